/*
 * sffn.h — activation-sparse gated FFN forward for NVIDIA B200 (sm_100a).
 *
 * The library computes, for T tokens x_t (rows of x),
 *
 *     g   = W_gate x_t + b            (dense gate)   or   z = bf16(x_t A), g = z B + b   (low-rank gate)
 *     a   = sigma(g)                  sigma = ReLU or SiLU
 *     keep_j  iff |a_j| > threshold   (relu-threshold mode)   or   j in top-k of |a_j|·||W_down[j,:]||_2 (wina-topk mode)
 *     v_j = round_to_operand_dtype(a_j)            (the TwELL value)
 *     u_j = <W_up[j,:], x_t>          only for kept j
 *     y_t = sum_{kept j} (v_j u_j) W_down[j,:]
 *
 * Sources (web pages, cited by title and section):
 *   - gated FFN structure and the low-rank (rank ratio 1/8) gate:
 *     "Meta FAIR and Inria's LoPA Gating Hits 3.31x Real GPU Speedup for LLM
 *     Inference", section "How LoPA Gating Restructures FFN Computation";
 *   - ReLU sparsity, the TwELL format written in the gate epilogue, the fused
 *     up/down pass that never stores h, and routing of highly active tokens
 *     to a dense tensor-core channel: "Sparser, Faster, Lighter Transformer
 *     Language Models" (news article), sections "稀疏不等於提速",
 *     "TwELL 減掉轉換開銷" and "Hybrid 應對非均勻稀疏";
 *   - the WINA score |hidden value| x ||weight column||_2 and per-token top-K:
 *     WINA framework explainer, sections 3.1 and 2.
 *
 * Layouts (all row-major, all pointers are DEVICE pointers, 16-byte aligned):
 *   x       [T][d_model]          operand dtype (bf16 or fp32)
 *   W_gate  [d_ff][d_model]       neuron-major: row j is neuron j (PyTorch Linear weight)
 *   A       [d_model][rank]       low-rank gate factor (x·A)
 *   B       [rank][d_ff]          low-rank gate factor (z·B)
 *   W_up    [d_ff][d_model]       neuron-major (PyTorch Linear weight of up_proj)
 *   W_down  [d_ff][d_model]       neuron-major: row j is neuron j's output row,
 *                                 i.e. the transpose of PyTorch's down_proj.weight
 *   gate_bias [d_ff] fp32 (optional)
 *   out     [T][d_model] fp32
 *
 * TwELL (tile-wise ELLPACK) as written by the gate epilogue, one record per
 * (token t, tile p) where a tile is 128 consecutive neurons:
 *   count[t][p]        int16: the TRUE number kept in the tile (may exceed C)
 *   idx[t][p][0..C)    int16: kept global neuron indices, ascending; pad -1
 *   val[t][p][0..C)    operand dtype: v of the kept neurons; pad +0.0
 * A token overflows iff some tile of it keeps more than C neurons; it is then
 * computed whole by the dense tensor-core fallback.  y does not depend on C.
 *
 * Ownership: the caller owns x, out and all weights.  Weights are borrowed
 * and must stay valid and unchanged for the life of the handle (the handle
 * keeps derived copies made at create time: a transposed W_down for the
 * tensor-core down projection, transposed low-rank factors, WINA norms).
 * The handle owns its workspace (TwELL, routing lists, scratch, status word).
 *
 * Errors: argument and shape errors are returned before any launch and leave
 * no side effect.  Launch failures return SFFN_ERR_CUDA.  Device-side problems
 * (a bounded wait that expired, an index out of range) are recorded in the
 * handle's device status word, which sffn_read_status() returns (and clears).
 * sffn_forward never blocks the host.  One handle serves one forward at a time
 * on one stream (not re-entrant); distinct handles are independent.
 */
#ifndef SFFN_H
#define SFFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SFFN_OK = 0,
  SFFN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad enum       */
  SFFN_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d_ff % 128 != 0) */
  SFFN_ERR_ALLOC = 3,         /* device allocation failed                          */
  SFFN_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed       */
  SFFN_ERR_TIMEOUT = 5,       /* a device-side bounded wait expired                */
  SFFN_ERR_DEVICE = 6,        /* a device-side range check failed                  */
  SFFN_ERR_NO_DEVICE = 7      /* no usable sm_100 device                           */
} sffn_status;

typedef enum { SFFN_BF16 = 0, SFFN_FP32 = 1 } sffn_dtype;
/* Selection of the kept neurons.
 *   RELU_THRESHOLD: keep iff |sigma(g)| > threshold;
 *   WINA_TOPK     : per token the k largest |sigma(g_j)|·||W_down[j,:]||_2 (WINA
 *                   framework explainer, section 3.1, hidden value = the gate
 *                   activation: only the kept neurons' W_up rows are read);
 *   WINA_FULL_H   : per token the k largest |sigma(g_j)·u_j|·||W_down[j,:]||_2,
 *                   the same score with the hidden value taken as the full
 *                   gated product: the up projection of every neuron is
 *                   computed (W_up read in full), the down projection is sparse.
 *                   Dense gate, bf16, tile_capacity 128. */
typedef enum { SFFN_MODE_RELU_THRESHOLD = 0, SFFN_MODE_WINA_TOPK = 1, SFFN_MODE_WINA_FULL_H = 2 } sffn_mode;
typedef enum { SFFN_ACT_RELU = 0, SFFN_ACT_SILU = 1 } sffn_act;

/* How the kept (token, neuron) pairs of non-overflow tokens are computed.
 *   ROWS : the fused up x down kernel streams only the kept rows of W_up
 *          and W_down, per block of 8 tokens (best when few tokens share a
 *          neuron: decode at T <= 8, sparse prefill).  At T <= 8 with a dense
 *          threshold gate the whole forward (gate, TwELL, routing, up x down,
 *          dense channel) runs as one persistent launch;
 *   TILES: tensor-core up and down over every 128-neuron tile that some token
 *          keeps, with the non-kept entries of h zeroed (best when the union
 *          of kept neurons covers most tiles: WINA, T in 16..256).  At
 *          T <= 32 in relu-threshold mode (dense or low-rank gate) the
 *          whole forward runs as one persistent launch;
 *   AUTO : ROWS for T <= 8 or T > 256 in relu-threshold mode, TILES otherwise. */
typedef enum { SFFN_PATH_AUTO = 0, SFFN_PATH_ROWS = 1, SFFN_PATH_TILES = 2 } sffn_path;

/* desc.flags */
#define SFFN_FLAG_DEBUG_GATE 1u   /* keep the dense fp32 gate g[T][d_ff] of the last forward */
#define SFFN_FLAG_SEPARATE 2u     /* separate gate, up x down and dense-channel launches instead
                                     of a single persistent launch (ROWS at T <= 8, TILES at
                                     T <= 32): diagnostics, tests */
#define SFFN_FLAG_COOPERATIVE 4u  /* launch the single persistent forward with the cooperative
                                     attribute (see sffn_forward) */
#define SFFN_FLAG_BACKWARD 8u     /* allocate the workspace of sffn_backward (relu-threshold
                                     mode, dense gate, bf16, no input_k or V) */

typedef struct sffn_desc {
  int d_model;          /* d: multiple of 8, 8..4096 (ROWS path needs d <= 4096)   */
  int d_ff;             /* F: multiple of 128, <= 32767 (int16 TwELL indices)      */
  int max_tokens;       /* workspace is sized for T <= max_tokens                  */
  int rank;             /* 0: dense W_gate; > 0: low-rank A,B (bf16 only), %64==0  */
  sffn_dtype dtype;     /* operand dtype; out is always fp32                       */
  sffn_mode mode;
  sffn_act act;
  float threshold;      /* relu-threshold: keep iff |sigma(g)| > threshold (>= 0)  */
  int k;                /* wina-topk: neurons kept per token, 0..d_ff              */
  int tile_capacity;    /* C: 8, 16, 32, 64 or 128                                 */
  int path;             /* sffn_path                                               */
  unsigned flags;       /* SFFN_FLAG_*                                             */
  const void* W_gate;   /* [d_ff][d_model]  (NULL iff rank > 0)                    */
  const void* A;        /* [d_model][rank]  (NULL iff rank == 0)                   */
  const void* B;        /* [rank][d_ff]     (NULL iff rank == 0)                   */
  const void* W_up;     /* [d_ff][d_model]                                         */
  const void* W_down;   /* [d_ff][d_model]                                         */
  const float* gate_bias; /* [d_ff] fp32 or NULL                                   */
  /* WINA on the input side (WINA explainer, section 3.1, applied to the layer
   * that consumes x, the stacked [W_gate; W_up]): per token keep the input_k
   * coordinates of largest |x_i|·c_i, c_i = ||column i of [W_gate; W_up]||_2
   * (fp64, rounded to fp32; the product rounded to fp32, equal scores to the
   * smaller index), zero the others, and run both projections on the result.
   * 0 = off; 1..d_model.  Dense gate, bf16. */
  int input_k;
  /* Orthogonalisation (WINA explainer, section 3.3): V [d_model][d_model] bf16,
   * the right singular vectors of [W_gate; W_up] (any V is accepted; the SVD
   * itself is the caller's).  At create time the handle stores W_gate·V and
   * W_up·V rounded to bf16 (2·d_ff·d_model·2 bytes), and every forward first
   * rotates its tokens, x' = bf16(x·V), so that W V V^T x = W x; the input-side
   * selection then acts on x' with the rotated column norms (the singular
   * values when V comes from the SVD).  NULL = off.  Dense gate, bf16. */
  const void* V;
} sffn_desc;

typedef struct sffn_handle sffn_handle;

/* Validate desc, allocate the workspace for max_tokens, build the TMA tensor
 * maps and the create-time derived data (transposed W_down; transposed A and
 * B; WINA norms), all on `cuda_stream` (a cudaStream_t, NULL = legacy default
 * stream).  Synchronises the stream before returning.  On error *out is NULL
 * and nothing stays allocated. */
sffn_status sffn_create(const sffn_desc* desc, void* cuda_stream, sffn_handle** out);

/* y = FFN(x) for T tokens, asynchronously on `cuda_stream`.  x: [T][d_model]
 * device, operand dtype; out: [T][d_model] fp32 device, fully overwritten.
 * 0 <= T <= max_tokens; T == 0 returns SFFN_OK and launches nothing.  Must not
 * overlap another forward of the same handle.  Each call takes the handle's
 * next epoch, passed to its kernels by value: it tags the forward's overflow
 * flags and, on the single-launch path, the scheduler words that the CTAs
 * exchange.  A forward captured into a CUDA graph and replayed would reuse
 * its epoch and could read a previous replay's scheduler words, so stream
 * capture of sffn_forward is not supported.
 *
 * The single persistent launches (ROWS path at T <= 8, TILES path at T <= 32
 * in relu-threshold mode, see sffn_path) have one CTA per SM and their CTAs wait on one
 * another, so each needs all of them resident at once.  That
 * holds when the forward has the GPU's SMs to itself or shares them with
 * ordinary kernels; it need not hold for an MPS client limited to part of the
 * SMs, a green context, or a concurrent persistent kernel that never yields
 * its SMs.  There every wait is bounded: the forward gives up after 2 s,
 * writes no valid out and records SFFN_ERR_TIMEOUT (sffn_read_status), and
 * nothing hangs.  Callers in such settings set SFFN_FLAG_COOPERATIVE: the
 * launch is then cooperative, so the driver holds it until the whole grid
 * fits, or refuses it (SFFN_ERR_CUDA) when it never can.  It costs about
 * 4 us per forward on B200, because a cooperative grid cannot start while
 * the previous forward's CTAs still hold SMs. */
sffn_status sffn_forward(sffn_handle* h, const void* x, int T, float* out, void* cuda_stream);

/* Same as sffn_forward but x and out are HOST buffers: copies x to the
 * handle's device staging buffer, runs the forward and copies y back, all on
 * `cuda_stream`, then synchronises it.  Page-locked host memory makes the
 * copies asynchronous DMA. */
sffn_status sffn_forward_host(sffn_handle* h, const void* x_host, int T, float* out_host,
                              void* cuda_stream);

/* Free everything the handle owns.  NULL is accepted (SFFN_OK). */
sffn_status sffn_destroy(sffn_handle* h);

const char* sffn_status_string(sffn_status s);

/* Synchronise `cuda_stream`, then return and clear the device status word
 * (SFFN_OK, SFFN_ERR_TIMEOUT or SFFN_ERR_DEVICE). */
sffn_status sffn_read_status(sffn_handle* h, void* cuda_stream);

/* Device views of the last forward's TwELL and overflow flags (valid until the
 * next forward or destroy).  count: int16 [T][n_tiles]; idx: int16
 * [T][n_tiles][C]; val: operand dtype [T][n_tiles][C]; overflow: uint32 [T],
 * equal to sffn_stats.epoch iff the token took the dense channel in the last
 * forward.  Test and bench use. */
sffn_status sffn_debug_twell(sffn_handle* h, const int16_t** count, const int16_t** idx,
                             const void** val, const uint32_t** overflow, int* n_tiles,
                             int* tile_capacity);

/* Test hook for the bounded waits of the single-launch forwards (ROWS path at
 * T <= 8, TILES path at T <= 32).  Until called again with (0, 0), those
 * forwards count
 * `phantom_ctas` (0 or 1) extra CTAs in their grid that never run, so every
 * wait on them expires, and limit their waits on other CTAs to `wait_us`
 * microseconds (0: the default of 2 s).  Such a forward's out is not valid
 * and it sets the status word's timeout (sffn_read_status returns
 * SFFN_ERR_TIMEOUT and clears the scheduler state); nothing faults or hangs.
 * Errors: SFFN_ERR_INVALID_ARG for a null handle or phantom_ctas not 0 or 1. */
sffn_status sffn_debug_decode_waits(sffn_handle* h, int phantom_ctas, unsigned wait_us);

/* The job lists of the TILES path's single launch (up to 32 tokens) for a
 * layer of d_model x d_ff (rank > 0: the low-rank gate) on n_cta CTAs, as the
 * handle builds them; host only, no device needed.  jobs receives n_jobs
 * records of 4 ints {type | finisher << 4 | count << 8, tile, k0 | k1 << 16,
 * id} (type 0 a z range, 1 a tile's gate and first up range, 2 a later up
 * range, 3 a down range; K in 64-wide blocks), off the n_cta + 1 offsets of
 * each CTA's list.  Test use: it lets the lists' coverage and wait order be
 * checked without a GPU.  Errors: SFFN_ERR_INVALID_ARG for sizes out of
 * range or buffers too small (*n_jobs then holds the count needed). */
sffn_status sffn_debug_tile_schedule(int d_model, int d_ff, int rank, int n_cta, int* jobs, int max_jobs,
                                     int* off, int* n_jobs);

/* Test hook: the next forward takes epoch `epoch` + 1 (0 is skipped).  The
 * single-launch decode forward's scheduler words carry the low 16 bits of the
 * epoch and are cleared here (synchronously) and at the start of every
 * window of 65536 epochs, so tests can cross those windows and the 32-bit
 * wrap.  Errors: SFFN_ERR_INVALID_ARG for a null handle; SFFN_ERR_CUDA if the
 * clear fails. */
sffn_status sffn_debug_set_epoch(sffn_handle* h, unsigned epoch);

/* Device view of the last forward's keep masks: uint32 [T][n_tiles][4], bit
 * (32 w + b) of word w set iff the token keeps neuron 128 p + 32 w + b of tile
 * p, with no capacity limit (an overflow token's full kept set).  Written by
 * the ROWS path only (undefined after a TILES forward).  Test and bench use. */
sffn_status sffn_debug_keep(sffn_handle* h, const uint32_t** keep);

/* Device view of the dense fp32 gate g[T][d_ff] of the last forward (only
 * with SFFN_FLAG_DEBUG_GATE; dense gate only).  Test use. */
sffn_status sffn_debug_gate(sffn_handle* h, const float** g);

/* Backward of the last forward: given that forward's x (device, [T][d_model]
 * bf16) and the upstream gradient dy = dL/dy (device, [T][d_model] fp32),
 * write dx [T][d_model], dW_gate, dW_up and dW_down [d_ff][d_model] (neuron-
 * major like the weights) and, if d_bias is not NULL, d_bias [d_ff], all fp32
 * device buffers, fully overwritten.  Source: "Sparser, Faster, Lighter
 * Transformer Language Models" (news article), section "Hybrid 應對非均勻稀疏"
 * (training over the sparse format).  The selection of the forward is held
 * fixed (its keep masks, every token's full kept set) and the rounding of the
 * stored value passes the gradient through:
 *     dh = dy W_down^T on kept pairs, du = dh·v, dg = dh·u·sigma'(g),
 *     dW_down = h^T dy, dW_up = du^T x, dW_gate = dg^T x, d_bias = sum_t dg,
 *     dx = du W_up + dg W_gate.
 * Only kept pairs are computed: a token pass (x and dy rows staged, the
 * kept rows of W_gate, W_up and W_down streamed; dx) and a neuron pass (the
 * dW rows and d_bias from each neuron's pairs, x and dy rows gathered).
 * Requires SFFN_FLAG_BACKWARD at create time (workspace 20·max_tokens·d_ff
 * bytes plus small arrays) and a last forward on the ROWS path with the same
 * T (else SFFN_ERR_INVALID_ARG).  Asynchronous on cuda_stream. */
sffn_status sffn_backward(sffn_handle* h, const void* x, const float* dy, int T, float* dx, float* dW_gate,
                          float* dW_up, float* dW_down, float* d_bias, void* cuda_stream);

/* Bytes of device memory the handle allocated (its whole workspace, one
 * allocation: TwELL, routing, scratch, status and the create-time derived
 * data).  A handle whose max_tokens is at most 8 and whose forwards all take
 * the single decode launch holds no transposed W_down and no h buffers. */
sffn_status sffn_workspace_bytes(const sffn_handle* h, size_t* bytes);

/* Device view of the WINA norms n_j (fp32 [d_ff]), wina-topk mode only. */
sffn_status sffn_debug_norms(sffn_handle* h, const float** norms);

/* Counters of the last forward, copied to the host (synchronises the stream):
 * number of overflow tokens, the number of kernel launches it made, the path
 * taken and the forward's epoch (see sffn_debug_twell). */
typedef struct sffn_stats {
  int n_overflow;
  int n_launches;
  int path;             /* the sffn_path actually taken (ROWS or TILES) */
  unsigned epoch;       /* overflow[t] == epoch marks the last forward's overflow tokens */
  unsigned launch_attrs; /* the last single persistent launch: bit 0 cooperative, bit 1
                            programmatic dependent launch (0 if none was made) */
} sffn_stats;
sffn_status sffn_get_stats(sffn_handle* h, void* cuda_stream, sffn_stats* st);

/* Per-kernel device timing (bench use).  Between sffn_timing_begin and
 * sffn_timing_end every stride-th forward records a CUDA event on its own
 * stream before each kernel launch and after the last one; no work is skipped
 * or added.  max_forwards bounds the forwards recorded (later ones are not
 * timed). */
sffn_status sffn_timing_begin(sffn_handle* h, int max_forwards, int stride);

/* Synchronise the recorded events and report, per kernel label (a short
 * name such as "gate" or "updown_rows", NUL-terminated, at most 31 chars), the
 * summed device time in ms and the number of launches timed.  At most
 * max_kernels labels are written; *n_kernels receives how many exist.
 * Timing is off afterwards. */
sffn_status sffn_timing_end(sffn_handle* h, int max_kernels, char (*names)[32], float* total_ms,
                            int* launches, int* n_kernels);

/* Allocation-free low-rank gate (no counterpart in the pages: an interface
 * convenience).  For callers that must not allocate device memory where they
 * run: code inside a runtime that owns all device memory (a pre-planned pool,
 * a plugin host with fixed buffers) or on a latency-critical path, where
 * cudaMalloc can synchronise the device or fail.  It computes the same TwELL
 * records as the low-rank gate of sffn_forward: z = bf16(x·A), g = z·B + b,
 * keep iff |sigma(g)| > threshold.  Inputs (device, 16-byte aligned):
 *   x [T][d_model] bf16; A_t [rank][d_model] bf16 (A transposed);
 *   B_t [d_ff][rank] bf16 (B transposed); gate_bias [d_ff] fp32 or NULL.
 * Outputs (device): count [T][d_ff/128] int16, idx [T][d_ff/128][C] int16,
 *   val [T][d_ff/128][C] bf16 (TwELL as described above), overflow [T]
 *   uint32: 1 iff the token overflows some tile, else 0.
 * Limits: T <= 64, d_model <= 4096 (multiple of 8), rank <= 1024 (multiple of
 * 64), d_ff <= 16384 (multiple of 128); larger sizes return
 * SFFN_ERR_UNSUPPORTED before anything runs.  Scratch lives in fixed device
 * arrays inside this library (1,179,696 bytes, about 1.2 MB, per GPU, held
 * until the process exits); the first call on a device looks their addresses
 * up, so make that call before any stream capture.  Every call shares that
 * scratch and clears what must start at zero, so calls that overlap on the
 * GPU (two streams, two threads) race and must be serialised by the caller.
 * Asynchronous on cuda_stream; no allocation, no host synchronisation.
 * Device-side errors (a bounded wait that expired) go to a status word that
 * all calls on the device share; sffn_lowrank_twell_noalloc_status reads it.
 * A call whose kernels recorded an error leaves its outputs undefined. */
sffn_status sffn_lowrank_twell_noalloc(const void* x, int T, int d_model, const void* A_t, int rank,
                                       const void* B_t, int d_ff, const float* gate_bias, int act,
                                       float threshold, int tile_capacity, int16_t* count, int16_t* idx,
                                       void* val, uint32_t* overflow, void* cuda_stream);

/* Status of the allocation-free calls on the current device: synchronises
 * `cuda_stream`, then returns and clears the device status word that those
 * calls' kernels share (SFFN_OK, SFFN_ERR_TIMEOUT or SFFN_ERR_DEVICE).  Errors
 * of every call since the last read accumulate in it.  SFFN_ERR_CUDA if the
 * synchronisation or the read fails. */
sffn_status sffn_lowrank_twell_noalloc_status(void* cuda_stream);

/* Test hook for the allocation-free calls' bounded waits.  While wait_us is
 * not 0, their kernels wait wait_us microseconds on a barrier that nothing
 * signals before they issue any copy, then record a timeout and return
 * without writing outputs (sffn_lowrank_twell_noalloc_status then returns
 * SFFN_ERR_TIMEOUT); nothing faults or hangs.  0 turns the hook off.
 * Process-wide; always SFFN_OK. */
sffn_status sffn_debug_noalloc_waits(unsigned wait_us);

/* ------------------------------------------------------------------------
 * Gated subspace linear layer (GSI).  Source: "Gated Subspace Inference for
 * Transformer Acceleration" (technical summary), section 2.1 (core
 * decomposition) and section 2.2 (gated residual pass-through).  For a linear
 * layer y = W x and an orthonormal basis V_k of the activation subspace:
 *
 *     g = V_k^T x,   r = x - V_k g,   M = W V_k  (cached at create time),
 *     y = M·bf16(g)   if ||r||^2 < eps^2·||x||^2   (fast path: reads only M)
 *     y = W x         otherwise                   (slow path: reads W)
 *
 * so a token on the fast path is off by at most ||W||_2·eps·||x|| (the
 * page's Theorem 4) and a token on the slow path is exact.
 *
 * Layouts (device pointers, 16-byte aligned, row-major): W [d_out][d_in] bf16
 * (PyTorch Linear weight), V_k [d_in][k] bf16 (orthonormal columns: the
 * caller's calibrated basis), x [T][d_in] bf16, y [T][d_out] fp32.  M is
 * stored as bf16(W V_k), and g is rounded to bf16 for the fast path; the
 * residual and the norms use the fp32 g.  The test is strict (rho = eps takes
 * the slow path) and x = 0 takes the slow path.
 * Limits: d_in % 8 == 0 and <= 8192; k % 8 == 0, k <= 512 and k <= d_in;
 * max_tokens <= 64 (decode batches); otherwise SFFN_ERR_UNSUPPORTED.
 * Ownership as for sffn_create: W and V_k are borrowed for the handle's life;
 * the handle owns M (d_out·k·2 bytes), V_k^T and its workspace. */
typedef struct sffn_gsi_desc {
  int d_in, d_out, k, max_tokens;
  float eps;            /* residual-ratio threshold (>= 0; 0: every token slow) */
  const void* W;        /* [d_out][d_in] bf16 */
  const void* Vk;       /* [d_in][k] bf16    */
} sffn_gsi_desc;

typedef struct sffn_gsi_handle sffn_gsi_handle;

/* Validate, allocate, transpose V_k and compute M on `cuda_stream`, then
 * synchronise it.  On error *out is NULL and nothing stays allocated. */
sffn_status sffn_gsi_create(const sffn_gsi_desc* desc, void* cuda_stream, sffn_gsi_handle** out);

/* y = GSI(x) for T tokens (0 <= T <= max_tokens; 0: nothing launched),
 * asynchronously on `cuda_stream`: three kernels (projection, residual norms,
 * routed output).  y is fully overwritten.  One forward at a time per handle. */
sffn_status sffn_gsi_forward(sffn_gsi_handle* h, const void* x, int T, float* y, void* cuda_stream);

sffn_status sffn_gsi_destroy(sffn_gsi_handle* h);

/* Number of tokens of the last forward that took the slow path (synchronises
 * the stream). */
sffn_status sffn_gsi_stats(sffn_gsi_handle* h, void* cuda_stream, int* n_slow);

/* Device views of the last forward (valid until the next forward or destroy):
 * g fp32 [T][k]; the per-CTA partial sums of r^2 and x^2, fp32
 * [n_part][T][2] (a token's ||r||^2 and ||x||^2 are their sums over the
 * n_part CTAs); and the cached image M bf16 [d_out][k].  Test use. */
sffn_status sffn_gsi_debug(sffn_gsi_handle* h, const float** g, const float** part, int* n_part,
                           const void** M);

/* Per-kernel device timing of the GSI forward, as sffn_timing_begin/end. */
sffn_status sffn_gsi_timing_begin(sffn_gsi_handle* h, int max_forwards, int stride);
sffn_status sffn_gsi_timing_end(sffn_gsi_handle* h, int max_kernels, char (*names)[32], float* total_ms,
                                int* launches, int* n_kernels);

/* ------------------------------------------------------------------------
 * Mixture of LoPA-gated sparse experts.  Source: "Meta FAIR and Inria's LoPA
 * Gating Hits 3.31x Real GPU Speedup for LLM Inference", section "Model
 * Casting and Quality at 90% Sparsity" (LoPA gating carries over to MoE
 * layers whose experts share the gated FFN structure) and section "How LoPA
 * Gating Restructures FFN Computation" (the low-rank gate).  The page gives
 * no routing rule; this library takes Mixtral's:
 *
 *     l[t][e] = <W_r[e], x_t>;  S_t = the top_k experts by l (ties to the
 *     smaller index);  w[t][e] = softmax of l[t][S_t];
 *     y_t = sum_{e in S_t} w[t][e] · FFN_e(x_t),
 *
 * each FFN_e the relu-threshold forward of sffn_forward with a low-rank gate
 * (A_e, B_e), its own W_up, W_down and bias.  A forward is a router launch,
 * each expert's sparse forward on a block of T rows (x_t where t is routed to
 * the expert, zero elsewhere: a zero row keeps no neuron, so the gate biases
 * must be <= 0, checked at create time) and a combine launch.
 *
 * Layouts as for sffn_desc; W_router [n_experts][d_model] bf16; the per-expert
 * pointer arrays are HOST arrays of n_experts device pointers (copied).
 * Limits: n_experts <= 64, top_k <= 8, max_tokens <= 1024. */
typedef struct sffn_moe_desc {
  int n_experts, top_k;
  int d_model, d_ff, rank, max_tokens, tile_capacity;
  float threshold;
  const void* W_router;
  const void* const* A;             /* [n_experts] -> [d_model][rank]   */
  const void* const* B;             /* [n_experts] -> [rank][d_ff]      */
  const void* const* W_up;          /* [n_experts] -> [d_ff][d_model]   */
  const void* const* W_down;        /* [n_experts] -> [d_ff][d_model]   */
  const float* const* gate_bias;    /* [n_experts] -> [d_ff], or NULL   */
} sffn_moe_desc;

typedef struct sffn_moe_handle sffn_moe_handle;

/* Create one sparse-FFN handle per expert and the routing workspace.
 * SFFN_ERR_UNSUPPORTED for a positive gate bias (see above). */
sffn_status sffn_moe_create(const sffn_moe_desc* desc, void* cuda_stream, sffn_moe_handle** out);

/* y = MoE(x) for T tokens (device x [T][d_model] bf16, out [T][d_model]
 * fp32), asynchronously on cuda_stream; no host synchronisation.  The
 * experts' forwards run side by side on up to eight streams of the handle,
 * which wait for the router on cuda_stream and which cuda_stream waits for
 * before the combine; work queued on cuda_stream after the call is ordered
 * after all of it. */
sffn_status sffn_moe_forward(sffn_moe_handle* h, const void* x, int T, float* out, void* cuda_stream);

sffn_status sffn_moe_destroy(sffn_moe_handle* h);

/* The handle of expert e (owned by the MoE handle): its TwELL and stats views
 * describe its last block of T rows. */
sffn_status sffn_moe_expert(sffn_moe_handle* h, int e, sffn_handle** expert);

/* Device views of the last forward's routing: sel int32 [T][top_k], weights
 * fp32 [T][top_k] and logits fp32 [T][n_experts].  Test use. */
sffn_status sffn_moe_debug(sffn_moe_handle* h, const int** sel, const float** w, const float** logits);

/* Synchronise and return (and clear) the first device-side error any expert
 * recorded (as sffn_read_status). */
sffn_status sffn_moe_read_status(sffn_moe_handle* h, void* cuda_stream);

/* Per-kernel device timing of the MoE forward (router, combine and every
 * expert's kernels, added by label), as sffn_timing_begin/end. */
sffn_status sffn_moe_timing_begin(sffn_moe_handle* h, int max_forwards, int stride);
sffn_status sffn_moe_timing_end(sffn_moe_handle* h, int max_kernels, char (*names)[32], float* total_ms,
                                int* launches, int* n_kernels);

/* Library version string. */
const char* sffn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SFFN_H */
