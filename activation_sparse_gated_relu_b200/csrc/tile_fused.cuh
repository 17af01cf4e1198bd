// The whole tile-path forward for up to 32 tokens in one persistent launch
// ([TwELL] "TwELL 減掉轉換開銷" and "Hybrid 應對非均勻稀疏"; [LoPA] "How LoPA
// Gating Restructures FFN Computation" for the low-rank gate).
//
// At 32 tokens nearly every neuron is kept by some token, so the up and down
// projections stream W_up and W_down^T whole through the tensor cores and the
// sparsity is applied as a mask on h.  One CTA per SM walks a static list of
// jobs, built on the host, over one TMA ring and four TMEM accumulator slots.
// Every job works on a pair of 128-row tiles (256 neurons, rank coordinates
// or output columns): a ring stage holds one 256-row weight box and one B
// tile (32 tokens) that both halves multiply, so the small B tiles cost half
// as much per weight byte as with one tile per stage.  "Tile" below means
// such a pair.
//
//   phase 0 (low-rank gate), the K blocks of z = x·A cut into pieces of a
//   few blocks, the first jobs of their CTAs (spread over the grid):
//     Z     a K range of z for 256 rank coordinates, a partial sum stored
//           and published.  Once every Z piece of its CTA has published,
//           each of the pair's last min(4, pieces) pieces adds all pieces'
//           partial sums in K order for its share of the pair's four parts
//           (a half of the rank coordinates x 16 tokens), rounds them to
//           bf16 and publishes each part
//   phase 1, a stream of 64-wide K blocks cut into one equal run per CTA:
//     MAIN  one tile (256 neurons): the first K range of u = x·W_up^T, then
//           the last K range of the gate GEMM (over W_gate, or over B with z
//           as the operand; last, so that z has long been published).  The
//           gate's earlier ranges come from GHELP jobs of the previous CTAs,
//           u's later ones from HELP jobs of the next; the MAIN adds them in
//           K order.  The TwELL emission (records, counts and overflow flags
//           exactly as the format defines them) runs on the complete gate;
//           h = v·u with v the kept activation values (zero elsewhere) is
//           written as a bf16 pair (hi + lo) and the tile is published
//     GHELP an earlier K range of one tile's gate, a partial sum
//     HELP  a later K range of one tile's u, a partial sum
//   phase 2, the down projection's K blocks cut the same way:
//     DOWN  a K range of y^T = W_down^T · h^T for 256 output columns, added
//           into out at L2 (after every CTA has zeroed its slice of out)
//
// Overflow tokens: the emission holds every kept value of the tile, not only
// the first C, and u is computed for every token, so a token whose record
// overflows gets the dense channel's h (keep ? bf16(sigma(g + b))·u : 0 over
// all neurons) from the same tiles; its TwELL record and overflow flag are
// still written as the format's routing record.
//
// Cross-CTA data goes through global memory with seq-tagged flags (the
// launch's own sequence number, so nothing needs clearing between launches):
// a producer writes, fences, then stores the flag with release semantics; the
// consumer acquires the flag and, before a TMA load of the data, fences the
// async proxy.  Every job waits only on jobs that come earlier in some CTA's
// list and do not wait themselves on later ones (Z ranges and HELP ranges
// open their runs, GHELP ranges close them; a gate waits for z, a MAIN for its
// helpers, DOWN for the mains), so with all CTAs resident every wait ends.  Every wait is
// bounded all the same: on a timeout the CTA records DEV_ERR_TIMEOUT, issues
// the copies its ring still expects, drains them and its MMAs, frees TMEM and
// returns.
//
// Warp roles (192 threads): warps 0-3 epilogue (thread = TMEM lane = one
// neuron, rank coordinate or output column), warp 4 TMA producer, warp 5 TMEM
// owner and MMA issuer.  Weights (every A operand) are constant for the
// handle's life, so the producer's first ring fills are issued before the
// grid dependency on the previous kernel of the stream.
#pragma once

#include "epilogues.cuh"
#include "tc_gemm.cuh"

namespace sffn {

constexpr int TF_BN = 32;                                  // tokens: one token tile
constexpr int TF_PAIR = 2;                                 // 128-row tiles per job tile
constexpr int TF_ROWS = TF_PAIR * TC_BM;                   // 256 weight rows per stage
constexpr int TF_A_BYTES = TF_PAIR * TC_A_BYTES;           // one 64 x 256 weight box (32 KB)
constexpr int TF_B_BYTES = TF_BN * TC_BK * 2;              // one B tile (4 KB)
constexpr int TF_STAGE_BYTES = TF_A_BYTES + 2 * TF_B_BYTES;  // weights + up to two B tiles (40 KB)
constexpr int TF_MAX_STAGES = 6;
constexpr int TF_NSLOT = 4;                                // TMEM accumulator slots
constexpr int TF_SLOT_COLS = TF_PAIR * 64;                 // a slot: per half 32 (or 64: hi | lo) columns
constexpr int TF_TILE_FLOATS = TF_PAIR * TF_BN * 128;      // a partial accumulator [2][32 tokens][128 rows]
constexpr int TF_ZMAXP = 8;                                // z pieces per rank pair at most

enum : int { TFJ_Z = 0, TFJ_MAIN = 1, TFJ_HELP = 2, TFJ_DOWN = 3, TFJ_GHELP = 4 };

// Job record (int4): x = type | fin << 4 | count << 8 | gcount << 16.  Z:
// count = pieces of its rank pair, gcount = this piece's index q among them,
// fin = it finishes some of the pair's four parts.  MAIN: count = up
// helpers, gcount = gate helpers.  y = tile pair (rank, neuron or
// output-column tiles 2y and 2y + 1), z = k0 | k1 << 16 (K blocks; MAIN: its
// gate range is [k0, gate end), its up range [0, k1)), w = id (Z: its piece
// slot, consecutive in K order within a rank pair; MAIN: its first helper
// slot, the gate helpers' slots before the up helpers'; HELP, GHELP: its slot).
__host__ __device__ inline int4 tf_job(int type, int fin, int count, int gcount, int tile, int k0, int k1, int id) {
  return make_int4(type | (fin << 4) | (count << 8) | (gcount << 16), tile, k0 | (k1 << 16), id);
}
// z of a rank pair is finished in four parts (half h = part / 2, tokens
// 16 (part % 2) .. + 15) by the pair's last min(4, pieces) pieces, part p by
// finisher p % that count; its flags f_z[4 pair + part]
constexpr int TF_ZPARTS = 4;

struct TfLayout {
  int stages, bars, scratch, total;
};
__host__ __device__ inline TfLayout tf_layout(int C) {
  TfLayout L;
  const int scratch = (twell32_smem(C) + 127) & ~127;
  L.stages = (TC_SMEM_BUDGET - 1024 - 256 - scratch) / TF_STAGE_BYTES;
  if (L.stages > TF_MAX_STAGES) L.stages = TF_MAX_STAGES;
  L.bars = L.stages * TF_STAGE_BYTES;
  L.scratch = L.bars + 256;
  L.total = 1024 + L.scratch + scratch;
  return L;
}

struct TfArgs {
  CUtensorMap mx;      // x [T][d], box 64 x 32
  CUtensorMap mz;      // z [maxT][R] (low rank)
  CUtensorMap mhi;     // h_hi [maxT][F]
  CUtensorMap mlo;     // h_lo [maxT][F]
  CUtensorMap mgate;   // the gate's A: W_gate [F][d], or B^T [F][R]; box 64 x 256
  CUtensorMap mAt;     // A^T [R][d] (low rank); box 64 x 256
  CUtensorMap mup;     // W_up [F][d]; box 64 x 256
  CUtensorMap mdT;     // W_down^T [d][F]; box 64 x 256
  const int4* jobs;
  const int* job_off;  // [n_chunks + 1]: CTA c runs jobs [job_off[c], job_off[c + 1])
  TwellParams tw;      // T, F, n_tiles, C, tau, act, TwELL outputs, overflow epoch (bias null)
  const float* bias;   // [F] or null: added to the gate before the emission
  float* zpart;        // [z pieces][2][32][128]
  float* upart;        // [helper slots][2][32][128]
  __nv_bfloat16* z;    // [maxT][R]
  __nv_bfloat16* h_hi; // [maxT][F]
  __nv_bfloat16* h_lo;
  int* f_zp;           // [z pieces]  = seq once the piece's partial sum is stored
  int* f_z;            // [R / 256][4] = seq once that part of z is stored
  int* f_up;           // [helper slots] = seq once the helper's partial is stored
  int* f_h;            // [F / 256]   = seq once h of the tile pair is stored
  int* f_zero;         // [n_chunks]  = seq once the CTA's slice of out is zeroed
  float* out;          // [T][d]
  int d, R, maxT, kb_gate, lowrank, n_chunks;
  int seq;             // this launch's sequence number (never 0)
  uint32_t* status;
  unsigned long long wait_ns;
};

enum : int { TFA_GATE = 0, TFA_AT = 1, TFA_UP = 2, TFA_DT = 3 };  // the A operand's tensor map

struct TfSeg {
  int amap;  // TFA_*
  int arow, k0, k1;
  int kind;  // B operand: 0 x; 1 z (flags f_z[4 (kb / 4) ..]); 2 the h pair (flag f_h[kb / 4])
};

__device__ __forceinline__ int tf_type(const int4& j) { return j.x & 15; }
__device__ __forceinline__ int tf_nseg(const int4& j) { return tf_type(j) == TFJ_MAIN ? 2 : 1; }
__device__ __forceinline__ TfSeg tf_seg(const TfArgs& a, const int4& j, int s) {
  const int t = j.y, k0 = j.z & 0xFFFF, k1 = (int)((unsigned)j.z >> 16);
  switch (tf_type(j)) {
    case TFJ_Z: return TfSeg{TFA_AT, t * TF_ROWS, k0, k1, 0};
    case TFJ_MAIN:  // the up range first: the gate's B operand (z) may be published later
      return s == 0 ? TfSeg{TFA_UP, t * TF_ROWS, 0, k1, 0}
                    : TfSeg{TFA_GATE, t * TF_ROWS, k0, a.kb_gate, a.lowrank ? 1 : 0};
    case TFJ_GHELP: return TfSeg{TFA_GATE, t * TF_ROWS, k0, k1, a.lowrank ? 1 : 0};
    case TFJ_HELP: return TfSeg{TFA_UP, t * TF_ROWS, k0, k1, 0};
    default: return TfSeg{TFA_DT, t * TF_ROWS, k0, k1, 2};
  }
}

// Walks the K blocks of a CTA's jobs in order (the host makes every segment
// non-empty).
struct TfIter {
  int j, j1, s, kb;
  int4 job;
  TfSeg seg;
  __device__ void init(const TfArgs& a, int j0, int jend) {
    j = j0;
    j1 = jend;
    s = 0;
    if (j < j1) {
      job = __ldg(a.jobs + j);
      seg = tf_seg(a, job, 0);
      kb = seg.k0;
    }
  }
  __device__ bool valid() const { return j < j1; }
  __device__ void next(const TfArgs& a) {
    if (++kb < seg.k1) return;
    if (++s < tf_nseg(job)) {
      seg = tf_seg(a, job, s);
      kb = seg.k0;
      return;
    }
    s = 0;
    if (++j < j1) {
      job = __ldg(a.jobs + j);
      seg = tf_seg(a, job, 0);
      kb = seg.k0;
    }
  }
};

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ int ld_relaxed_gpu(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Non-blocking test of an mbarrier phase (try_wait may suspend the thread for
// a while; the producer has other copies to issue meanwhile).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Named barrier over n threads that also returns the AND of their predicates.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// mbarrier wait bounded by `limit`; false if the abort flag is (or becomes)
// set or the limit expires (then the flag is set and the timeout recorded).
__device__ __forceinline__ bool tf_mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             uint32_t* status, unsigned long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        atomicOr(status, DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Poll a seq-tagged flag of another CTA (acquire), bounded likewise.
__device__ __forceinline__ bool tf_flag_wait(const int* f, int seq, volatile int* abort_flag, uint32_t* status,
                                             unsigned long long limit) {
  if (ld_acquire_gpu(f) == seq) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(f) == seq) return true;
    if ((it & 7u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        atomicOr(status, DEV_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__global__ void __launch_bounds__(TC_THREADS, 1) k_tile_fused(const __grid_constant__ TfArgs a) {
  constexpr uint32_t NCOLS = tmem_cols_for(TF_NSLOT * TF_SLOT_COLS);
  constexpr uint32_t IDESC = idesc_bf16_f32(TC_BM, TF_BN);        // B: 32 token rows
  constexpr uint32_t IDESC2 = idesc_bf16_f32(TC_BM, 2 * TF_BN);   // B: the h pair, hi rows then lo rows
  const TfLayout L = tf_layout(a.tw.C);
  const int STAGES = L.stages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + TF_MAX_STAGES;
  uint64_t* accfull = empty + TF_MAX_STAGES;  // [TF_NSLOT]
  uint64_t* accfree = accfull + TF_NSLOT;     // [TF_NSLOT]
  uint64_t* mma_done = accfree + TF_NSLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* scratch = smem + L.scratch;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int j0 = __ldg(a.job_off + cta), j1 = __ldg(a.job_off + cta + 1);
  const int seq = a.seq;
  const int T = a.tw.T;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < TF_NSLOT; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accfree[b], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      // Two cursors over the same block sequence: weight boxes run ahead as
      // ring stages free up; each B load follows once its operand is
      // published.  A stage's barrier expects both.
      tma_prefetch_desc(&a.mgate);
      tma_prefetch_desc(&a.mup);
      tma_prefetch_desc(&a.mdT);
      if (a.lowrank) tma_prefetch_desc(&a.mAt);
      TfIter ia, ib;
      ia.init(a, j0, j1);
      ib.init(a, j0, j1);
      int ai = 0, bi = 0;
      auto stage = [&](int i) { return smem + (size_t)(i % STAGES) * TF_STAGE_BYTES; };
      auto issue_a = [&](int i) {
        uint64_t* bar = &full[i % STAGES];
        mbar_expect_tx(bar, (uint32_t)(TF_A_BYTES + (ia.seg.kind == 2 ? 2 : 1) * TF_B_BYTES));
        const int c0 = ia.kb * TC_BK, c1 = ia.seg.arow;
        switch (ia.seg.amap) {  // (one call per map: the maps stay kernel parameters)
          case TFA_GATE: tma_load_2d(stage(i), &a.mgate, bar, c0, c1); break;
          case TFA_AT: tma_load_2d(stage(i), &a.mAt, bar, c0, c1); break;
          case TFA_UP: tma_load_2d(stage(i), &a.mup, bar, c0, c1); break;
          default: tma_load_2d(stage(i), &a.mdT, bar, c0, c1); break;
        }
      };
      auto issue_b = [&](int i) {
        uint64_t* bar = &full[i % STAGES];
        uint8_t* sb = stage(i) + TF_A_BYTES;
        const int c0 = ib.kb * TC_BK;
        if (ib.seg.kind == 0) {
          tma_load_2d(sb, &a.mx, bar, c0, 0);
        } else if (ib.seg.kind == 1) {
          tma_load_2d(sb, &a.mz, bar, c0, 0);
        } else {  // hi rows then lo rows: one 64-row B operand
          tma_load_2d(sb, &a.mhi, bar, c0, 0);
          tma_load_2d(sb + TF_B_BYTES, &a.mlo, bar, c0, 0);
        }
      };
      // the weights' first stages, before the previous grid has finished
      while (ia.valid() && ai < STAGES) {
        issue_a(ai++);
        ia.next(a);
      }
      griddep_wait();
      // tile pairs [hz_lo, hz_hi) of the B operand kind hz_kind are known to
      // be published; flags are read eight at a time (independent loads, one
      // acquire fence), since a down range walks many tiles
      int hz_kind = -1, hz_lo = 0, hz_hi = 0;
      bool abort = false;
      uint64_t t_last = globaltimer();
      for (uint32_t spin = 0;; ++spin) {
        bool prog = false;
        while (bi < ai) {
          if (!abort && ib.seg.kind != 0) {
            const int tile = ib.kb >> 2;  // 4 K blocks of 64 per 256-row pair
            if (ib.seg.kind != hz_kind || tile < hz_lo || tile >= hz_hi) {
              // flags of up to 8 pairs of h, or 2 pairs of z (four parts each)
              const int per = ib.seg.kind == 1 ? TF_ZPARTS : 1;
              const int* f = ib.seg.kind == 1 ? a.f_z + tile * TF_ZPARTS : a.f_h + tile;
              const int nf = min(8, (((ib.seg.k1 - 1) >> 2) - tile + 1) * per);
              int fv[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) fv[q] = q < nf ? ld_relaxed_gpu(f + q) : 0;
              int nq = 0;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (nq == q && fv[q] == seq) ++nq;
              const int n = nq / per;  // whole pairs
              if (n == 0) break;
              fence_acq_rel_gpu();          // acquire what those flags' releases published
              fence_proxy_async_global();   // written by generic stores, read by TMA
              hz_kind = ib.seg.kind;
              hz_lo = tile;
              hz_hi = tile + n;
            }
          }
          issue_b(bi++);
          ib.next(a);
          prog = true;
        }
        if (!abort && ia.valid()) {
          const int f = ai / STAGES;
          if (mbar_test_wait(&empty[ai % STAGES], (uint32_t)((f - 1) & 1))) {
            issue_a(ai++);
            ia.next(a);
            prog = true;
            if (!ia.valid()) griddep_launch();  // this CTA streams no more weights
          }
        }
        if (bi >= ai && (abort || !ia.valid())) break;
        if (prog) {
          t_last = globaltimer();
        } else {
          __nanosleep(64);  // leave the issue slots to the epilogue warps
        }
        if (!prog && (spin & 15u) == 0u && !abort) {
          if (*abort_flag) {
            abort = true;
          } else if (globaltimer() - t_last > a.wait_ns) {
            abort = true;
            *abort_flag = 1;
            atomicOr(a.status, DEV_ERR_TIMEOUT);
          }
        }
      }
      // the last fill of every stage has landed before the CTA can exit
      for (int s = 0; s < STAGES && s < ai; ++s) {
        const int last = s + STAGES * ((ai - 1 - s) / STAGES);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&full[s], (uint32_t)((last / STAGES) & 1))) {
          if (globaltimer() - t0 > a.wait_ns) {
            atomicOr(a.status, DEV_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      // Per stage, both 128-row halves of the weight box against the stage's
      // B tile, into the two halves of the segment's accumulator slot.
      int i = 0, c = 0;
      bool ok = true;
      for (int jj = j0; jj < j1 && ok; ++jj) {
        const int4 job = __ldg(a.jobs + jj);
        for (int sg = 0; sg < tf_nseg(job) && ok; ++sg, ++c) {
          const TfSeg seg = tf_seg(a, job, sg);
          const int slot = c % TF_NSLOT, use = c / TF_NSLOT;
          if (use > 0 && !tf_mbar_wait(&accfree[slot], (uint32_t)((use - 1) & 1), abort_flag, a.status, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem + (uint32_t)(slot * TF_SLOT_COLS);
          const uint32_t idesc = seg.kind == 2 ? IDESC2 : IDESC;
          for (int kb = seg.k0; kb < seg.k1; ++kb, ++i) {
            const int s = i % STAGES;
            if (!tf_mbar_wait(&full[s], (uint32_t)((i / STAGES) & 1), abort_flag, a.status, a.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint8_t* st = smem + (size_t)s * TF_STAGE_BYTES;
            const uint64_t bd = sdesc_k_sw128(smem_u32(st + TF_A_BYTES));
#pragma unroll
            for (int h = 0; h < TF_PAIR; ++h) {
              const uint64_t ad = sdesc_k_sw128(smem_u32(st + h * TC_A_BYTES));
#pragma unroll
              for (int k = 0; k < TC_BK / 16; ++k)
                tc_mma(dcol + (uint32_t)(h * 64), ad + 2u * k, bd + 2u * k, idesc, (kb == seg.k0 && k == 0) ? 0u : 1u);
            }
            tc_commit(&empty[s]);
          }
          if (ok) tc_commit(&accfull[slot]);
        }
      }
      // every MMA of this CTA has completed before TMEM is freed
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(mma_done, 0)) {
        if (globaltimer() - t0 > a.wait_ns) {
          atomicOr(a.status, DEV_ERR_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int etid = threadIdx.x;  // 0..127
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const int rows = min(TF_BN, a.maxT);  // rows of z and h that the B loads read
    griddep_wait();  // out and the workspace belong to the stream order
    {
      // this CTA's slice of out, zeroed before any DOWN job adds into it
      const long long n = (long long)T * a.d;
      if ((reinterpret_cast<uintptr_t>(a.out) & 15u) == 0) {
        float4* o4 = reinterpret_cast<float4*>(a.out);
        for (long long e = (long long)cta * 128 + etid; e < n / 4; e += (long long)gridDim.x * 128)
          o4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        for (long long e = (long long)cta * 128 + etid; e < n; e += (long long)gridDim.x * 128) a.out[e] = 0.f;
      }
      __threadfence();
      named_bar_sync(1, 128);
      if (etid == 0) st_release_gpu(a.f_zero + cta, seq);
    }
    int c = 0;
    bool zero_seen = false;
    // accumulator slot of segment c: wait for it (one thread waits; the
    // barrier's reduction gives all 128 the outcome) ...
    auto take = [&](int cs) -> bool {
      const int slot = cs % TF_NSLOT, use = cs / TF_NSLOT;
      bool ok = true;
      if (etid == 0) ok = tf_mbar_wait(&accfull[slot], (uint32_t)(use & 1), abort_flag, a.status, a.wait_ns);
      if (!named_bar_and(1, 128, ok)) return false;
      tc_fence_after();
      return true;
    };
    // ... read half h (32 columns, or 64: hi | lo) ...
    auto ld_half = [&](int cs, int h, float* v, bool pair64) {
      const uint32_t col = tl + (uint32_t)((cs % TF_NSLOT) * TF_SLOT_COLS + h * 64);
      tmem_ld16(col, v);
      tmem_ld16(col + 16, v + 16);
      if (pair64) {  // the lo half's product, added to the hi half's
        float w[TF_BN];
        tmem_ld16(col + 32, w);
        tmem_ld16(col + 48, w + 16);
#pragma unroll
        for (int t = 0; t < TF_BN; ++t) v[t] += w[t];
      }
    };
    // ... and hand the slot back to the MMAs
    auto release = [&](int cs) {
      tc_fence_before();
      named_bar_sync(1, 128);
      if (etid == 0) mbar_arrive(&accfree[cs % TF_NSLOT]);
    };
    // wait for the flags f[0 .. n) of other CTAs, one thread per flag (the
    // loads in parallel); the barrier's reduction gives all 128 the outcome
    auto wait_flags = [&](const int* f, int n) -> bool {
      bool ok = true;
      for (int q = etid; q < n && ok; q += 128) ok = tf_flag_wait(f + q, seq, abort_flag, a.status, a.wait_ns);
      ok = named_bar_and(1, 128, ok);
      fence_acq_rel_gpu();
      return ok;
    };
    auto publish = [&](int* flag) {
      __threadfence();
      named_bar_sync(1, 128);
      if (etid == 0) st_release_gpu(flag, seq);
    };
    // partial sum [2][32][128] of slot q: element (h, t) of this thread
    auto part = [&](float* base, int q, int h, int t) { return base + ((size_t)q * TF_PAIR + h) * (TF_BN * 128) + t * 128 + etid; };

    for (int jj = j0; jj < j1; ++jj) {
      const int4 job = __ldg(a.jobs + jj);
      const int type = tf_type(job), tile = job.y, id = job.w;
      const int count = (job.x >> 8) & 0xFF, gcount = (job.x >> 16) & 0xFF;
      const int cs = c;
      c += tf_nseg(job);
      if (type == TFJ_Z) {
        // (the z jobs open the list: every piece stores and publishes its
        // partial sum before any of them waits, see below)
        if (!take(cs)) break;
#pragma unroll
        for (int h = 0; h < TF_PAIR; ++h) {
          float v[TF_BN];
          ld_half(cs, h, v, false);
#pragma unroll
          for (int t = 0; t < TF_BN; ++t) __stcg(part(a.zpart, id, h, t), v[t]);
        }
        release(cs);
        publish(a.f_zp + id);
        const bool last_z = jj + 1 == j1 || tf_type(__ldg(a.jobs + jj + 1)) != TFJ_Z;
        bool ok = true;
        for (int jf = j0; last_z && jf <= jj && ok; ++jf) {
          // the finishers among this list's z pieces: every piece's partial
          // sum of the rank pair, in K order, for their parts of z
          const int4 zj = __ldg(a.jobs + jf);
          if (!((zj.x >> 4) & 1)) continue;
          const int zq = (zj.x >> 16) & 0xFF, zc = (zj.x >> 8) & 0xFF, zt = zj.y;
          const int first = zj.w - zq, nfin = min(TF_ZPARTS, zc), f = zq - (zc - nfin);
          ok = wait_flags(a.f_zp + first, zc);
          for (int pt = f; pt < TF_ZPARTS && ok; pt += nfin) {
            const int h = pt >> 1, r = (zt * TF_PAIR + h) * 128 + etid;
#pragma unroll 1
            for (int t0 = (pt & 1) * 16; t0 < (pt & 1) * 16 + 16; t0 += 8) {
              // eight tokens of every piece, all loads in flight together
              float pv[TF_ZMAXP][8];
#pragma unroll
              for (int qq = 0; qq < TF_ZMAXP; ++qq)
#pragma unroll
                for (int t = 0; t < 8; ++t) pv[qq][t] = qq < zc ? __ldcg(part(a.zpart, first + qq, h, t0 + t)) : 0.f;
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                float zs = 0.f;
#pragma unroll
                for (int qq = 0; qq < TF_ZMAXP; ++qq)
                  if (qq < zc) zs += pv[qq][t];
                const int tt = t0 + t;
                if (r < a.R && tt < rows) a.z[(size_t)tt * a.R + r] = __float2bfloat16_rn(tt < T ? zs : 0.f);
              }
            }
            fence_proxy_async_global();  // read by other CTAs' TMA loads
            publish(a.f_z + zt * TF_ZPARTS + pt);
          }
        }
        if (!ok) break;
      } else if (type == TFJ_MAIN) {
        // slot cs: this job's up range; slot cs + 1: its gate range.  Per
        // half: g = the earlier K ranges' partial sums, then the gate range,
        // then the bias, in K order; the TwELL emission; u = the up range
        // plus the later K ranges' partial sums; h = v·u as hi + lo
        if (count > 0 && !wait_flags(a.f_up + id + gcount, count)) break;
        if (gcount > 0 && !wait_flags(a.f_up + id, gcount)) break;
        if (!take(cs + 1)) break;  // (the gate range comes after the up range)
        for (int h = 0; h < TF_PAIR; ++h) {
          const int p = tile * TF_PAIR + h;     // the 128-neuron tile
          if (p >= a.tw.n_tiles) break;         // (uniform: the pair's second tile may not exist)
          const int j = p * 128 + etid;
          const float bj = a.bias ? __ldg(a.bias + j) : 0.f;
          float g[TF_BN];
#pragma unroll
          for (int t = 0; t < TF_BN; ++t) g[t] = 0.f;
          for (int q = 0; q < gcount; ++q) {
            float pv[TF_BN];
#pragma unroll
            for (int t = 0; t < TF_BN; ++t) pv[t] = __ldcg(part(a.upart, id + q, h, t));
#pragma unroll
            for (int t = 0; t < TF_BN; ++t) g[t] += pv[t];
          }
          {
            float gv[TF_BN];
            ld_half(cs + 1, h, gv, false);
#pragma unroll
            for (int t = 0; t < TF_BN; ++t) g[t] = (gcount > 0 ? g[t] + gv[t] : gv[t]) + bj;
          }
          twell_tile32<TF_BN>(a.tw, g, j, 0, etid, scratch, 1);  // (a.tw.bias is null)
          float u[TF_BN];
          ld_half(cs, h, u, false);
          for (int q = gcount; q < gcount + count; ++q) {
            float pv[TF_BN];
#pragma unroll
            for (int t = 0; t < TF_BN; ++t) pv[t] = __ldcg(part(a.upart, id + q, h, t));
#pragma unroll
            for (int t = 0; t < TF_BN; ++t) u[t] += pv[t];
          }
          const uint32_t* masks = reinterpret_cast<const uint32_t*>(scratch);                 // [32][4]
          const uint16_t* vals = reinterpret_cast<const uint16_t*>(scratch + TF_BN * 4 * 4);  // [32][TW32_VP]
          const int wq = etid >> 5, bit = etid & 31;
#pragma unroll
          for (int t = 0; t < TF_BN; ++t) {
            if (t >= rows) break;
            float hv = 0.f;
            if (t < T && ((masks[t * 4 + wq] >> bit) & 1u))
              hv = __uint_as_float((uint32_t)vals[t * TW32_VP + etid] << 16) * u[t];
            const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
            const __nv_bfloat16 lo = __float2bfloat16_rn(hv - __bfloat162float(hi));
            a.h_hi[(size_t)t * a.tw.F + j] = hi;
            a.h_lo[(size_t)t * a.tw.F + j] = lo;
          }
        }
        release(cs);
        release(cs + 1);
        fence_proxy_async_global();  // read by other CTAs' TMA loads
        publish(a.f_h + tile);
      } else if (type == TFJ_HELP || type == TFJ_GHELP) {
        if (!take(cs)) break;
#pragma unroll
        for (int h = 0; h < TF_PAIR; ++h) {
          float v[TF_BN];
          ld_half(cs, h, v, false);
#pragma unroll
          for (int t = 0; t < TF_BN; ++t) __stcg(part(a.upart, id, h, t), v[t]);
        }
        release(cs);
        publish(a.f_up + id);
      } else {
        if (!take(cs)) break;
        float y[TF_PAIR][TF_BN];
#pragma unroll
        for (int h = 0; h < TF_PAIR; ++h) ld_half(cs, h, y[h], true);
        release(cs);
        if (!zero_seen) {  // every CTA's slice of out is zeroed
          if (!wait_flags(a.f_zero, a.n_chunks)) break;
          zero_seen = true;
        }
#pragma unroll
        for (int h = 0; h < TF_PAIR; ++h) {
          const int colo = (tile * TF_PAIR + h) * 128 + etid;
          if (colo < a.d) {
#pragma unroll
            for (int t = 0; t < TF_BN; ++t)
              if (t < T) atomicAdd(a.out + (size_t)t * a.d + colo, y[h][t]);
          }
        }
      }
    }
  }
  griddep_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

}  // namespace sffn
