// C ABI of the activation-sparse gated FFN forward (see include/sffn.h):
// argument validation, workspace, TMA tensor maps and the launch sequence.
//
// Launch sequence of one bf16 forward (all on the caller's stream):
//   gate    tensor-core tile kernel, epilogue = TwELL emission (threshold) or
//           dense value + score (WINA, then the top-k kernel emits TwELL);
//           low-rank gate = two tile kernels (z = bf16(x·A) split over K, then
//           g = z·B with the TwELL epilogue); up to 8 tokens: a row-streaming
//           gate over every SM with the same epilogue
//   ROWS    fused up x down over the kept rows of each 8-token block
//           (non-overflow tokens; the kernel also routes the overflow tokens,
//           and the gate zeroes out when the kernel adds partial sums into it)
//   TILES   tensor-core u per tile with h from TwELL (non-overflow tokens);
//           the first tile's CTA routes the overflow tokens, the gate zeroes out
//   dense   tensor-core recompute of g and u for overflow tokens -> h
//   down    tensor-core y = h·W_down for the h rows (overflow rows on ROWS,
//           all rows on TILES)
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/sffn.h"
#include "epilogues.cuh"
#include "decode_fused.cuh"
#include "tc_gate_persist.cuh"
#include "gate_rows.cuh"
#include "gsi.cuh"
#include "moe.cuh"
#include "backward.cuh"
#include "rows_mma.cuh"
#include "tile_fused.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"

using namespace sffn;

#define SFFN_VERSION_STRING "sffn 0.1.0 (sm_100a)"

namespace {

constexpr int kNumSMsFallback = 148;
constexpr int kMaxMarks = 12;
enum KernelLabel { L_GATE_Z, L_GATE, L_WINA_TOPK, L_ROUTER, L_UPDOWN_ROWS, L_TILE_H, L_FALLBACK_H, L_DOWN,
                   L_GATE_F32, L_ROWS_F32, L_FALLBACK_F32, L_DECODE, L_ROTATE_X, L_INPUT_SELECT,
                   L_GSI_PROJECT, L_GSI_RESID, L_GSI_OUT, L_MOE_ROUTE, L_MOE_COMBINE,
                   L_BWD_INDEX, L_BWD_TOKEN, L_BWD_NEURON, L_BWD_DENSE, L_TILE_FUSED, L_COUNT };
const char* const kLabelNames[L_COUNT] = {"gate_lowrank_z", "gate", "wina_topk", "router", "updown_rows",
                                          "tile_h", "fallback_h", "down", "gate_f32", "rows_f32",
                                          "fallback_f32", "decode_fused", "rotate_x", "input_select",
                                          "gsi_project", "gsi_resid", "gsi_out", "moe_route", "moe_combine",
                                          "bwd_index", "bwd_token", "bwd_neuron", "bwd_dense", "tile_fused"};
constexpr int kMaxTokensLimit = 16384;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][inner] matrix, box = 64 x box_rows,
// 128-byte swizzle (the K-major operand layout of the tile kernel).
bool make_map(CUtensorMap* m, const void* base, long long inner, long long rows, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int pick_bn(int n) { return n <= 16 ? 16 : n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : 256; }
int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// K splits of the z = x·A GEMM: only with one token tile (up to 256 tokens),
// at most Z_MAX_SPLITS, at least 4 K blocks each, and no more CTAs than SMs
// (the splits' sum is a serial step at the end, so few long splits beat many)
int z_splits(int d, int m_tiles, int tok_tiles, int n_sm) {
  if (tok_tiles != 1) return 1;
  return std::max(1, std::min({Z_MAX_SPLITS, cdiv(d, 64) / 4, n_sm / m_tiles}));
}

// Job lists of the tile path's single launch (tile_fused.cuh) for n_chunks
// CTAs, in 64-wide K blocks:
//   phase 0 (low-rank gate): each rank tile's z range cut into pieces of
//     about kZPiece blocks, spread over the CTAs as their first jobs;
//   phase 1: the stream [gate of tile 0][up of tile 0] ... [gate of tile
//     P-1][up of tile P-1] cut into n_chunks runs, each CTA's run shortened
//     by its z blocks so that phases 0 and 1 together are even;
//   phase 2: the stream [down of output tile 0] ... [down of output tile
//     Md-1] cut into n_chunks runs of equal length.
// A tile here is the kernel's unit, a pair of 128-row tiles (P, Rt and Md
// count pairs).
// Phase-1 cuts are moved so that the run holding the end of a tile's gate
// also holds at least kMinPiece blocks of its up range (the MAIN job), and so
// that no gate or up piece shorter than kMinPiece is cut off (2 for down).
// The earlier pieces of a gate (GHELP) and the later pieces of an up range
// (HELP) are partial sums that the MAIN adds in K order; a tile's helper
// slots are consecutive, gate pieces first.  The z pieces of a rank tile have
// consecutive slots in K order; the last one adds them up.
struct TfSchedule {
  std::vector<int4> jobs;
  std::vector<int> off;   // [n_chunks + 1]
  int n_zp = 0, n_help = 0;
  bool ok = true;
};

TfSchedule tf_schedule(int n_chunks, int kd, int kg, int P, int Rt, int Md, int Kf) {
  constexpr int kMinPiece = 2, kZPiece = 8;
  struct Item {
    int type, tile;
    long long s, e;
  };
  TfSchedule S;
  // phase 0: z pieces, piece i of nz to chunk i * n_chunks / nz
  const int zper = Rt ? std::min(TF_ZMAXP, std::max(1, cdiv(kd, kZPiece))) : 0, nz = Rt * zper;
  std::vector<std::vector<int4>> zjobs(n_chunks);
  std::vector<long long> zload(n_chunks, 0);
  for (int i = 0; i < nz; ++i) {
    const int r = i / zper, q = i % zper;
    const int k0 = (int)((long long)kd * q / zper), k1 = (int)((long long)kd * (q + 1) / zper);
    const int c = (int)((long long)i * n_chunks / nz);
    if (k1 <= k0) S.ok = false;
    zjobs[c].push_back(tf_job(TFJ_Z, q >= zper - std::min(TF_ZPARTS, zper) ? 1 : 0, zper, q, r, k0, k1, i));
    zload[c] += k1 - k0;
  }
  S.n_zp = nz;

  std::vector<Item> p1, p2;
  long long pos = 0;
  for (int p = 0; p < P; ++p) {
    p1.push_back({TFJ_MAIN, p, pos, pos + kg});  // the gate
    pos += kg;
    p1.push_back({TFJ_HELP, p, pos, pos + kd});  // the up range
    pos += kd;
  }
  const long long W1 = pos;
  pos = 0;
  for (int m = 0; m < Md; ++m, pos += Kf) p2.push_back({TFJ_DOWN, m, pos, pos + Kf});
  const long long W2 = pos;

  // target[i] = where run i - 1 should end (before the moves)
  auto cuts = [&](long long W, const std::vector<Item>& items, int minp, const std::vector<long long>& target) {
    std::vector<long long> c(n_chunks + 1, 0);
    size_t k = 0;
    for (int i = 1; i <= n_chunks; ++i) {
      long long x = std::min(std::max(target[i], 0LL), W);
      if (i < n_chunks) {
        while (k < items.size() && items[k].e <= x) ++k;
        if (k < items.size()) {
          const Item& q = items[k];
          const long long len = q.e - q.s, m = std::min<long long>(minp, len);
          if (x < q.s + m) x = q.type == TFJ_HELP ? q.s + m : q.s;  // an up range's first blocks stay with its gate
          if (x > q.e - m && x < q.e) x = q.type == TFJ_MAIN ? q.e - m : q.e;  // a gate's last blocks too
        }
      } else {
        x = W;
      }
      c[i] = std::max(x, c[i - 1]);
    }
    return c;
  };
  std::vector<long long> t1(n_chunks + 1, 0), t2(n_chunks + 1, 0);
  {
    long long tot = W1;
    for (long long v : zload) tot += v;
    double acc = 0.0;
    for (int i = 1; i <= n_chunks; ++i) {
      acc += (double)tot / n_chunks - (double)zload[i - 1];
      t1[i] = (long long)(acc + 0.5);
      t2[i] = W2 * i / n_chunks;
    }
  }
  const std::vector<long long> c1 = cuts(W1, p1, kMinPiece, t1), c2 = cuts(W2, p2, 2, t2);

  // pass 1: pieces per chunk, helper slots numbered in stream order
  std::vector<int> gcount(P, 0), ucount(P, 0), hfirst(P, -1), main_job(P, -1);
  struct Piece {
    int type, tile, k0, k1, id;
  };
  std::vector<std::vector<Piece>> per(n_chunks);
  int hp = 0;
  auto overlap = [](const Item& q, long long lo, long long hi, long long& s0, long long& s1) {
    s0 = std::max(lo, q.s);
    s1 = std::min(hi, q.e);
    return s0 < s1;
  };
  for (int c = 0; c < n_chunks; ++c) {
    long long s0, s1;
    for (size_t k = 0; k < p1.size(); ++k) {
      const Item& q = p1[k];
      if (!overlap(q, c1[c], c1[c + 1], s0, s1)) continue;
      const int k0 = (int)(s0 - q.s), k1 = (int)(s1 - q.s);
      if (q.type == TFJ_MAIN && s1 == q.e) {  // the gate's last piece: the MAIN job
        const Item& u = p1[k + 1];
        const long long u1 = std::min(c1[c + 1], u.e);
        if (u1 <= u.s) S.ok = false;  // no up blocks after the gate
        per[c].push_back({TFJ_MAIN, q.tile, k0, (int)(u1 - u.s), -1});
      } else if (q.type == TFJ_MAIN) {
        if (hfirst[q.tile] < 0) hfirst[q.tile] = hp;
        ++gcount[q.tile];
        per[c].push_back({TFJ_GHELP, q.tile, k0, k1, hp++});
      } else if (s0 != q.s) {  // an up range's start belongs to the MAIN job
        if (hfirst[q.tile] < 0) hfirst[q.tile] = hp;
        ++ucount[q.tile];
        per[c].push_back({TFJ_HELP, q.tile, k0, k1, hp++});
      }
    }
    for (const Item& q : p2)
      if (overlap(q, c2[c], c2[c + 1], s0, s1)) per[c].push_back({TFJ_DOWN, q.tile, (int)(s0 - q.s), (int)(s1 - q.s), 0});
  }
  // pass 2: records
  S.off.assign(n_chunks + 1, 0);
  for (int c = 0; c < n_chunks; ++c) {
    S.off[c] = (int)S.jobs.size();
    for (const int4& z : zjobs[c]) S.jobs.push_back(z);
    for (const Piece& q : per[c]) {
      if (q.k1 > 0xFFFF) S.ok = false;
      if (q.type == TFJ_MAIN) {
        if (main_job[q.tile] >= 0 || q.k0 >= kg || q.k1 < 1 || gcount[q.tile] > 0xFF || ucount[q.tile] > 0xFF)
          S.ok = false;
        main_job[q.tile] = (int)S.jobs.size();
        S.jobs.push_back(tf_job(TFJ_MAIN, 0, ucount[q.tile], gcount[q.tile], q.tile, q.k0, q.k1,
                                std::max(hfirst[q.tile], 0)));
      } else {
        if (q.k1 <= q.k0) S.ok = false;
        S.jobs.push_back(tf_job(q.type, 0, 0, 0, q.tile, q.k0, q.k1, q.id));
      }
    }
  }
  S.off[n_chunks] = (int)S.jobs.size();
  if (zper > TF_ZMAXP) S.ok = false;
  for (int p = 0; p < P; ++p)
    if (main_job[p] < 0) S.ok = false;
  S.n_help = hp;
  return S;
}

// Launch with programmatic dependent launch: the kernel may be scheduled while
// the previous kernel on the stream drains; it calls griddepcontrol.wait before
// touching data an earlier kernel writes or reads.  cluster_x > 1 also sets
// the thread-block cluster size.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

template <int BN, class Epi>
cudaError_t launch_tc_bn(dim3 grid, cudaStream_t st, const CUtensorMap& a0, const CUtensorMap& b0,
                         const CUtensorMap& a1, const CUtensorMap& b1, const TcArgs& args,
                         const typename Epi::Params& ep) {
  return launch_pdl(k_tc_gemm<BN, Epi>, grid, dim3(TC_THREADS), TcCfgOf<BN, Epi>::SMEM, st, 1, a0, b0, a1, b1, args, ep);
}

template <class Epi>
cudaError_t launch_tc(int BN, dim3 grid, cudaStream_t st, const CUtensorMap& a0, const CUtensorMap& b0,
                      const CUtensorMap& a1, const CUtensorMap& b1, const TcArgs& args,
                      const typename Epi::Params& ep) {
  switch (BN) {
    case 16: return launch_tc_bn<16, Epi>(grid, st, a0, b0, a1, b1, args, ep);
    case 32: return launch_tc_bn<32, Epi>(grid, st, a0, b0, a1, b1, args, ep);
    case 64: return launch_tc_bn<64, Epi>(grid, st, a0, b0, a1, b1, args, ep);
    case 128: return launch_tc_bn<128, Epi>(grid, st, a0, b0, a1, b1, args, ep);
    default: return launch_tc_bn<256, Epi>(grid, st, a0, b0, a1, b1, args, ep);
  }
}

// The persistent gate for as many 128-neuron x BN-token tiles as there are
// SMs or more: one CTA per SM walks the tiles (tc_gate_persist.cuh).
cudaError_t launch_gate_persist(int BN, int n_sm, int n_work, cudaStream_t st, const CUtensorMap& a,
                                const CUtensorMap& b, const TcArgs& args, const TwellParams& tw) {
  const dim3 grid(std::min(n_sm, n_work)), block(TP_THREADS);
  const size_t smem = (size_t)tp_layout(BN, tw.C).total;
  switch (BN) {
    case 16: return launch_pdl(k_tc_gate_persist<16>, grid, block, smem, st, 1, a, b, args, tw);
    case 32: return launch_pdl(k_tc_gate_persist<32>, grid, block, smem, st, 1, a, b, args, tw);
    case 64: return launch_pdl(k_tc_gate_persist<64>, grid, block, smem, st, 1, a, b, args, tw);
    case 128: return launch_pdl(k_tc_gate_persist<128>, grid, block, smem, st, 1, a, b, args, tw);
    default: return launch_pdl(k_tc_gate_persist<256>, grid, block, smem, st, 1, a, b, args, tw);
  }
}
cudaError_t set_gate_persist_attrs(int C) {
  cudaError_t e = cudaSuccess;
  e = e ? e : cudaFuncSetAttribute(k_tc_gate_persist<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, tp_layout(16, C).total);
  e = e ? e : cudaFuncSetAttribute(k_tc_gate_persist<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, tp_layout(32, C).total);
  e = e ? e : cudaFuncSetAttribute(k_tc_gate_persist<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, tp_layout(64, C).total);
  e = e ? e : cudaFuncSetAttribute(k_tc_gate_persist<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, tp_layout(128, C).total);
  e = e ? e : cudaFuncSetAttribute(k_tc_gate_persist<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, tp_layout(256, C).total);
  return e;
}

template <class Epi>
cudaError_t set_tc_attrs() {
  cudaError_t e = cudaSuccess;
  e = e ? e : cudaFuncSetAttribute(k_tc_gemm<16, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfgOf<16, Epi>::SMEM);
  e = e ? e : cudaFuncSetAttribute(k_tc_gemm<32, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfgOf<32, Epi>::SMEM);
  e = e ? e : cudaFuncSetAttribute(k_tc_gemm<64, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfgOf<64, Epi>::SMEM);
  e = e ? e : cudaFuncSetAttribute(k_tc_gemm<128, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfgOf<128, Epi>::SMEM);
  e = e ? e : cudaFuncSetAttribute(k_tc_gemm<256, Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfgOf<256, Epi>::SMEM);
  return e;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

// Per-kernel device timing (sffn_timing_begin / sffn_gsi_timing_begin): CUDA
// events recorded on the launching stream before each kernel of every
// stride-th forward and after its last one.
struct KTiming {
  bool tm_on = false;
  bool tm_prev = false;             // the last tmark_begin opened a record
  int tm_max = 0, tm_n = 0, tm_cur = -1, tm_stride = 1, tm_seen = 0;
  std::vector<cudaEvent_t> tm_ev;   // [tm_max][kMaxMarks + 1]
  std::vector<int> tm_lab;          // [tm_max][kMaxMarks]
  std::vector<int> tm_nk;           // [tm_max]
};

struct sffn_handle : KTiming {
  sffn_desc desc;
  int dev = 0, n_sm = kNumSMsFallback;
  int d = 0, F = 0, P = 0, R = 0, C = 0, maxT = 0, esize = 2;
  bool f32 = false, wina = false, lowrank = false;
  bool fullh = false;            // WINA with the full-h score (wina is set too)
  // effective gate and up weights: the caller's, or their orthogonalised copies
  const __nv_bfloat16* Wg = nullptr;
  const __nv_bfloat16* Wu = nullptr;
  uint32_t epoch = 0;
  // workspace
  int16_t* count = nullptr;
  int16_t* idx = nullptr;
  void* val = nullptr;
  uint32_t* ovf = nullptr;
  uint32_t* kmask = nullptr;
  int* ovf_list = nullptr;
  int* ovf_count = nullptr;
  __nv_bfloat16* xo = nullptr;
  __nv_bfloat16* h_hi = nullptr;
  __nv_bfloat16* h_lo = nullptr;
  float* scores = nullptr;
  void* vdense = nullptr;
  float* norms = nullptr;
  __nv_bfloat16* z = nullptr;
  __nv_bfloat16* zo = nullptr;
  float* zpart = nullptr;   // split-K partials of z (up to 256 tokens)
  int* tickets = nullptr;
  __nv_bfloat16* At = nullptr;
  __nv_bfloat16* Bt = nullptr;
  __nv_bfloat16* WdT = nullptr;
  float* gdebug = nullptr;
  uint32_t* status = nullptr;
  void* xstage = nullptr;
  float* ostage = nullptr;
  float* hfull = nullptr;        // full-h WINA: h = v·u [T][F]
  float* colnorm = nullptr;      // input-side WINA: column norms of [W_gate; W_up] [d]
  double* colacc = nullptr;      // their fp64 sums (create time)
  __nv_bfloat16* xsel = nullptr; // input-side WINA: the selected x [T][d]
  __nv_bfloat16* Vt = nullptr;   // orthogonalisation: V^T [d][d]
  __nv_bfloat16* Wg_rot = nullptr;  // W_gate·V [F][d]
  __nv_bfloat16* Wu_rot = nullptr;  // W_up·V [F][d]
  __nv_bfloat16* xrot = nullptr;    // x·V [T][d]
  CUtensorMap tmVt;              // V^T rows as the A operand of x·V
  // backward workspace (SFFN_FLAG_BACKWARD)
  int* bw_wordpre = nullptr;
  int* bw_nnz = nullptr;
  int* bw_rowptr = nullptr;
  int2* bw_chunks = nullptr;
  int* bw_nchunks = nullptr;
  int* bw_counter = nullptr;
  float* bw_du = nullptr;
  float* bw_dg = nullptr;
  float* bw_h = nullptr;
  int* bw_colcnt = nullptr;
  int* bw_colptr = nullptr;
  int* bw_cscpos = nullptr;
  int* bw_csctok = nullptr;
  int bw_smem = 0;
  // the dense channel of the heavy (overflow) tokens; NP = max_tokens rounded up to 64
  int bw_NP = 0;
  int* bw_heavy = nullptr;
  int* bw_hlist = nullptr;
  int* bw_nheavy = nullptr;
  float* bw_dbh = nullptr;
  __nv_bfloat16 *bw_xh = nullptr, *bw_dyh_hi = nullptr, *bw_dyh_lo = nullptr;       // [NP][d]
  __nv_bfloat16 *bw_xhT = nullptr, *bw_dyhT_hi = nullptr, *bw_dyhT_lo = nullptr;    // [d][NP]
  float *bw_g = nullptr, *bw_u = nullptr;                                            // [NP][F]
  __nv_bfloat16 *bw_du_hi = nullptr, *bw_du_lo = nullptr, *bw_dg_hi = nullptr, *bw_dg_lo = nullptr;  // [NP][F]
  __nv_bfloat16 *bw_duT_hi = nullptr, *bw_duT_lo = nullptr, *bw_dgT_hi = nullptr, *bw_dgT_lo = nullptr;
  __nv_bfloat16 *bw_hT_hi = nullptr, *bw_hT_lo = nullptr;                            // [F][NP]
  __nv_bfloat16 *bw_WuT = nullptr, *bw_WgT = nullptr;                                // [d][F]
  CUtensorMap bm_Wd, bm_WuT, bm_WgT, bm_duT_hi, bm_duT_lo, bm_dgT_hi, bm_dgT_lo, bm_hT_hi, bm_hT_lo;  // A (128 rows)
  CUtensorMap bm_xh, bm_dyh_hi, bm_dyh_lo, bm_du_hi, bm_du_lo, bm_dg_hi, bm_dg_lo, bm_xhT, bm_dyhT_hi,
      bm_dyhT_lo;                                                                    // B (256 rows)
  void* arena = nullptr;         // the one device allocation all of the above live in
  size_t arena_bytes = 0;
  bool dense_bufs = false;       // xo, h_hi, h_lo and W_down^T exist (paths other than the single launch)
  // A-operand tensor maps (box 64 x 128)
  CUtensorMap tmWgate, tmWup, tmWdT, tmAt, tmBt;
  int last_T = 0, last_path = 0, last_launches = 0;
  int rows_nslot = 0, rows_lcap = 0, rows_smem = 0;
  bool rows_ok = false;                // the fused row kernel supports this shape
  int gate_stages = 0, down_stages = 0;  // ring depth of the gate and down tile kernels (0: all)
  // row-streaming gate for up to 8 tokens: tile staging, tickets, ring slots, shared memory
  float* gstage = nullptr;
  int* gtick = nullptr;
  int gr_nslot = 0, gr_smem = 0;
  bool gr_ok = false;
  // single persistent launch for T <= 8: scheduler words, published row lists, launch shape
  int* dsched = nullptr;
  int dsched_ints = 0;
  uint32_t* wl_id = nullptr;
  uint4* wl_val = nullptr;
  int dec_maxr = 0, dec_smem = 0, dec_grid = 0;
  bool dec_ok = false;
  bool dec_pdl = true;           // the single launch also asks for programmatic dependent launch
  unsigned last_attrs = 0;       // attributes of the last single launch (sffn_stats.launch_attrs)
  int dec_phantom = 0;           // test hook (sffn_debug_decode_waits)
  unsigned long long dec_wait_ns = SFFN_WAIT_LIMIT_NS;
  bool last_fused = false;     // the last forward was a single launch: its routing is the ovf flags
  uint32_t last_epoch = 0;
  // single persistent launch of the tile path (T <= 32): job lists, partial
  // sums and seq-tagged flags (tile_fused.cuh)
  int4* tf_jobs = nullptr;
  int* tf_off = nullptr;
  float* tf_upart = nullptr;
  float* tf_zpart = nullptr;
  int* tf_flags = nullptr;
  int tf_flag_ints = 0, tf_max_jobs = 0, tf_max_zp = 0, tf_max_help = 0;
  int tf_off_z = 0, tf_off_up = 0, tf_off_h = 0, tf_off_zero = 0;  // flag arrays in tf_flags (ints)
  int tf_smem = 0, tf_grid = 0, tf_chunks = 0;
  int tf_seq = 0;                // the last launch's sequence number
  bool tf_ok = false;
  bool tf_pdl = true;
  CUtensorMap tf_mgate, tf_mAt, tf_mup, tf_mdT;  // its weight maps (box 64 x 256)
};

namespace {

void timing_free(KTiming* h);

void free_handle(sffn_handle* h) {
  if (!h) return;
  timing_free(h);
  if (h->arena) cudaFree(h->arena);
  delete h;
}

// Carves the handle's workspace out of one device allocation: run once with
// base == nullptr to size it, then again with the allocation's base.  Every
// buffer starts on a 256-byte boundary (TMA and 16-byte vector accesses).
struct Arena {
  uint8_t* base = nullptr;
  size_t size = 0;
  template <typename T>
  void take(T** p, size_t bytes) {
    size = (size + 255) & ~size_t(255);
    *p = base ? reinterpret_cast<T*>(base + size) : nullptr;
    size += bytes ? bytes : 16;
  }
};

template <typename T>
bool dalloc(T** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  void* q = nullptr;
  if (cudaMalloc(&q, bytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  *p = static_cast<T*>(q);
  return true;
}

void tmark(KTiming* h, cudaStream_t st, int label) {
  if (!h->tm_on || h->tm_cur < 0) return;
  const int f = h->tm_cur, i = h->tm_nk[f];
  if (i >= kMaxMarks) return;
  cudaEventRecord(h->tm_ev[(size_t)f * (kMaxMarks + 1) + i], st);
  h->tm_lab[(size_t)f * kMaxMarks + i] = label;
  h->tm_nk[f] = i + 1;
}

void tmark_begin(KTiming* h) {
  h->tm_cur = -1;
  if (h->tm_on && (h->tm_seen++ % h->tm_stride) == 0 && h->tm_n < h->tm_max) {
    h->tm_cur = h->tm_n++;
    h->tm_nk[h->tm_cur] = 0;
  }
  h->tm_prev = h->tm_cur >= 0;
}

// A record for a pass that follows a forward (the backward, a MoE combine):
// opened exactly when the forward's own record was, so the stride counts
// forwards only.
void tmark_follow(KTiming* h) {
  h->tm_cur = -1;
  if (h->tm_on && h->tm_prev && h->tm_n < h->tm_max) {
    h->tm_cur = h->tm_n++;
    h->tm_nk[h->tm_cur] = 0;
  }
}

void tmark_end(KTiming* h, cudaStream_t st) {
  if (!h->tm_on || h->tm_cur < 0) return;
  const int f = h->tm_cur;
  cudaEventRecord(h->tm_ev[(size_t)f * (kMaxMarks + 1) + h->tm_nk[f]], st);
  h->tm_cur = -1;
}

void timing_free(KTiming* h) {
  for (cudaEvent_t e : h->tm_ev)
    if (e) cudaEventDestroy(e);
  h->tm_ev.clear();
  h->tm_lab.clear();
  h->tm_nk.clear();
  h->tm_on = false;
  h->tm_max = h->tm_n = 0;
  h->tm_cur = -1;
}

sffn_status validate(const sffn_desc* d) {
  if (!d) return SFFN_ERR_INVALID_ARG;
  if (d->d_model <= 0 || d->d_ff <= 0 || d->max_tokens <= 0 || d->rank < 0) return SFFN_ERR_INVALID_ARG;
  if (d->dtype != SFFN_BF16 && d->dtype != SFFN_FP32) return SFFN_ERR_INVALID_ARG;
  if (d->mode != SFFN_MODE_RELU_THRESHOLD && d->mode != SFFN_MODE_WINA_TOPK && d->mode != SFFN_MODE_WINA_FULL_H)
    return SFFN_ERR_INVALID_ARG;
  if (d->act != SFFN_ACT_RELU && d->act != SFFN_ACT_SILU) return SFFN_ERR_INVALID_ARG;
  if (d->path < SFFN_PATH_AUTO || d->path > SFFN_PATH_TILES) return SFFN_ERR_INVALID_ARG;
  const int C = d->tile_capacity;
  if (C != 8 && C != 16 && C != 32 && C != 64 && C != 128) return SFFN_ERR_INVALID_ARG;
  if (d->mode == SFFN_MODE_RELU_THRESHOLD && (!(d->threshold >= 0.0f) || !std::isfinite(d->threshold)))
    return SFFN_ERR_INVALID_ARG;
  if (d->mode != SFFN_MODE_RELU_THRESHOLD && (d->k < 0 || d->k > d->d_ff)) return SFFN_ERR_INVALID_ARG;
  if (d->input_k < 0 || d->input_k > d->d_model) return SFFN_ERR_INVALID_ARG;
  if (d->V && !aligned16(d->V)) return SFFN_ERR_INVALID_ARG;
  if (!d->W_up || !d->W_down) return SFFN_ERR_INVALID_ARG;
  if (d->rank == 0 && (!d->W_gate || d->A || d->B)) return SFFN_ERR_INVALID_ARG;
  if (d->rank > 0 && (d->W_gate || !d->A || !d->B)) return SFFN_ERR_INVALID_ARG;
  const void* ptrs[] = {d->W_gate, d->A, d->B, d->W_up, d->W_down, d->gate_bias};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return SFFN_ERR_INVALID_ARG;
  if (d->d_model % 8 != 0) return SFFN_ERR_UNSUPPORTED;
  if (d->d_ff % 128 != 0 || d->d_ff > 32767) return SFFN_ERR_UNSUPPORTED;
  if (d->max_tokens > kMaxTokensLimit) return SFFN_ERR_UNSUPPORTED;
  if (d->d_model > 4096) return SFFN_ERR_UNSUPPORTED;
  if (d->mode != SFFN_MODE_RELU_THRESHOLD && C != 128) return SFFN_ERR_UNSUPPORTED;
  // the WINA variants of the full-h score, the input side and the
  // orthogonalisation: dense gate, bf16 operands
  if ((d->mode == SFFN_MODE_WINA_FULL_H || d->input_k > 0 || d->V) && (d->rank > 0 || d->dtype != SFFN_BF16))
    return SFFN_ERR_UNSUPPORTED;
  if (d->rank > 0 && (d->dtype != SFFN_BF16 || d->rank % 64 != 0 || d->rank > 4096)) return SFFN_ERR_UNSUPPORTED;
  if (d->dtype == SFFN_FP32 && d->d_ff > 8192) return SFFN_ERR_UNSUPPORTED;
  if ((d->flags & SFFN_FLAG_DEBUG_GATE) && d->rank > 0) return SFFN_ERR_UNSUPPORTED;
  if (d->flags & ~(SFFN_FLAG_DEBUG_GATE | SFFN_FLAG_SEPARATE | SFFN_FLAG_COOPERATIVE | SFFN_FLAG_BACKWARD))
    return SFFN_ERR_INVALID_ARG;
  // the backward: threshold selection, dense gate, bf16, the plain input
  if ((d->flags & SFFN_FLAG_BACKWARD) && (d->mode != SFFN_MODE_RELU_THRESHOLD || d->rank > 0 ||
                                          d->dtype != SFFN_BF16 || d->input_k > 0 || d->V))
    return SFFN_ERR_UNSUPPORTED;
  return SFFN_OK;
}

}  // namespace

extern "C" {

const char* sffn_version(void) { return SFFN_VERSION_STRING; }

const char* sffn_status_string(sffn_status s) {
  switch (s) {
    case SFFN_OK: return "ok";
    case SFFN_ERR_INVALID_ARG: return "invalid argument";
    case SFFN_ERR_UNSUPPORTED: return "unsupported configuration";
    case SFFN_ERR_ALLOC: return "device allocation failed";
    case SFFN_ERR_CUDA: return "CUDA error";
    case SFFN_ERR_TIMEOUT: return "device-side wait timed out";
    case SFFN_ERR_DEVICE: return "device-side range check failed";
    case SFFN_ERR_NO_DEVICE: return "no usable sm_100 device";
  }
  return "unknown status";
}

sffn_status sffn_create(const sffn_desc* desc, void* cuda_stream, sffn_handle** out) {
  if (!out) return SFFN_ERR_INVALID_ARG;
  *out = nullptr;
  sffn_status vs = validate(desc);
  if (vs != SFFN_OK) return vs;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_NO_DEVICE;
  }
  int major = 0, nsm = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return SFFN_ERR_NO_DEVICE;
  if (!get_encode()) return SFFN_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  sffn_handle* h = new (std::nothrow) sffn_handle();
  if (!h) return SFFN_ERR_ALLOC;
  h->desc = *desc;
  h->dev = dev;
  h->n_sm = nsm > 0 ? nsm : kNumSMsFallback;
  h->d = desc->d_model;
  h->F = desc->d_ff;
  h->P = desc->d_ff / 128;
  h->R = desc->rank;
  h->C = desc->tile_capacity;
  h->maxT = desc->max_tokens;
  h->f32 = desc->dtype == SFFN_FP32;
  h->esize = h->f32 ? 4 : 2;
  h->wina = desc->mode == SFFN_MODE_WINA_TOPK || desc->mode == SFFN_MODE_WINA_FULL_H;
  h->fullh = desc->mode == SFFN_MODE_WINA_FULL_H;
  h->Wg = static_cast<const __nv_bfloat16*>(desc->W_gate);
  h->Wu = static_cast<const __nv_bfloat16*>(desc->W_up);
  h->lowrank = desc->rank > 0;
  const size_t T = (size_t)h->maxT, d = (size_t)h->d, F = (size_t)h->F, P = (size_t)h->P, C = (size_t)h->C;
  const size_t R = (size_t)h->R;
  cudaError_t e = cudaSuccess;
  int max_smem = 0;
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const bool dense_gate_bf16 = !h->f32 && !h->wina && !h->lowrank;
  // the low-rank gate's z = bf16(x·A) streams the rank rows of A^T at up to
  // 8 tokens
  const bool lowrank_rows = !h->f32 && !h->wina && h->lowrank && h->R % 128 == 0;

  // ------------------------------------------- kernel attributes and shapes
  if (!h->f32) {
    e = e ? e : set_tc_attrs<EpiGateTwell>();
    e = e ? e : set_gate_persist_attrs(h->C);
    e = e ? e : set_tc_attrs<EpiWina>();
    e = e ? e : set_tc_attrs<EpiLowRankZ>();
    e = e ? e : set_tc_attrs<EpiFallbackH>();
    e = e ? e : set_tc_attrs<EpiTwellH>();
    e = e ? e : set_tc_attrs<EpiDownOut>();
    e = e ? e : set_tc_attrs<EpiWinaFullH>();
    e = e ? e : set_tc_attrs<EpiStoreBf16>();
    // fused up x down: ring slots and list capacity from the shared memory budget
    int lcap = 512, ns = RW_NSMAX;
    auto fits = [&](int l, int n) { return RowsSmem::make(h->P, l, h->d, n).total <= max_smem; };
    while (ns > 2 && !fits(lcap, ns)) --ns;
    while (lcap > 64 && !fits(lcap, ns)) lcap -= 64;
    h->rows_nslot = ns;
    h->rows_lcap = lcap;
    h->rows_smem = RowsSmem::make(h->P, lcap, h->d, ns).total;
    // the x rows and the ring double as the [8][d] fp32 partial-output buffer
    h->rows_ok = h->d % RW_DIV == 0 && h->d <= RW_MAXJ * RW_DIV &&
                 (long long)(ns + 1) * RowsSmem::stage(h->d) >= 32LL * (h->d + 4) &&
                 h->P <= RW_THREADS &&
                 h->rows_smem <= max_smem;
    e = e ? e : cudaFuncSetAttribute(k_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, h->rows_smem);
    if (lowrank_rows) {
      // z = bf16(x·A) streams the d-long rank rows of A^T through two slots
      h->gr_nslot = 2;
      h->gr_smem = GateRowsSmem::make(h->d, 2).total;
      h->gr_ok = h->d % RW_DIV == 0 && h->d <= RW_MAXJ * RW_DIV && h->gr_smem <= max_smem;
      if (h->gr_ok)
        e = e ? e : cudaFuncSetAttribute(k_gate_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, h->gr_smem);
    }
    if (dense_gate_bf16) {
      // row-streaming gate: the same staged-row layout, two ring slots
      const int gns = 2;
      h->gr_nslot = gns;
      h->gr_smem = GateRowsSmem::make(h->d, gns).total;
      h->gr_ok = h->d % RW_DIV == 0 && h->d <= RW_MAXJ * RW_DIV && h->gr_smem <= max_smem;
      if (h->gr_ok)
        e = e ? e : cudaFuncSetAttribute(k_gate_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, h->gr_smem);
      // the single persistent launch: one CTA per SM, all resident at once (a CTA
      // may wait for another's list or zeroed slice of out), lists sized for the
      // most gate groups one CTA takes
      const int G = h->n_sm, NG = (int)(F / RW_G), gmax = cdiv(NG, G);
      h->dec_grid = G;
      h->dec_maxr = gmax * RW_G;
      h->dec_smem = DecodeSmem::make(h->C, h->dec_maxr, h->d).total;
      h->dec_ok = h->gr_ok && h->rows_ok && h->dec_smem <= max_smem && G <= RW_THREADS && F < (1 << 24) &&
                  h->dec_maxr < (1 << 16);
      if (h->dec_ok && !e) {
        e = cudaFuncSetAttribute(k_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, h->dec_smem);
        int nb = 0;
        if (!e) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_decode, RW_THREADS, h->dec_smem);
        h->dec_ok = !e && nb >= 1;
      }
    }
  }
  if (!e && h->wina) {
    const int tk_smem = topk_smem_bytes((int)F, (int)P, (int)C);
    e = cudaFuncSetAttribute(k_wina_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, tk_smem);
  }
  if (!e && desc->input_k > 0)
    e = cudaFuncSetAttribute(k_input_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             input_select_smem_bytes((int)d));
  if (!e && (desc->flags & SFFN_FLAG_BACKWARD)) {
    h->bw_smem = BwdTokenSmem::make((int)d).total;
    e = cudaFuncSetAttribute(k_bwd_token, cudaFuncAttributeMaxDynamicSharedMemorySize, h->bw_smem);
    e = e ? e : set_tc_attrs<EpiStoreGU>();
    e = e ? e : set_tc_attrs<EpiBwdDh>();
    e = e ? e : set_tc_attrs<EpiAddF32>();
    e = e ? e : set_tc_attrs<EpiAddF32Dual>();
  }
  if (!e) e = cudaFuncSetAttribute(k_router, cudaFuncAttributeMaxDynamicSharedMemorySize, router_smem_bytes((int)T));
  if (!e && h->f32) {
    e = cudaFuncSetAttribute(k_rows_f32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)((d + 2 * P * C) * 4));
    e = e ? e : cudaFuncSetAttribute(k_fallback_f32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)((d + F) * 4));
  }
  if (e) {
    cudaGetLastError();
    free_handle(h);
    return SFFN_ERR_CUDA;
  }
  // Every forward of a handle whose token count never exceeds 8 takes the
  // single decode launch (ROWS path, no SFFN_FLAG_SEPARATE), which reads
  // W_down by rows and keeps h in registers: such a handle holds neither the
  // transposed W_down nor the h and overflow-row buffers of the other paths.
  h->dense_bufs = !h->f32 && !(h->dec_ok && h->maxT <= 8 && !(desc->flags & SFFN_FLAG_SEPARATE) &&
                               desc->path != SFFN_PATH_TILES);

  // The tile path's single launch (up to 32 tokens, threshold selection): one
  // CTA per SM, all resident at once; job lists for the grid and for the
  // grid plus one never-launched CTA (the bounded-wait test hook).
  TfSchedule tf_s0, tf_s1;
  if (h->dense_bufs && !h->wina) {
    const TfLayout TL = tf_layout(h->C);
    // (jobs work on pairs of 128-row tiles)
    const int kd = cdiv(d, 64), kg = h->lowrank ? cdiv(R, 64) : kd, Rt = h->lowrank ? cdiv(R, 256) : 0;
    const int P2 = cdiv(P, 2), Md2 = cdiv(d, 256);
    h->tf_grid = h->n_sm;
    h->tf_chunks = h->n_sm;
    h->tf_smem = TL.total;
    tf_s0 = tf_schedule(h->tf_grid, kd, kg, P2, Rt, Md2, (int)(F / 64));
    tf_s1 = tf_schedule(h->tf_grid + 1, kd, kg, P2, Rt, Md2, (int)(F / 64));
    h->tf_ok = tf_s0.ok && tf_s1.ok && TL.stages >= 4 && TL.total <= max_smem;
    if (h->tf_ok) {
      h->tf_max_jobs = (int)std::max(tf_s0.jobs.size(), tf_s1.jobs.size());
      h->tf_max_help = std::max(tf_s0.n_help, tf_s1.n_help);
      h->tf_max_zp = std::max(tf_s0.n_zp, tf_s1.n_zp);
      // flags: z pieces, z parts, helper slots, tile pairs, CTAs (with the hook's extra one)
      h->tf_off_z = h->tf_max_zp;
      h->tf_off_up = h->tf_off_z + Rt * TF_ZPARTS;
      h->tf_off_h = h->tf_off_up + h->tf_max_help;
      h->tf_off_zero = h->tf_off_h + P2;
      h->tf_flag_ints = h->tf_off_zero + h->tf_grid + 1;
      e = cudaFuncSetAttribute(k_tile_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, h->tf_smem);
      int nb = 0;
      if (!e) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_tile_fused, TC_THREADS, h->tf_smem);
      h->tf_ok = !e && nb >= 1;
      if (e) {
        cudaGetLastError();
        e = cudaSuccess;
      }
    }
  }

  // ------------------------------------------ workspace: one allocation
  Arena ar;
  auto plan = [&](Arena& a) {
    a.take(&h->count, T * P * 2);
    a.take(&h->idx, T * P * C * 2);
    a.take(&h->val, T * P * C * h->esize);
    a.take(&h->ovf, T * 4);
    a.take(&h->kmask, T * P * 16);
    a.take(&h->ovf_list, T * 4);
    a.take(&h->ovf_count, 16);
    a.take(&h->status, 16);
    a.take(&h->xstage, T * d * h->esize);
    a.take(&h->ostage, T * d * 4);
    if (h->dense_bufs) {
      a.take(&h->xo, T * d * 2);
      a.take(&h->h_hi, T * F * 2);
      a.take(&h->h_lo, T * F * 2);
      a.take(&h->WdT, d * F * 2);
    }
    if (h->wina) {
      a.take(&h->scores, T * F * 4);
      a.take(&h->vdense, T * F * h->esize);
      a.take(&h->norms, F * 4);
    }
    if (h->fullh) a.take(&h->hfull, T * F * 4);
    if (desc->input_k > 0) {
      a.take(&h->colnorm, d * 4);
      a.take(&h->colacc, d * 8);
      a.take(&h->xsel, T * d * 2);
    }
    if (desc->V) {
      a.take(&h->Vt, d * d * 2);
      a.take(&h->Wg_rot, F * d * 2);
      a.take(&h->Wu_rot, F * d * 2);
      a.take(&h->xrot, T * d * 2);
    }
    if (h->lowrank) {
      a.take(&h->z, T * R * 2);
      a.take(&h->zo, T * R * 2);
      a.take(&h->zpart, (R / 128 + 1) * Z_MAX_SPLITS * (size_t)pick_bn((int)std::min<size_t>(T, 256)) * 128 * 4);
      a.take(&h->tickets, (R / 128 + 1) * 4);
      a.take(&h->At, R * d * 2);
      a.take(&h->Bt, F * R * 2);
    }
    if (desc->flags & SFFN_FLAG_DEBUG_GATE) a.take(&h->gdebug, T * F * 4);
    if (dense_gate_bf16 || lowrank_rows) {
      const size_t tiles = std::max(P, R / 128);   // the gate's tiles, or z's (low rank)
      a.take(&h->gstage, tiles * 8 * 128 * 4);
      a.take(&h->gtick, tiles * 4);
    }
    if (desc->flags & SFFN_FLAG_BACKWARD) {
      const size_t W32 = F / 32, pairs = T * F;
      a.take(&h->bw_wordpre, T * W32 * 4);
      a.take(&h->bw_nnz, T * 4);
      a.take(&h->bw_rowptr, (T + 1) * 4);
      a.take(&h->bw_chunks, (T + pairs / BW_CH + 1) * 8);
      a.take(&h->bw_nchunks, 16);
      a.take(&h->bw_counter, 16);
      a.take(&h->bw_du, pairs * 4);
      a.take(&h->bw_dg, pairs * 4);
      a.take(&h->bw_h, pairs * 4);
      a.take(&h->bw_colcnt, ((T + BW_TCH - 1) / BW_TCH) * F * 4);
      a.take(&h->bw_colptr, (F + 1) * 4);
      a.take(&h->bw_cscpos, pairs * 4);
      a.take(&h->bw_csctok, pairs * 4);
      const size_t NP = (T + 63) / 64 * 64;
      h->bw_NP = (int)NP;
      a.take(&h->bw_heavy, T * 4);
      a.take(&h->bw_hlist, T * 4);
      a.take(&h->bw_nheavy, 16);
      a.take(&h->bw_dbh, F * 4);
      a.take(&h->bw_xh, NP * d * 2);
      a.take(&h->bw_dyh_hi, NP * d * 2);
      a.take(&h->bw_dyh_lo, NP * d * 2);
      a.take(&h->bw_xhT, d * NP * 2);
      a.take(&h->bw_dyhT_hi, d * NP * 2);
      a.take(&h->bw_dyhT_lo, d * NP * 2);
      a.take(&h->bw_g, NP * F * 4);
      a.take(&h->bw_u, NP * F * 4);
      a.take(&h->bw_du_hi, NP * F * 2);
      a.take(&h->bw_du_lo, NP * F * 2);
      a.take(&h->bw_dg_hi, NP * F * 2);
      a.take(&h->bw_dg_lo, NP * F * 2);
      a.take(&h->bw_duT_hi, F * NP * 2);
      a.take(&h->bw_duT_lo, F * NP * 2);
      a.take(&h->bw_dgT_hi, F * NP * 2);
      a.take(&h->bw_dgT_lo, F * NP * 2);
      a.take(&h->bw_hT_hi, F * NP * 2);
      a.take(&h->bw_hT_lo, F * NP * 2);
      a.take(&h->bw_WuT, d * F * 2);
      a.take(&h->bw_WgT, d * F * 2);
    }
    if (h->tf_ok) {
      a.take(&h->tf_jobs, (size_t)h->tf_max_jobs * 16);
      a.take(&h->tf_off, (size_t)(h->tf_grid + 2) * 4);
      a.take(&h->tf_upart, (size_t)h->tf_max_help * TF_TILE_FLOATS * 4);
      a.take(&h->tf_zpart, (size_t)h->tf_max_zp * TF_TILE_FLOATS * 4);
      a.take(&h->tf_flags, (size_t)h->tf_flag_ints * 4);
    }
    if (h->dec_ok) {
      h->dsched_ints = decode_sched_ints((int)P, h->dec_grid + 1);
      a.take(&h->dsched, (size_t)h->dsched_ints * 4);
      a.take(&h->wl_id, (size_t)h->dec_grid * h->dec_maxr * 4);
      a.take(&h->wl_val, (size_t)h->dec_grid * h->dec_maxr * 16);
    }
  };
  plan(ar);                      // sizes
  if (!dalloc(&h->arena, ar.size)) {
    free_handle(h);
    return SFFN_ERR_ALLOC;
  }
  h->arena_bytes = ar.size;
  ar.base = static_cast<uint8_t*>(h->arena);
  ar.size = 0;
  plan(ar);                      // addresses

  e = e ? e : cudaMemsetAsync(h->ovf, 0, T * 4, st);
  e = e ? e : cudaMemsetAsync(h->status, 0, 16, st);
  e = e ? e : cudaMemsetAsync(h->ovf_count, 0, 16, st);
  if (h->gtick) e = e ? e : cudaMemsetAsync(h->gtick, 0, std::max(P, R / 128) * 4, st);
  if (h->lowrank) e = e ? e : cudaMemsetAsync(h->tickets, 0, (R / 128 + 1) * 4, st);
  if (h->dsched) e = e ? e : cudaMemsetAsync(h->dsched, 0, (size_t)h->dsched_ints * 4, st);
  if (h->tf_ok) {
    e = e ? e : cudaMemsetAsync(h->tf_flags, 0, (size_t)h->tf_flag_ints * 4, st);
    e = e ? e : cudaMemcpyAsync(h->tf_jobs, tf_s0.jobs.data(), tf_s0.jobs.size() * 16, cudaMemcpyHostToDevice, st);
    e = e ? e : cudaMemcpyAsync(h->tf_off, tf_s0.off.data(), tf_s0.off.size() * 4, cudaMemcpyHostToDevice, st);
  }
  // create-time derived data
  const dim3 tb(32, 8);
  if (!e && h->WdT) {
    k_transpose_bf16<<<dim3(cdiv(d, 32), cdiv(F, 32)), tb, 0, st>>>(
        static_cast<const __nv_bfloat16*>(desc->W_down), h->WdT, (int)F, (int)d);
    e = cudaGetLastError();
  }
  if (!e && h->lowrank) {
    k_transpose_bf16<<<dim3(cdiv(R, 32), cdiv(d, 32)), tb, 0, st>>>(static_cast<const __nv_bfloat16*>(desc->A),
                                                                    h->At, (int)d, (int)R);
    k_transpose_bf16<<<dim3(cdiv(F, 32), cdiv(R, 32)), tb, 0, st>>>(static_cast<const __nv_bfloat16*>(desc->B),
                                                                    h->Bt, (int)R, (int)F);
    e = cudaGetLastError();
  }
  if (!e && h->wina) {
    if (h->f32)
      k_row_norms<float><<<cdiv(F, 8), 256, 0, st>>>(static_cast<const float*>(desc->W_down), (int)F, (int)d,
                                                      h->norms);
    else
      k_row_norms<__nv_bfloat16><<<cdiv(F, 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(desc->W_down),
                                                             (int)F, (int)d, h->norms);
    e = cudaGetLastError();
  }
  // [WINA] section 3.3: the gate and up weights right-multiplied by V,
  // rounded to bf16 (D[neuron][n] = sum_k W[neuron][k]·V^T[n][k] on the
  // tile kernel); the forwards then use these copies
  if (!e && desc->V) {
    k_transpose_bf16<<<dim3(cdiv(d, 32), cdiv(d, 32)), tb, 0, st>>>(static_cast<const __nv_bfloat16*>(desc->V),
                                                                    h->Vt, (int)d, (int)d);
    e = cudaGetLastError();
    CUtensorMap mW, mV;
    const int BNr = 256;
    if (!e && !make_map(&mV, h->Vt, d, d, BNr)) e = cudaErrorInvalidValue;
    for (int which = 0; which < 2 && !e; ++which) {
      const void* Wsrc = which == 0 ? desc->W_gate : desc->W_up;
      __nv_bfloat16* Wdst = which == 0 ? h->Wg_rot : h->Wu_rot;
      if (!make_map(&mW, Wsrc, d, F, 128)) {
        e = cudaErrorInvalidValue;
        break;
      }
      TcArgs ra{};
      ra.n_phase = 1;
      ra.kb_total[0] = cdiv(d, 64);
      ra.n_rows = (int)d;
      ra.status = h->status;
      StoreParams sp{Wdst, (long long)d, (int)F, (int)d, 0};
      e = launch_tc<EpiStoreBf16>(BNr, dim3(P, cdiv(d, BNr), 1), st, mW, mV, mW, mV, ra, sp);
    }
    h->Wg = h->Wg_rot;
    h->Wu = h->Wu_rot;
  }
  // input-side WINA: column norms of the (orthogonalised) [W_gate; W_up]
  if (!e && desc->input_k > 0) {
    e = cudaMemsetAsync(h->colacc, 0, d * 8, st);
    if (!e) {
      k_col_sumsq<<<dim3(cdiv(d, 256), 64), 256, 0, st>>>(h->Wg, h->Wu, (int)F, (int)d, h->colacc);
      k_col_norms_finish<<<cdiv(d, 256), 256, 0, st>>>(h->colacc, (int)d, h->colnorm);
      e = cudaGetLastError();
    }
  }
  // the backward's dense channel: W_up^T and W_gate^T (the A operands of dx)
  // and the tensor maps of its buffers
  if (!e && h->bw_WuT) {
    k_transpose_bf16<<<dim3(cdiv(d, 32), cdiv(F, 32)), tb, 0, st>>>(h->Wu, h->bw_WuT, (int)F, (int)d);
    k_transpose_bf16<<<dim3(cdiv(d, 32), cdiv(F, 32)), tb, 0, st>>>(h->Wg, h->bw_WgT, (int)F, (int)d);
    e = cudaGetLastError();
    const long long NP = h->bw_NP;
    bool mk = make_map(&h->bm_Wd, desc->W_down, d, F, 128) && make_map(&h->bm_WuT, h->bw_WuT, F, d, 128) &&
              make_map(&h->bm_WgT, h->bw_WgT, F, d, 128) && make_map(&h->bm_duT_hi, h->bw_duT_hi, NP, F, 128) &&
              make_map(&h->bm_duT_lo, h->bw_duT_lo, NP, F, 128) && make_map(&h->bm_dgT_hi, h->bw_dgT_hi, NP, F, 128) &&
              make_map(&h->bm_dgT_lo, h->bw_dgT_lo, NP, F, 128) && make_map(&h->bm_hT_hi, h->bw_hT_hi, NP, F, 128) &&
              make_map(&h->bm_hT_lo, h->bw_hT_lo, NP, F, 128) && make_map(&h->bm_xh, h->bw_xh, d, NP, 256) &&
              make_map(&h->bm_dyh_hi, h->bw_dyh_hi, d, NP, 256) && make_map(&h->bm_dyh_lo, h->bw_dyh_lo, d, NP, 256) &&
              make_map(&h->bm_du_hi, h->bw_du_hi, F, NP, 256) && make_map(&h->bm_du_lo, h->bw_du_lo, F, NP, 256) &&
              make_map(&h->bm_dg_hi, h->bw_dg_hi, F, NP, 256) && make_map(&h->bm_dg_lo, h->bw_dg_lo, F, NP, 256) &&
              make_map(&h->bm_xhT, h->bw_xhT, NP, d, 256) && make_map(&h->bm_dyhT_hi, h->bw_dyhT_hi, NP, d, 256) &&
              make_map(&h->bm_dyhT_lo, h->bw_dyhT_lo, NP, d, 256);
    if (!e && !mk) e = cudaErrorInvalidValue;
  }
  // A-operand tensor maps
  if (!e && !h->f32) {
    bool mok = true;
    if (!h->lowrank) mok = mok && make_map(&h->tmWgate, h->Wg, h->d, h->F, 128);
    mok = mok && make_map(&h->tmWup, h->Wu, h->d, h->F, 128);
    if (h->Vt) mok = mok && make_map(&h->tmVt, h->Vt, h->d, h->d, 128);
    if (h->WdT) mok = mok && make_map(&h->tmWdT, h->WdT, h->F, h->d, 128);
    if (h->tf_ok) {
      mok = mok && make_map(&h->tf_mgate, h->lowrank ? static_cast<const void*>(h->Bt) : h->Wg, h->lowrank ? h->R : h->d,
                            h->F, TF_ROWS);
      mok = mok && make_map(&h->tf_mup, h->Wu, h->d, h->F, TF_ROWS);
      mok = mok && make_map(&h->tf_mdT, h->WdT, h->F, h->d, TF_ROWS);
      if (h->lowrank) mok = mok && make_map(&h->tf_mAt, h->At, h->d, h->R, TF_ROWS);
    }
    if (h->lowrank) {
      mok = mok && make_map(&h->tmAt, h->At, h->d, h->R, 128);
      mok = mok && make_map(&h->tmBt, h->Bt, h->R, h->F, 128);
    }
    if (!mok) {
      cudaStreamSynchronize(st);
      free_handle(h);
      return SFFN_ERR_CUDA;
    }
  }
  if (!e) e = cudaStreamSynchronize(st);
  if (e) {
    cudaGetLastError();
    cudaStreamSynchronize(st);
    free_handle(h);
    return SFFN_ERR_CUDA;
  }
  *out = h;
  return SFFN_OK;
}

sffn_status sffn_destroy(sffn_handle* h) {
  if (!h) return SFFN_OK;
  cudaDeviceSynchronize();
  free_handle(h);
  return SFFN_OK;
}

// The single decode launch's CTAs wait on one another (row lists, zeroed
// slices of out), so all of them must be resident at once: one CTA per SM,
// checked against the occupancy at create time.  With SFFN_FLAG_COOPERATIVE
// it is launched cooperatively, so that when the grid cannot be co-resident
// (an SM-limited MPS client, a green context, SMs held by another persistent
// kernel) the driver holds the launch until the whole grid fits or fails it
// up front, instead of the resident CTAs waiting out their limits.  That
// costs about 4 us per forward (the grid cannot start while the previous
// forward's CTAs hold SMs), so it is not the default.  Programmatic
// dependent launch is requested; if the driver refuses it beside the
// cooperative attribute, the launch is repeated, and later ones made,
// without it.
static cudaError_t launch_decode(sffn_handle* h, const DecodeArgs& da, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->dec_grid);
  cfg.blockDim = dim3(RW_THREADS);
  cfg.dynamicSmemBytes = (size_t)h->dec_smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  const bool coop = (h->desc.flags & SFFN_FLAG_COOPERATIVE) != 0;
  if (coop) {
    at[n].id = cudaLaunchAttributeCooperative;
    at[n].val.cooperative = 1;
    ++n;
  }
  if (h->dec_pdl) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_decode, da);
  if (e == cudaSuccess) {
    h->last_attrs = (coop ? 1u : 0u) | (h->dec_pdl ? 2u : 0u);
    return e;
  }
  cudaGetLastError();
  if (coop && h->dec_pdl && e != cudaErrorCooperativeLaunchTooLarge) {
    h->dec_pdl = false;
    return launch_decode(h, da, st);
  }
  return e;
}

// The tile path's single launch (tile_fused.cuh), launched like the decode
// one: one CTA per SM, cooperative with SFFN_FLAG_COOPERATIVE, programmatic
// dependent launch unless the driver refuses it beside the cooperative
// attribute.
static cudaError_t launch_tile_fused(sffn_handle* h, const TfArgs& ta, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->tf_grid);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = (size_t)h->tf_smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  int n = 0;
  const bool coop = (h->desc.flags & SFFN_FLAG_COOPERATIVE) != 0;
  if (coop) {
    at[n].id = cudaLaunchAttributeCooperative;
    at[n].val.cooperative = 1;
    ++n;
  }
  if (h->tf_pdl) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_tile_fused, ta);
  if (e == cudaSuccess) {
    h->last_attrs = (coop ? 1u : 0u) | (h->tf_pdl ? 2u : 0u);
    return e;
  }
  cudaGetLastError();
  if (coop && h->tf_pdl && e != cudaErrorCooperativeLaunchTooLarge) {
    h->tf_pdl = false;
    return launch_tile_fused(h, ta, st);
  }
  return e;
}

// Uploads the job lists of the fused tile launch for n_chunks runs (the grid,
// or the grid plus the test hook's CTA that never runs).  Synchronous.
static bool tf_upload(sffn_handle* h, int n_chunks) {
  const int kd = cdiv(h->d, 64), kg = h->lowrank ? cdiv(h->R, 64) : kd, Rt = h->lowrank ? cdiv(h->R, 256) : 0;
  const TfSchedule S = tf_schedule(n_chunks, kd, kg, cdiv(h->P, 2), Rt, cdiv(h->d, 256), h->F / 64);
  if (!S.ok || (int)S.jobs.size() > h->tf_max_jobs || S.n_help > h->tf_max_help || S.n_zp > h->tf_max_zp)
    return false;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(h->tf_jobs, S.jobs.data(), S.jobs.size() * 16, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(h->tf_off, S.off.data(), S.off.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  h->tf_chunks = n_chunks;
  return true;
}

static sffn_status forward_bf16(sffn_handle* h, const void* x, int T, float* out, cudaStream_t st) {
  const sffn_desc& D = h->desc;
  const int d = h->d, F = h->F, P = h->P;
  int launches = 0;
  const uint32_t epoch = h->epoch;
  const int BN = pick_bn(T);
  const int ntile_tok = cdiv(T, BN);

  // [WINA] section 3.3: each token's input rotated by the same V as the
  // weights, x' = bf16(x·V), computed as V^T·x^T on the tile kernel and
  // stored transposed
  if (h->Vt) {
    CUtensorMap mx0;
    if (!make_map(&mx0, x, d, T, BN)) return SFFN_ERR_CUDA;
    TcArgs ra{};
    ra.n_phase = 1;
    ra.kb_total[0] = cdiv(d, 64);
    ra.n_rows = T;
    ra.status = h->status;
    StoreParams sp{h->xrot, (long long)d, d, T, 1};
    tmark(h, st, L_ROTATE_X);
    if (launch_tc<EpiStoreBf16>(BN, dim3(cdiv(d, 128), ntile_tok, 1), st, h->tmVt, mx0, h->tmVt, mx0, ra, sp))
      return SFFN_ERR_CUDA;
    ++launches;
    x = h->xrot;
  }
  // [WINA] section 3.1 on the input side: keep the input_k coordinates of
  // largest |x_i|·c_i per token, zero the rest; both projections see the result
  if (h->xsel) {
    InputSelectArgs ia{static_cast<const __nv_bfloat16*>(x), h->colnorm, h->xsel, T, d, D.input_k};
    tmark(h, st, L_INPUT_SELECT);
    if (launch_pdl(k_input_select, dim3(T), dim3(1024), (size_t)input_select_smem_bytes(d), st, 1, ia))
      return SFFN_ERR_CUDA;
    ++launches;
    x = h->xsel;
  }
  int path = D.path;
  if (path == SFFN_PATH_AUTO) path = (h->rows_ok && (T <= 8 || T > 256)) ? SFFN_PATH_ROWS : SFFN_PATH_TILES;
  if (h->wina) path = SFFN_PATH_TILES;  // the top-k kernel writes no per-token keep masks
  if (path == SFFN_PATH_ROWS && !h->rows_ok) return SFFN_ERR_UNSUPPORTED;
  const bool rows = path == SFFN_PATH_ROWS;
  const int nblk = cdiv(T, 8);
  // the row kernel's CTAs per 8-token block: all SMs over one block at
  // decode; at least two for many blocks (prefill at 4096 tokens: 796.8 ->
  // 761.7 us per step with two, 765.3 with three; the shorter CTAs leave a
  // smaller last wave)
  int rows_split = rows ? std::max(nblk > 1 ? 2 : 1, h->n_sm / nblk) : 1;
  // down projection split over d_ff so that its grid covers the SMs.  On the
  // ROWS path it takes the overflow rows only, whose count is on the device:
  // the split assumes two token tiles of them (at 4096 tokens with ~10 %
  // overflow, two tiles of 256, a split of 4 measured 64.7 us, 2 84.3 us and
  // 9 96.2 us)
  const int m_tiles_down = cdiv(d, 128);
  const int est_rows_tiles = rows ? std::min(ntile_tok, 2) : ntile_tok;
  const int kb_down = cdiv(F, 64);
  const int sk_down = std::max(1, std::min(kb_down / 4, h->n_sm / (m_tiles_down * est_rows_tiles)));

  cudaError_t e = cudaSuccess;
  TwellParams tw;
  tw.bias = D.gate_bias;
  tw.tau = h->wina ? 0.f : D.threshold;
  tw.act = D.act;
  tw.T = T;
  tw.F = F;
  tw.n_tiles = P;
  tw.C = h->C;
  tw.count = h->count;
  tw.idx = h->idx;
  tw.val = h->val;
  tw.val_f32 = 0;
  tw.ovf = h->ovf;
  tw.epoch = epoch;
  tw.kmask = rows ? h->kmask : nullptr;
  tw.gdebug = h->gdebug;

  // ---------------------------------------- one persistent launch at T <= 8
  if (rows && T <= 8 && h->dec_ok && !(D.flags & SFFN_FLAG_SEPARATE)) {
    DecodeArgs da{};
    da.x = static_cast<const __nv_bfloat16*>(x);
    da.W_gate = h->Wg;
    da.W_up = h->Wu;
    da.W_down = static_cast<const __nv_bfloat16*>(D.W_down);
    da.tw = tw;
    da.gstage = h->gstage;
    da.sched = h->dsched;
    da.wl_id = h->wl_id;
    da.wl_val = h->wl_val;
    da.maxr = h->dec_maxr;
    da.out = out;
    da.d = d;
    da.status = h->status;
    da.wait_ns = h->dec_wait_ns;
    da.phantom = h->dec_phantom;
    tmark(h, st, L_DECODE);
    if (launch_decode(h, da, st)) return SFFN_ERR_CUDA;
    h->last_path = SFFN_PATH_ROWS;
    h->last_launches = launches + 1;
    h->last_fused = true;
    return SFFN_OK;
  }

  // ----------------------------- tile path: one persistent launch at T <= 32
  // (at 32 tokens, d 4096, d_ff 14336: 77.0 against the separate launches'
  // 94.2 us with the low-rank gate of rank 512, 86.7 against 102.2 us with
  // the dense gate)
  if (!rows && !h->wina && T <= TF_BN && h->tf_ok && !(D.flags & SFFN_FLAG_SEPARATE)) {
    TfArgs ta{};
    bool mok = make_map(&ta.mx, x, d, T, TF_BN) && make_map(&ta.mhi, h->h_hi, F, h->maxT, TF_BN) &&
               make_map(&ta.mlo, h->h_lo, F, h->maxT, TF_BN);
    if (h->lowrank) mok = mok && make_map(&ta.mz, h->z, h->R, h->maxT, TF_BN);
    else ta.mz = ta.mx;  // unused
    if (!mok) return SFFN_ERR_CUDA;
    ta.mgate = h->tf_mgate;
    ta.mAt = h->lowrank ? h->tf_mAt : h->tf_mgate;  // (unused with the dense gate)
    ta.mup = h->tf_mup;
    ta.mdT = h->tf_mdT;
    ta.jobs = h->tf_jobs;
    ta.job_off = h->tf_off;
    ta.tw = tw;
    ta.tw.bias = nullptr;  // the kernel adds it before the emission
    ta.bias = D.gate_bias;
    ta.zpart = h->tf_zpart;
    ta.upart = h->tf_upart;
    ta.z = h->z;
    ta.h_hi = h->h_hi;
    ta.h_lo = h->h_lo;
    ta.f_zp = h->tf_flags;
    ta.f_z = h->tf_flags + h->tf_off_z;
    ta.f_up = h->tf_flags + h->tf_off_up;
    ta.f_h = h->tf_flags + h->tf_off_h;
    ta.f_zero = h->tf_flags + h->tf_off_zero;
    ta.out = out;
    ta.d = d;
    ta.R = h->R;
    ta.maxT = h->maxT;
    ta.kb_gate = h->lowrank ? cdiv(h->R, 64) : cdiv(d, 64);
    ta.lowrank = h->lowrank ? 1 : 0;
    ta.n_chunks = h->tf_chunks;
    if (++h->tf_seq <= 0) {  // sequence numbers are positive: restart, clearing the flags
      if (cudaMemsetAsync(h->tf_flags, 0, (size_t)h->tf_flag_ints * 4, st) != cudaSuccess) return SFFN_ERR_CUDA;
      h->tf_seq = 1;
    }
    ta.seq = h->tf_seq;
    ta.status = h->status;
    ta.wait_ns = h->dec_wait_ns;
    tmark(h, st, L_TILE_FUSED);
    if (launch_tile_fused(h, ta, st)) return SFFN_ERR_CUDA;
    h->last_path = SFFN_PATH_TILES;
    h->last_launches = launches + 1;
    h->last_fused = true;
    return SFFN_OK;
  }

  // the other paths: tensor maps of x and of the workspace rows they use
  if (!h->dense_bufs) return SFFN_ERR_UNSUPPORTED;  // unreachable: such handles always take the single launch
  CUtensorMap mx, mxo, mhi, mlo, mz, mzo;
  bool mok = make_map(&mx, x, d, T, BN) && make_map(&mxo, h->xo, d, h->maxT, BN) &&
             make_map(&mhi, h->h_hi, F, h->maxT, BN) && make_map(&mlo, h->h_lo, F, h->maxT, BN);
  if (h->lowrank)
    mok = mok && make_map(&mz, h->z, h->R, h->maxT, BN) && make_map(&mzo, h->zo, h->R, h->maxT, BN);
  if (!mok) return SFFN_ERR_CUDA;

  // ---------------------------------------------------------------- gate
  const bool lr_rows = h->lowrank && h->gr_ok && T <= 8;
  const CUtensorMap* gateA = &h->tmWgate;
  const CUtensorMap* gateB = &mx;
  int gate_kb = cdiv(d, 64);
  if (lr_rows) {
    // up to 8 tokens: z = bf16(x·A) by streaming the rank rows of A^T
    GateRowsArgs zr{};
    zr.x = static_cast<const __nv_bfloat16*>(x);
    zr.W_gate = h->At;
    zr.tw.T = T;
    zr.tw.F = h->R;
    zr.tw.n_tiles = h->R / 128;
    zr.gstage = h->gstage;
    zr.tick = h->gtick;
    zr.d = d;
    zr.nslot = h->gr_nslot;
    zr.status = h->status;
    zr.zout = h->z;
    tmark(h, st, L_GATE_Z);
    e = launch_pdl(k_gate_rows, dim3(std::min(h->n_sm, h->R / RW_G)), dim3(RW_THREADS), (size_t)h->gr_smem, st, 1,
                   zr);
    ++launches;
    if (e) return SFFN_ERR_CUDA;
    // the gate over B (15 MB at d = 4096, d_ff = 14336, rank 512) stays on
    // the tile kernel: streaming B^T's short rows measured slower (21.8 vs
    // 16.4 us per launch at 8 tokens), the row kernel's fixed cost dominating
    gateA = &h->tmBt;
    gateB = &mz;
    gate_kb = cdiv(h->R, 64);
  } else if (h->lowrank) {
    // z = bf16(x·A): rows are rank coordinates, split over d
    const int mt = cdiv(h->R, 128);
    const int sk = z_splits(d, mt, ntile_tok, h->n_sm);
    TcArgs za{};
    za.n_phase = 1;
    za.kb_total[0] = cdiv(d, 64);
    za.n_rows = T;
    za.status = h->status;
    ZParams zp{T, h->R, sk, h->zpart, h->z, h->tickets};
    tmark(h, st, L_GATE_Z);
    e = launch_tc<EpiLowRankZ>(BN, dim3(mt, ntile_tok, sk), st, h->tmAt, mx, h->tmAt, mx, za, zp);
    ++launches;
    if (e) return SFFN_ERR_CUDA;
    gateA = &h->tmBt;
    gateB = &mz;
    gate_kb = cdiv(h->R, 64);
  }
  TcArgs ga{};
  ga.n_phase = 1;
  ga.kb_total[0] = gate_kb;
  ga.n_rows = T;
  ga.status = h->status;
  ga.stages = h->gate_stages;
  if (!rows || rows_split > 1) {  // later kernels add partial sums into out
    ga.zero_out = reinterpret_cast<float4*>(out);
    ga.zero_n4 = (long long)T * d / 4;
  }
  if (h->wina) {
    tmark(h, st, L_GATE);
    if (h->fullh) {
      // g and u of every neuron in one tile kernel (two accumulators)
      TcArgs fa = ga;
      fa.n_phase = 2;
      fa.kb_total[1] = cdiv(d, 64);
      WinaFullHParams fp{D.gate_bias, D.act, T, F, h->norms, static_cast<__nv_bfloat16*>(h->vdense), h->scores,
                         h->hfull};
      e = launch_tc<EpiWinaFullH>(BN, dim3(P, ntile_tok, 1), st, h->tmWgate, mx, h->tmWup, mx, fa, fp);
    } else {
      WinaParams wp{D.gate_bias, D.act, T, F, h->norms, h->vdense, 0, h->scores};
      e = launch_tc<EpiWina>(BN, dim3(P, ntile_tok, 1), st, *gateA, *gateB, *gateA, *gateB, ga, wp);
    }
    ++launches;
    if (e) return SFFN_ERR_CUDA;
    TopkArgs ta{h->scores, h->vdense, 0, T, F, D.k, P, h->C, h->count, h->idx, h->val, h->ovf, epoch};
    if (h->fullh) {  // the top-k also writes the down projection's masked h rows
      ta.hfull = h->hfull;
      ta.h_hi = h->h_hi;
      ta.h_lo = h->h_lo;
    }
    tmark(h, st, L_WINA_TOPK);
    ++launches;
    if (launch_pdl(k_wina_topk, dim3(T), dim3(1024), (size_t)topk_smem_bytes(F, P, h->C), st, 1, ta))
      return SFFN_ERR_CUDA;
  } else {
    tmark(h, st, L_GATE);
    if (h->gr_ok && T <= 8 && !h->lowrank) {
      // up to 8 tokens: stream whole W_gate rows over every SM
      GateRowsArgs gr{};
      gr.x = static_cast<const __nv_bfloat16*>(x);
      gr.W_gate = h->Wg;
      gr.tw = tw;
      gr.gstage = h->gstage;
      gr.tick = h->gtick;
      gr.zero_out = ga.zero_out;
      gr.zero_n4 = ga.zero_n4;
      gr.d = d;
      gr.nslot = h->gr_nslot;
      gr.status = h->status;
      e = launch_pdl(k_gate_rows, dim3(std::min(h->n_sm, F / RW_G)), dim3(RW_THREADS), (size_t)h->gr_smem, st, 1,
                     gr);
    } else if (P * ntile_tok > h->n_sm && !(D.flags & SFFN_FLAG_SEPARATE)) {
      // at least a tile per SM: the persistent gate overlaps each tile's
      // TwELL emission with the next tile's MMAs
      e = launch_gate_persist(BN, h->n_sm, P * ntile_tok, st, *gateA, *gateB, ga, tw);
    } else {
      e = launch_tc<EpiGateTwell>(BN, dim3(P, ntile_tok, 1), st, *gateA, *gateB, *gateA, *gateB, ga, tw);
    }
    ++launches;
    if (e) return SFFN_ERR_CUDA;
  }

  // ------------------------------------------ non-overflow tokens
  if (rows) {
    RowsArgs rw{};
    rw.x = static_cast<const __nv_bfloat16*>(x);
    rw.W_up = h->Wu;
    rw.W_down = static_cast<const __nv_bfloat16*>(D.W_down);
    rw.count = h->count;
    rw.idx = h->idx;
    rw.val = static_cast<const __nv_bfloat16*>(h->val);
    rw.kmask = reinterpret_cast<const uint4*>(h->kmask);
    rw.ovf = h->ovf;
    rw.epoch = epoch;
    rw.ovf_list = h->ovf_list;
    rw.ovf_count = h->ovf_count;
    rw.xo = reinterpret_cast<uint4*>(h->xo);
    rw.z = h->lowrank ? reinterpret_cast<const uint4*>(h->z) : nullptr;
    rw.zo = reinterpret_cast<uint4*>(h->zo);
    rw.r_vec = h->R / 8;
    rw.zero_ovf_rows = rows_split == 1 && sk_down > 1 ? 1 : 0;
    rw.out = out;
    rw.T = T;
    rw.d = d;
    rw.F = F;
    rw.n_tiles = P;
    rw.C = h->C;
    rw.atomic = rows_split > 1 ? 1 : 0;
    rw.nslot = h->rows_nslot;
    rw.lcap = h->rows_lcap;
    rw.status = h->status;
    tmark(h, st, L_UPDOWN_ROWS);
    ++launches;
    if (launch_pdl(k_rows, dim3(rows_split, nblk, 1), dim3(RW_THREADS), (size_t)h->rows_smem, st, 1, rw))
      return SFFN_ERR_CUDA;
  } else if (!h->fullh) {  // (full-h: the top-k kernel wrote h)
    TcArgs ua{};
    ua.n_phase = 1;
    ua.kb_total[0] = cdiv(d, 64);
    ua.n_rows = T;
    ua.status = h->status;
    TwellHParams hp{T, F, P, h->C, h->count, h->idx, static_cast<const __nv_bfloat16*>(h->val), h->ovf, epoch,
                    h->h_hi, h->h_lo, RouteParams{}};
    // the first tile's CTA routes the overflow tokens for the dense channel
    hp.route.ovf_list = h->ovf_list;
    hp.route.ovf_count = h->ovf_count;
    hp.route.x = static_cast<const uint4*>(x);
    hp.route.xo = reinterpret_cast<uint4*>(h->xo);
    hp.route.d_vec = d / 8;
    hp.route.z = h->lowrank ? reinterpret_cast<const uint4*>(h->z) : nullptr;
    hp.route.zo = reinterpret_cast<uint4*>(h->zo);
    hp.route.r_vec = h->R / 8;
    tmark(h, st, L_TILE_H);
    e = launch_tc<EpiTwellH>(BN, dim3(P, ntile_tok, 1), st, h->tmWup, mx, h->tmWup, mx, ua, hp);
    ++launches;
    if (e) return SFFN_ERR_CUDA;
  }

  // ------------------------------------- dense channel for overflow tokens
  if (!h->wina) {
    TcArgs fa{};
    fa.n_phase = 2;
    fa.kb_total[0] = h->lowrank ? cdiv(h->R, 64) : cdiv(d, 64);
    fa.kb_total[1] = cdiv(d, 64);
    fa.n_rows = T;
    fa.n_rows_dev = h->ovf_count;
    fa.status = h->status;
    HParams hp{};
    hp.bias = D.gate_bias;
    hp.tau = D.threshold;
    hp.act = D.act;
    hp.F = F;
    hp.n_rows_dev = h->ovf_count;
    hp.n_rows = T;
    hp.row_map = rows ? nullptr : h->ovf_list;
    hp.h_hi = h->h_hi;
    hp.h_lo = h->h_lo;
    const CUtensorMap& a0 = h->lowrank ? h->tmBt : h->tmWgate;
    const CUtensorMap& b0 = h->lowrank ? mzo : mxo;
    tmark(h, st, L_FALLBACK_H);
    e = launch_tc<EpiFallbackH>(BN, dim3(P, ntile_tok, 1), st, a0, b0, h->tmWup, mxo, fa, hp);
    ++launches;
    if (e) return SFFN_ERR_CUDA;
  }

  // ----------------------------------------------------- down projection
  {
    TcArgs da{};
    da.n_phase = 1;  // each stage multiplies one W_down^T tile by h_hi and h_lo
    da.kb_total[0] = kb_down;
    da.stages = h->down_stages;
    da.n_rows = T;
    da.n_rows_dev = rows ? h->ovf_count : nullptr;
    da.status = h->status;
    OutParams op{};
    op.out = out;
    op.d = d;
    op.n_rows_dev = rows ? h->ovf_count : nullptr;
    op.n_rows = T;
    op.row_map = rows ? h->ovf_list : nullptr;
    op.atomic = sk_down > 1 ? 1 : 0;
    tmark(h, st, L_DOWN);
    e = launch_tc<EpiDownOut>(BN, dim3(m_tiles_down, ntile_tok, sk_down), st, h->tmWdT, mhi, h->tmWdT, mlo, da,
                              op);
    ++launches;
    if (e) return SFFN_ERR_CUDA;
  }
  h->last_path = path;
  h->last_launches = launches;
  return SFFN_OK;
}

static sffn_status forward_f32(sffn_handle* h, const void* x, int T, float* out, cudaStream_t st) {
  const sffn_desc& D = h->desc;
  const int d = h->d, F = h->F, P = h->P;
  const uint32_t epoch = h->epoch;
  int launches = 0;
  GateF32Args ga{};
  ga.x = static_cast<const float*>(x);
  ga.W_gate = static_cast<const float*>(D.W_gate);
  ga.d = d;
  ga.wina = h->wina ? 1 : 0;
  ga.tw.bias = D.gate_bias;
  ga.tw.tau = D.threshold;
  ga.tw.act = D.act;
  ga.tw.T = T;
  ga.tw.F = F;
  ga.tw.n_tiles = P;
  ga.tw.C = h->C;
  ga.tw.count = h->count;
  ga.tw.idx = h->idx;
  ga.tw.val = h->val;
  ga.tw.val_f32 = 1;
  ga.tw.ovf = h->ovf;
  ga.tw.epoch = epoch;
  ga.tw.kmask = nullptr;
  ga.tw.gdebug = h->gdebug;
  ga.wp = WinaParams{D.gate_bias, D.act, T, F, h->norms, h->vdense, 1, h->scores};
  tmark(h, st, L_GATE_F32);
  ++launches;
  if (launch_pdl(k_gate_f32, dim3(P, cdiv(T, 16)), dim3(128), 0, st, 1, ga)) return SFFN_ERR_CUDA;
  if (h->wina) {
    TopkArgs ta{h->scores, h->vdense, 1, T, F, D.k, P, h->C, h->count, h->idx, h->val, h->ovf, epoch};
    tmark(h, st, L_WINA_TOPK);
    ++launches;
    if (launch_pdl(k_wina_topk, dim3(T), dim3(1024), (size_t)topk_smem_bytes(F, P, h->C), st, 1, ta))
      return SFFN_ERR_CUDA;
  }
  RouterArgs ra{};
  ra.T = T;
  ra.ovf = h->ovf;
  ra.epoch = epoch;
  ra.ovf_list = h->ovf_list;
  ra.ovf_count = h->ovf_count;
  ra.zero_all = 0;
  tmark(h, st, L_ROUTER);
  ++launches;
  if (launch_pdl(k_router, dim3(1), dim3(1024), (size_t)router_smem_bytes(T), st, 1, ra)) return SFFN_ERR_CUDA;
  RowsF32Args rf{static_cast<const float*>(x), static_cast<const float*>(D.W_up), static_cast<const float*>(D.W_down),
                 h->count, h->idx, static_cast<const float*>(h->val), h->ovf, epoch, out, T, d, P, h->C};
  tmark(h, st, L_ROWS_F32);
  ++launches;
  if (launch_pdl(k_rows_f32, dim3(T), dim3(256), (size_t)(d + 2 * P * h->C) * 4, st, 1, rf)) return SFFN_ERR_CUDA;
  if (!h->wina) {
    FallbackF32Args fa{static_cast<const float*>(x), static_cast<const float*>(D.W_gate),
                       static_cast<const float*>(D.W_up), static_cast<const float*>(D.W_down), D.gate_bias,
                       D.threshold, D.act, h->ovf_list, h->ovf_count, out, d, F};
    tmark(h, st, L_FALLBACK_F32);
    ++launches;
    if (launch_pdl(k_fallback_f32, dim3(T), dim3(256), (size_t)(d + F) * 4, st, 1, fa)) return SFFN_ERR_CUDA;
  }
  h->last_path = SFFN_PATH_ROWS;
  h->last_launches = launches;
  return SFFN_OK;
}

sffn_status sffn_forward(sffn_handle* h, const void* x, int T, float* out, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (T < 0 || T > h->maxT) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  ++h->epoch;
  if (h->epoch == 0) ++h->epoch;  // 0 marks "never overflowed"
  // the single-launch schedule's words carry the low 16 bits of the epoch:
  // cleared at the start of every window of 65536 epochs, no word left by an
  // earlier launch carries the current tag
  if (h->dsched && ((h->epoch & 0xFFFFu) == 0u || h->epoch == 1u)) {
    if (cudaMemsetAsync(h->dsched, 0, (size_t)h->dsched_ints * 4, st) != cudaSuccess) return SFFN_ERR_CUDA;
  }
  h->last_T = T;
  h->last_epoch = h->epoch;
  h->last_fused = false;
  tmark_begin(h);
  const sffn_status r = h->f32 ? forward_f32(h, x, T, out, st) : forward_bf16(h, x, T, out, st);
  tmark_end(h, st);
  return r;
}

static sffn_status timing_begin_impl(KTiming* h, int max_forwards, int stride) {
  if (!h || max_forwards <= 0 || max_forwards > 100000 || stride <= 0) return SFFN_ERR_INVALID_ARG;
  timing_free(h);
  h->tm_stride = stride;
  h->tm_seen = 0;
  const size_t nev = (size_t)max_forwards * (kMaxMarks + 1);
  h->tm_ev.assign(nev, nullptr);
  for (size_t i = 0; i < nev; ++i) {
    if (cudaEventCreate(&h->tm_ev[i]) != cudaSuccess) {
      cudaGetLastError();
      timing_free(h);
      return SFFN_ERR_CUDA;
    }
  }
  h->tm_lab.assign((size_t)max_forwards * kMaxMarks, 0);
  h->tm_nk.assign(max_forwards, 0);
  h->tm_max = max_forwards;
  h->tm_n = 0;
  h->tm_on = true;
  return SFFN_OK;
}

static sffn_status timing_end_impl(KTiming* h, int max_kernels, char (*names)[32], float* total_ms,
                                   int* launches, int* n_kernels) {
  if (!h || !h->tm_on) return SFFN_ERR_INVALID_ARG;
  double acc[L_COUNT] = {0};
  int cnt[L_COUNT] = {0};
  sffn_status rs = SFFN_OK;
  for (int f = 0; f < h->tm_n && rs == SFFN_OK; ++f) {
    const int nk = h->tm_nk[f];
    cudaEvent_t* ev = &h->tm_ev[(size_t)f * (kMaxMarks + 1)];
    if (cudaEventSynchronize(ev[nk]) != cudaSuccess) {
      rs = SFFN_ERR_CUDA;
      break;
    }
    for (int i = 0; i < nk; ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) {
        rs = SFFN_ERR_CUDA;
        break;
      }
      const int lab = h->tm_lab[(size_t)f * kMaxMarks + i];
      acc[lab] += ms;
      cnt[lab] += 1;
    }
  }
  int n = 0;
  for (int l = 0; l < L_COUNT; ++l) {
    if (!cnt[l]) continue;
    if (n < max_kernels) {
      if (names) {
        std::strncpy(names[n], kLabelNames[l], 31);
        names[n][31] = 0;
      }
      if (total_ms) total_ms[n] = (float)acc[l];
      if (launches) launches[n] = cnt[l];
    }
    ++n;
  }
  if (n_kernels) *n_kernels = n;
  timing_free(h);
  cudaGetLastError();
  return rs;
}

sffn_status sffn_timing_begin(sffn_handle* h, int max_forwards, int stride) {
  return timing_begin_impl(h, max_forwards, stride);
}

sffn_status sffn_timing_end(sffn_handle* h, int max_kernels, char (*names)[32], float* total_ms, int* launches,
                            int* n_kernels) {
  return timing_end_impl(h, max_kernels, names, total_ms, launches, n_kernels);
}

sffn_status sffn_forward_host(sffn_handle* h, const void* x_host, int T, float* out_host, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (T < 0 || T > h->maxT) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  if (!x_host || !out_host) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const size_t xb = (size_t)T * h->d * h->esize, ob = (size_t)T * h->d * 4;
  if (cudaMemcpyAsync(h->xstage, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess) return SFFN_ERR_CUDA;
  sffn_status s = sffn_forward(h, h->xstage, T, h->ostage, cuda_stream);
  if (s != SFFN_OK) return s;
  if (cudaMemcpyAsync(out_host, h->ostage, ob, cudaMemcpyDeviceToHost, st) != cudaSuccess) return SFFN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SFFN_ERR_CUDA;
  return SFFN_OK;
}

sffn_status sffn_read_status(sffn_handle* h, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint32_t w = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SFFN_ERR_CUDA;
  if (cudaMemcpy(&w, h->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return SFFN_ERR_CUDA;
  if (w) {
    cudaMemset(h->status, 0, 4);
    // a CTA that gave up may have left scheduler words of the single-launch
    // decode kernel set: start the next forward from zero
    if (h->dsched) cudaMemset(h->dsched, 0, (size_t)h->dsched_ints * 4);
  }
  if (w & DEV_ERR_TIMEOUT) return SFFN_ERR_TIMEOUT;
  if (w & DEV_ERR_RANGE) return SFFN_ERR_DEVICE;
  return SFFN_OK;
}

sffn_status sffn_debug_twell(sffn_handle* h, const int16_t** count, const int16_t** idx, const void** val,
                             const uint32_t** overflow, int* n_tiles, int* tile_capacity) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (count) *count = h->count;
  if (idx) *idx = h->idx;
  if (val) *val = h->val;
  if (overflow) *overflow = h->ovf;
  if (n_tiles) *n_tiles = h->P;
  if (tile_capacity) *tile_capacity = h->C;
  return SFFN_OK;
}

sffn_status sffn_debug_set_epoch(sffn_handle* h, unsigned epoch) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (h->dsched && cudaMemset(h->dsched, 0, (size_t)h->dsched_ints * 4) != cudaSuccess) return SFFN_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SFFN_ERR_CUDA;
  h->epoch = epoch;
  return SFFN_OK;
}

sffn_status sffn_debug_decode_waits(sffn_handle* h, int phantom_ctas, unsigned wait_us) {
  if (!h || phantom_ctas < 0 || phantom_ctas > 1) return SFFN_ERR_INVALID_ARG;
  if (h->tf_ok && h->tf_chunks != h->tf_grid + phantom_ctas && !tf_upload(h, h->tf_grid + phantom_ctas))
    return SFFN_ERR_CUDA;
  h->dec_phantom = phantom_ctas;
  h->dec_wait_ns = wait_us ? (unsigned long long)wait_us * 1000ull : SFFN_WAIT_LIMIT_NS;
  return SFFN_OK;
}

sffn_status sffn_debug_tile_schedule(int d_model, int d_ff, int rank, int n_cta, int* jobs, int max_jobs,
                                     int* off, int* n_jobs) {
  if (d_model <= 0 || d_model > 4096 || d_model % 8 || d_ff <= 0 || d_ff % 128 || d_ff > 32767 || rank < 0 ||
      rank % 64 || rank > 4096 || n_cta <= 0 || n_cta > 4096 || !n_jobs)
    return SFFN_ERR_INVALID_ARG;
  const int kd = cdiv(d_model, 64), kg = rank ? rank / 64 : kd, Rt = rank ? cdiv(rank, 256) : 0;
  const TfSchedule S = tf_schedule(n_cta, kd, kg, cdiv(d_ff / 128, 2), Rt, cdiv(d_model, 256), d_ff / 64);
  if (!S.ok) return SFFN_ERR_UNSUPPORTED;
  *n_jobs = (int)S.jobs.size();
  if (!jobs || !off || max_jobs < (int)S.jobs.size()) return SFFN_ERR_INVALID_ARG;
  std::memcpy(jobs, S.jobs.data(), S.jobs.size() * sizeof(int4));
  std::memcpy(off, S.off.data(), S.off.size() * sizeof(int));
  return SFFN_OK;
}

sffn_status sffn_debug_keep(sffn_handle* h, const uint32_t** keep) {
  if (!h || !keep) return SFFN_ERR_INVALID_ARG;
  *keep = h->kmask;
  return SFFN_OK;
}

sffn_status sffn_debug_gate(sffn_handle* h, const float** g) {
  if (!h || !g) return SFFN_ERR_INVALID_ARG;
  if (!h->gdebug) return SFFN_ERR_UNSUPPORTED;
  *g = h->gdebug;
  return SFFN_OK;
}

sffn_status sffn_workspace_bytes(const sffn_handle* h, size_t* bytes) {
  if (!h || !bytes) return SFFN_ERR_INVALID_ARG;
  *bytes = h->arena_bytes;
  return SFFN_OK;
}

sffn_status sffn_debug_norms(sffn_handle* h, const float** norms) {
  if (!h || !norms) return SFFN_ERR_INVALID_ARG;
  if (!h->norms) return SFFN_ERR_UNSUPPORTED;
  *norms = h->norms;
  return SFFN_OK;
}

sffn_status sffn_get_stats(sffn_handle* h, void* cuda_stream, sffn_stats* st) {
  if (!h || !st) return SFFN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int n = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SFFN_ERR_CUDA;
  if (h->last_fused) {
    // the single launch routes implicitly (an overflow token's kept rows are
    // in the row lists); its record of the routing is the per-token flags
    std::vector<uint32_t> f(std::max(h->last_T, 1));
    if (cudaMemcpy(f.data(), h->ovf, (size_t)h->last_T * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return SFFN_ERR_CUDA;
    for (int t = 0; t < h->last_T; ++t) n += f[t] == h->last_epoch;
  } else if (cudaMemcpy(&n, h->ovf_count, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    return SFFN_ERR_CUDA;
  }
  st->n_overflow = n;
  st->n_launches = h->last_launches;
  st->path = h->last_path;
  st->epoch = h->epoch;
  st->launch_attrs = h->last_fused ? h->last_attrs : 0u;
  return SFFN_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free low-rank gate -> TwELL.
//
// Some callers cannot allocate device memory at the point where they run the
// gate: code embedded in a runtime that owns all device memory (a serving
// engine with a pre-planned pool, a plugin host that hands out fixed buffers)
// and code on a latency-critical path, where cudaMalloc may synchronise the
// device or fail when memory is reserved or fragmented.  For them this entry
// point computes z = bf16(x·A) and the TwELL records of sigma(z·B + b) with
// the same kernels as sffn_forward, but keeps its scratch (the split-K fp32
// partials of z, its per-tile tickets, z itself and a status word) in
// file-scope device arrays of fixed size that every GPU loading this library
// holds until the process exits.  It calls no allocator: inputs and outputs
// come from the caller.
namespace {

constexpr int kNaMaxT = 64, kNaMaxD = 4096, kNaMaxR = 1024, kNaMaxF = 16384;
constexpr int kNaTickets = kNaMaxR / 128;
// Scratch held per GPU: the fp32 split partials of z, (1024/128 row tiles) x
// 4 splits x 64 tokens x 128 rows x 4 B = 1 MiB; z itself, 64 x 1024 x 2 B =
// 128 KiB; the tickets and the status word: 1,179,696 bytes in all (~1.2 MB).

static __device__ __align__(256) float g_na_zpart[(kNaMaxR / 128) * Z_MAX_SPLITS * kNaMaxT * 128];
static __device__ __align__(256) __nv_bfloat16 g_na_z[kNaMaxT * kNaMaxR];
static __device__ __align__(256) int g_na_tickets[kNaTickets];
static __device__ __align__(256) uint32_t g_na_status[4];

struct NaScratch {
  float* zpart = nullptr;
  __nv_bfloat16* z = nullptr;
  int* tickets = nullptr;
  uint32_t* status = nullptr;
  bool ready = false;
};
constexpr int kNaMaxDevices = 64;
NaScratch g_na_dev[kNaMaxDevices];
std::mutex g_na_mu;
// test hook (sffn_debug_noalloc_waits): hold time of the calls' kernels, ns
std::atomic<unsigned long long> g_na_hold_ns{0};

// Device addresses of the scratch arrays for the current device (looked up
// once per device; the host-side names of the arrays are not device addresses).
sffn_status na_setup(int dev, NaScratch** out) {
  if (dev < 0 || dev >= kNaMaxDevices) return SFFN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_na_mu);
  NaScratch& s = g_na_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_na_zpart) != cudaSuccess) goto fail;
    s.zpart = static_cast<float*>(p);
    if (cudaGetSymbolAddress(&p, g_na_z) != cudaSuccess) goto fail;
    s.z = static_cast<__nv_bfloat16*>(p);
    if (cudaGetSymbolAddress(&p, g_na_tickets) != cudaSuccess) goto fail;
    s.tickets = static_cast<int*>(p);
    if (cudaGetSymbolAddress(&p, g_na_status) != cudaSuccess) goto fail;
    s.status = static_cast<uint32_t*>(p);
    if (set_tc_attrs<EpiLowRankZ>() != cudaSuccess || set_tc_attrs<EpiGateTwell>() != cudaSuccess) goto fail;
    s.ready = true;
  }
  *out = &s;
  return SFFN_OK;
fail:
  cudaGetLastError();
  return SFFN_ERR_CUDA;
}

}  // namespace

extern "C" sffn_status sffn_lowrank_twell_noalloc(const void* x, int T, int d_model, const void* A_t, int rank,
                                                  const void* B_t, int d_ff, const float* gate_bias, int act,
                                                  float threshold, int tile_capacity, int16_t* count, int16_t* idx,
                                                  void* val, uint32_t* overflow, void* cuda_stream) {
  if (!x || !A_t || !B_t || !count || !idx || !val || !overflow) return SFFN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(A_t) || !aligned16(B_t)) return SFFN_ERR_INVALID_ARG;
  if (gate_bias && (reinterpret_cast<uintptr_t>(gate_bias) & 3u)) return SFFN_ERR_INVALID_ARG;
  if (act != SFFN_ACT_RELU && act != SFFN_ACT_SILU) return SFFN_ERR_INVALID_ARG;
  if (!(threshold >= 0.0f) || !std::isfinite(threshold)) return SFFN_ERR_INVALID_ARG;
  const int C = tile_capacity;
  if (C != 8 && C != 16 && C != 32 && C != 64 && C != 128) return SFFN_ERR_INVALID_ARG;
  if (T < 0 || d_model <= 0 || rank <= 0 || d_ff <= 0) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  // the scratch arrays bound the problem size
  if (T > kNaMaxT || d_model > kNaMaxD || rank > kNaMaxR || d_ff > kNaMaxF) return SFFN_ERR_UNSUPPORTED;
  if (d_model % 8 != 0 || rank % 64 != 0 || d_ff % 128 != 0) return SFFN_ERR_UNSUPPORTED;
  int dev = 0, major = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_NO_DEVICE;
  }
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return SFFN_ERR_NO_DEVICE;
  NaScratch* sc = nullptr;
  sffn_status ss = na_setup(dev, &sc);
  if (ss != SFFN_OK) return ss;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const int P = d_ff / 128, BN = pick_bn(T), ntile = cdiv(T, BN), mt = cdiv(rank, 128);
  const int sk = z_splits(d_model, mt, ntile, nsm > 0 ? nsm : kNumSMsFallback);
  // the split tickets and the caller's overflow flags start at zero
  cudaError_t e = cudaMemsetAsync(sc->tickets, 0, sizeof(int) * kNaTickets, st);
  e = e ? e : cudaMemsetAsync(overflow, 0, (size_t)T * sizeof(uint32_t), st);
  if (e) {
    cudaGetLastError();
    return SFFN_ERR_CUDA;
  }
  CUtensorMap mAt, mx, mBt, mz;
  if (!make_map(&mAt, A_t, d_model, rank, 128) || !make_map(&mx, x, d_model, T, BN) ||
      !make_map(&mBt, B_t, rank, d_ff, 128) || !make_map(&mz, sc->z, rank, T, BN))
    return SFFN_ERR_CUDA;
  const unsigned long long hold = g_na_hold_ns.load();
  TcArgs za{};
  za.n_phase = 1;
  za.kb_total[0] = cdiv(d_model, 64);
  za.n_rows = T;
  za.status = sc->status;
  za.hold_ns = hold;
  ZParams zp{T, rank, sk, sc->zpart, sc->z, sc->tickets};
  if (launch_tc<EpiLowRankZ>(BN, dim3(mt, ntile, sk), st, mAt, mx, mAt, mx, za, zp) != cudaSuccess)
    return SFFN_ERR_CUDA;
  TcArgs ga{};
  ga.n_phase = 1;
  ga.kb_total[0] = cdiv(rank, 64);
  ga.n_rows = T;
  ga.status = sc->status;
  ga.hold_ns = hold;
  TwellParams tw;
  tw.bias = gate_bias;
  tw.tau = threshold;
  tw.act = act;
  tw.T = T;
  tw.F = d_ff;
  tw.n_tiles = P;
  tw.C = C;
  tw.count = count;
  tw.idx = idx;
  tw.val = val;
  tw.val_f32 = 0;
  tw.ovf = overflow;
  tw.epoch = 1;
  tw.kmask = nullptr;
  tw.gdebug = nullptr;
  if (launch_tc<EpiGateTwell>(BN, dim3(P, ntile, 1), st, mBt, mz, mBt, mz, ga, tw) != cudaSuccess)
    return SFFN_ERR_CUDA;
  return SFFN_OK;
}

extern "C" sffn_status sffn_lowrank_twell_noalloc_status(void* cuda_stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_NO_DEVICE;
  }
  NaScratch* sc = nullptr;
  sffn_status ss = na_setup(dev, &sc);
  if (ss != SFFN_OK) return ss;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  uint32_t w = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemcpy(&w, sc->status, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_CUDA;
  }
  if (w && cudaMemset(sc->status, 0, sizeof(w)) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_CUDA;
  }
  if (w & DEV_ERR_TIMEOUT) return SFFN_ERR_TIMEOUT;
  if (w & DEV_ERR_RANGE) return SFFN_ERR_DEVICE;
  return SFFN_OK;
}

extern "C" sffn_status sffn_debug_noalloc_waits(unsigned wait_us) {
  g_na_hold_ns.store((unsigned long long)wait_us * 1000ull);
  return SFFN_OK;
}

// ---------------------------------------------------------------------------
// Gated subspace linear layer ("Gated Subspace Inference for Transformer
// Acceleration", sections 2.1 and 2.2): y = M·bf16(V_k^T x) for tokens whose
// residual ratio ||x - V_k V_k^T x|| / ||x|| is below eps, y = W x for the
// others, with M = bf16(W V_k) made at create time.
struct sffn_gsi_handle : KTiming {
  sffn_gsi_desc desc;
  int dev = 0, n_sm = kNumSMsFallback;
  void* arena = nullptr;
  size_t arena_bytes = 0;
  __nv_bfloat16* Vkt = nullptr;   // [k][d_in]
  __nv_bfloat16* M = nullptr;     // [d_out][k]
  float* g[2] = {nullptr, nullptr};   // [maxT][k], alternate forwards (one is cleared for the next)
  float* part = nullptr;          // [grid_resid][maxT][2]
  int* n_slow = nullptr;          // [4]
  uint32_t* status = nullptr;     // [4]
  int smem_proj = 0, smem_resid = 0, smem_out = 0;
  int grid_proj = 0, grid_resid = 0, grid_out = 0;
  int parity = 0;
  int last_T = 0;
};

namespace {

sffn_status gsi_validate(const sffn_gsi_desc* d) {
  if (!d || !d->W || !d->Vk) return SFFN_ERR_INVALID_ARG;
  if (d->d_in <= 0 || d->d_out <= 0 || d->k <= 0 || d->max_tokens <= 0) return SFFN_ERR_INVALID_ARG;
  if (!(d->eps >= 0.0f) || std::isnan(d->eps)) return SFFN_ERR_INVALID_ARG;
  if (!aligned16(d->W) || !aligned16(d->Vk)) return SFFN_ERR_INVALID_ARG;
  if (d->k > d->d_in) return SFFN_ERR_INVALID_ARG;
  if (d->d_in % 8 || d->k % 8 || d->d_in > 8192 || d->k > 512 || d->max_tokens > 64) return SFFN_ERR_UNSUPPORTED;
  return SFFN_OK;
}

void gsi_free(sffn_gsi_handle* h) {
  if (!h) return;
  timing_free(h);
  if (h->arena) cudaFree(h->arena);
  delete h;
}

}  // namespace

extern "C" sffn_status sffn_gsi_create(const sffn_gsi_desc* desc, void* cuda_stream, sffn_gsi_handle** out) {
  if (!out) return SFFN_ERR_INVALID_ARG;
  *out = nullptr;
  sffn_status vs = gsi_validate(desc);
  if (vs != SFFN_OK) return vs;
  int dev = 0, major = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_NO_DEVICE;
  }
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10) return SFFN_ERR_NO_DEVICE;
  if (!get_encode()) return SFFN_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  sffn_gsi_handle* h = new (std::nothrow) sffn_gsi_handle();
  if (!h) return SFFN_ERR_ALLOC;
  h->desc = *desc;
  h->dev = dev;
  h->n_sm = nsm > 0 ? nsm : kNumSMsFallback;
  const size_t di = desc->d_in, dout = desc->d_out, k = desc->k, T = desc->max_tokens;
  Arena ar;
  h->grid_proj = cdiv(di, GSI_PROJ_ROWS);
  h->grid_resid = cdiv(di, GSI_RESID_ROWS);
  h->grid_out = h->n_sm;
  auto plan = [&](Arena& a) {
    a.take(&h->Vkt, k * di * 2);
    a.take(&h->M, dout * k * 2);
    a.take(&h->g[0], T * k * 4);
    a.take(&h->g[1], T * k * 4);
    a.take(&h->part, (size_t)h->grid_resid * T * 2 * 4);
    a.take(&h->n_slow, 16);
    a.take(&h->status, 16);
  };
  plan(ar);
  if (!dalloc(&h->arena, ar.size)) {
    gsi_free(h);
    return SFFN_ERR_ALLOC;
  }
  h->arena_bytes = ar.size;
  ar.base = static_cast<uint8_t*>(h->arena);
  ar.size = 0;
  plan(ar);
  h->smem_proj = (GSI_THREADS / ((int)k / 2)) * GSI_TC * (int)k * 4;
  h->smem_resid = GSI_TC * (int)k * 4;
  h->smem_out = GsiOutSmem::make((int)T, (int)k, (int)di).total;
  cudaError_t e = cudaMemsetAsync(h->status, 0, 16, st);
  e = e ? e : cudaMemsetAsync(h->n_slow, 0, 16, st);
  e = e ? e : cudaMemsetAsync(h->g[0], 0, T * k * 4, st);
  e = e ? e : cudaMemsetAsync(h->g[1], 0, T * k * 4, st);
  e = e ? e : cudaFuncSetAttribute(k_gsi_project, cudaFuncAttributeMaxDynamicSharedMemorySize, h->smem_proj);
  e = e ? e : cudaFuncSetAttribute(k_gsi_resid, cudaFuncAttributeMaxDynamicSharedMemorySize, h->smem_resid);
  e = e ? e : cudaFuncSetAttribute(k_gsi_out, cudaFuncAttributeMaxDynamicSharedMemorySize, h->smem_out);
  e = e ? e : set_tc_attrs<EpiStoreBf16>();
  // V_k^T, then the cached image M = bf16(W V_k): D[o][j] = sum_i W[o][i] V_k^T[j][i]
  if (!e) {
    k_transpose_bf16<<<dim3(cdiv(k, 32), cdiv(di, 32)), dim3(32, 8), 0, st>>>(
        static_cast<const __nv_bfloat16*>(desc->Vk), h->Vkt, (int)di, (int)k);
    e = cudaGetLastError();
  }
  if (!e) {
    CUtensorMap mW, mV;
    const int BNr = 256;
    if (!make_map(&mW, desc->W, (long long)di, (long long)dout, 128) ||
        !make_map(&mV, h->Vkt, (long long)di, (long long)k, BNr)) {
      e = cudaErrorInvalidValue;
    } else {
      TcArgs ra{};
      ra.n_phase = 1;
      ra.kb_total[0] = cdiv(di, 64);
      ra.n_rows = (int)k;
      ra.status = h->status;
      StoreParams sp{h->M, (long long)k, (int)dout, (int)k, 0};
      e = launch_tc<EpiStoreBf16>(BNr, dim3(cdiv(dout, 128), cdiv(k, BNr), 1), st, mW, mV, mW, mV, ra, sp);
    }
  }
  if (!e) e = cudaStreamSynchronize(st);
  if (e) {
    cudaGetLastError();
    cudaStreamSynchronize(st);
    gsi_free(h);
    return SFFN_ERR_CUDA;
  }
  *out = h;
  return SFFN_OK;
}

extern "C" sffn_status sffn_gsi_forward(sffn_gsi_handle* h, const void* x, int T, float* y, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (T < 0 || T > h->desc.max_tokens) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  if (!x || !y || !aligned16(x) || !aligned16(y)) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  GsiArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.Vk = static_cast<const __nv_bfloat16*>(h->desc.Vk);
  a.M = h->M;
  a.W = static_cast<const __nv_bfloat16*>(h->desc.W);
  a.g = h->g[h->parity];
  a.g_next = h->g[h->parity ^ 1];
  a.part = h->part;
  a.n_slow = h->n_slow;
  a.y = y;
  a.T = T;
  a.d_in = h->desc.d_in;
  a.d_out = h->desc.d_out;
  a.k = h->desc.k;
  a.maxT = h->desc.max_tokens;
  a.grid_resid = h->grid_resid;
  a.eps2 = h->desc.eps * h->desc.eps;
  h->last_T = T;
  tmark_begin(h);
  tmark(h, st, L_GSI_PROJECT);
  if (launch_pdl(k_gsi_project, dim3(h->grid_proj), dim3(GSI_THREADS), (size_t)h->smem_proj, st, 1, a))
    return SFFN_ERR_CUDA;
  tmark(h, st, L_GSI_RESID);
  if (launch_pdl(k_gsi_resid, dim3(h->grid_resid), dim3(GSI_THREADS), (size_t)h->smem_resid, st, 1, a))
    return SFFN_ERR_CUDA;
  tmark(h, st, L_GSI_OUT);
  if (launch_pdl(k_gsi_out, dim3(h->grid_out), dim3(GSI_OUT_THREADS), (size_t)h->smem_out, st, 1, a))
    return SFFN_ERR_CUDA;
  tmark_end(h, st);
  h->parity ^= 1;   // the launches went out: the next forward sums into the other buffer
  return SFFN_OK;
}

extern "C" sffn_status sffn_gsi_destroy(sffn_gsi_handle* h) {
  if (!h) return SFFN_OK;
  cudaDeviceSynchronize();
  gsi_free(h);
  return SFFN_OK;
}

extern "C" sffn_status sffn_gsi_stats(sffn_gsi_handle* h, void* cuda_stream, int* n_slow) {
  if (!h || !n_slow) return SFFN_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess ||
      cudaMemcpy(n_slow, h->n_slow, 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_CUDA;
  }
  return SFFN_OK;
}

extern "C" sffn_status sffn_gsi_debug(sffn_gsi_handle* h, const float** g, const float** part, int* n_part,
                                      const void** M) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (g) *g = h->g[h->parity ^ 1];   // the last forward's buffer
  if (part) *part = h->part;
  if (n_part) *n_part = h->grid_resid;
  if (M) *M = h->M;
  return SFFN_OK;
}

extern "C" sffn_status sffn_gsi_timing_begin(sffn_gsi_handle* h, int max_forwards, int stride) {
  return timing_begin_impl(h, max_forwards, stride);
}

extern "C" sffn_status sffn_gsi_timing_end(sffn_gsi_handle* h, int max_kernels, char (*names)[32], float* total_ms,
                                           int* launches, int* n_kernels) {
  return timing_end_impl(h, max_kernels, names, total_ms, launches, n_kernels);
}

// ---------------------------------------------------------------------------
// Mixture of LoPA-gated sparse experts (see moe.cuh): a router launch, every
// expert's own sparse forward on its block of T rows (x where the token is
// routed to it, zero elsewhere), a combine launch.
struct sffn_moe_handle : KTiming {
  int E = 0, top_k = 0, d = 0, F = 0, maxT = 0;
  const void* Wr = nullptr;
  std::vector<sffn_handle*> experts;
  void* arena = nullptr;
  __nv_bfloat16* xe = nullptr;    // [E][maxT][d]
  float* ye = nullptr;            // [E][maxT][d]
  int* sel = nullptr;             // [maxT][top_k]
  float* w = nullptr;             // [maxT][top_k]
  float* logits = nullptr;        // [maxT][E]
  int last_T = 0;
  // the experts' forwards run side by side: expert e on stream e % kMoeStreams,
  // forked after the router and joined before the combine
  std::vector<cudaStream_t> es;
  cudaEvent_t ev_fork = nullptr;
  std::vector<cudaEvent_t> ev_join;
};

namespace {
constexpr int kMoeStreams = 8;
void moe_free(sffn_moe_handle* h) {
  if (!h) return;
  for (sffn_handle* e : h->experts) sffn_destroy(e);
  for (cudaStream_t s : h->es)
    if (s) cudaStreamDestroy(s);
  for (cudaEvent_t ev : h->ev_join)
    if (ev) cudaEventDestroy(ev);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  timing_free(h);
  if (h->arena) cudaFree(h->arena);
  delete h;
}
}  // namespace

extern "C" sffn_status sffn_moe_create(const sffn_moe_desc* md, void* cuda_stream, sffn_moe_handle** out) {
  if (!out) return SFFN_ERR_INVALID_ARG;
  *out = nullptr;
  if (!md || !md->W_router || !md->A || !md->B || !md->W_up || !md->W_down) return SFFN_ERR_INVALID_ARG;
  if (md->n_experts < 1 || md->top_k < 1 || md->top_k > md->n_experts) return SFFN_ERR_INVALID_ARG;
  if (md->n_experts > MOE_MAX_E || md->top_k > MOE_MAX_K) return SFFN_ERR_UNSUPPORTED;
  if (md->rank <= 0 || md->d_model <= 0 || md->max_tokens <= 0) return SFFN_ERR_INVALID_ARG;
  if (!aligned16(md->W_router)) return SFFN_ERR_INVALID_ARG;
  if (md->d_model % 8 || md->max_tokens > 1024) return SFFN_ERR_UNSUPPORTED;
  // unrouted rows are zero: they must keep nothing, so the gate bias is <= 0
  for (int e = 0; e < md->n_experts; ++e) {
    sffn_desc d{};
    d.d_model = md->d_model;
    d.d_ff = md->d_ff;
    d.max_tokens = md->max_tokens;
    d.rank = md->rank;
    d.dtype = SFFN_BF16;
    d.mode = SFFN_MODE_RELU_THRESHOLD;
    d.act = SFFN_ACT_RELU;
    d.threshold = md->threshold;
    d.tile_capacity = md->tile_capacity;
    d.A = md->A[e];
    d.B = md->B[e];
    d.W_up = md->W_up[e];
    d.W_down = md->W_down[e];
    d.gate_bias = md->gate_bias ? md->gate_bias[e] : nullptr;
    const sffn_status vs = validate(&d);
    if (vs != SFFN_OK) return vs;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SFFN_ERR_NO_DEVICE;
  }
  int major = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return SFFN_ERR_NO_DEVICE;
  sffn_moe_handle* h = new (std::nothrow) sffn_moe_handle();
  if (!h) return SFFN_ERR_ALLOC;
  h->E = md->n_experts;
  h->top_k = md->top_k;
  h->d = md->d_model;
  h->F = md->d_ff;
  h->maxT = md->max_tokens;
  h->Wr = md->W_router;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (md->gate_bias) {   // a positive bias would keep neurons of the zero rows: checked on the host copy
    std::vector<float> b((size_t)md->d_ff);
    for (int e = 0; e < md->n_experts; ++e) {
      if (!md->gate_bias[e]) continue;
      if (cudaMemcpy(b.data(), md->gate_bias[e], b.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        moe_free(h);
        return SFFN_ERR_CUDA;
      }
      for (float v : b)
        if (!(v <= 0.0f)) {
          moe_free(h);
          return SFFN_ERR_UNSUPPORTED;
        }
    }
  }
  for (int e = 0; e < h->E; ++e) {
    sffn_desc d{};
    d.d_model = md->d_model;
    d.d_ff = md->d_ff;
    d.max_tokens = md->max_tokens;
    d.rank = md->rank;
    d.dtype = SFFN_BF16;
    d.mode = SFFN_MODE_RELU_THRESHOLD;
    d.act = SFFN_ACT_RELU;
    d.threshold = md->threshold;
    d.tile_capacity = md->tile_capacity;
    d.A = md->A[e];
    d.B = md->B[e];
    d.W_up = md->W_up[e];
    d.W_down = md->W_down[e];
    d.gate_bias = md->gate_bias ? md->gate_bias[e] : nullptr;
    sffn_handle* eh = nullptr;
    const sffn_status cs = sffn_create(&d, cuda_stream, &eh);
    if (cs != SFFN_OK) {
      moe_free(h);
      return cs;
    }
    h->experts.push_back(eh);
  }
  {
    const int ns = std::min(h->E, kMoeStreams);
    bool ok = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < ns && ok; ++i) {
      cudaStream_t s = nullptr;
      cudaEvent_t ev = nullptr;
      ok = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess;
      if (ok) h->es.push_back(s);
      ok = ok && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess;
      if (ok) h->ev_join.push_back(ev);
    }
    if (!ok) {
      cudaGetLastError();
      moe_free(h);
      return SFFN_ERR_CUDA;
    }
  }
  const size_t E = h->E, T = h->maxT, dd = h->d, K = h->top_k;
  Arena ar;
  auto plan = [&](Arena& a) {
    a.take(&h->xe, E * T * dd * 2);
    a.take(&h->ye, E * T * dd * 4);
    a.take(&h->sel, T * K * 4);
    a.take(&h->w, T * K * 4);
    a.take(&h->logits, T * E * 4);
  };
  plan(ar);
  if (!dalloc(&h->arena, ar.size)) {
    moe_free(h);
    return SFFN_ERR_ALLOC;
  }
  ar.base = static_cast<uint8_t*>(h->arena);
  ar.size = 0;
  plan(ar);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    moe_free(h);
    return SFFN_ERR_CUDA;
  }
  *out = h;
  return SFFN_OK;
}

extern "C" sffn_status sffn_moe_forward(sffn_moe_handle* h, const void* x, int T, float* out, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (T < 0 || T > h->maxT) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  if (!x || !out || !aligned16(x) || !aligned16(out)) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  h->last_T = T;
  tmark_begin(h);
  MoeRouteArgs ra{static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(h->Wr), h->xe,
                  h->sel, h->w, h->logits, T, h->d, h->E, h->top_k};
  tmark(h, st, L_MOE_ROUTE);
  if (launch_pdl(k_moe_route, dim3(T), dim3(256), 0, st, 1, ra)) return SFFN_ERR_CUDA;
  tmark_end(h, st);
  // the experts side by side: each stream waits for the router, the
  // combine waits for every stream
  const int ns = (int)h->es.size();
  if (cudaEventRecord(h->ev_fork, st) != cudaSuccess) return SFFN_ERR_CUDA;
  for (int i = 0; i < ns; ++i)
    if (cudaStreamWaitEvent(h->es[i], h->ev_fork, 0) != cudaSuccess) return SFFN_ERR_CUDA;
  sffn_status res = SFFN_OK;
  for (int e = 0; e < h->E && res == SFFN_OK; ++e)
    res = sffn_forward(h->experts[e], h->xe + (size_t)e * T * h->d, T, h->ye + (size_t)e * T * h->d,
                       h->es[e % ns]);
  // joined even after a failed expert, so that the experts already queued
  // stay ordered before the caller's later work on its stream
  for (int i = 0; i < ns; ++i)
    if ((cudaEventRecord(h->ev_join[i], h->es[i]) != cudaSuccess ||
         cudaStreamWaitEvent(st, h->ev_join[i], 0) != cudaSuccess) && res == SFFN_OK)
      res = SFFN_ERR_CUDA;
  if (res != SFFN_OK) return res;
  tmark_follow(h);
  MoeCombineArgs ca{h->ye, h->sel, h->w, out, T, h->d, h->top_k};
  tmark(h, st, L_MOE_COMBINE);
  if (launch_pdl(k_moe_combine, dim3(std::max(1, cdiv(h->d / 4, 256)), T), dim3(256), 0, st, 1, ca))
    return SFFN_ERR_CUDA;
  tmark_end(h, st);
  return SFFN_OK;
}

extern "C" sffn_status sffn_moe_destroy(sffn_moe_handle* h) {
  if (!h) return SFFN_OK;
  cudaDeviceSynchronize();
  moe_free(h);
  return SFFN_OK;
}

extern "C" sffn_status sffn_moe_expert(sffn_moe_handle* h, int e, sffn_handle** expert) {
  if (!h || !expert || e < 0 || e >= h->E) return SFFN_ERR_INVALID_ARG;
  *expert = h->experts[e];
  return SFFN_OK;
}

extern "C" sffn_status sffn_moe_debug(sffn_moe_handle* h, const int** sel, const float** w, const float** logits) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (sel) *sel = h->sel;
  if (w) *w = h->w;
  if (logits) *logits = h->logits;
  return SFFN_OK;
}

extern "C" sffn_status sffn_moe_read_status(sffn_moe_handle* h, void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  sffn_status worst = SFFN_OK;
  for (sffn_handle* e : h->experts) {
    const sffn_status s = sffn_read_status(e, cuda_stream);
    if (s != SFFN_OK && worst == SFFN_OK) worst = s;
  }
  return worst;
}

extern "C" sffn_status sffn_moe_timing_begin(sffn_moe_handle* h, int max_forwards, int stride) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  sffn_status s = timing_begin_impl(h, 2 * max_forwards, stride);
  for (size_t e = 0; e < h->experts.size() && s == SFFN_OK; ++e) s = timing_begin_impl(h->experts[e], max_forwards, stride);
  return s;
}

extern "C" sffn_status sffn_moe_timing_end(sffn_moe_handle* h, int max_kernels, char (*names)[32], float* total_ms,
                                           int* launches, int* n_kernels) {
  // the router and combine launches, then every expert's kernels, added by label
  if (!h) return SFFN_ERR_INVALID_ARG;
  std::vector<std::vector<char>> nm;
  std::vector<float> ms;
  std::vector<int> ln;
  auto collect = [&](KTiming* t) -> sffn_status {
    char tn[L_COUNT][32];
    float tm[L_COUNT];
    int tl[L_COUNT], n = 0;
    const sffn_status s = timing_end_impl(t, L_COUNT, tn, tm, tl, &n);
    if (s != SFFN_OK) return s;
    for (int i = 0; i < std::min(n, (int)L_COUNT); ++i) {
      size_t j = 0;
      while (j < nm.size() && std::strcmp(nm[j].data(), tn[i]) != 0) ++j;
      if (j == nm.size()) {
        nm.emplace_back(tn[i], tn[i] + 32);
        ms.push_back(0.f);
        ln.push_back(0);
      }
      ms[j] += tm[i];
      ln[j] += tl[i];
    }
    return SFFN_OK;
  };
  sffn_status s = collect(h);
  for (size_t e = 0; e < h->experts.size() && s == SFFN_OK; ++e) s = collect(h->experts[e]);
  const int n = (int)nm.size();
  for (int i = 0; i < std::min(n, max_kernels); ++i) {
    if (names) std::memcpy(names[i], nm[i].data(), 32);
    if (total_ms) total_ms[i] = ms[i];
    if (launches) launches[i] = ln[i];
  }
  if (n_kernels) *n_kernels = n;
  return s;
}

// ---------------------------------------------------------------------------
// Backward of the last forward (see backward.cuh).
extern "C" sffn_status sffn_backward(sffn_handle* h, const void* x, const float* dy, int T, float* dx,
                                     float* dW_gate, float* dW_up, float* dW_down, float* d_bias,
                                     void* cuda_stream) {
  if (!h) return SFFN_ERR_INVALID_ARG;
  if (!(h->desc.flags & SFFN_FLAG_BACKWARD)) return SFFN_ERR_UNSUPPORTED;
  if (T < 0 || T > h->maxT) return SFFN_ERR_INVALID_ARG;
  if (T == 0) return SFFN_OK;
  if (!x || !dy || !dx || !dW_gate || !dW_up || !dW_down) return SFFN_ERR_INVALID_ARG;
  const void* ptrs[] = {x, dy, dx, dW_gate, dW_up, dW_down};
  for (const void* p : ptrs)
    if (!aligned16(p)) return SFFN_ERR_INVALID_ARG;
  if (d_bias && (reinterpret_cast<uintptr_t>(d_bias) & 3u)) return SFFN_ERR_INVALID_ARG;
  // the keep masks of the last forward: it must have been a ROWS-path forward of these T tokens
  if (h->last_T != T || h->last_path != SFFN_PATH_ROWS) return SFFN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  BwdArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.dy = dy;
  a.W_gate = h->Wg;
  a.W_up = h->Wu;
  a.W_down = static_cast<const __nv_bfloat16*>(h->desc.W_down);
  a.bias = h->desc.gate_bias;
  a.kmask = h->kmask;
  a.T = T;
  a.d = h->d;
  a.F = h->F;
  a.n_words = h->F / 32;
  a.act = h->desc.act;
  a.wordpre = h->bw_wordpre;
  a.nnz = h->bw_nnz;
  a.rowptr = h->bw_rowptr;
  a.chunks = h->bw_chunks;
  a.n_chunks = h->bw_nchunks;
  a.counter = h->bw_counter;
  a.du = h->bw_du;
  a.dg = h->bw_dg;
  a.hv = h->bw_h;
  a.colcnt = h->bw_colcnt;
  a.colptr = h->bw_colptr;
  a.cscpos = h->bw_cscpos;
  a.csctok = h->bw_csctok;
  a.dx = dx;
  a.dW_gate = dW_gate;
  a.dW_up = dW_up;
  a.dW_down = dW_down;
  a.db = d_bias;
  a.ovf = h->ovf;
  a.epoch = h->last_epoch;
  a.heavy = h->bw_heavy;
  a.hlist = h->bw_hlist;
  a.n_heavy = h->bw_nheavy;
  a.dbh = d_bias ? h->bw_dbh : nullptr;
  const int NP = h->bw_NP, d = h->d, F = h->F, P = h->P;
  tmark_follow(h);
  tmark(h, st, L_BWD_INDEX);
  if (launch_pdl(k_bwd_rows, dim3(T), dim3(BW_THREADS), 0, st, 1, a)) return SFFN_ERR_CUDA;
  if (launch_pdl(k_bwd_scan, dim3(1), dim3(1024), 0, st, 1, a)) return SFFN_ERR_CUDA;
  tmark(h, st, L_BWD_TOKEN);
  if (launch_pdl(k_bwd_token, dim3(2 * h->n_sm), dim3(BW_THREADS), (size_t)h->bw_smem, st, 1, a))
    return SFFN_ERR_CUDA;
  // dense channel of the heavy tokens ([TwELL] hybrid routing): their x and
  // dy rows gathered (and transposed), g and u over every neuron, dh with the
  // pair values, dx = du W_up + dg W_gate on the tensor cores
  {
    tmark(h, st, L_BWD_DENSE);
    HeavyPrepArgs pa{a.x, dy, h->bw_hlist, h->bw_nheavy, h->bw_xh, h->bw_dyh_hi, h->bw_dyh_lo, h->bw_xhT,
                     h->bw_dyhT_hi, h->bw_dyhT_lo, h->bw_dbh, d, F, NP};
    if (launch_pdl(k_bwd_heavy_prep, dim3(cdiv(d, 32), NP / 32), dim3(32, 8), 0, st, 1, pa)) return SFFN_ERR_CUDA;
    const int BN = 256, ntok = cdiv(NP, BN);
    TcArgs ga{};
    ga.n_phase = 2;
    ga.kb_total[0] = ga.kb_total[1] = cdiv(d, 64);
    ga.n_rows = T;
    ga.n_rows_dev = h->bw_nheavy;
    ga.status = h->status;
    GuParams gp{h->bw_g, h->bw_u, h->bw_nheavy, F};
    if (launch_tc<EpiStoreGU>(BN, dim3(P, ntok, 1), st, h->tmWgate, h->bm_xh, h->tmWup, h->bm_xh, ga, gp))
      return SFFN_ERR_CUDA;
    TcArgs da{};
    da.n_phase = 1;
    da.kb_total[0] = cdiv(d, 64);
    da.n_rows = T;
    da.n_rows_dev = h->bw_nheavy;
    da.status = h->status;
    BwdDhParams dp{h->bw_g, h->bw_u, h->desc.gate_bias, h->kmask, F / 32, h->bw_hlist, h->bw_nheavy, F, NP,
                   h->desc.act, h->bw_du_hi, h->bw_du_lo, h->bw_dg_hi, h->bw_dg_lo, h->bw_duT_hi, h->bw_duT_lo,
                   h->bw_dgT_hi, h->bw_dgT_lo, h->bw_hT_hi, h->bw_hT_lo, h->bw_dbh};
    if (launch_tc<EpiBwdDh>(BN, dim3(P, ntok, 1), st, h->bm_Wd, h->bm_dyh_hi, h->bm_Wd, h->bm_dyh_lo, da, dp))
      return SFFN_ERR_CUDA;
    // dx rows of the heavy tokens: W_up^T (du hi + lo), then W_gate^T (dg hi + lo) added
    TcArgs xa{};
    xa.n_phase = 1;
    xa.kb_total[0] = cdiv(F, 64);
    xa.n_rows = T;
    xa.n_rows_dev = h->bw_nheavy;
    xa.status = h->status;
    OutParams op{dx, d, h->bw_nheavy, T, h->bw_hlist, 0};
    if (launch_tc<EpiDownOut>(BN, dim3(cdiv(d, 128), ntok, 1), st, h->bm_WuT, h->bm_du_hi, h->bm_WuT, h->bm_du_lo,
                              xa, op))
      return SFFN_ERR_CUDA;
    op.atomic = 1;
    if (launch_tc<EpiDownOut>(BN, dim3(cdiv(d, 128), ntok, 1), st, h->bm_WgT, h->bm_dg_hi, h->bm_WgT, h->bm_dg_lo,
                              xa, op))
      return SFFN_ERR_CUDA;
  }
  tmark(h, st, L_BWD_INDEX);
  const dim3 gcol(cdiv(h->F, 256), cdiv(T, BW_TCH));
  if (launch_pdl(k_bwd_colcount, gcol, dim3(256), 0, st, 1, a)) return SFFN_ERR_CUDA;
  if (launch_pdl(k_bwd_colprefix, dim3(cdiv(h->F, 256)), dim3(256), 0, st, 1, a)) return SFFN_ERR_CUDA;
  if (launch_pdl(k_bwd_scan2, dim3(1), dim3(1024), 0, st, 1, a)) return SFFN_ERR_CUDA;
  if (launch_pdl(k_bwd_colfill, gcol, dim3(256), 0, st, 1, a)) return SFFN_ERR_CUDA;
  tmark(h, st, L_BWD_NEURON);
  // one 16-byte piece per thread up to d = 2048 (fewer registers, more CTAs per SM), two up to 4096
  const cudaError_t en = h->d <= 8 * BW_THREADS
                             ? launch_pdl(k_bwd_neuron<1>, dim3(h->F), dim3(BW_THREADS), 0, st, 1, a)
                             : launch_pdl(k_bwd_neuron<2>, dim3(h->F), dim3(BW_THREADS), 0, st, 1, a);
  if (en) return SFFN_ERR_CUDA;
  // the heavy tokens' dW rows, added: K = the heavy tokens (device count),
  // A = the neuron-major pair values (hi, then lo), B = x^T or dy^T (hi + lo)
  {
    tmark(h, st, L_BWD_DENSE);
    const int BN = 256;
    TcArgs wa{};
    wa.n_phase = 2;
    wa.acc_same = 1;
    wa.kb_dev = h->bw_nheavy;
    wa.n_rows = d;
    wa.status = h->status;
    const dim3 gw(P, cdiv(d, BN), 1);
    AddParams ap{dW_up, (long long)d, F, d};
    if (launch_tc<EpiAddF32>(BN, gw, st, h->bm_duT_hi, h->bm_xhT, h->bm_duT_lo, h->bm_xhT, wa, ap))
      return SFFN_ERR_CUDA;
    ap.dst = dW_gate;
    if (launch_tc<EpiAddF32>(BN, gw, st, h->bm_dgT_hi, h->bm_xhT, h->bm_dgT_lo, h->bm_xhT, wa, ap))
      return SFFN_ERR_CUDA;
    ap.dst = dW_down;
    if (launch_tc<EpiAddF32Dual>(BN, gw, st, h->bm_hT_hi, h->bm_dyhT_hi, h->bm_hT_lo, h->bm_dyhT_lo, wa, ap))
      return SFFN_ERR_CUDA;
  }
  tmark_end(h, st);
  return SFFN_OK;
}
