// Epilogues of the tensor-core tile kernel.  In every one of them the 128
// epilogue threads hold one accumulator row each (a neuron, a low-rank
// coordinate or an output column) and 16 consecutive columns (tokens) at a
// time, read from TMEM with tcgen05.ld.
#pragma once

#include "ptx.cuh"

namespace sffn {

enum : int { ACT_RELU = 0, ACT_SILU = 1 };

__device__ __forceinline__ float act_fn(float g, int act) {
  return act == ACT_RELU ? fmaxf(g, 0.0f) : g / (1.0f + expf(-g));
}

// ------------------------------------------------------------------ TwELL
// TwELL emission for one chunk of 16 tokens, shared by the tensor-core gate
// and the fp32 SIMT gate.  Called by 128 threads (4 full warps); thread etid
// owns neuron j of tile p = j / 128 (j % 128 == etid) and holds g (pre-bias)
// for tokens t0..t0+15.  Kept neurons are compacted per token with warp
// ballots: the rank of neuron j among the kept neurons of its tile is the
// popcount of the kept bits of lower lanes in lower warps and in its own warp,
// which is its slot (ascending neuron order).
struct TwellParams {
  const float* bias;  // [F] or null
  float tau;
  int act;
  int T, F, n_tiles, C;
  int16_t* count;     // [T][n_tiles]
  int16_t* idx;       // [T][n_tiles][C]
  void* val;          // [T][n_tiles][C] bf16 or fp32
  int val_f32;
  uint32_t* ovf;      // [T]: = epoch iff the token overflows in this forward
  uint32_t epoch;
  uint32_t* kmask;    // [T][n_tiles][4] kept bits of every (token, tile), or null
  float* gdebug;      // [T][F] dense gate (debug), or null
};

__device__ __forceinline__ void twell_chunk(const TwellParams& o, const float* g, int j, int t0, int etid,
                                            uint32_t* masks /*[4][16]*/) {
  const int w = etid >> 5, lane = etid & 31;
  const int p = j >> 7;
  const float b = o.bias ? o.bias[j] : 0.0f;
  float a[16];
  uint32_t keep = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float gv = g[i] + b;
    a[i] = act_fn(gv, o.act);
    const bool in = (t0 + i) < o.T;
    const bool k = in && fabsf(a[i]) > o.tau;
    keep |= (k ? 1u : 0u) << i;
    if (o.gdebug && in) o.gdebug[(size_t)(t0 + i) * o.F + j] = gv;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, k);
    if (lane == 0) masks[w * 16 + i] = bal;
  }
  named_bar_sync(1, 128);
  if (o.kmask && etid < 64) {
    const int i = etid & 15, ww = etid >> 4;
    if (t0 + i < o.T) o.kmask[((size_t)(t0 + i) * o.n_tiles + p) * 4 + ww] = masks[ww * 16 + i];
  }
  const uint32_t lt = lanemask_lt();
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int t = t0 + i;
    if (t >= o.T) break;
    const uint32_t m0 = masks[i], m1 = masks[16 + i], m2 = masks[32 + i], m3 = masks[48 + i];
    const int c0 = __popc(m0), c1 = __popc(m1), c2 = __popc(m2), c3 = __popc(m3);
    const int total = c0 + c1 + c2 + c3;
    const uint32_t mw = w == 0 ? m0 : w == 1 ? m1 : w == 2 ? m2 : m3;
    const int pre = (w > 0 ? c0 : 0) + (w > 1 ? c1 : 0) + (w > 2 ? c2 : 0) + __popc(mw & lt);
    const size_t base = ((size_t)t * o.n_tiles + p) * o.C;
    if (((keep >> i) & 1u) && pre < o.C) {
      o.idx[base + pre] = (int16_t)j;
      if (o.val_f32)
        reinterpret_cast<float*>(o.val)[base + pre] = a[i];
      else
        reinterpret_cast<__nv_bfloat16*>(o.val)[base + pre] = __float2bfloat16_rn(a[i]);
    }
    if (etid >= total && etid < o.C) {
      o.idx[base + etid] = -1;
      if (o.val_f32)
        reinterpret_cast<float*>(o.val)[base + etid] = 0.0f;
      else
        reinterpret_cast<__nv_bfloat16*>(o.val)[base + etid] = __float2bfloat16_rn(0.0f);
    }
    if (etid == 0) {
      o.count[(size_t)t * o.n_tiles + p] = (int16_t)total;
      if (total > o.C) o.ovf[t] = o.epoch;
    }
  }
}

// TwELL emission for one 128-neuron tile and up to NT (8 or 32) tokens
// t0..t0+NT-1 (bf16 values), by the 128 threads of four full warps.  It is the same format as
// twell_chunk, but its phases keep every thread busy and write whole records:
//   1. thread = neuron: activation, keep bit, bf16 value into a staging
//      block; warp ballots give each token's 128-bit keep mask;
//   2. four threads per token, one per 32-bit mask word: each ranks its kept
//      neurons after the lower words' counts.  The first C ranks go to the
//      token's staged record (ascending neuron order); pads fill slots at or
//      after the count.  Count, overflow epoch and keep mask are written
//      here;
//   3. the staged [NT][C] idx and val records go out as 16-byte vectors.
// (Thread-per-neuron stores of 2-byte slots kept one warp per scheduler
// waiting on dependent latencies and flooded L2 with partial writes.)
constexpr int TW32_VP = 128 + 8;   // padded staged-value row (bf16 elements)
__host__ __device__ constexpr int twell_smem(int NT, int C) { return NT * 4 * 4 + NT * TW32_VP * 2 + NT * C * 2 * 2; }
__host__ __device__ constexpr int twell32_smem(int C) { return twell_smem(32, C); }

template <int NT = 32>
__device__ __forceinline__ void twell_tile32(const TwellParams& o, const float* g, int j, int t0, int etid,
                                             uint8_t* scratch, uint32_t bar_id) {
  const int w = etid >> 5, lane = etid & 31;
  const int p = j >> 7, n_in = j & 127;
  const int C = o.C;
  uint32_t* masks = reinterpret_cast<uint32_t*>(scratch);                         // [NT tokens][4]
  uint16_t* vals = reinterpret_cast<uint16_t*>(scratch + NT * 4 * 4);             // [NT][TW32_VP]
  uint16_t* sidx = reinterpret_cast<uint16_t*>(scratch + NT * 4 * 4 + NT * TW32_VP * 2);  // [NT][C]
  uint16_t* sval = sidx + NT * C;                                                  // [NT][C]
  const float b = o.bias ? o.bias[j] : 0.0f;
  const int ntok = min(NT, o.T - t0);  // tokens of this call (the rest are masked)
  // 1. thread = neuron
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    if (i >= ntok) {  // uniform: tokens beyond T keep nothing
      if (lane == 0) masks[i * 4 + w] = 0u;
      continue;
    }
    const float gv = g[i] + b;
    const float a = act_fn(gv, o.act);
    const bool in = (t0 + i) < o.T;
    const bool k = in && fabsf(a) > o.tau;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, k);
    if (lane == 0) masks[i * 4 + w] = bal;
    vals[i * TW32_VP + n_in] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
    if (o.gdebug && in) o.gdebug[(size_t)(t0 + i) * o.F + j] = gv;
  }
  named_bar_sync(bar_id, 128);
  // 2. four threads per token
  if (etid < 4 * NT && t0 + (etid >> 2) < o.T) {
    const int tt = etid >> 2, wq = etid & 3, t = t0 + tt;
    const uint4 m4 = reinterpret_cast<const uint4*>(masks)[tt];
    const int c0 = __popc(m4.x), c1 = __popc(m4.y), c2 = __popc(m4.z), c3 = __popc(m4.w);
    const int total = c0 + c1 + c2 + c3;
    int rank = (wq > 0 ? c0 : 0) + (wq > 1 ? c1 : 0) + (wq > 2 ? c2 : 0);
    uint32_t m = wq == 0 ? m4.x : wq == 1 ? m4.y : wq == 2 ? m4.z : m4.w;
    const int q = C >> 2;  // pad slots this thread owns: [wq q, (wq + 1) q)
    for (int sl = wq * q; sl < (wq + 1) * q; ++sl)
      if (sl >= total) {
        sidx[tt * C + sl] = 0xFFFFu;   // -1
        sval[tt * C + sl] = 0u;        // +0
      }
    while (m != 0u && rank < C) {
      const int bit = __ffs(m) - 1;
      m &= m - 1u;
      const int n = wq * 32 + bit;
      sidx[tt * C + rank] = (uint16_t)(p * 128 + n);
      sval[tt * C + rank] = vals[tt * TW32_VP + n];
      ++rank;
    }
    if (wq == 0 && t < o.T) {
      o.count[(size_t)t * o.n_tiles + p] = (int16_t)total;
      if (total > C) o.ovf[t] = o.epoch;
      if (o.kmask) reinterpret_cast<uint4*>(o.kmask)[(size_t)t * o.n_tiles + p] = m4;
    }
  }
  named_bar_sync(bar_id, 128);
  // 3. whole records out, 8 slots per 16-byte vector
  {
    const int nvec = C >> 3;
    for (int e = etid; e < 2 * NT * nvec; e += 128) {
      const int arr = e / (NT * nvec), r = e - arr * NT * nvec;
      const int tt = r / nvec, v = r - tt * nvec, t = t0 + tt;
      if (t >= o.T) continue;
      const uint4 val = reinterpret_cast<const uint4*>((arr ? sval : sidx) + tt * C)[v];
      uint16_t* dst = arr ? reinterpret_cast<uint16_t*>(o.val) : reinterpret_cast<uint16_t*>(o.idx);
      reinterpret_cast<uint4*>(dst + ((size_t)t * o.n_tiles + p) * C)[v] = val;
    }
  }
  named_bar_sync(bar_id, 128);  // the staging is free for the next call
}

struct EpiGateTwell {
  static constexpr int N_ACC = 1;
  static constexpr int EPI_SMEM = twell32_smem(128);
  using Params = TwellParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t* scratch) {
    const int j = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= o.T) break;
      float g[32];
      tmem_ld16(tmem + c, g);
      if (BN > 16) {
        tmem_ld16(tmem + c + 16, g + 16);
      } else {
#pragma unroll
        for (int i = 16; i < 32; ++i) g[i] = 0.f;
      }
      twell_tile32(o, g, j, n0 + c, etid, scratch, 1);
    }
  }
};

// ------------------------------------------------------------------- WINA
// Dense activation and score for the per-token top-k: v = round(sigma(g+b)),
// s = |sigma(g+b)|·n_j, both [T][F].
struct WinaParams {
  const float* bias;
  int act, T, F;
  const float* norms;
  void* vdense;       // [T][F] bf16 or fp32
  int val_f32;
  float* scores;      // [T][F]
};

__device__ __forceinline__ void wina_chunk(const WinaParams& o, const float* g, int j, int t0) {
  const float b = o.bias ? o.bias[j] : 0.0f;
  const float n = o.norms[j];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int t = t0 + i;
    if (t < o.T) {
      const float a = act_fn(g[i] + b, o.act);
      const size_t off = (size_t)t * o.F + j;
      if (o.val_f32)
        reinterpret_cast<float*>(o.vdense)[off] = a;
      else
        reinterpret_cast<__nv_bfloat16*>(o.vdense)[off] = __float2bfloat16_rn(a);
      o.scores[off] = fabsf(a) * n;
    }
  }
}

struct EpiWina {
  static constexpr int N_ACC = 1;
  using Params = WinaParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int j = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= o.T) break;
      float g[16];
      tmem_ld16(tmem + c, g);
      wina_chunk(o, g, j, n0 + c);
    }
  }
};

// ------------------------------------------------------- WINA, full-h score
// [WINA] section 3.1 with the hidden value taken as the whole gated product:
// the tile kernel runs two phases into two accumulators, g = W_gate·x (col 0)
// and u = W_up·x (col BN), for every neuron of the tile.  Per (token, neuron):
// a = sigma(g + b), v = round(a) (the TwELL value), s = |a·u|·n_j (the score
// of the unrounded product) and h = v·u (fp32, what the down projection adds
// for a kept neuron).
struct WinaFullHParams {
  const float* bias;
  int act, T, F;
  const float* norms;
  __nv_bfloat16* vdense;  // [T][F]
  float* scores;          // [T][F]
  float* hfull;           // [T][F]
};

struct EpiWinaFullH {
  static constexpr int N_ACC = 2;
  using Params = WinaFullHParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int j = m0 + etid;
    const float b = o.bias ? o.bias[j] : 0.0f;
    const float n = o.norms[j];
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= o.T) break;
      float g[16], u[16];
      tmem_ld16(tmem + c, g);
      tmem_ld16(tmem + BN + c, u);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = n0 + c + i;
        if (t < o.T) {
          const float a = act_fn(g[i] + b, o.act);
          const __nv_bfloat16 v = __float2bfloat16_rn(a);
          const size_t off = (size_t)t * o.F + j;
          o.vdense[off] = v;
          o.scores[off] = fabsf(a * u[i]) * n;
          o.hfull[off] = __bfloat162float(v) * u[i];
        }
      }
    }
  }
};

// -------------------------------------------------- plain bf16 store of D
// D[128 rows][BN cols] rounded to bf16 and stored row-major: out[r][c] at
// r·ld + c (transpose = 0) or out[c][r] at c·ld + r (transpose = 1), rows
// below `rows` and columns below `cols` only.  Used for the orthogonalising
// rotations ([WINA] section 3.3): W' = W·V (rows = neurons) and x' = x·V
// (computed as V^T·x^T, rows = input coordinates, stored transposed).
struct StoreParams {
  __nv_bfloat16* out;
  long long ld;
  int rows, cols, transpose;
};

struct EpiStoreBf16 {
  static constexpr int N_ACC = 1;
  using Params = StoreParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int r = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= o.cols) break;
      float v[16];
      tmem_ld16(tmem + c, v);
      if (r < o.rows) {
        if (o.transpose) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (n0 + c + i < o.cols) o.out[(size_t)(n0 + c + i) * o.ld + r] = __float2bfloat16_rn(v[i]);
        } else {
          __align__(16) __nv_bfloat16 pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = __float2bfloat16_rn(v[i]);
          __nv_bfloat16* dst = o.out + (size_t)r * o.ld + n0 + c;
          if (n0 + c + 16 <= o.cols && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
            reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(pk)[0];
            reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(pk)[1];
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (n0 + c + i < o.cols) dst[i] = pk[i];
          }
        }
      }
    }
  }
};

// ------------------------------------------------------- low-rank gate: z
// z = round_bf16(x·A).  The tile's rows are rank coordinates r, its columns
// tokens.  With a split K every CTA stores its fp32 partial in its split's
// slot; the CTA that completes the tile's ticket adds the splits in
// ascending K order (the same order on every forward, so z is reproducible),
// rounds and stores z, and clears the ticket.
constexpr int Z_MAX_SPLITS = 4;  // the last CTA's loads of every split go out at once

struct ZParams {
  int T, R, splits;
  float* zpart;            // [row tiles x token tiles][splits][BN][128] fp32 (splits > 1)
  __nv_bfloat16* z;        // [maxT][R]
  int* tickets;            // [row tiles x token tiles], zero between forwards
};

struct EpiLowRankZ {
  static constexpr int N_ACC = 1;
  using Params = ZParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int split, int etid, uint8_t* scratch) {
    const int r = m0 + etid;
    const bool rin = r < o.R;
    if (o.splits == 1) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        if (n0 + c >= o.T) break;
        float g[16];
        tmem_ld16(tmem + c, g);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (n0 + c + i < o.T && rin) o.z[(size_t)(n0 + c + i) * o.R + r] = __float2bfloat16_rn(g[i]);
      }
      return;
    }
    const int slot = blockIdx.x * gridDim.y + blockIdx.y;
    float* base = o.zpart + (size_t)slot * o.splits * BN * 128;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= o.T) break;
      float g[16];
      tmem_ld16(tmem + c, g);
#pragma unroll
      for (int i = 0; i < 16; ++i) __stcg(&base[((size_t)split * BN + c + i) * 128 + etid], g[i]);
    }
    int* last = reinterpret_cast<int*>(scratch);
    __threadfence();
    named_bar_sync(1, 128);
    if (etid == 0) *last = atomicAdd(&o.tickets[slot], 1) == o.splits - 1;
    named_bar_sync(1, 128);
    if (!*last) return;
    __threadfence();
    const int tend = min(o.T - n0, BN);
#pragma unroll 1
    for (int c = 0; c < tend; c += 16) {
      float h[Z_MAX_SPLITS][16];
#pragma unroll
      for (int q = 0; q < Z_MAX_SPLITS; ++q)
#pragma unroll
        for (int i = 0; i < 16; ++i)
          h[q][i] = q < o.splits ? __ldcg(&base[((size_t)q * BN + c + i) * 128 + etid]) : 0.f;
      float g[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {  // splits added in ascending K order
        g[i] = h[0][i];
#pragma unroll
        for (int q = 1; q < Z_MAX_SPLITS; ++q)
          if (q < o.splits) g[i] += h[q][i];
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (c + i < tend && rin) o.z[(size_t)(n0 + c + i) * o.R + r] = __float2bfloat16_rn(g[i]);
    }
    if (etid == 0) o.tickets[slot] = 0;
  }
};

// -------------------------------------------------- dense fallback: h rows
// Overflow tokens ([TwELL] hybrid routing): both accumulators hold g (col 0)
// and u (col BN) for the gathered overflow rows.  h = keep ? bf16(a)·u : 0 is
// written as a bf16 pair (hi + lo, hi = bf16(h), lo = bf16(h - hi)) so the
// tensor-core down projection loses no more than 2^-16 relative of h.
struct HParams {
  const float* bias;
  float tau;
  int act, F;
  const int* n_rows_dev;    // number of valid rows (overflow count)
  int n_rows;               // used when n_rows_dev is null
  const int* row_map;       // output row of gathered row o (or null: identity)
  __nv_bfloat16* h_hi;      // [maxT][F]
  __nv_bfloat16* h_lo;
  int val_f32;              // stored value rounding: 0 bf16
};

__device__ __forceinline__ void store_h(const HParams& o, int row, int j, float h) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(h);
  const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
  const size_t off = (size_t)row * o.F + j;
  o.h_hi[off] = hi;
  o.h_lo[off] = lo;
}

struct EpiFallbackH {
  static constexpr int N_ACC = 2;
  using Params = HParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int n_rows = o.n_rows_dev ? *o.n_rows_dev : o.n_rows;
    const int j = m0 + etid;
    const float b = o.bias ? o.bias[j] : 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= n_rows) break;
      float g[16], u[16];
      tmem_ld16(tmem + c, g);
      tmem_ld16(tmem + BN + c, u);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = n0 + c + i;
        if (r < n_rows) {
          const float a = act_fn(g[i] + b, o.act);
          const bool keep = fabsf(a) > o.tau;
          const float v = __bfloat162float(__float2bfloat16_rn(a));
          store_h(o, o.row_map ? o.row_map[r] : r, j, keep ? v * u[i] : 0.0f);
        }
      }
    }
  }
};

// ------------------------------------------- tile path: h from TwELL values
// Non-overflow tokens on the tile path: the accumulator holds u for a
// 128-neuron tile; the kept values come from the token's TwELL record, which
// is scattered into a shared [32 tokens][128 neurons] table, 32 tokens at a
// time.  Overflow tokens are skipped (their rows come from the fallback).
// Hybrid routing ([TwELL] "Hybrid 應對非均勻稀疏") for the tile path, done
// by the epilogue warps of the first tile's CTA before their own tile: the
// tokens whose TwELL record overflowed go whole to the dense channel, which
// runs after this kernel.  They are listed in token order and counted, and
// their x (and z) rows are gathered for the dense channel's B operand.
struct RouteParams {
  int* ovf_list;      // [maxT] (null: no routing in this launch)
  int* ovf_count;     // [1]
  const uint4* x;     // [T][d/8]
  uint4* xo;
  int d_vec;
  const uint4* z;     // [T][R/8] or null
  uint4* zo;
  int r_vec;
};

__device__ __forceinline__ void route_overflow(const RouteParams& r, const uint32_t* ovf, uint32_t epoch, int T,
                                               int etid, int* sh /*[8]*/) {
  const int w = etid >> 5, lane = etid & 31;
  int base = 0;
  for (int c = 0; c < T; c += 128) {
    const int t = c + etid;
    const bool o = t < T && ovf[t] == epoch;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, o);
    if (lane == 0) sh[w] = __popc(bal);
    named_bar_sync(1, 128);
    int pre = base;
    for (int q = 0; q < w; ++q) pre += sh[q];
    if (o) r.ovf_list[pre + __popc(bal & lanemask_lt())] = t;
    base += sh[0] + sh[1] + sh[2] + sh[3];
    named_bar_sync(1, 128);
  }
  if (etid == 0) *r.ovf_count = base;
  // gathers: the list entries this thread wrote are visible to the CTA after the barrier
  __threadfence_block();
  named_bar_sync(1, 128);
  for (int o = 0; o < base; ++o) {
    const int t = r.ovf_list[o];
    for (int v = etid; v < r.d_vec; v += 128) r.xo[(size_t)o * r.d_vec + v] = r.x[(size_t)t * r.d_vec + v];
    if (r.z)
      for (int v = etid; v < r.r_vec; v += 128) r.zo[(size_t)o * r.r_vec + v] = r.z[(size_t)t * r.r_vec + v];
  }
  named_bar_sync(1, 128);
}

struct TwellHParams {
  int T, F, n_tiles, C;
  const int16_t* count;
  const int16_t* idx;
  const __nv_bfloat16* val;
  const uint32_t* ovf;
  uint32_t epoch;
  __nv_bfloat16* h_hi;
  __nv_bfloat16* h_lo;
  RouteParams route;  // done by the CTA of tile (0, 0) when route.ovf_list is set
};

struct EpiTwellH {
  static constexpr int N_ACC = 1;
  using Params = TwellHParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t* scratch) {
    uint16_t* tab = reinterpret_cast<uint16_t*>(scratch);            // [32][128]
    int* live = reinterpret_cast<int*>(scratch + 32 * 128 * 2);        // [32]
    const int p = m0 >> 7, j = m0 + etid;
    if (o.route.ovf_list && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
      route_overflow(o.route, o.ovf, o.epoch, o.T, etid, live);
    HParams hp;
    hp.F = o.F;
    hp.h_hi = o.h_hi;
    hp.h_lo = o.h_lo;
#pragma unroll 1
    for (int c32 = 0; c32 < BN; c32 += 32) {
      if (n0 + c32 >= o.T) break;
      for (int e = etid; e < 32 * 128 / 2; e += 128) reinterpret_cast<uint32_t*>(tab)[e] = 0u;
      if (etid < 32) {
        const int t = n0 + c32 + etid;
        live[etid] = (t < o.T && o.ovf[t] != o.epoch) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      {
        const int tl = etid >> 2, q = etid & 3;
        const int t = n0 + c32 + tl;
        if (live[tl]) {
          const size_t rec = (size_t)t * o.n_tiles + p;
          const int cnt = min((int)o.count[rec], o.C);
          for (int s = q; s < cnt; s += 4) {
            const int jj = o.idx[rec * o.C + s] - m0;
            if (jj >= 0 && jj < 128)
              tab[tl * 128 + jj] = reinterpret_cast<const uint16_t*>(o.val)[rec * o.C + s];
          }
        }
      }
      named_bar_sync(1, 128);
#pragma unroll 1
      for (int c = 0; c < 32; c += 16) {
        if (c32 + c >= BN) break;
        float u[16];
        tmem_ld16(tmem + c32 + c, u);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tl = c + i;
          if (live[tl]) {
            const float v = __uint_as_float((uint32_t)tab[tl * 128 + etid] << 16);
            store_h(hp, n0 + c32 + tl, j, v * u[i]);
          }
        }
      }
      named_bar_sync(1, 128);
    }
  }
};

// -------------------------------------------------- down projection output
// D^T tile: rows are output columns (m0 + etid), columns are h rows; every
// stage multiplies one W_down^T tile by both halves of h (hi and lo) into the
// one accumulator.  With a split K the partial sums are added into out
// (zeroed beforehand by the router, the gate or the fused row kernel).
struct OutParams {
  float* out;          // [T][d]
  int d;
  const int* n_rows_dev;
  int n_rows;
  const int* row_map;  // out row of h row r (null: identity)
  int atomic;
};

struct EpiDownOut {
  static constexpr int N_ACC = 1;
  static constexpr bool DUAL_B = true;  // B0 = h_hi, B1 = h_lo, one accumulator
  using Params = OutParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int n_rows = o.n_rows_dev ? *o.n_rows_dev : o.n_rows;
    const int col = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= n_rows) break;
      float y[16];
      tmem_ld16(tmem + c, y);
      if (col < o.d) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = n0 + c + i;
          if (r < n_rows) {
            const int row = o.row_map ? o.row_map[r] : r;
            float* dst = &o.out[(size_t)row * o.d + col];
            if (o.atomic)
              atomicAdd(dst, y[i]);
            else
              *dst = y[i];
          }
        }
      }
    }
  }
};

}  // namespace sffn
