// SIMT kernels: the overflow router, the fused sparse up x down pass over
// kept rows, the WINA per-token top-k, the fp32 path and create-time helpers.
#pragma once

#include "epilogues.cuh"
#include "ptx.cuh"

namespace sffn {

// Exclusive scan of one int per thread over the whole block (<= 32 warps).
// warp_tot: shared scratch of >= 33 ints.  Returns the exclusive prefix and
// sets *total (all threads).  Contains __syncthreads.
__device__ __forceinline__ int block_scan_excl(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nw ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, ti, o);
      if (lane >= o) ti += n;
    }
    if (lane < nw) warp_tot[lane] = ti - t;
    if (lane == 31) warp_tot[32] = ti;
  }
  __syncthreads();
  const int excl = warp_tot[warp] + inc - v;
  *total = warp_tot[32];
  __syncthreads();
  return excl;
}

// ---------------------------------------------------------------- router
// Hybrid routing ([TwELL] "Hybrid 應對非均勻稀疏") for the tile path and the
// fp32 path: a token whose TwELL record overflowed in some tile goes whole to
// the dense channel.  Every CTA ranks the overflow tokens itself (the flags
// are few); CTA 0 publishes the overflow list and its count; all CTAs then
// gather the overflow rows of x (and z) and, if asked, zero the output that
// later kernels accumulate into.  (The fused row kernel routes its own
// blocks.)
struct RouterArgs {
  int T;
  const uint32_t* ovf;
  uint32_t epoch;
  int* ovf_list;           // [maxT]
  int* ovf_count;          // [1]
  const uint4* x;          // [T][d] bf16 as 16-byte vectors, or null (no gather)
  uint4* xo;               // [maxT][d]
  int d_vec;               // d / 8
  const uint4* z;          // [T][R] bf16, or null
  uint4* zo;
  int r_vec;               // R / 8
  float4* out;             // [T][d] fp32
  int d4;                  // d / 4
  int zero_all;            // zero all T rows of out
};

__host__ __device__ inline int router_smem_bytes(int T) { return T * 4; }

__global__ void __launch_bounds__(1024) k_router(const RouterArgs a) {
  extern __shared__ int rs_list[];   // [T] overflow list
  __shared__ int scan_tmp[33];
  griddep_wait();
  int base = 0;
  for (int c = 0; c < a.T; c += blockDim.x) {
    const int t = c + threadIdx.x;
    const int f = (t < a.T && a.ovf[t] == a.epoch) ? 1 : 0;
    int tot;
    const int ex = block_scan_excl(f, scan_tmp, &tot);
    if (f) rs_list[base + ex] = t;
    base += tot;
  }
  __syncthreads();
  const int n_o = base;
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < n_o; i += blockDim.x) a.ovf_list[i] = rs_list[i];
    if (threadIdx.x == 0) *a.ovf_count = n_o;
  }
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long gstride = (long long)gridDim.x * blockDim.x;
  if (a.x) {
    const long long n = (long long)n_o * a.d_vec;
    for (long long e = gtid; e < n; e += gstride) {
      const int o = (int)(e / a.d_vec), v = (int)(e % a.d_vec);
      a.xo[(size_t)o * a.d_vec + v] = a.x[(size_t)rs_list[o] * a.d_vec + v];
    }
  }
  if (a.z) {
    const long long n = (long long)n_o * a.r_vec;
    for (long long e = gtid; e < n; e += gstride) {
      const int o = (int)(e / a.r_vec), v = (int)(e % a.r_vec);
      a.zo[(size_t)o * a.r_vec + v] = a.z[(size_t)rs_list[o] * a.r_vec + v];
    }
  }
  if (a.zero_all) {
    const long long n = (long long)a.T * a.d4;
    for (long long e = gtid; e < n; e += gstride) a.out[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ------------------------------------------------------------ WINA top-k
// [WINA] section 3.1 / section 2: per token keep the k largest scores
// s_tj = |a_tj|·n_j, equal scores going to the smaller index, and write the
// kept neurons as TwELL.  Scores are non-negative, so their fp32 bit patterns
// order like the values: a 4-pass 8-bit radix select finds the k-th largest
// pattern K and how many entries equal to K are kept; tie ranks follow index
// order through per-tile counts.  One CTA (1024 threads) per token.
struct TopkArgs {
  const float* scores;   // [T][F]
  const void* vdense;    // [T][F] bf16 or fp32
  int val_f32;
  int T, F, k, n_tiles, C;
  int16_t* count;
  int16_t* idx;
  void* val;
  uint32_t* ovf;
  uint32_t epoch;
  const float* hfull;    // full-h variant: [T][F] h = v·u; the kept entries go to
  __nv_bfloat16* h_hi;   // h_hi/h_lo [T][F] (hi + lo split), the others are zeroed
  __nv_bfloat16* h_lo;   // (null: TwELL only)
};

// keys, histograms, tie prefix (padded to 16 bytes), per-warp staged records
__host__ __device__ inline int topk_smem_bytes(int F, int n_tiles, int C) {
  return F * 4 + 32 * 256 * 4 + ((n_tiles + 3) & ~3) * 4 + 32 * 3 * C * 2;
}

// The k-th largest of n non-negative fp32 bit patterns in shared memory, by a
// 4-pass 8-bit radix select (1024 threads, per-warp histograms hist[32][256]).
// Returns K, the k-th largest pattern, and *rem, how many entries equal to K
// belong to the k largest (ties are then broken by the caller, by index).
// Needs 0 < k < n.
__device__ __forceinline__ uint32_t radix_select_kth(const uint32_t* keys, int n, int k, uint32_t* hist,
                                                     int* wtot, int* wpre, uint32_t* sel, int* rem_out) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t prefix = 0, mask = 0;
  int rem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int e = tid; e < 32 * 256; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += blockDim.x) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[warp * 256 + ((key >> shift) & 255u)], 1u);
    }
    __syncthreads();
    // bins in descending order: four threads per bin (thread group g = bin
    // 255 - g) add the 32 per-warp counts, then a scan over the groups gives
    // every bin the number of keys in higher bins
    const int g = tid >> 2, part = tid & 3, bin = 255 - g;
    int c = 0;
    for (int w2 = part; w2 < 32; w2 += 4) c += (int)hist[w2 * 256 + bin];
    c += __shfl_xor_sync(0xFFFFFFFFu, c, 1);
    c += __shfl_xor_sync(0xFFFFFFFFu, c, 2);
    int inc = c;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += nn;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const int v = wtot[lane];
      int vi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nn = __shfl_up_sync(0xFFFFFFFFu, vi, o);
        if (lane >= o) vi += nn;
      }
      wpre[lane] = vi - v;
    }
    __syncthreads();
    const int ex = wpre[warp] + inc - c;
    if (part == 0 && ex < rem && ex + c >= rem) {
      sel[0] = (uint32_t)bin;
      sel[1] = (uint32_t)(rem - ex);
    }
    __syncthreads();
    prefix |= sel[0] << shift;
    mask |= 255u << shift;
    rem = (int)sel[1];
    __syncthreads();
  }
  *rem_out = rem;
  return prefix;
}

__global__ void __launch_bounds__(1024) k_wina_topk(const TopkArgs a) {
  extern __shared__ uint32_t tk_keys[];   // [F] keys, [32][256] histograms, [n_tiles] tie prefix, [32] records
  uint32_t* hist = tk_keys + a.F;
  int* eqpre = reinterpret_cast<int*>(hist + 32 * 256);
  uint16_t* recs = reinterpret_cast<uint16_t*>(eqpre + ((a.n_tiles + 3) & ~3));
  __shared__ int wtot[32], wpre[32];
  __shared__ uint32_t sel[4];  // prefix, remaining
  griddep_wait();
  const int t = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* sc = a.scores + (size_t)t * a.F;
  // F is a multiple of 128: 16-byte loads, several in flight per thread
#pragma unroll 4
  for (int j = 4 * tid; j < a.F; j += 4 * blockDim.x)
    *reinterpret_cast<uint4*>(&tk_keys[j]) = *reinterpret_cast<const uint4*>(&sc[j]);
  const int k = a.k;
  const bool keep_all = k >= a.F, keep_none = k <= 0;
  int rem = k;
  uint32_t prefix = 0;
  if (!keep_all && !keep_none) {
    __syncthreads();
    prefix = radix_select_kth(tk_keys, a.F, k, hist, wtot, wpre, sel, &rem);
  }
  // tie prefix over tiles: number of keys equal to K in lower tiles
  const uint32_t K = prefix;
  for (int p = warp; p < a.n_tiles; p += 32) {
    int c = 0;
    for (int q = 0; q < 4; ++q) c += __popc(__ballot_sync(0xFFFFFFFFu, tk_keys[p * 128 + q * 32 + lane] == K));
    if (lane == 0) eqpre[p] = c;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix over the tiles: lane l takes tiles [8l, 8l + 8)
    int loc[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int p = 8 * lane + i;
      loc[i] = p < a.n_tiles ? eqpre[p] : 0;
      sum += loc[i];
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += n;
    }
    int run = inc - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int p = 8 * lane + i;
      if (p < a.n_tiles) eqpre[p] = run;
      run += loc[i];
    }
  }
  __syncthreads();
  // records: each warp stages a tile's record (ascending neuron order, pads
  // after the count) in shared memory and writes it as 16-byte vectors
  const uint32_t lt = lanemask_lt();
  uint16_t* ridx = recs + warp * 3 * a.C;                 // [C] idx, then [C] values (2 or 4 bytes)
  uint16_t* rval = ridx + a.C;
  const int vb = a.val_f32 ? 4 : 2;
  for (int p = warp; p < a.n_tiles; p += 32) {
    int run = 0, ties = eqpre[p];
    const size_t rec = (size_t)t * a.n_tiles + p;
    for (int sl = lane; sl < a.C; sl += 32) {
      ridx[sl] = 0xFFFFu;  // -1
      rval[sl] = 0u;       // +0
      if (a.val_f32) rval[a.C + sl] = 0u;
    }
    __syncwarp();
    for (int q = 0; q < 4; ++q) {
      const int j = p * 128 + q * 32 + lane;
      const uint32_t key = tk_keys[j];
      const uint32_t eqb = __ballot_sync(0xFFFFFFFFu, key == K);
      const int tie_rank = ties + __popc(eqb & lt);
      const bool keep = keep_all || (!keep_none && (key > K || (key == K && tie_rank < rem)));
      ties += __popc(eqb);
      const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
      const int slot = run + __popc(kb & lt);
      if (keep && slot < a.C) {
        ridx[slot] = (uint16_t)j;
        if (a.val_f32)
          reinterpret_cast<float*>(rval)[slot] = reinterpret_cast<const float*>(a.vdense)[(size_t)t * a.F + j];
        else
          rval[slot] = reinterpret_cast<const uint16_t*>(a.vdense)[(size_t)t * a.F + j];
      }
      run += __popc(kb);
      if (a.hfull) {  // full-h variant: the down projection's h row, zero where not kept
        const size_t off = (size_t)t * a.F + j;
        const float hv = keep ? a.hfull[off] : 0.0f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
        a.h_hi[off] = hi;
        a.h_lo[off] = __float2bfloat16_rn(hv - __bfloat162float(hi));
      }
    }
    __syncwarp();
    const int ni = a.C >> 3, nvv = a.C * vb / 16;  // 16-byte vectors of idx and of values
    for (int e = lane; e < ni + nvv; e += 32) {
      if (e < ni) {
        reinterpret_cast<uint4*>(a.idx + rec * a.C)[e] = reinterpret_cast<const uint4*>(ridx)[e];
      } else {
        uint8_t* dst = reinterpret_cast<uint8_t*>(a.val) + rec * a.C * vb;
        reinterpret_cast<uint4*>(dst)[e - ni] = reinterpret_cast<const uint4*>(rval)[e - ni];
      }
    }
    if (lane == 0) {
      a.count[rec] = (int16_t)run;
      if (run > a.C) a.ovf[t] = a.epoch;
    }
    __syncwarp();
  }
}

// ------------------------------------------------- WINA on the input side
// [WINA] section 3.1 applied to the layer that consumes x, the stacked
// [W_gate; W_up]: per token keep the k input coordinates with the largest
// s_i = |x_i|·c_i (c = the stacked matrix's column norms; the product
// rounded once to fp32, equal scores to the smaller index) and zero the rest.
// One CTA (1024 threads) per token; d <= 4 x 1024.
struct InputSelectArgs {
  const __nv_bfloat16* x;   // [T][d]
  const float* colnorm;     // [d]
  __nv_bfloat16* xsel;      // [T][d]
  int T, d, k;
};

__host__ __device__ inline int input_select_smem_bytes(int d) { return d * 4 + 32 * 256 * 4; }

__global__ void __launch_bounds__(1024) k_input_select(const InputSelectArgs a) {
  extern __shared__ uint32_t is_keys[];   // [d] keys, [32][256] histograms
  uint32_t* hist = is_keys + a.d;
  __shared__ int wtot[33], wpre[32];
  __shared__ uint32_t sel[4];
  griddep_wait();
  const int t = blockIdx.x, tid = threadIdx.x;
  const __nv_bfloat16* xr = a.x + (size_t)t * a.d;
  for (int i = tid; i < a.d; i += blockDim.x)
    is_keys[i] = __float_as_uint(fabsf(__bfloat162float(xr[i])) * a.colnorm[i]);
  __syncthreads();
  const int k = a.k;
  int rem = k;
  uint32_t K = 0;
  const bool keep_all = k >= a.d;
  if (!keep_all && k > 0) K = radix_select_kth(is_keys, a.d, k, hist, wtot, wpre, sel, &rem);
  // ties at K: the rem lowest indices.  Thread tid owns the contiguous
  // coordinates [4 tid, 4 tid + 4): a block scan of its tie count ranks them
  const int i0 = 4 * tid;
  int eq = 0;
  for (int q = 0; q < 4; ++q) eq += (i0 + q < a.d && is_keys[i0 + q] == K) ? 1 : 0;
  int tot;
  int rank = block_scan_excl(eq, wtot, &tot);
  __nv_bfloat16* out = a.xsel + (size_t)t * a.d;
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + q;
    if (i >= a.d) break;
    const uint32_t key = is_keys[i];
    bool keep = keep_all;
    if (!keep_all && k > 0) {
      keep = key > K;
      if (key == K) keep = rank++ < rem;
    }
    out[i] = keep ? xr[i] : __float2bfloat16_rn(0.0f);
  }
}

// Column norms of the stacked [W_gate; W_up] (create time): c_i = sqrt of the
// sum over both matrices' rows of W[j][i]^2, accumulated in fp64 and rounded
// to fp32.  One thread per column (consecutive threads read consecutive
// columns of a row), rows split across gridDim.y with fp64 atomics into
// acc[d], then k_col_norms_finish rounds.
__global__ void k_col_sumsq(const __nv_bfloat16* __restrict__ Wg, const __nv_bfloat16* __restrict__ Wu, int F,
                            int d, double* acc) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= d) return;
  const int per = (2 * F + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * per, r1 = min(2 * F, r0 + per);
  double s = 0.0;
  for (int r = r0; r < r1; ++r) {
    const __nv_bfloat16* W = r < F ? Wg : Wu;
    const double v = (double)__bfloat162float(W[(size_t)(r < F ? r : r - F) * d + i]);
    s += v * v;
  }
  atomicAdd(&acc[i], s);
}

__global__ void k_col_norms_finish(const double* acc, int d, float* c) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < d) c[i] = (float)sqrt(acc[i]);
}

// ---------------------------------------------------------------- fp32 path
// The fp32 configuration has no full-precision tensor-core MMA, so its gate
// is a SIMT tile: 128 threads = the 128 neurons of one tile, 16 tokens.  K
// goes in chunks of 64: the tile's 128 W_gate row pieces and the tokens' x
// pieces are staged in shared memory by coalesced loads (rows padded to 65
// floats, so that each thread reads its own row bank-conflict free), then
// every thread accumulates its neuron's 16 dot products.  The same TwELL (or
// WINA score) emission as the tensor-core epilogue follows.
struct GateF32Args {
  const float* x;       // [T][d]
  const float* W_gate;  // [F][d]
  int d;
  int wina;             // 0: TwELL emission, 1: WINA dense value + score
  TwellParams tw;
  WinaParams wp;
};

constexpr int GF_K = 64;

__global__ void __launch_bounds__(128) k_gate_f32(const GateF32Args a) {
  __shared__ float ws[128][GF_K + 1];
  __shared__ __align__(16) float xs[16][GF_K];
  __shared__ uint32_t masks[2][64];
  griddep_wait();
  const int p = blockIdx.x, t0 = blockIdx.y * 16;
  const int etid = threadIdx.x, j = p * 128 + etid;
  const int T = a.wina ? a.wp.T : a.tw.T;
  const int d = a.d;
  float g[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) g[i] = 0.f;
  const float* wtile = a.W_gate + (size_t)p * 128 * d;
  for (int k0 = 0; k0 < d; k0 += GF_K) {
    const int kn = min(GF_K, d - k0);
    __syncthreads();
    // all of a thread's loads go out before its first store (64 W and 8 x
    // values per thread per chunk): one memory latency per chunk, not 72
    if ((d & 3) == 0) {
      float4 wv[16], xv[2];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int e = etid + 128 * q, r = e >> 4, c = 4 * (e & 15);
        wv[q] = c < kn ? __ldg(reinterpret_cast<const float4*>(wtile + (size_t)r * d + k0 + c))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e = etid + 128 * q, i = e >> 4, c = 4 * (e & 15), t = t0 + i;
        xv[q] = (t < T && c < kn) ? __ldg(reinterpret_cast<const float4*>(a.x + (size_t)t * d + k0 + c))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int e = etid + 128 * q, r = e >> 4, c = 4 * (e & 15);
        ws[r][c] = wv[q].x;
        ws[r][c + 1] = wv[q].y;
        ws[r][c + 2] = wv[q].z;
        ws[r][c + 3] = wv[q].w;
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e = etid + 128 * q, i = e >> 4, c = 4 * (e & 15);
        *reinterpret_cast<float4*>(&xs[i][c]) = xv[q];
      }
    } else {
#pragma unroll 8
      for (int e = etid; e < 128 * GF_K; e += 128) {
        const int r = e / GF_K, c = e % GF_K;
        ws[r][c] = c < kn ? wtile[(size_t)r * d + k0 + c] : 0.f;
      }
#pragma unroll 8
      for (int e = etid; e < 16 * GF_K; e += 128) {
        const int i = e / GF_K, c = e % GF_K;
        const int t = t0 + i;
        xs[i][c] = (t < T && c < kn) ? a.x[(size_t)t * d + k0 + c] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < GF_K; ++kk) {
      const float w = ws[etid][kk];
#pragma unroll
      for (int i = 0; i < 16; ++i) g[i] = fmaf(w, xs[i][kk], g[i]);
    }
  }
  if (a.wina)
    wina_chunk(a.wp, g, j, t0);
  else
    twell_chunk(a.tw, g, j, t0, etid, masks[0]);
}

// Sparse up x down for one fp32 token per CTA: its TwELL neurons are gathered
// into shared memory, one warp per neuron computes u = <W_up[j], x_t> and
// h = v·u, then every thread adds h·W_down[j] into its own output columns.
struct RowsF32Args {
  const float* x;
  const float* W_up;
  const float* W_down;
  const int16_t* count;
  const int16_t* idx;
  const float* val;
  const uint32_t* ovf;
  uint32_t epoch;
  float* out;
  int T, d, n_tiles, C;
};

__global__ void __launch_bounds__(256) k_rows_f32(const RowsF32Args a) {
  extern __shared__ float rf_smem[];   // xs[d], then hj[cap], then jj[cap] (int)
  griddep_wait();
  const int t = blockIdx.x;
  if (t >= a.T || a.ovf[t] == a.epoch) return;
  const int cap = a.n_tiles * a.C;
  float* xs = rf_smem;
  float* hv = xs + a.d;
  int* jj = reinterpret_cast<int*>(hv + cap);
  __shared__ int scan_tmp[33];
  __shared__ int n_keep;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < a.d; i += blockDim.x) xs[i] = a.x[(size_t)t * a.d + i];
  // gather the kept list in tile order (ascending j)
  int base = 0;
  for (int p0 = 0; p0 < a.n_tiles; p0 += blockDim.x) {
    const int p = p0 + tid;
    const int c = p < a.n_tiles ? min((int)a.count[(size_t)t * a.n_tiles + p], a.C) : 0;
    int tot;
    const int ex = block_scan_excl(c, scan_tmp, &tot);
    for (int sl = 0; sl < c; ++sl) {
      const size_t r = ((size_t)t * a.n_tiles + p) * a.C + sl;
      jj[base + ex + sl] = a.idx[r];
      hv[base + ex + sl] = a.val[r];
    }
    base += tot;
  }
  if (tid == 0) n_keep = base;
  __syncthreads();
  const int nk = n_keep;
  for (int e = warp; e < nk; e += blockDim.x / 32) {
    const float* wr = a.W_up + (size_t)jj[e] * a.d;
    float u = 0.f;
    for (int i = lane; i < a.d; i += 32) u = fmaf(wr[i], xs[i], u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xFFFFFFFFu, u, o);
    if (lane == 0) hv[e] = hv[e] * u;
  }
  __syncthreads();
  for (int i = tid; i < a.d; i += blockDim.x) {
    float y = 0.f;
    for (int e = 0; e < nk; ++e) y = fmaf(hv[e], a.W_down[(size_t)jj[e] * a.d + i], y);
    a.out[(size_t)t * a.d + i] = y;
  }
}

// Dense fallback for one fp32 overflow token per CTA: every neuron is
// recomputed (gate, activation, threshold, up), h is kept in shared memory and
// the down projection follows.
struct FallbackF32Args {
  const float* x;
  const float* W_gate;
  const float* W_up;
  const float* W_down;
  const float* bias;
  float tau;
  int act;
  const int* ovf_list;
  const int* ovf_count;
  float* out;
  int d, F;
};

__global__ void __launch_bounds__(256) k_fallback_f32(const FallbackF32Args a) {
  extern __shared__ float ff_smem[];   // xs[d], h[F]
  griddep_wait();
  const int o = blockIdx.x;
  if (o >= *a.ovf_count) return;
  const int t = a.ovf_list[o];
  float* xs = ff_smem;
  float* h = xs + a.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < a.d; i += blockDim.x) xs[i] = a.x[(size_t)t * a.d + i];
  __syncthreads();
  for (int j = warp; j < a.F; j += blockDim.x / 32) {
    const float* wg = a.W_gate + (size_t)j * a.d;
    const float* wu = a.W_up + (size_t)j * a.d;
    float g = 0.f, u = 0.f;
    for (int i = lane; i < a.d; i += 32) {
      g = fmaf(wg[i], xs[i], g);
      u = fmaf(wu[i], xs[i], u);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      g += __shfl_xor_sync(0xFFFFFFFFu, g, s);
      u += __shfl_xor_sync(0xFFFFFFFFu, u, s);
    }
    if (lane == 0) {
      const float av = act_fn(g + (a.bias ? a.bias[j] : 0.f), a.act);
      h[j] = fabsf(av) > a.tau ? av * u : 0.f;
    }
  }
  __syncthreads();
  for (int i = tid; i < a.d; i += blockDim.x) {
    float y = 0.f;
    for (int j = 0; j < a.F; ++j) {
      const float hj = h[j];
      if (hj != 0.f) y = fmaf(hj, a.W_down[(size_t)j * a.d + i], y);
    }
    a.out[(size_t)t * a.d + i] = y;
  }
}

// ------------------------------------------------------------- create time
// out[c][r] = in[r][c] for a rows x cols bf16 matrix (32x32 tiles).
__global__ void k_transpose_bf16(const __nv_bfloat16* in, __nv_bfloat16* out, int rows, int cols) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][i];
  }
}

// n_j = ||W_down[j,:]||_2, accumulated in fp64 and rounded to fp32 ([WINA] 3.1).
template <typename Tw>
__global__ void k_row_norms(const Tw* W, int F, int d, float* norms) {
  const int j = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= F) return;
  double s = 0.0;
  for (int i = lane; i < d; i += 32) {
    const double v = (double)(float)W[(size_t)j * d + i];
    s += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) norms[j] = (float)sqrt(s);
}

}  // namespace sffn
