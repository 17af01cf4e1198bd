// Backward pass of the activation-sparse gated FFN (relu-threshold selection,
// dense gate): training over the sparse format ("Sparser, Faster, Lighter
// Transformer Language Models", news article, section "Hybrid 應對非均勻稀疏").
// With the forward's selection held fixed and the rounding of the stored
// value passed straight through, for upstream dy:
//     dh = dy W_down^T (kept), du = dh·v, dg = dh·u·sigma'(g),
//     dW_down = h^T dy, dW_up = du^T x, dW_gate = dg^T x, db = sum_t dg,
//     dx = du W_up + dg W_gate.
// Only the kept (token, neuron) pairs are touched.  They come from the
// forward's keep masks (kmask [T][P][4] words: every token's full kept set,
// overflow tokens included), in two orders:
//   token-major (CSR): pair p of token t sits at rowptr[t] + its rank among
//     the token's kept neurons (ascending);
//   neuron-major (CSC): for neuron j, the CSR positions of its pairs in token
//     order.
// Kernels, in launch order:
//   k_bwd_rows     per token: kept count, per-word rank prefix; zeroes dx of
//                  tokens split over several chunks
//   k_bwd_scan     (one CTA) CSR offsets and the chunk table: each token's kept
//                  list cut into chunks of BW_CH pairs
//   k_bwd_token    persistent: CTAs take chunks from a counter; per chunk
//                  the token's x and dy rows in shared memory, the chunk's
//                  neurons listed, warp = neuron: g, u, dh (three row dot
//                  products), then du, dg, h per pair (stored in CSR order)
//                  and du·W_up[j] + dg·W_gate[j] into the warp's dx row;
//                  the warps' rows summed into dx (added when the token has
//                  several chunks)
//   k_bwd_colcount thread = (chunk of 64 tokens, neuron): pairs counted;
//                  k_bwd_scan2 turns the counts into offsets
//   k_bwd_colfill  thread = (chunk, neuron): the CSR positions of its pairs
//   k_bwd_neuron   CTA = neuron: dW_gate, dW_up and dW_down rows and db
//                  from its pairs (x and dy rows gathered), no atomics
#pragma once

#include "epilogues.cuh"
#include "ptx.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"

namespace sffn {

constexpr int BW_THREADS = 256;
constexpr int BW_CH = 256;           // kept pairs per chunk of the token pass

struct BwdArgs {
  const __nv_bfloat16* x;       // [T][d]
  const float* dy;              // [T][d]
  const __nv_bfloat16* W_gate;  // [F][d]
  const __nv_bfloat16* W_up;    // [F][d]
  const __nv_bfloat16* W_down;  // [F][d]
  const float* bias;            // [F] or null
  const uint32_t* kmask;        // [T][n_words]
  int T, d, F, n_words;         // n_words = F / 32
  int act;
  int* wordpre;                 // [T][n_words] exclusive rank prefix within the token
  int* nnz;                     // [T]
  int* rowptr;                  // [T + 1]
  int2* chunks;                 // [max_chunks] (token, first rank)
  int* n_chunks;                // [1]
  int* counter;                 // [1] chunk counter of k_bwd_token
  float* du;                    // [pairs]
  float* dg;                    // [pairs]
  float* hv;                    // [pairs]
  int* colcnt;                  // [T / BW_TCH][F] pairs per (token chunk, neuron), then their offsets
  int* colptr;                  // [F + 1]
  int* cscpos;                  // [pairs] CSR position of the pair
  int* csctok;                  // [pairs] its token
  float* dx;                    // [T][d]
  float* dW_gate;               // [F][d]
  float* dW_up;                 // [F][d]
  float* dW_down;               // [F][d]
  float* db;                    // [F] or null
  // hybrid routing: the forward's overflow tokens ("heavy") take the dense
  // tensor-core channel instead of the sparse passes
  const uint32_t* ovf;          // [T] overflow epochs of the forward
  uint32_t epoch;               // the forward's epoch
  int* heavy;                   // [T] 1 for a heavy token
  int* hlist;                   // [T] heavy tokens in token order
  int* n_heavy;                 // [1]
  float* dbh;                   // [F] heavy tokens' d_bias contributions (added by the neuron pass)
};

// Exclusive scan of a[0..n) into out[0..n], out[n] = total (one CTA of 1024).
__device__ __forceinline__ void cta_scan_excl(const int* a, int n, int* out, int* tmp) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per, i1 = min(n, i0 + per);
  int s = 0;
  for (int i = i0; i < i1; ++i) s += a[i];
  int tot;
  int run = block_scan_excl(s, tmp, &tot);
  for (int i = i0; i < i1; ++i) {
    const int v = a[i];
    out[i] = run;
    run += v;
  }
  if (threadIdx.x == 0) out[n] = tot;
}

__global__ void __launch_bounds__(BW_THREADS) k_bwd_rows(const BwdArgs a) {
  __shared__ int tmp[33];
  griddep_wait();
  const int t = blockIdx.x;
  const uint32_t* km = a.kmask + (size_t)t * a.n_words;
  const int per = (a.n_words + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per, w1 = min(a.n_words, w0 + per);
  int s = 0;
  for (int w = w0; w < w1; ++w) s += __popc(km[w]);
  int tot;
  int run = block_scan_excl(s, tmp, &tot);
  for (int w = w0; w < w1; ++w) {
    a.wordpre[(size_t)t * a.n_words + w] = run;
    run += __popc(km[w]);
  }
  const bool hv = a.ovf && a.ovf[t] == a.epoch;
  if (threadIdx.x == 0) {
    a.nnz[t] = hv ? 0 : tot;   // a heavy token's pairs go to the dense channel
    if (a.heavy) a.heavy[t] = hv ? 1 : 0;
  }
  if (!hv && tot > BW_CH)    // several chunks add into dx
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) a.dx[(size_t)t * a.d + i] = 0.0f;
}

__global__ void __launch_bounds__(1024) k_bwd_scan(const BwdArgs a) {
  __shared__ int tmp[33];
  griddep_wait();
  cta_scan_excl(a.nnz, a.T, a.rowptr, tmp);
  __syncthreads();
  // chunk table: token t owns ceil(nnz_t / BW_CH) chunks (at least one, so
  // that a token that keeps nothing still gets dx = 0)
  const int per = (a.T + blockDim.x - 1) / blockDim.x;
  const int t0 = threadIdx.x * per, t1 = min(a.T, t0 + per);
  auto is_heavy = [&](int t) { return a.heavy && a.heavy[t]; };
  int s = 0;
  for (int t = t0; t < t1; ++t) s += is_heavy(t) ? 0 : max(1, (a.nnz[t] + BW_CH - 1) / BW_CH);
  int tot;
  int run = block_scan_excl(s, tmp, &tot);
  for (int t = t0; t < t1; ++t) {
    const int nc = is_heavy(t) ? 0 : max(1, (a.nnz[t] + BW_CH - 1) / BW_CH);
    for (int c = 0; c < nc; ++c) a.chunks[run + c] = make_int2(t, c * BW_CH);
    run += nc;
  }
  __syncthreads();
  if (a.hlist) {   // the heavy tokens in token order
    int hs = 0;
    for (int t = t0; t < t1; ++t) hs += is_heavy(t) ? 1 : 0;
    int htot;
    int hr = block_scan_excl(hs, tmp, &htot);
    for (int t = t0; t < t1; ++t)
      if (is_heavy(t)) a.hlist[hr++] = t;
    if (threadIdx.x == 0) *a.n_heavy = htot;
  }
  if (threadIdx.x == 0) {
    *a.n_chunks = tot;
    *a.counter = 0;
  }
}

// x and dy of the chunk's token, the chunk's neurons, per-warp dx rows
struct BwdTokenSmem {
  int x, dy, list, dxw, total;
  __host__ __device__ static BwdTokenSmem make(int d) {
    BwdTokenSmem s;
    int o = 0;
    s.x = o;    o += d * 2;
    s.dy = o;   o += d * 4;
    s.list = o; o += BW_CH * 4;
    s.dxw = o;  o += (BW_THREADS / 32) * d * 4;
    s.total = o + 16;
    return s;
  }
};

__global__ void __launch_bounds__(BW_THREADS) k_bwd_token(const BwdArgs a) {
  extern __shared__ __align__(16) uint8_t bw_s[];
  const BwdTokenSmem L = BwdTokenSmem::make(a.d);
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(bw_s + L.x);
  float* dys = reinterpret_cast<float*>(bw_s + L.dy);
  int* list = reinterpret_cast<int*>(bw_s + L.list);
  float* dxw = reinterpret_cast<float*>(bw_s + L.dxw);
  __shared__ int s_chunk;
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = BW_THREADS / 32;
  const int dv = a.d / 8;
  const int nch = *a.n_chunks;
  int cur_t = -1;
  for (;;) {
    __syncthreads();
    if (threadIdx.x == 0) s_chunk = atomicAdd(a.counter, 1);
    __syncthreads();
    const int c = s_chunk;
    if (c >= nch) break;
    const int2 ch = a.chunks[c];
    const int t = ch.x, r0 = ch.y;
    const int nz = a.nnz[t];
    const int n = min(BW_CH, nz - r0);
    if (t != cur_t) {   // stage the token's x and dy rows
      for (int v = threadIdx.x; v < dv; v += blockDim.x) {
        reinterpret_cast<uint4*>(xs)[v] = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d)[v];
        reinterpret_cast<float4*>(dys)[2 * v] = reinterpret_cast<const float4*>(a.dy + (size_t)t * a.d)[2 * v];
        reinterpret_cast<float4*>(dys)[2 * v + 1] =
            reinterpret_cast<const float4*>(a.dy + (size_t)t * a.d)[2 * v + 1];
      }
      cur_t = t;
    }
    // the chunk's neurons: the kept ones of rank r0 .. r0 + n - 1
    const uint32_t* km = a.kmask + (size_t)t * a.n_words;
    const int* wp = a.wordpre + (size_t)t * a.n_words;
    for (int w = threadIdx.x; w < a.n_words; w += blockDim.x) {
      uint32_t m = km[w];
      int rk = wp[w];
      if (rk >= r0 + n || rk + __popc(m) <= r0) continue;
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        if (rk >= r0 && rk < r0 + n) list[rk - r0] = w * 32 + b;
        ++rk;
      }
    }
    for (int i = threadIdx.x; i < nwarp * a.d; i += blockDim.x) dxw[i] = 0.0f;
    __syncthreads();
    float* myacc = dxw + warp * a.d;
    constexpr int PB = 8;   // 16-byte pieces per lane loaded at once (d <= 2048 in one batch)
    for (int q = warp; q < n; q += nwarp) {
      const int j = list[q];
      const uint4* rg = reinterpret_cast<const uint4*>(a.W_gate + (size_t)j * a.d);
      const uint4* ru = reinterpret_cast<const uint4*>(a.W_up + (size_t)j * a.d);
      const uint4* rd = reinterpret_cast<const uint4*>(a.W_down + (size_t)j * a.d);
      float sg = 0.f, su = 0.f, sd = 0.f;
      uint4 pg[PB], pu[PB];
      for (int vb = 0; vb < dv; vb += 32 * PB) {
        uint4 pd[PB];
#pragma unroll
        for (int i = 0; i < PB; ++i) {   // every piece's loads go out before the first use
          const int v = vb + lane + 32 * i;
          const bool in = v < dv;
          pg[i] = in ? __ldg(rg + v) : make_uint4(0, 0, 0, 0);
          pu[i] = in ? __ldg(ru + v) : make_uint4(0, 0, 0, 0);
          pd[i] = in ? __ldg(rd + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < PB; ++i) {
          const int v = vb + lane + 32 * i;
          if (v >= dv) break;
          const uint4 px = reinterpret_cast<const uint4*>(xs)[v];
          const float4 y0 = reinterpret_cast<const float4*>(dys)[2 * v];
          const float4 y1 = reinterpret_cast<const float4*>(dys)[2 * v + 1];
          const float yy[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
          const uint32_t gg[4] = {pg[i].x, pg[i].y, pg[i].z, pg[i].w}, uu[4] = {pu[i].x, pu[i].y, pu[i].z, pu[i].w};
          const uint32_t dd[4] = {pd[i].x, pd[i].y, pd[i].z, pd[i].w}, xx[4] = {px.x, px.y, px.z, px.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xx[e]));
            const float2 fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gg[e]));
            const float2 fu = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uu[e]));
            const float2 fd = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dd[e]));
            sg += fg.x * fx.x + fg.y * fx.y;
            su += fu.x * fx.x + fu.y * fx.y;
            sd += fd.x * yy[2 * e] + fd.y * yy[2 * e + 1];
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sg += __shfl_xor_sync(0xFFFFFFFFu, sg, o);
        su += __shfl_xor_sync(0xFFFFFFFFu, su, o);
        sd += __shfl_xor_sync(0xFFFFFFFFu, sd, o);
      }
      const float g = sg + (a.bias ? a.bias[j] : 0.0f);
      const float act = act_fn(g, a.act);
      const float v = __bfloat162float(__float2bfloat16_rn(act));
      // sigma'(g): 1 for ReLU on a kept neuron (the forward kept it, so g >
      // threshold >= 0), s(1 + g(1 - s)) for SiLU
      float slope = 1.0f;
      if (a.act == ACT_SILU) {
        const float sgm = 1.0f / (1.0f + expf(-g));
        slope = sgm * (1.0f + g * (1.0f - sgm));
      }
      const float du = sd * v, dg = sd * su * slope;
      if (lane == 0) {
        const int pos = a.rowptr[t] + r0 + q;
        a.du[pos] = du;
        a.dg[pos] = dg;
        a.hv[pos] = v * su;
      }
      // dx row of this warp: du·W_up[j] + dg·W_gate[j]; the last batch's
      // pieces are still in registers, earlier batches (d > 2048) reload
      for (int vb = 0; vb < dv; vb += 32 * PB) {
        const bool last = vb + 32 * PB >= dv;
#pragma unroll
        for (int i = 0; i < PB; ++i) {
          const int v8 = vb + lane + 32 * i;
          if (v8 >= dv) break;
          const uint4 qu = last ? pu[i] : __ldg(ru + v8), qg = last ? pg[i] : __ldg(rg + v8);
          const uint32_t uu[4] = {qu.x, qu.y, qu.z, qu.w}, gg[4] = {qg.x, qg.y, qg.z, qg.w};
          float4* acc = reinterpret_cast<float4*>(myacc + 8 * v8);
          float4 a0 = acc[0], a1 = acc[1];
          float r[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fu = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uu[e]));
            const float2 fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gg[e]));
            r[2 * e] = du * fu.x + dg * fg.x;
            r[2 * e + 1] = du * fu.y + dg * fg.y;
          }
          a0.x += r[0]; a0.y += r[1]; a0.z += r[2]; a0.w += r[3];
          a1.x += r[4]; a1.y += r[5]; a1.z += r[6]; a1.w += r[7];
          acc[0] = a0;
          acc[1] = a1;
        }
      }
    }
    __syncthreads();
    const bool split = nz > BW_CH;
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) {
      float s = 0.0f;
      for (int w = 0; w < nwarp; ++w) s += dxw[w * a.d + i];
      float* dst = a.dx + (size_t)t * a.d + i;
      if (split)
        atomicAdd(dst, s);
      else
        *dst = s;
    }
  }
}

// The column index, in parallel over (token chunk, neuron): thread = one
// neuron over BW_TCH consecutive tokens.  k_bwd_colcount writes the count
// of each (chunk, neuron); k_bwd_scan2 turns them into offsets (chunks in
// token order inside each neuron, neurons one after another); k_bwd_colfill
// writes each chunk's pairs at its offset, so every neuron's list is in token
// order, the same on every run (k_bwd_colprefix and k_bwd_scan2 between them).
constexpr int BW_TCH = 64;

__global__ void k_bwd_colcount(const BwdArgs a) {
  griddep_wait();
  const int j = blockIdx.x * blockDim.x + threadIdx.x, tc = blockIdx.y;
  if (j >= a.F) return;
  const int w = j >> 5;
  const uint32_t bit = 1u << (j & 31);
  const int t0 = tc * BW_TCH, t1 = min(a.T, t0 + BW_TCH);
  int c = 0;
  for (int t = t0; t < t1; ++t)
    c += (!(a.heavy && a.heavy[t]) && (__ldg(a.kmask + (size_t)t * a.n_words + w) & bit)) ? 1 : 0;
  a.colcnt[(size_t)tc * a.F + j] = c;
}

// per neuron (thread): its chunks' counts turned into exclusive prefixes in
// place, the total into colptr[j]
__global__ void k_bwd_colprefix(const BwdArgs a) {
  griddep_wait();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= a.F) return;
  const int nch = (a.T + BW_TCH - 1) / BW_TCH;
  int run = 0;
  for (int c = 0; c < nch; ++c) {
    const int v = a.colcnt[(size_t)c * a.F + j];
    a.colcnt[(size_t)c * a.F + j] = run;
    run += v;
  }
  a.colptr[j] = run;
}

// colptr: exclusive scan of the neurons' totals, in place (one CTA)
__global__ void __launch_bounds__(1024) k_bwd_scan2(const BwdArgs a) {
  __shared__ int tmp[33];
  griddep_wait();
  const int per = (a.F + blockDim.x - 1) / blockDim.x;
  const int i0 = threadIdx.x * per, i1 = min(a.F, i0 + per);
  int sum = 0;
  for (int i = i0; i < i1; ++i) sum += a.colptr[i];
  int tot;
  int run = block_scan_excl(sum, tmp, &tot);
  for (int i = i0; i < i1; ++i) {
    const int v = a.colptr[i];
    a.colptr[i] = run;
    run += v;
  }
  if (threadIdx.x == 0) a.colptr[a.F] = tot;
}

__global__ void k_bwd_colfill(const BwdArgs a) {
  griddep_wait();
  const int j = blockIdx.x * blockDim.x + threadIdx.x, tc = blockIdx.y;
  if (j >= a.F) return;
  const int w = j >> 5, b = j & 31;
  const uint32_t bit = 1u << b, below = bit - 1u;
  const int t0 = tc * BW_TCH, t1 = min(a.T, t0 + BW_TCH);
  int k = a.colptr[j] + a.colcnt[(size_t)tc * a.F + j];
  for (int t = t0; t < t1; ++t) {
    const uint32_t m = __ldg(a.kmask + (size_t)t * a.n_words + w);
    if ((m & bit) && !(a.heavy && a.heavy[t])) {
      a.cscpos[k] = a.rowptr[t] + a.wordpre[(size_t)t * a.n_words + w] + __popc(m & below);
      a.csctok[k] = t;
      ++k;
    }
  }
}

// dW rows of neuron j (blockIdx.x): its pairs' tokens and values staged in
// shared memory BW_NB at a time, then thread = 8 consecutive columns per
// 16-byte piece (d / 8 pieces over the CTA), BW_PB pairs' x and dy pieces
// loaded before use (two CTAs per SM).
constexpr int BW_NB = 256;
constexpr int BW_PB = 4;   // pairs whose x and dy pieces are loaded at once

template <int MAXV>   // 16-byte pieces per thread: d <= MAXV x 8 x 256
__global__ void __launch_bounds__(BW_THREADS, 2) k_bwd_neuron(const BwdArgs a) {
  __shared__ int s_tok[BW_NB];
  __shared__ float s_du[BW_NB], s_dg[BW_NB], s_h[BW_NB];
  __shared__ float s_red[BW_THREADS / 32];
  griddep_wait();
  const int j = blockIdx.x;
  const int p0 = a.colptr[j], p1 = a.colptr[j + 1];
  const int dv = a.d / 8;
  float ag[MAXV][8], au[MAXV][8], ad[MAXV][8];
#pragma unroll
  for (int m = 0; m < MAXV; ++m)
#pragma unroll
    for (int e = 0; e < 8; ++e) ag[m][e] = au[m][e] = ad[m][e] = 0.0f;
  float dbs = 0.0f;
  for (int pb = p0; pb < p1; pb += BW_NB) {
    const int nb = min(BW_NB, p1 - pb);
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
      const int pos = a.cscpos[pb + i];
      s_tok[i] = a.csctok[pb + i];
      s_du[i] = a.du[pos];
      s_dg[i] = a.dg[pos];
      s_h[i] = a.hv[pos];
      dbs += a.dg[pos];
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
      const int v = threadIdx.x + m * BW_THREADS;
      if (v >= dv) break;
      for (int i0 = 0; i0 < nb; i0 += BW_PB) {
        uint4 xq[BW_PB];
        float4 y0[BW_PB], y1[BW_PB];
#pragma unroll
        for (int q = 0; q < BW_PB; ++q) {
          if (i0 + q < nb) {
            const int t = s_tok[i0 + q];
            xq[q] = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d) + v);
            y0[q] = __ldg(reinterpret_cast<const float4*>(a.dy + (size_t)t * a.d) + 2 * v);
            y1[q] = __ldg(reinterpret_cast<const float4*>(a.dy + (size_t)t * a.d) + 2 * v + 1);
          } else {
            xq[q] = make_uint4(0, 0, 0, 0);
            y0[q] = y1[q] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int q = 0; q < BW_PB; ++q) {
          const float cu = i0 + q < nb ? s_du[i0 + q] : 0.0f;
          const float cg = i0 + q < nb ? s_dg[i0 + q] : 0.0f;
          const float ch = i0 + q < nb ? s_h[i0 + q] : 0.0f;
          const uint32_t xx[4] = {xq[q].x, xq[q].y, xq[q].z, xq[q].w};
          const float yy[8] = {y0[q].x, y0[q].y, y0[q].z, y0[q].w, y1[q].x, y1[q].y, y1[q].z, y1[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xx[e]));
            ag[m][2 * e] += cg * fx.x;
            ag[m][2 * e + 1] += cg * fx.y;
            au[m][2 * e] += cu * fx.x;
            au[m][2 * e + 1] += cu * fx.y;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) ad[m][e] += ch * yy[e];
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MAXV; ++m) {
    const int v = threadIdx.x + m * BW_THREADS;
    if (v >= dv) break;
    float4* og = reinterpret_cast<float4*>(a.dW_gate + (size_t)j * a.d) + 2 * v;
    float4* ou = reinterpret_cast<float4*>(a.dW_up + (size_t)j * a.d) + 2 * v;
    float4* od = reinterpret_cast<float4*>(a.dW_down + (size_t)j * a.d) + 2 * v;
    og[0] = make_float4(ag[m][0], ag[m][1], ag[m][2], ag[m][3]);
    og[1] = make_float4(ag[m][4], ag[m][5], ag[m][6], ag[m][7]);
    ou[0] = make_float4(au[m][0], au[m][1], au[m][2], au[m][3]);
    ou[1] = make_float4(au[m][4], au[m][5], au[m][6], au[m][7]);
    od[0] = make_float4(ad[m][0], ad[m][1], ad[m][2], ad[m][3]);
    od[1] = make_float4(ad[m][4], ad[m][5], ad[m][6], ad[m][7]);
  }
  if (a.db) {   // d_bias[j] = sum of dg over the pairs, in pair order within each thread's share
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dbs += __shfl_xor_sync(0xFFFFFFFFu, dbs, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = dbs;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.0f;
      for (int w = 0; w < BW_THREADS / 32; ++w) s += s_red[w];
      a.db[j] = s + (a.dbh ? a.dbh[j] : 0.0f);
    }
  }
}

// ------------------------------------------------ dense channel (heavy tokens)
// Heavy token o (hlist[o]) in the dense buffers; NP = max_tokens rounded up
// to 64 (the K padding of the GEMMs over tokens).
struct HeavyPrepArgs {
  const __nv_bfloat16* x;       // [T][d]
  const float* dy;              // [T][d]
  const int* hlist;
  const int* n_heavy;
  __nv_bfloat16* xh;            // [NP][d]   x rows of the heavy tokens
  __nv_bfloat16* dyh_hi;        // [NP][d]   dy rows, split hi + lo
  __nv_bfloat16* dyh_lo;
  __nv_bfloat16* xhT;           // [d][NP]   transposed, zero past n_heavy up to a multiple of 64
  __nv_bfloat16* dyhT_hi;       // [d][NP]
  __nv_bfloat16* dyhT_lo;
  float* dbh;                   // [F] zeroed here
  int d, F, NP;
};

// grid (d / 32, NP / 32), block (32, 8): a 32 x 32 tile of (heavy token,
// column), read by token rows and written transposed through shared memory
__global__ void k_bwd_heavy_prep(const HeavyPrepArgs a) {
  __shared__ float tx[32][33], ty[32][33];
  griddep_wait();
  const int nh = *a.n_heavy;
  const int npad = (nh + 63) & ~63;
  const int i0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int j = threadIdx.y * 32 + threadIdx.x; j < a.F; j += 256) a.dbh[j] = 0.0f;
  if (o0 >= npad) return;
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int o = o0 + r, i = i0 + threadIdx.x;
    float xv = 0.f, yv = 0.f;
    if (o < nh && i < a.d) {
      const int t = a.hlist[o];
      xv = __bfloat162float(a.x[(size_t)t * a.d + i]);
      yv = a.dy[(size_t)t * a.d + i];
      const __nv_bfloat16 yh = __float2bfloat16_rn(yv);
      a.xh[(size_t)o * a.d + i] = a.x[(size_t)t * a.d + i];
      a.dyh_hi[(size_t)o * a.d + i] = yh;
      a.dyh_lo[(size_t)o * a.d + i] = __float2bfloat16_rn(yv - __bfloat162float(yh));
    }
    tx[r][threadIdx.x] = xv;
    ty[r][threadIdx.x] = yv;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int i = i0 + r, o = o0 + threadIdx.x;
    if (i < a.d && o < npad) {
      const float yv = ty[threadIdx.x][r];
      const __nv_bfloat16 yh = __float2bfloat16_rn(yv);
      a.xhT[(size_t)i * a.NP + o] = __float2bfloat16_rn(tx[threadIdx.x][r]);
      a.dyhT_hi[(size_t)i * a.NP + o] = yh;
      a.dyhT_lo[(size_t)i * a.NP + o] = __float2bfloat16_rn(yv - __bfloat162float(yh));
    }
  }
}

// g and u of the heavy tokens, every neuron: two accumulators (W_gate, then
// W_up, against the heavy x rows); stored fp32 [NP][F]
struct GuParams {
  float* g;
  float* u;
  const int* n_rows_dev;
  int F;
};

struct EpiStoreGU {
  static constexpr int N_ACC = 2;
  using Params = GuParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int n = *o.n_rows_dev, j = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= n) break;
      float g[16], u[16];
      tmem_ld16(tmem + c, g);
      tmem_ld16(tmem + BN + c, u);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = n0 + c + i;
        if (r < n) {
          o.g[(size_t)r * o.F + j] = g[i];
          o.u[(size_t)r * o.F + j] = u[i];
        }
      }
    }
  }
};

// dh = dy W_down^T for the heavy tokens (dy split hi + lo, one accumulator);
// the epilogue forms the pair values: with the keep bit of the forward,
// v = bf16(sigma(g + b)), du = dh·v, dg = dh·u·sigma'(g), h = v·u (zero where
// not kept).  Written hi + lo: token-major [NP][F] (du, dg: the dx GEMMs'
// B operands) and neuron-major [F][NP] (du, dg, h: the dW GEMMs' A operands,
// zero in the K padding past the last heavy token).  d_bias sums go to dbh.
struct BwdDhParams {
  const float* g;
  const float* u;
  const float* bias;
  const uint32_t* kmask;
  int n_words;
  const int* hlist;
  const int* n_rows_dev;
  int F, NP, act;
  __nv_bfloat16 *du_hi, *du_lo, *dg_hi, *dg_lo;          // [NP][F]
  __nv_bfloat16 *duT_hi, *duT_lo, *dgT_hi, *dgT_lo;      // [F][NP]
  __nv_bfloat16 *hT_hi, *hT_lo;                          // [F][NP]
  float* dbh;                                            // [F]
};

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

struct EpiBwdDh {
  static constexpr int N_ACC = 1;
  static constexpr bool DUAL_B = true;   // dy hi + lo
  using Params = BwdDhParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int n = *o.n_rows_dev, npad = (n + 63) & ~63, j = m0 + etid;
    const float b = o.bias ? o.bias[j] : 0.0f;
    const int w = j >> 5;
    const uint32_t bit = 1u << (j & 31);
    float dbs = 0.0f;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= npad) break;
      float dh[16];
      tmem_ld16(tmem + c, dh);
      __align__(16) __nv_bfloat16 Tdu_h[16], Tdu_l[16], Tdg_h[16], Tdg_l[16], Th_h[16], Th_l[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = n0 + c + i;
        float du = 0.f, dg = 0.f, hv = 0.f;
        if (r < n) {
          const int t = o.hlist[r];
          if (o.kmask[(size_t)t * o.n_words + w] & bit) {
            const float gg = o.g[(size_t)r * o.F + j] + b;
            const float uu = o.u[(size_t)r * o.F + j];
            const float v = __bfloat162float(__float2bfloat16_rn(act_fn(gg, o.act)));
            float slope = 1.0f;
            if (o.act == ACT_SILU) {
              const float sg = 1.0f / (1.0f + expf(-gg));
              slope = sg * (1.0f + gg * (1.0f - sg));
            }
            du = dh[i] * v;
            dg = dh[i] * uu * slope;
            hv = v * uu;
          }
          __nv_bfloat16 hi, lo;
          split_bf16(du, hi, lo);
          o.du_hi[(size_t)r * o.F + j] = hi;
          o.du_lo[(size_t)r * o.F + j] = lo;
          split_bf16(dg, hi, lo);
          o.dg_hi[(size_t)r * o.F + j] = hi;
          o.dg_lo[(size_t)r * o.F + j] = lo;
          dbs += dg;
        }
        split_bf16(du, Tdu_h[i], Tdu_l[i]);
        split_bf16(dg, Tdg_h[i], Tdg_l[i]);
        split_bf16(hv, Th_h[i], Th_l[i]);
      }
      // neuron-major: 16 consecutive tokens of row j, two 16-byte stores each
      const size_t off = (size_t)j * o.NP + n0 + c;
      __nv_bfloat16* dst[6] = {o.duT_hi, o.duT_lo, o.dgT_hi, o.dgT_lo, o.hT_hi, o.hT_lo};
      const __nv_bfloat16* src[6] = {Tdu_h, Tdu_l, Tdg_h, Tdg_l, Th_h, Th_l};
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        reinterpret_cast<uint4*>(dst[q] + off)[0] = reinterpret_cast<const uint4*>(src[q])[0];
        reinterpret_cast<uint4*>(dst[q] + off)[1] = reinterpret_cast<const uint4*>(src[q])[1];
      }
    }
    if (dbs != 0.0f) atomicAdd(&o.dbh[j], dbs);
  }
};

// D[rows][cols] added into dst (fp32, row-major, ld), rows below `rows` and
// columns below `cols`: the heavy tokens' share of dW_gate, dW_up, dW_down
struct AddParams {
  float* dst;
  long long ld;
  int rows, cols;
};

template <bool DUAL>
struct EpiAddF32T {
  static constexpr int N_ACC = 1;
  static constexpr bool DUAL_B = DUAL;     // B split hi + lo ...
  static constexpr bool DUAL_ALL = DUAL;   // ... in both phases (A hi, then A lo)
  using Params = AddParams;
  template <int BN>
  __device__ static void run(const Params& o, uint32_t tmem, int m0, int n0, int, int etid, uint8_t*) {
    const int r = m0 + etid;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      if (n0 + c >= o.cols) break;
      float v[16];
      tmem_ld16(tmem + c, v);
      if (r < o.rows) {
        float* dst = o.dst + (size_t)r * o.ld + n0 + c;
        if (n0 + c + 16 <= o.cols) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float4 p = reinterpret_cast<float4*>(dst)[q];
            p.x += v[4 * q];
            p.y += v[4 * q + 1];
            p.z += v[4 * q + 2];
            p.w += v[4 * q + 3];
            reinterpret_cast<float4*>(dst)[q] = p;
          }
        } else {
          for (int i = 0; i < 16 && n0 + c + i < o.cols; ++i) dst[i] += v[i];
        }
      }
    }
  }
};
using EpiAddF32 = EpiAddF32T<false>;
using EpiAddF32Dual = EpiAddF32T<true>;

}  // namespace sffn
