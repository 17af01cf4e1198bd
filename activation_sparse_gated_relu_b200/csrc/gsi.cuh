// Gated subspace linear layer ("Gated Subspace Inference for Transformer
// Acceleration", sections 2.1 and 2.2): for y = W x with W [d_out][d_in] and
// an orthonormal basis V_k [d_in][k] of the activation subspace,
//     g = V_k^T x,  r = x - V_k g,  M = W V_k (cached at create time),
// and per token y = M·bf16(g) when ||r||^2 < eps^2 ||x||^2 (fast path: only
// the d_out x k image is read), y = W x otherwise (slow path).
//
// Decode batches (a few tokens) make every step a matrix-vector stream, bound
// by HBM: each kernel gives whole rows to warps, loads them as 16-byte
// vectors several rows (or several pieces of a row) ahead, keeps the tokens'
// operands in shared memory and reduces each row's dot products with warp
// shuffles.  Three launches (programmatic dependent launch between them):
//   k_gsi_project  g[t][j] = <V_k^T[j], x_t> for the k basis rows; zeroes the
//                  norm accumulators
//   k_gsi_resid    r_t[i] = x_t[i] - <V_k[i], g_t> for the d_in rows of V_k;
//                  sum_i r_t[i]^2 and sum_i x_t[i]^2 per token (atomics)
//   k_gsi_out      per token route, then y[t][o] = <M[o], bf16(g_t)> (fast)
//                  or <W[o], x_t> (slow) for the d_out rows
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int GSI_TC = 8;          // tokens per chunk in shared memory
constexpr int GSI_THREADS = 512;   // 16 warps

struct GsiArgs {
  const __nv_bfloat16* x;      // [T][d_in]
  const __nv_bfloat16* Vkt;    // [k][d_in]
  const __nv_bfloat16* Vk;     // [d_in][k]
  const __nv_bfloat16* M;      // [d_out][k]
  const __nv_bfloat16* W;      // [d_out][d_in]
  float* g;                    // [T][k] fp32
  float* rn2;                  // [T] sum of r^2
  float* xn2;                  // [T] sum of x^2
  int* n_slow;                 // [1] slow tokens of the forward (written by k_gsi_out's CTA 0)
  float* y;                    // [T][d_out]
  int T, d_in, d_out, k;
  float eps2;                  // eps^2 (fp32)
};

__device__ __forceinline__ float bf16x2_dot(uint32_t a, uint32_t b) {
  const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
  const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b));
  return fa.x * fb.x + fa.y * fb.y;
}

__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
  return bf16x2_dot(a.x, b.x) + bf16x2_dot(a.y, b.y) + bf16x2_dot(a.z, b.z) + bf16x2_dot(a.w, b.w);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// g = V_k^T x: one warp per basis row j (d_in elements), the chunk's tokens'
// x rows in shared memory; the lane's 16-byte pieces of the row go out four
// ahead of their use.
__global__ void __launch_bounds__(GSI_THREADS) k_gsi_project(const GsiArgs a) {
  extern __shared__ uint4 gsi_xs[];   // [GSI_TC][d_in / 8]
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dv = a.d_in / 8;
  if (blockIdx.x == 0)
    for (int t = threadIdx.x; t < a.T; t += blockDim.x) {
      a.rn2[t] = 0.0f;
      a.xn2[t] = 0.0f;
    }
  const int nw = gridDim.x * (GSI_THREADS / 32), gw = blockIdx.x * (GSI_THREADS / 32) + warp;
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    __syncthreads();
    for (int e = threadIdx.x; e < nt * dv; e += blockDim.x)
      gsi_xs[e] = reinterpret_cast<const uint4*>(a.x)[(size_t)t0 * dv + e];
    __syncthreads();
    for (int j = gw; j < a.k; j += nw) {
      const uint4* row = reinterpret_cast<const uint4*>(a.Vkt) + (size_t)j * dv;
      float acc[GSI_TC];
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) acc[i] = 0.0f;
      for (int v0 = lane; v0 < dv; v0 += 32 * 4) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = v0 + 32 * u < dv ? __ldg(row + v0 + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (v0 + 32 * u >= dv) break;
#pragma unroll
          for (int i = 0; i < GSI_TC; ++i)
            if (i < nt) acc[i] += dot8(w[u], gsi_xs[i * dv + v0 + 32 * u]);
        }
      }
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) {
        if (i >= nt) break;
        const float s = warp_sum(acc[i]);
        if (lane == 0) a.g[(size_t)(t0 + i) * a.k + j] = s;
      }
    }
  }
}

// r = x - V_k g and the two squared norms: one warp per row i of V_k (k
// elements, k / 8 16-byte pieces spread over the lanes), g of the chunk's
// tokens in shared memory; each warp keeps its tokens' partial sums in
// registers and adds them once into rn2 / xn2.
__global__ void __launch_bounds__(GSI_THREADS) k_gsi_resid(const GsiArgs a) {
  extern __shared__ float gsi_gs[];   // [GSI_TC][k]
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kv = a.k / 8;
  const int nw = gridDim.x * (GSI_THREADS / 32), gw = blockIdx.x * (GSI_THREADS / 32) + warp;
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    __syncthreads();
    for (int e = threadIdx.x; e < nt * a.k; e += blockDim.x) gsi_gs[e] = a.g[(size_t)t0 * a.k + e];
    __syncthreads();
    float r2[GSI_TC], x2[GSI_TC];
#pragma unroll
    for (int i = 0; i < GSI_TC; ++i) r2[i] = x2[i] = 0.0f;
    for (int row = gw; row < a.d_in; row += nw) {
      const uint4* vr = reinterpret_cast<const uint4*>(a.Vk) + (size_t)row * kv;
      float acc[GSI_TC];
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) acc[i] = 0.0f;
      for (int v = lane; v < kv; v += 32) {
        const uint4 w = __ldg(vr + v);
        const uint32_t wp[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wp[q]));
#pragma unroll
          for (int i = 0; i < GSI_TC; ++i)
            if (i < nt) {
              const float* gi = gsi_gs + i * a.k + 8 * v + 2 * q;
              acc[i] += f.x * gi[0] + f.y * gi[1];
            }
        }
      }
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) {
        if (i >= nt) break;
        const float s = warp_sum(acc[i]);
        const float xv = __bfloat162float(a.x[(size_t)(t0 + i) * a.d_in + row]);
        const float rv = xv - s;
        r2[i] += rv * rv;
        x2[i] += xv * xv;
      }
    }
    if (lane == 0)
      for (int i = 0; i < nt; ++i) {
        atomicAdd(&a.rn2[t0 + i], r2[i]);
        atomicAdd(&a.xn2[t0 + i], x2[i]);
      }
  }
}

// y: every CTA first decides each token's path (the same decision in every
// CTA: the norms are final once this kernel may read them), stages bf16(g) of
// the fast tokens and x of the slow tokens, then its warps take output rows:
// <M[o], bf16(g_t)> for fast tokens (k elements) and, only if some token is
// slow, <W[o], x_t> for slow tokens (d_in elements).
struct GsiOutSmem {
  int ghat, xs, flags, total;
  __host__ __device__ static GsiOutSmem make(int T, int k, int d_in) {
    GsiOutSmem s;
    int o = 0;
    s.ghat = o;  o += ((T * k * 2 + 15) & ~15);       // bf16 [T][k]
    s.xs = o;    o += GSI_TC * d_in * 2;              // bf16 [GSI_TC][d_in] (slow tokens, a chunk)
    s.flags = o; o += ((T * 4 + 15) & ~15) + 16;      // slow token list [T] and its count
    s.total = o;
    return s;
  }
};

__global__ void __launch_bounds__(GSI_THREADS) k_gsi_out(const GsiArgs a) {
  extern __shared__ __align__(16) uint8_t gsi_o[];
  const GsiOutSmem L = GsiOutSmem::make(a.T, a.k, a.d_in);
  __nv_bfloat16* ghat = reinterpret_cast<__nv_bfloat16*>(gsi_o + L.ghat);
  uint4* xs = reinterpret_cast<uint4*>(gsi_o + L.xs);
  int* slow = reinterpret_cast<int*>(gsi_o + L.flags);
  int* nslow = slow + a.T;
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int t = 0; t < a.T; ++t)
      if (!(a.rn2[t] < a.eps2 * a.xn2[t])) slow[n++] = t;
    *nslow = n;
    if (blockIdx.x == 0) *a.n_slow = n;
  }
  for (int e = threadIdx.x; e < a.T * a.k; e += blockDim.x) ghat[e] = __float2bfloat16_rn(a.g[e]);
  __syncthreads();
  const int ns = *nslow;
  const int kv = a.k / 8, dv = a.d_in / 8;
  const int nw = gridDim.x * (GSI_THREADS / 32), gw = blockIdx.x * (GSI_THREADS / 32) + warp;
  // fast path: tokens in chunks of GSI_TC; slow tokens' outputs are written
  // by the slow pass below
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    for (int o = gw; o < a.d_out; o += nw) {
      const uint4* mr = reinterpret_cast<const uint4*>(a.M) + (size_t)o * kv;
      float acc[GSI_TC];
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) acc[i] = 0.0f;
      for (int v = lane; v < kv; v += 32) {
        const uint4 w = __ldg(mr + v);
#pragma unroll
        for (int i = 0; i < GSI_TC; ++i)
          if (i < nt) acc[i] += dot8(w, reinterpret_cast<const uint4*>(ghat + (size_t)(t0 + i) * a.k)[v]);
      }
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) {
        if (i >= nt) break;
        const float s = warp_sum(acc[i]);
        if (lane == 0) a.y[(size_t)(t0 + i) * a.d_out + o] = s;
      }
    }
  }
  if (ns == 0) return;
  // slow path: chunks of the slow tokens, x rows staged, W rows streamed four
  // 16-byte pieces per lane ahead
  __syncwarp();
  for (int s0 = 0; s0 < ns; s0 += GSI_TC) {
    const int nt = min(GSI_TC, ns - s0);
    __syncthreads();
    for (int e = threadIdx.x; e < nt * dv; e += blockDim.x) {
      const int i = e / dv, v = e - i * dv;
      xs[e] = reinterpret_cast<const uint4*>(a.x)[(size_t)slow[s0 + i] * dv + v];
    }
    __syncthreads();
    for (int o = gw; o < a.d_out; o += nw) {
      const uint4* wr = reinterpret_cast<const uint4*>(a.W) + (size_t)o * dv;
      float acc[GSI_TC];
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) acc[i] = 0.0f;
      for (int v0 = lane; v0 < dv; v0 += 32 * 4) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = v0 + 32 * u < dv ? __ldg(wr + v0 + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (v0 + 32 * u >= dv) break;
#pragma unroll
          for (int i = 0; i < GSI_TC; ++i)
            if (i < nt) acc[i] += dot8(w[u], xs[i * dv + v0 + 32 * u]);
        }
      }
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) {
        if (i >= nt) break;
        const float s = warp_sum(acc[i]);
        if (lane == 0) a.y[(size_t)slow[s0 + i] * a.d_out + o] = s;
      }
    }
  }
}

}  // namespace sffn
