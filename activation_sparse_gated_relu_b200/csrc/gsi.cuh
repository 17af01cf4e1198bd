// Gated subspace linear layer ("Gated Subspace Inference for Transformer
// Acceleration", sections 2.1 and 2.2): for y = W x with W [d_out][d_in] and
// an orthonormal basis V_k [d_in][k] of the activation subspace,
//     g = V_k^T x,  r = x - V_k g,  M = W V_k (cached at create time),
// and per token y = M·bf16(g) when ||r||^2 < eps^2 ||x||^2 (fast path: only
// the d_out x k image is read), y = W x otherwise (slow path).
//
// Decode batches (a few tokens) make every step a matrix-vector stream, bound
// by HBM.  Every kernel hands each CTA a contiguous range of rows, so its
// loads are one sequential stream, and issues a whole batch of loads before
// using any.  Three launches (programmatic dependent launch between them):
//   k_gsi_project  rows i of V_k: thread = two basis columns j, partial sums
//                  of g[t][j] = sum_i V_k[i][j] x_t[i] over the CTA's rows,
//                  added into g (red.add; g is cleared by the previous
//                  forward's k_gsi_out, two buffers alternating)
//   k_gsi_resid    rows i of V_k: warp = row, lane = 8 basis columns;
//                  r_t[i] = x_t[i] - <V_k[i], g_t>; per-CTA sums of r^2 and
//                  x^2 per token written out (no atomics)
//   k_gsi_out      every CTA adds those partial norms and decides each
//                  token's path; rows o of M (and of W for slow tokens):
//                  y[t][o] = <M[o], bf16(g_t)> or <W[o], x_t>
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int GSI_TC = 8;          // tokens per chunk
constexpr int GSI_THREADS = 256;   // 8 warps
constexpr int GSI_ROWS = 6;        // rows a warp loads at once in k_gsi_out (register budget of 512 threads)
constexpr int GSI_OUT_THREADS = 512;   // 16 warps: a whole batch of rows in flight per SM

struct GsiArgs {
  const __nv_bfloat16* x;      // [T][d_in]
  const __nv_bfloat16* Vk;     // [d_in][k]
  const __nv_bfloat16* M;      // [d_out][k]
  const __nv_bfloat16* W;      // [d_out][d_in]
  float* g;                    // [T][k] fp32: summed into, zero on entry
  float* g_next;               // [T][k]: the buffer the next forward sums into (cleared here)
  float* part;                 // [grid_resid][maxT][2]: per-CTA sums of r^2 and x^2
  int* n_slow;                 // [1] slow tokens of the forward (written by k_gsi_out's CTA 0)
  float* y;                    // [T][d_out]
  int T, d_in, d_out, k;
  int maxT;                    // g_next is cleared for this many tokens
  int grid_resid;              // CTAs of k_gsi_resid (partials to add)
  float eps2;                  // eps^2 (fp32)
};

__device__ __forceinline__ float2 bf2(uint32_t a) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Sum of v[i] over the warp's lanes for 8 values at once, by halving
// exchanges (9 shuffles instead of 40): lane l returns the sum of v[(l >> 2) & 7].
__device__ __forceinline__ float warp_sum8(const float (&v)[8]) {
  const int lane = threadIdx.x & 31;
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float w[4], u[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? v[i] : v[i + 4];
    w[i] = (b4 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xFFFFFFFFu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? w[i] : w[i + 2];
    u[i] = (b3 ? w[i + 2] : w[i]) + __shfl_xor_sync(0xFFFFFFFFu, send, 8);
  }
  float s = (b2 ? u[1] : u[0]) + __shfl_xor_sync(0xFFFFFFFFu, b2 ? u[0] : u[1], 4);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 2);
  s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
  return s;
}

__device__ __forceinline__ void row_range(int rows, int& r0, int& r1) {
  r0 = (int)((long long)rows * blockIdx.x / gridDim.x);
  r1 = (int)((long long)rows * (blockIdx.x + 1) / gridDim.x);
}

// g partial sums: rows [r0, r1) of V_k (at most GSI_PROJ_ROWS per CTA).
// Thread = one column pair (2 c, 2 c + 1) of one row group: with k / 2 pairs
// per row, 256 / (k / 2) groups take interleaved rows, all of a thread's row
// loads go out before their use, the groups' sums meet in shared memory and
// the CTA adds its partial g into g (red.add).
constexpr int GSI_PROJ_ROWS = 32;

__global__ void __launch_bounds__(GSI_THREADS) k_gsi_project(const GsiArgs a) {
  __shared__ float xs[GSI_TC][GSI_PROJ_ROWS];
  extern __shared__ float gsi_red[];     // [groups][GSI_TC][k]
  griddep_wait();
  int r0, r1;
  row_range(a.d_in, r0, r1);
  const int nr = r1 - r0;
  const int cpr = a.k / 2, groups = GSI_THREADS / cpr;
  const int pair = threadIdx.x % cpr, grp = threadIdx.x / cpr;
  const bool own = grp < groups;
  const uint32_t* V = reinterpret_cast<const uint32_t*>(a.Vk) + (size_t)r0 * cpr + pair;   // bf16 pairs
  // this thread's rows: grp, grp + groups, ... < nr, at most GSI_PROJ_ROWS / 1
  constexpr int MAXQ = GSI_PROJ_ROWS;
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    __syncthreads();
    for (int e = threadIdx.x; e < GSI_TC * GSI_PROJ_ROWS; e += blockDim.x) {
      const int i = e / GSI_PROJ_ROWS, q = e % GSI_PROJ_ROWS;
      xs[i][q] = (i < nt && q < nr) ? __bfloat162float(a.x[(size_t)(t0 + i) * a.d_in + r0 + q]) : 0.0f;
    }
    __syncthreads();
    float acc[GSI_TC][2];
#pragma unroll
    for (int i = 0; i < GSI_TC; ++i) acc[i][0] = acc[i][1] = 0.0f;
    if (own) {
#pragma unroll 1
      for (int qb = grp; qb < nr; qb += 16 * groups) {
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int q = qb + u * groups;
          w[u] = q < nr && q < MAXQ ? __ldg(V + (size_t)q * cpr) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int q = qb + u * groups;
          if (q >= nr) break;
          const float2 f = bf2(w[u]);
#pragma unroll
          for (int i = 0; i < GSI_TC; ++i) {
            const float xv = xs[i][q];
            acc[i][0] += f.x * xv;
            acc[i][1] += f.y * xv;
          }
        }
      }
      float* rr = gsi_red + (size_t)grp * GSI_TC * a.k;
#pragma unroll
      for (int i = 0; i < GSI_TC; ++i) {
        rr[i * a.k + 2 * pair] = acc[i][0];
        rr[i * a.k + 2 * pair + 1] = acc[i][1];
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nt * a.k; e += blockDim.x) {
      float sum = 0.0f;
      for (int q = 0; q < groups; ++q) sum += gsi_red[(size_t)q * GSI_TC * a.k + e];
      red_add_f32(&a.g[(size_t)t0 * a.k + e], sum);
    }
  }
}

// Residual norms: rows [r0, r1) of V_k (at most 4 per warp), warp = row,
// lane = 8 consecutive basis columns per 16-byte piece (k / 8 pieces per
// row), the warp's rows loaded before use; g of the chunk in shared memory.
// Each CTA writes its sums of r^2 and x^2 per token.
constexpr int GSI_RESID_ROWS = 32;   // rows per CTA (4 per warp)

__global__ void __launch_bounds__(GSI_THREADS) k_gsi_resid(const GsiArgs a) {
  extern __shared__ float gsi_gs[];   // [GSI_TC][k]
  __shared__ float red[GSI_THREADS / 32][GSI_TC][2];
  griddep_wait();
  int r0, r1;
  row_range(a.d_in, r0, r1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = GSI_THREADS / 32;
  const int kv = a.k / 8;
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    __syncthreads();
    for (int e = threadIdx.x; e < GSI_TC * a.k; e += blockDim.x)
      gsi_gs[e] = e < nt * a.k ? a.g[(size_t)t0 * a.k + e] : 0.0f;
    __syncthreads();
    float r2 = 0.0f, x2 = 0.0f;   // of token (lane >> 2) & 7
    for (int rb = r0 + warp; rb < r1; rb += 4 * nwarp) {
      float acc[4][GSI_TC];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < GSI_TC; ++i) acc[u][i] = 0.0f;
      for (int v = lane; v < kv; v += 32) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int row = rb + u * nwarp;
          w[u] = row < r1 ? __ldg(reinterpret_cast<const uint4*>(a.Vk) + (size_t)row * kv + v) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t wp[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const float2 f = bf2(wp[qq]);
#pragma unroll
            for (int i = 0; i < GSI_TC; ++i) {
              const float2 gg = *reinterpret_cast<const float2*>(gsi_gs + i * a.k + 8 * v + 2 * qq);
              acc[u][i] += f.x * gg.x + f.y * gg.y;
            }
          }
        }
      }
      const int ti = (lane >> 2) & 7;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int row = rb + u * nwarp;
        const float s = warp_sum8(acc[u]);
        if ((lane & 3) == 0 && ti < nt && row < r1) {
          const float xv = __bfloat162float(a.x[(size_t)(t0 + ti) * a.d_in + row]);
          const float rv = xv - s;
          r2 += rv * rv;
          x2 += xv * xv;
        }
      }
    }
    if ((lane & 3) == 0) {
      red[warp][(lane >> 2) & 7][0] = r2;
      red[warp][(lane >> 2) & 7][1] = x2;
    }
    __syncthreads();
    if (threadIdx.x < 2 * nt) {
      const int i = threadIdx.x >> 1, c = threadIdx.x & 1;
      float s = 0.0f;
      for (int w = 0; w < nwarp; ++w) s += red[w][i][c];
      a.part[((size_t)blockIdx.x * a.maxT + t0 + i) * 2 + c] = s;
    }
  }
}

// Output rows [r0, r1): every CTA adds the residual kernel's partial norms
// and decides the route of each token (the same decision in every CTA), then
// each warp loads GSI_ROWS rows of M at once (one 16-byte piece per lane per
// row, k <= 256; two pieces for k <= 512) and reduces the eight tokens' dot
// products with warp_sum8.  Slow tokens then stream their W rows.
struct GsiOutSmem {
  int ghat, xs, slow, total;
  __host__ __device__ static GsiOutSmem make(int T, int k, int d_in) {
    GsiOutSmem s;
    int o = 0;
    s.ghat = o;  o += (T * k * 2 + 15) & ~15;         // bf16 [T][k]
    s.xs = o;    o += GSI_TC * d_in * 2;              // bf16 [GSI_TC][d_in] (a chunk of slow tokens)
    s.slow = o;  o += ((T + 1) * 4 + 15) & ~15;       // slow token list and its count
    s.total = o;
    return s;
  }
};

__global__ void __launch_bounds__(GSI_OUT_THREADS) k_gsi_out(const GsiArgs a) {
  extern __shared__ __align__(16) uint8_t gsi_o[];
  const GsiOutSmem L = GsiOutSmem::make(a.T, a.k, a.d_in);
  __nv_bfloat16* ghat = reinterpret_cast<__nv_bfloat16*>(gsi_o + L.ghat);
  uint4* xs = reinterpret_cast<uint4*>(gsi_o + L.xs);
  int* slow = reinterpret_cast<int*>(gsi_o + L.slow);
  int* nslow = slow + a.T;
  griddep_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = GSI_OUT_THREADS / 32;
  // routes: warp w adds the partial norms of tokens w, w + 8, ...
  for (int t = warp; t < a.T; t += nwarp) {
    float r2 = 0.0f, x2 = 0.0f;
    for (int c = lane; c < a.grid_resid; c += 32) {
      r2 += a.part[((size_t)c * a.maxT + t) * 2];
      x2 += a.part[((size_t)c * a.maxT + t) * 2 + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      r2 += __shfl_xor_sync(0xFFFFFFFFu, r2, o);
      x2 += __shfl_xor_sync(0xFFFFFFFFu, x2, o);
    }
    if (lane == 0) slow[t] = !(r2 < a.eps2 * x2);
  }
  for (int e = threadIdx.x; e < a.T * a.k; e += blockDim.x) ghat[e] = __float2bfloat16_rn(a.g[e]);
  __syncthreads();
  if (threadIdx.x == 0) {   // compact the slow tokens in token order
    int n = 0;
    for (int t = 0; t < a.T; ++t)
      if (slow[t]) slow[n++] = t;
    *nslow = n;
    if (blockIdx.x == 0) *a.n_slow = n;
  }
  // the next forward sums its g into the other buffer: clear it here
  {
    const long long n = (long long)a.maxT * a.k;
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
      a.g_next[e] = 0.0f;
  }
  __syncthreads();
  const int ns = *nslow;
  int r0, r1;
  row_range(a.d_out, r0, r1);
  const int kv = a.k / 8;
  // fast path (every token; slow tokens are overwritten below)
  for (int t0 = 0; t0 < a.T; t0 += GSI_TC) {
    const int nt = min(GSI_TC, a.T - t0);
    for (int ob = r0 + warp * GSI_ROWS; ob < r1; ob += nwarp * GSI_ROWS) {
      const int nr = min(GSI_ROWS, r1 - ob);
      float acc[GSI_ROWS][GSI_TC];
#pragma unroll
      for (int r = 0; r < GSI_ROWS; ++r)
#pragma unroll
        for (int i = 0; i < GSI_TC; ++i) acc[r][i] = 0.0f;
      for (int v = lane; v < kv; v += 32) {
        uint4 w[GSI_ROWS];
#pragma unroll
        for (int r = 0; r < GSI_ROWS; ++r)
          w[r] = r < nr ? __ldg(reinterpret_cast<const uint4*>(a.M) + (size_t)(ob + r) * kv + v)
                        : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < GSI_TC; ++i) {   // one token's 8 values of bf16(g) at a time
          const uint4 gq = i < nt ? reinterpret_cast<const uint4*>(ghat + (size_t)(t0 + i) * a.k)[v]
                                  : make_uint4(0, 0, 0, 0);
          const uint32_t gp[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const float2 gf = bf2(gp[qq]);
#pragma unroll
            for (int r = 0; r < GSI_ROWS; ++r) {
              const uint32_t wq = qq == 0 ? w[r].x : qq == 1 ? w[r].y : qq == 2 ? w[r].z : w[r].w;
              const float2 f = bf2(wq);
              acc[r][i] += f.x * gf.x + f.y * gf.y;
            }
          }
        }
      }
      const int ti = (lane >> 2) & 7;
#pragma unroll
      for (int r = 0; r < GSI_ROWS; ++r) {
        const float s = warp_sum8(acc[r]);
        if ((lane & 3) == 0 && ti < nt && r < nr) a.y[(size_t)(t0 + ti) * a.d_out + ob + r] = s;
      }
    }
  }
  if (ns == 0) return;
  // slow path: chunks of the slow tokens, x rows staged, W rows (d_in
  // elements) streamed four 16-byte pieces per lane ahead
  const int dv = a.d_in / 8;
  for (int s0 = 0; s0 < ns; s0 += GSI_TC) {
    const int nt = min(GSI_TC, ns - s0);
    __syncthreads();
    for (int e = threadIdx.x; e < GSI_TC * dv; e += blockDim.x) {
      const int i = e / dv, v = e - i * dv;
      xs[e] = i < nt ? reinterpret_cast<const uint4*>(a.x)[(size_t)slow[s0 + i] * dv + v] : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int o = r0 + warp; o < r1; o += nwarp) {
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
          const uint32_t wp[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
          for (int i = 0; i < GSI_TC; ++i) {
            const uint4 xq = xs[i * dv + v0 + 32 * u];
            const uint32_t xp[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float2 f = bf2(wp[qq]), xf = bf2(xp[qq]);
              acc[i] += f.x * xf.x + f.y * xf.y;
            }
          }
        }
      }
      const float s = warp_sum8(acc);
      const int ti = (lane >> 2) & 7;
      if ((lane & 3) == 0 && ti < nt) a.y[(size_t)slow[s0 + ti] * a.d_out + o] = s;
    }
  }
}

}  // namespace sffn
