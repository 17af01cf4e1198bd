// Mixture of LoPA-gated sparse experts ("Meta FAIR and Inria's LoPA Gating
// Hits 3.31x Real GPU Speedup for LLM Inference", section "Model Casting and
// Quality at 90% Sparsity": LoPA gating carries over to MoE layers whose
// experts share the gated FFN structure).  Routing as in Mixtral: the top_k
// experts by router logit (ties to the smaller index), softmax over the kept
// logits, y_t = sum of w_te · FFN_e(x_t).
//
//   k_moe_route    one CTA per token: logits <W_r[e], x_t> (a warp per
//                  expert), the top_k, their softmax weights, and the token's
//                  row in every expert's input block: x_t where routed, zero
//                  elsewhere
//   (each expert's own sparse forward on its block of T rows: a zero row
//    keeps no neuron when the gate bias is <= 0, so it reads no W_up/W_down
//    row and adds nothing)
//   k_moe_combine  y[t] = sum_k w[t][k] · y_e[t] over the token's experts
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int MOE_MAX_E = 64;
constexpr int MOE_MAX_K = 8;

struct MoeRouteArgs {
  const __nv_bfloat16* x;     // [T][d]
  const __nv_bfloat16* Wr;    // [E][d]
  __nv_bfloat16* xe;          // [E][T][d] expert input blocks
  int* sel;                   // [T][top_k]
  float* w;                   // [T][top_k]
  float* logits;              // [T][E] (debug)
  int T, d, E, top_k;
};

__global__ void __launch_bounds__(256) k_moe_route(const MoeRouteArgs a) {
  __shared__ float lg[MOE_MAX_E];
  __shared__ int s_sel[MOE_MAX_K];
  __shared__ float s_w[MOE_MAX_K];
  __shared__ uint64_t routed;          // bit e: the token goes to expert e
  griddep_wait();
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.d);
  const int dv = a.d / 8;
  for (int e = warp; e < a.E; e += nw) {
    const uint4* wr = reinterpret_cast<const uint4*>(a.Wr + (size_t)e * a.d);
    float s = 0.0f;
    for (int v = lane; v < dv; v += 32) {
      const uint4 p = __ldg(wr + v), q = xr[v];
      const uint32_t pp[4] = {p.x, p.y, p.z, p.w}, qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pp[i]));
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qq[i]));
        s += f.x * g.x + f.y * g.y;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) lg[e] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // top_k by repeated selection: the largest remaining logit, the smaller
    // index among equals
    uint64_t taken = 0;
    for (int kk = 0; kk < a.top_k; ++kk) {
      int best = -1;
      for (int e = 0; e < a.E; ++e)
        if (!((taken >> e) & 1ull) && (best < 0 || lg[e] > lg[best])) best = e;
      taken |= 1ull << best;
      s_sel[kk] = best;
    }
    float mx = lg[s_sel[0]], den = 0.0f;
    for (int kk = 0; kk < a.top_k; ++kk) {
      s_w[kk] = expf(lg[s_sel[kk]] - mx);
      den += s_w[kk];
    }
    for (int kk = 0; kk < a.top_k; ++kk) {
      a.sel[t * a.top_k + kk] = s_sel[kk];
      a.w[t * a.top_k + kk] = s_w[kk] / den;
    }
    routed = taken;
  }
  if (a.logits)
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.logits[(size_t)t * a.E + e] = lg[e];
  __syncthreads();
  const uint64_t r = routed;
  for (int e = 0; e < a.E; ++e) {
    uint4* dst = reinterpret_cast<uint4*>(a.xe + ((size_t)e * a.T + t) * a.d);
    const bool on = (r >> e) & 1ull;
    for (int v = threadIdx.x; v < dv; v += blockDim.x) dst[v] = on ? xr[v] : make_uint4(0, 0, 0, 0);
  }
}

struct MoeCombineArgs {
  const float* ye;            // [E][T][d] expert outputs
  const int* sel;             // [T][top_k]
  const float* w;             // [T][top_k]
  float* y;                   // [T][d]
  int T, d, top_k;
};

__global__ void __launch_bounds__(256) k_moe_combine(const MoeCombineArgs a) {
  griddep_wait();
  const int t = blockIdx.y;
  const int d4 = a.d / 4;
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < d4; v += gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int kk = 0; kk < a.top_k; ++kk) {
      const int e = a.sel[t * a.top_k + kk];
      const float wk = a.w[t * a.top_k + kk];
      const float4 p = reinterpret_cast<const float4*>(a.ye + ((size_t)e * a.T + t) * a.d)[v];
      acc.x += wk * p.x;
      acc.y += wk * p.y;
      acc.z += wk * p.z;
      acc.w += wk * p.w;
    }
    reinterpret_cast<float4*>(a.y + (size_t)t * a.d)[v] = acc;
  }
}

}  // namespace sffn
