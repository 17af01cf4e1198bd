// Gate GEMM for a single block of up to 8 tokens, streaming whole W_gate rows
// ([TwELL] TwELL section: the gate is dense and HBM-bound at decode, and its
// epilogue writes TwELL directly, with no conversion kernel).
//
// The dense gate g = x·W_gate^T + b has one weight row per neuron.  At a few
// tokens it moves about 1 byte per FLOP, so the copy engine, not the tensor
// core, sets its time.  Tile-shaped TMA loads of 128 rows x 128 bytes ran at
// about 35 GB/s per SM for the 1 MB each CTA streams; whole-row bulk copies
// run faster.  This kernel therefore streams W_gate like the fused row kernel
// streams W_up.  Every SM takes an equal contiguous range of 8-neuron groups
// (an 8-row stage of 8 KB bulk copies) through a ring of two slots (a third
// slot measured slower: more rows in flight cost HBM efficiency).  The
// up-style warp MMA gives g^T[token][neuron] for each group: tokens are M,
// padded to 16 with zero rows, from a staged x block; the rows are N.  The
// 16 warps' partial sums meet in shared memory.
//
// A TwELL tile holds 128 neurons, which one CTA's range may split.  Every
// CTA writes its groups' g into a per-tile fp32 staging block, and the CTA
// whose ticket completes the tile reads the whole tile back.  That CTA emits
// TwELL exactly as the tile-kernel epilogue does: counts, ascending indices,
// bf16 values, pads, keep masks and overflow epochs.
//
// The low-rank gate ([LoPA]) runs it at up to 8 tokens over the rank rows of
// A^T with x, storing z = bf16(x·A) instead of emitting TwELL (the gate over
// B then runs on the tile kernel).
#pragma once

#include "epilogues.cuh"
#include "rows_mma.cuh"

namespace sffn {

struct GateRowsArgs {
  const __nv_bfloat16* x;      // [T][d]
  const __nv_bfloat16* W_gate; // [F][d]
  TwellParams tw;              // T, F, n_tiles, C, bias, tau, act and the TwELL outputs
  float* gstage;               // [n_tiles][8][128] fp32 gate values of a tile being assembled
  int* tick;                   // [n_tiles] groups done per tile, zero between forwards
  float4* zero_out;            // if set, zeroed (zero_n4 float4) for the kernel that adds into it
  long long zero_n4;
  int d;
  int nslot;                   // ring slots (<= RW_NSMAX)
  uint32_t* status;
  __nv_bfloat16* zout;         // if set: store bf16(g) [T][F] (no bias) instead of emitting TwELL
                               // (the low-rank gate's z = bf16(x·A) with W_gate = A^T)
};

struct GateRowsSmem {
  int xs, ring, bars, ured, scratch, total;
  __host__ __device__ static GateRowsSmem make(int d, int nslot) {
    GateRowsSmem s;
    int o = 0;
    s.xs = o;      o += RowsSmem::stage(d);
    s.ring = o;    o += nslot * RowsSmem::stage(d);
    s.bars = o;    o += ((RW_NSMAX + 1) * 8 + 15) & ~15;
    s.ured = o;    o += 2 * RW_WARPS * 32 * 8;      // double-buffered warp partials
    s.scratch = o; o += twell32_smem(128) + 16;     // TwELL staging, then ticket result and abort flag
    s.total = o;
    return s;
  }
};

__global__ void __launch_bounds__(RW_THREADS, 1) k_gate_rows(const GateRowsArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int d = a.d;
  const int ns = max(2, min(a.nslot, RW_NSMAX));
  const GateRowsSmem L = GateRowsSmem::make(d, ns);
  const int RS = RowsSmem::pitch(d), SB = RowsSmem::stage(d);
  uint8_t* ring = sm + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* xbar = full + RW_NSMAX;
  float2* ured = reinterpret_cast<float2*>(sm + L.ured);
  uint8_t* tw_stage = sm + L.scratch;
  volatile int* done_flag = reinterpret_cast<volatile int*>(sm + L.scratch + twell32_smem(128));
  volatile int* abort_flag = done_flag + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.tw.T, F = a.tw.F;
  const int nj = d / RW_DIV;
  const int NG = F / RW_G;                                   // 8-neuron groups
  const int g0 = (int)((long long)NG * blockIdx.x / gridDim.x);
  const int g1 = (int)((long long)NG * (blockIdx.x + 1) / gridDim.x);
  const int n_stages = g1 - g0;
  constexpr int GPT = 128 / RW_G;                            // groups per TwELL tile

  griddep_wait();  // x, and the outputs earlier kernels read, belong to the stream order
  const int nvalid = min(8, T);
  if (tid == 0) {
    for (int i = 0; i < ns; ++i) mbar_init(&full[i], 1);
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_expect_tx(xbar, (uint32_t)(nvalid * d * 2));
    for (int t = 0; t < nvalid; ++t) bulk_g2s(sm + L.xs + t * RS, a.x + (size_t)t * d, (uint32_t)d * 2u, xbar);
  }
  for (int e = tid; e < (8 - nvalid) * (d >> 3); e += blockDim.x) {
    const int t = nvalid + e / (d >> 3), v = e % (d >> 3);
    *reinterpret_cast<uint4*>(sm + L.xs + t * RS + v * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  if (a.zero_out) {
    for (long long e = (long long)blockIdx.x * blockDim.x + tid; e < a.zero_n4; e += (long long)gridDim.x * blockDim.x)
      a.zero_out[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();

  // stage q = group g0 + q: warp w (lane 0) copies its row w
  auto issue_stage = [&](int q) {
    if (q >= n_stages || lane != 0 || warp >= RW_G) return;
    const int slot = q % ns;
    if (warp == 0) mbar_expect_tx(&full[slot], (uint32_t)(RW_G * d * 2));
    const int row = (g0 + q) * RW_G + warp;
    bulk_g2s(ring + (size_t)slot * SB + warp * RS, a.W_gate + (size_t)row * d, (uint32_t)d * 2u, &full[slot]);
  };
  for (int q = 0; q < ns; ++q) issue_stage(q);
  int issued_end = min(ns, n_stages);
  mbar_wait(xbar, 0, abort_flag, a.status);

  const uint32_t lrow = (uint32_t)((lane & 7) * RS + 16 * ((lane >> 3) & 1) + 32 * warp);
  const uint32_t hi_off = (lane >> 4) ? 32u * RW_WARPS : 0u;
  const uint32_t xsl = smem_u32(sm + L.xs) + lrow;
  const uint32_t ring_s = smem_u32(ring);
  for (int q = 0; q < n_stages; ++q) {
    const int slot = q % ns;
    const bool ok = mbar_wait(&full[slot], (uint32_t)((q / ns) & 1), abort_flag, a.status);
    const uint32_t sbs = ring_s + (uint32_t)(slot * SB) + lrow;
    float cu[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
#pragma unroll
      for (int j = 0; j < RW_MAXJ; j += 2) {
        if (j < nj) {
          const uint32_t off = 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u);
          uint32_t x0, x1, x2, x3, b0, b1, b2, b3;
          ldsm_x4(xsl + off, x0, x1, x2, x3);
          ldsm_x4(sbs + off, b0, b1, b2, b3);
          mma_bf16_16816(cu, x0, 0u, x1, 0u, b0, b1);
          if (j + 1 < nj) mma_bf16_16816(cu, x2, 0u, x3, 0u, b2, b3);
        }
      }
    }
    float2* ub = ured + (q & 1) * RW_WARPS * 32;
    ub[warp * 32 + lane] = make_float2(cu[0], cu[1]);
    __syncthreads();
    issue_stage(q + ns);  // the slot is free
    if (q + ns < n_stages) issued_end = q + ns + 1;
    if (warp < 4) {
      // warp 0 sums the partials of (token lane/4, neurons 2(lane%4), +1) into
      // the tile's staging block; the CTA's last group of a tile takes a ticket
      const int grp = g0 + q, p = grp / GPT;
      const bool last_of_tile = q == n_stages - 1 || (grp + 1) % GPT == 0;
      if (warp == 0) {
        float u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int w = 0; w < RW_WARPS; ++w) {
          const float2 v = ub[w * 32 + lane];
          u0 += v.x;
          u1 += v.y;
        }
        const int tok = lane >> 2, n = (grp % GPT) * RW_G + 2 * (lane & 3);
        float* gs = a.gstage + ((size_t)p * 8 + tok) * 128 + n;
        __stcg(gs, u0);
        __stcg(gs + 1, u1);
        if (last_of_tile) {
          __threadfence();
          __syncwarp();
          if (lane == 0) {
            const int n_done = grp - max(g0, p * GPT) + 1;
            *done_flag = atomicAdd(&a.tick[p], n_done) + n_done == GPT;
          }
          __syncwarp();
        }
      }
      if (last_of_tile) {
        named_bar_sync(2, 128);
        if (*done_flag) {
          // the whole tile is in: emit TwELL for it (one neuron per thread;
          // after an abort the values are void, which the status word says)
          __threadfence();
          float g[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = i < 8 ? __ldcg(a.gstage + ((size_t)p * 8 + i) * 128 + tid) : 0.f;
          if (a.zout) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < T) a.zout[(size_t)i * F + p * 128 + tid] = __float2bfloat16_rn(g[i]);
          } else {
            twell_tile32(a.tw, g, p * 128 + tid, 0, tid, tw_stage, 1);
          }
          if (tid == 0) a.tick[p] = 0;
        }
        named_bar_sync(2, 128);  // done_flag is read by all four warps before it is rewritten
      }
    }
  }
  // drain copies still in flight (only after an abort)
  if (tid == 0 && *abort_flag) {
    const uint64_t tx = globaltimer();
    while (!mbar_try_wait(xbar, 0u)) {
      if (globaltimer() - tx > SFFN_WAIT_LIMIT_NS) break;
    }
    for (int k = 0; k < ns && k < issued_end; ++k) {
      const int last = issued_end - 1 - k;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&full[last % ns], (uint32_t)((last / ns) & 1))) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) break;
      }
    }
  }
}

}  // namespace sffn
