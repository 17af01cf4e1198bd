// Persistent tensor-core gate with the TwELL emission overlapped with the
// next tile's MMAs ([TwELL] "TwELL 減掉轉換開銷": the gate GEMM's epilogue
// writes TwELL directly).  For many tokens (prefill) the gate is a dense
// tensor-core GEMM, D[128 neurons x BN tokens] per tile, and the TwELL
// emission of a tile takes longer than its MMAs.  With one CTA per tile the
// tensor pipe idles while each CTA emits.  Here one CTA per SM walks the
// tiles w = blockIdx.x, blockIdx.x + gridDim.x, ... and keeps two TMEM
// accumulators: the MMA warp fills one while the emission reads the other.
//
// Warp roles: warps 0 .. 4 TP_EPI_WG - 1 emit, as TP_EPI_WG warpgroups that
// take interleaved 32-token chunks of a tile (warp w reads TMEM lanes
// 32 (w % 4) .. +31, one neuron per thread; each warpgroup has its own
// staging block and named barrier); the next warp issues the TMA loads of the
// A (W_gate) and B (x) k-blocks through a ring that runs on across tiles; the
// last owns TMEM and issues the MMAs.  Barriers: full/empty per ring stage,
// accfull per accumulator (MMA -> emission) and accfree per accumulator (all
// emission warpgroups -> MMA).  Every wait is bounded; on a timeout the CTA
// records DEV_ERR_TIMEOUT, drains its copies and MMAs, frees TMEM and returns.
#pragma once

#include "epilogues.cuh"
#include "tc_gemm.cuh"

namespace sffn {

constexpr int TP_EPI_WG = 4;                 // emission warpgroups
constexpr int TP_EPI_WARPS = 4 * TP_EPI_WG;
constexpr int TP_THREADS = TP_EPI_WARPS * 32 + 64;
constexpr int TP_PRODUCER = TP_EPI_WARPS, TP_MMA = TP_EPI_WARPS + 1;  // warp indices

struct TpLayout {
  int stages, stage_bytes, bars, scratch, scratch_wg, total;
};
__host__ __device__ inline TpLayout tp_layout(int BN, int C) {
  TpLayout L;
  L.stage_bytes = TC_A_BYTES + BN * TC_BK * 2;
  L.scratch_wg = (twell32_smem(C) + 127) & ~127;
  const int fixed = 1024 /*align slack*/ + 256 /*barriers*/ + TP_EPI_WG * L.scratch_wg;
  L.stages = (TC_SMEM_BUDGET - fixed) / L.stage_bytes;
  if (L.stages > 8) L.stages = 8;
  L.bars = L.stages * L.stage_bytes;
  L.scratch = L.bars + 256;
  L.total = 1024 + L.scratch + TP_EPI_WG * L.scratch_wg;
  return L;
}

// args: kb_total[0] (K blocks), n_rows (tokens), status, zero_out/zero_n4.
template <int BN>
__global__ void __launch_bounds__(TP_THREADS, 1)
k_tc_gate_persist(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                  const TcArgs args, const TwellParams tw) {
  static_assert(2 * BN <= 512, "two accumulators must fit in TMEM");
  constexpr uint32_t NCOLS = tmem_cols_for(2 * BN);
  constexpr uint32_t IDESC = idesc_bf16_f32(TC_BM, BN);
  const TpLayout L = tp_layout(BN, tw.C);
  const int STAGES = L.stages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + STAGES;
  uint64_t* accfull = empty + STAGES;  // [2]
  uint64_t* accfree = accfull + 2;     // [2]
  uint64_t* mma_done = accfree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = tw.n_tiles;
  const int n_work = P * ((args.n_rows + BN - 1) / BN);
  const int KB = args.kb_total[0];

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accfree[b], TP_EPI_WG);  // one arrival per emission warpgroup
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == TP_MMA) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  if (warp == TP_PRODUCER && lane == 0) {
    tma_prefetch_desc(&mA);
    tma_prefetch_desc(&mB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // x and the outputs belong to the stream order

  if (warp == TP_PRODUCER) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_work && ok; w += gridDim.x) {
        const int m0 = (w % P) * TC_BM, n0 = (w / P) * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, f = it / STAGES;
          if (f > 0 && !mbar_wait(&empty[s], (f - 1) & 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + (size_t)s * L.stage_bytes;
          mbar_expect_tx(&full[s], (uint32_t)L.stage_bytes);
          tma_load_2d(st, &mA, &full[s], kb * TC_BK, m0);
          tma_load_2d(st + TC_A_BYTES, &mB, &full[s], kb * TC_BK, n0);
        }
      }
      // the last fill of every stage has landed before the CTA can exit
      for (int s = 0; s < STAGES && s < it; ++s) {
        const int last = s + STAGES * ((it - 1 - s) / STAGES);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&full[s], (last / STAGES) & 1)) {
          if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) {
            atomicOr(args.status, DEV_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
  } else if (warp == TP_MMA) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      int it = 0, i = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < n_work && ok; w += gridDim.x, ++i) {
        const int b = i & 1;
        // the emission is done with this accumulator's previous tile
        if (i >= 2 && !mbar_wait(&accfree[b], (uint32_t)(((i >> 1) - 1) & 1), abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES, f = it / STAGES;
          if (!mbar_wait(&full[s], f & 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + (size_t)s * L.stage_bytes;
          const uint64_t ad = sdesc_k_sw128(smem_u32(st));
          const uint64_t bd = sdesc_k_sw128(smem_u32(st + TC_A_BYTES));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k)
            tc_mma(dcol, ad + 2u * k, bd + 2u * k, IDESC, (kb == 0 && k == 0) ? 0u : 1u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&accfull[b]);
      }
      // every MMA of this CTA has completed before TMEM is freed
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(mma_done, 0)) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) {
          atomicOr(args.status, DEV_ERR_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ----------------------------------------------------------- emission
    if (args.zero_out) {  // an output that later kernels accumulate into
      for (long long e = (long long)blockIdx.x * (TP_EPI_WARPS * 32) + threadIdx.x; e < args.zero_n4;
           e += (long long)gridDim.x * (TP_EPI_WARPS * 32))
        args.zero_out[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int wg = warp >> 2, etid = threadIdx.x & 127;
    const uint32_t tlane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint8_t* scratch = smem + L.scratch + wg * L.scratch_wg;
    int i = 0;
    for (int w = blockIdx.x; w < n_work; w += gridDim.x, ++i) {
      const int b = i & 1;
      if (!mbar_wait(&accfull[b], (uint32_t)((i >> 1) & 1), abort_flag, args.status)) break;
      tc_fence_after();
      const int m0 = (w % P) * TC_BM, n0 = (w / P) * BN;
      const int j = m0 + etid;
#pragma unroll 1
      for (int c = 32 * wg; c < BN; c += 32 * TP_EPI_WG) {  // this warpgroup's 32-token chunks
        if (n0 + c >= tw.T) break;
        float g[32];
        tmem_ld16(tlane + (uint32_t)(b * BN + c), g);
        tmem_ld16(tlane + (uint32_t)(b * BN + c + 16), g + 16);
        twell_tile32(tw, g, j, n0 + c, etid, scratch, 1 + wg);
      }
      // this warpgroup has read the accumulator: the MMAs may refill it
      tc_fence_before();
      named_bar_sync(1 + wg, 128);
      if (etid == 0) mbar_arrive(&accfree[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == TP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

}  // namespace sffn
