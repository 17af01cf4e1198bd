// Tensor-core tile kernel for sm_100a: TMA -> shared memory -> tcgen05.mma ->
// TMEM -> epilogue.  One CTA computes D[128 x BN] = A[m0:m0+128, K] ·
// B[n0:n0+BN, K]^T for one or two GEMM phases (two accumulators, or one that
// both phases add into), over a K range that may be split across gridDim.z.
//
// Warp roles (192 threads): warps 0-3 run the epilogue (warp w reads TMEM
// lanes 32w..32w+31, one accumulator row per thread), warp 4 issues the TMA
// loads, warp 5 owns TMEM and issues the MMAs.  Every wait is bounded; on a
// timeout the CTA records DEV_ERR_TIMEOUT, drains its own copies and MMAs,
// frees TMEM and returns.
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int TC_THREADS = 192;
constexpr int TC_BM = 128;           // rows per tile (TMEM lanes)
constexpr int TC_BK = 64;            // bf16 elements per 128-byte swizzled row
constexpr int TC_A_BYTES = TC_BM * TC_BK * 2;

// NB = B operands per stage: 2 when one A tile multiplies two B tiles into
// the same accumulator (the hi and lo halves of a split bf16 operand).  EPI =
// the epilogue's shared scratch; the ring takes what is left of 227 KB.
constexpr int TC_SMEM_BUDGET = 227 * 1024;
template <int BN, int NB = 1, int EPI = 9 * 1024>
struct TcCfg {
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE_BYTES = TC_A_BYTES + NB * B_BYTES;
  static constexpr int EPI_SMEM = (EPI + 127) & ~127;
  static constexpr int STAGES_RAW = (TC_SMEM_BUDGET - 1024 - 256 - EPI_SMEM) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : (STAGES_RAW < 2 ? 2 : STAGES_RAW);
  static constexpr int SMEM = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256 /*barriers*/ + EPI_SMEM;
  static_assert(SMEM <= TC_SMEM_BUDGET, "shared memory budget");
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : n <= 256 ? 256u : 512u;
}

struct TcArgs {
  int n_phase;          // 1 or 2
  int acc_same;         // 1: both phases accumulate into one accumulator
  int kb_total[2];      // 64-wide K blocks of each phase (before the split)
  int n_rows;           // valid B rows (columns of D); CTAs with n0 >= n_rows exit
  const int* n_rows_dev;  // if set, the valid B row count is read from the device
  uint32_t* status;
  float4* zero_out;     // if set, the CTAs zero zero_n4 float4 here (after the grid dependency)
  long long zero_n4;
  int stages;           // ring stages in use (0: all that fit); fewer bound the bytes in flight
  const int* kb_dev;    // if set, every phase's K is *kb_dev rows (64-wide blocks rounded up), read
                        // from the device after the grid dependency (a count an earlier kernel wrote)
  unsigned long long hold_ns;  // test hook (0: off): before issuing any copy the producer waits
                               // this long on a barrier that nothing signals, then records a
                               // timeout and the CTA returns without output
};

template <class E, class = void>
struct epi_dual_b {
  static constexpr bool value = false;
};
template <class E>
struct epi_dual_b<E, decltype(void(E::DUAL_B))> {
  static constexpr bool value = E::DUAL_B;
};
// DUAL_ALL: every phase multiplies its A by the same pair (B0 + B1) (without
// it, a phase after the first reads its single B from mB1)
template <class E, class = void>
struct epi_dual_all {
  static constexpr bool value = false;
};
template <class E>
struct epi_dual_all<E, decltype(void(E::DUAL_ALL))> {
  static constexpr bool value = E::DUAL_ALL;
};
template <class E, class = void>
struct epi_smem {
  static constexpr int value = 9 * 1024;
};
template <class E>
struct epi_smem<E, decltype(void(E::EPI_SMEM))> {
  static constexpr int value = E::EPI_SMEM;
};
template <int BN, class Epi>
using TcCfgOf = TcCfg<BN, epi_dual_b<Epi>::value ? 2 : 1, epi_smem<Epi>::value>;

// Epilogue contract:
//   struct Epi { struct Params; static constexpr int N_ACC;
//     __device__ static void run(const Params&, uint32_t tmem, int m0, int n0,
//                                int split, int etid, uint8_t* scratch); };
// run() is called by the 128 epilogue threads (etid 0..127) once the
// accumulators are complete; accumulator a lives at TMEM column a*BN.

template <int BN, class Epi>
__global__ void __launch_bounds__(TC_THREADS, 1)
k_tc_gemm(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mB0,
          const __grid_constant__ CUtensorMap mA1, const __grid_constant__ CUtensorMap mB1,
          const TcArgs args, const typename Epi::Params ep) {
  using Cfg = TcCfgOf<BN, Epi>;
  constexpr bool DUAL = epi_dual_b<Epi>::value;  // phase 0 only: A · (B0 + B1) per stage
  constexpr int NB = DUAL ? 2 : 1;
  const int STAGES = args.stages > 0 && args.stages < Cfg::STAGES ? args.stages : Cfg::STAGES;
  constexpr uint32_t NCOLS = tmem_cols_for(Epi::N_ACC * BN);
  constexpr uint32_t IDESC = idesc_bf16_f32(TC_BM, BN);
  static_assert(2 * Cfg::STAGES * 8 + 8 + 8 <= 256, "barrier area");

  const int m0 = blockIdx.x * TC_BM;
  const int n0 = blockIdx.y * BN;
  if (args.n_rows_dev) griddep_wait();  // the row count comes from an earlier kernel
  const int n_rows = args.n_rows_dev ? *args.n_rows_dev : args.n_rows;
  if (n0 >= n_rows) return;  // uniform: the whole CTA leaves before any setup

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * TC_A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* scratch = smem + STAGES * Cfg::STAGE_BYTES + 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&mA0);
    tma_prefetch_desc(&mB0);
    if (args.n_phase > 1 || DUAL) {
      tma_prefetch_desc(&mA1);
      tma_prefetch_desc(&mB1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // inputs and outputs may belong to earlier kernels on the stream

  const int S = gridDim.z, sk = blockIdx.z;
  int kb_tot[2] = {args.kb_total[0], args.kb_total[1]};
  if (args.kb_dev) {
    const int kd = (*args.kb_dev + TC_BK - 1) / TC_BK;
    kb_tot[0] = kb_tot[1] = kd;
  }

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      int it = 0;
      bool ok = true;
      if (args.hold_ns) {
        // no copy is in flight yet: the wait runs out, the MMA warp sees the
        // abort flag, and the epilogue writes nothing
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&full[0], 0)) {
          if (globaltimer() - t0 > args.hold_ns) break;
        }
        *abort_flag = 1;
        atomicOr(args.status, DEV_ERR_TIMEOUT);
        ok = false;
      }
      for (int ph = 0; ph < args.n_phase && ok; ++ph) {
        const CUtensorMap* ma = ph == 0 ? &mA0 : &mA1;
        const CUtensorMap* mb = (ph == 0 || epi_dual_all<Epi>::value) ? &mB0 : &mB1;
        const int kb0 = (int)((long long)kb_tot[ph] * sk / S);
        const int kb1 = (int)((long long)kb_tot[ph] * (sk + 1) / S);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES, f = it / STAGES;
          if (f > 0 && !mbar_wait(&empty[s], (f - 1) & 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], Cfg::STAGE_BYTES);
          tma_load_2d(sA + s * TC_A_BYTES, ma, &full[s], kb * TC_BK, m0);
          tma_load_2d(sB + s * NB * Cfg::B_BYTES, mb, &full[s], kb * TC_BK, n0);
          if (DUAL) tma_load_2d(sB + (s * NB + 1) * Cfg::B_BYTES, &mB1, &full[s], kb * TC_BK, n0);
        }
      }
      // Drain: the last fill of every stage has landed before the CTA can exit.
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
  } else if (warp == 5) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      int it = 0;
      bool ok = true;
      for (int ph = 0; ph < args.n_phase && ok; ++ph) {
        const uint32_t dcol = args.acc_same ? 0u : (uint32_t)(ph * BN);
        const int kb0 = (int)((long long)kb_tot[ph] * sk / S);
        const int kb1 = (int)((long long)kb_tot[ph] * (sk + 1) / S);
        bool first = (ph == 0) || !args.acc_same;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES, f = it / STAGES;
          if (!mbar_wait(&full[s], f & 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(smem_u32(sA + s * TC_A_BYTES));
          const uint64_t bd = sdesc_k_sw128(smem_u32(sB + s * NB * Cfg::B_BYTES));
          const uint64_t bd1 = sdesc_k_sw128(smem_u32(sB + (s * NB + 1) * Cfg::B_BYTES));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            tc_mma(tmem + dcol, ad + 2u * k, bd + 2u * k, IDESC, (first && k == 0) ? 0u : 1u);
            if (DUAL) tc_mma(tmem + dcol, ad + 2u * k, bd1 + 2u * k, IDESC, 1u);
          }
          first = false;
          tc_commit(&empty[s]);
        }
      }
      // An accumulator whose K range is empty stays unwritten: only happens
      // when the split exceeds the K blocks, which the host never launches.
      tc_commit(accf);
      if (!ok) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(accf, 0)) {
          if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    if (args.zero_out) {  // an output that later kernels accumulate into
      const long long ncta = (long long)gridDim.x * gridDim.y * gridDim.z;
      const long long cta = ((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
      for (long long e = cta * 128 + threadIdx.x; e < args.zero_n4; e += ncta * 128)
        args.zero_out[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);
    // a CTA whose K range is empty (a device-side K of 0) has no accumulator to read
    bool any_k = false;
    for (int ph = 0; ph < args.n_phase; ++ph)
      any_k |= (long long)kb_tot[ph] * (sk + 1) / S > (long long)kb_tot[ph] * sk / S;
    if (mbar_wait(accf, 0, abort_flag, args.status) && !*abort_flag && any_k) {
      tc_fence_after();
      Epi::template run<BN>(ep, tlane, m0, n0, sk, threadIdx.x, scratch);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

}  // namespace sffn
