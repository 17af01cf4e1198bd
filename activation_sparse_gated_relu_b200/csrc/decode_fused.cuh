// The whole forward for one block of up to 8 tokens in one persistent launch
// ([TwELL] sections "TwELL 減掉轉換開銷" and "Hybrid 應對非均勻稀疏"): the gate
// with its TwELL emission, the overflow routing, the fused sparse up x down of
// the non-overflow tokens and the dense channel of the overflow tokens.
//
// With one CTA per SM, every phase streams weight rows through the same
// ring of shared-memory stages (8 whole rows of 8 KB per stage, one bulk copy
// per row) and computes on warp MMAs, as the separate row-streaming kernels
// do (gate_rows.cuh, rows_mma.cuh).  Keeping the phases in one launch removes
// a kernel boundary (grid drain, launch, prologue) between each, shares the
// staged x block and the partial output registers, and drops the dense
// channel's launches when no token overflows (the common case at decode).
//
//   G  gate: CTA s takes an equal range of 8-neuron groups of W_gate and
//      writes their gate values (fp32, for the TwELL values) and keep bits
//      (one byte per token and group);
//   -- grid barrier: every gate value and keep bit in --
//   R  rows: every CTA derives the per-tile counts, the overflow tokens and
//      the union of the live tokens' keep masks from the keep bits, ranks
//      the union and takes an equal range; its W_up rows then W_down rows
//      stream through the ring, u and h stay in registers, y accumulates in
//      registers.  While its first stages are in flight, CTA p writes tile
//      p's TwELL records (the format's output; nothing here waits for them)
//      and CTA 0 lists and counts the overflow tokens;
//   D  dense channel, only if some token overflowed: D1 streams W_gate and
//      W_up rows over the CTA's gate range and writes h = bf16(sigma(g))·u
//      of the overflow tokens (0 where not kept); after a second grid
//      barrier, D2 streams W_down rows over the same range and adds
//      h·W_down into the same partial-output registers;
//   the partial outputs go into out (zeroed in G, before the first barrier)
//   by bulk reduce-add copies at L2.
//
// The grid barriers need every CTA resident: the host launches exactly the
// number of CTAs that fit at once (one per SM), and every wait is bounded
// (a timeout sets the status word and the CTA gives up instead of hanging).
#pragma once

#include "epilogues.cuh"
#include "rows_mma.cuh"

namespace sffn {

struct DecodeArgs {
  const __nv_bfloat16* x;        // [T][d]
  const __nv_bfloat16* W_gate;   // [F][d]
  const __nv_bfloat16* W_up;
  const __nv_bfloat16* W_down;
  const __nv_bfloat16* zero_row; // >= d bf16 zeros
  TwellParams tw;                // T, F, n_tiles, C, bias, tau, act, TwELL outputs, keep masks, epochs
  float* gstage;                 // [n_tiles][8][128] fp32 gate values (before the bias)
  uint8_t* kbits;                // [8][d_ff / 8] keep bits, one byte per (token, 8-neuron group)
  unsigned* gbar;                // [2] grid barrier: arrivals, generation
  int* ovf_list;                 // [8]
  int* ovf_count;                // [1]
  float* hdense;                 // [8][F] h of the overflow tokens (dense channel)
  float* out;                    // [T][d]
  int d, nslot, lcap;
  uint32_t* status;
};

struct DecodeSmem {
  int xs, ring, bars, uni, emit, ured, misc, total;
  // uni: the rank bookkeeping of R; emit: the TwELL staging (8 tokens)
  __host__ __device__ static int rank_bytes(int n_tiles, int lcap) {
    return (((n_tiles + 1) * 4 + 15) & ~15) + n_tiles * 16 + lcap * 4 + lcap * 4 + lcap * 16;
  }
  __host__ __device__ static DecodeSmem make(int n_tiles, int C, int lcap, int d, int nslot) {
    DecodeSmem s;
    int o = 0;
    s.xs = o;      o += RowsSmem::stage(d);
    s.ring = o;    o += nslot * RowsSmem::stage(d);
    s.bars = o;    o += ((RW_NSMAX + 1) * 8 + 15) & ~15;
    s.uni = o;     o += rank_bytes(n_tiles, lcap);
    s.emit = o;    o += twell_smem(8, C);
    s.ured = o;    o += 2 * RW_WARPS * 32 * 8;
    s.misc = o;    o += 64 * 4;
    s.total = o;
    return s;
  }
};

// Bounded grid-wide barrier over all CTAs of the launch (all resident).
// Returns false (and records a timeout) if the other CTAs do not arrive.
__device__ __forceinline__ bool grid_barrier(unsigned* gbar, volatile int* abort_flag, uint32_t* status,
                                             volatile int* shared_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    const unsigned gen = atomicAdd(&gbar[1], 0u);
    if (atomicAdd(&gbar[0], 1u) == gridDim.x - 1) {
      atomicExch(&gbar[0], 0u);
      __threadfence();
      atomicAdd(&gbar[1], 1u);
    } else {
      const uint64_t t0 = globaltimer();
      while (atomicAdd(&gbar[1], 0u) == gen) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) {
          atomicOr(status, DEV_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    *shared_ok = ok;
  }
  __syncthreads();
  return *shared_ok != 0;
}

__global__ void __launch_bounds__(RW_THREADS, 1) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int d = a.d, T = a.tw.T, F = a.tw.F, P = a.tw.n_tiles, C = a.tw.C;
  const int ns = max(2, min(a.nslot, RW_NSMAX));
  const DecodeSmem L = DecodeSmem::make(P, C, a.lcap, d, ns);
  const int RS = RowsSmem::pitch(d), SB = RowsSmem::stage(d);
  uint8_t* ring = sm + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* xbar = full + RW_NSMAX;
  float2* ured = reinterpret_cast<float2*>(sm + L.ured);
  int* misc = reinterpret_cast<int*>(sm + L.misc);
  volatile int* abort_flag = misc + 40;
  volatile int* bar_ok = misc + 42;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, s = blockIdx.x;
  const int nj = d / RW_DIV;
  const int NG = F / RW_G;
  const int g0 = (int)((long long)NG * s / G), g1 = (int)((long long)NG * (s + 1) / G);
  constexpr int GPT = 128 / RW_G;  // 8-neuron groups per TwELL tile
  const uint32_t ring_s = smem_u32(ring);
  const uint32_t lrow = (uint32_t)((lane & 7) * RS + 16 * ((lane >> 3) & 1) + 32 * warp);
  const uint32_t hi_off = (lane >> 4) ? 32u * RW_WARPS : 0u;
  const uint32_t xsl = smem_u32(sm + L.xs) + lrow;
  int gsq = 0;         // stages issued and consumed by earlier phases (slot and parity base)
  int issued_end = 0;  // stages issued so far (for the drain after an abort)

  griddep_wait();  // x, out and the workspace belong to the stream order
  // ---------------------------------------------------------------- setup
  const int nvalid = min(8, T);
  if (tid == 0) {
    for (int i = 0; i < ns; ++i) mbar_init(&full[i], 1);
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_expect_tx(xbar, (uint32_t)(nvalid * d * 2));
    for (int t = 0; t < nvalid; ++t) bulk_g2s(sm + L.xs + t * RS, a.x + (size_t)t * d, (uint32_t)d * 2u, xbar);
    // the gate's first stages go out with x, ahead of the zeroing below
    for (int q = 0; q < ns && q < g1 - g0; ++q) {
      mbar_expect_tx(&full[q], (uint32_t)(RW_G * d * 2));
      for (int r = 0; r < RW_G; ++r)
        bulk_g2s(ring + (size_t)q * SB + r * RS, a.W_gate + (size_t)((g0 + q) * RW_G + r) * d, (uint32_t)d * 2u, &full[q]);
    }
  }
  for (int e = tid; e < (8 - nvalid) * (d >> 3); e += blockDim.x) {
    const int t = nvalid + e / (d >> 3), v = e % (d >> 3);
    *reinterpret_cast<uint4*>(sm + L.xs + t * RS + v * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  {  // this CTA's slice of out starts at zero: every phase adds into it at the end
    const long long n4 = (long long)T * d / 4;
    const long long q0 = n4 * s / G, q1 = n4 * (s + 1) / G;
    for (long long e = q0 + tid; e < q1; e += blockDim.x)
      reinterpret_cast<float4*>(a.out)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();

  // stage of 8 rows of matrix W starting at row r0 (or the given row ids)
  auto issue_rows = [&](int gs, const __nv_bfloat16* W, const int* rowid, int nrows, int row0) {
    if (lane != 0 || warp >= RW_G) return;
    const int slot = gs % ns;
    if (warp == 0) mbar_expect_tx(&full[slot], (uint32_t)(RW_G * d * 2));
    const __nv_bfloat16* src =
        warp < nrows ? W + (size_t)(rowid ? rowid[warp] : row0 + warp) * d : a.zero_row;
    bulk_g2s(ring + (size_t)slot * SB + warp * RS, src, (uint32_t)d * 2u, &full[slot]);
  };
  // up-style product of a staged stage: the warp's partial of
  // u^T[token lane/4][neurons 2(lane%4), +1] over its k steps
  auto up_partial = [&](uint32_t sbs, bool ok, float* cu) {
    cu[0] = cu[1] = cu[2] = cu[3] = 0.f;
    if (!ok) return;
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
  };
  float acc[RW_MAXJ][4];
#pragma unroll
  for (int j = 0; j < RW_MAXJ; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[j][k] = 0.f;
  // down product of a staged stage of 8 W_down rows with h (bh, bl) into acc
  auto down_acc = [&](uint32_t sbs, bool ok, uint32_t bh, uint32_t bl) {
    if (!ok) return;
#pragma unroll
    for (int j = 0; j < RW_MAXJ; j += 2) {
      if (j < nj) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(sbs + 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u), a0, a1, a2, a3);
        mma_bf16_1688(acc[j], a0, a1, bh);
        mma_bf16_1688(acc[j], a0, a1, bl);
        if (j + 1 < nj) {
          mma_bf16_1688(acc[j + 1], a2, a3, bh);
          mma_bf16_1688(acc[j + 1], a2, a3, bl);
        }
      }
    }
  };
  auto split_hilo = [](float h0, float h1, uint32_t& bh, uint32_t& bl) {
    const __nv_bfloat16 a0 = __float2bfloat16_rn(h0), a1 = __float2bfloat16_rn(h1);
    bh = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
    bl = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h0 - __bfloat162float(a0))) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h1 - __bfloat162float(a1))) << 16);
  };
  mbar_wait(xbar, 0, abort_flag, a.status);

  // ------------------------------------------------------------ G: gate
  {
    const int n_st = g1 - g0;  // the first ns stages were issued in the setup
    issued_end = gsq + min(ns, n_st);
    for (int q = 0; q < n_st; ++q) {
      const int gs = gsq + q, slot = gs % ns;
      // warp 0's bias pair for this group, loaded before the wait
      float b0 = 0.f, b1 = 0.f;
      if (warp == 0 && a.tw.bias) {
        const int n = (g0 + q) * RW_G + 2 * (lane & 3);
        b0 = __ldg(a.tw.bias + n);
        b1 = __ldg(a.tw.bias + n + 1);
      }
      const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
      float cu[4];
      up_partial(ring_s + (uint32_t)(slot * SB) + lrow, ok, cu);
      float2* ub = ured + (q & 1) * RW_WARPS * 32;
      ub[warp * 32 + lane] = make_float2(cu[0], cu[1]);
      __syncthreads();
      if (q + ns < n_st) {
        issue_rows(gs + ns, a.W_gate, nullptr, RW_G, (g0 + q + ns) * RW_G);
        issued_end = gs + ns + 1;
      }
      if (warp == 0) {
        // warp 0 sums the warps' partials into the tile's staging block
        const int grp = g0 + q, p = grp / GPT;
        float u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int w = 0; w < RW_WARPS; ++w) {
          const float2 v = ub[w * 32 + lane];
          u0 += v.x;
          u1 += v.y;
        }
        float* gsg = a.gstage + ((size_t)p * 8 + (lane >> 2)) * 128 + (grp % GPT) * RW_G + 2 * (lane & 3);
        __stcg(gsg, u0);
        __stcg(gsg + 1, u1);
        // keep bits of (token lane/4, neurons 2(lane%4), +1), gathered into one byte per token
        const int t = lane >> 2;
        const bool k0 = t < T && fabsf(act_fn(u0 + b0, a.tw.act)) > a.tw.tau;
        const bool k1 = t < T && fabsf(act_fn(u1 + b1, a.tw.act)) > a.tw.tau;
        uint32_t bits = ((k0 ? 1u : 0u) | (k1 ? 2u : 0u)) << (2 * (lane & 3));
        bits |= __shfl_xor_sync(0xFFFFFFFFu, bits, 1);
        bits |= __shfl_xor_sync(0xFFFFFFFFu, bits, 2);
        if ((lane & 3) == 0) a.kbits[(size_t)t * NG + grp] = (uint8_t)bits;
      }
    }
    gsq += n_st;
  }
  // every gate value and keep bit in, every slice of out zeroed
  grid_barrier(a.gbar, abort_flag, a.status, bar_ok);

  // ------------------------------------------------------------ R: rows
  int* tpre = reinterpret_cast<int*>(sm + L.uni);
  uint4* ums = reinterpret_cast<uint4*>(sm + L.uni + (((P + 1) * 4 + 15) & ~15));
  int* nid = reinterpret_cast<int*>(ums + P);
  uint32_t* lmask = reinterpret_cast<uint32_t*>(nid + a.lcap);
  uint4* lval = reinterpret_cast<uint4*>(lmask + a.lcap);
  // per (token, tile) keep masks from the keep bits: counts, overflow tokens
  // ([TwELL] hybrid: a token overflows iff some tile keeps more than C),
  // then the union of the live (valid, not overflowing) tokens' masks
  uint4 km[8];
  if (tid == 0) {
    misc[50] = 0;
    misc[51] = 0;
  }
  __syncthreads();
  if (tid < P) {
    uint32_t ob = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      km[i] = i < T ? __ldcg(reinterpret_cast<const uint4*>(a.kbits + (size_t)i * NG) + tid) : make_uint4(0, 0, 0, 0);
      const int c = __popc(km[i].x) + __popc(km[i].y) + __popc(km[i].z) + __popc(km[i].w);
      if (c > C) ob |= 1u << i;
    }
    if (ob) atomicOr(reinterpret_cast<unsigned*>(&misc[51]), ob);
  }
  __syncthreads();
  if (tid == 0) misc[50] = (int)(((1u << T) - 1u) & ~(uint32_t)misc[51]);
  __syncthreads();
  const uint32_t live = (uint32_t)misc[50], obits = (uint32_t)misc[51];
  if (tid < P) {
    uint4 u = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((live >> i) & 1u) {
        u.x |= km[i].x;
        u.y |= km[i].y;
        u.z |= km[i].z;
        u.w |= km[i].w;
      }
    ums[tid] = u;
  }
  // overflow routing ([TwELL] hybrid): the overflow tokens, in token order,
  // take the dense channel (phase D below)
  if (s == 0 && tid == 0) {
    int o = 0;
    for (int i = 0; i < 8; ++i)
      if ((obits >> i) & 1u) a.ovf_list[o++] = i;
    *a.ovf_count = o;
  }
  __syncthreads();
  // exclusive prefix of the tile union counts; this CTA's rank range
  if (warp == 0) {
    int run = 0;
    for (int p0 = 0; p0 < P; p0 += 32) {
      const int p = p0 + lane;
      int c = 0;
      if (p < P) {
        const uint4 m = ums[p];
        c = __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
      }
      int inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, inc, o);
        if (lane >= o) inc += n;
      }
      if (p < P) tpre[p] = run + inc - c;
      run += __shfl_sync(0xFFFFFFFFu, inc, 31);
    }
    if (lane == 0) tpre[P] = run;
  }
  __syncthreads();
  // the TwELL records of tile s (and s + G, ...) by warps 0-3, the same
  // emission as the tile kernels'; the rows phase does not wait for them
  auto emit_tiles = [&]() {
    if (warp >= 4) return;
    for (int p = s; p < P; p += G) {
      float g[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = __ldcg(a.gstage + ((size_t)p * 8 + i) * 128 + tid);
      twell_tile32<8>(a.tw, g, p * 128 + tid, 0, tid, sm + L.emit, 1);
    }
  };
  {
    const int U = tpre[P];
    const int r0 = (int)((long long)U * s / G), r1 = (int)((long long)U * (s + 1) / G);
    if (r0 >= r1) emit_tiles();  // no rows for this CTA
    for (int c0 = r0; c0 < r1; c0 += a.lcap) {
      const int c1 = min(r1, c0 + a.lcap), Lc = c1 - c0;
      const int n_groups = (Lc + RW_G - 1) / RW_G;
      const int n_st = n_groups * 2;  // per group: its W_up rows, then its W_down rows
      for (int p = tid; p < P; p += blockDim.x) {
        if (tpre[p] <= c0 && c0 < tpre[p + 1]) misc[48] = p;
        if (tpre[p] < c1 && c1 <= tpre[p + 1]) misc[49] = p;
      }
      __syncthreads();
      const int pa = misc[48], pb = misc[49];
      for (int e = tid; e < (pb - pa + 1) * 128; e += blockDim.x) {
        const int p = pa + (e >> 7), bit = e & 127;
        const uint4 m = ums[p];
        if ((word4(m, bit >> 5) >> (bit & 31)) & 1u) {
          const int rank = tpre[p] + popc_below(m, bit);
          if (rank >= c0 && rank < c1) nid[rank - c0] = p * 128 + bit;
        }
      }
      for (int e = tid; e < Lc; e += blockDim.x) {
        lmask[e] = 0u;
        lval[e] = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
      auto issue_r = [&](int q) {
        const int n0 = (q >> 1) * RW_G;
        issue_rows(gsq + q, (q & 1) ? a.W_down : a.W_up, nid + n0, min(RW_G, Lc - n0), 0);
      };
      for (int q = 0; q < ns && q < n_st; ++q) issue_r(q);
      issued_end = gsq + min(ns, n_st);
      if (c0 == r0) emit_tiles();  // while the first stages are in flight
      // h's bf16 values v = bf16(sigma(g + b)) of the live tokens' kept
      // pairs of this chunk's neurons: one thread per (neuron, token)
      for (int e = tid; e < Lc * 8; e += blockDim.x) {
        const int r = e >> 3, i = e & 7;
        const int n = nid[r];
        if (!((live >> i) & 1u)) continue;
        if (!((a.kbits[(size_t)i * NG + (n >> 3)] >> (n & 7)) & 1u)) continue;
        const float gv = __ldcg(a.gstage + ((size_t)(n >> 7) * 8 + i) * 128 + (n & 127)) +
                         (a.tw.bias ? a.tw.bias[n] : 0.f);
        reinterpret_cast<uint16_t*>(&lval[r])[i] = __bfloat16_as_ushort(__float2bfloat16_rn(act_fn(gv, a.tw.act)));
        atomicOr(&lmask[r], 1u << i);
      }
      __syncthreads();
      for (int g = 0; g < n_groups; ++g) {
        const int n0 = g * RW_G, nn = min(RW_G, Lc - n0);
        uint32_t bh = 0u, bl = 0u;
        {  // up stage
          const int q = 2 * g, gs = gsq + q, slot = gs % ns;
          const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
          float cu[4];
          up_partial(ring_s + (uint32_t)(slot * SB) + lrow, ok, cu);
          ured[warp * 32 + lane] = make_float2(cu[0], cu[1]);
          __syncthreads();
          if (q + ns < n_st) {
            issue_r(q + ns);
            issued_end = gs + ns + 1;
          }
          const int tn = lane >> 2, rr = 2 * (lane & 3);
          float u0 = 0.f, u1 = 0.f;
#pragma unroll
          for (int w = 0; w < RW_WARPS; ++w) {
            const float2 v = ured[w * 32 + lane];
            u0 += v.x;
            u1 += v.y;
          }
          float hv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = rr + e, n = n0 + r;
            float h = 0.f;
            if (r < nn && ((lmask[n] >> tn) & 1u)) {
              const float v = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(&lval[n])[tn] << 16);
              h = v * (e ? u1 : u0);
            }
            hv[e] = h;
          }
          split_hilo(hv[0], hv[1], bh, bl);
        }
        {  // down stage
          const int q = 2 * g + 1, gs = gsq + q, slot = gs % ns;
          const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
          down_acc(ring_s + (uint32_t)(slot * SB) + lrow, ok, bh, bl);
          __syncthreads();
          if (q + ns < n_st) {
            issue_r(q + ns);
            issued_end = gs + ns + 1;
          }
        }
      }
      gsq += n_st;
      __syncthreads();
      if (*abort_flag) break;
    }
  }

  // -------------------------------------------- D: dense channel (overflow)
  if (obits != 0u && !*abort_flag) {
    const int n_st = 2 * (g1 - g0);  // per group: its W_gate rows, then its W_up rows
    auto issue_d1 = [&](int q) {
      issue_rows(gsq + q, (q & 1) ? a.W_up : a.W_gate, nullptr, RW_G, (g0 + (q >> 1)) * RW_G);
    };
    for (int q = 0; q < ns && q < n_st; ++q) issue_d1(q);
    issued_end = gsq + min(ns, n_st);
    for (int q = 0; q < n_st; ++q) {
      const int gs = gsq + q, slot = gs % ns;
      const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
      float cu[4];
      up_partial(ring_s + (uint32_t)(slot * SB) + lrow, ok, cu);
      float2* ub = ured + (q & 1) * RW_WARPS * 32;  // g partials, then u partials
      ub[warp * 32 + lane] = make_float2(cu[0], cu[1]);
      __syncthreads();
      if (q + ns < n_st) {
        issue_d1(q + ns);
        issued_end = gs + ns + 1;
      }
      if (q & 1) {
        // h_tj = bf16(sigma(g + b))·u where kept, for the overflow tokens; 0 otherwise
        if (warp == 0) {
          float gv[2] = {0.f, 0.f}, uv[2] = {0.f, 0.f};
#pragma unroll
          for (int w = 0; w < RW_WARPS; ++w) {
            const float2 vg = ured[w * 32 + lane], vu = ured[RW_WARPS * 32 + w * 32 + lane];
            gv[0] += vg.x;
            gv[1] += vg.y;
            uv[0] += vu.x;
            uv[1] += vu.y;
          }
          const int t = lane >> 2, j = (g0 + (q >> 1)) * RW_G + 2 * (lane & 3);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float gb = gv[e] + (a.tw.bias ? a.tw.bias[j + e] : 0.f);
            const float act = act_fn(gb, a.tw.act);
            const bool keep = ((obits >> t) & 1u) && fabsf(act) > a.tw.tau;
            const float v = __bfloat162float(__float2bfloat16_rn(act));
            a.hdense[(size_t)t * F + j + e] = keep ? v * uv[e] : 0.f;
          }
        }
        __syncthreads();  // the partials are read before the next group writes them
      }
    }
    gsq += n_st;
    // every overflow token's h is in
    grid_barrier(a.gbar, abort_flag, a.status, bar_ok);
    const int n_st2 = g1 - g0;
    for (int q = 0; q < ns && q < n_st2; ++q) issue_rows(gsq + q, a.W_down, nullptr, RW_G, (g0 + q) * RW_G);
    issued_end = gsq + min(ns, n_st2);
    for (int q = 0; q < n_st2; ++q) {
      const int gs = gsq + q, slot = gs % ns;
      // this lane's B fragment: h of token lane/4 at neurons 2(lane%4), +1 of the group
      const int j = (g0 + q) * RW_G + 2 * (lane & 3);
      const float2 hv = __ldcg(reinterpret_cast<const float2*>(a.hdense + (size_t)(lane >> 2) * F + j));
      uint32_t bh, bl;
      split_hilo(hv.x, hv.y, bh, bl);
      const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
      down_acc(ring_s + (uint32_t)(slot * SB) + lrow, ok, bh, bl);
      __syncthreads();
      if (q + ns < n_st2) {
        issue_rows(gs + ns, a.W_down, nullptr, RW_G, (g0 + q + ns) * RW_G);
        issued_end = gs + ns + 1;
      }
    }
    gsq += n_st2;
  }

  // drain copies still in flight (only after an abort): the last fill of every slot
  if (tid == 0 && *abort_flag) {
    for (int k = 0; k < ns && k < issued_end; ++k) {
      const int last = issued_end - 1 - k;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&full[last % ns], (uint32_t)((last / ns) & 1))) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) break;
      }
    }
  }
  __syncthreads();
  const bool okall = !*abort_flag;

  // partial y -> red[8][d] (rows padded by 4 floats against bank conflicts,
  // over the x block and the ring), then out by bulk reduce-add per token
  const int RP = d + 4;
  float* red = reinterpret_cast<float*>(sm + L.xs);
#pragma unroll
  for (int j = 0; j < RW_MAXJ; ++j) {
    const int row = 16 * (warp + RW_WARPS * j) + (lane >> 2);
    if (j < nj) {
      const int t = 2 * (lane & 3);
      red[t * RP + row] = acc[j][0];
      red[(t + 1) * RP + row] = acc[j][1];
      red[t * RP + row + 8] = acc[j][2];
      red[(t + 1) * RP + row + 8] = acc[j][3];
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (tid < nvalid && okall) {
    asm volatile("fence.proxy.async.global;" ::: "memory");  // after the other CTAs' zeroing of out
    bulk_reduce_add_f32(a.out + (size_t)tid * d, red + tid * RP, (uint32_t)d * 4u);
    bulk_commit();
    bulk_wait_all();
  }
}

}  // namespace sffn
