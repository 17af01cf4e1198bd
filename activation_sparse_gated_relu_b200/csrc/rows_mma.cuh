// Fused sparse up x down over the kept rows of a block of 8 tokens
// ([TwELL] "TwELL 減掉轉換開銷": one pass computes both projections and never
// stores h in global memory).
//
// One CTA (16 warps) takes a block of 8 tokens and a contiguous range of the
// block's union of kept neurons, ranked tile by tile from the union of the
// live (non-overflow) tokens' keep masks, so that every CTA streams the same
// number of rows.  CTA 0 of each block also routes the block's overflow
// tokens to the dense channel (list, count, gathered rows).
//
// Neurons are processed in groups of 8, and groups in pairs (A, B): the W_up
// rows of A, then of B, then the W_down rows of A and of B pass through a
// ring of shared-memory stages, one stage = 8 whole rows (8 x d bf16), each
// row brought by one 1-D bulk copy (8 KB at d = 4096: the copy size at which
// one SM's bulk-copy traffic reaches the HBM rate, where 2 KB pieces fall
// about a fifth short).  Rows are padded by 16 bytes so that ldmatrix is free
// of bank conflicts.  The warps issue the 8 copies of a stage in parallel;
// one CTA barrier frees both W_up stages of a pair (whose up product is one
// MMA chain over both) and another both W_down stages, and each freed slot is
// refilled at once with the stage nslot ahead.
//
// Both contractions are warp-level tensor-core MMAs (bf16 inputs, fp32
// accumulate) on the staged rows:
//   up:   u[16 neurons][8 tokens] = W_up rows · x^T over a pair of groups
//         (m16n8k16: the pair's 16 rows as M, the 8 tokens as N, both via
//         ldmatrix) -- warp w takes every 16th 16-wide k step; the 16 warps'
//         partial sums meet in shared memory, laid out so that every lane
//         adds up the 16 partials at its position in the down product's B
//         fragment (token lane/4, neurons 2 (lane%4) and +1);
//   h:    h_tj = v_tj·u_tj where (t, j) is kept, else 0, split into
//         hi = bf16(h) and lo = bf16(h - hi) (so the bf16 MMA operand loses at
//         most 2^-16 of h), straight into the down product's B fragment;
//   down: y^T[d][8 tokens] += W_down rows^T (ldmatrix.trans) · (h_hi + h_lo)
//         (m16n8k8, the 8 neurons as K) -- warp w owns every 16th 16-row
//         output tile, held in registers for the whole CTA.
// At the end the per-CTA partial y goes to out: plain stores when one CTA
// owns the block, otherwise bulk reduce-add copies, one per live token, that
// the bulk-copy engine adds into out at L2.  (Summing first over a
// thread-block cluster through distributed shared memory measured slower:
// its remote loads ran at about 40 GB/s per SM.)
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int RW_WARPS = 16;
constexpr int RW_THREADS = RW_WARPS * 32;
constexpr int RW_G = 8;             // neurons per group = rows per stage (up N, down K)
constexpr int RW_MAXJ = 16;         // k steps (up) and output tiles (down) per warp: d <= 4096
constexpr int RW_DIV = 256;         // d must be a multiple of 16 warps x 16
constexpr int RW_NSMAX = 6;         // ring slots at most

struct RowsArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* W_up;
  const __nv_bfloat16* W_down;
  const int16_t* count;
  const int16_t* idx;
  const __nv_bfloat16* val;
  const uint4* kmask;        // [T][n_tiles] 128-bit keep masks from the gate epilogue
  const uint32_t* ovf;       // [T] overflow epochs
  uint32_t epoch;
  // overflow routing (CTA 0 of every block): compacted list, count, gathered rows
  int* ovf_list;
  int* ovf_count;
  uint4* xo;                 // [T][d / 8] gathered x rows of overflow tokens
  const uint4* z;            // low-rank z rows to gather (or null)
  uint4* zo;
  int r_vec;
  int zero_ovf_rows;         // zero out's rows of overflow tokens (split down adds into them)
  float* out;
  int T, d, F, n_tiles, C;
  int atomic;
  int nslot, lcap;          // ring slots (<= RW_NSMAX), neuron-id list capacity
  uint32_t* status;
};

struct RowsSmem {
  // byte offsets inside the dynamic shared memory
  int xs, ring, bars, tpre, ums, nid, lmask, lval, ured, misc, total;
  __host__ __device__ static int pitch(int d) { return d * 2 + 16; }   // padded staged row (bytes)
  __host__ __device__ static int stage(int d) { return RW_G * pitch(d); }
  __host__ __device__ static RowsSmem make(int n_tiles, int lcap, int d, int nslot) {
    RowsSmem s;
    int o = 0;
    s.xs = o;    o += stage(d);           // the block's 8 x rows, staged like weight rows
    s.ring = o;  o += nslot * stage(d);
    s.bars = o;  o += ((RW_NSMAX + 1) * 8 + 15) & ~15;  // ring slots, then the x rows; keeps 16-B alignment
    s.tpre = o;  o += ((n_tiles + 1) * 4 + 15) & ~15;
    s.ums = o;   o += n_tiles * 16;
    s.nid = o;   o += lcap * 4;
    s.lmask = o; o += lcap * 4;
    s.lval = o;  o += lcap * 16;
    s.ured = o;  o += 2 * RW_WARPS * 32 * 8;  // the partials of a pair of groups
    s.misc = o;  o += 64 * 4;
    s.total = o;
    return s;
  }
};

__device__ __forceinline__ uint32_t word4(const uint4& m, int q) {
  return q == 0 ? m.x : q == 1 ? m.y : q == 2 ? m.z : m.w;
}

// number of set bits of the 128-bit mask below position bit
__device__ __forceinline__ int popc_below(const uint4& m, int bit) {
  const int q = bit >> 5;
  int c = __popc(word4(m, q) & ((1u << (bit & 31)) - 1u));
  if (q > 0) c += __popc(m.x);
  if (q > 1) c += __popc(m.y);
  if (q > 2) c += __popc(m.z);
  return c;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D[16x8] += A[16x16] (row) · B[16x8] (col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D[16x8] += A[16x8] (row) · B[8x8] (col), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_1688(float* c, uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__global__ void __launch_bounds__(RW_THREADS, 1) k_rows(const RowsArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int d = a.d;
  const int ns = max(2, min(a.nslot, RW_NSMAX));  // ring slots, all kept in flight
  const RowsSmem L = RowsSmem::make(a.n_tiles, a.lcap, d, ns);
  const int RS = RowsSmem::pitch(d), SB = RowsSmem::stage(d);
  uint8_t* ring = sm + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* xbar = full + RW_NSMAX;
  int* tpre = reinterpret_cast<int*>(sm + L.tpre);
  uint4* ums = reinterpret_cast<uint4*>(sm + L.ums);
  int* nid = reinterpret_cast<int*>(sm + L.nid);
  uint32_t* lmask = reinterpret_cast<uint32_t*>(sm + L.lmask);
  uint4* lval = reinterpret_cast<uint4*>(sm + L.lval);
  float2* ured = reinterpret_cast<float2*>(sm + L.ured);
  int* misc = reinterpret_cast<int*>(sm + L.misc);
  volatile int* abort_flag = misc + 40;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = a.n_tiles, b = blockIdx.y, S = gridDim.x, s = blockIdx.x;
  const int tb0 = b * 8;
  const int nj = d / RW_DIV;         // k steps (up) and output tiles (down) of each warp

  griddep_wait();  // keep masks, TwELL and overflow epochs come from the gate
  // 1. barriers; the block's x rows go out at once as bulk copies into the x
  // block (staged like weight rows: the up product's A operand comes from
  // them by ldmatrix), rows beyond T are zeroed; then the live tokens of the
  // block (valid, not overflowing) and the union of their keep masks, tile
  // by tile
  const int nvalid = max(0, min(8, a.T - tb0));
  if (tid == 0) {
    for (int i = 0; i < ns; ++i) mbar_init(&full[i], 1);
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_expect_tx(xbar, (uint32_t)(nvalid * d * 2));
    for (int t = 0; t < nvalid; ++t)
      bulk_g2s(sm + L.xs + t * RS, a.x + (size_t)(tb0 + t) * d, (uint32_t)d * 2u, xbar);
  }
  for (int e = tid; e < (8 - nvalid) * (d >> 3); e += blockDim.x) {
    const int t = nvalid + e / (d >> 3), v = e % (d >> 3);
    *reinterpret_cast<uint4*>(sm + L.xs + t * RS + v * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  uint4 km[8];
  if (tid < P) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      km[i] = tb0 + i < a.T ? a.kmask[(size_t)(tb0 + i) * P + tid] : make_uint4(0, 0, 0, 0);
  }
  if (warp == 0) {
    const int t = tb0 + lane;
    const bool v = lane < 8 && t < a.T;
    const bool o = v && a.ovf[t] == a.epoch;
    const uint32_t vb = __ballot_sync(0xFFFFFFFFu, v), obb = __ballot_sync(0xFFFFFFFFu, o);
    if (lane == 0) {
      misc[50] = (int)(vb & ~obb);
      misc[51] = (int)obb;
      misc[52] = 0;
    }
  }
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
  // overflow routing ([TwELL] hybrid): CTA 0 of the block ranks the block's
  // overflow tokens after those of earlier blocks, lists them and gathers
  // their rows for the dense channel; the last block writes the count
  if (s == 0) {
    int before = 0;
    for (int t = tid; t < tb0; t += blockDim.x) before += a.ovf[t] == a.epoch ? 1 : 0;
    if (before) atomicAdd(&misc[52], before);
  }
  __syncthreads();
  if (s == 0 && (obits != 0u || b == (int)gridDim.y - 1)) {
    const int base = misc[52];
    if (b == (int)gridDim.y - 1 && tid == 0) *a.ovf_count = base + __popc(obits);
    const int dv = d >> 3, d4 = d >> 2;
    int o = base;
    for (int i = 0; i < 8; ++i) {
      if (!((obits >> i) & 1u)) continue;
      const int t = tb0 + i;
      if (tid == 0) a.ovf_list[o] = t;
      const uint4* xr = reinterpret_cast<const uint4*>(a.x) + (size_t)t * dv;
      for (int v = tid; v < dv; v += blockDim.x) a.xo[(size_t)o * dv + v] = xr[v];
      if (a.z)
        for (int v = tid; v < a.r_vec; v += blockDim.x) a.zo[(size_t)o * a.r_vec + v] = a.z[(size_t)t * a.r_vec + v];
      if (a.zero_ovf_rows)
        for (int v = tid; v < d4; v += blockDim.x)
          reinterpret_cast<float4*>(a.out)[(size_t)t * d4 + v] = make_float4(0.f, 0.f, 0.f, 0.f);
      ++o;
    }
  }
  // 2. exclusive prefix of the tile union counts
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
  const int U = tpre[P];
  const int r0 = (int)((long long)U * s / S), r1 = (int)((long long)U * (s + 1) / S);

  float acc[RW_MAXJ][4];
#pragma unroll
  for (int j = 0; j < RW_MAXJ; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[j][k] = 0.f;

  const uint32_t ring_s = smem_u32(ring);
  int sbase = 0;        // stages of earlier chunks (uniform), for slot and parity
  int issued_end = 0;   // stages issued so far (global numbering, uniform)

  for (int c0 = r0; c0 < r1; c0 += a.lcap) {
    const int c1 = min(r1, c0 + a.lcap), Lc = c1 - c0;
    const int n_groups = (Lc + RW_G - 1) / RW_G;
    // groups go in pairs (A, B): stages W_up A, W_up B, W_down A, W_down B, so
    // that one barrier frees two stages and the up products share x; a
    // missing last B has no rows
    const int n_pairs = (n_groups + 1) >> 1;
    const int n_stages = n_pairs * 4;
    // a. tiles overlapping [c0, c1): pa holds rank c0, pb holds rank c1 - 1
    for (int p = tid; p < P; p += blockDim.x) {
      if (tpre[p] <= c0 && c0 < tpre[p + 1]) misc[48] = p;
      if (tpre[p] < c1 && c1 <= tpre[p + 1]) misc[49] = p;
    }
    __syncthreads();
    const int pa = misc[48], pb = misc[49];
    // b. neuron ids of ranks [c0, c1), one thread per (tile, bit)
    const int nbits = (pb - pa + 1) * 128;
    for (int e = tid; e < nbits; e += blockDim.x) {
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
    // c. stage q of this chunk (group 2 (q / 4) + q % 2; W_up rows if q % 4 < 2):
    // warp w (lane 0) copies row w; padding rows copy nothing (their u is
    // never used, and the down product masks their stale rows out)
    auto issue_stage = [&](int q) {
      if (q >= n_stages || lane != 0 || warp >= RW_G) return;
      const int gs = sbase + q, slot = gs % ns;
      const int g = 2 * (q >> 2) + (q & 1);
      const bool up = (q & 2) == 0;
      const uint32_t bytes = (uint32_t)d * 2u;
      const int n0 = g * RW_G, nn = max(0, min(RW_G, Lc - n0));
      if (warp == 0) mbar_expect_tx(&full[slot], bytes * (uint32_t)nn);
      if (warp < nn)
        bulk_g2s(ring + (size_t)slot * SB + warp * RS, (up ? a.W_up : a.W_down) + (size_t)nid[n0 + warp] * d, bytes,
                 &full[slot]);
    };
    for (int q = 0; q < ns; ++q) issue_stage(q);
    issued_end = sbase + min(ns, n_stages);
    // d. scatter TwELL values of the live tokens: one thread per (slot, token, tile)
    {
      const int n_items = a.C * 8 * (pb - pa + 1);
      for (int e = tid; e < n_items; e += blockDim.x) {
        const int sl = e % a.C, rest = e / a.C;
        const int i = rest & 7, p = pa + (rest >> 3);
        if (!((live >> i) & 1u)) continue;
        const size_t rec = (size_t)(tb0 + i) * P + p;
        const int cnt = min((int)a.count[rec], a.C);
        if (sl >= cnt) continue;
        const int bit = (int)a.idx[rec * a.C + sl] - p * 128;
        if (bit < 0 || bit >= 128) {
          atomicOr(a.status, DEV_ERR_RANGE);
          continue;
        }
        const int rank = tpre[p] + popc_below(ums[p], bit);
        if (rank >= c0 && rank < c1) {
          reinterpret_cast<uint16_t*>(&lval[rank - c0])[i] =
              reinterpret_cast<const uint16_t*>(a.val)[rec * a.C + sl];
          atomicOr(&lmask[rank - c0], 1u << i);
        }
      }
    }
    __syncthreads();
    if (sbase == 0) mbar_wait(xbar, 0, abort_flag, a.status);  // the x rows have landed

    // e. consume the stages in order, a pair of groups at a time; one barrier
    // frees both W_up stages, another both W_down stages.
    // ldmatrix lanes: 0-7 rows 0-7 at column c, 8-15 rows 0-7 at column c + 8,
    // 16-31 the same for the warp's next k step (or output tile)
    const uint32_t lrow = (uint32_t)((lane & 7) * RS + 16 * ((lane >> 3) & 1) + 32 * warp);
    const uint32_t xsl = smem_u32(sm + L.xs) + lrow;
    const uint32_t hi_off = (lane >> 4) ? 32u * RW_WARPS : 0u;  // lanes 16-31: the next k step / tile
    auto stage_wait = [&](int q) {
      const int gs = sbase + q;
      return mbar_wait(&full[gs % ns], (uint32_t)((gs / ns) & 1), abort_flag, a.status);
    };
    auto stage_addr = [&](int q) { return ring_s + (uint32_t)(((sbase + q) % ns) * SB) + lrow; };
    // h of one group as the down product's B fragment (hi, lo), from the 16
    // warps' partials at this lane's fragment position (token lane/4, neurons
    // 2(lane%4) and +1)
    auto group_h = [&](const float2* ub, int n0, int nn, uint32_t& bh, uint32_t& bl) {
      const int tn = lane >> 2, r0 = 2 * (lane & 3);
      float u0 = 0.f, u1 = 0.f;
#pragma unroll
      for (int w = 0; w < RW_WARPS; ++w) {
        const float2 v = ub[w * 32 + lane];
        u0 += v.x;
        u1 += v.y;
      }
      float hv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = r0 + e, n = n0 + r;
        float h = 0.f;
        if (r < nn && ((lmask[n] >> tn) & 1u)) {
          const float v = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(&lval[n])[tn] << 16);
          h = v * (e ? u1 : u0);
        }
        hv[e] = h;
      }
      const __nv_bfloat16 h0 = __float2bfloat16_rn(hv[0]), h1 = __float2bfloat16_rn(hv[1]);
      bh = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      bl = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hv[0] - __bfloat162float(h0))) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hv[1] - __bfloat162float(h1))) << 16);
    };
    // y^T[d][token] += W_down rows^T · h over a group's nn neurons: this
    // lane's A fragments hold rows 2(lane%4) and +1, and the rows of padding
    // neurons (stale slot data; h is zero there, and 0 * inf would not be)
    // are cleared
    auto down_group = [&](uint32_t sbs, uint32_t bh, uint32_t bl, int nn) {
      const int r0 = 2 * (lane & 3);
      const uint32_t keep = (r0 < nn ? 0xFFFFu : 0u) | (r0 + 1 < nn ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int j = 0; j < RW_MAXJ; j += 2) {
        if (j < nj) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(sbs + 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u), a0, a1, a2, a3);
          a0 &= keep;
          a1 &= keep;
          a2 &= keep;
          a3 &= keep;
          mma_bf16_1688(acc[j], a0, a1, bh);
          mma_bf16_1688(acc[j], a0, a1, bl);
          if (j + 1 < nj) {
            mma_bf16_1688(acc[j + 1], a2, a3, bh);
            mma_bf16_1688(acc[j + 1], a2, a3, bl);
          }
        }
      }
    };
    for (int pr = 0; pr < n_pairs; ++pr) {
      const int q0 = 4 * pr;
      const int nA = RW_G * 2 * pr, nB = nA + RW_G;
      const int nnA = min(RW_G, Lc - nA), nnB = max(0, min(RW_G, Lc - nB));
      // up: u[neuron][token] partials of both groups over this warp's k
      // steps, the pair's 16 rows as the MMA's M (group A rows 0-7, group B
      // rows 8-15) and the 8 tokens as its N: no half-empty tiles.  Rows of
      // padding neurons (and all of B's when the pair has one group) hold
      // stale data; each D row depends on its own A row only, and group_h
      // reads none of them.
      const bool okA = stage_wait(q0);
      const bool okB = stage_wait(q0 + 1);
      float cu[4] = {0.f, 0.f, 0.f, 0.f};
      if (okA && okB) {
        const uint32_t sa = stage_addr(q0), sb = stage_addr(q0 + 1);
#pragma unroll
        for (int j = 0; j < RW_MAXJ; j += 2) {
          if (j < nj) {
            const uint32_t off = 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u);
            uint32_t x0, x1, x2, x3, a0, a1, a2, a3, b0, b1, b2, b3;
            ldsm_x4(xsl + off, x0, x1, x2, x3);
            ldsm_x4(sa + off, a0, a1, a2, a3);
            ldsm_x4(sb + off, b0, b1, b2, b3);
            mma_bf16_16816(cu, a0, b0, a1, b1, x0, x1);
            if (j + 1 < nj) mma_bf16_16816(cu, a2, b2, a3, b3, x2, x3);
          }
        }
      }
      {  // into ured as [group][warp][token][neuron]: group_h's float2 at
         // (warp, lane) is its token's two neurons 2 (lane % 4) and + 1
        float* uf = reinterpret_cast<float*>(ured);
        const int n = lane >> 2, t = 2 * (lane & 3);
        uf[(warp * 8 + t) * 8 + n] = cu[0];
        uf[(warp * 8 + t + 1) * 8 + n] = cu[1];
        uf[RW_WARPS * 64 + (warp * 8 + t) * 8 + n] = cu[2];
        uf[RW_WARPS * 64 + (warp * 8 + t + 1) * 8 + n] = cu[3];
      }
      __syncthreads();
      issue_stage(q0 + ns);  // both W_up slots are free
      issue_stage(q0 + 1 + ns);
      if (q0 + ns < n_stages) issued_end = sbase + min(n_stages, q0 + 2 + ns);
      uint32_t bhA, blA, bhB = 0u, blB = 0u;
      group_h(ured, nA, nnA, bhA, blA);
      if (nnB > 0) group_h(ured + RW_WARPS * 32, nB, nnB, bhB, blB);
      // down: both groups into the partial y
      if (stage_wait(q0 + 2)) down_group(stage_addr(q0 + 2), bhA, blA, nnA);
      if (stage_wait(q0 + 3) && nnB > 0) down_group(stage_addr(q0 + 3), bhB, blB, nnB);
      __syncthreads();
      issue_stage(q0 + 2 + ns);  // both W_down slots are free
      issue_stage(q0 + 3 + ns);
      if (q0 + 2 + ns < n_stages) issued_end = sbase + min(n_stages, q0 + 4 + ns);
    }
    sbase += n_stages;
    __syncthreads();
    if (*abort_flag) break;
  }
  // drain copies still in flight (only after an abort): the last fill of every slot
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
  __syncthreads();
  const bool okall = !*abort_flag;

  // 4. partial y -> red[8][d] (fp32, over the x rows and the free ring; rows
  // padded by 4 floats, so that the four token rows a warp writes at once
  // fall in different banks), then out
  const int RP = d + 4, n4p = RP >> 2;
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
  const int n4 = d >> 2;
  if (a.atomic) {
    // the bulk-copy engine adds each live token's partial row into out at L2
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < 8 && ((live >> tid) & 1u) && okall) {
      bulk_reduce_add_f32(a.out + (size_t)(tb0 + tid) * d, red + tid * RP, (uint32_t)d * 4u);
      bulk_commit();
      bulk_wait_all();
    }
  } else {
    __syncthreads();
    for (int e = tid; e < 8 * n4; e += blockDim.x) {
      const int t = e / n4, q = e - t * n4;
      if (!((live >> t) & 1u) || !okall) continue;
      reinterpret_cast<float4*>(a.out + (size_t)(tb0 + t) * d)[q] = reinterpret_cast<const float4*>(red)[t * n4p + q];
    }
  }
}

}  // namespace sffn
