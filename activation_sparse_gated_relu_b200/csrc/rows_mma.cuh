// Fused sparse up x down over the kept rows of a block of 8 tokens
// ([TwELL] "TwELL 減掉轉換開銷": one pass computes both projections and never
// stores h in global memory).
//
// One CTA (16 warps) takes a block of 8 tokens and a contiguous range of the
// block's union of kept neurons, ranked tile by tile from the union of the
// live (non-overflow) tokens' keep masks, so that every CTA streams the same
// number of rows.  CTA 0 of each block also routes the block's overflow
// tokens to the dense channel (list, count, gathered rows).  Neurons are
// processed in groups of 16.  A group's W_up rows and then its W_down rows
// (contiguous, neuron-major) pass through a ring of shared-memory stages, one
// stage = the same 1024-column chunk of the 16 rows (16 KB... 32 KB), each
// row chunk brought by a 1-D bulk copy that one of the 16 warps issues, so
// the copies of a stage go out in parallel; rows are padded by 16 bytes so
// ldmatrix is free of bank conflicts.  One CTA barrier per stage releases its
// slot, which the warps refill at once with the stage NS ahead.
//
// Both contractions are warp-level tensor-core MMAs (m16n8k16, bf16 inputs,
// fp32 accumulate) on the staged rows:
//   up:   u[16 neurons][8 tokens] = W_up rows (ldmatrix) · x^T -- warp w takes
//         every 16th 16-wide k step, whose x fragments it keeps in registers;
//         the 16 warps' partial sums meet in shared memory and every warp
//         adds them up itself;
//   h:    h_tj = v_tj·u_tj where (t, j) is kept, else 0, split into
//         hi = bf16(h) and lo = bf16(h - hi) (so the bf16 MMA operand loses at
//         most 2^-16 of h);
//   down: y^T[d][8 tokens] += W_down rows^T (ldmatrix.trans) · (h_hi + h_lo)
//         -- warp w owns every 16th 16-row output tile, held in registers for
//         the whole CTA.
// At the end the per-CTA partial y goes to out: plain stores when one CTA
// owns the block, otherwise summed over the CTAs of a thread-block cluster
// through distributed shared memory (each CTA of the cluster owns one column
// slice) and added into out by bulk reduce-add copies, one per live token.
#pragma once

#include "ptx.cuh"

namespace sffn {

constexpr int RW_WARPS = 16;
constexpr int RW_THREADS = RW_WARPS * 32;
constexpr int RW_G = 16;            // neurons per group (MMA M of up, K of down)
constexpr int RW_CHUNK = 1024;      // columns of a row per stage
constexpr int RW_MAXC = 4;          // chunks per row: d <= 4096
constexpr int RW_MAXJ = RW_CHUNK / 256;  // k steps (or output tiles) per warp and chunk
constexpr int RW_DIV = 256;         // d must be a multiple of 16 warps x 16
constexpr int RW_NS = 6;            // ring stages

struct RowsArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* W_up;
  const __nv_bfloat16* W_down;
  const __nv_bfloat16* zero_row;   // >= 2 KB of zeros (rows of padding neurons)
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
  int nslot, lcap;
  uint32_t* status;
};

struct RowsSmem {
  // byte offsets inside the dynamic shared memory
  int ring, bars, tpre, ums, nid, lmask, lval, ured, misc, total;
  static constexpr int RSTRIDE = RW_CHUNK * 2 + 16;    // padded staged row chunk (bytes)
  static constexpr int STAGE = RW_G * RSTRIDE;
  __host__ __device__ static RowsSmem make(int n_tiles, int lcap) {
    RowsSmem s;
    int o = 0;
    s.ring = o;  o += RW_NS * STAGE;
    s.bars = o;  o += RW_NS * 8;
    s.tpre = o;  o += ((n_tiles + 1) * 4 + 15) & ~15;
    s.ums = o;   o += n_tiles * 16;
    s.nid = o;   o += lcap * 4;
    s.lmask = o; o += lcap * 4;
    s.lval = o;  o += lcap * 16;
    s.ured = o;  o += RW_WARPS * 32 * 16;
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

__global__ void __launch_bounds__(RW_THREADS, 1) k_rows(const RowsArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const RowsSmem L = RowsSmem::make(a.n_tiles, a.lcap);
  constexpr int RS = RowsSmem::RSTRIDE, SB = RowsSmem::STAGE;
  uint8_t* ring = sm + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  int* tpre = reinterpret_cast<int*>(sm + L.tpre);
  uint4* ums = reinterpret_cast<uint4*>(sm + L.ums);
  int* nid = reinterpret_cast<int*>(sm + L.nid);
  uint32_t* lmask = reinterpret_cast<uint32_t*>(sm + L.lmask);
  uint4* lval = reinterpret_cast<uint4*>(sm + L.lval);
  float4* ured = reinterpret_cast<float4*>(sm + L.ured);
  int* misc = reinterpret_cast<int*>(sm + L.misc);
  volatile int* abort_flag = misc + 40;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = a.n_tiles, b = blockIdx.y, S = gridDim.x, s = blockIdx.x;
  const int tb0 = b * 8;
  const int d = a.d;
  const int nchunk = (d + RW_CHUNK - 1) / RW_CHUNK;
  const int spg = 2 * nchunk;        // stages per group: up chunks, then down chunks

  griddep_wait();  // keep masks, TwELL and overflow epochs come from the gate
  // 1. live tokens of the block (valid, not overflowing) and the union of
  // their keep masks, tile by tile; barriers
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
      for (int i = 0; i < RW_NS; ++i) mbar_init(&full[i], 1);
      *abort_flag = 0;
      fence_mbar_init();
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
  // x^T fragments of this warp's k steps (16(w + 16 j) in every chunk), in
  // registers; zero beyond T
  uint32_t xb[RW_MAXC][RW_MAXJ][2];
  {
    const int t = tb0 + (lane >> 2);
#pragma unroll
    for (int c = 0; c < RW_MAXC; ++c)
#pragma unroll
      for (int j = 0; j < RW_MAXJ; ++j) {
        xb[c][j][0] = xb[c][j][1] = 0u;
        const int k = c * RW_CHUNK + 16 * (warp + RW_WARPS * j);
        if (k < d && t < a.T) {
          const uint32_t* xr = reinterpret_cast<const uint32_t*>(a.x + (size_t)t * d + k + 2 * (lane & 3));
          xb[c][j][0] = xr[0];
          xb[c][j][1] = xr[4];
        }
      }
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

  float acc[RW_MAXC][RW_MAXJ][4];
#pragma unroll
  for (int c = 0; c < RW_MAXC; ++c)
#pragma unroll
    for (int j = 0; j < RW_MAXJ; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[c][j][k] = 0.f;

  const uint32_t ring_s = smem_u32(ring);
  int sbase = 0;        // stages of earlier chunks (uniform), for slot and parity
  int issued_end = 0;   // stages issued so far (global numbering, uniform)

  for (int c0 = r0; c0 < r1; c0 += a.lcap) {
    const int c1 = min(r1, c0 + a.lcap), Lc = c1 - c0;
    const int n_groups = (Lc + RW_G - 1) / RW_G;
    const int n_stages = n_groups * spg;
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
    // c. stage q of this chunk: warp w (lane 0) copies row w's column chunk;
    // padding rows of W_down stages copy zeros, of W_up stages nothing
    auto issue_stage = [&](int q) {
      if (q >= n_stages || lane != 0) return;
      const int gs = sbase + q, slot = gs % RW_NS;
      const int g = q / spg, st = q - g * spg;
      const bool up = st < nchunk;
      const int ch = up ? st : st - nchunk;
      const int cols = min(RW_CHUNK, d - ch * RW_CHUNK);
      const uint32_t bytes = (uint32_t)cols * 2u;
      const int n0 = g * RW_G, nn = min(RW_G, Lc - n0);
      const int nrows = up ? nn : RW_G;
      if (warp == 0) mbar_expect_tx(&full[slot], bytes * (uint32_t)nrows);
      if (warp < nrows) {
        const __nv_bfloat16* src =
            warp < nn ? (up ? a.W_up : a.W_down) + (size_t)nid[n0 + warp] * d + ch * RW_CHUNK : a.zero_row;
        bulk_g2s(ring + (size_t)slot * SB + warp * RS, src, bytes, &full[slot]);
      }
    };
    for (int q = 0; q < RW_NS; ++q) issue_stage(q);
    issued_end = sbase + min(RW_NS, n_stages);
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

    // e. consume the stages in order; one barrier per stage releases its slot
    for (int g = 0; g < n_groups; ++g) {
      const int n0 = g * RW_G, nn = min(RW_G, Lc - n0);
      float cu[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t bh0 = 0u, bh1 = 0u, bl0 = 0u, bl1 = 0u;
#pragma unroll
      for (int st = 0; st < 2 * RW_MAXC; ++st) {
        const bool up = st < RW_MAXC;
        const int ch = up ? st : st - RW_MAXC;
        if (ch >= nchunk) continue;
        const int q = g * spg + (up ? ch : nchunk + ch);
        const int gs = sbase + q, slot = gs % RW_NS;
        const bool ok = mbar_wait(&full[slot], (uint32_t)((gs / RW_NS) & 1), abort_flag, a.status);
        const uint32_t sbs = ring_s + (uint32_t)(slot * SB);
        if (ok && up) {
          // A rows = the 16 neurons; lane supplies row (lane & 7) + 8((lane >> 3) & 1)
          const uint32_t arow = sbs + (uint32_t)(((lane & 7) + 8 * ((lane >> 3) & 1)) * RS);
#pragma unroll
          for (int j = 0; j < RW_MAXJ; ++j) {
            const int kk = 16 * (warp + RW_WARPS * j);        // chunk-local k
            if (ch * RW_CHUNK + kk < d) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4(arow + (kk + 8 * (lane >> 4)) * 2, a0, a1, a2, a3);
              mma_bf16_16816(cu, a0, a1, a2, a3, xb[ch][j][0], xb[ch][j][1]);
            }
          }
        } else if (ok) {
          // A = stored [neuron k][d] rows; lane supplies k = (lane & 7) + 8(lane >> 4)
          const uint32_t krow = sbs + (uint32_t)(((lane & 7) + 8 * (lane >> 4)) * RS);
          const int moff = 8 * ((lane >> 3) & 1);
#pragma unroll
          for (int j = 0; j < RW_MAXJ; ++j) {
            const int mm = 16 * (warp + RW_WARPS * j);        // chunk-local output row
            if (ch * RW_CHUNK + mm < d) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(krow + (mm + moff) * 2, a0, a1, a2, a3);
              mma_bf16_16816(acc[ch][j], a0, a1, a2, a3, bh0, bh1);
              mma_bf16_16816(acc[ch][j], a0, a1, a2, a3, bl0, bl1);
            }
          }
        }
        const bool last_up = up && ch == nchunk - 1;
        if (last_up) ured[warp * 32 + lane] = make_float4(cu[0], cu[1], cu[2], cu[3]);
        __syncthreads();
        // the slot is free: refill it with the stage RW_NS ahead
        issue_stage(q + RW_NS);
        if (sbase + q + RW_NS < sbase + n_stages) issued_end = sbase + q + RW_NS + 1;
        if (last_up) {
          // h for the group: lane needs neurons k0 = 2(l&3) (+1, +8, +9) of token l>>2;
          // element (row r, col c) of a warp's partial lives in lane 4(r&7) + (c>>1),
          // register (c&1) + 2(r>>3)
          const int tn = lane >> 2, k0 = 2 * (lane & 3);
          float hv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = k0 + (e & 1) + 8 * (e >> 1);
            const float* pu = reinterpret_cast<const float*>(ured) + (4 * (r & 7) + (tn >> 1)) * 4 + (tn & 1) +
                              2 * (r >> 3);
            float u = 0.f;
#pragma unroll
            for (int w = 0; w < RW_WARPS; ++w) u += pu[w * 128];
            const int n = n0 + r;
            float h = 0.f;
            if (r < nn && ((lmask[n] >> tn) & 1u)) {
              const float v = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(&lval[n])[tn] << 16);
              h = v * u;
            }
            hv[e] = h;
          }
          uint32_t hb[4], lb[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(hv[e]);
            hb[e] = (uint32_t)__bfloat16_as_ushort(hi);
            lb[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hv[e] - __bfloat162float(hi)));
          }
          bh0 = hb[0] | (hb[1] << 16);
          bh1 = hb[2] | (hb[3] << 16);
          bl0 = lb[0] | (lb[1] << 16);
          bl1 = lb[2] | (lb[3] << 16);
          __syncthreads();  // every warp has read the partials before the next group writes them
        }
      }
    }
    sbase += n_stages;
    __syncthreads();
    if (*abort_flag) break;
  }
  // drain copies still in flight (only after an abort): the last fill of every slot
  if (tid == 0 && *abort_flag) {
    for (int k = 0; k < RW_NS && k < issued_end; ++k) {
      const int last = issued_end - 1 - k;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&full[last % RW_NS], (uint32_t)((last / RW_NS) & 1))) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) break;
      }
    }
  }
  __syncthreads();
  const bool okall = !*abort_flag;

  // 4. partial y -> red[8][d] (fp32, in the free ring), then out
  float* red = reinterpret_cast<float*>(ring);
#pragma unroll
  for (int c = 0; c < RW_MAXC; ++c)
#pragma unroll
    for (int j = 0; j < RW_MAXJ; ++j) {
      const int row = c * RW_CHUNK + 16 * (warp + RW_WARPS * j) + (lane >> 2);
      if (row < d) {
        const int t = 2 * (lane & 3);
        red[t * d + row] = acc[c][j][0];
        red[(t + 1) * d + row] = acc[c][j][1];
        red[t * d + row + 8] = acc[c][j][2];
        red[(t + 1) * d + row + 8] = acc[c][j][3];
      }
    }
  const uint32_t CS = cluster_nctarank();
  const int n4 = d >> 2;
  if (a.atomic && CS > 1) {
    // the cluster's CTAs sum their partials over distributed shared memory,
    // each one column slice, into a slice buffer behind red; the bulk-copy
    // engine then adds each live token's slice row into out at L2
    cluster_sync();
    const uint32_t rank = cluster_ctarank();
    const int q0 = (int)(n4 * rank / CS), q1 = (int)(n4 * (rank + 1) / CS);
    const int width = q1 - q0;
    const uint32_t red_s = smem_u32(red);
    float4* slice = reinterpret_cast<float4*>(red + 8 * d);
    for (int e0 = tid; e0 < 8 * width; e0 += blockDim.x) {
      const int t = e0 / width, q = q0 + (e0 - t * width);
      if (!((live >> t) & 1u)) continue;
      const uint32_t off = (uint32_t)((t * n4 + q) * 16);
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (uint32_t r = 0; r < CS; ++r) {
        const float4 v = ld_shared_cluster_f4(mapa_shared(red_s + off, r));
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      slice[e0] = sum;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < 8 && ((live >> tid) & 1u) && okall) {
      bulk_reduce_add_f32(a.out + (size_t)(tb0 + tid) * d + 4 * q0, slice + tid * width, (uint32_t)width * 16u);
      bulk_commit();
      bulk_wait_all();
    }
    cluster_sync();
  } else if (a.atomic) {
    fence_proxy_async_smem();
    __syncthreads();
    if (tid < 8 && ((live >> tid) & 1u) && okall) {
      bulk_reduce_add_f32(a.out + (size_t)(tb0 + tid) * d, red + tid * d, (uint32_t)d * 4u);
      bulk_commit();
      bulk_wait_all();
    }
  } else {
    __syncthreads();
    for (int e = tid; e < 8 * n4; e += blockDim.x) {
      const int t = e / n4, q = e - t * n4;
      if (!((live >> t) & 1u) || !okall) continue;
      reinterpret_cast<float4*>(a.out + (size_t)(tb0 + t) * d)[q] = reinterpret_cast<const float4*>(red)[t * n4 + q];
    }
  }
}

}  // namespace sffn
