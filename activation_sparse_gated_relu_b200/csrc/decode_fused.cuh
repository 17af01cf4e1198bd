// The whole forward for one block of up to 8 tokens in one persistent launch
// ([TwELL] sections "TwELL 減掉轉換開銷" and "Hybrid 應對非均勻稀疏"): the gate
// with its TwELL emission, the overflow flags and the fused sparse up x down
// of every kept neuron.
//
// With one CTA per SM, every phase streams whole weight rows through shared-
// memory stages (8 rows of 8 KB per stage, one bulk copy per row) and
// computes on warp MMAs, as the separate row-streaming kernels do
// (gate_rows.cuh, rows_mma.cuh).  There is no grid-wide barrier:
//
//   G  CTA s gates an equal range of 8-neuron groups of W_gate through three
//      slots (the two ring slots and the x block: x sits in registers while
//      the partial y is not yet live).  Its warp 0 turns each group's gate
//      values into the TwELL staging block (fp32, shared with the other CTAs
//      of the tile) and into CTA s's own row list: one record per neuron of
//      the range that some token keeps (the neuron, its token mask and the 8
//      tokens' bf16 values bf16(sigma(g + b))), copied to global memory as it
//      grows.  The list is complete when the range is, with no other CTA's
//      results.
//   R  the list's 8-record items go through the two ring slots as a W_up
//      stage and a W_down stage each, with x back in the x block; u and h
//      stay in registers, y accumulates in registers.  The first item's
//      stages are issued while the last gate stages are still in use, so the
//      stream does not pause between G and R.  Each list is published as
//      soon as its gate phase ends (its length, tagged with the forward's
//      epoch, after a release fence); its owner keeps the first half of its
//      items and takes the rest in claims of one, and a CTA whose own list is
//      exhausted steals half of the largest remainder of another CTA's list:
//      the work of an SM that gated slowly, or whose range keeps more
//      neurons, spreads over the others.
//   y  every CTA zeroes a slice of out when it starts (its publication
//      announces that too); each CTA's partial y goes into out by bulk
//      reduce-add copies at L2, eight pieces per token row.
//   TwELL: while those copies run, warps 4-7 of CTA s write the records of
//      the tiles [e_lo, e_hi) assigned to it, from the staged gate values of
//      the CTAs that gated them (complete once those have published).
//
// Overflow tokens.  The hybrid format sends a token that keeps more than C
// neurons of some tile to a dense channel, which computes
// y = sum_j h_j W_down[j] over all d_ff neurons with h_j = 0 where the token
// does not keep j.  Here a token's row list has no capacity, so the same sum
// over the kept neurons is what R computes for every token: an overflow
// token's dense-channel result comes out of the same stream, and it costs at
// most its extra kept rows rather than a second pass over all three matrices.
// The TwELL records and the per-token overflow flags are still written
// exactly as the format defines them; the flags are the routing's record.
//
// The only waits on other CTAs are a steal while some list is not yet
// published, the zeroed slices of out and the completeness of a tile to
// write; all CTAs are resident (the host launches one per SM), every wait is
// bounded, and a timeout sets the status word.
#pragma once

#include "epilogues.cuh"
#include "rows_mma.cuh"

namespace sffn {

struct DecodeArgs {
  const __nv_bfloat16* x;        // [T][d]
  const __nv_bfloat16* W_gate;   // [F][d]
  const __nv_bfloat16* W_up;
  const __nv_bfloat16* W_down;
  TwellParams tw;                // T, F, n_tiles, C, bias, tau, act, TwELL outputs, keep masks, epochs
  float* gstage;                 // [n_tiles][8][128] fp32 gate values (before the bias)
  int* sched;                    // [decode_sched_ints(n_tiles, grid)] zero before the first launch
  uint32_t* wl_id;               // [grid][maxr] published records: neuron | token mask << 24
  uint4* wl_val;                 // [grid][maxr] published records: 8 tokens' bf16 values
  int maxr;                      // records per list (>= 8 x the most groups a CTA gates)
  float* out;                    // [T][d]
  int d;
  uint32_t* status;
  unsigned long long wait_ns;    // limit of the waits on other CTAs
  int phantom;                   // test hook: CTAs counted in the grid that never run (0 or 1)
};

// Scheduler words, in ints from the start of DecodeArgs::sched.  A list
// length carries the forward's epoch, so a value left by an earlier launch
// never reads as this launch's, and its owner sets the claim count before it
// publishes the length: nothing needs resetting between launches.
struct DecodeSched {
  int P, G;
  __host__ __device__ int pub(int v) const { return v; }        // (epoch << 16) | (list length + 1)
  __host__ __device__ int claim(int v) const { return G + v; }  // items taken from list v
  __host__ __device__ int total() const { return 2 * G; }
};
__host__ __device__ inline int decode_sched_ints(int P, int G) { return DecodeSched{P, G}.total(); }

constexpr int DEC_NS = 2;  // ring slots (the gate also streams through the x block)

struct DecodeSmem {
  int xs, ring, bars, lid, lval, ib, emit, ured, vcnt, misc, total;
  __host__ __device__ static DecodeSmem make(int C, int maxr, int d) {
    DecodeSmem s;
    int o = 0;
    s.xs = o;    o += RowsSmem::stage(d);
    s.ring = o;  o += DEC_NS * RowsSmem::stage(d);
    s.bars = o;  o += ((RW_NSMAX + 1) * 8 + 15) & ~15;
    s.lid = o;   o += (maxr * 4 + 15) & ~15;       // own list: packed ids
    s.lval = o;  o += maxr * 16;                   // own list: values
    s.ib = o;    o += 2 * 8 * 4 + 2 * 8 * 16;      // two item buffers (ids, then values)
    s.emit = o;  o += twell_smem(8, C);
    s.ured = o;  o += 2 * RW_WARPS * 32 * 8;
    s.vcnt = o;  o += RW_THREADS * 4;              // steal scan: list lengths
    s.misc = o;  o += 64 * 4;
    s.total = o;
    return s;
  }
};

// misc[] slots
enum : int {
  DM_ABORT = 0, DM_CNT = 1, DM_RISS = 2, DM_EMOK = 3, DM_CHV = 4, DM_CHK = 5, DM_CHK1 = 6,
  DM_VCNT = 7, DM_OWNMORE = 8, DM_RES = 9, DM_LK0 = 12, DM_XLK = 15,
  DM_RED = 16
};

__global__ void __launch_bounds__(RW_THREADS, 1) k_decode(const DecodeArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int d = a.d, T = a.tw.T, F = a.tw.F, P = a.tw.n_tiles;
  const DecodeSmem L = DecodeSmem::make(a.tw.C, a.maxr, d);
  const int RS = RowsSmem::pitch(d), SB = RowsSmem::stage(d);
  uint8_t* ring = sm + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* xbar = full + RW_NSMAX;
  uint32_t* lid = reinterpret_cast<uint32_t*>(sm + L.lid);
  uint4* lval = reinterpret_cast<uint4*>(sm + L.lval);
  uint32_t* ib_id = reinterpret_cast<uint32_t*>(sm + L.ib);   // [2][8]
  uint4* ib_val = reinterpret_cast<uint4*>(sm + L.ib + 64);   // [2][8]
  float2* ured = reinterpret_cast<float2*>(sm + L.ured);
  int* vcs = reinterpret_cast<int*>(sm + L.vcnt);
  int* misc = reinterpret_cast<int*>(sm + L.misc);
  volatile int* abort_flag = misc + DM_ABORT;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, s = blockIdx.x;
  const DecodeSched S{P, G + 1};  // one spare slot: the test hook's CTA that never runs
  const int GS = G + a.phantom;    // the CTAs whose lists and zeroed slices are awaited
  int* sc = a.sched;
  const int nj = d / RW_DIV;
  const int NG = F / RW_G;
  const int g0 = (int)((long long)NG * s / G), g1 = (int)((long long)NG * (s + 1) / G);
  const int n_g = g1 - g0;  // gate stages: stage k < n_g holds W_gate rows of group g0 + k
  constexpr int GPT = 128 / RW_G;  // 8-neuron groups per TwELL tile
  const uint32_t ring_s = smem_u32(ring);
  const uint32_t lrow = (uint32_t)((lane & 7) * RS + 16 * ((lane >> 3) & 1) + 32 * warp);
  const uint32_t hi_off = (lane >> 4) ? 32u * RW_WARPS : 0u;
  const uint32_t xsl = smem_u32(sm + L.xs) + lrow;

  // ---------------------------------------------------------------- setup
  // The gate streams through three slots, the two ring slots and the x
  // block: x moves into registers for the gate (the partial y is not live
  // yet), and the x block's last gate stage hands it back to a second copy of
  // x for the rows phase, which streams through the two ring slots.
  const int nvalid = min(8, T);
  const bool x_slot = n_g >= 3;  // the gate uses the x block as a third slot
  auto g_fills = [&](int sl) { return n_g > sl ? (n_g - sl + 2) / 3 : 0; };    // gate stages in slot sl
  auto g_last = [&](int sl) { return n_g > sl ? sl + 3 * ((n_g - 1 - sl) / 3) : -1; };
  auto slot_at = [&](int sl) -> uint8_t* { return sl < 2 ? ring + (size_t)sl * SB : sm + L.xs; };
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&full[i], 1);
    mbar_init(xbar, 1);
    misc[DM_ABORT] = 0;
    misc[DM_LK0] = misc[DM_LK0 + 1] = misc[DM_LK0 + 2] = -1;
    fence_mbar_init();
    // the gate's first stages: the weights stay unchanged for the handle's
    // life, so they load before the previous grid on the stream has finished
    for (int q = 0; q < 2 && q < n_g; ++q) {
      mbar_expect_tx(&full[q], (uint32_t)(RW_G * d * 2));
      misc[DM_LK0 + q] = 0;
      for (int r = 0; r < RW_G; ++r)
        bulk_g2s(ring + (size_t)q * SB + r * RS, a.W_gate + (size_t)((g0 + q) * RW_G + r) * d, (uint32_t)d * 2u, &full[q]);
    }
  }
  griddep_wait();  // x, out and the workspace belong to the stream order
  if (tid == 0) {
    mbar_expect_tx(xbar, (uint32_t)(nvalid * d * 2));
    misc[DM_XLK] = 1;
    for (int t = 0; t < nvalid; ++t) bulk_g2s(sm + L.xs + t * RS, a.x + (size_t)t * d, (uint32_t)d * 2u, xbar);
  }
  for (int e = tid; e < (8 - nvalid) * (d >> 3); e += blockDim.x) {
    const int t = nvalid + e / (d >> 3), v = e % (d >> 3);
    *reinterpret_cast<uint4*>(sm + L.xs + t * RS + v * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  {  // every CTA adds its partial y into all of out at the end; the list's
     // publication (below) tells the others this slice is zero
    const long long n4 = (long long)T * d / 4;
    const long long q0 = n4 * s / G, q1 = n4 * (s + 1) / G;
    for (long long e = q0 + tid; e < q1; e += blockDim.x)
      reinterpret_cast<float4*>(a.out)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();

  // gate stage q: 8 consecutive W_gate rows into slot q % 3 (lane 0 of warps 0-7, one row each)
  auto issue_gate = [&](int q) {
    if (lane != 0 || warp >= RW_G) return;
    const int sl = q % 3;
    if (warp == 0) {
      mbar_expect_tx(&full[sl], (uint32_t)(RW_G * d * 2));
      misc[DM_LK0 + sl] = (q / 3) & 1;
    }
    bulk_g2s(slot_at(sl) + warp * RS, a.W_gate + (size_t)((g0 + q) * RW_G + warp) * d, (uint32_t)d * 2u, &full[sl]);
  };
  // rows stage kr: item kr/2's W_up rows (kr even) or W_down rows (kr odd)
  // from item buffer b into ring slot kr % 2.  Absent records copy nothing:
  // their slot rows keep stale weights, which the products mask out (a
  // shared zero row, copied by every CTA at once, made one L2 slice a hot
  // spot at the end of the rows phase).
  auto r_par = [&](int kr) { return (uint32_t)((g_fills(kr & 1) + (kr >> 1)) & 1); };
  auto issue_item = [&](int kr, int b) {
    if (lane != 0 || warp >= RW_G) return;
    const int sl = kr & 1;
    if (warp == 0) {
      int present = 0;
#pragma unroll
      for (int r = 0; r < RW_G; ++r) present += ib_id[b * 8 + r] != 0u;
      mbar_expect_tx(&full[sl], (uint32_t)(present * d * 2));
      misc[DM_LK0 + sl] = (int)r_par(kr);
    }
    const uint32_t id = ib_id[b * 8 + warp];
    if (id == 0u) return;
    const __nv_bfloat16* W = (kr & 1) ? a.W_down : a.W_up;
    bulk_g2s(ring + (size_t)sl * SB + warp * RS, W + (size_t)(id & 0xFFFFFFu) * d, (uint32_t)d * 2u, &full[sl]);
  };
  // up-style product of a staged stage: the warp's partial of
  // u^T[token lane/4][rows 2(lane%4), +1] over its k steps, x from the x block
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
  // h as bf16 hi + lo halves (the down product's B fragment)
  auto split_hilo = [](float h0, float h1, uint32_t& bh, uint32_t& bl) {
    const __nv_bfloat16 a0 = __float2bfloat16_rn(h0), a1 = __float2bfloat16_rn(h1);
    bh = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
    bl = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h0 - __bfloat162float(a0))) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(h1 - __bfloat162float(a1))) << 16);
  };
  // x into registers for the gate: the A fragments of the warp's k steps
  uint32_t xr[RW_MAXJ / 2][4];
  mbar_wait(xbar, 0, abort_flag, a.status);
#pragma unroll
  for (int jp = 0; jp < RW_MAXJ / 2; ++jp) {
    const int j = 2 * jp;
    if (j < nj) {
      ldsm_x4(xsl + 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u), xr[jp][0], xr[jp][1], xr[jp][2], xr[jp][3]);
    } else {
      xr[jp][0] = xr[jp][1] = xr[jp][2] = xr[jp][3] = 0u;
    }
  }
  __syncthreads();  // every warp holds x: the x block is the gate's third slot
  if (x_slot) issue_gate(2);

  // ------------------------------------------------------------ G: gate
  // warp 0's running state: records in the own list, stages of the first
  // item already issued
  int cnt = 0, r_iss = 0;
  // warp 0 turns group qq's partials (in ured[qq & 1]) into its gate values,
  // keep decisions and list records
  auto gate_group = [&](int qq, float b0, float b1) {
    const float2* ub = ured + (qq & 1) * RW_WARPS * 32;
    const int grp = g0 + qq, p = grp / GPT;
    float u0 = 0.f, u1 = 0.f;
#pragma unroll
    for (int w = 0; w < RW_WARPS; ++w) {
      const float2 v = ub[w * 32 + lane];
      u0 += v.x;
      u1 += v.y;
    }
    // g^T[token lane/4][rows 2(lane%4), +1] into the tile's staging block
    const int t = lane >> 2, c = lane & 3;
    float* gsg = a.gstage + ((size_t)p * 8 + t) * 128 + (grp % GPT) * RW_G + 2 * c;
    __stcg(gsg, u0);
    __stcg(gsg + 1, u1);
    // keep decisions ([TwELL]: |sigma(g + b)| > tau) and the records of the
    // group's rows that some token keeps, appended in row order
    const float a0 = act_fn(u0 + b0, a.tw.act), a1 = act_fn(u1 + b1, a.tw.act);
    const bool k0 = t < T && fabsf(a0) > a.tw.tau, k1 = t < T && fabsf(a1) > a.tw.tau;
    const uint32_t bal0 = __ballot_sync(0xFFFFFFFFu, k0), bal1 = __ballot_sync(0xFFFFFFFFu, k1);
    uint32_t ra = 0u;  // row r = 2c' + e is kept by token t' iff bit 4t' + c' of bal_e
#pragma unroll
    for (int r = 0; r < RW_G; ++r)
      if (((((r & 1) ? bal1 : bal0) >> (r >> 1)) & 0x11111111u) != 0u) ra |= 1u << r;
    if ((ra >> (2 * c)) & 1u)
      reinterpret_cast<uint16_t*>(&lval[cnt + __popc(ra & ((1u << (2 * c)) - 1u))])[t] =
          k0 ? __bfloat16_as_ushort(__float2bfloat16_rn(a0)) : (uint16_t)0;
    if ((ra >> (2 * c + 1)) & 1u)
      reinterpret_cast<uint16_t*>(&lval[cnt + __popc(ra & ((2u << (2 * c)) - 1u))])[t] =
          k1 ? __bfloat16_as_ushort(__float2bfloat16_rn(a1)) : (uint16_t)0;
    if (lane < RW_G && ((ra >> lane) & 1u)) {
      const uint32_t bal = (lane & 1) ? bal1 : bal0;
      uint32_t tm = 0u;
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) tm |= ((bal >> (4 * tt + (lane >> 1))) & 1u) << tt;
      lid[cnt + __popc(ra & ((1u << lane) - 1u))] = (uint32_t)(grp * RW_G + lane) | (tm << 24);
    }
    __syncwarp();
    if (lane < __popc(ra)) {  // the new records go out now; the publication orders them
      const int i = cnt + lane;
      a.wl_id[(size_t)s * a.maxr + i] = lid[i];
      a.wl_val[(size_t)s * a.maxr + i] = lval[i];
    }
    cnt += __popc(ra);
    __syncwarp();
  };
  // warp 0: the first item (own records 0-7) into ring slots 0 and 1 (rows
  // stages 0 and 1) once their last gate stages are read and the list has it
  auto early_rows = [&](int q_read) {
    while (r_iss < 2 && g_last(r_iss) <= q_read && cnt >= 8) {
      if (lane == 0) {
        mbar_expect_tx(&full[r_iss], (uint32_t)(RW_G * d * 2));
        misc[DM_LK0 + r_iss] = (int)r_par(r_iss);
      }
      if (lane < RW_G)
        bulk_g2s(ring + (size_t)r_iss * SB + lane * RS,
                 (r_iss ? a.W_down : a.W_up) + (size_t)(lid[lane] & 0xFFFFFFu) * d, (uint32_t)d * 2u, &full[r_iss]);
      ++r_iss;
    }
  };
  for (int q = 0; q < n_g; ++q) {
    const int sl = q % 3;
    float b0 = 0.f, b1 = 0.f;  // warp 0's bias pair, loaded before the wait
    if (warp == 0 && a.tw.bias) {
      const int n = (g0 + q) * RW_G + 2 * (lane & 3);
      b0 = __ldg(a.tw.bias + n);
      b1 = __ldg(a.tw.bias + n + 1);
    }
    const bool ok = mbar_wait(&full[sl], (uint32_t)((q / 3) & 1), abort_flag, a.status);
    // this stage's partials: two chains of MMAs against x in registers
    float ca[4] = {0.f, 0.f, 0.f, 0.f}, cb[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      const uint32_t sbs = smem_u32(slot_at(sl)) + lrow;
#pragma unroll
      for (int jp = 0; jp < RW_MAXJ / 2; ++jp) {
        const int j = 2 * jp;
        if (j < nj) {
          uint32_t b0r, b1r, b2r, b3r;
          ldsm_x4(sbs + 32u * RW_WARPS * j + (j + 1 < nj ? hi_off : 0u), b0r, b1r, b2r, b3r);
          mma_bf16_16816(ca, xr[jp][0], 0u, xr[jp][1], 0u, b0r, b1r);
          if (j + 1 < nj) mma_bf16_16816(cb, xr[jp][2], 0u, xr[jp][3], 0u, b2r, b3r);
        }
      }
    }
    ured[(q & 1) * RW_WARPS * 32 + warp * 32 + lane] = make_float2(ca[0] + cb[0], ca[1] + cb[1]);
    __syncthreads();
    // the slot is free: the stream's next gate stage, or x back into the x block
    if (q + 3 < n_g) {
      issue_gate(q + 3);
    } else if (sl == 2 && tid == 0) {
      mbar_expect_tx(xbar, (uint32_t)(nvalid * d * 2));
      misc[DM_XLK] = 2;
      for (int t = 0; t < nvalid; ++t) bulk_g2s(sm + L.xs + t * RS, a.x + (size_t)t * d, (uint32_t)d * 2u, xbar);
    }
    if (warp == 0) {
      early_rows(q);
      gate_group(q, b0, b1);
    }
  }
  if (n_g > 0 && warp == 0) early_rows(n_g - 1);
  if (x_slot) {  // the second copy of x: rows of absent tokens are zero again
    for (int e = tid; e < (8 - nvalid) * (d >> 3); e += blockDim.x) {
      const int t = nvalid + e / (d >> 3), v = e % (d >> 3);
      *reinterpret_cast<uint4*>(sm + L.xs + t * RS + v * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  float acc[RW_MAXJ][4];  // the partial y: live from here on
#pragma unroll
  for (int j = 0; j < RW_MAXJ; ++j)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[j][k] = 0.f;
  // down product of a staged stage of 8 W_down rows with h (bh, bl) into
  // acc; keep (per 16-bit half) clears the rows of absent records, whose
  // slot rows hold stale data (h is zero there, and 0 * inf would not be)
  auto down_acc = [&](uint32_t sbs, bool ok, uint32_t bh, uint32_t bl, uint32_t keep) {
    if (!ok) return;
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
  if (tid == 0) {  // warp 0's totals; the claim state starts on the own list
    const int items = (cnt + 7) >> 3;
    misc[DM_CNT] = cnt;
    misc[DM_RISS] = r_iss;
    misc[DM_CHV] = s;
    misc[DM_CHK] = 0;
    misc[DM_CHK1] = min(items, max(1, (items + 1) >> 1));
    misc[DM_VCNT] = cnt;
    misc[DM_OWNMORE] = misc[DM_CHK1] < items;
  }
  __syncthreads();

  // ------------------------------------------------------ own list, steals
  const int cnt_own = misc[DM_CNT], r_issued = misc[DM_RISS];
  const int items_own = (cnt_own + 7) >> 3;
  const int k_pre = min(items_own, max(1, (items_own + 1) >> 1));  // items the owner keeps outright
  const uint32_t epoch = a.tw.epoch;
  // Publication of the own list (its length, tagged with the epoch, after the
  // claim count and a release fence that also covers the records, the gate
  // values and the zeroed slice of out), right away: a CTA that gated late
  // is the one whose remainder the others wait for.  Measured against
  // publishing once the first item's stages were under way: 1 us less per
  // forward at 1, 4 and 8 tokens.
  bool all_seen = false;    // uniform: a steal scan found every list published
  if (tid == 0) {
    sc[S.claim(s)] = k_pre;
    fence_acq_rel_gpu();
    atomicExch(sc + S.pub(s), (int)(((epoch & 0xFFFFu) << 16) | (uint32_t)(cnt_own + 1)));
  }

  // The next item into item buffer `buf` (block-wide).  Returns ACQ_GOT, or
  // ACQ_NONE when no list anywhere has work left, or (only when `wait` is
  // false) ACQ_LATER when nothing is stealable yet but some lists are still
  // being gated: the caller has an item in flight and asks again, waiting,
  // once that item is done.  The items of the current claim come first (one
  // barrier); then own items, one per claim; then the largest published
  // remainder, half of it per steal.  Only tid 0 writes the claim state in
  // misc, between barriers.
  enum { ACQ_NONE = 0, ACQ_GOT = 1, ACQ_LATER = 2 };
  auto acquire = [&](int buf, bool wait) -> int {
    if (misc[DM_CHK] >= misc[DM_CHK1]) {
      if (__syncthreads_or(*abort_flag)) return ACQ_NONE;
      if (tid == 0) {
        int got = 0;
        if (misc[DM_OWNMORE]) {
          const int c = atomicAdd(sc + S.claim(s), 1);
          if (c < items_own) {
            misc[DM_CHV] = s;
            misc[DM_CHK] = c;
            misc[DM_CHK1] = c + 1;
            misc[DM_VCNT] = cnt_own;
            got = 1;
          } else {
            misc[DM_OWNMORE] = 0;
          }
        }
        misc[DM_RES] = got;
      }
      __syncthreads();
      if (!misc[DM_RES]) {
        uint64_t t0 = 0;
        if (tid == 0) t0 = globaltimer();
        for (;;) {
          int key = -1;
          bool unpub = false;
          if (tid < GS && tid != s) {
            const uint32_t pv = (uint32_t)ld_acquire_gpu(sc + S.pub(tid));
            const int len = (int)(pv & 0xFFFFu) - 1;
            if ((pv >> 16) != (epoch & 0xFFFFu) || len < 0) {
              unpub = true;  // not yet published in this launch
            } else {
              vcs[tid] = len;
              const int rem = ((len + 7) >> 3) - __ldcg(sc + S.claim(tid));
              if (rem > 0) key = (rem << 9) | tid;
            }
          }
#pragma unroll
          for (int o = 16; o; o >>= 1) key = max(key, __shfl_xor_sync(0xFFFFFFFFu, key, o));
          if (lane == 0) misc[DM_RED + warp] = key;
          const int n_unpub = __syncthreads_count(unpub);
          if (tid == 0) {
            int best = -1;
            for (int w = 0; w < RW_WARPS; ++w) best = max(best, misc[DM_RED + w]);
            int res = 0;  // 0: look again, 1: claimed, 2: no work left (3: and every list seen), 4: later
            if (best >= 0) {
              const int v = best & 511, vc = vcs[v], it = (vc + 7) >> 3;
              const int m = max(1, (best >> 9) >> 1);
              const int c = atomicAdd(sc + S.claim(v), m);
              if (c < it) {
                misc[DM_CHV] = v;
                misc[DM_CHK] = c;
                misc[DM_CHK1] = min(c + m, it);
                misc[DM_VCNT] = vc;
                res = 1;
              }
            } else if (n_unpub > 0) {  // lists still being gated: wait for them, bounded
              if (!wait) {
                res = 4;
              } else if (globaltimer() - t0 > a.wait_ns) {
                atomicOr(a.status, DEV_ERR_TIMEOUT);
                *abort_flag = 1;
                res = 2;
              } else {
                __nanosleep(256);
              }
            } else {
              res = 3;
            }
            misc[DM_RES] = res;
          }
          __syncthreads();
          if (misc[DM_RES] != 0) break;
        }
        const int res = misc[DM_RES];
        if (res == 4) return ACQ_LATER;
        if (res >= 2) {
          all_seen = res == 3;
          return ACQ_NONE;
        }
      }
    }
    const int v = misc[DM_CHV], k = misc[DM_CHK], vc = misc[DM_VCNT];
    if (tid < RW_G) {
      const int i = k * RW_G + tid;
      uint32_t id = 0u;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (i < vc) {
        if (v == s) {
          id = lid[i];
          val = lval[i];
        } else {
          id = __ldcg(a.wl_id + (size_t)v * a.maxr + i);
          val = __ldcg(a.wl_val + (size_t)v * a.maxr + i);
        }
      }
      ib_id[buf * 8 + tid] = id;
      ib_val[buf * 8 + tid] = val;
    }
    __syncthreads();  // the item buffer is complete; every thread has read the claim state
    if (tid == 0) misc[DM_CHK] = k + 1;  // read again only after the loop's next barrier
    return ACQ_GOT;
  };

  // ------------------------------------------------------------ R: rows
  // rows stage 2i is item i's W_up stage, 2i + 1 its W_down stage
  const bool have_first = acquire(0, true) == ACQ_GOT;
  if (have_first)
    for (int r = r_issued; r < 2; ++r) issue_item(r, 0);  // those G did not issue
  if (x_slot) mbar_wait(xbar, 1, abort_flag, a.status);  // the second copy of x
  if (have_first) {
    int kr = 0, cur = 0;
    __syncthreads();  // the claim state acquire(0) left
    int nx = acquire(1, false);
    for (;;) {
      const bool have_next = nx == ACQ_GOT;
      uint32_t bh, bl, keep;
      {  // W_up stage: u of the item's rows, then h = v·u where the token keeps the row
        const int sl = kr & 1;
        const bool ok = mbar_wait(&full[sl], r_par(kr), abort_flag, a.status);
        float cu[4];
        up_partial(ring_s + (uint32_t)(sl * SB) + lrow, ok, cu);
        ured[warp * 32 + lane] = make_float2(cu[0], cu[1]);
        __syncthreads();
        if (have_next) issue_item(kr + 2, cur ^ 1);
        float u0 = 0.f, u1 = 0.f;
#pragma unroll
        for (int w = 0; w < RW_WARPS; ++w) {
          const float2 v = ured[w * 32 + lane];
          u0 += v.x;
          u1 += v.y;
        }
        const int tn = lane >> 2, rr = 2 * (lane & 3);
        float hv[2];
        keep = 0u;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t id = ib_id[cur * 8 + rr + e];
          if (id != 0u) keep |= 0xFFFFu << (16 * e);
          float h = 0.f;
          if ((id >> (24 + tn)) & 1u) {
            const float v = __uint_as_float(
                (uint32_t)reinterpret_cast<const uint16_t*>(&ib_val[cur * 8 + rr + e])[tn] << 16);
            h = v * (e ? u1 : u0);
          }
          hv[e] = h;
        }
        split_hilo(hv[0], hv[1], bh, bl);
      }
      {  // W_down stage: y += h·W_down
        const int k = kr + 1, sl = k & 1;
        const bool ok = mbar_wait(&full[sl], r_par(k), abort_flag, a.status);
        down_acc(ring_s + (uint32_t)(sl * SB) + lrow, ok, bh, bl, keep);
        __syncthreads();
        if (have_next) issue_item(kr + 3, cur ^ 1);
      }
      kr += 2;
      if (nx == ACQ_LATER) {  // nothing in flight now: wait for a list, then issue its stages
        nx = acquire(cur ^ 1, true);
        if (nx == ACQ_GOT) {
          issue_item(kr, cur ^ 1);
          issue_item(kr + 1, cur ^ 1);
        }
      }
      if (nx != ACQ_GOT) break;
      cur ^= 1;
      nx = acquire(cur ^ 1, false);
    }
  }
  // This CTA streams no more weights: the next forward's launch may begin
  // (its CTAs take an SM as ours leave and load their first gate stages
  // while the output copies of this one run).
  griddep_launch();

  // ------------------------------------------------------------- TwELL
  // ([TwELL] "TwELL 減掉轉換開銷") CTA s writes the records of tiles [e_lo,
  // e_hi) with warps 4-7, the tile kernels' emission from the staged gate
  // values, while the reduce copies of y run.  A tile is complete once the
  // CTAs that gated its groups have published their lists (the last steal
  // scan usually saw them all).  The emission also flags each token that
  // keeps more than C neurons of the tile (the hybrid routing: in this kernel
  // such a token's kept rows were in the row lists like any other's).
  const int e_lo = (int)(((long long)s * P + G - 1) / G), e_hi = (int)(((long long)(s + 1) * P + G - 1) / G);
  const bool emitter = warp >= 4 && warp < 8 && e_lo < e_hi;
  const int et = tid - 128;
  float eg[8];
  if (emitter) {
    if (et == 0) {
      int good = !*abort_flag;
      if (good && !all_seen) {
        // the CTA that gates group g: the v with g0(v) <= g < g1(v)
        auto gater = [&](int g) {
          int v = (int)((long long)g * G / NG);
          while (v + 1 < G && (int)((long long)NG * (v + 1) / G) <= g) ++v;
          while (v > 0 && (int)((long long)NG * v / G) > g) --v;
          return v;
        };
        const uint64_t t0 = globaltimer();
        for (int v = gater(e_lo * GPT); v <= gater(e_hi * GPT - 1) && good; ++v) {
          for (;;) {
            const uint32_t pv = (uint32_t)ld_acquire_gpu(sc + S.pub(v));
            if ((pv >> 16) == (epoch & 0xFFFFu) && (pv & 0xFFFFu) != 0u) break;
            if (globaltimer() - t0 > a.wait_ns) {
              atomicOr(a.status, DEV_ERR_TIMEOUT);
              good = 0;
              break;
            }
            __nanosleep(128);
          }
        }
      }
      misc[DM_EMOK] = good;
    }
    named_bar_sync(1, 128);
    if (misc[DM_EMOK]) {  // the first tile's values, loading while y goes out
      const float b = a.tw.bias ? __ldg(a.tw.bias + e_lo * 128 + et) : 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) eg[i] = __ldcg(a.gstage + ((size_t)e_lo * 8 + i) * 128 + et) + b;
    }
  }

  // ---------------------------------------------------------------- y out
  // drain copies still in flight (only after an abort): the last x copy and
  // the last fill of every slot (misc holds the parity of each last phase)
  if (tid == 0 && *abort_flag) {
    const uint64_t tx = globaltimer();
    while (!mbar_try_wait(xbar, (uint32_t)((misc[DM_XLK] - 1) & 1))) {
      if (globaltimer() - tx > SFFN_WAIT_LIMIT_NS) break;
    }
    for (int sl = 0; sl < 3; ++sl) {
      const int par = misc[DM_LK0 + sl];
      if (par < 0) continue;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&full[sl], (uint32_t)par)) {
        if (globaltimer() - t0 > SFFN_WAIT_LIMIT_NS) break;
      }
    }
  }
  __syncthreads();
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
  // every CTA's slice of out is zero (it published its list after zeroing;
  // the last steal scan may have seen every list already)
  if (tid < GS && !all_seen) {
    const uint64_t t0 = globaltimer();
    for (;;) {
      const uint32_t pv = (uint32_t)ld_acquire_gpu(sc + S.pub(tid));
      if ((pv >> 16) == (epoch & 0xFFFFu) && (pv & 0xFFFFu) != 0u) break;
      if (globaltimer() - t0 > a.wait_ns) {
        atomicOr(a.status, DEV_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      __nanosleep(64);
    }
  }
  const bool okall = !__syncthreads_or(*abort_flag);
  // eight pieces per token row, each CTA starting at a different piece so
  // that the grid's adds spread over the output's L2 lines
  if (tid < nvalid * 8 && okall) {
    const int t = tid >> 3, c = ((tid & 7) + s) & 7, n = d >> 3;
    asm volatile("fence.proxy.async.global;" ::: "memory");  // after the other CTAs' zeroing of out
    bulk_reduce_add_f32(a.out + (size_t)t * d + c * n, red + t * RP + c * n, (uint32_t)n * 4u);
    bulk_commit();
    bulk_wait_read();  // the grid's end completes the writes
  }
  if (emitter && misc[DM_EMOK]) {
    TwellParams twb = a.tw;  // the emission gets g + b
    twb.bias = nullptr;
    for (int p = e_lo; p < e_hi; ++p) {
      float g[8];
      if (p == e_lo) {
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = eg[i];
      } else {
        const float b = a.tw.bias ? __ldg(a.tw.bias + p * 128 + et) : 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = __ldcg(a.gstage + ((size_t)p * 8 + i) * 128 + et) + b;
      }
      twell_tile32<8>(twb, g, p * 128 + et, 0, et, sm + L.emit, 1);
    }
  }
}

}  // namespace sffn
