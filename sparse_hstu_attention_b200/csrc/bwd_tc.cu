// SLA HSTU attention backward on the 5th-generation tensor cores (tcgen05).
//
// With x_ij = alpha q_i.k_j, P_ij = M SiLU(x)/N and dP_ij = dO_i.v_j:
//   dV_j = sum_i P_ij dO_i,   dK_j = sum_i dS_ij q_i,   dQ_i = sum_j dS_ij k_j,
//   dS_ij = M dP_ij SiLU'(x_ij) alpha/N
// (the chain rule through "Bending the Scaling Law Curve in Large-Scale
// Recommendation Systems", section 3, Eq. 3, under the SLA mask of section
// 4.2.1, Eq. 7).  With h = x/2, t = tanh(h) and u = 1 + t: SiLU(x) = h u and
// SiLU'(x) = (u/2)(1 + 2h - h u); one MUFU op per score.
//
// Two launches of one kernel template, neither using atomics on the data:
//   KV pass: a resident 128-key tile (K, V) meets streamed 64-row query tiles
//     (Q, dO):  S^T = K Q^T, dP^T = V dO^T  ->  P^T, dS^T (bf16, TMEM)
//     -> dV += P^T dO, dK += dS^T Q, both accumulated in TMEM.
//   Q pass: a resident 128-row query tile (Q, dO) meets streamed 64-key tiles
//     (K, V):  S = Q K^T, dP = dO V^T  ->  dS (bf16, TMEM)  ->  dQ += dS K.
// The Q pass recomputes S and dP instead of scattering dQ partial sums from
// the KV pass: 40% more tensor work, but no fp32 dQ workspace, no atomics and
// a deterministic result.
//
// Roles (persistent CTAs, one per SM; work units are handed out by an atomic
// counter so the long prefix-key units of the KV pass, which every later row
// sees, start first and the rest fill in around them):
//   warp 0      takes units from the counter, decodes each once into a
//               4-slot shared-memory ring the other roles read, and loads the
//               resident tiles (once per unit) and streamed tiles (4-stage
//               ring) by TMA
//   warp 1      TMEM allocation; one lane issues every UMMA and commit
//   warps 2..17 pointwise: two groups of eight take alternate steps; P and
//               dS (bf16) are written over the first half of each warp's own
//               fp32 score columns; then the epilogue: accumulators -> bf16
//               -> a staging buffer -> global by TMA (row by row for tiles
//               that run past the sequence end)
// TMEM columns: X1 (scores) [0,64) [64,128), X2 (dP) [128,192) [192,256),
// ACC1 [256,256+d), ACC2 [384,384+d).  Bf16 of fp32 columns [32c, 32c+32) of
// an X buffer lives in its columns [32c, 32c+16); the accumulating MMA for
// streamed rows [16k, 16k+16) reads 8 columns there.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace hstu {

bool make_tma_2d(CUtensorMap* m, const void* ptr, int64_t T, int HD, int64_t rs, int box_w,
                 int box_h, bool sw128);
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kRes = 128, kStr = 64, kMaxSt = 4, kPwWarps = 16, kUSlots = 4, kPwWarp0 = 2;
constexpr int kThreads = 32 * (kPwWarp0 + kPwWarps);
constexpr uint32_t kColX1 = 0, kColX2 = 128, kColAcc1 = 256, kColAcc2 = 384, kTmemCols = 512;

template <int D>
struct BCfg {
  // Streamed-tile ring depth (a slot is freed by a commit after the
  // accumulating MMAs of its step).
  static constexpr int kSt = D == 128 ? 3 : 4;
  static constexpr int SW = D >= 64 ? 128 : 64;
  static constexpr int BOXW = SW / 2;
  static constexpr int NB = D / BOXW;      // boxes per tile row
  static constexpr int RTILE = kRes * D * 2;
  static constexpr int STILE = kStr * D * 2;
  static constexpr int RBLK = kRes * SW;
  static constexpr int SBLK = kStr * SW;
  // Two resident buffers (tiles A1, A2 each), so the next unit's resident
  // tiles load while the current unit runs; a finished unit's buffer also
  // stages its epilogue (ACC1 over A1, ACC2 over A2) for the TMA stores.
  static constexpr int ABUF = 2 * RTILE;
  static constexpr int OFF_B1 = 2 * ABUF;
  static constexpr int OFF_B2 = OFF_B1 + kSt * STILE;
  static constexpr int OFF_BAR = OFF_B2 + kSt * STILE;
  static constexpr int OFF_UNIT = OFF_BAR + 512;
  static constexpr int OFF_SLOT = OFF_UNIT + kUSlots * (int)sizeof(UnitRec);
  static constexpr int SMEM = OFF_SLOT + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr uint32_t SWZ = SW == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t SBO = 8 * SW;
  static constexpr uint32_t IDESC_X = idesc_bf16(kRes, kStr, false, false);
  static constexpr uint32_t IDESC_ACC = idesc_bf16(kRes, D, false, true);
};

enum {
  B_A_FULL = 0, B_A_EMPTY = 2, B_B_FULL = 4, B_B_EMPTY = B_B_FULL + kMaxSt,
  B_X_FULL = B_B_EMPTY + kMaxSt,
  B_OP_FULL = B_X_FULL + 2, B_ACC_FULL = B_OP_FULL + 2, B_ACC_EMPTY, B_U_FULL,
  B_U_EMPTY = B_U_FULL + kUSlots, B_DRAIN = B_U_EMPTY + kUSlots, B_OST,  // OST: accumulator x box
  B_COUNT = B_OST + 4
};
static_assert(8 * B_COUNT <= 512, "barrier area");

// Unit u of the dynamic schedule: work-list entry u / H, head u % H; the
// streamed tiles that meet its resident tile.  u < 0 ends the schedule.
template <bool KV>
__device__ void decode_bunit(const AttnArgs& a, const int2* items, int u, UnitRec* r) {
  if (u < 0) {
    r->nsteps = -1;
    return;
  }
  const int idx = u / a.H;
  const int h = u - idx * a.H;
  const int2 it = items[idx];
  const SeqGeom g = seq_geom(a, it.x);
  const int t0 = it.y * kRes;
  const int t1 = imin(t0 + kRes, g.L);
  unit_rec_fill(r, h, g.s0, g.L, g.Lh, t0, t1,
                KV ? k_tile_q_tiles(t0, t1, g.L, g.Lh, a.K1, a.K2e, kStr)
                   : q_tile_key_tiles(t0, t1, g.Lh, a.K1, a.K2e, kStr));
}

template <int D, bool KV>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tma1, const __grid_constant__ CUtensorMap tma2,
                  const __grid_constant__ CUtensorMap tmb1, const __grid_constant__ CUtensorMap tmb2,
                  const __grid_constant__ CUtensorMap tmo1, const __grid_constant__ CUtensorMap tmo2,
                  const AttnArgs a) {
  using C = BCfg<D>;
  constexpr int kSt = C::kSt;
  constexpr int kNacc = KV ? 2 : 1;  // accumulators: dV, dK or dQ
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sA = base;  // resident buffer ab: A1 at sA + ab * ABUF, A2 RTILE further
  const uint32_t sB1 = base + C::OFF_B1, sB2 = base + C::OFF_B2;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  UnitRec* ring = reinterpret_cast<UnitRec*>(base_ptr + C::OFF_UNIT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_SLOT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (load_status(a.ws) != 0) return;
  const int2* items = KV ? a.items2 : a.items;
  const int total = (KV ? a.ws->n_items2 : a.ws->n_items) * a.H;
  int* sched = KV ? &a.ws->sched2 : &a.ws->sched;

  if (threadIdx.x == 0) {
    for (int ab = 0; ab < 2; ++ab) {
      mbar_init(bar(B_A_FULL + ab), 1);
      mbar_init(bar(B_A_EMPTY + ab), 1 + C::NB);  // last X commit + one per box stored
    }
    for (int s = 0; s < kSt; ++s) {
      mbar_init(bar(B_B_FULL + s), 1);
      mbar_init(bar(B_B_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_X_FULL + b), 1);
      mbar_init(bar(B_OP_FULL + b), kPwWarps / 2);  // one arrive per warp of group b
    }
    mbar_init(bar(B_ACC_FULL), 1);
    mbar_init(bar(B_ACC_EMPTY), kPwWarps);
    for (int s = 0; s < kUSlots; ++s) {
      mbar_init(bar(B_U_FULL + s), 1);
      mbar_init(bar(B_U_EMPTY + s), 1 + kPwWarps);  // MMA lane + pointwise warps
    }
    mbar_init(bar(B_DRAIN), 1);
    for (int w = 0; w < kNacc; ++w)
      for (int b = 0; b < C::NB; ++b)
        mbar_init(bar(B_OST + 2 * w + b), 4 * (C::BOXW / 32));  // warps staging one box
    fence_barrier_init();
    prefetch_tmap(&tma1);
    prefetch_tmap(&tma2);
    prefetch_tmap(&tmb1);
    prefetch_tmap(&tmb2);
    prefetch_tmap(&tmo1);
    prefetch_tmap(&tmo2);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------- scheduler + producer
    // The whole warp walks the schedule (warp-uniform values); lane 0 takes
    // units from the counter, decodes them, arms barriers and issues copies.
    uint32_t an = 0, bn = 0;
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(B_U_EMPTY + slot), ((kk / kUSlots) & 1) ^ 1, a.ws);
      if (!ok) break;
      if (lane == 0) {
        const int u = atomicAdd(sched, 1);
        decode_bunit<KV>(a, items, u < total ? u : -1, &ring[slot]);
        mbar_arrive(bar(B_U_FULL + slot));
      }
      __syncwarp();
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt < 0) break;
      if (nt == 0) continue;
      const int h = r->h, s0 = r->s0;
      // resident buffer an % 2: free once the unit two back is done with it
      const uint32_t ab = an & 1;
      ok = warp_wait(bar(B_A_EMPTY + ab), ((an >> 1) & 1) ^ 1, a.ws);
      if (!ok) break;
      if (lane == 0) {
        const uint32_t a1 = sA + ab * C::ABUF, fb = bar(B_A_FULL + ab);
        mbar_expect_tx(fb, 2 * C::RTILE);
        for (int b = 0; b < C::NB; ++b) {
          tma_load_2d(a1 + b * C::RBLK, &tma1, fb, h * D + b * C::BOXW, s0 + r->t0);
          tma_load_2d(a1 + C::RTILE + b * C::RBLK, &tma2, fb, h * D + b * C::BOXW, s0 + r->t0);
        }
      }
      ++an;
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt && ok; ++n, c.next(r)) {
        const int s = bn % kSt;
        ok = warp_wait(bar(B_B_EMPTY + s), ((bn / kSt) & 1) ^ 1, a.ws);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(bar(B_B_FULL + s), 2 * C::STILE);
          const int y = s0 + c.j * kStr;
          for (int b = 0; b < C::NB; ++b) {
            tma_load_2d(sB1 + s * C::STILE + b * C::SBLK, &tmb1, bar(B_B_FULL + s),
                        h * D + b * C::BOXW, y);
            tma_load_2d(sB2 + s * C::STILE + b * C::SBLK, &tmb2, bar(B_B_FULL + s),
                        h * D + b * C::BOXW, y);
          }
        }
        ++bn;
      }
    }
    if (lane == 0 && load_status(a.ws) != 0) {  // drain copies in flight before exiting
      for (uint32_t ab = 0; ab < 2; ++ab) {
        const uint32_t armed = an / 2 + (ab < (an & 1) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(B_A_FULL + ab), (armed - 1) & 1);
      }
      for (int s = 0; s < kSt; ++s) {
        const uint32_t armed = bn / kSt + (s < (int)(bn % kSt) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(B_B_FULL + s), (armed - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // One lane alone: a tcgen05.mma costs its issuing thread about as long as
    // a 128x64 MMA takes to execute, so the waits and commits here stay
    // single-threaded.  Step n: X(n) = the two score MMAs into X buffer n % 2,
    // then the accumulating MMAs of step n - 1 (whose bf16 operands the
    // pointwise warps have written by then).
    if (lane == 0) {
      uint32_t an = 0, bn = 0, xc = 0, accn = 0;
      bool ok = true;
      // Descriptor bases; offsets only add to the start-address field.
      const uint64_t dA = smem_desc(sA, 16, C::SBO, C::SWZ);
      const uint64_t dB1 = smem_desc(sB1, 16, C::SBO, C::SWZ);
      const uint64_t dB2 = smem_desc(sB2, 16, C::SBO, C::SWZ);
      const uint64_t mB1 = smem_desc(sB1, C::SBLK, C::SBO, C::SWZ);  // MN-major views
      const uint64_t mB2 = smem_desc(sB2, C::SBLK, C::SBO, C::SWZ);
      auto koff = [](int ks, int blk) -> uint32_t {  // k-step ks of a K-major tile, 16-byte units
        return (uint32_t)((((ks * 32) / C::SW) * blk + (ks * 32) % C::SW) >> 4);
      };
      // accumulating MMAs of the step with ring counter bm / X counter xm
      auto acc = [&](uint32_t bm, uint32_t xm, bool first) -> bool {
        const uint32_t b = xm & 1;
        if (!mbar_wait(bar(B_OP_FULL + b), (xm >> 1) & 1, a.ws)) return false;
        if (first && !mbar_wait(bar(B_ACC_EMPTY), (accn & 1) ^ 1, a.ws)) return false;
        tc_fence_after();
        const int s = bm % kSt;
        const uint32_t so = (uint32_t)(s * C::STILE) >> 4;
#pragma unroll
        for (int ks = 0; ks < kStr / 16; ++ks) {
          const uint32_t accum = (!first || ks > 0) ? 1u : 0u;
          const uint32_t ko = so + ((uint32_t)(ks * 16 * C::SW) >> 4);
          const uint32_t xo = b * 64 + (ks >> 1) * 32 + (ks & 1) * 8;
          if (KV) {
            mma_ts(tmem + kColAcc1, tmem + kColX1 + xo, mB2 + ko, C::IDESC_ACC, accum);  // dV += P^T dO
            mma_ts(tmem + kColAcc2, tmem + kColX2 + xo, mB1 + ko, C::IDESC_ACC, accum);  // dK += dS^T Q
          } else {
            mma_ts(tmem + kColAcc1, tmem + kColX2 + xo, mB1 + ko, C::IDESC_ACC, accum);  // dQ += dS K
          }
        }
        tc_commit(bar(B_B_EMPTY + s));
        return true;
      };
      for (int kk = 0; ok; ++kk) {
        const int slot = kk % kUSlots;
        ok = mbar_wait(bar(B_U_FULL + slot), (kk / kUSlots) & 1, a.ws);
        if (!ok) break;
        const int nt = ring[slot].nsteps;
        mbar_arrive(bar(B_U_EMPTY + slot));
        if (nt < 0) break;
        if (nt == 0) continue;
        const uint32_t ab = an & 1;
        ok = mbar_wait(bar(B_A_FULL + ab), (an >> 1) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dA1 = dA + ((ab * C::ABUF) >> 4), dA2 = dA1 + (C::RTILE >> 4);
        const uint32_t bn0 = bn, xc0 = xc;
        for (int n = 0; n < nt; ++n) {
          const int s = bn % kSt;
          ok = mbar_wait(bar(B_B_FULL + s), (bn / kSt) & 1, a.ws);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = xc & 1;
          const uint32_t so = (uint32_t)(s * C::STILE) >> 4;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            mma_ss(tmem + kColX1 + b * 64, dA1 + koff(ks, C::RBLK), dB1 + so + koff(ks, C::SBLK),
                   C::IDESC_X, ks > 0 ? 1u : 0u);
            mma_ss(tmem + kColX2 + b * 64, dA2 + koff(ks, C::RBLK), dB2 + so + koff(ks, C::SBLK),
                   C::IDESC_X, ks > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_X_FULL + b));
          if (n + 1 == nt) tc_commit(bar(B_A_EMPTY + ab));  // last use of the resident tiles
          if (n > 0) {
            ok = acc(bn - 1, xc - 1, n == 1);
            if (!ok) break;
          }
          ++bn;
          ++xc;
        }
        if (!ok) break;
        ok = acc(bn0 + nt - 1, xc0 + nt - 1, nt == 1);
        if (!ok) break;
        tc_commit(bar(B_ACC_FULL));
        ++an;
        ++accn;
      }
      tc_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ pointwise + epilogue
    // Two groups of eight warps take alternate steps (group g owns X buffer
    // g), so one group's TMEM latency overlaps the other's arithmetic; the two
    // warps of a group on one 32-lane TMEM quarter split the step's 64
    // streamed columns in halves.  The epilogue uses all sixteen warps: warp
    // `chunk` of a quarter handles accumulator columns [32 chunk, +32).
    const int pw = warp - kPwWarp0;
    const int grp = pw >> 3;              // X buffer / step parity of this warp
    const int quarter = warp & 3;
    const int chunk = pw >> 2;            // 0..3
    const int half = chunk & 1;           // streamed-column half within the group
    const int row = quarter * 32 + lane;  // resident row of this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint64_t half_alpha2 = f2s(0.5f * a.alpha);
    // dS is produced as 2 dP SiLU'(x): its consumers take alpha / (2N)
    const float sc1 = KV ? a.inv_n : 0.5f * a.alpha * a.inv_n;  // ACC1: dV or dQ
    const float sc2 = 0.5f * a.alpha * a.inv_n;                 // ACC2: dK
    bf16* out1 = KV ? a.dv : a.dq;
    const int64_t rs1 = KV ? a.dv_rs : a.dq_rs;
    const int col = half * 32;
    const bool has_acc = chunk < D / 32;
    // epilogue staging (see the forward kernel): box of this warp's chunk,
    // its first 16-byte chunk within a box row, and the box's storing warp
    const int box = (chunk * 32) / C::BOXW;
    const int box_c0 = ((chunk * 32) % C::BOXW) / 8;
    const bool box_leader = has_acc && quarter == 0 && (chunk * 32) % C::BOXW == 0;
    const uint32_t swz = C::SW == 128 ? (uint32_t)(row & 7) : (uint32_t)((row >> 1) & 3);
    uint32_t xc = 0, accn = 0, an = 0;
    // Box leaders: resident buffer whose epilogue stores were issued but not
    // yet released.  The wait for the stores to read it is deferred past this
    // warp's next step (the producer reuses the buffer only two units on).
    int pend_ab = -1;
    auto release = [&]() {
      if (pend_ab >= 0) {
        if (lane == 0) {
          bulk_wait_read_all();
          mbar_arrive(bar(B_A_EMPTY + pend_ab));
        }
        __syncwarp();
        pend_ab = -1;
      }
    };
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(B_U_FULL + slot), (kk / kUSlots) & 1, a.ws);
      if (!ok) break;
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt < 0) {
        warp_arrive(bar(B_U_EMPTY + slot));
        break;
      }
      const int h = r->h, s0 = r->s0, Lh = r->Lh, t0 = r->t0, t1 = r->t1;
      const int rr = t0 + row;  // this thread's resident position in the sequence
      bf16* o1 = out1 + (int64_t)(s0 + rr) * rs1 + h * D + chunk * 32;
      bf16* o2 = a.dk + (int64_t)(s0 + rr) * a.dk_rs + h * D + chunk * 32;
      if (nt == 0) {
        if (has_acc && rr < t1) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            reinterpret_cast<uint4*>(o1)[v] = z;
            if (KV) reinterpret_cast<uint4*>(o2)[v] = z;
          }
        }
        warp_arrive(bar(B_U_EMPTY + slot));
        continue;
      }
      const KeyMask km = key_mask(rr, r->L, Lh, a.K1, a.K2e);
      const RowMask rm = row_mask(rr, r->L, Lh, a.K1, a.K2e);
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt; ++n, ++xc, c.next(r)) {
        const uint32_t b = xc & 1;
        if ((int)b != grp) continue;  // the other group's step
        ok = warp_wait(bar(B_X_FULL + b), (xc >> 1) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const int c0 = c.j * kStr;  // first streamed position of this step
        const bool full = KV ? tile_full(c0, c0 + kStr, t0, t0 + kRes, Lh, a.K1, a.K2e)
                             : tile_full(t0, t0 + kRes, c0, c0 + kStr, Lh, a.K1, a.K2e);
        const uint32_t xs_addr = lane_base + kColX1 + b * 64 + col;
        const uint32_t xd_addr = lane_base + kColX2 + b * 64 + col;
        uint32_t xs0[16], xs1[16], xd0[16], xd1[16];
        tmem_ld16(xs_addr, xs0);
        tmem_ld16(xs_addr + 16, xs1);
        tmem_ld16(xd_addr, xd0);
        tmem_ld16(xd_addr + 16, xd1);
        tmem_ld_wait2(xs0, xs1);
        tmem_ld_wait2(xd0, xd1);
        // Fully visible tiles skip the mask; others clear invisible entries by
        // one bit test against this thread's 32-position visibility mask.
        const uint32_t bits =
            full ? 0xFFFFFFFFu : (KV ? key_mask_bits(km, c0 + col) : row_mask_bits(rm, c0 + col));
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          bwd_pair(xs0[2 * e], xs0[2 * e + 1], xd0[2 * e], xd0[2 * e + 1], half_alpha2, pp[e], dd[e]);
          bwd_pair(xs1[2 * e], xs1[2 * e + 1], xd1[2 * e], xd1[2 * e + 1], half_alpha2, pp[8 + e],
                   dd[8 + e]);
        }
        if (!full) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            pp[e] = mask_pair(pp[e], bits, e);
            dd[e] = mask_pair(dd[e], bits, e);
          }
        }
        // over the first half of the columns this warp just read
        if (KV) tmem_st16(xs_addr, pp);
        tmem_st16(xd_addr, dd);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(bar(B_OP_FULL + b));
        release();
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = warp_wait(bar(B_ACC_FULL), accn & 1, a.ws);
      if (!ok) break;
      tc_fence_after();
      const bool whole = t1 - t0 == kRes;
      // This unit's resident buffer: its last X MMA is complete (ACC_FULL
      // follows it), and it is reloaded only after the stores below read it.
      const uint32_t ab = an & 1;
#pragma unroll 1
      for (int which = 0; which < kNacc; ++which) {
        uint32_t o[16];
        if (has_acc) {
          uint32_t x0[16], x1[16];
          const uint32_t cbase = lane_base + (which ? kColAcc2 : kColAcc1) + chunk * 32;
          tmem_ld16(cbase, x0);
          tmem_ld16(cbase + 16, x1);
          tmem_ld_wait2(x0, x1);
          const float sc = which ? sc2 : sc1;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            o[e] = pack_bf16x2(__uint_as_float(x0[2 * e]) * sc, __uint_as_float(x0[2 * e + 1]) * sc);
            o[8 + e] =
                pack_bf16x2(__uint_as_float(x1[2 * e]) * sc, __uint_as_float(x1[2 * e + 1]) * sc);
          }
        }
        if (which + 1 == kNacc) {
          // every accumulator is in registers or staged: the next unit may start
          tc_fence_before();
          warp_arrive(bar(B_ACC_EMPTY));
          ++accn;
        }
        if (!has_acc) continue;
        if (whole) {
          const uint32_t rowaddr = sA + ab * C::ABUF + which * C::RTILE + box * C::RBLK + row * C::SW;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(rowaddr + ((((uint32_t)(box_c0 + q)) ^ swz) << 4), o[4 * q], o[4 * q + 1],
                         o[4 * q + 2], o[4 * q + 3]);
          fence_proxy_async_smem();  // staged rows visible to the TMA store
        } else if (rr < t1) {
          uint4* dst = reinterpret_cast<uint4*>(which ? o2 : o1);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
        warp_arrive(bar(B_OST + 2 * which + box));
      }
      if (box_leader) {
        // one thread per box stores each accumulator's box; the resident
        // buffer is freed once the stores have read it
        release();
        for (int which = 0; which < kNacc; ++which) {
          ok = mbar_wait(bar(B_OST + 2 * which + box), an & 1, a.ws) && ok;
          if (lane == 0 && ok && whole) {
            tma_store_2d(which ? &tmo2 : &tmo1, sA + ab * C::ABUF + which * C::RTILE + box * C::RBLK,
                         h * D + box * C::BOXW, s0 + t0);
            bulk_commit_group();
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (whole) {
          pend_ab = (int)ab;
        } else {
          if (lane == 0) mbar_arrive(bar(B_A_EMPTY + ab));
          __syncwarp();
        }
      }
      ++an;
      warp_arrive(bar(B_U_EMPTY + slot));
    }
    // stores still in flight must complete before the CTA exits
    if (ok) release();
    if (box_leader && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool KV>
cudaError_t launch_pass(const AttnArgs& a, cudaStream_t st) {
  using C = BCfg<D>;
  const int HD = a.H * D;
  const bool sw = C::SW == 128;
  // resident: KV -> K, V ; Q pass -> Q, dO.   streamed: KV -> Q, dO ; Q pass -> K, V.
  // stored:   KV -> dV, dK ; Q pass -> dQ.
  const void* r1 = KV ? (const void*)a.k : (const void*)a.q;
  const void* r2 = KV ? (const void*)a.v : (const void*)a.dout;
  const void* s1 = KV ? (const void*)a.q : (const void*)a.k;
  const void* s2 = KV ? (const void*)a.dout : (const void*)a.v;
  const int64_t rr1 = KV ? a.k_rs : a.q_rs, rr2 = KV ? a.v_rs : a.do_rs;
  const int64_t rs1 = KV ? a.q_rs : a.k_rs, rs2 = KV ? a.do_rs : a.v_rs;
  const void* w1 = KV ? (const void*)a.dv : (const void*)a.dq;
  const int64_t ws1 = KV ? a.dv_rs : a.dq_rs;
  CUtensorMap m1, m2, m3, m4, m5, m6;
  if (!make_tma_2d(&m1, r1, a.T, HD, rr1, C::BOXW, kRes, sw) ||
      !make_tma_2d(&m2, r2, a.T, HD, rr2, C::BOXW, kRes, sw) ||
      !make_tma_2d(&m3, s1, a.T, HD, rs1, C::BOXW, kStr, sw) ||
      !make_tma_2d(&m4, s2, a.T, HD, rs2, C::BOXW, kStr, sw) ||
      !make_tma_2d(&m5, w1, a.T, HD, ws1, C::BOXW, kRes, sw) ||
      !make_tma_2d(&m6, KV ? (const void*)a.dk : w1, a.T, HD, KV ? a.dk_rs : ws1, C::BOXW, kRes,
                   sw))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel<D, KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t units = max_items(a.T, a.B) * a.H;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  bwd_tc_kernel<D, KV><<<grid, kThreads, C::SMEM, st>>>(m1, m2, m3, m4, m5, m6, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_tc(const AttnArgs& a, int d, bool kv_pass, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (d == 32) return kv_pass ? launch_pass<32, true>(a, st) : launch_pass<32, false>(a, st);
  if (d == 64) return kv_pass ? launch_pass<64, true>(a, st) : launch_pass<64, false>(a, st);
  return kv_pass ? launch_pass<128, true>(a, st) : launch_pass<128, false>(a, st);
}

}  // namespace hstu
