// SLA HSTU attention backward for head_dim 128 in ONE pass over key tiles, on
// the 5th-generation tensor cores (tcgen05 / TMEM / TMA).
//
// With x_ij = alpha q_i.k_j, P_ij = M SiLU(x)/N and dP_ij = dO_i.v_j:
//   dV_j = sum_i P_ij dO_i,   dK_j = sum_i dS_ij q_i,   dQ_i = sum_j dS_ij k_j,
//   dS_ij = M dP_ij SiLU'(x_ij) alpha/N
// (the chain rule through "Bending the Scaling Law Curve in Large-Scale
// Recommendation Systems", section 3, Eq. 3, under the SLA mask of section
// 4.2.1, Eq. 7).
//
// A resident 128-key tile (K, V) meets streamed 64-row query tiles (Q, dO):
//   S^T = K Q^T, dP^T = V dO^T            (tensor cores, fp32 in TMEM)
//   P^T, dS^T                              (pointwise warps, bf16)
//   dV += P^T dO, dK += dS^T Q            (TMEM accumulators: each key tile has
//                                          one owner, so no atomics on dK, dV)
//   dQ^T(step) = K^T dS^T                 (128 x 64 fp32 in TMEM)
//   dQ workspace += dQ(step)               (fp32 reductions in L2, by the
//                                          pointwise warps that drained it)
// and a second kernel turns the fp32 dQ workspace into bf16 dq, applying
// alpha / (2N).  Against a separate query-major pass that recomputes S and dP
// this saves two of the seven tile contractions per (key tile, query tile)
// pair; the price is the fp32 workspace and the order of the dQ additions,
// which is not fixed (dq is reproducible to fp32 rounding, not bitwise).
//
// Roles (persistent CTAs, one per SM; units handed out by an atomic counter,
// prefix-key units first):
//   warp 0      scheduler + TMA producer of the 4-stage Q / dO ring
//   warp 18     TMA loads of K and V (one buffer each)
//   warp 1      TMEM allocation; the warp computes every MMA operand, one
//               elected lane issues each batch of UMMAs and its commits
//   warps 2..17 pointwise, all sixteen on every step (16 query columns
//               each); then the dQ drain of the step before; at the end of
//               a unit, they store dK and dV
// TMEM columns:
//   X1(b) = [64b, 64b+64)       S^T (fp32); after the pointwise: per 16-column
//                               group g, P^T bf16 in [16g, 16g+8) and dS^T
//                               bf16 in [16g+8, 16g+16)
//   X2(b) = [128+64b, 192+64b)  dP^T (fp32); then the step's dQ^T (lanes =
//                               head-dim index, columns = query rows)
//   ACC1 = [256, 384) dV,  ACC2 = [384, 512) dK
// Shared memory (227 KB): K 32 KB, V 32 KB, Q and dO 4 x 16 KB each, dS^T
// 2 x 16 KB (the B operand of the dQ MMA), barriers and the unit ring.
#include <cudaTypedefs.h>
#include <type_traits>

#include "sm100.cuh"

namespace hstu {

bool make_tma_2d(CUtensorMap* m, const void* ptr, int64_t T, int HD, int64_t rs, int box_w,
                 int box_h, bool sw128);
int device_sm_count();

namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kRes = 128, kStr = 64, kSt = 4, kPwWarps = 16, kUSlots = 4, kPwWarp0 = 2;
constexpr int kKvWarp = kPwWarp0 + kPwWarps;  // the K / V loader
constexpr int kThreads = 32 * (kKvWarp + 1);
constexpr uint32_t kColX1 = 0, kColX2 = 128, kColAcc1 = 256, kColAcc2 = 384, kTmemCols = 512;
constexpr int SW = 128, BOXW = 64, NB = D / BOXW;
constexpr int RTILE = kRes * D * 2;     // resident tile, two 64-column boxes
constexpr int STILE = kStr * D * 2;     // streamed tile, two boxes
constexpr int RBLK = kRes * SW;         // one box of a resident tile
constexpr int SBLK = kStr * SW;         // one box of a streamed tile
constexpr int DSTILE = kRes * kStr * 2;  // dS^T: [128 keys][64 rows] bf16, one box
constexpr int OFF_K = 0;
// One K buffer: the next unit's K loads once the current unit's last dQ MMA
// is done.  Measured against two buffers with three Q / dO stages, the
// kernel ran ~1% faster; the 32 KB then went to a fourth Q / dO stage.
constexpr int kKBufs = 1;
constexpr int OFF_V = OFF_K + kKBufs * RTILE;
constexpr int OFF_B1 = OFF_V + RTILE;
constexpr int OFF_B2 = OFF_B1 + kSt * STILE;
constexpr int OFF_DS = OFF_B2 + kSt * STILE;
constexpr int OFF_BAR = OFF_DS + 2 * DSTILE;
constexpr int OFF_UNIT = OFF_BAR + 512;
constexpr int OFF_SLOT = OFF_UNIT + kUSlots * (int)sizeof(UnitRec);
// relative attention bias: per-unit histograms of the bias gradient, two
// (alternating units), each in two copies (warps of even and odd index add
// into separate copies, halving same-address atomics), 32 position then 32
// time buckets each
constexpr int kHistBins = 64;
constexpr int OFF_HIST = OFF_SLOT + 16;
constexpr int kHistCopies = 2;
constexpr int SMEM = OFF_HIST + 2 * kHistCopies * kHistBins * 4 + 1024;
static_assert(SMEM <= 232448, "shared memory budget");
constexpr uint32_t SBO = 8 * SW;
// 128 x 64 scores, both operands K-major
constexpr uint32_t IDESC_X = idesc_bf16(kRes, kStr, false, false);
// 128 x 128 accumulators: A = P^T / dS^T from TMEM, B = dO / Q MN-major
constexpr uint32_t IDESC_ACC = idesc_bf16(kRes, D, false, true);
// 128 x 64 dQ^T: A = K^T and B = dS^T, both read MN-major from their tiles
constexpr uint32_t IDESC_DQ = idesc_bf16(D, kStr, true, true);

enum {
  F_K_FULL = 0, F_K_EMPTY = 2, F_V_FULL = 4, F_V_EMPTY, F_B_FULL,
  F_B_EMPTY = F_B_FULL + kSt, F_X_FULL = F_B_EMPTY + kSt, F_OP_FULL = F_X_FULL + 2,
  F_DQ_FULL = F_OP_FULL + 2, F_DQ_EMPTY = F_DQ_FULL + 2, F_ACC_FULL = F_DQ_EMPTY + 2,
  F_ACC_EMPTY, F_U_FULL, F_U_EMPTY = F_U_FULL + kUSlots, F_DRAIN = F_U_EMPTY + kUSlots,
  F_H_DONE, F_H_ZERO = F_H_DONE + 2, F_COUNT = F_H_ZERO + 2
};
static_assert(8 * F_COUNT <= 512, "barrier area");

// Unit u of the schedule: the prefix key tiles of every problem first (the
// longest units: every later row sees a prefix key), then the other key
// tiles, problem after problem; within a problem's part, item u / H, head
// u % H.  Past the last unit the record ends the schedule.
__device__ void decode_kv_unit(const GroupSet& gs, int u, UnitRec* r) {
  for (int part = 0; part < 2 && u >= 0; ++part) {
    for (int p = 0; p < kMaxGroups && p < gs.G; ++p) {
      const AttnArgs& a = gs.g[p];
      const int n_pre = a.ws->n_items2_pre;
      const int units = (part == 0 ? n_pre : a.ws->n_items2 - n_pre) * a.H;
      if (u < units) {
        const int idx = u / a.H;
        const int h = u - idx * a.H;
        const int2 it = a.items2[(part == 0 ? 0 : n_pre) + idx];
        const SeqGeom g = seq_geom(a, it.x);
        const int t0 = it.y * kRes;
        const int t1 = imin(t0 + kRes, g.L);
        unit_rec_fill(r, h, g.s0, g.L, g.Lh, t0, t1,
                      k_tile_q_tiles(t0, t1, g.L, g.Lh, a.K1, a.K2e, kStr));
        r->grp = p;
        return;
      }
      u -= units;
    }
  }
  r->nsteps = -1;
}

// k-step ks of a K-major 128B-swizzled tile whose 64-column boxes are `blk`
// bytes apart, in the 16-byte units of a descriptor's start address.
__host__ __device__ constexpr uint32_t koff_k(int ks, int blk) {
  return (uint32_t)((((ks * 32) / SW) * blk + (ks * 32) % SW) >> 4);
}

// k, v, q, dout maps of every problem of a launch.
struct BwdMaps {
  CUtensorMap k[kMaxGroups], v[kMaxGroups], q[kMaxGroups], dout[kMaxGroups];
};

// Adds two (bin, value) pairs per lane (one per table; bin < 0: nothing)
// into the shared histogram: a segmented sum over runs of consecutive lanes
// with equal bins (five shuffle steps for every run at once), then one
// shared atomic from each run's last lane.  Equal bins in separate runs
// stay correct (one atomic per run).  Called by the whole warp.
__device__ __forceinline__ void warp_flush_runs(float* hst, int bp, float vp, int bt, float vt,
                                                int lane) {
  const uint32_t full = 0xffffffffu;
  const int bp_prev = __shfl_up_sync(full, bp, 1), bt_prev = __shfl_up_sync(full, bt, 1);
  const int bp_next = __shfl_down_sync(full, bp, 1), bt_next = __shfl_down_sync(full, bt, 1);
  const uint32_t below = (2u << lane) - 1u;  // lanes 0..lane
  const uint32_t hp = __ballot_sync(full, lane == 0 || bp != bp_prev) & below;
  const uint32_t ht = __ballot_sync(full, lane == 0 || bt != bt_prev) & below;
  const int sp = 31 - __clz(hp), st = 31 - __clz(ht);  // first lane of my run
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float up = __shfl_up_sync(full, vp, o), ut = __shfl_up_sync(full, vt, o);
    if (lane - o >= sp) vp += up;
    if (lane - o >= st) vt += ut;
  }
  if (bp >= 0 && (lane == 31 || bp_next != bp)) atomicAdd(hst + bp, vp);
  if (bt >= 0 && (lane == 31 || bt_next != bt)) atomicAdd(hst + bt, vt);
}

// Fire-and-forget fp32 addition in L2 (the result is unused, so this is a
// reduction, not a round trip).
__device__ __forceinline__ void red_add_f32(float* p, uint32_t v) { atomicAdd(p, __uint_as_float(v)); }

// RAB: the relative attention bias is added to every recomputed score and
// its gradient is accumulated per unit in a shared-memory histogram.  Each
// thread keeps runs of equal buckets along its key's query columns: in a
// 16-column round where every lane's buckets span at most two neighbouring
// values (the position bucket only grows along the columns; the time bucket
// is bounded by the round's earliest and latest query) a score adds its
// gradient to two or three register totals; finished runs wait in one slot
// per table and are added into the histogram once per step, runs of lanes
// with equal buckets summed by a segmented shuffle scan first
// (same-address shared atomics from many lanes were the cost).  One
// pointwise warp flushes the unit's sums into this head's table gradients.
// STALL (the wait-timeout test hook only): each pointwise warp withholds its
// OP_FULL arrive of the first step it processes, so the MMA warp's wait for
// those operands runs into the launch's wait limit.
template <bool RAB, bool STALL = false>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kvq_kernel(const __grid_constant__ BwdMaps maps, const __grid_constant__ GroupSet gs) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sK = base + OFF_K, sV = base + OFF_V, sB1 = base + OFF_B1, sB2 = base + OFF_B2;
  const uint32_t sDS = base + OFF_DS;
  const uint32_t bar0 = base + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  UnitRec* ring = reinterpret_cast<UnitRec*>(base_ptr + OFF_UNIT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + OFF_SLOT);
  float* hist = reinterpret_cast<float*>(base_ptr + OFF_HIST);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* const ws = gs.common;  // status word and scheduler of the launch
  // a problem's device-side input check failed: report it for the launch
  for (int p = 0; p < kMaxGroups && p < gs.G; ++p) {
    const int st = load_status(gs.g[p].ws);
    if (st != 0) {
      if (threadIdx.x == 0) set_status(ws, st);
      return;
    }
  }
  if (load_status(ws) != 0) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(F_K_FULL + i), 1);
      mbar_init(bar(F_K_EMPTY + i), 1);                // commit after the unit's last dQ MMA
      mbar_init(bar(F_X_FULL + i), 1);
      mbar_init(bar(F_OP_FULL + i), kPwWarps);         // one arrive per pointwise warp
      mbar_init(bar(F_DQ_FULL + i), 1);
      mbar_init(bar(F_DQ_EMPTY + i), kPwWarps);
    }
    mbar_init(bar(F_V_FULL), 1);
    mbar_init(bar(F_V_EMPTY), 1);                      // commit after the unit's last X MMA
    for (int s = 0; s < kSt; ++s) {
      mbar_init(bar(F_B_FULL + s), 1);
      mbar_init(bar(F_B_EMPTY + s), 1);
    }
    mbar_init(bar(F_ACC_FULL), 1);
    mbar_init(bar(F_ACC_EMPTY), kPwWarps);
    for (int s = 0; s < kUSlots; ++s) {
      mbar_init(bar(F_U_FULL + s), 1);
      mbar_init(bar(F_U_EMPTY + s), 2 + kPwWarps);  // MMA, K / V loader, pointwise warps
    }
    mbar_init(bar(F_DRAIN), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(F_H_DONE + i), kPwWarps);  // every pointwise warp's sums are in
      mbar_init(bar(F_H_ZERO + i), 1);         // flushed and cleared
    }
    fence_barrier_init();
    for (int p = 0; p < kMaxGroups && p < gs.G; ++p) {
      if (gs.g[p].T == 0) continue;  // no map was built
      prefetch_tmap(&maps.k[p]);
      prefetch_tmap(&maps.v[p]);
      prefetch_tmap(&maps.q[p]);
      prefetch_tmap(&maps.dout[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (RAB)
    for (int i = threadIdx.x; i < 2 * kHistCopies * kHistBins; i += blockDim.x) hist[i] = 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------- scheduler + producer
    // The whole warp walks the schedule (warp-uniform values); lane 0 takes
    // units from the counter, decodes them, arms barriers and issues copies.
    // The K / V tiles come from their own warp (kKvWarp), so this stream of
    // Q / dO tiles runs into the next unit while its V still waits for the
    // current unit's last score MMA.
    uint32_t bn = 0;  // streamed loads issued
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(F_U_EMPTY + slot), ((kk / kUSlots) & 1) ^ 1, ws);
      if (!ok) break;
      if (lane == 0) {
        decode_kv_unit(gs, atomicAdd(&ws->sched2, 1), &ring[slot]);
        mbar_arrive(bar(F_U_FULL + slot));
      }
      __syncwarp();
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt < 0) break;
      if (nt == 0) continue;
      const int h = r->h;
      const int p = r->grp;
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt && ok; ++n, c.next(r)) {
        const int s = bn % kSt;
        ok = warp_wait(bar(F_B_EMPTY + s), ((bn / kSt) & 1) ^ 1, ws);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(F_B_FULL + s);
          mbar_expect_tx(fb, 2 * STILE);
          const int y = r->s0 + c.j * kStr;
          for (int b = 0; b < NB; ++b) {
            tma_load_2d(sB1 + s * STILE + b * SBLK, &maps.q[p], fb, h * D + b * BOXW, y);
            tma_load_2d(sB2 + s * STILE + b * SBLK, &maps.dout[p], fb, h * D + b * BOXW, y);
          }
        }
        ++bn;
      }
    }
    if (lane == 0 && load_status(ws) != 0) {  // drain copies in flight before exiting
      for (int s = 0; s < kSt; ++s) {
        const uint32_t armed = bn / kSt + (s < (int)(bn % kSt) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(F_B_FULL + s), (armed - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp walks the schedule and computes every operand (TMEM
    // addresses, descriptor bases, barrier addresses) together, so they are
    // warp-uniform; one elected lane then issues each batch of UMMAs with
    // only immediate offsets added, and the commits that close it.  A lone
    // lane (a divergent branch) pays ~60 clk per tcgen05.mma against ~10 here.
    // Step n: the S^T MMAs into X1, then (once the dQ^T two steps back has
    // been read out of X2) the dP^T MMAs into X2; then the MMAs of step n - 1
    // that consume its bf16 P^T / dS^T: dQ^T first (its drain overlaps the
    // rest), then dV and dK.
    {
      uint32_t an = 0, bn = 0, xc = 0, accn = 0;
      bool ok = true;
      // Descriptor bases; offsets only add to the start-address field.
      const uint64_t dK0 = smem_desc(sK, 16, SBO, kSwizzle128B);      // K, K-major
      const uint64_t dKt0 = smem_desc(sK, RBLK, SBO, kSwizzle128B);   // K^T, MN-major
      const uint64_t dV = smem_desc(sV, 16, SBO, kSwizzle128B);
      const uint64_t dB1 = smem_desc(sB1, 16, SBO, kSwizzle128B);
      const uint64_t dB2 = smem_desc(sB2, 16, SBO, kSwizzle128B);
      const uint64_t mB1 = smem_desc(sB1, SBLK, SBO, kSwizzle128B);  // MN-major views
      const uint64_t mB2 = smem_desc(sB2, SBLK, SBO, kSwizzle128B);
      // dS^T is one 128-byte-wide box: the leading byte offset is never used
      const uint64_t dDS = smem_desc(sDS, DSTILE, SBO, kSwizzle128B);
      constexpr uint32_t kRows16 = (16 * SW) >> 4;  // 16 rows of an MN-major tile, 16-byte units
      // MMAs of the step with ring counter bm / X counter xm, K buffer kb
      auto acc = [&](uint32_t bm, uint32_t xm, uint32_t kb, bool first, bool last) -> bool {
        const uint32_t b = xm & 1;
        if (!warp_wait(bar(F_OP_FULL + b), (xm >> 1) & 1, ws)) return false;
        if (first && !warp_wait(bar(F_ACC_EMPTY), (accn & 1) ^ 1, ws)) return false;
        tc_fence_after();
        const int s = bm % kSt;
        const uint32_t so = (uint32_t)(s * STILE) >> 4;
        const uint64_t aq = dKt0 + ((kb * RTILE) >> 4), bq = dDS + ((b * DSTILE) >> 4);
        const uint64_t b1 = mB1 + so, b2 = mB2 + so;
        const uint32_t dq_t = tmem + kColX2 + b * 64, x1 = tmem + kColX1 + b * 64;
        const uint32_t bar_dq = bar(F_DQ_FULL + b), bar_k = bar(F_K_EMPTY + kb);
        const uint32_t bar_b = bar(F_B_EMPTY + s);
        const uint32_t acc0 = first ? 0u : 1u;
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kRes / 16; ++ks)  // dQ^T = K^T dS^T over the read-out dP^T
            mma_ss(dq_t, aq + ks * kRows16, bq + ks * kRows16, IDESC_DQ, ks > 0 ? 1u : 0u);
          tc_commit(bar_dq);
          if (last) tc_commit(bar_k);  // last use of this K buffer
#pragma unroll
          for (int ks = 0; ks < kStr / 16; ++ks) {
            // queries [16 ks, +16): P^T at columns 32 (ks / 2) + 16 (ks % 2), dS^T 8 further
            const uint32_t xo = (ks >> 1) * 32 + (ks & 1) * 16;
            mma_ts(tmem + kColAcc1, x1 + xo, b2 + ks * kRows16, IDESC_ACC,
                   ks > 0 ? 1u : acc0);  // dV += P^T dO
            mma_ts(tmem + kColAcc2, x1 + xo + 8, b1 + ks * kRows16, IDESC_ACC,
                   ks > 0 ? 1u : acc0);  // dK += dS^T Q
          }
          tc_commit(bar_b);
        }
        __syncwarp();
        return true;
      };
      for (int kk = 0; ok; ++kk) {
        const int slot = kk % kUSlots;
        ok = warp_wait(bar(F_U_FULL + slot), (kk / kUSlots) & 1, ws);
        if (!ok) break;
        const int nt = __shfl_sync(0xffffffffu, ring[slot].nsteps, 0);
        warp_arrive(bar(F_U_EMPTY + slot));
        if (nt < 0) break;
        if (nt == 0) continue;
        const uint32_t kb = an % kKBufs;
        ok = warp_wait(bar(F_K_FULL + kb), (an / kKBufs) & 1, ws) &&
             warp_wait(bar(F_V_FULL), an & 1, ws);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dK = dK0 + ((kb * RTILE) >> 4);
        const uint32_t bn0 = bn, xc0 = xc;
        for (int n = 0; n < nt; ++n) {
          const int s = bn % kSt;
          ok = warp_wait(bar(F_B_FULL + s), (bn / kSt) & 1, ws);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = xc & 1;
          const uint32_t so = (uint32_t)(s * STILE) >> 4;
          const uint64_t bq = dB1 + so, bo = dB2 + so;
          const uint32_t x1 = tmem + kColX1 + b * 64, x2 = tmem + kColX2 + b * 64;
          if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)  // S^T = K Q^T
              mma_ss(x1, dK + koff_k(ks, RBLK), bq + koff_k(ks, SBLK), IDESC_X, ks > 0 ? 1u : 0u);
          }
          __syncwarp();
          // X2(b) still holds the dQ^T of step xc - 2 until its drain is done
          ok = warp_wait(bar(F_DQ_EMPTY + b), ((xc >> 1) & 1) ^ 1, ws);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bar_x = bar(F_X_FULL + b), bar_v = bar(F_V_EMPTY);
          const bool last_v = n + 1 == nt;
          if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)  // dP^T = V dO^T
              mma_ss(x2, dV + koff_k(ks, RBLK), bo + koff_k(ks, SBLK), IDESC_X, ks > 0 ? 1u : 0u);
            tc_commit(bar_x);
            if (last_v) tc_commit(bar_v);  // last use of V
          }
          __syncwarp();
          if (n > 0) {
            ok = acc(bn - 1, xc - 1, kb, n == 1, false);
            if (!ok) break;
          }
          ++bn;
          ++xc;
        }
        if (!ok) break;
        ok = acc(bn0 + nt - 1, xc0 + nt - 1, kb, nt == 1, true);
        if (!ok) break;
        if (elect_one()) tc_commit(bar(F_ACC_FULL));
        __syncwarp();
        ++an;
        ++accn;
      }
      if (elect_one()) tc_commit(bar(F_DRAIN));
      __syncwarp();
      drain_wait(bar(F_DRAIN), 0);
    }
    __syncwarp();
  } else if (warp == kKvWarp) {
    // -------------------------------------------------------- K / V loader
    // Per unit with steps: K once the previous unit's last dQ MMA is done,
    // then V once the previous unit's last score MMA is done.
    uint32_t kn = 0, vn = 0;  // K, V loads issued
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(F_U_FULL + slot), (kk / kUSlots) & 1, ws);
      if (!ok) break;
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt > 0) {
        const int h = r->h, y0 = r->s0 + r->t0, p = r->grp;
        const uint32_t kb = kn % kKBufs;
        ok = warp_wait(bar(F_K_EMPTY + kb), ((kn / kKBufs) & 1) ^ 1, ws);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(F_K_FULL + kb);
          mbar_expect_tx(fb, RTILE);
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sK + kb * RTILE + b * RBLK, &maps.k[p], fb, h * D + b * BOXW, y0);
        }
        ++kn;
        ok = warp_wait(bar(F_V_EMPTY), (vn & 1) ^ 1, ws);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(F_V_FULL);
          mbar_expect_tx(fb, RTILE);
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sV + b * RBLK, &maps.v[p], fb, h * D + b * BOXW, y0);
        }
        ++vn;
      }
      warp_arrive(bar(F_U_EMPTY + slot));
      if (nt < 0) break;
    }
    if (lane == 0 && load_status(ws) != 0) {  // drain copies in flight before exiting
      for (uint32_t kb = 0; kb < (uint32_t)kKBufs; ++kb) {
        const uint32_t armed = kn / kKBufs + (kb < (kn % kKBufs) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(F_K_FULL + kb), (armed - 1) & 1);
      }
      if (vn > 0) drain_wait(bar(F_V_FULL), (vn - 1) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ pointwise + drains
    // All sixteen warps work on every step: the four warps on one 32-lane
    // TMEM quarter split the step's 64 query columns in chunks of 16 (the
    // step's pointwise latency, which the MMA of the step after next waits
    // for, is that of one 16-column round).  Per step a warp turns its 16
    // scores per key into P^T and dS^T (bf16, TMEM) and copies dS^T into
    // shared memory for the dQ MMA; then it drains the PREVIOUS step's dQ^T
    // (done by now: the MMA lane issued it right after this step's dP^T),
    // reading its 16 columns (query rows) for the 32 head-dim lanes of its
    // quarter and adding them to the fp32 workspace, so no warp ever waits
    // for a dQ^T.  A unit's last dQ^T is drained before its epilogue.  Unit
    // epilogue: warp `chunk` of a quarter stores accumulator columns
    // [32 chunk, +32) of dV and dK.
    const int pw = warp - kPwWarp0;
    const int quarter = warp & 3;
    const int chunk = pw >> 2;            // 0..3
    const int row = quarter * 32 + lane;  // key row (and head-dim lane of dQ^T)
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int col = chunk * 16;           // this warp's query columns of a step
    const uint32_t ds_row = sDS + (uint32_t)row * SW;
    const uint32_t swz = (uint32_t)(row & 7);
    uint32_t xc = 0, accn = 0;
    bool withhold = STALL;  // the test hook's one withheld arrive
    uint32_t hu = 0;  // units with steps so far (histogram buffer hu & 1)
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(F_U_FULL + slot), (kk / kUSlots) & 1, ws);
      if (!ok) break;
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt < 0) {
        warp_arrive(bar(F_U_EMPTY + slot));
        break;
      }
      const int h = r->h, s0 = r->s0, L = r->L, Lh = r->Lh, t0 = r->t0, t1 = r->t1;
      const AttnArgs& A = gs.g[r->grp];
      const int K1 = A.K1, K2e = A.K2e;
      const uint64_t half_alpha2 = f2s(0.5f * A.alpha);
      // dS is produced as 2 dP SiLU'(x): its consumers take alpha / (2N)
      const float sc_dv = A.inv_n, sc_dk = 0.5f * A.alpha * A.inv_n;
      const int rr = t0 + row;  // this thread's key position in the sequence
      bf16* o1 = A.dv + (int64_t)(s0 + rr) * A.dv_rs + h * D + chunk * 32;
      bf16* o2 = A.dk + (int64_t)(s0 + rr) * A.dk_rs + h * D + chunk * 32;
      if (nt == 0) {  // keys no row sees
        if (rr < t1) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            reinterpret_cast<uint4*>(o1)[v] = z;
            reinterpret_cast<uint4*>(o2)[v] = z;
          }
        }
        warp_arrive(bar(F_U_EMPTY + slot));
        continue;
      }
      const KeyMask km = key_mask(rr, L, Lh, K1, K2e);
      // dQ workspace ([H][T][D]) column of this lane (head-dim index `row`)
      // at the sequence start
      float* dqa = A.dqacc + ((int64_t)h * A.T + s0) * D + row;
      // relative attention bias: this head's tables, this key's timestamp and
      // the unit's histogram buffer (free once the unit two back was flushed)
      float tabp = 0.f, tabt = 0.f;  // half of bucket min(lane, nb - 1)
      int32_t tj = 0;
      float* const hst0 = hist + (hu & 1) * kHistCopies * kHistBins;  // the unit's copies
      float* hst = hst0 + (pw % kHistCopies) * kHistBins;
      if constexpr (RAB) {
        tabp = rab_lane_table(A.rab_pos, A.nbp, h, lane);
        tabt = rab_lane_table(A.rab_time, A.nbt, h, lane);
        tj = (A.ts && rr < L) ? __ldg(A.ts + s0 + rr) : 0;
        ok = warp_wait(bar(F_H_ZERO + (hu & 1)), ((hu >> 1) & 1) ^ 1, ws);
        if (!ok) break;
      }
      // runs of equal buckets (position, time) along this key's query
      // columns, which only grow through the unit's steps.  Bins hold the
      // buckets before the tables' clamp (0..31 each); the flush folds bins
      // past a table's last bucket into it.
      int run_p = -1, run_t = -1;
      float sum_p = 0.f, sum_t = 0.f;
      // a finished run waits in one pending slot per table until the end of
      // the step, when the warp sums runs of lanes with equal bins; a second
      // one in the same step goes straight into the histogram
      int pend_p = -1, pend_t = -1;
      float psum_p = 0.f, psum_t = 0.f;
      auto run_add = [&](int& run, float& sum, int& pend, float& psum, int bin, float g) {
        const bool c = bin != run;
        if (c && pend >= 0) {  // a second finished run in this step
          atomicAdd(hst + run, sum);
          sum = 0.f;
          run = -1;
        }
        const bool mv = c && run >= 0;
        pend = mv ? run : pend;
        psum = mv ? sum : psum;
        sum = c ? g : sum + g;
        run = bin;
      };
      // Reads step xd's dQ^T (first query row q0) out of X2 and adds this
      // warp's 16 rows of it to the workspace; rows past the sequence end are
      // skipped.
      auto drain = [&](uint32_t xd, int q0) -> bool {
        const uint32_t bb = xd & 1;
        if (!warp_wait(bar(F_DQ_FULL + bb), (xd >> 1) & 1, ws)) return false;
        tc_fence_after();
        uint32_t g[16];
        tmem_ld16(lane_base + kColX2 + bb * 64 + col, g);
        tmem_ld_wait(g);
        tc_fence_before();
        warp_arrive(bar(F_DQ_EMPTY + bb));
        const int qq = q0 + col;
        const int nv = L - qq;
        float* p = dqa + (int64_t)qq * D;
        if (nv >= 16) {
#pragma unroll
          for (int e = 0; e < 16; ++e) red_add_f32(p + e * D, g[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (e < nv) red_add_f32(p + e * D, g[e]);
        }
        return true;
      };
      int prev_c0 = 0;  // first query row of the previous step of this unit
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt; ++n, ++xc, c.next(r)) {
        const uint32_t b = xc & 1;
        const int c0 = c.j * kStr;  // first query row of this step
        // relative attention bias: the 16 queries' timestamps (lanes 0..15),
        // loaded before the wait for the scores
        int32_t tql = 0;
        bool tq_ok = false;  // this lane's query column is in the sequence
        if constexpr (RAB) {
          const int ql = c0 + col + lane;
          tq_ok = lane < 16 && ql < L;
          tql = (A.ts && tq_ok) ? __ldg(A.ts + s0 + ql) : 0;
        }
        ok = warp_wait(bar(F_X_FULL + b), (xc >> 1) & 1, ws);
        if (!ok) break;
        tc_fence_after();
        const bool full = tile_full(c0, c0 + kStr, t0, t0 + kRes, Lh, K1, K2e);
        const uint32_t xs_addr = lane_base + kColX1 + b * 64 + col;
        const uint32_t xd_addr = lane_base + kColX2 + b * 64 + col;
        const uint32_t dsr = ds_row + b * DSTILE;
        // Fully visible tiles skip the mask; others clear invisible entries by
        // one bit test against this key's visibility mask of the chunk's rows.
        const uint32_t bits = full ? 0xFFFFFFFFu : key_mask_bits(km, c0 + col);
        // One round of the chunk's 16 query columns: P^T (8 packed columns)
        // then dS^T (8) over the 16 score columns it read, and dS^T copied to
        // 16-byte chunks 2 chunk, +1 of this key's 128-byte swizzled row of
        // the dS^T tile.
#pragma unroll
        for (int r = 0; r < 1; ++r) {
          uint32_t xs[16], xd[16], pp[8], dd[8];
          tmem_ld16(xs_addr + 16 * r, xs);
          tmem_ld16(xd_addr + 16 * r, xd);
          tmem_ld_wait2(xs, xd);
          if constexpr (RAB) {
            // Bounds of the round's buckets for this key: the position bucket
            // only grows along the columns (first and last column), the time
            // difference lies between those to the round's earliest and latest
            // query.  When every lane's buckets take at most two neighbouring
            // values, each score only adds its gradient to the round's total
            // and to the upper buckets' totals; else each score extends its
            // runs one by one.
            const int b0p = rab_log_bucket(rab_pos_u(__viaddmin_s32(c0 + col, 16 * r, Lh), 1 - rr));
            const int b1p =
                rab_log_bucket(rab_pos_u(__viaddmin_s32(c0 + col, 16 * r + 15, Lh), 1 - rr));
            const bool in_round = tq_ok && (lane >> 4) == r;
            const int32_t tmin = __reduce_min_sync(0xffffffffu, in_round ? tql : INT32_MAX);
            const int32_t tmax = __reduce_max_sync(0xffffffffu, in_round ? tql : INT32_MIN);
            uint32_t dlo, dhi;
            if (tj <= tmin) {
              dlo = (uint32_t)tmin - (uint32_t)tj;
              dhi = (uint32_t)tmax - (uint32_t)tj;
            } else if (tj >= tmax) {
              dlo = (uint32_t)tj - (uint32_t)tmax;
              dhi = (uint32_t)tj - (uint32_t)tmin;
            } else {
              dlo = 0u;
              dhi = max((uint32_t)tmax - (uint32_t)tj, (uint32_t)tj - (uint32_t)tmin);
            }
            const int b0t = rab_log_bucket(dlo + 1u) & 31;
            const int b1t = rab_log_bucket(dhi + 1u) & 31;
            const bool two = (uint32_t)(b1p - b0p) <= 1u && (uint32_t)(b1t - b0t) <= 1u;
            const bool flat = b1p == b0p && b1t == b0t;
            // every lane's buckets constant over the round: one bias for all
            // its scores, and the round's total goes to one bin per table
            // (the same values and order of additions as the two-bucket form)
            auto rab_flat = [&](auto all_c) {
              constexpr bool kAll = decltype(all_c)::value;
              const float hb = rab_half_bias(tabp, tabt, b0p, b0t);
              float acc = 0.f;
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int k = 16 * r + 2 * e;
                float ga, gb;
                bwd_pair_bias(xs[2 * e], xs[2 * e + 1], xd[2 * e], xd[2 * e + 1], half_alpha2, hb,
                              hb, pp[e], dd[e], ga, gb);
                if (!kAll && !((bits >> k) & 1u)) ga = 0.f;
                if (!kAll && !((bits >> (k + 1)) & 1u)) gb = 0.f;
                acc += ga;
                acc += gb;
              }
              if (acc != 0.f) {
                run_add(run_p, sum_p, pend_p, psum_p, b0p, acc);
                run_add(run_t, sum_t, pend_t, psum_t, 32 + b0t, acc);
              }
            };
            // every lane's buckets take at most two neighbouring values: the
            // upper position bucket starts at a column kp of the round (the
            // position difference only grows along it), a score is in the
            // upper time bucket from the difference thr_t on; the four table
            // values are read once, and each score picks its bias and its
            // upper-bucket sums by two predicates (the same values as the
            // per-score form below)
            auto rab_two = [&](auto all_c) {
              constexpr bool kAll = decltype(all_c)::value;
              const int kp =
                  b1p != b0p
                      ? (int)max((int64_t)0, ((int64_t)1 << (b0p + 1)) - 1 + rr - (c0 + col + 16 * r))
                      : 16;
              const bool two_t = b1t != b0t;
              const uint32_t thr_t = (2u << b0t) - 1u;  // 2^(b0t + 1) - 1 (b0t <= 30 when used)
              const float hp0 = __shfl_sync(0xffffffffu, tabp, b0p);
              const float hp1 = __shfl_sync(0xffffffffu, tabp, b0p + 1);
              const float ht0 = __shfl_sync(0xffffffffu, tabt, b0t);
              const float ht1 = __shfl_sync(0xffffffffu, tabt, b0t + 1);
              float acc = 0.f, ahp = 0.f, aht = 0.f;  // round total, upper buckets
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int k = 16 * r + 2 * e;
                const uint32_t da = __sad(__shfl_sync(0xffffffffu, tql, k), tj, 0u);
                const uint32_t db = __sad(__shfl_sync(0xffffffffu, tql, k + 1), tj, 0u);
                const bool upa = two_t && da >= thr_t, upb = two_t && db >= thr_t;
                const bool ppa = 2 * e >= kp, ppb = 2 * e + 1 >= kp;
                const float ba = (ppa ? hp1 : hp0) + (upa ? ht1 : ht0);
                const float bb = (ppb ? hp1 : hp0) + (upb ? ht1 : ht0);
                float ga, gb;
                bwd_pair_bias(xs[2 * e], xs[2 * e + 1], xd[2 * e], xd[2 * e + 1], half_alpha2, ba,
                              bb, pp[e], dd[e], ga, gb);
                if (!kAll && !((bits >> k) & 1u)) ga = 0.f;
                if (!kAll && !((bits >> (k + 1)) & 1u)) gb = 0.f;
                acc += ga;
                ahp += ppa ? ga : 0.f;
                aht += upa ? ga : 0.f;
                acc += gb;
                ahp += ppb ? gb : 0.f;
                aht += upb ? gb : 0.f;
              }
              // lower then upper bucket (an exact zero adds nothing)
              const float lop = acc - ahp, lot = acc - aht;
              if (lop != 0.f) run_add(run_p, sum_p, pend_p, psum_p, b0p, lop);
              if (ahp != 0.f) run_add(run_p, sum_p, pend_p, psum_p, b0p + 1, ahp);
              if (lot != 0.f) run_add(run_t, sum_t, pend_t, psum_t, 32 + b0t, lot);
              if (aht != 0.f) run_add(run_t, sum_t, pend_t, psum_t, 33 + b0t, aht);
            };
            // other rounds: each score extends its runs one by one
            auto rab_round = [&]() {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int k = 16 * r + 2 * e;
                const int bpa = rab_log_bucket(rab_pos_u(__viaddmin_s32(c0 + col, k, Lh), 1 - rr));
                const int bpb =
                    rab_log_bucket(rab_pos_u(__viaddmin_s32(c0 + col, k + 1, Lh), 1 - rr));
                const int bta =
                    rab_log_bucket(rab_time_u(__shfl_sync(0xffffffffu, tql, k), tj)) & 31;
                const int btb =
                    rab_log_bucket(rab_time_u(__shfl_sync(0xffffffffu, tql, k + 1), tj)) & 31;
                const float ba = rab_half_bias(tabp, tabt, bpa, bta);
                const float bb = rab_half_bias(tabp, tabt, bpb, btb);
                float ga, gb;
                bwd_pair_bias(xs[2 * e], xs[2 * e + 1], xd[2 * e], xd[2 * e + 1], half_alpha2, ba,
                              bb, pp[e], dd[e], ga, gb);
                if ((bits >> k) & 1u) {
                  run_add(run_p, sum_p, pend_p, psum_p, bpa, ga);
                  run_add(run_t, sum_t, pend_t, psum_t, 32 + bta, ga);
                }
                if ((bits >> (k + 1)) & 1u) {
                  run_add(run_p, sum_p, pend_p, psum_p, bpb, gb);
                  run_add(run_t, sum_t, pend_t, psum_t, 32 + btb, gb);
                }
              }
            };
            if (__all_sync(0xffffffffu, flat)) {
              if (full)
                rab_flat(std::true_type{});
              else
                rab_flat(std::false_type{});
            } else if (!__all_sync(0xffffffffu, two))
              rab_round();
            else if (full)
              rab_two(std::true_type{});
            else
              rab_two(std::false_type{});
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              bwd_pair(xs[2 * e], xs[2 * e + 1], xd[2 * e], xd[2 * e + 1], half_alpha2, pp[e],
                       dd[e]);
          }
          if (!full) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              pp[e] = mask_pair(pp[e], bits, e);
              dd[e] = mask_pair(dd[e], bits, e);
            }
          }
          tmem_st8(xs_addr + 16 * r, pp);
          tmem_st8(xs_addr + 16 * r + 8, dd);
#pragma unroll
          for (int q = 0; q < 2; ++q)
            st_shared_v4(dsr + ((((uint32_t)(2 * chunk + q)) ^ swz) << 4), dd[4 * q],
                         dd[4 * q + 1], dd[4 * q + 2], dd[4 * q + 3]);
        }
        if constexpr (RAB) {  // the step's finished runs, equal bins added up first
          if (__any_sync(0xffffffffu, (pend_p >= 0) | (pend_t >= 0))) {
            warp_flush_runs(hst, pend_p, psum_p, pend_t, psum_t, lane);
            pend_p = pend_t = -1;
          }
        }
        fence_proxy_async_smem();  // visible to the dQ MMA
        tmem_st_wait();
        tc_fence_before();
        if (!withhold) warp_arrive(bar(F_OP_FULL + b));
        withhold = false;
        // the previous step's dQ^T, issued right after this step's dP^T
        if (n > 0) {
          ok = drain(xc - 1, prev_c0);
          if (!ok) break;
        }
        prev_c0 = c0;
      }
      if (!ok) break;
      ok = drain(xc - 1, prev_c0);  // the unit's last step
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = warp_wait(bar(F_ACC_FULL), accn & 1, ws);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        uint32_t x0[16], x1[16], o[16];
        const uint32_t cbase = lane_base + (which ? kColAcc2 : kColAcc1) + chunk * 32;
        tmem_ld16(cbase, x0);
        tmem_ld16(cbase + 16, x1);
        tmem_ld_wait2(x0, x1);
        const float sc = which ? sc_dk : sc_dv;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          o[e] = pack_bf16x2(__uint_as_float(x0[2 * e]) * sc, __uint_as_float(x0[2 * e + 1]) * sc);
          o[8 + e] =
              pack_bf16x2(__uint_as_float(x1[2 * e]) * sc, __uint_as_float(x1[2 * e + 1]) * sc);
        }
        if (which == 1) {  // both accumulators read: the next unit may start
          tc_fence_before();
          warp_arrive(bar(F_ACC_EMPTY));
          ++accn;
        }
        if (rr < t1) {
          uint4* dst = reinterpret_cast<uint4*>(which ? o2 : o1);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        }
      }
      if constexpr (RAB) {
        // the unit's last runs, lanes with equal buckets added up first
        warp_flush_runs(hst, run_p, sum_p, run_t, sum_t, lane);
        // this warp's sums of the unit are in; the first pointwise warp adds
        // the unit's histogram into this head's table gradients (dS2 is
        // 2 dP SiLU'(x); the gradient takes dP SiLU'(x) / N) and clears it
        warp_arrive(bar(F_H_DONE + (hu & 1)));
        if (pw == 0) {
          ok = warp_wait(bar(F_H_DONE + (hu & 1)), (hu >> 1) & 1, ws);
          if (!ok) break;
          const float sc = 0.5f * A.inv_n;
          for (int bin = lane; bin < kHistBins; bin += 32) {
            float v = 0.f;
            for (int cp = 0; cp < kHistCopies; ++cp) v += hst0[cp * kHistBins + bin];
            if (v != 0.f) {
              if (bin < 32) {
                if (A.d_rab_pos) atomicAdd(A.d_rab_pos + h * A.nbp + imin(bin, A.nbp - 1), v * sc);
              } else if (A.d_rab_time) {
                atomicAdd(A.d_rab_time + h * A.nbt + imin(bin - 32, A.nbt - 1), v * sc);
              }
            }
            for (int cp = 0; cp < kHistCopies; ++cp) hst0[cp * kHistBins + bin] = 0.f;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(F_H_ZERO + (hu & 1)));
          __syncwarp();
        }
        ++hu;
      }
      warp_arrive(bar(F_U_EMPTY + slot));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The STU layer's form of the step after the one-pass backward: the
// pre-activation gradients of the Q, K, V blocks, in one pass over the rows,
//   dq = bf16(scale * workspace * SiLU'(pre_q))
//   dk = bf16(dk * SiLU'(pre_k)),  dv likewise      (in place)
// and per block the column sums of the three (the bias gradient), stored
// to db_part[block] for silu_db_reduce_kernel.  Thread j: block part j / ch
// (0 Q, 1 K, 2 V; ch = H * D / 8 threads each, a multiple of 32, so parts are
// warp-uniform), columns [8 (j % ch), +8); a block takes a contiguous range
// of rows.
__global__ void __launch_bounds__(384, 2) silu_qkv_kernel(const AttnArgs a, float scale) {
  const int HD = a.H * D, ch = HD / 8;
  const int j = threadIdx.x;
  const int part = j / ch;
  const int cj = (j - part * ch) * 8;
  const int h = cj / D, cd = cj - h * D;
  const int64_t T = a.T;
  const int64_t per = (T + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = blockIdx.x * per, r1 = r0 + per < T ? r0 + per : T;
  const bf16* pre = (part == 0 ? a.pre_q : part == 1 ? a.pre_k : a.pre_v) + cj;
  bf16* g = part == 0 ? a.dq : part == 1 ? a.dk : a.dv;
  const int64_t g_rs = part == 0 ? a.dq_rs : part == 1 ? a.dk_rs : a.dv_rs;
  float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  // kRows rows per round: every load of the round first (the gradient, as
  // fp32 workspace or bf16, and the pre-activation), then the arithmetic and
  // the stores, so that a thread keeps kRows rows of loads in flight
  constexpr int kRows = 3;
  for (int64_t t0 = r0; t0 < r1; t0 += kRows) {
    // ga / gb: the two fp32 halves of a dQ row (Q part) as raw bits, or
    // ga the bf16 dK / dV row (K, V parts)
    uint4 ga[kRows], gb[kRows], pw[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int64_t t = t0 + k < r1 ? t0 + k : t0;  // a missing row repeats the first
      if (part == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(a.dqacc + ((int64_t)h * T + t) * D + cd);
        ga[k] = __ldcs(src);
        gb[k] = __ldcs(src + 1);
      } else {
        ga[k] = *reinterpret_cast<const uint4*>(g + t * g_rs + cj);
      }
      pw[k] = __ldg(reinterpret_cast<const uint4*>(pre + t * a.pre_rs));
    }
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
      const int64_t t = t0 + k;
      if (t >= r1) break;
      float x[8];
      if (part == 0) {
        x[0] = __uint_as_float(ga[k].x) * scale; x[1] = __uint_as_float(ga[k].y) * scale;
        x[2] = __uint_as_float(ga[k].z) * scale; x[3] = __uint_as_float(ga[k].w) * scale;
        x[4] = __uint_as_float(gb[k].x) * scale; x[5] = __uint_as_float(gb[k].y) * scale;
        x[6] = __uint_as_float(gb[k].z) * scale; x[7] = __uint_as_float(gb[k].w) * scale;
      } else {
        const uint32_t ww[4] = {ga[k].x, ga[k].y, ga[k].z, ga[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[2 * e] = __uint_as_float(ww[e] << 16);
          x[2 * e + 1] = __uint_as_float(ww[e] & 0xFFFF0000u);
        }
      }
      const uint32_t pp[4] = {pw[k].x, pw[k].y, pw[k].z, pw[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] *= silu_grad(__uint_as_float(pp[e] << 16));
        x[2 * e + 1] *= silu_grad(__uint_as_float(pp[e] & 0xFFFF0000u));
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sum[e] += x[e];
      uint4 o;
      o.x = pack_bf16x2(x[0], x[1]);
      o.y = pack_bf16x2(x[2], x[3]);
      o.z = pack_bf16x2(x[4], x[5]);
      o.w = pack_bf16x2(x[6], x[7]);
      *reinterpret_cast<uint4*>(g + t * g_rs + cj) = o;
    }
  }
  float4* dst = reinterpret_cast<float4*>(a.db_part + ((int64_t)blockIdx.x * 3 + part) * HD + cj);
  dst[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
  dst[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
}

// db_{q,k,v}[c] += the blocks' partial sums.  Block (x, y) owns 32
// consecutive columns of the 3 * H * D and the partials of blocks y, y +
// gridDim.y, ...; its warp w takes every eighth of those (lane = column, so
// each read is 128 contiguous bytes), then the eight warps' totals are added
// and one atomic per column and block row goes out.
__global__ void __launch_bounds__(256) silu_db_reduce_kernel(const AttnArgs a, int nblk) {
  __shared__ float s_part[8][32];
  const int HD = a.H * D;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;  // in [0, 3 HD)
  const int part = col / HD, c = col - part * HD;
  float v = 0.f;
#pragma unroll 4
  for (int b = blockIdx.y + gridDim.y * w; b < nblk; b += 8 * gridDim.y)
    v += a.db_part[((int64_t)b * 3 + part) * HD + c];
  s_part[w][lane] = v;
  __syncthreads();
  if (w == 0) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += s_part[k][lane];
    atomicAdd((part == 0 ? a.db_q : part == 1 ? a.db_k : a.db_v) + c, t);
  }
}

// dq[t, h, :] = bf16(scale * workspace[h, t, :]), eight head-dim values per
// thread and step.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc,
                                                         bf16* __restrict__ dq, int64_t dq_rs,
                                                         int64_t T, int H, float scale) {
  constexpr int kChunks = D / 8;
  const int64_t n = T * H * kChunks;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t th = i / kChunks;  // t * H + h
    const int c = (int)(i - th * kChunks) * 8;
    const int64_t t = th / H;
    const int h = (int)(th - t * H);
    const float4* src = reinterpret_cast<const float4*>(acc + ((int64_t)h * T + t) * D + c);
    const float4 x0 = __ldcs(src), x1 = __ldcs(src + 1);
    uint4 o;
    o.x = pack_bf16x2(x0.x * scale, x0.y * scale);
    o.y = pack_bf16x2(x0.z * scale, x0.w * scale);
    o.z = pack_bf16x2(x1.x * scale, x1.y * scale);
    o.w = pack_bf16x2(x1.z * scale, x1.w * scale);
    *reinterpret_cast<uint4*>(dq + t * dq_rs + h * D + c) = o;
  }
}

}  // namespace

cudaError_t launch_bwd_fused_grouped(const GroupSet& gs, cudaStream_t st) {
  if (gs.G < 1 || gs.G > kMaxGroups) return cudaErrorInvalidValue;
  BwdMaps m;
  memset(&m, 0, sizeof(m));
  int64_t units = 0;
  cudaError_t e;
  bool rab = false;  // a problem with a relative attention bias
  for (int p = 0; p < gs.G; ++p) {
    const AttnArgs& a = gs.g[p];
    rab = rab || a.rab_pos != nullptr || a.rab_time != nullptr;
    // its table gradients are overwritten (also when it has no tokens)
    if (a.d_rab_pos &&
        (e = cudaMemsetAsync(a.d_rab_pos, 0, sizeof(float) * a.H * a.nbp, st)) != cudaSuccess)
      return e;
    if (a.d_rab_time &&
        (e = cudaMemsetAsync(a.d_rab_time, 0, sizeof(float) * a.H * a.nbt, st)) != cudaSuccess)
      return e;
    if (a.T == 0) continue;  // no units; its maps stay unused
    const int HD = a.H * D;
    if (!make_tma_2d(&m.k[p], a.k, a.T, HD, a.k_rs, BOXW, kRes, true) ||
        !make_tma_2d(&m.v[p], a.v, a.T, HD, a.v_rs, BOXW, kRes, true) ||
        !make_tma_2d(&m.q[p], a.q, a.T, HD, a.q_rs, BOXW, kStr, true) ||
        !make_tma_2d(&m.dout[p], a.dout, a.T, HD, a.do_rs, BOXW, kStr, true))
      return cudaErrorInvalidValue;
    if (!gs.cleared &&
        (e = cudaMemsetAsync(a.dqacc, 0, dq_workspace_bytes(a.T, a.H, D), st)) != cudaSuccess)
      return e;
    units += max_items(a.T, a.B) * a.H;
  }
  if (units == 0) return cudaSuccess;
  auto kern = rab ? bwd_kvq_kernel<true> : bwd_kvq_kernel<false>;
  if (gs.stall) kern = bwd_kvq_kernel<false, true>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  kern<<<grid, kThreads, SMEM, st>>>(m, gs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int p = 0; p < gs.G; ++p) {
    const AttnArgs& a = gs.g[p];
    if (a.T == 0) continue;
    if (a.pre_q != nullptr) {  // STU layer: SiLU' of Q, K, V and the bias gradient
      const int HD = a.H * D;
      // one wave of blocks (as many as fit on every SM), at least ~128 rows
      // each, at most kSiluBlocks
      int per_sm = 1;
      if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, silu_qkv_kernel,
                                                             3 * HD / 8, 0)) != cudaSuccess)
        return e;
      const int64_t wave = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
      const int64_t want = (a.T + 127) / 128;
      int64_t nb = want < wave ? want : wave;
      nb = nb < kSiluBlocks ? nb : kSiluBlocks;
      const int nblk = (int)(nb > 0 ? nb : 1);
      silu_qkv_kernel<<<nblk, 3 * HD / 8, 0, st>>>(a, 0.5f * a.alpha * a.inv_n);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      silu_db_reduce_kernel<<<dim3(3 * HD / 32, 8), 256, 0, st>>>(a, nblk);
    } else {
      dq_convert_kernel<<<sms * 8, 256, 0, st>>>(a.dqacc, a.dq, a.dq_rs, a.T, a.H,
                                                 0.5f * a.alpha * a.inv_n);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_bwd_fused(const AttnArgs& a, cudaStream_t st, bool cleared) {
  if (a.T == 0) return cudaSuccess;
  GroupSet gs;
  memset(&gs, 0, sizeof(gs));
  gs.g[0] = a;
  gs.common = a.ws;
  gs.G = 1;
  gs.cleared = cleared ? 1 : 0;
  return launch_bwd_fused_grouped(gs, st);
}

}  // namespace hstu
