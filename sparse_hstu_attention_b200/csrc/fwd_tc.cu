// SLA HSTU attention forward on the 5th-generation tensor cores (tcgen05).
//
//   out_i = (1/N) sum_j M(i,j) SiLU(alpha q_i.k_j) v_j
// ("Bending the Scaling Law Curve in Large-Scale Recommendation Systems",
// section 3, Eq. 3, under the Semi-Local Attention mask of section 4.2.1,
// Eq. 7; candidates per the M-FALCON mask of the HSTU notes.)
//
// Persistent, warp-specialised: one CTA per SM walks (head, 128-row query
// tile) work units.  Per unit only the key tiles that the SLA mask leaves
// non-empty are visited (global prefix, local band, candidates' diagonal).
//   warp 0      decodes each unit once into a 4-slot shared-memory ring that
//               the other roles read, and loads Q tiles (two alternating
//               buffers) and K tiles (ring) by TMA, 128B-swizzled boxes of
//               64 head-dim columns.
//   warp 1      allocates TMEM; one lane issues UMMA: S = Q K^T (M=128,
//               N=128, K=d) into one of three TMEM score buffers, and
//               O += P V (M=128, N=d, K=128) with P read from TMEM.  S runs
//               two key tiles ahead of P V, so the pointwise stage of a tile
//               has two tile periods of tensor work to hide behind.
//   warp 2      loads V tiles into their own ring, so a K load never queues
//               behind a V slot that is still being read.
//   warps 3..18 pointwise: two groups of eight take alternate key tiles;
//               TMEM -> registers, P = SiLU(alpha S) (masked only on partial
//               tiles) as bf16 written back over the scores it replaces;
//               after a unit's last key tile all sixteen run the epilogue:
//               O * (1/N) -> bf16 -> global, rows past the sequence end not
//               written.
// TMEM columns: score buffers [0,128) [128,256) [256,384), O [384,384+d).
// P of score columns [32c, 32c+32) lives in columns [32c, 32c+16) of the
// same buffer; the P V MMA for keys [16k, 16k+16) reads 8 columns there.
// A score buffer is rewritten only by an S MMA issued after the P V MMA that
// read it (tcgen05.mma from one thread executes in issue order).
// SiLU(x) = h + h tanh(h), h = x/2: one MUFU op per score; 1/N applied once.
// Every wait is bounded; on a timeout the kernel records HSTU_SLA_ERR_TIMEOUT,
// drains what it issued and frees TMEM.
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace hstu {

bool make_tma_2d(CUtensorMap* m, const void* ptr, int64_t T, int HD, int64_t rs, int box_w,
                 int box_h, bool sw128);
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 128, kPwWarps = 16, kSBufs = 3, kUSlots = 4;
constexpr int kPwWarp0 = 3;                         // first pointwise warp
constexpr int kThreads = 32 * (kPwWarp0 + kPwWarps);
constexpr uint32_t kColS = 0, kColO = 384, kTmemCols = 512;

template <int D>
struct Cfg {
  // Ring depths, as deep as 227 KB of shared memory allows.  A K slot is
  // free again once the S MMA that read it has completed, which the score
  // buffer's S_FULL barrier already signals; that reuse needs kKSt <= 3 (a
  // buffer's next S cannot complete before the load that waits on it).
  static constexpr int kKSt = 3;
  static constexpr int kVSt = D == 128 ? 2 : 4;
  static constexpr int SW = D >= 64 ? 128 : 64;   // swizzle span (bytes) = one box row
  static constexpr int BOXW = SW / 2;             // bf16 elements per box row
  static constexpr int NB = D / BOXW;             // boxes per tile
  static constexpr int BLK = 128 * SW;            // bytes per box (128 rows)
  static constexpr int TILE = 128 * D * 2;        // bytes per Q / K / V tile
  static constexpr int OFF_Q = 0;                 // two Q buffers
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = (2 + kKSt) * TILE;
  static constexpr int OFF_BAR = (2 + kKSt + kVSt) * TILE;
  static constexpr int OFF_UNIT = OFF_BAR + 512;
  static constexpr int OFF_SLOT = OFF_UNIT + kUSlots * (int)sizeof(UnitRec);
  static constexpr int SMEM = OFF_SLOT + 16 + 1024;  // + 1 KB alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr uint32_t SWZ = SW == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t SBO = 8 * SW;             // stride of 8-row groups
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kBN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
};

// Barrier slots (8 bytes each) after the tiles.
constexpr int kMaxSt = 4;
enum {
  BAR_Q_FULL = 0, BAR_Q_EMPTY = 2, BAR_K_FULL = 4, BAR_V_FULL = BAR_K_FULL + kMaxSt, BAR_V_EMPTY = BAR_V_FULL + kMaxSt,
  BAR_S_FULL = BAR_V_EMPTY + kMaxSt, BAR_P_FULL = BAR_S_FULL + kSBufs,
  BAR_O_FULL = BAR_P_FULL + kSBufs, BAR_O_EMPTY, BAR_U_FULL, BAR_U_EMPTY = BAR_U_FULL + kUSlots,
  BAR_DRAIN = BAR_U_EMPTY + kUSlots, BAR_OST, BAR_COUNT = BAR_OST + 2
};
static_assert(8 * BAR_COUNT <= 512, "barrier area");

// Unit u of the schedule (units are taken from an atomic counter in order, so
// a CTA that drew short units takes more of them).  The problems' units follow
// one another; within problem p, unit u is head u / n_items, query tile
// items[u % n_items]; the record gets the key tiles it meets.  Past the last
// unit the record ends the schedule.
__device__ void decode_unit(const GroupSet& gs, int u, UnitRec* r) {
  for (int p = 0; p < kMaxGroups && p < gs.G; ++p) {
    const AttnArgs& a = gs.g[p];
    const int n_items = a.ws->n_items;
    const int units = n_items * a.H;
    if (u < units) {
      const int h = u / n_items;
      const int2 it = a.items[u - h * n_items];
      const SeqGeom g = seq_geom(a, it.x);
      const int t0 = it.y * kBM;
      const int t1 = imin(t0 + kBM, g.L);
      unit_rec_fill(r, h, g.s0, g.L, g.Lh, t0, t1,
                    q_tile_key_tiles(t0, t1, g.Lh, a.K1, a.K2e, kBN));
      r->grp = p;
      return;
    }
    u -= units;
  }
  r->nsteps = -1;
}

// q, k, v, out maps of every problem of a launch.
struct FwdMaps {
  CUtensorMap q[kMaxGroups], k[kMaxGroups], v[kMaxGroups], o[kMaxGroups];
};

// RAB: add the relative attention bias to every score (AttnArgs::rab_*).
// STALL (the wait-timeout test hook only): each pointwise warp withholds
// its P_FULL arrive of the first tile it processes, so the MMA warp's wait
// for that P runs into the launch's wait limit.
template <int D, bool RAB, bool STALL = false>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ FwdMaps maps, const __grid_constant__ GroupSet gs) {
  using C = Cfg<D>;
  constexpr int kKSt = C::kKSt, kVSt = C::kVSt;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  UnitRec* ring = reinterpret_cast<UnitRec*>(base_ptr + C::OFF_UNIT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_SLOT);

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
    for (int qb = 0; qb < 2; ++qb) {
      mbar_init(bar(BAR_Q_FULL + qb), 1);
      mbar_init(bar(BAR_Q_EMPTY + qb), 1 + C::NB);  // last S commit + one per O box stored
    }
    for (int s = 0; s < kKSt; ++s) {
      mbar_init(bar(BAR_K_FULL + s), 1);
    }
    for (int s = 0; s < kVSt; ++s) {
      mbar_init(bar(BAR_V_FULL + s), 1);
      mbar_init(bar(BAR_V_EMPTY + s), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(bar(BAR_S_FULL + b), 1);
      mbar_init(bar(BAR_P_FULL + b), kPwWarps / 2);  // one arrive per warp of the tile's group
    }
    mbar_init(bar(BAR_O_FULL), 1);
    mbar_init(bar(BAR_O_EMPTY), kPwWarps);
    for (int s = 0; s < kUSlots; ++s) {
      mbar_init(bar(BAR_U_FULL + s), 1);
      mbar_init(bar(BAR_U_EMPTY + s), kPwWarps + 2);  // MMA, V loader, pointwise warps
    }
    mbar_init(bar(BAR_DRAIN), 1);
    for (int b = 0; b < C::NB; ++b) mbar_init(bar(BAR_OST + b), 4 * (C::BOXW / 32));
    fence_barrier_init();
    for (int p = 0; p < kMaxGroups && p < gs.G; ++p) {
      if (gs.g[p].T == 0) continue;  // no map was built
      prefetch_tmap(&maps.q[p]);
      prefetch_tmap(&maps.k[p]);
      prefetch_tmap(&maps.v[p]);
      prefetch_tmap(&maps.o[p]);
    }
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
    // ------------------------------------------- unit decoder, Q and K loads
    // The whole warp walks the schedule (every value stays warp-uniform);
    // lane 0 decodes units, arms the barriers and issues the copies.  Unit
    // kk + 1 is decoded right after unit kk's first K load is issued, so its
    // global reads overlap the copies in flight.
    uint32_t qn = 0, kn = 0;
    bool ok = true;
    auto publish = [&](int kk) -> bool {
      const int slot = kk % kUSlots;
      if (!warp_wait(bar(BAR_U_EMPTY + slot), ((kk / kUSlots) & 1) ^ 1, ws)) return false;
      if (lane == 0) {
        decode_unit(gs, atomicAdd(&ws->sched, 1), &ring[slot]);
        mbar_arrive(bar(BAR_U_FULL + slot));
      }
      __syncwarp();
      return true;
    };
    ok = publish(0);
    for (int kk = 0; ok; ++kk) {
      const UnitRec* r = &ring[kk % kUSlots];
      const int nt = r->nsteps;
      if (nt < 0) break;
      if (nt == 0) {
        ok = publish(kk + 1);
        continue;
      }
      const int h = r->h, s0 = r->s0;
      const CUtensorMap* tmq = &maps.q[r->grp];
      const CUtensorMap* tmk = &maps.k[r->grp];
      // Q tiles alternate between two buffers, so the next unit's Q is loaded
      // while the current unit still runs.
      const uint32_t qb = qn & 1;
      ok = warp_wait(bar(BAR_Q_EMPTY + qb), ((qn >> 1) & 1) ^ 1, ws);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(bar(BAR_Q_FULL + qb), C::TILE);
        for (int b = 0; b < C::NB; ++b)
          tma_load_2d(sQ + qb * C::TILE + b * C::BLK, tmq, bar(BAR_Q_FULL + qb),
                      h * D + b * C::BOXW, s0 + r->t0);
      }
      ++qn;
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt && ok; ++n, c.next(r)) {
        // the slot's previous tile, kn - kKSt, must have been read by its S MMA
        const int s = kn % kKSt;
        if (kn >= (uint32_t)kKSt) {
          const uint32_t prev = kn - kKSt;
          ok = warp_wait(bar(BAR_S_FULL + prev % kSBufs), (prev / kSBufs) & 1, ws);
          if (!ok) break;
        }
        if (lane == 0) {
          mbar_expect_tx(bar(BAR_K_FULL + s), C::TILE);
          for (int b = 0; b < C::NB; ++b)
            tma_load_2d(sK + s * C::TILE + b * C::BLK, tmk, bar(BAR_K_FULL + s),
                        h * D + b * C::BOXW, s0 + c.j * kBN);
        }
        ++kn;
        if (n == 0) ok = publish(kk + 1);
      }
    }
    // If any role gave up, every load issued must still land before the CTA
    // exits (each barrier has at most its last armed phase outstanding).
    if (lane == 0 && load_status(ws) != 0) {
      for (uint32_t qb = 0; qb < 2; ++qb) {
        const uint32_t armed = qn / 2 + (qb < (qn & 1) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(BAR_Q_FULL + qb), (armed - 1) & 1);
      }
      for (int s = 0; s < kKSt; ++s) {
        const uint32_t armed = kn / kKSt + (s < (int)(kn % kKSt) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(BAR_K_FULL + s), (armed - 1) & 1);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------- V loads
    uint32_t vn = 0;
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(BAR_U_FULL + slot), (kk / kUSlots) & 1, ws);
      if (!ok) break;
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps, h = r->h, s0 = r->s0;
      const CUtensorMap* tmv = &maps.v[nt > 0 ? r->grp : 0];
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt && ok; ++n, c.next(r)) {
        const int s = vn % kVSt;
        ok = warp_wait(bar(BAR_V_EMPTY + s), ((vn / kVSt) & 1) ^ 1, ws);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(bar(BAR_V_FULL + s), C::TILE);
          for (int b = 0; b < C::NB; ++b)
            tma_load_2d(sV + s * C::TILE + b * C::BLK, tmv, bar(BAR_V_FULL + s),
                        h * D + b * C::BOXW, s0 + c.j * kBN);
        }
        ++vn;
      }
      warp_arrive(bar(BAR_U_EMPTY + slot));
      if (nt < 0) break;
    }
    if (lane == 0 && load_status(ws) != 0) {
      for (int s = 0; s < kVSt; ++s) {
        const uint32_t armed = vn / kVSt + (s < (int)(vn % kVSt) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(BAR_V_FULL + s), (armed - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    // The whole warp runs this role converged and computes every descriptor
    // together (warp-uniform values); one elected lane issues each UMMA and
    // commit.  Per tile there are only two commits (S_FULL, which also frees
    // the K slot, and V_EMPTY).
    // Tiles are numbered across units: tile t uses score buffer t % 3, K slot
    // t % kKSt and V slot t % kVSt; its P V is issued once S of tile t + 2 is
    // issued, or earlier while the warp waits for a copy, so P V of a unit's
    // last tiles overlaps S of the next unit's first.
    {
      constexpr uint32_t kAll = 0xffffffffu;
      uint32_t qn = 0, tc = 0, pvc = 0, on = 0;
      uint32_t pend = 0;  // 2 bits per tile in [pvc, tc): first / last of its unit
      bool ok = true;
      // Descriptor bases; a k-step / stage only adds to the start-address field
      // (smem addresses stay below 2^18, so the 14-bit field never carries).
      const uint64_t dQ = smem_desc(sQ, 16, C::SBO, C::SWZ);
      const uint64_t dK = smem_desc(sK, 16, C::SBO, C::SWZ);
      const uint64_t dV = smem_desc(sV, C::BLK, C::SBO, C::SWZ);
      auto kstep = [](int ks) -> uint32_t {  // byte offset of k-step ks in a K-major tile
        return (uint32_t)(((ks * 32) / C::SW) * C::BLK + (ks * 32) % C::SW);
      };
      auto commit = [&](uint32_t b) {
        if (elect_one()) tc_commit(b);
        __syncwarp();
      };
      // O += P V for tile pvc, its operands known to be ready.  Every operand
      // is computed by the whole warp (warp-uniform); one elected lane issues
      // the batch with immediate offsets only (a lone lane in a divergent
      // branch pays ~60 clk per tcgen05.mma against ~10 here).
      auto pv_issue = [&]() {
        const uint32_t f = pend & 3u;
        pend >>= 2;
        const bool first = (f & 1u) != 0, last = (f & 2u) != 0;
        const uint32_t b = pvc % kSBufs;
        const int s = pvc % kVSt;
        tc_fence_after();
        const uint64_t dv = dV + ((uint32_t)(s * C::TILE) >> 4);
        const uint32_t pa = tmem + kColS + b * 128;
        const uint32_t acc0 = first ? 0u : 1u;
        const uint32_t bar_v = bar(BAR_V_EMPTY + s), bar_o = bar(BAR_O_FULL);
        if (elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks)
            mma_ts(tmem + kColO, pa + (ks >> 1) * 32 + (ks & 1) * 8,
                   dv + ((uint32_t)(ks * 16 * C::SW) >> 4), C::IDESC_O, ks > 0 ? 1u : acc0);
          tc_commit(bar_v);
          if (last) tc_commit(bar_o);
        }
        __syncwarp();
        if (last) ++on;
        ++pvc;
      };
      auto pv_ready = [&]() -> bool {  // P, V (and O, for a unit's first) of tile pvc
        return __all_sync(
            kAll, mbar_test_wait(bar(BAR_P_FULL + pvc % kSBufs), (pvc / kSBufs) & 1) &&
                      mbar_test_wait(bar(BAR_V_FULL + pvc % kVSt), (pvc / kVSt) & 1) &&
                      ((pend & 1u) == 0 || mbar_test_wait(bar(BAR_O_EMPTY), (on & 1) ^ 1)));
      };
      auto pv = [&]() -> bool {  // blocking form
        if (!warp_wait(bar(BAR_P_FULL + pvc % kSBufs), (pvc / kSBufs) & 1, ws)) return false;
        if (!warp_wait(bar(BAR_V_FULL + pvc % kVSt), (pvc / kVSt) & 1, ws)) return false;
        if ((pend & 1u) && !warp_wait(bar(BAR_O_EMPTY), (on & 1) ^ 1, ws)) return false;
        pv_issue();
        return true;
      };
      // Waits for a load / the next unit while issuing every deferred P V as
      // soon as its operands are ready.  What these waits depend on (the
      // producer's next copies, which may wait for a unit's epilogue to free
      // its Q buffer or ring slot) can depend on deferred P V, so they must
      // never sit behind such a wait.
      auto wait_issuing = [&](uint32_t b, uint32_t parity) -> bool {
        if (__all_sync(kAll, mbar_test_wait(b, parity))) return true;
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 1;; ++it) {
          // try_wait may suspend the warp in hardware until the phase
          // completes, leaving the issue slots of its sub-partition to the
          // pointwise warps there; deferred P V readiness is polled between
          if (__all_sync(kAll, mbar_try_wait(b, parity))) return true;
          if (pvc != tc && pv_ready()) {
            pv_issue();
            continue;
          }
          if ((it & 255u) == 0) {
            if (__any_sync(kAll, load_status(ws) != 0)) return false;
            if (__any_sync(kAll, globaltimer() - t0 > wait_limit(ws, kWaitLimitNs))) {
              if (lane == 0) set_status(ws, HSTU_SLA_ERR_TIMEOUT);
              return false;
            }
          }
        }
      };
      for (int kk = 0; ok; ++kk) {
        const int slot = kk % kUSlots;
        ok = wait_issuing(bar(BAR_U_FULL + slot), (kk / kUSlots) & 1);
        if (!ok) break;
        const int nt = __shfl_sync(kAll, ring[slot].nsteps, 0);
        warp_arrive(bar(BAR_U_EMPTY + slot));
        if (nt < 0) break;
        if (nt == 0) continue;
        const uint32_t qb = qn & 1;
        ok = wait_issuing(bar(BAR_Q_FULL + qb), (qn >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        for (int n = 0; n < nt; ++n) {
          const int s = tc % kKSt;
          ok = wait_issuing(bar(BAR_K_FULL + s), (tc / kKSt) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = tc % kSBufs;
          const uint64_t dk = dK + ((uint32_t)(s * C::TILE) >> 4);
          const uint64_t dq = dQ + ((uint32_t)(qb * C::TILE) >> 4);
          const uint32_t sd = tmem + kColS + b * 128;
          const uint32_t bar_s = bar(BAR_S_FULL + b), bar_q = bar(BAR_Q_EMPTY + qb);
          const bool last_q = n + 1 == nt;
          if (elect_one()) {
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_ss(sd, dq + (kstep(ks) >> 4), dk + (kstep(ks) >> 4), C::IDESC_S,
                     ks > 0 ? 1u : 0u);
            tc_commit(bar_s);
            if (last_q) tc_commit(bar_q);  // last S read of this Q tile
          }
          __syncwarp();
          pend |= ((n == 0 ? 1u : 0u) | (n + 1 == nt ? 2u : 0u)) << (2 * (tc - pvc));
          ++tc;
          // the score buffer of tile tc (next S) is free once P V of tc - 3
          // is issued: keep at most two tiles' P V pending
          if (tc - pvc > 2) {
            ok = pv();
            if (!ok) break;
          }
        }
        ++qn;
      }
      while (ok && pvc != tc) ok = pv();
      // Every MMA issued must finish before TMEM is released.
      commit(bar(BAR_DRAIN));
      drain_wait(bar(BAR_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------- pointwise and epilogue
    // Two groups of eight warps take alternate key tiles, so one group's TMEM
    // load / store latency overlaps the other's arithmetic.  Within a group,
    // the two warps on a 32-lane TMEM quarter split the tile's 128 columns in
    // halves.  The epilogue uses all sixteen: warp `chunk` of a quarter writes
    // O columns [32 chunk, +32).
    const int pw = warp - kPwWarp0;        // 0..15
    const int grp = pw >> 3;               // tile parity of this warp
    const int quarter = warp & 3;          // TMEM lanes [32*quarter, +32)
    const int chunk = pw >> 2;             // 0..3
    const int half = chunk & 1;            // column half within the group
    const int row = quarter * 32 + lane;   // row of the 128-row tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool has_o = chunk < D / 32;     // this warp writes an O chunk
    // Epilogue store: a tile that lies inside its sequence is staged as bf16
    // in the unit's Q buffer (no S MMA reads it any more) in the swizzled
    // layout of a TMA box and stored by one thread per box; that thread
    // releases the Q buffer once the store has read it.  Tiles that run past
    // the sequence end are written row by row, rows past the end skipped.
    const int box = (chunk * 32) / C::BOXW;          // O box of this warp's chunk
    const int box_c0 = ((chunk * 32) % C::BOXW) / 8;  // its first 16-byte chunk in a box row
    const bool box_leader = has_o && quarter == 0 && (chunk * 32) % C::BOXW == 0;
    const uint32_t swz = C::SW == 128 ? (uint32_t)(row & 7) : (uint32_t)((row >> 1) & 3);
    // A unit's epilogue is deferred until this warp has done its first key
    // tile of the next unit (whose scores are ready by then), so the P of a
    // unit's first tiles does not wait for the previous unit's last P V and
    // epilogue.  The deferred unit keeps its ring slot until then.  Every
    // epilogue and Q-buffer release completes before the warp waits on a
    // tile of the unit after next, whose Q load depends on them.
    uint32_t tc = 0, on = 0, qn = 0;
    bool withhold = STALL;  // the test hook's one withheld arrive
    bool ep_pend = false;
    int e_h = 0, e_s0 = 0, e_t0 = 0, e_t1 = 0, e_slot = 0, e_grp = 0;
    uint32_t e_qn = 0;
    int rel_qb = -1;  // box leaders: Q buffer whose O stores are issued, not yet released
    auto release = [&]() {
      if (rel_qb >= 0) {
        if (lane == 0) {
          bulk_wait_read_all();
          mbar_arrive(bar(BAR_Q_EMPTY + rel_qb));
        }
        __syncwarp();
        rel_qb = -1;
      }
    };
    auto epilogue = [&]() -> bool {
      ep_pend = false;
      if (!warp_wait(bar(BAR_O_FULL), on & 1, ws)) return false;
      tc_fence_after();
      const uint32_t qb = e_qn & 1;
      const bool whole = e_t1 - e_t0 == kBM;
      const int i = e_t0 + row;
      const AttnArgs& E = gs.g[e_grp];
      const float inv_n = E.inv_n;
      uint32_t o[16];
      if (has_o) {
        uint32_t r0[16], r1[16];
        tmem_ld16(lane_base + kColO + chunk * 32, r0);
        tmem_ld16(lane_base + kColO + chunk * 32 + 16, r1);
        tmem_ld_wait2(r0, r1);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          o[e] = pack_bf16x2(__uint_as_float(r0[2 * e]) * inv_n,
                             __uint_as_float(r0[2 * e + 1]) * inv_n);
          o[8 + e] = pack_bf16x2(__uint_as_float(r1[2 * e]) * inv_n,
                                 __uint_as_float(r1[2 * e + 1]) * inv_n);
        }
      }
      // O is in registers: the next unit's P V may overwrite it
      tc_fence_before();
      warp_arrive(bar(BAR_O_EMPTY));
      ++on;
      bool good = true;
      if (has_o) {
        if (whole) {
          const uint32_t rowaddr = sQ + qb * C::TILE + box * C::BLK + row * C::SW;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_shared_v4(rowaddr + ((((uint32_t)(box_c0 + v)) ^ swz) << 4), o[4 * v],
                         o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          fence_proxy_async_smem();  // staged rows visible to the TMA store
        } else if (i < e_t1) {
          uint4* dst = reinterpret_cast<uint4*>(E.out + (int64_t)(e_s0 + i) * E.o_rs + e_h * D +
                                                chunk * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
        warp_arrive(bar(BAR_OST + box));
        if (box_leader) {
          release();
          good = mbar_wait(bar(BAR_OST + box), e_qn & 1, ws);
          if (lane == 0 && good && whole) {
            tma_store_2d(&maps.o[e_grp], sQ + qb * C::TILE + box * C::BLK, e_h * D + box * C::BOXW,
                         e_s0 + e_t0);
            bulk_commit_group();
          }
          good = __all_sync(0xffffffffu, good);
          if (good) {
            if (whole) {
              rel_qb = (int)qb;  // released after this warp's next tile
            } else {
              if (lane == 0) mbar_arrive(bar(BAR_Q_EMPTY + qb));
              __syncwarp();
            }
          }
        }
      }
      warp_arrive(bar(BAR_U_EMPTY + e_slot));
      return good;
    };
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int slot = kk % kUSlots;
      ok = warp_wait(bar(BAR_U_FULL + slot), (kk / kUSlots) & 1, ws);
      if (!ok) break;
      const UnitRec* r = &ring[slot];
      const int nt = r->nsteps;
      if (nt <= 0) {
        if (ep_pend) {
          ok = epilogue();
          if (!ok) break;
        }
        release();
        if (nt < 0) {
          warp_arrive(bar(BAR_U_EMPTY + slot));
          break;
        }
        // no visible key anywhere in the tile
        const int i = r->t0 + row;
        if (has_o && i < r->t1) {
          const AttnArgs& A = gs.g[r->grp];
          uint4* dst = reinterpret_cast<uint4*>(A.out + (int64_t)(r->s0 + i) * A.o_rs +
                                                r->h * D + chunk * 32);
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = z;
        }
        warp_arrive(bar(BAR_U_EMPTY + slot));
        continue;
      }
      const int h = r->h, s0 = r->s0, Lh = r->Lh, t0 = r->t0, t1 = r->t1;
      const int i = t0 + row;  // row within the sequence
      const AttnArgs& A = gs.g[r->grp];
      const int K1 = A.K1, K2e = A.K2e;
      const uint64_t half_alpha2 = f2s(0.5f * A.alpha);
      const RowMask m = row_mask(i, r->L, Lh, K1, K2e);
      // relative attention bias: half of this head's tables' bucket
      // min(lane, nb - 1) in this lane, and this row's timestamp
      float tabp = 0.f, tabt = 0.f;
      int32_t ti = 0;
      if constexpr (RAB) {
        tabp = rab_lane_table(A.rab_pos, A.nbp, h, lane);
        tabt = rab_lane_table(A.rab_time, A.nbt, h, lane);
        ti = (A.ts && i < r->L) ? __ldg(A.ts + s0 + i) : 0;
      }
      SpanCursor c;
      c.begin(r);
      for (int n = 0; n < nt; ++n, ++tc, c.next(r)) {
        if ((int)(tc & 1) != grp) continue;  // the other group's tile
        const uint32_t b = tc % kSBufs;
        const int j0 = c.j * kBN;
        // relative attention bias: this warp's 2 x 32 keys' timestamps, one
        // per lane and round, loaded before the wait for the scores
        int32_t tjr[2] = {0, 0};
        if constexpr (RAB) {
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int jl = j0 + half * 64 + sub * 32 + lane;
            tjr[sub] = (A.ts && jl < r->L) ? __ldg(A.ts + s0 + jl) : 0;
          }
        }
        ok = warp_wait(bar(BAR_S_FULL + b), (tc / kSBufs) & 1, ws);
        if (!ok) break;
        tc_fence_after();
        const bool full = tile_full(t0, t0 + kBM, j0, j0 + kBN, Lh, K1, K2e);
        // P = SiLU(alpha S) = h + h tanh(h) with h = alpha S / 2.  Tiles that
        // are entirely visible skip the mask; the others clear invisible
        // entries with one bit test each against this row's 32-key bitmask.
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const int col = half * 64 + sub * 32;
          const uint32_t taddr = lane_base + kColS + b * 128 + col;
          uint32_t c0[16], c1[16];
          tmem_ld16(taddr, c0);
          tmem_ld16(taddr + 16, c1);
          tmem_ld_wait2(c0, c1);
          uint32_t p[16];
          if constexpr (RAB) {
            // the 32 keys' timestamps, one per lane, then each score's bias:
            // key j = j0 + col + k has u_pos = max(pb - k, 1)
            const int32_t tjl = tjr[sub];
            const int pb = imin(i, Lh) + 1 - (j0 + col);
            // Both buckets are monotone in their difference, so the round's
            // extreme differences bound them: the position over u_pos in
            // [max(pb - 31, 1), max(pb, 1)], the time over the keys'
            // timestamp range [tmin, tmax] (|ti - tj| is largest at an end
            // and smallest at an end, or 0 inside).  When every lane's two
            // buckets are constant over the round, one bias serves all 32
            // scores (the same value the per-score path computes).
            const int32_t tmin = __reduce_min_sync(0xffffffffu, tjl);
            const int32_t tmax = __reduce_max_sync(0xffffffffu, tjl);
            // |ti - tj| as an exact uint32; its bucket as the per-score path
            // uses it (a shuffle lane: 2^32 - 1 lands in lane 31)
            auto tbucket = [](uint32_t dlt) {
              return dlt == 0xffffffffu ? 31 : rab_log_bucket(dlt + 1u);
            };
            const uint32_t da = __sad(ti, tmin, 0u), db = __sad(ti, tmax, 0u);
            const uint32_t d_hi = da > db ? da : db;
            const uint32_t d_lo = (ti >= tmin && ti <= tmax) ? 0u : (da < db ? da : db);
            const int bp_hi = rab_log_bucket(rab_pos_u(pb, 0));
            const int bt_hi = tbucket(d_hi);
            const bool flat =
                rab_log_bucket(rab_pos_u(pb, -31)) == bp_hi && tbucket(d_lo) == bt_hi;
            if (__all_sync(0xffffffffu, flat)) {
              const float hb = rab_half_bias(tabp, tabt, bp_hi, bt_hi);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                p[e] = silu_pair_bias(e < 8 ? c0[2 * e] : c1[2 * e - 16],
                                      e < 8 ? c0[2 * e + 1] : c1[2 * e - 15], half_alpha2, hb, hb);
            } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float ba = rab_half_bias(
                  tabp, tabt, rab_log_bucket(rab_pos_u(pb, -2 * e)),
                  rab_log_bucket(rab_time_u(ti, __shfl_sync(0xffffffffu, tjl, 2 * e))));
              const float bb = rab_half_bias(
                  tabp, tabt, rab_log_bucket(rab_pos_u(pb, -2 * e - 1)),
                  rab_log_bucket(rab_time_u(ti, __shfl_sync(0xffffffffu, tjl, 2 * e + 1))));
              p[e] = silu_pair_bias(e < 8 ? c0[2 * e] : c1[2 * e - 16],
                                    e < 8 ? c0[2 * e + 1] : c1[2 * e - 15], half_alpha2, ba, bb);
            }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              p[e] = silu_pair(c0[2 * e], c0[2 * e + 1], half_alpha2);
              p[8 + e] = silu_pair(c1[2 * e], c1[2 * e + 1], half_alpha2);
            }
          }
          if (!full) {
            const uint32_t bits = row_mask_bits(m, j0 + col);
#pragma unroll
            for (int e = 0; e < 16; ++e) p[e] = mask_pair(p[e], bits, e);
          }
          tmem_st16(taddr, p);  // over the first half of the scores just read
        }
        tmem_st_wait();
        tc_fence_before();
        if (!withhold) warp_arrive(bar(BAR_P_FULL + b));
        withhold = false;
        if (ep_pend) {
          ok = epilogue();
          if (!ok) break;
        } else {
          release();
        }
      }
      if (!ok) break;
      if (ep_pend) {  // no tile of this unit for this warp's group
        ok = epilogue();
        if (!ok) break;
      }
      release();
      ep_pend = true;
      e_h = h; e_s0 = s0; e_t0 = t0; e_t1 = t1; e_slot = slot; e_qn = qn; e_grp = r->grp;
      ++qn;
    }
    // stores still in flight must complete before the CTA exits
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

template <int D>
cudaError_t launch_d(const GroupSet& gs, cudaStream_t st) {
  using C = Cfg<D>;
  FwdMaps m;
  memset(&m, 0, sizeof(m));
  int64_t units = 0;
  for (int p = 0; p < gs.G; ++p) {
    const AttnArgs& a = gs.g[p];
    if (a.T == 0) continue;  // no units; its maps stay unused
    const int HD = a.H * D;
    if (!make_tma_2d(&m.q[p], a.q, a.T, HD, a.q_rs, C::BOXW, kBM, C::SW == 128) ||
        !make_tma_2d(&m.k[p], a.k, a.T, HD, a.k_rs, C::BOXW, kBN, C::SW == 128) ||
        !make_tma_2d(&m.v[p], a.v, a.T, HD, a.v_rs, C::BOXW, kBN, C::SW == 128) ||
        !make_tma_2d(&m.o[p], a.out, a.T, HD, a.o_rs, C::BOXW, kBM, C::SW == 128))
      return cudaErrorInvalidValue;
    units += max_items(a.T, a.B) * a.H;
  }
  if (units == 0) return cudaSuccess;
  bool rab = false;  // any problem with a relative attention bias takes the bias kernel
  for (int p = 0; p < gs.G; ++p) rab = rab || gs.g[p].rab_pos != nullptr || gs.g[p].rab_time != nullptr;
  auto kern = rab ? fwd_tc_kernel<D, true> : fwd_tc_kernel<D, false>;
  if (gs.stall) {
    if constexpr (D == 128) kern = fwd_tc_kernel<D, false, true>;
    else return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  kern<<<grid, kThreads, C::SMEM, st>>>(m, gs);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_grouped(const GroupSet& gs, int d, cudaStream_t st) {
  if (gs.G < 1 || gs.G > kMaxGroups) return cudaErrorInvalidValue;
  if (d == 32) return launch_d<32>(gs, st);
  if (d == 64) return launch_d<64>(gs, st);
  return launch_d<128>(gs, st);
}

cudaError_t launch_fwd_tc(const AttnArgs& a, int d, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  GroupSet gs;
  memset(&gs, 0, sizeof(gs));
  gs.g[0] = a;
  gs.common = a.ws;
  gs.G = 1;
  return launch_fwd_grouped(gs, d, st);
}

}  // namespace hstu
