// SLA HSTU attention backward on the 5th-generation tensor cores (tcgen05).
//
// With x_ij = alpha q_i.k_j, P_ij = M SiLU(x)/N and dP_ij = dO_i.v_j:
//   dV_j = sum_i P_ij dO_i,   dK_j = sum_i dS_ij q_i,   dQ_i = sum_j dS_ij k_j,
//   dS_ij = M dP_ij SiLU'(x_ij) alpha/N
// (the chain rule through "Bending the Scaling Law Curve in Large-Scale
// Recommendation Systems", section 3, Eq. 3, under the SLA mask of section
// 4.2.1, Eq. 7).  With h = x/2 and t = tanh(h): SiLU(x) = h + h t and
// SiLU'(x) = (1 + t)/2 * (1 + h - h t); one MUFU op per score.
//
// Two launches of one kernel template, neither using atomics:
//   KV pass: a resident 128-key tile (K, V) meets streamed 64-row query tiles
//     (Q, dO):  S^T = K Q^T, dP^T = V dO^T  ->  P^T, dS^T (bf16, TMEM)
//     -> dV += P^T dO, dK += dS^T Q, both accumulated in TMEM.
//   Q pass: a resident 128-row query tile (Q, dO) meets streamed 64-key tiles
//     (K, V):  S = Q K^T, dP = dO V^T  ->  dS (bf16, TMEM)  ->  dQ += dS K.
// The Q pass recomputes S and dP instead of scattering dQ partial sums from
// the KV pass: 40% more tensor work, but no fp32 dQ workspace, no atomics and
// a deterministic result.
//
// Roles (persistent CTAs, one per SM, work units handed out dynamically by an
// atomic counter so the long prefix-key units of the KV pass, which every
// later row sees, start first and the rest fill in around them):
//   warp 0      scheduler + TMA producer (resident tiles once per unit,
//               streamed tiles through a 4-stage ring)
//   warp 1      TMEM allocation; one lane issues every UMMA
//   warps 2..17 pointwise (P, dS into TMEM, aliasing the fp32 scores they
//               replace) and the epilogue (accumulators -> bf16 -> global);
//               four warps per 32-lane TMEM quarter hide TMEM latency
// TMEM columns: X1 (scores) [0,64) [64,128), X2 (dP) [128,192) [192,256),
// ACC1 [256,256+d), ACC2 [384,384+d).
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace hstu {

bool make_tma_2d(CUtensorMap* m, const void* ptr, int64_t T, int HD, int64_t rs, int box_w,
                 int box_h, bool sw128);
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kRes = 128, kStr = 64, kStages = 4, kPwWarps = 16;
constexpr int kThreads = 64 + 32 * kPwWarps;
constexpr uint32_t kColX1 = 0, kColX2 = 128, kColAcc1 = 256, kColAcc2 = 384, kTmemCols = 512;

template <int D>
struct BCfg {
  static constexpr int SW = D >= 64 ? 128 : 64;
  static constexpr int BOXW = SW / 2;
  static constexpr int NB = D / BOXW;
  static constexpr int RTILE = kRes * D * 2;
  static constexpr int STILE = kStr * D * 2;
  static constexpr int RBLK = kRes * SW;
  static constexpr int SBLK = kStr * SW;
  static constexpr int OFF_A1 = 0;
  static constexpr int OFF_A2 = RTILE;
  static constexpr int OFF_B1 = 2 * RTILE;
  static constexpr int OFF_B2 = 2 * RTILE + kStages * STILE;
  static constexpr int OFF_BAR = 2 * RTILE + 2 * kStages * STILE;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  static constexpr uint32_t SWZ = SW == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t SBO = 8 * SW;
  static constexpr uint32_t IDESC_X = idesc_bf16(kRes, kStr, false, false);
  static constexpr uint32_t IDESC_ACC = idesc_bf16(kRes, D, false, true);
};

enum {
  B_A_FULL = 0, B_A_EMPTY, B_B_FULL, B_B_EMPTY = B_B_FULL + kStages,
  B_X_FULL = B_B_EMPTY + kStages, B_OP_FULL = B_X_FULL + 2, B_ACC_FULL = B_OP_FULL + 2,
  B_ACC_EMPTY, B_U_FULL, B_U_EMPTY = B_U_FULL + 2, B_DRAIN = B_U_EMPTY + 2, B_PW_SYNC,
  B_COUNT = B_PW_SYNC + 2
};

struct BUnit {
  int h, s0, L, Lh, t0, t1;  // resident tile rows [t0, t1) of the sequence
  Spans sp;                  // streamed tiles (64 rows) that meet it
  int nsteps;
};

template <bool KV>
__device__ __forceinline__ BUnit bunit_at(const AttnArgs& a, const int2* items, int u) {
  BUnit w;
  const int idx = u / a.H;
  w.h = u - idx * a.H;
  const int2 it = items[idx];
  const SeqGeom g = seq_geom(a, it.x);
  w.s0 = g.s0; w.L = g.L; w.Lh = g.Lh;
  w.t0 = it.y * kRes;
  w.t1 = imin(w.t0 + kRes, g.L);
  w.sp = KV ? k_tile_q_tiles(w.t0, w.t1, g.L, g.Lh, a.K1, a.K2e, kStr)
            : q_tile_key_tiles(w.t0, w.t1, g.Lh, a.K1, a.K2e, kStr);
  w.nsteps = w.sp.count();
  return w;
}

template <int D, bool KV>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tma1, const __grid_constant__ CUtensorMap tma2,
                  const __grid_constant__ CUtensorMap tmb1, const __grid_constant__ CUtensorMap tmb2,
                  const AttnArgs a) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sA1 = base + C::OFF_A1, sA2 = base + C::OFF_A2;
  const uint32_t sB1 = base + C::OFF_B1, sB2 = base + C::OFF_B2;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  volatile int* s_unit = reinterpret_cast<volatile int*>(base_ptr + C::OFF_BAR + 8 * B_COUNT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + 8 * B_COUNT + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (load_status(a.ws) != 0) return;
  const int2* items = KV ? a.items2 : a.items;
  const int total = (KV ? a.ws->n_items2 : a.ws->n_items) * a.H;
  int* sched = KV ? &a.ws->sched2 : &a.ws->sched;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_A_FULL), 1);
    mbar_init(bar(B_A_EMPTY), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_B_FULL + s), 1);
      mbar_init(bar(B_B_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_X_FULL + b), 1);
      mbar_init(bar(B_OP_FULL + b), kPwWarps / 2);  // one arrive per warp of group b
      mbar_init(bar(B_PW_SYNC + b), kPwWarps / 2);
      mbar_init(bar(B_U_FULL + b), 1);
      mbar_init(bar(B_U_EMPTY + b), 1 + kPwWarps);  // MMA warp + pointwise warps
    }
    mbar_init(bar(B_ACC_FULL), 1);
    mbar_init(bar(B_ACC_EMPTY), kPwWarps);
    mbar_init(bar(B_DRAIN), 1);
    fence_barrier_init();
    prefetch_tmap(&tma1);
    prefetch_tmap(&tma2);
    prefetch_tmap(&tmb1);
    prefetch_tmap(&tmb2);
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
    // units from the counter, arms barriers and issues the copies.
    uint32_t k = 0, an = 0, bn = 0;
    bool ok = true;
    for (;;) {
      const uint32_t slot = k & 1;
      ok = warp_wait(bar(B_U_EMPTY + slot), ((k >> 1) & 1) ^ 1, a.ws);
      if (!ok) break;
      int u = 0;
      if (lane == 0) {
        u = atomicAdd(sched, 1);
        if (u >= total) u = -1;
        s_unit[slot] = u;
        mbar_arrive(bar(B_U_FULL + slot));
      }
      u = __shfl_sync(0xffffffffu, u, 0);
      ++k;
      if (u < 0) break;
      const BUnit w = bunit_at<KV>(a, items, u);
      if (w.nsteps == 0) continue;
      ok = warp_wait(bar(B_A_EMPTY), (an & 1) ^ 1, a.ws);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(bar(B_A_FULL), 2 * C::RTILE);
        for (int b = 0; b < C::NB; ++b) {
          tma_load_2d(sA1 + b * C::RBLK, &tma1, bar(B_A_FULL), w.h * D + b * C::BOXW, w.s0 + w.t0);
          tma_load_2d(sA2 + b * C::RBLK, &tma2, bar(B_A_FULL), w.h * D + b * C::BOXW, w.s0 + w.t0);
        }
      }
      ++an;
      for (int n = 0; n < w.nsteps; ++n) {
        const int s = bn % kStages;
        ok = warp_wait(bar(B_B_EMPTY + s), ((bn / kStages) & 1) ^ 1, a.ws);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(bar(B_B_FULL + s), 2 * C::STILE);
          const int y = w.s0 + w.sp.at(n) * kStr;
          for (int b = 0; b < C::NB; ++b) {
            tma_load_2d(sB1 + s * C::STILE + b * C::SBLK, &tmb1, bar(B_B_FULL + s),
                        w.h * D + b * C::BOXW, y);
            tma_load_2d(sB2 + s * C::STILE + b * C::SBLK, &tmb2, bar(B_B_FULL + s),
                        w.h * D + b * C::BOXW, y);
          }
        }
        ++bn;
      }
      if (!ok) break;
    }
    if (lane == 0 && load_status(a.ws) != 0) {  // drain copies in flight before exiting
      if (an > 0) drain_wait(bar(B_A_FULL), (an - 1) & 1);
      for (int s = 0; s < kStages; ++s) {
        const uint32_t armed = bn / kStages + (s < (int)(bn % kStages) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(B_B_FULL + s), (armed - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // Whole warp, warp-uniform descriptors; lane 0 issues every UMMA / commit.
    uint32_t k = 0, an = 0, bn = 0, xc = 0, accn = 0;
    bool ok = true;
    // Descriptor bases; offsets only add to the start-address field.
    const uint64_t dA1 = smem_desc(sA1, 16, C::SBO, C::SWZ);
    const uint64_t dA2 = smem_desc(sA2, 16, C::SBO, C::SWZ);
    const uint64_t dB1 = smem_desc(sB1, 16, C::SBO, C::SWZ);
    const uint64_t dB2 = smem_desc(sB2, 16, C::SBO, C::SWZ);
    const uint64_t mB1 = smem_desc(sB1, C::SBLK, C::SBO, C::SWZ);  // MN-major views
    const uint64_t mB2 = smem_desc(sB2, C::SBLK, C::SBO, C::SWZ);
    auto koff = [](int ks, int blk) -> uint32_t {  // k-step ks of a K-major tile, 16-byte units
      return (uint32_t)((((ks * 32) / C::SW) * blk + (ks * 32) % C::SW) >> 4);
    };
    auto acc = [&](uint32_t bm, uint32_t xm, bool first) -> bool {
      const uint32_t b = xm & 1;
      if (!warp_wait(bar(B_OP_FULL + b), (xm >> 1) & 1, a.ws)) return false;
      if (first && !warp_wait(bar(B_ACC_EMPTY), (accn & 1) ^ 1, a.ws)) return false;
      tc_fence_after();
      const int s = bm % kStages;
      if (lane == 0) {
        const uint32_t so = (uint32_t)(s * C::STILE) >> 4;
#pragma unroll
        for (int ks = 0; ks < kStr / 16; ++ks) {
          const uint32_t accum = (!first || ks > 0) ? 1u : 0u;
          const uint32_t ko = so + ((uint32_t)(ks * 16 * C::SW) >> 4);
          if (KV) {
            mma_ts(tmem + kColAcc1, tmem + kColX1 + b * 64 + ks * 8, mB2 + ko, C::IDESC_ACC,
                   accum);  // dV += P^T dO
            mma_ts(tmem + kColAcc2, tmem + kColX2 + b * 64 + ks * 8, mB1 + ko, C::IDESC_ACC,
                   accum);  // dK += dS^T Q
          } else {
            mma_ts(tmem + kColAcc1, tmem + kColX2 + b * 64 + ks * 8, mB1 + ko, C::IDESC_ACC,
                   accum);  // dQ += dS K
          }
        }
        tc_commit(bar(B_B_EMPTY + s));
      }
      __syncwarp();
      return true;
    };
    for (;;) {
      const uint32_t slot = k & 1;
      ok = warp_wait(bar(B_U_FULL + slot), (k >> 1) & 1, a.ws);
      if (!ok) break;
      const int u = s_unit[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_U_EMPTY + slot));
      ++k;
      if (u < 0) break;
      const BUnit w = bunit_at<KV>(a, items, u);
      if (w.nsteps == 0) continue;
      ok = warp_wait(bar(B_A_FULL), an & 1, a.ws);
      if (!ok) break;
      tc_fence_after();
      const uint32_t bn0 = bn, xc0 = xc;
      for (int n = 0; n < w.nsteps; ++n) {
        const int s = bn % kStages;
        ok = warp_wait(bar(B_B_FULL + s), (bn / kStages) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b = xc & 1;
        if (lane == 0) {
          const uint32_t so = (uint32_t)(s * C::STILE) >> 4;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            mma_ss(tmem + kColX1 + b * 64, dA1 + koff(ks, C::RBLK), dB1 + so + koff(ks, C::SBLK),
                   C::IDESC_X, ks > 0 ? 1u : 0u);
            mma_ss(tmem + kColX2 + b * 64, dA2 + koff(ks, C::RBLK), dB2 + so + koff(ks, C::SBLK),
                   C::IDESC_X, ks > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_X_FULL + b));
          if (n + 1 == w.nsteps) tc_commit(bar(B_A_EMPTY));  // last use of the resident tiles
        }
        __syncwarp();
        if (n > 0) {
          ok = acc(bn - 1, xc - 1, n == 1);
          if (!ok) break;
        }
        ++bn;
        ++xc;
      }
      if (!ok) break;
      ok = acc(bn0 + w.nsteps - 1, xc0 + w.nsteps - 1, w.nsteps == 1);
      if (!ok) break;
      if (lane == 0) tc_commit(bar(B_ACC_FULL));
      __syncwarp();
      ++an;
      ++accn;
    }
    if (lane == 0) {
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
    // `chunk` of a quarter writes accumulator columns [32 chunk, +32).
    const int pw = warp - 2;
    const int grp = pw >> 3;              // X buffer / step parity of this warp
    const int quarter = warp & 3;
    const int chunk = pw >> 2;            // 0..3
    const int half = chunk & 1;           // streamed-column half within the group
    const int row = quarter * 32 + lane;  // resident row of this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float half_alpha = 0.5f * a.alpha;
    const float sc1 = KV ? a.inv_n : a.alpha * a.inv_n;  // ACC1: dV or dQ
    const float sc2 = a.alpha * a.inv_n;                 // ACC2: dK
    bf16* out1 = KV ? a.dv : a.dq;
    const int64_t rs1 = KV ? a.dv_rs : a.dq_rs;
    const int col = half * 32;
    const bool has_acc = chunk < D / 32;
    uint32_t k = 0, xc = 0, accn = 0;
    bool ok = true;
    for (;;) {
      const uint32_t slot = k & 1;
      ok = warp_wait(bar(B_U_FULL + slot), (k >> 1) & 1, a.ws);
      if (!ok) break;
      const int u = s_unit[slot];
      warp_arrive(bar(B_U_EMPTY + slot));
      ++k;
      if (u < 0) break;
      const BUnit w = bunit_at<KV>(a, items, u);
      const int r = w.t0 + row;  // this thread's resident position in the sequence
      bf16* o1 = out1 + (int64_t)(w.s0 + r) * rs1 + w.h * D + chunk * 32;
      bf16* o2 = a.dk + (int64_t)(w.s0 + r) * a.dk_rs + w.h * D + chunk * 32;
      if (w.nsteps == 0) {
        if (has_acc && r < w.t1) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            reinterpret_cast<uint4*>(o1)[v] = z;
            if (KV) reinterpret_cast<uint4*>(o2)[v] = z;
          }
        }
        continue;
      }
      const KeyMask km = key_mask(r, w.L, w.Lh, a.K1, a.K2e);
      const RowMask rm = row_mask(r, w.L, w.Lh, a.K1, a.K2e);
      for (int n = 0; n < w.nsteps; ++n, ++xc) {
        const uint32_t b = xc & 1;
        if ((int)b != grp) continue;  // the other group's step
        ok = warp_wait(bar(B_X_FULL + b), (xc >> 1) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const int c0 = w.sp.at(n) * kStr;  // first streamed position of this step
        const bool full = KV ? tile_full(c0, c0 + kStr, w.t0, w.t0 + kRes, w.Lh, a.K1, a.K2e)
                             : tile_full(w.t0, w.t0 + kRes, c0, c0 + kStr, w.Lh, a.K1, a.K2e);
        uint32_t xs0[16], xs1[16], xd0[16], xd1[16];
        tmem_ld16(lane_base + kColX1 + b * 64 + col, xs0);
        tmem_ld16(lane_base + kColX1 + b * 64 + col + 16, xs1);
        tmem_ld16(lane_base + kColX2 + b * 64 + col, xd0);
        tmem_ld16(lane_base + kColX2 + b * 64 + col + 16, xd1);
        tmem_ld_wait2(xs0, xs1);
        tmem_ld_wait2(xd0, xd1);
        // every score of the group is in registers before P / dS overwrite
        // them (a bounded barrier over the group's warps, one phase per step)
        warp_arrive(bar(B_PW_SYNC + b));
        ok = warp_wait(bar(B_PW_SYNC + b), (xc >> 1) & 1, a.ws);
        if (!ok) break;
        // P = SiLU(x) and dS = dP SiLU'(x) for x = alpha S, with h = x/2 and
        // t = tanh(h): SiLU = h + h t, SiLU' = (1 + t)/2 (1 + h - h t).
        // Fully visible tiles skip the mask; others clear invisible entries
        // by one bit test against this thread's 32-position visibility mask.
        const uint32_t bits =
            full ? 0xFFFFFFFFu : (KV ? key_mask_bits(km, c0 + col) : row_mask_bits(rm, c0 + col));
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const uint32_t* xs = sub ? xs1 : xs0;
          const uint32_t* xd = sub ? xd1 : xd0;
          uint32_t pp[8], dd[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            bwd_pair(xs[2 * e], xs[2 * e + 1], xd[2 * e], xd[2 * e + 1], half_alpha, pp[e], dd[e]);
            if (!full) {
              pp[e] = mask_pair(pp[e], bits, 8 * sub + e);
              dd[e] = mask_pair(dd[e], bits, 8 * sub + e);
            }
          }
          if (KV) tmem_st8(lane_base + kColX1 + b * 64 + col / 2 + 8 * sub, pp);
          tmem_st8(lane_base + kColX2 + b * 64 + col / 2 + 8 * sub, dd);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(bar(B_OP_FULL + b));
      }
      if (!ok) break;
      ok = warp_wait(bar(B_ACC_FULL), accn & 1, a.ws);
      if (!ok) break;
      tc_fence_after();
      if (has_acc) {
#pragma unroll
        for (int which = 0; which < (KV ? 2 : 1); ++which) {
          uint32_t v0[16], v1[16];
          const uint32_t cbase = lane_base + (which ? kColAcc2 : kColAcc1) + chunk * 32;
          tmem_ld16(cbase, v0);
          tmem_ld16(cbase + 16, v1);
          tmem_ld_wait2(v0, v1);
          if (r < w.t1) {
            const float sc = which ? sc2 : sc1;
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              o[e] = pack_bf16x2(__uint_as_float(v0[2 * e]) * sc, __uint_as_float(v0[2 * e + 1]) * sc);
              o[8 + e] =
                  pack_bf16x2(__uint_as_float(v1[2 * e]) * sc, __uint_as_float(v1[2 * e + 1]) * sc);
            }
            uint4* dst = reinterpret_cast<uint4*>(which ? o2 : o1);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
      }
      tc_fence_before();
      warp_arrive(bar(B_ACC_EMPTY));
      ++accn;
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

template <int D, bool KV>
cudaError_t launch_pass(const AttnArgs& a, cudaStream_t st) {
  using C = BCfg<D>;
  const int HD = a.H * D;
  const bool sw = C::SW == 128;
  // resident: KV -> K, V ; Q pass -> Q, dO.   streamed: KV -> Q, dO ; Q pass -> K, V.
  const void* r1 = KV ? (const void*)a.k : (const void*)a.q;
  const void* r2 = KV ? (const void*)a.v : (const void*)a.dout;
  const void* s1 = KV ? (const void*)a.q : (const void*)a.k;
  const void* s2 = KV ? (const void*)a.dout : (const void*)a.v;
  const int64_t rr1 = KV ? a.k_rs : a.q_rs, rr2 = KV ? a.v_rs : a.do_rs;
  const int64_t rs1 = KV ? a.q_rs : a.k_rs, rs2 = KV ? a.do_rs : a.v_rs;
  CUtensorMap m1, m2, m3, m4;
  if (!make_tma_2d(&m1, r1, a.T, HD, rr1, C::BOXW, kRes, sw) ||
      !make_tma_2d(&m2, r2, a.T, HD, rr2, C::BOXW, kRes, sw) ||
      !make_tma_2d(&m3, s1, a.T, HD, rs1, C::BOXW, kStr, sw) ||
      !make_tma_2d(&m4, s2, a.T, HD, rs2, C::BOXW, kStr, sw))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel<D, KV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t units = max_items(a.T, a.B) * a.H;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  bwd_tc_kernel<D, KV><<<grid, kThreads, C::SMEM, st>>>(m1, m2, m3, m4, a);
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
