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
//   warp 0      TMA producer: Q tiles into two alternating buffers, K and V
//               tiles (128 keys) into a 2-stage ring; 128B-swizzled boxes
//               of 64 head-dim columns.
//   warp 1      allocates TMEM; one lane issues UMMA: S = Q K^T into one of
//               two TMEM S buffers (M=128, N=128, K=d), then O += P V with P
//               read from TMEM (M=128, N=d, K=128) into the O accumulator.
//   warps 2..17 pointwise: TMEM -> registers, P = SiLU(alpha S) (masked only
//               on partial tiles) as bf16 back into TMEM; after the last key
//               tile, the epilogue: O * (1/N) -> bf16 -> global, rows past the
//               sequence end not written.  Four warps share each 32-lane TMEM
//               quarter, one per 32-column chunk, so TMEM load/store latency
//               is hidden across warps.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+d) P0 [384,448) P1 [448,512).
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

constexpr int kBM = 128, kBN = 128, kPwWarps = 16;
constexpr int kThreads = 64 + 32 * kPwWarps;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384, kTmemCols = 512;

// K/V ring depth: as deep as 227 KB of shared memory allows.
template <int D>
constexpr int fwd_stages() { return D == 128 ? 2 : 4; }

template <int D>
struct Cfg {
  static constexpr int kStages = fwd_stages<D>();
  static constexpr int SW = D >= 64 ? 128 : 64;   // swizzle span (bytes) = one box row
  static constexpr int BOXW = SW / 2;             // bf16 elements per box row
  static constexpr int NB = D / BOXW;             // boxes per tile
  static constexpr int BLK = 128 * SW;            // bytes per box (128 rows)
  static constexpr int TILE = 128 * D * 2;        // bytes per Q / K / V tile
  static constexpr int OFF_Q = 0;                      // two Q buffers
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = TILE * (2 + kStages);
  static constexpr int OFF_BAR = TILE * (2 + 2 * kStages);
  static_assert(OFF_BAR + 256 + 1024 <= 232448, "shared memory budget");
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers + 1 KB alignment slack
  static constexpr uint32_t SWZ = SW == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr uint32_t SBO = 8 * SW;             // stride of 8-row groups
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kBN, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, D, false, true);
  static constexpr int COLS_PER_PW = kBN / (kPwWarps / 4);  // S columns per pointwise warp (32)
};

// Barrier slots (8 bytes each) after the tiles.
constexpr int kMaxStages = 4;
enum {
  BAR_Q_FULL = 0, BAR_Q_EMPTY = 2, BAR_K_FULL = 4, BAR_K_EMPTY = BAR_K_FULL + kMaxStages,
  BAR_V_FULL = BAR_K_EMPTY + kMaxStages, BAR_V_EMPTY = BAR_V_FULL + kMaxStages,
  BAR_S_FULL = BAR_V_EMPTY + kMaxStages, BAR_P_FULL = BAR_S_FULL + 2, BAR_O_FULL = BAR_P_FULL + 2,
  BAR_O_EMPTY, BAR_DRAIN, BAR_COUNT
};

struct Unit {
  int h, s0, L, Lh, r0, r1;
  Spans sp;
  int ntiles;
};

__device__ __forceinline__ Unit unit_at(const AttnArgs& a, int n_items, int u) {
  Unit w;
  w.h = u / n_items;
  const int2 it = a.items[u - w.h * n_items];
  const SeqGeom g = seq_geom(a, it.x);
  w.s0 = g.s0; w.L = g.L; w.Lh = g.Lh;
  w.r0 = it.y * kBM;
  w.r1 = imin(w.r0 + kBM, g.L);
  w.sp = q_tile_key_tiles(w.r0, w.r1, g.Lh, a.K1, a.K2e, kBN);
  w.ntiles = w.sp.count();
  return w;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const AttnArgs a) {
  using C = Cfg<D>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V;
  const uint32_t bar0 = base + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + 8 * BAR_COUNT);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (load_status(a.ws) != 0) return;  // device-side input check failed
  const int n_items = a.ws->n_items;
  const int total = n_items * a.H;

  if (threadIdx.x == 0) {
    for (int qb = 0; qb < 2; ++qb) {
      mbar_init(bar(BAR_Q_FULL + qb), 1);
      mbar_init(bar(BAR_Q_EMPTY + qb), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_K_FULL + s), 1);
      mbar_init(bar(BAR_K_EMPTY + s), 1);
      mbar_init(bar(BAR_V_FULL + s), 1);
      mbar_init(bar(BAR_V_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BAR_S_FULL + b), 1);
      mbar_init(bar(BAR_P_FULL + b), kPwWarps / 2);  // one arrive per warp of group b
    }
    mbar_init(bar(BAR_O_FULL), 1);
    mbar_init(bar(BAR_O_EMPTY), kPwWarps);
    mbar_init(bar(BAR_DRAIN), 1);
    fence_barrier_init();
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
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
    // ------------------------------------------------------------ producer
    // The whole warp walks the schedule (so every value stays warp-uniform);
    // lane 0 arms the barriers and issues the copies.
    uint32_t qn = 0, kv = 0, kn = 0, vn = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit w = unit_at(a, n_items, u);
      if (w.ntiles == 0) continue;
      // Q tiles alternate between two buffers, so the next unit's Q is loaded
      // while the current unit still runs.
      const uint32_t qb = qn & 1;
      ok = warp_wait(bar(BAR_Q_EMPTY + qb), ((qn >> 1) & 1) ^ 1, a.ws);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(bar(BAR_Q_FULL + qb), C::TILE);
        for (int b = 0; b < C::NB; ++b)
          tma_load_2d(sQ + qb * C::TILE + b * C::BLK, &tmq, bar(BAR_Q_FULL + qb),
                      w.h * D + b * C::BOXW, w.s0 + w.r0);
      }
      ++qn;
      for (int n = 0; n < w.ntiles && ok; ++n) {
        const int y = w.s0 + w.sp.at(n) * kBN;
        const int s = kv % kStages;
        const uint32_t ph = (kv / kStages) & 1;
        ok = warp_wait(bar(BAR_K_EMPTY + s), ph ^ 1, a.ws);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(bar(BAR_K_FULL + s), C::TILE);
          for (int b = 0; b < C::NB; ++b)
            tma_load_2d(sK + s * C::TILE + b * C::BLK, &tmk, bar(BAR_K_FULL + s),
                        w.h * D + b * C::BOXW, y);
        }
        ++kn;
        ok = warp_wait(bar(BAR_V_EMPTY + s), ph ^ 1, a.ws);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(bar(BAR_V_FULL + s), C::TILE);
          for (int b = 0; b < C::NB; ++b)
            tma_load_2d(sV + s * C::TILE + b * C::BLK, &tmv, bar(BAR_V_FULL + s),
                        w.h * D + b * C::BOXW, y);
        }
        ++vn;
        ++kv;
      }
    }
    // If any role gave up, every load issued must still land before the CTA
    // exits (each barrier has at most its last armed phase outstanding).
    if (lane == 0 && load_status(a.ws) != 0) {
      for (uint32_t qb = 0; qb < 2; ++qb) {
        const uint32_t armed = qn / 2 + (qb < (qn & 1) ? 1u : 0u);
        if (armed > 0) drain_wait(bar(BAR_Q_FULL + qb), (armed - 1) & 1);
      }
      for (int s = 0; s < kStages; ++s) {
        const uint32_t k_armed = kn / kStages + (s < (int)(kn % kStages) ? 1u : 0u);
        const uint32_t v_armed = vn / kStages + (s < (int)(vn % kStages) ? 1u : 0u);
        if (k_armed > 0) drain_wait(bar(BAR_K_FULL + s), (k_armed - 1) & 1);
        if (v_armed > 0) drain_wait(bar(BAR_V_FULL + s), (v_armed - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    // The whole warp runs the loop with warp-uniform descriptors; lane 0
    // issues every UMMA and commit (a commit tracks the issuing thread's MMAs).
    uint32_t qn = 0, kv = 0, tc = 0, on = 0;
    bool ok = true;
    // Descriptor bases; a k-step / stage only adds to the start-address field
    // (smem addresses stay below 2^18, so the 14-bit field never carries).
    const uint64_t dQ = smem_desc(sQ, 16, C::SBO, C::SWZ);
    const uint64_t dK = smem_desc(sK, 16, C::SBO, C::SWZ);
    const uint64_t dV = smem_desc(sV, C::BLK, C::SBO, C::SWZ);
    auto kstep = [](int ks) -> uint32_t {  // byte offset of k-step ks in a K-major tile
      return (uint32_t)(((ks * 32) / C::SW) * C::BLK + (ks * 32) % C::SW);
    };
    // O += P(tile m) V(tile m); kvm / tcm: that tile's ring / S-buffer counters.
    auto pv = [&](uint32_t kvm, uint32_t tcm, bool first) -> bool {
      const uint32_t b = tcm & 1;
      if (!warp_wait(bar(BAR_P_FULL + b), (tcm >> 1) & 1, a.ws)) return false;
      const int s = kvm % kStages;
      if (!warp_wait(bar(BAR_V_FULL + s), (kvm / kStages) & 1, a.ws)) return false;
      if (first && !warp_wait(bar(BAR_O_EMPTY), (on & 1) ^ 1, a.ws)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint64_t dv = dV + ((uint32_t)(s * C::TILE) >> 4);
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks)
          mma_ts(tmem + kColO, tmem + kColP0 + b * 64 + ks * 8,
                 dv + ((uint32_t)(ks * 16 * C::SW) >> 4), C::IDESC_O,
                 (!first || ks > 0) ? 1u : 0u);
        tc_commit(bar(BAR_V_EMPTY + s));
      }
      __syncwarp();
      return true;
    };
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit w = unit_at(a, n_items, u);
      if (w.ntiles == 0) continue;
      const uint32_t qb = qn & 1;
      ok = warp_wait(bar(BAR_Q_FULL + qb), (qn >> 1) & 1, a.ws);
      if (!ok) break;
      tc_fence_after();
      const uint32_t kv0 = kv, tc0 = tc;
      for (int n = 0; n < w.ntiles; ++n) {
        const int s = kv % kStages;
        ok = warp_wait(bar(BAR_K_FULL + s), (kv / kStages) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const uint32_t b = tc & 1;
        if (lane == 0) {
          const uint64_t dk = dK + ((uint32_t)(s * C::TILE) >> 4);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            mma_ss(tmem + kColS0 + b * 128, dQ + ((qb * C::TILE + kstep(ks)) >> 4),
                   dk + (kstep(ks) >> 4),
                   C::IDESC_S, ks > 0 ? 1u : 0u);
          tc_commit(bar(BAR_S_FULL + b));
          tc_commit(bar(BAR_K_EMPTY + s));
          if (n + 1 == w.ntiles) tc_commit(bar(BAR_Q_EMPTY + qb));  // last use of this Q tile
        }
        __syncwarp();
        if (n > 0) {
          ok = pv(kv - 1, tc - 1, n == 1);
          if (!ok) break;
        }
        ++kv;
        ++tc;
      }
      if (!ok) break;
      ok = pv(kv0 + w.ntiles - 1, tc0 + w.ntiles - 1, w.ntiles == 1);
      if (!ok) break;
      if (lane == 0) tc_commit(bar(BAR_O_FULL));
      __syncwarp();
      ++qn;
      ++on;
    }
    // Every MMA issued must finish before TMEM is released.
    if (lane == 0) {
      tc_commit(bar(BAR_DRAIN));
      drain_wait(bar(BAR_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ----------------------------------------------- pointwise and epilogue
    // Two groups of eight warps take alternate S tiles (group g owns S buffer
    // g), so one group's TMEM load / store latency overlaps the other's
    // arithmetic.  Within a group, the two warps on a 32-lane TMEM quarter
    // split the tile's 128 columns in halves.  The epilogue uses all sixteen:
    // warp `chunk` of a quarter writes O columns [32 chunk, +32).
    const int pw = warp - 2;               // 0..15
    const int grp = pw >> 3;               // S buffer / tile parity of this warp
    const int quarter = warp & 3;          // TMEM lanes [32*quarter, +32)
    const int chunk = pw >> 2;             // 0..3
    const int half = chunk & 1;            // column half within the group
    const int row = quarter * 32 + lane;   // row of the 128-row tile
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float half_alpha = 0.5f * a.alpha;
    const bool has_o = chunk < D / 32;     // this warp writes an O chunk
    uint32_t tc = 0, on = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit w = unit_at(a, n_items, u);
      const int i = w.r0 + row;  // row within the sequence
      bf16* orow = a.out + (int64_t)(w.s0 + i) * a.o_rs + w.h * D + chunk * 32;
      if (w.ntiles == 0) {  // no visible key anywhere in the tile
        if (has_o && i < w.r1) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 4; ++v) reinterpret_cast<uint4*>(orow)[v] = z;
        }
        continue;
      }
      const RowMask m = row_mask(i, w.L, w.Lh, a.K1, a.K2e);
      for (int n = 0; n < w.ntiles; ++n, ++tc) {
        const uint32_t b = tc & 1;
        if ((int)b != grp) continue;  // the other group's tile
        ok = warp_wait(bar(BAR_S_FULL + b), (tc >> 1) & 1, a.ws);
        if (!ok) break;
        tc_fence_after();
        const int j0 = w.sp.at(n) * kBN;
        const bool full = tile_full(w.r0, w.r0 + kBM, j0, j0 + kBN, w.Lh, a.K1, a.K2e);
        // P = SiLU(alpha S) = h + h tanh(h) with h = alpha S / 2.  Tiles that
        // are entirely visible skip the mask; the others clear invisible
        // entries with one bit test each against this row's 32-key bitmask.
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const int col = half * 64 + sub * 32;
          uint32_t c0[16], c1[16];
          tmem_ld16(lane_base + kColS0 + b * 128 + col, c0);
          tmem_ld16(lane_base + kColS0 + b * 128 + col + 16, c1);
          tmem_ld_wait2(c0, c1);
          uint32_t p[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = silu_pair(c0[2 * e], c0[2 * e + 1], half_alpha);
            p[8 + e] = silu_pair(c1[2 * e], c1[2 * e + 1], half_alpha);
          }
          if (!full) {
            const uint32_t bits = row_mask_bits(m, j0 + col);
#pragma unroll
            for (int e = 0; e < 16; ++e) p[e] = mask_pair(p[e], bits, e);
          }
          tmem_st16(lane_base + kColP0 + b * 64 + col / 2, p);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(bar(BAR_P_FULL + b));
      }
      if (!ok) break;
      // epilogue
      ok = warp_wait(bar(BAR_O_FULL), on & 1, a.ws);
      if (!ok) break;
      tc_fence_after();
      if (has_o) {
        uint32_t r0[16], r1[16];
        tmem_ld16(lane_base + kColO + chunk * 32, r0);
        tmem_ld16(lane_base + kColO + chunk * 32 + 16, r1);
        tmem_ld_wait2(r0, r1);
        if (i < w.r1) {
          uint32_t o[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            o[e] = pack_bf16x2(__uint_as_float(r0[2 * e]) * a.inv_n,
                               __uint_as_float(r0[2 * e + 1]) * a.inv_n);
            o[8 + e] = pack_bf16x2(__uint_as_float(r1[2 * e]) * a.inv_n,
                                   __uint_as_float(r1[2 * e + 1]) * a.inv_n);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
      }
      tc_fence_before();
      warp_arrive(bar(BAR_O_EMPTY));
      ++on;
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

template <int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D>;
  CUtensorMap mq, mk, mv;
  const int HD = a.H * D;
  if (!make_tma_2d(&mq, a.q, a.T, HD, a.q_rs, C::BOXW, kBM, C::SW == 128) ||
      !make_tma_2d(&mk, a.k, a.T, HD, a.k_rs, C::BOXW, kBN, C::SW == 128) ||
      !make_tma_2d(&mv, a.v, a.T, HD, a.v_rs, C::BOXW, kBN, C::SW == 128))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t units = max_items(a.T, a.B) * a.H;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  fwd_tc_kernel<D><<<grid, kThreads, C::SMEM, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const AttnArgs& a, int d, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (d == 32) return launch_d<32>(a, st);
  if (d == 64) return launch_d<64>(a, st);
  return launch_d<128>(a, st);
}

}  // namespace hstu
