// Dense bf16 GEMM on the 5th-generation tensor cores (tcgen05 / TMEM / TMA)
// for the STU layer's projections: f1 of Eq. 2 (the UVQK projection), f2 of
// Eq. 4 (the output projection) and their backward contractions, of "Bending
// the Scaling Law Curve in Large-Scale Recommendation Systems", section 3
// (and the addmm steps of its Listing 1, section 4.2.2).
//
//   D[m, n] = sum_k A[m, k] B[n, k]      (bf16 operands, fp32 accumulation)
//
// Each operand is read either K-major (row m of A / row n of B holds its K
// values contiguously: activations x [T, d_in] as A, or a weight W [N, K]
// as B) or MN-major (row k holds the M / N values contiguously: a weight
// W [K, N] as B, or activations read transposed for a weight gradient).
// Epilogues, fused on the TMEM read-out:
//   kEpiStore      out  = bf16(D)
//   kEpiBiasSilu   out2 = bf16(D + bias),  out = bf16(SiLU(D + bias))
//   kEpiBiasResid  out  = bf16(D + bias + resid)
//   kEpiRedF32     outf += D              (fp32 reductions: split-K partial
//                                          sums of a weight gradient)
//
// Tiles of 128 x 256 (one 128x256x16 UMMA per 16 of K, the full-rate shape),
// K in blocks of 64 (one 128-byte swizzle atom), 4-stage TMA ring, two TMEM
// accumulators so a tile's epilogue overlaps the next tile's main loop.
// Persistent CTAs walk tiles (split, m block, n block) with n fastest, so
// consecutive tiles share their A rows in L2.
// Roles: warp 0 TMA producer, warp 1 TMEM allocation + one MMA-issuing lane,
// warps 2..9 epilogue (warp w reads TMEM lanes 32 (w % 4) .. +32 and half of
// the tile's columns).
#include <cudaTypedefs.h>
#include <string.h>

#include "sm100.cuh"
#include "stu_common.cuh"

namespace hstu {

bool make_tma_2d(CUtensorMap* m, const void* ptr, int64_t T, int HD, int64_t rs, int box_w,
                 int box_h, bool sw128);
bool make_tma_2d_u8(CUtensorMap* m, const void* ptr, int64_t T, int W, int64_t rs, int box_w,
                    int box_h);
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter, each half of the tile's columns
constexpr int kThreads = 32 * (2 + 8);
constexpr int A_TILE = kBM * kBK * 2;  // 16 KB
constexpr int B_TILE = kBN * kBK * 2;  // 32 KB
constexpr int MN_BOX = 64 * kBK * 2;   // one 64 (M or N) x 64 (K) box of an MN-major tile
// bf16 outputs leave through shared memory and TMA: each epilogue warp
// stages 32-row x 32-column boxes (64-byte rows, 64B-swizzled) of each
// output; with two buffers the store of one chunk reads shared memory while
// the next chunk is computed.
constexpr int STG_BOX = 32 * 64;
constexpr int STG_BUF = 2 * STG_BOX;  // out, out2
// Shared-memory plan: the fp32 reductions take 4 ring stages and no staging;
// bf16 operands with bf16 outputs 4 stages (the main loop is the longer side)
// and one staging buffer; 8-bit operands (half the ring stages per tile) 3
// stages and two staging buffers (the epilogue is the longer side).
template <int EPI, bool F8>
struct GLayout {
  static constexpr int kStages = EPI == kEpiRedF32 ? 4 : (F8 ? 3 : 4);
  static constexpr int kStgBufs = F8 ? 2 : 1;
  static constexpr int STG_WARP = kStgBufs * STG_BUF;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kStages * A_TILE;
  static constexpr int OFF_STG = OFF_B + kStages * B_TILE;
  static constexpr int OFF_BAR = OFF_STG + (EPI == kEpiRedF32 ? 0 : kEpiWarps * STG_WARP);
  static constexpr int OFF_SLOT = OFF_BAR + 128;
  static constexpr int SMEM = OFF_SLOT + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};
constexpr int kMaxStages = 4;
constexpr uint32_t kTmemCols = 2 * kBN;

enum { G_FULL = 0, G_EMPTY = kMaxStages, G_ACC_FULL = 2 * kMaxStages, G_ACC_EMPTY = G_ACC_FULL + 2,
       G_COUNT = G_ACC_EMPTY + 2 };
static_assert(8 * G_COUNT <= 128, "barrier area");

struct TileInfo {
  int m0, n0, k0, nkb;  // first row / column / k, number of 64-wide k blocks
};

// bk: elements per k block (64 bf16 or 128 8-bit values: 128 bytes either way)
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& g, int t, int tiles_m, int tiles_n,
                                              int bk) {
  TileInfo ti;
  const int nb = t % tiles_n;
  const int rest = t / tiles_n;
  const int mb = rest % tiles_m;
  const int split = rest / tiles_m;
  ti.m0 = mb * kBM;
  ti.n0 = nb * kBN;
  ti.k0 = split * g.k_split;
  const int k1 = min(g.K, ti.k0 + g.k_split);
  ti.nkb = k1 > ti.k0 ? (k1 - ti.k0 + bk - 1) / bk : 0;
  return ti;
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile(
      "{\n .reg .u64 g;\n cvta.to.global.u64 g, %0;\n"
      " red.relaxed.gpu.global.add.v4.f32 [g], {%1, %2, %3, %4};\n}\n" ::"l"(p),
      "f"(a), "f"(b), "f"(c), "f"(d)
      : "memory");
}

// SiLU(v) = h + h tanh(h) with h = v / 2 (one MUFU op)
__device__ __forceinline__ float silu_f(float v) {
  float t;
  const float h = 0.5f * v;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

template <bool A_MN, bool B_MN, int EPI, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                   const __grid_constant__ CUtensorMap tmo, const __grid_constant__ CUtensorMap tmo2,
                   const GemmArgs g) {
  static_assert(!F8 || (!A_MN && !B_MN), "8-bit operands are read K-major");
  constexpr int kBKe = F8 ? 2 * kBK : kBK;  // elements per 128-byte k block
  using Lay = GLayout<EPI, F8>;
  constexpr int kStgBufs = Lay::kStgBufs, STG_WARP = Lay::STG_WARP;
  constexpr int kStages = Lay::kStages, OFF_A = Lay::OFF_A, OFF_B = Lay::OFF_B;
  constexpr int OFF_STG = Lay::OFF_STG, OFF_BAR = Lay::OFF_BAR, OFF_SLOT = Lay::OFF_SLOT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sA = base + OFF_A, sB = base + OFF_B;
  const uint32_t bar0 = base + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + OFF_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (g.M + kBM - 1) / kBM, tiles_n = g.N / kBN;
  const int ntiles = tiles_m * tiles_n * g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(G_FULL + s), 1);
      mbar_init(bar(G_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(G_ACC_FULL + b), 1);
      mbar_init(bar(G_ACC_EMPTY + b), kEpiWarps);
    }
    fence_barrier_init();
    prefetch_tmap(&tma);
    prefetch_tmap(&tmb);
    if (EPI != kEpiRedF32) prefetch_tmap(&tmo);
    if (EPI == kEpiBiasSilu) prefetch_tmap(&tmo2);
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
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(g, t, tiles_m, tiles_n, kBKe);
        for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
          const int s = it % kStages;
          ok = mbar_wait(bar(G_EMPTY + s), ((it / kStages) & 1) ^ 1, g.ws);
          if (!ok) break;
          const uint32_t fb = bar(G_FULL + s);
          mbar_expect_tx(fb, A_TILE + B_TILE);
          const int k = ti.k0 + kb * kBKe;
          const uint32_t a = sA + s * A_TILE, b = sB + s * B_TILE;
          if (A_MN) {  // [K][M]: two 64-wide column boxes
            tma_load_2d(a, &tma, fb, ti.m0, k);
            tma_load_2d(a + MN_BOX, &tma, fb, ti.m0 + 64, k);
          } else {     // [M][K]: 128 rows x 64 k
            tma_load_2d(a, &tma, fb, k, ti.m0);
          }
          if (B_MN) {  // [K][N]: four 64-wide column boxes
            for (int j = 0; j < kBN / 64; ++j) tma_load_2d(b + j * MN_BOX, &tmb, fb, ti.n0 + 64 * j, k);
          } else {     // [N][K]: 256 rows x 64 k
            tma_load_2d(b, &tmb, fb, k, ti.n0);
          }
        }
      }
      if (load_status(g.ws) != 0) {  // drain copies in flight before exiting
        for (int s = 0; s < kStages; ++s) {
          const uint32_t armed = it / kStages + (s < (int)(it % kStages) ? 1u : 0u);
          if (armed > 0) drain_wait(bar(G_FULL + s), (armed - 1) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp computes every operand (warp-uniform); one elected lane
    // issues each k block's UMMAs with immediate offsets and its commit.
    {
      constexpr uint32_t IDESC = F8 ? idesc_e4m3(kBM, kBN) : idesc_bf16(kBM, kBN, A_MN, B_MN);
      // K-major: a 16-wide k step moves 32 bytes inside the 128-byte row;
      // MN-major: it moves 16 rows of 128 bytes.  Units of 16 bytes.
      constexpr uint32_t kStepA = A_MN ? 128u : 2u, kStepB = B_MN ? 128u : 2u;
      const uint64_t dA = A_MN ? smem_desc(sA, MN_BOX, 1024, kSwizzle128B)
                               : smem_desc(sA, 16, 1024, kSwizzle128B);
      const uint64_t dB = B_MN ? smem_desc(sB, MN_BOX, 1024, kSwizzle128B)
                               : smem_desc(sB, 16, 1024, kSwizzle128B);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(g, t, tiles_m, tiles_n, kBKe);
        if (ti.nkb == 0) continue;
        const uint32_t buf = tc & 1;
        ok = warp_wait(bar(G_ACC_EMPTY + buf), ((tc >> 1) & 1) ^ 1, g.ws);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc_t = tmem + buf * kBN;
        for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
          const int s = it % kStages;
          ok = warp_wait(bar(G_FULL + s), (it / kStages) & 1, g.ws);
          if (!ok) break;
          tc_fence_after();
          const uint64_t a = dA + ((uint32_t)(s * A_TILE) >> 4);
          const uint64_t b = dB + ((uint32_t)(s * B_TILE) >> 4);
          const uint32_t acc0 = kb > 0 ? 1u : 0u;
          const uint32_t bar_e = bar(G_EMPTY + s);
          if (elect_one()) {
            // four 32-byte k steps per 128-byte block (16 bf16 or 32 8-bit values each)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              if constexpr (F8)
                mma_ss_f8(acc_t, a + ks * kStepA, b + ks * kStepB, IDESC, ks > 0 ? 1u : acc0);
              else
                mma_ss(acc_t, a + ks * kStepA, b + ks * kStepB, IDESC, ks > 0 ? 1u : acc0);
            }
            tc_commit(bar_e);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc_commit(bar(G_ACC_FULL + buf));
        __syncwarp();
        ++tc;
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int col0 = ((warp - 2) >> 2) * (kBN / 2);  // this warp's half of the columns
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t stg = base + OFF_STG + (uint32_t)(warp - 2) * STG_WARP;
    const uint32_t stg_row = (uint32_t)lane * 64;          // 64-byte staged rows
    const uint32_t swz = (uint32_t)((lane >> 1) & 3);     // 64B swizzle of row `lane`
    uint32_t ec = 0;  // chunks this warp has staged
    uint32_t tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const TileInfo ti = tile_info(g, t, tiles_m, tiles_n, kBKe);
      if (ti.nkb == 0) continue;
      const uint32_t buf = tc & 1;
      const int m = ti.m0 + quarter * 32 + lane;
      const bool live = m < g.M;
      // residual epilogue: the first chunk's residual row segment is read
      // before the accumulator wait, each later one a chunk ahead
      uint4 res_a[4], res_b[4];
      auto load_res = [&](int i, uint4(&r)[4]) {
        if (EPI == kEpiBiasResid && live) {
          const uint4* rp = reinterpret_cast<const uint4*>(g.resid + (int64_t)m * g.ldr + ti.n0 +
                                                           col0 + 32 * i);
#pragma unroll
          for (int q = 0; q < 4; ++q) r[q] = rp[q];
        }
      };
      load_res(0, res_a);
      ok = warp_wait(bar(G_ACC_FULL + buf), (tc >> 1) & 1, g.ws);
      if (!ok) break;
      tc_fence_after();
      if constexpr (EPI == kEpiRedF32) {
#pragma unroll 1
        for (int c = col0; c < col0 + kBN / 2; c += 32) {
          uint32_t v[32];
          tmem_ld32(lane_base + buf * kBN + c, v);
          tmem_ld_wait(v);
          if (c + 32 == col0 + kBN / 2) {  // this warp's share read out
            tc_fence_before();
            warp_arrive(bar(G_ACC_EMPTY + buf));
          }
          if (live) {
            float* dst = g.outf + (int64_t)m * g.ldf + ti.n0 + c;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4(dst + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                         __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
      } else {
        // 32-column chunks; the next chunk's TMEM load is in flight while this
        // one is converted and staged
        uint32_t va[32], vb[32];
        tmem_ld32(lane_base + buf * kBN + col0, va);
        tmem_ld_wait(va);
        auto chunk = [&](int i, uint32_t(&v)[32], uint32_t(&vn)[32], uint4(&res)[4],
                         uint4(&res_n)[4]) {
          constexpr int kChunks = kBN / 2 / 32;
          if (i + 1 < kChunks) {
            tmem_ld32(lane_base + buf * kBN + col0 + 32 * (i + 1), vn);
            load_res(i + 1, res_n);
          } else {  // this warp's share of the accumulator is in registers
            tc_fence_before();
            warp_arrive(bar(G_ACC_EMPTY + buf));
          }
          const int n = ti.n0 + col0 + 32 * i;
          float f[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
          if constexpr (F8) {  // row scale of A times column scale of B
            const float sm = live ? g.sa[m] : 0.f;
            const float4* sp = reinterpret_cast<const float4*>(g.sb + n);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 s4 = __ldg(sp + e);
              f[4 * e] *= sm * s4.x;
              f[4 * e + 1] *= sm * s4.y;
              f[4 * e + 2] *= sm * s4.z;
              f[4 * e + 3] *= sm * s4.w;
            }
          }
          if (EPI == kEpiBiasSilu || EPI == kEpiBiasResid) {
            const float4* bp = reinterpret_cast<const float4*>(g.bias + n);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 b4 = __ldg(bp + e);
              f[4 * e] += b4.x;
              f[4 * e + 1] += b4.y;
              f[4 * e + 2] += b4.z;
              f[4 * e + 3] += b4.w;
            }
          }
          if (EPI == kEpiBiasResid && live) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 r4 = res[q];
              const uint32_t w[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                f[8 * q + 2 * h] += __uint_as_float(w[h] << 16);
                f[8 * q + 2 * h + 1] += __uint_as_float(w[h] & 0xFFFF0000u);
              }
            }
          }
          uint32_t o[16], o2[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = pack_bf16x2(f[2 * e], f[2 * e + 1]);
          if (EPI == kEpiBiasSilu) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              o2[e] = o[e];  // pre-activation
              o[e] = pack_bf16x2(silu_f(f[2 * e]), silu_f(f[2 * e + 1]));
            }
          }
          // the buffer's previous store (two chunks back) must have read it
          const uint32_t sb = stg + (uint32_t)(ec % kStgBufs) * STG_BUF;
          if (ec >= (uint32_t)kStgBufs) {
            if (lane == 0) {
              if (kStgBufs == 2) bulk_wait_read_1();
              else bulk_wait_read_all();
            }
            __syncwarp();
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t off = stg_row + ((((uint32_t)q) ^ swz) << 4);
            st_shared_v4(sb + off, o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            if (EPI == kEpiBiasSilu)
              st_shared_v4(sb + STG_BOX + off, o2[4 * q], o2[4 * q + 1], o2[4 * q + 2],
                           o2[4 * q + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {  // rows past M are clipped by the store
            const int y = ti.m0 + quarter * 32;
            tma_store_2d(&tmo, sb, n, y);
            if (EPI == kEpiBiasSilu) tma_store_2d(&tmo2, sb + STG_BOX, n, y);
            bulk_commit_group();
          }
          ++ec;
          if (i + 1 < kChunks) tmem_ld_wait(vn);
        };
        chunk(0, va, vb, res_a, res_b);
        chunk(1, vb, va, res_b, res_a);
        chunk(2, va, vb, res_a, res_b);
        chunk(3, vb, va, res_b, res_a);
      }
      ++tc;
    }
    if (lane == 0) bulk_wait_all();  // every store complete before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool A_MN, bool B_MN, int EPI, bool F8 = false>
cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo,
                     const CUtensorMap& mo2, const GemmArgs& g, int ntiles, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN, EPI, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GLayout<EPI, F8>::SMEM);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  gemm_tc_kernel<A_MN, B_MN, EPI, F8>
      <<<ntiles < sms ? ntiles : sms, kThreads, GLayout<EPI, F8>::SMEM, st>>>(ma, mb, mo, mo2, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmOperand& A, const GemmOperand& B, GemmArgs g, int epi,
                        cudaStream_t st) {
  if (g.M == 0 || g.N == 0) return cudaSuccess;
  // split-K only for the reducing epilogue; each split covers whole k blocks
  if (epi != kEpiRedF32) g.splits = 1;
  if (g.splits < 1) g.splits = 1;
  const bool f8 = A.fp8 || B.fp8;
  if (f8 && (!A.fp8 || !B.fp8 || A.mn_major || B.mn_major || epi == kEpiRedF32 ||
             g.sa == nullptr || g.sb == nullptr))
    return cudaErrorNotSupported;
  const int bke = f8 ? 2 * kBK : kBK;
  const int kb_total = (g.K + bke - 1) / bke;
  const int kb_per = (kb_total + g.splits - 1) / g.splits;
  g.k_split = kb_per * bke;
  g.splits = kb_per > 0 ? (kb_total + kb_per - 1) / kb_per : 1;
  CUtensorMap ma, mb;
  // K-major operand: rows = M (or N), columns = K.  MN-major: rows = K.
  if (f8) {
    if (!make_tma_2d_u8(&ma, A.ptr, g.M, g.K, A.ld, 128, kBM) ||
        !make_tma_2d_u8(&mb, B.ptr, g.N, g.K, B.ld, 128, kBN))
      return cudaErrorInvalidValue;
  } else if (!(A.mn_major ? make_tma_2d(&ma, A.ptr, g.K, g.M, A.ld, 64, kBK, true)
                          : make_tma_2d(&ma, A.ptr, g.M, g.K, A.ld, kBK, kBM, true)) ||
             !(B.mn_major ? make_tma_2d(&mb, B.ptr, g.K, g.N, B.ld, 64, kBK, true)
                          : make_tma_2d(&mb, B.ptr, g.N, g.K, B.ld, kBK, kBN, true))) {
    return cudaErrorInvalidValue;
  }
  // bf16 outputs: 64-column x 32-row boxes, 128B-swizzled like the staging
  CUtensorMap mo, mo2;
  memset(&mo, 0, sizeof(mo));
  memset(&mo2, 0, sizeof(mo2));
  if (epi != kEpiRedF32 && !make_tma_2d(&mo, g.out, g.M, g.N, g.ldo, 32, 32, false))
    return cudaErrorInvalidValue;
  if (epi == kEpiBiasSilu && !make_tma_2d(&mo2, g.out2, g.M, g.N, g.ldo2, 32, 32, false))
    return cudaErrorInvalidValue;
  const int ntiles = ((g.M + kBM - 1) / kBM) * (g.N / kBN) * g.splits;
  if (f8) {  // the forward projections in E4M3
    if (epi == kEpiBiasSilu) return launch_t<false, false, kEpiBiasSilu, true>(ma, mb, mo, mo2, g, ntiles, st);
    if (epi == kEpiBiasResid) return launch_t<false, false, kEpiBiasResid, true>(ma, mb, mo, mo2, g, ntiles, st);
    if (epi == kEpiStore) return launch_t<false, false, kEpiStore, true>(ma, mb, mo, mo2, g, ntiles, st);
    return cudaErrorNotSupported;
  }
#define HSTU_GEMM_CASE(AM, BM_, E) \
  if (A.mn_major == AM && B.mn_major == BM_ && epi == E) \
    return launch_t<AM, BM_, E>(ma, mb, mo, mo2, g, ntiles, st);
  HSTU_GEMM_CASE(false, true, kEpiBiasSilu)    // x^ W1 + b1 -> SiLU      (W1 stored [K][N])
  HSTU_GEMM_CASE(false, true, kEpiBiasResid)   // y W2 + b2 + x           (W2 stored [K][N])
  HSTU_GEMM_CASE(false, false, kEpiStore)      // dOut W2^T, dPre W1^T     (W read [N][K])
  HSTU_GEMM_CASE(false, true, kEpiStore)
  HSTU_GEMM_CASE(true, true, kEpiRedF32)       // x^T dPre, y^T dOut       (both [K][*])
  HSTU_GEMM_CASE(false, false, kEpiRedF32)
#undef HSTU_GEMM_CASE
  return cudaErrorNotSupported;
}

}  // namespace hstu
