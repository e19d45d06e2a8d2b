// Warp-synchronous SLA forward (mma.sync m16n8k16 bf16, cp.async double
// buffering).  One CTA of 4 warps per (sequence, 64-row query tile, head);
// it walks only the key tiles the SLA mask leaves non-empty for its rows
// (global prefix, local band, candidates' diagonal) and evaluates the mask
// only on tiles that are not entirely visible.
//
//   out_i = (1/N) sum_j M(i,j) SiLU(alpha q_i.k_j) v_j
// ("Bending the Scaling Law Curve in Large-Scale Recommendation Systems",
// section 3, Eq. 3 and section 4.2.1, Eq. 7).  SiLU(x) = h + h tanh(h) with
// h = x/2, one MUFU op per score; 1/N is applied once to the accumulator.
#include "mma_sm80.cuh"
#include "sla_common.cuh"

namespace hstu {
namespace {

constexpr int kBM = 64, kBN = 64, kThreads = 128;

// Rows [tok0, tok0 + 64) of X (row stride rs, head offset hoff) into a
// [64][D + 8] smem tile; rows >= nvalid are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(bf16* s, const bf16* X, int64_t rs, int64_t tok0,
                                          int nvalid, int hoff) {
  constexpr int LD = D + 8, CPR = D / 8;
  for (int c = threadIdx.x; c < 64 * CPR; c += kThreads) {
    int r = c / CPR, cc = c - r * CPR;
    bool ok = r < nvalid;
    const bf16* src = ok ? X + (tok0 + r) * rs + hoff + cc * 8 : X;
    cp_async_16(s + r * LD + cc * 8, src, ok);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) fwd_mma_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int LD = D + 8, TILE = 64 * LD, KD = D / 16;
  bf16* sQ = reinterpret_cast<bf16*>(smem_raw);
  bf16* sK = sQ + TILE;      // 2 stages
  bf16* sV = sK + 2 * TILE;  // 2 stages

  if (load_status(a.ws) != 0) return;
  if ((int)blockIdx.x >= a.ws->n_items) return;
  const int2 it = a.items[blockIdx.x];
  const int h = blockIdx.y, hoff = h * D;
  const SeqGeom g = seq_geom(a, it.x);
  const int r0 = it.y * kBM, r1 = imin(r0 + kBM, g.L);
  const Spans sp = q_tile_key_tiles(r0, r1, g.Lh, a.K1, a.K2e, kBN);
  const int ntiles = sp.count();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;

  load_tile<D>(sQ, a.q, a.q_rs, g.s0 + r0, r1 - r0, hoff);
  cp_async_commit();
  if (ntiles > 0) {
    const int kt = sp.at(0), nv = imin(kBN, g.L - kt * kBN);
    load_tile<D>(sK, a.k, a.k_rs, g.s0 + kt * kBN, nv, hoff);
    load_tile<D>(sV, a.v, a.v_rs, g.s0 + kt * kBN, nv, hoff);
    cp_async_commit();
    cp_async_wait<1>();
  } else {
    cp_async_wait<0>();
  }
  __syncthreads();

  uint32_t qf[KD][4];
#pragma unroll
  for (int kk = 0; kk < KD; ++kk)
    ldsm_x4(qf[kk], sQ + (warp * 16 + (lane & 15)) * LD + kk * 16 + (lane >> 4) * 8);

  const int ra = r0 + warp * 16 + gq, rb = ra + 8;
  const RowMask ma = row_mask(ra, g.L, g.Lh, a.K1, a.K2e);
  const RowMask mb = row_mask(rb, g.L, g.Lh, a.K1, a.K2e);
  const float half_alpha = 0.5f * a.alpha;

  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  for (int n = 0; n < ntiles; ++n) {
    const int stage = n & 1;
    if (n + 1 < ntiles) {
      const int kt = sp.at(n + 1), nv = imin(kBN, g.L - kt * kBN);
      load_tile<D>(sK + (stage ^ 1) * TILE, a.k, a.k_rs, g.s0 + kt * kBN, nv, hoff);
      load_tile<D>(sV + (stage ^ 1) * TILE, a.v, a.v_rs, g.s0 + kt * kBN, nv, hoff);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j0 = sp.at(n) * kBN, j1 = imin(j0 + kBN, g.L);
    const bf16* k_s = sK + stage * TILE;
    const bf16* v_s = sV + stage * TILE;

    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ldsm_x4(b, k_s + (np * 16 + (lane >> 4) * 8 + (lane & 7)) * LD + kk * 16 +
                       ((lane >> 3) & 1) * 8);
        mma_bf16(s[2 * np], qf[kk], b[0], b[1]);
        mma_bf16(s[2 * np + 1], qf[kk], b[2], b[3]);
      }
    }
    const bool full = tile_full(r0, r1, j0, j1, g.Lh, a.K1, a.K2e);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float p = silu_from_half(s[nt][e] * half_alpha);
        if (!full) {
          const int j = j0 + nt * 8 + 2 * tq + (e & 1);
          const bool vis = (e < 2) ? ma(j) : mb(j);
          p = vis ? p : 0.f;
        }
        s[nt][e] = p;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t af[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                        pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                        pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b[4];
        ldsm_x4_t(b, v_s + (kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * LD + dp * 16 +
                         (lane >> 4) * 8);
        mma_bf16(o[2 * dp], af, b[0], b[1]);
        mma_bf16(o[2 * dp + 1], af, b[2], b[3]);
      }
    }
    __syncthreads();
  }

  // Epilogue: scale by 1/N, stage this warp's 16 rows in its own rows of sQ,
  // then 16-byte row-predicated stores (rows past the sequence end are not
  // written: they belong to the next sequence).
  bf16* so = sQ + warp * 16 * LD;
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    *reinterpret_cast<uint32_t*>(so + gq * LD + nt * 8 + 2 * tq) =
        pack_bf16(o[nt][0] * a.inv_n, o[nt][1] * a.inv_n);
    *reinterpret_cast<uint32_t*>(so + (gq + 8) * LD + nt * 8 + 2 * tq) =
        pack_bf16(o[nt][2] * a.inv_n, o[nt][3] * a.inv_n);
  }
  __syncwarp();
  constexpr int CPR = D / 8;
  for (int c = lane; c < 16 * CPR; c += 32) {
    const int r = c / CPR, cc = c - r * CPR, row = r0 + warp * 16 + r;
    if (row < r1)
      *reinterpret_cast<uint4*>(a.out + (int64_t)(g.s0 + row) * a.o_rs + hoff + cc * 8) =
          *reinterpret_cast<const uint4*>(so + r * LD + cc * 8);
  }
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  const int smem = 5 * 64 * (D + 8) * 2;
  cudaError_t e = cudaFuncSetAttribute(fwd_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)max_items(a.T, a.B), a.H);
  fwd_mma_kernel<D><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_mma(const AttnArgs& a, int d, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (d == 32) return launch_d<32>(a, st);
  if (d == 64) return launch_d<64>(a, st);
  return launch_d<128>(a, st);
}

}  // namespace hstu
