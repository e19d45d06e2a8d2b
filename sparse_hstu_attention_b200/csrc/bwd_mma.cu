// Warp-synchronous SLA backward (mma.sync m16n8k16 bf16), key-tile parallel.
// One CTA of 4 warps per (sequence, 64-key tile, head); each warp owns 16 keys
// and keeps their dK and dV in registers for the whole sweep over the query
// tiles that see the key tile, so dK/dV need no atomics.  dQ contributions go
// to an fp32 workspace with vector atomics and are converted at the end.
//
// With x_ij = alpha q_i.k_j, P_ij = M SiLU(x)/N, dP_ij = dO_i.v_j:
//   dV_j = sum_i P_ij dO_i,  dS_ij = M dP_ij SiLU'(x) alpha/N,
//   dK_j = sum_i dS_ij q_i,  dQ_i = sum_j dS_ij k_j
// (the chain rule through "Bending the Scaling Law Curve in Large-Scale
// Recommendation Systems", section 3, Eq. 3, under the SLA mask of section
// 4.2.1, Eq. 7).  With t = tanh(x/2): sigmoid(x) = (1 + t)/2, SiLU(x) =
// x sigmoid(x), SiLU'(x) = sigmoid(x) (1 + x (1 - sigmoid(x))).
#include "mma_sm80.cuh"
#include "sla_common.cuh"

namespace hstu {
namespace {

constexpr int kBM = 64, kBN = 64, kThreads = 128;

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
__global__ void __launch_bounds__(kThreads, 1) bwd_mma_kernel(const AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  constexpr int LD = D + 8, TILE = 64 * LD, KD = D / 16, LDS = 64 + 8;
  bf16* sK = reinterpret_cast<bf16*>(smem_raw);
  bf16* sV = sK + TILE;
  bf16* sQ = sV + TILE;       // 2 stages
  bf16* sDO = sQ + 2 * TILE;  // 2 stages
  bf16* sDS = sDO + 2 * TILE; // [64 keys][64 rows + 8]

  if (load_status(a.ws) != 0) return;
  if ((int)blockIdx.x >= a.ws->n_items) return;
  const int2 it = a.items[blockIdx.x];
  const int h = blockIdx.y, hoff = h * D;
  const SeqGeom g = seq_geom(a, it.x);
  const int j0 = it.y * kBN, j1 = imin(j0 + kBN, g.L);
  const Spans sp = k_tile_q_tiles(j0, j1, g.L, g.Lh, a.K1, a.K2e, kBM);
  const int nq = sp.count();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;

  load_tile<D>(sK, a.k, a.k_rs, g.s0 + j0, j1 - j0, hoff);
  load_tile<D>(sV, a.v, a.v_rs, g.s0 + j0, j1 - j0, hoff);
  cp_async_commit();
  if (nq > 0) {
    const int i0 = sp.at(0) * kBM, nv = imin(kBM, g.L - i0);
    load_tile<D>(sQ, a.q, a.q_rs, g.s0 + i0, nv, hoff);
    load_tile<D>(sDO, a.dout, a.do_rs, g.s0 + i0, nv, hoff);
    cp_async_commit();
  }

  const int ka = j0 + warp * 16 + gq, kb = ka + 8;
  const float alpha = a.alpha, half_alpha = 0.5f * a.alpha;
  const float dq_scale = a.alpha * a.inv_n;

  float dv[D / 8][4], dk[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dv[i][e] = dk[i][e] = 0.f;

  for (int n = 0; n < nq; ++n) {
    const int stage = n & 1;
    if (n + 1 < nq) {
      const int i0n = sp.at(n + 1) * kBM, nv = imin(kBM, g.L - i0n);
      load_tile<D>(sQ + (stage ^ 1) * TILE, a.q, a.q_rs, g.s0 + i0n, nv, hoff);
      load_tile<D>(sDO + (stage ^ 1) * TILE, a.dout, a.do_rs, g.s0 + i0n, nv, hoff);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int i0 = sp.at(n) * kBM, i1 = imin(i0 + kBM, g.L);
    const bf16* q_s = sQ + stage * TILE;
    const bf16* do_s = sDO + stage * TILE;

    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 64 rows.
    float st[8][4], dpt[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KD; ++kk) {
      uint32_t kf[4], vf[4];
      ldsm_x4(kf, sK + (warp * 16 + (lane & 15)) * LD + kk * 16 + (lane >> 4) * 8);
      ldsm_x4(vf, sV + (warp * 16 + (lane & 15)) * LD + kk * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int off = (np * 16 + (lane >> 4) * 8 + (lane & 7)) * LD + kk * 16 +
                        ((lane >> 3) & 1) * 8;
        uint32_t b[4];
        ldsm_x4(b, q_s + off);
        mma_bf16(st[2 * np], kf, b[0], b[1]);
        mma_bf16(st[2 * np + 1], kf, b[2], b[3]);
        ldsm_x4(b, do_s + off);
        mma_bf16(dpt[2 * np], vf, b[0], b[1]);
        mma_bf16(dpt[2 * np + 1], vf, b[2], b[3]);
      }
    }
    // P^T (unscaled by 1/N) into st, dS^T (unscaled by alpha/N) into dpt.
    const bool full = tile_full(i0, i1, j0, j1, g.Lh, a.K1, a.K2e);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = st[nt][e] * alpha, hx = st[nt][e] * half_alpha;
        const float t = tanh_approx(hx);
        const float sg = fmaf(0.5f, t, 0.5f);
        const float silu = fmaf(hx, t, hx);
        const float dsilu = sg * fmaf(x, 1.f - sg, 1.f);
        bool vis = true;
        if (!full) {
          const int i = i0 + nt * 8 + 2 * tq + (e & 1), j = (e < 2) ? ka : kb;
          vis = sla_visible(i, j, g.L, g.Lh, a.K1, a.K2e);
        }
        st[nt][e] = vis ? silu : 0.f;
        dpt[nt][e] = vis ? dpt[nt][e] * dsilu : 0.f;
      }
    }
    // dV += P^T dO, dK += dS^T Q (k = the 64 rows).
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pf[4] = {pack_bf16(st[2 * kk][0], st[2 * kk][1]),
                        pack_bf16(st[2 * kk][2], st[2 * kk][3]),
                        pack_bf16(st[2 * kk + 1][0], st[2 * kk + 1][1]),
                        pack_bf16(st[2 * kk + 1][2], st[2 * kk + 1][3])};
      uint32_t sf[4] = {pack_bf16(dpt[2 * kk][0], dpt[2 * kk][1]),
                        pack_bf16(dpt[2 * kk][2], dpt[2 * kk][3]),
                        pack_bf16(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]),
                        pack_bf16(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3])};
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int off = (kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * LD + dp * 16 +
                        (lane >> 4) * 8;
        uint32_t b[4];
        ldsm_x4_t(b, do_s + off);
        mma_bf16(dv[2 * dp], pf, b[0], b[1]);
        mma_bf16(dv[2 * dp + 1], pf, b[2], b[3]);
        ldsm_x4_t(b, q_s + off);
        mma_bf16(dk[2 * dp], sf, b[0], b[1]);
        mma_bf16(dk[2 * dp + 1], sf, b[2], b[3]);
      }
    }
    // dS^T -> smem, then dQ (64 rows x D) = dS K; warp w takes rows 16w..16w+15.
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      *reinterpret_cast<uint32_t*>(sDS + (warp * 16 + gq) * LDS + nt * 8 + 2 * tq) =
          pack_bf16(dpt[nt][0], dpt[nt][1]);
      *reinterpret_cast<uint32_t*>(sDS + (warp * 16 + gq + 8) * LDS + nt * 8 + 2 * tq) =
          pack_bf16(dpt[nt][2], dpt[nt][3]);
    }
    __syncthreads();
    uint32_t dsf[4][4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      ldsm_x4_t(dsf[kk], sDS + (kk * 16 + (lane >> 4) * 8 + (lane & 7)) * LDS + warp * 16 +
                             ((lane >> 3) & 1) * 8);
    const int ra = i0 + warp * 16 + gq, rb = ra + 8;
    float* dqa = a.dq_acc + ((int64_t)(g.s0 + ra) * a.H + h) * D;
    float* dqb = a.dq_acc + ((int64_t)(g.s0 + rb) * a.H + h) * D;
#pragma unroll
    for (int dc = 0; dc < D / 32; ++dc) {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int dp = 0; dp < 2; ++dp) {
          uint32_t b[4];
          ldsm_x4_t(b, sK + (kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * LD + dc * 32 +
                           dp * 16 + (lane >> 4) * 8);
          mma_bf16(acc[2 * dp], dsf[kk], b[0], b[1]);
          mma_bf16(acc[2 * dp + 1], dsf[kk], b[2], b[3]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int c = dc * 32 + nt * 8 + 2 * tq;
        if (ra < i1)
          atomicAdd(reinterpret_cast<float2*>(dqa + c),
                    make_float2(acc[nt][0] * dq_scale, acc[nt][1] * dq_scale));
        if (rb < i1)
          atomicAdd(reinterpret_cast<float2*>(dqb + c),
                    make_float2(acc[nt][2] * dq_scale, acc[nt][3] * dq_scale));
      }
    }
    __syncthreads();
  }

  // Epilogue: dV * 1/N and dK * alpha/N, staged through smem, row-predicated.
  cp_async_wait<0>();
  __syncthreads();
  bf16* sv = sQ;          // 64 x LD
  bf16* sk = sQ + TILE;   // 64 x LD
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {
    const int r = warp * 16 + gq, c = nt * 8 + 2 * tq;
    *reinterpret_cast<uint32_t*>(sv + r * LD + c) =
        pack_bf16(dv[nt][0] * a.inv_n, dv[nt][1] * a.inv_n);
    *reinterpret_cast<uint32_t*>(sv + (r + 8) * LD + c) =
        pack_bf16(dv[nt][2] * a.inv_n, dv[nt][3] * a.inv_n);
    *reinterpret_cast<uint32_t*>(sk + r * LD + c) =
        pack_bf16(dk[nt][0] * dq_scale, dk[nt][1] * dq_scale);
    *reinterpret_cast<uint32_t*>(sk + (r + 8) * LD + c) =
        pack_bf16(dk[nt][2] * dq_scale, dk[nt][3] * dq_scale);
  }
  __syncthreads();
  constexpr int CPR = D / 8;
  for (int c = threadIdx.x; c < 64 * CPR; c += kThreads) {
    const int r = c / CPR, cc = c - r * CPR, j = j0 + r;
    if (j < j1) {
      *reinterpret_cast<uint4*>(a.dv + (int64_t)(g.s0 + j) * a.dv_rs + hoff + cc * 8) =
          *reinterpret_cast<const uint4*>(sv + r * LD + cc * 8);
      *reinterpret_cast<uint4*>(a.dk + (int64_t)(g.s0 + j) * a.dk_rs + hoff + cc * 8) =
          *reinterpret_cast<const uint4*>(sk + r * LD + cc * 8);
    }
  }
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t st) {
  const int smem = (6 * 64 * (D + 8) + 64 * 72) * 2;
  cudaError_t e = cudaFuncSetAttribute(bwd_mma_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)max_items(a.T, a.B), a.H);
  bwd_mma_kernel<D><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_mma(const AttnArgs& a, int d, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  if (d == 32) return launch_d<32>(a, st);
  if (d == 64) return launch_d<64>(a, st);
  return launch_d<128>(a, st);
}

}  // namespace hstu
