// Row- and column-wise kernels of the STU layer ("Bending the Scaling Law
// Curve in Large-Scale Recommendation Systems", section 3, Eq. 1-5; HSTU's
// "Actions Speak Louder than Words", section 3.1):
//   LayerNorm before the UVQK projection (Eq. 1), the gated norm
//   y = LayerNorm(A V) * U after the attention (Eq. 4), their backward with
//   the affine-parameter gradients, SiLU' on the projection's gradient with
//   the bias gradient, and the attention truncation of section 4.3 (keep the
//   contextual prefix, the last `tail` history tokens and the candidates, as
//   TorchEasyRec's "Mid-stack Attention Truncation" bullet states).
// Rows are d_model wide (W = 256, 512 or 1024); one warp per row, lane l
// owning the 16-byte chunks l, l + 32, ... of the row.
#include "sm100.cuh"
#include "stu_common.cuh"

namespace hstu {
namespace {

constexpr int kRowWarps = 8;  // rows per 256-thread block

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void load8(const bf16* p, float* f) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    f[2 * h] = __uint_as_float(w[h] << 16);
    f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void store8(bf16* p, const float* f) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

using sm100::silu_grad;

// LayerNorm (biased variance) of each row, then the affine map; GATED also
// multiplies by the gate row u.  Saves the row mean and 1/sqrt(var + eps).
// With yq set, also writes the row in E4M3 with a per-row scale: the FP8
// quantization fused into the norm that precedes each projection ("Bending
// the Scaling Law Curve...", section 4.2.2, mixed-precision training and
// inference; Figure 4).  A warp takes kLnRows rows and issues every row's
// loads (x, the gate) before its first reduction, holding them as packed
// bf16, so several rows' latencies overlap; gamma and beta are read where
// they are used (the same 2 W floats for every warp: L1 hits).
template <int NV>
constexpr int ln_rows() { return NV >= 4 ? 2 : 4; }

__device__ __forceinline__ void unpack8(const uint4 r, float* f) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    f[2 * h] = __uint_as_float(w[h] << 16);
    f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void ldg8f(const float* p, float* f) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <int NV, bool GATED>
__global__ void __launch_bounds__(32 * kRowWarps) ln_fwd_kernel(const LnArgs a) {
  constexpr int W = NV * 256;
  const int lane = threadIdx.x & 31;
  constexpr int kLnRows = ln_rows<NV>();
  const int64_t row0 = ((int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5)) * kLnRows;
  if (row0 >= a.T) return;
  uint4 xp[kLnRows][NV], up[GATED ? kLnRows : 1][NV];
#pragma unroll
  for (int r = 0; r < kLnRows; ++r) {
    const int64_t row = row0 + r < a.T ? row0 + r : row0;  // a missing row repeats the first
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      xp[r][v] = *reinterpret_cast<const uint4*>(a.x + row * a.ldx + 8 * (lane + 32 * v));
      if (GATED)
        up[GATED ? r : 0][v] =
            *reinterpret_cast<const uint4*>(a.u + row * a.ldu + 8 * (lane + 32 * v));
    }
  }
#pragma unroll
  for (int r = 0; r < kLnRows; ++r) {
    const int64_t row = row0 + r;
    if (row >= a.T) break;
    float x[NV][8];
#pragma unroll
    for (int v = 0; v < NV; ++v) unpack8(xp[r][v], x[v]);
    float mean = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
      for (int e = 0; e < 8; ++e) mean += x[v][e];
    mean = warp_sum(mean) * (1.0f / W);
    float q = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
      for (int e = 0; e < 8; ++e) q += (x[v][e] - mean) * (x[v][e] - mean);
    const float rstd = rsqrtf(warp_sum(q) * (1.0f / W) + a.eps);
    float amax = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int c = 8 * (lane + 32 * v);
      float gm[8], bt[8], u[8];
      ldg8f(a.gamma + c, gm);
      ldg8f(a.beta + c, bt);
      if (GATED) unpack8(up[GATED ? r : 0][v], u);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[v][e] = (x[v][e] - mean) * rstd * gm[e] + bt[e];  // x now holds y
        if (GATED) x[v][e] *= u[e];
      }
      store8(a.y + row * a.ldy + c, x[v]);
      if (a.yq) {  // quantize what the bf16 output holds
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          x[v][e] = __bfloat162float(__float2bfloat16(x[v][e]));
          amax = fmaxf(amax, fabsf(x[v][e]));
        }
      }
    }
    if (a.yq) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float scale = amax > 0.f ? amax * (1.0f / 448.0f) : 1.0f;
      const float inv = 1.0f / scale;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const int c = 8 * (lane + 32 * v);
        uint2 w;
        w.x = sm100::pack_e4m3x2(x[v][0] * inv, x[v][1] * inv) |
              (sm100::pack_e4m3x2(x[v][2] * inv, x[v][3] * inv) << 16);
        w.y = sm100::pack_e4m3x2(x[v][4] * inv, x[v][5] * inv) |
              (sm100::pack_e4m3x2(x[v][6] * inv, x[v][7] * inv) << 16);
        *reinterpret_cast<uint2*>(a.yq + row * a.ldyq + c) = w;
      }
      if (lane == 0) a.yscale[row] = scale;
    }
    if (lane == 0) {
      a.mean[row] = mean;
      a.rstd[row] = rstd;
    }
  }
}

// Weight quantizer: a block owns 64 output columns.  It first takes each
// column's max |W[k][n]| over all K (4 row phases x 64 columns, one reduce),
// then converts 64 x 64 chunks through shared memory so that the transposed
// rows of Wq are written 16 bytes at a time.
__global__ void __launch_bounds__(256) quant_wt_kernel(const bf16* W, int64_t ldw, int K,
                                                       uint8_t* Wq, int64_t ldq, float* scale) {
  __shared__ float s_amax[4][64];
  __shared__ __align__(16) uint8_t s_q[64][80];  // [n][k], rows padded to 80 bytes
  const int c = threadIdx.x & 63, r = threadIdx.x >> 6;
  const int n0 = blockIdx.x * 64;
  const bf16* col = W + n0 + c;
  float amax = 0.f;
#pragma unroll 4
  for (int k = r; k < K; k += 4) amax = fmaxf(amax, fabsf(__bfloat162float(col[(int64_t)k * ldw])));
  s_amax[r][c] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(s_amax[0][c], s_amax[1][c]), fmaxf(s_amax[2][c], s_amax[3][c]));
  const float sc = amax > 0.f ? amax * (1.0f / 448.0f) : 1.0f;
  const float inv = 1.0f / sc;
  if (r == 0) scale[n0 + c] = sc;
  const int orow = threadIdx.x >> 2, ochunk = (threadIdx.x & 3) * 16;
  for (int k0 = 0; k0 < K; k0 += 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int kk = r + 4 * i;
      const float f = __bfloat162float(col[(int64_t)(k0 + kk) * ldw]) * inv;
      s_q[c][kk] = (uint8_t)sm100::pack_e4m3x2(f, 0.f);
    }
    __syncthreads();
    *reinterpret_cast<uint4*>(Wq + (int64_t)(n0 + orow) * ldq + k0 + ochunk) =
        *reinterpret_cast<const uint4*>(&s_q[orow][ochunk]);
    __syncthreads();
  }
}

// Backward of the above.  Plain: dx = resid_grad + LN'(dy * gamma).
// Gated: dz = dy * u, du = dy * z (times SiLU'(pre_u), since the gate is a
// SiLU output), dx = LN'(dz * gamma).  Two passes over each row, both from
// registers: every load of the row (x, dy, the gate and its pre-activation,
// the residual gradient) is issued first and held as packed bf16, so a row
// costs one memory latency; dgamma / dbeta (and, gated, the column sums of du: the
// gate's bias gradient) accumulate in shared memory over the rows a block
// visits (per warp, each lane updating only its own columns, for W <= 512;
// shared atomics beyond), then once per block and column in global memory.
template <int NV, bool GATED>
__global__ void __launch_bounds__(32 * kRowWarps, GATED ? 2 : 3) ln_bwd_kernel(const LnArgs a) {
  constexpr int W = NV * 256;
  constexpr bool kPerWarp = NV <= 2;
  constexpr int kAcc = kPerWarp ? kRowWarps : 1;
  // shared memory: gamma, beta, then the dgamma, dbeta (and, gated, du)
  // accumulators, kAcc rows of W each; dynamic for the gated form (past the
  // 48 KB of static shared memory at W = 512)
  float* ln_smem;
  if constexpr (GATED) {
    extern __shared__ __align__(16) float ln_dyn[];
    ln_smem = ln_dyn;
  } else {
    __shared__ __align__(16) float ln_static[(2 + 2 * kAcc) * W];
    ln_smem = ln_static;
  }
  float* s_g = ln_smem;
  float* s_b = s_g + W;
  float* s_dg = s_b + W;
  float* s_db = s_dg + kAcc * W;
  float* s_du = s_db + kAcc * W;
  for (int c = threadIdx.x; c < W; c += blockDim.x) {
    s_g[c] = a.gamma[c];
    s_b[c] = a.beta[c];
    for (int w = 0; w < kAcc; ++w) {
      s_dg[w * W + c] = s_db[w * W + c] = 0.f;
      if (GATED) s_du[w * W + c] = 0.f;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int acc_row = kPerWarp ? (threadIdx.x >> 5) : 0;
  float* my_dg = s_dg + acc_row * W;
  float* my_db = s_db + acc_row * W;
  float* my_du = s_du + acc_row * W;
  const int64_t nwarps = (int64_t)gridDim.x * kRowWarps;
  for (int64_t row = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5); row < a.T;
       row += nwarps) {
    // every load of the row first, held as packed bf16 for both passes
    uint4 xp[NV], dyp[NV], up[GATED ? NV : 1], pup[GATED ? NV : 1], rp[NV];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int c = 8 * (lane + 32 * v);
      xp[v] = *reinterpret_cast<const uint4*>(a.x + row * a.ldx + c);
      dyp[v] = *reinterpret_cast<const uint4*>(a.dy + row * a.lddy + c);
      if (GATED) {
        up[GATED ? v : 0] = *reinterpret_cast<const uint4*>(a.u + row * a.ldu + c);
        pup[GATED ? v : 0] = *reinterpret_cast<const uint4*>(a.pre_u + row * a.ldpu + c);
      }
      if (a.resid_grad) rp[v] = *reinterpret_cast<const uint4*>(a.resid_grad + row * a.ldr + c);
    }
    const float mean = a.mean[row], rstd = a.rstd[row];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int c = 8 * (lane + 32 * v);
      float x[8], dy[8], u[8], pu[8], du[8], tg[8], tb[8];
      unpack8(xp[v], x);
      unpack8(dyp[v], dy);
      if (GATED) {
        unpack8(up[GATED ? v : 0], u);
        unpack8(pup[GATED ? v : 0], pu);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xh = (x[e] - mean) * rstd;
        float dz = dy[e];
        if (GATED) {
          du[e] = dy[e] * (s_g[c + e] * xh + s_b[c + e]) * silu_grad(pu[e]);
          dz = dy[e] * u[e];
        }
        tg[e] = dz * xh;
        tb[e] = dz;
        const float g = dz * s_g[c + e];
        s1 += g;
        s2 += g * xh;
      }
      if (kPerWarp) {  // this lane's own 8 columns of its warp's row
        float4* pg = reinterpret_cast<float4*>(my_dg + c);
        float4* pb = reinterpret_cast<float4*>(my_db + c);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float4 g4 = pg[h], b4 = pb[h];
          g4.x += tg[4 * h]; g4.y += tg[4 * h + 1]; g4.z += tg[4 * h + 2]; g4.w += tg[4 * h + 3];
          b4.x += tb[4 * h]; b4.y += tb[4 * h + 1]; b4.z += tb[4 * h + 2]; b4.w += tb[4 * h + 3];
          pg[h] = g4;
          pb[h] = b4;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          atomicAdd(my_dg + c + e, tg[e]);
          atomicAdd(my_db + c + e, tb[e]);
        }
      }
      if (GATED) {
        store8(a.du + row * a.lddu + c, du);
        if (a.dbias_u) {
          if (kPerWarp) {
            float4* pu4 = reinterpret_cast<float4*>(my_du + c);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float4 u4 = pu4[h];
              u4.x += du[4 * h]; u4.y += du[4 * h + 1]; u4.z += du[4 * h + 2];
              u4.w += du[4 * h + 3];
              pu4[h] = u4;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) atomicAdd(my_du + c + e, du[e]);
          }
        }
      }
    }
    const float m1 = warp_sum(s1) * (1.0f / W), m2 = warp_sum(s2) * (1.0f / W);
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int c = 8 * (lane + 32 * v);
      float x[8], dy[8], u[8], dx[8], r[8];
      unpack8(xp[v], x);
      unpack8(dyp[v], dy);
      if (GATED) unpack8(up[GATED ? v : 0], u);
      if (a.resid_grad) unpack8(rp[v], r);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xh = (x[e] - mean) * rstd;
        const float g = (GATED ? dy[e] * u[e] : dy[e]) * s_g[c + e];
        dx[e] = rstd * (g - m1 - xh * m2);
        if (a.resid_grad) dx[e] += r[e];
      }
      store8(a.dx + row * a.lddx + c, dx);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < W; c += blockDim.x) {
    float g = 0.f, b = 0.f;
    float u = 0.f;
    for (int w = 0; w < kAcc; ++w) {
      g += s_dg[w * W + c];
      b += s_db[w * W + c];
      if (GATED) u += s_du[w * W + c];
    }
    atomicAdd(a.dgamma + c, g);
    atomicAdd(a.dbeta + c, b);
    if (GATED && a.dbias_u) atomicAdd(a.dbias_u + c, u);
  }
}

// Column-parallel pass over [T][W] in 256-thread blocks: W / 8 threads own
// columns [8t, 8t + 8) of a row; 256 / (W / 8) such groups take interleaved
// rows of the block's chunk.  SCALE multiplies columns >= c0 by SiLU'(pre)
// in place; every column's (scaled) values are summed, per block in shared
// memory, then into dbias.
constexpr int kColThreads = 256;
template <bool SCALE>
__global__ void __launch_bounds__(kColThreads) colsum_kernel(bf16* g, int64_t ldg, const bf16* pre,
                                                             int64_t ldp, int64_t T, int W,
                                                             int c0, float* dbias, int rows) {
  const int ncol = W / 8, groups = kColThreads / ncol;
  const int t = threadIdx.x % ncol, grp = threadIdx.x / ncol;
  const int c = 8 * t;
  const int64_t r0 = (int64_t)blockIdx.x * rows;
  const int64_t r1 = r0 + rows < T ? r0 + rows : T;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (grp < groups) {
    const bool scale = SCALE && c >= c0;
    for (int64_t r = r0 + grp; r < r1; r += groups) {
      float v[8];
      load8(g + r * ldg + c, v);
      if (scale) {
        float p[8];
        load8(pre + r * ldp + c, p);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= silu_grad(p[e]);
        store8(g + r * ldg + c, v);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += v[e];
    }
  }
  if (groups == 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicAdd(dbias + c + e, acc[e]);
    return;
  }
  // several row groups: sum them through shared memory, column by column
  __shared__ float s_sum[kColThreads * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s_sum[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  for (int col = threadIdx.x; col < W; col += kColThreads) {
    const int tt = col / 8, e = col % 8;
    float sum = 0.f;
    for (int q = 0; q < groups; ++q) sum += s_sum[(q * ncol + tt) * 8 + e];
    atomicAdd(dbias + col, sum);
  }
}

// New offsets after truncation (one thread; B is small).
__global__ void trunc_offsets_kernel(const int32_t* offs, const int32_t* nts, int B, int c,
                                     int tail, int32_t* new_offs) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int32_t o = 0;
  new_offs[0] = 0;
  for (int b = 0; b < B; ++b) {
    const int L = offs[b + 1] - offs[b];
    const int drop = trunc_drop(L, nts ? nts[b] : 0, c, tail);
    o += L - drop;
    new_offs[b + 1] = o;
  }
}

__device__ __forceinline__ int find_seq(const int32_t* offs, int B, int64_t r) {
  int lo = 0, hi = B;  // offs[lo] <= r < offs[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offs[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

// Gather (rows of the truncated layout from the full one) or scatter (rows of
// the full layout from the truncated one; dropped rows become zero).  One warp
// per output row.
__global__ void __launch_bounds__(256) trunc_rows_kernel(const bf16* src, int64_t lds,
                                                         const int32_t* offs,
                                                         const int32_t* new_offs,
                                                         const int32_t* nts, int B, int c,
                                                         int tail, int W, bf16* dst, int64_t ldd,
                                                         int64_t T_out, int scatter) {
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= T_out) return;
  const int32_t* out_offs = scatter ? offs : new_offs;
  const int32_t* in_offs = scatter ? new_offs : offs;
  const int b = find_seq(out_offs, B, r);
  const int L = offs[b + 1] - offs[b];
  const int drop = trunc_drop(L, nts ? nts[b] : 0, c, tail);
  const int p = (int)(r - out_offs[b]);
  int64_t s;  // source row, or -1 for a dropped row (scatter)
  if (scatter) s = (p < c || p >= c + drop) ? in_offs[b] + p - (p >= c ? drop : 0) : -1;
  else s = in_offs[b] + p + (p >= c ? drop : 0);
  uint4* d = reinterpret_cast<uint4*>(dst + r * ldd);
  const uint4* q = s >= 0 ? reinterpret_cast<const uint4*>(src + s * lds) : nullptr;
  for (int j = lane; j < W / 8; j += 32) d[j] = q ? q[j] : make_uint4(0, 0, 0, 0);
}

}  // namespace

cudaError_t launch_ln_fwd(const LnArgs& a, bool gated, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
#define HSTU_LN(NV)                                                                     \
  if (a.W == NV * 256) {                                                                \
    constexpr int rows = kRowWarps * ln_rows<NV>();                                     \
    const int grid = (int)((a.T + rows - 1) / rows);                                    \
    if (gated) ln_fwd_kernel<NV, true><<<grid, 32 * kRowWarps, 0, st>>>(a);             \
    else ln_fwd_kernel<NV, false><<<grid, 32 * kRowWarps, 0, st>>>(a);                  \
    return cudaGetLastError();                                                          \
  }
  HSTU_LN(1) HSTU_LN(2) HSTU_LN(4)
#undef HSTU_LN
  return cudaErrorNotSupported;
}

cudaError_t launch_quant_wt(const bf16* W, int64_t ldw, int K, int N, uint8_t* Wq, int64_t ldq,
                            float* scale, cudaStream_t st) {
  if (K % 64 != 0 || N % 64 != 0 || ldq % 16 != 0) return cudaErrorNotSupported;
  if (N == 0) return cudaSuccess;
  quant_wt_kernel<<<N / 64, 256, 0, st>>>(W, ldw, K, Wq, ldq, scale);
  return cudaGetLastError();
}

template <int NV, bool GATED>
cudaError_t launch_ln_bwd_t(const LnArgs& a, cudaStream_t st) {
  constexpr int W = NV * 256;
  constexpr int kAcc = NV <= 2 ? kRowWarps : 1;
  // dynamic shared memory for the gated form only (its carveout: what two
  // blocks need, the rest of the SM's 256 KB stays L1)
  constexpr int bytes = GATED ? (2 + 3 * kAcc) * W * (int)sizeof(float) : 0;
  if (GATED) {
    cudaError_t e = cudaFuncSetAttribute(ln_bwd_kernel<NV, GATED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(ln_bwd_kernel<NV, GATED>,
                               cudaFuncAttributePreferredSharedMemoryCarveout,
                               (2 * (bytes + 1024) * 100 + 228 * 1024 - 1) / (228 * 1024));
    if (e != cudaSuccess) return e;
  }
  // whole waves: as many blocks as fit on every SM at once (rows are strided
  // over the grid), fewer for short batches
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, ln_bwd_kernel<NV, GATED>, 32 * kRowWarps, bytes);
  if (e != cudaSuccess) return e;
  const int64_t need = (a.T + kRowWarps - 1) / kRowWarps;
  const int64_t cap = (int64_t)device_sm_count() * (per_sm > 0 ? per_sm : 1);
  const int grid = (int)(need < cap ? need : cap);
  ln_bwd_kernel<NV, GATED><<<grid, 32 * kRowWarps, bytes, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ln_bwd(const LnArgs& a, bool gated, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
#define HSTU_LNB(NV)                                                                    \
  if (a.W == NV * 256) {                                                                \
    if (gated) return launch_ln_bwd_t<NV, true>(a, st);                                 \
    return launch_ln_bwd_t<NV, false>(a, st);                                           \
  }
  HSTU_LNB(1) HSTU_LNB(2) HSTU_LNB(4)
#undef HSTU_LNB
  return cudaErrorNotSupported;
}

// Rows per block: about 64 rows' worth of 16-byte loads per thread.
int colsum_rows(int W) { return 64 * (kColThreads / (W / 8)); }

bool colsum_width_ok(int W) {
  return W % 8 == 0 && W / 8 <= kColThreads && kColThreads % (W / 8) == 0;
}

cudaError_t launch_silu_bwd_colsum(bf16* g, int64_t ldg, const bf16* pre, int64_t ldp, int64_t T,
                                   int W, int c0, float* dbias, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (!colsum_width_ok(W)) return cudaErrorNotSupported;
  const int rows = colsum_rows(W);
  const int grid = (int)((T + rows - 1) / rows);
  colsum_kernel<true><<<grid, kColThreads, 0, st>>>(g, ldg, pre, ldp, T, W, c0, dbias, rows);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const bf16* g, int64_t ldg, int64_t T, int W, float* dbias,
                          cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (!colsum_width_ok(W)) return cudaErrorNotSupported;
  const int rows = colsum_rows(W);
  const int grid = (int)((T + rows - 1) / rows);
  colsum_kernel<false><<<grid, kColThreads, 0, st>>>(const_cast<bf16*>(g), ldg, nullptr, 0, T, W,
                                                     W, dbias, rows);
  return cudaGetLastError();
}

cudaError_t launch_trunc_offsets(const int32_t* offs, const int32_t* nts, int B, int c, int tail,
                                 int32_t* new_offs, cudaStream_t st) {
  trunc_offsets_kernel<<<1, 32, 0, st>>>(offs, nts, B, c, tail, new_offs);
  return cudaGetLastError();
}

cudaError_t launch_trunc_rows(const bf16* src, int64_t lds, const int32_t* offs,
                              const int32_t* new_offs, const int32_t* nts, int B, int c, int tail,
                              int W, bf16* dst, int64_t ldd, int64_t T_out, bool scatter,
                              cudaStream_t st) {
  if (T_out == 0) return cudaSuccess;
  const int grid = (int)((T_out + 7) / 8);
  trunc_rows_kernel<<<grid, 256, 0, st>>>(src, lds, offs, new_offs, nts, B, c, tail, W, dst, ldd,
                                          T_out, scatter ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace hstu
