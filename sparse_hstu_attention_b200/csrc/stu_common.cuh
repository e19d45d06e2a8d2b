// Device-side declarations of the STU-layer kernels: the tcgen05 GEMM and the
// row-wise / column-wise kernels around it (LayerNorm, gated norm, SiLU'
// with the bias gradient, jagged truncation).
#pragma once

#include "sla_common.cuh"

namespace hstu {

int device_sm_count();

// Attention truncation ("Bending the Scaling Law Curve in Large-Scale
// Recommendation Systems", section 4.3; TorchEasyRec's attention truncation
// fields): a sequence of length L with nt candidates keeps its contextual
// prefix [0, c), its last `tail` history rows and its candidates; the history
// rows in between, max(0, L - nt - c - tail) of them, are dropped.  The one
// definition of the rule, used by the device kernels and the host helper.
__host__ __device__ __forceinline__ int trunc_drop(int L, int nt, int c, int tail) {
  const int d = L - nt - c - tail;
  return d > 0 ? d : 0;
}

// GEMM epilogues (gemm_tc.cu)
enum { kEpiStore = 0, kEpiBiasSilu = 1, kEpiBiasResid = 2, kEpiRedF32 = 3 };

// One GEMM operand: bf16 matrix, row stride `ld` elements.  K-major: rows are
// the M (or N) index; MN-major: rows are the K index.
struct GemmOperand {
  const void* ptr;
  int64_t ld;      // elements (bytes for 8-bit operands)
  bool mn_major;
  bool fp8 = false;  // E4M3 bytes (K-major only)
};

struct GemmArgs {
  int M, N, K;       // D is M x N (N a multiple of 256); K the contraction length
  int k_split;       // K per split (set by launch_gemm)
  int splits;        // requested split-K factor (kEpiRedF32 only)
  const float* bias;  // [N]
  const bf16* resid;  // [M][N], row stride ldr
  int64_t ldr;
  bf16* out;          // [M][N] bf16, row stride ldo
  int64_t ldo;
  bf16* out2;         // kEpiBiasSilu: pre-activation [M][N], row stride ldo2
  int64_t ldo2;
  float* outf;        // kEpiRedF32: [M][N] fp32 accumulated into, row stride ldf
  int64_t ldf;
  WsHeader* ws;       // status word for the bounded waits
  const float* sa;    // 8-bit operands: D[m][n] is scaled by sa[m] * sb[n]
  const float* sb;
};

cudaError_t launch_gemm(const GemmOperand& A, const GemmOperand& B, GemmArgs g, int epi,
                        cudaStream_t st);

// Row-wise kernels over rows of width W (a multiple of 256; the STU layer's
// d_model), one warp per row (stu_ops.cu).
struct LnArgs {
  int64_t T;
  int W;
  float eps;
  const bf16* x;       // LayerNorm input [T][W], row stride ldx
  int64_t ldx;
  const bf16* u;       // gated norm: gate [T][W], row stride ldu
  int64_t ldu;
  const float* gamma;  // [W]
  const float* beta;   // [W]
  bf16* y;             // output [T][W], row stride ldy
  int64_t ldy;
  float* mean;         // [T]
  float* rstd;         // [T]
  uint8_t* yq;         // optional E4M3 copy of y [T][W] (row stride ldyq bytes), with
  int64_t ldyq;        //   yq[t] * yscale[t] ~ y[t] (per-row scale, max |y[t]| / 448)
  float* yscale;
  // backward
  const bf16* dy;      // gradient of y [T][W], row stride lddy
  int64_t lddy;
  const bf16* resid_grad;  // added to dx (residual branch), [T][W], row stride ldr, or null
  int64_t ldr;
  bf16* dx;            // [T][W], row stride lddx
  int64_t lddx;
  bf16* du;            // gated norm: d(gate) * SiLU'(pre_u), [T][W], row stride lddu
  int64_t lddu;
  const bf16* pre_u;   // gate pre-activation [T][W], row stride ldpu
  int64_t ldpu;
  float* dgamma;       // [W], accumulated into
  float* dbeta;        // [W], accumulated into
  float* dbias_u;      // gated norm, optional: column sums of du accumulated into [W]
};
cudaError_t launch_ln_fwd(const LnArgs& a, bool gated, cudaStream_t st);
// E4M3 copy of a weight W [K][N] (x W convention) transposed to [N][K] (row
// stride ldq bytes) with one scale per output column: Wq[n][k] * scale[n] ~ W[k][n].
cudaError_t launch_quant_wt(const bf16* W, int64_t ldw, int K, int N, uint8_t* Wq, int64_t ldq,
                            float* scale, cudaStream_t st);
cudaError_t launch_ln_bwd(const LnArgs& a, bool gated, cudaStream_t st);

// g[t][c] *= SiLU'(pre[t][c]) for columns [c0, W) and dbias[c] += sum_t of the
// result over all W columns (columns below c0 are taken as already scaled).
cudaError_t launch_silu_bwd_colsum(bf16* g, int64_t ldg, const bf16* pre, int64_t ldp, int64_t T,
                                   int W, int c0, float* dbias, cudaStream_t st);
// dbias[c] += sum_t g[t][c]
cudaError_t launch_colsum(const bf16* g, int64_t ldg, int64_t T, int W, float* dbias,
                          cudaStream_t st);

// Jagged truncation: per sequence keep [0, c) + the last `tail` history rows
// + the candidates; rows [c, c + drop) are dropped, drop = max(0, Lh - c - tail).
cudaError_t launch_trunc_offsets(const int32_t* offs, const int32_t* nts, int B, int c, int tail,
                                 int32_t* new_offs, cudaStream_t st);
cudaError_t launch_trunc_rows(const bf16* src, int64_t lds, const int32_t* offs,
                              const int32_t* new_offs, const int32_t* nts, int B, int c, int tail,
                              int W, bf16* dst, int64_t ldd, int64_t T_out, bool scatter,
                              cudaStream_t st);

}  // namespace hstu
