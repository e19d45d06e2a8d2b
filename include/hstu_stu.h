/*
 * hstu_stu.h -- C ABI of the STU layer around the SLA attention (B200, sm_100a).
 *
 * One STU layer ("Bending the Scaling Law Curve in Large-Scale Recommendation
 * Systems", section 3, Eq. 1-5, and the forward / backward of its Listing 1
 * in section 4.2.2), on a jagged batch of T tokens of width d_model = H * d:
 *
 *     x^          = LayerNorm(x) * ln1_w + ln1_b
 *     pre         = x^ W1 + b1                  W1: [d_model][4 d_model]
 *     U, V, Q, K  = split(SiLU(pre))            column blocks of d_model, in
 *                                               that order
 *     A           = SLA attention of Q, K, V    (hstu_sla.h, heads of d)
 *     y           = (LayerNorm(A) * ln2_w + ln2_b) * U
 *     out         = y W2 + b2 + x               W2: [d_model][d_model]
 *
 * The backward takes dout = dL/dout and produces dx and the gradients of
 * every parameter (fp32).  Attention truncation (section 4.3; TorchEasyRec's
 * "Mid-stack Attention Truncation") keeps, per
 * sequence, the contextual prefix [0, c), the last `tail` history tokens and
 * all candidates: rows [c, c + drop) go, drop = max(0, Lh - c - tail).
 *
 * Conventions are those of hstu_sla.h: device pointers, caller-owned
 * buffers, asynchronous on `stream`, HSTU_SLA_* return codes, no traps.
 * All matrices are row-major with rows contiguous (row stride = width):
 * activations bf16, LayerNorm parameters, biases and gradients fp32.
 * d_model must be 256, 512 or 1024 and d one of the attention head dims.
 */
#ifndef HSTU_STU_H_
#define HSTU_STU_H_

#include "hstu_sla.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t B, H, d;             /* d_model = H * d */
  int64_t total_tokens;        /* T = seq_offsets[B] */
  int32_t max_seq_len;
  const int32_t* seq_offsets;  /* device [B + 1] */
  const int32_t* num_targets;  /* device [B] or NULL */
  int32_t contextual_len, K1, K2;
  float alpha, N;              /* attention scale and normaliser */
  float ln_eps;                /* LayerNorm epsilon */
  /* parameters (device) */
  const float* ln1_w;          /* [d_model] */
  const float* ln1_b;
  const void* w1;              /* bf16 [d_model][4 d_model] */
  const float* b1;             /* [4 d_model] */
  const float* ln2_w;          /* [d_model] */
  const float* ln2_b;
  const void* w2;              /* bf16 [d_model][d_model] */
  const float* b2;             /* [d_model] */
  /* activations (device, bf16) */
  const void* x;               /* [T][d_model] layer input */
  void* out;                   /* [T][d_model] layer output */
  /* saved by the forward for the backward (caller-owned) */
  void* xn;                    /* [T][d_model]    x^ */
  void* pre;                   /* [T][4 d_model]  pre-activation */
  void* uvqk;                  /* [T][4 d_model]  SiLU(pre) = U | V | Q | K */
  void* av;                    /* [T][d_model]    attention output */
  void* y;                     /* [T][d_model]    gated norm output */
  float* stats;                /* [4][T]          mean / rstd of both norms */
  /* FP8 forward projections (section 4.2.2, mixed-precision training and
   * inference; appendix E.1, Tables 7 and 10): with fp8 = 1 the forward computes x^ W1 and y W2 with E4M3
   * operands and fp32 accumulation.  Each LayerNorm also writes its output
   * row in E4M3 with one scale per row (max |row| / 448, into the workspace),
   * and the weights come pre-quantized by hstu_quant_weight_e4m3 (one scale
   * per output column).  Everything saved for the backward stays bf16 and the
   * backward itself is unchanged (bf16 GEMMs against w1 / w2).  fp8 = 0 reads
   * none of the four fields below. */
  int32_t fp8;
  const void* w1q;             /* E4M3 [4 d_model][d_model]: W1 transposed */
  const float* w1s;            /* [4 d_model] column scales of W1 */
  const void* w2q;             /* E4M3 [d_model][d_model]:   W2 transposed */
  const float* w2s;            /* [d_model] */
  /* Selective activation rematerialisation (section 4.2.2 and its code
   * Listing 1): with remat = 1 the forward keeps for the backward only what
   * the listing saves, x (the caller's input), u (the U block of SiLU(pre),
   * [T][d_model], written here), av and stats; xn, pre, uvqk and y are
   * scratch in the workspace (their pointers are not read and may be NULL).
   * The backward recomputes x^ = LayerNorm(x) and pre, U | V | Q | K with the
   * same kernels (so the same bits), and y = LayerNorm(av) * u, then runs the
   * usual backward.  Workspaces: HSTU_STU_WS_FWD_REMAT / HSTU_STU_WS_BWD_REMAT.
   * Not with fp8 = 1 (HSTU_SLA_ERR_UNSUPPORTED). */
  int32_t remat;
  void* u;                     /* bf16 [T][d_model]; read only with remat = 1 */
} hstu_stu_layer_params;

typedef struct {
  hstu_stu_layer_params fwd;   /* as given to (and filled by) the forward */
  const void* dout;            /* bf16 [T][d_model] */
  void* dx;                    /* bf16 [T][d_model] */
  /* scratch (bf16) */
  void* dy;                    /* [T][d_model] */
  void* dav;                   /* [T][d_model] */
  void* dpre;                  /* [T][4 d_model] */
  void* dxn;                   /* [T][d_model] */
  /* parameter gradients (fp32, same shapes as the parameters); overwritten */
  float* d_ln1_w;
  float* d_ln1_b;
  float* d_w1;
  float* d_b1;
  float* d_ln2_w;
  float* d_ln2_b;
  float* d_w2;
  float* d_b2;
} hstu_stu_layer_bwd_params;

/* Workspace bytes for hstu_stu_layer_fwd (which = HSTU_SLA_WS_FWD, or
 * HSTU_STU_WS_FWD_FP8 when fp8 = 1: the E4M3 activation rows on top, or
 * HSTU_STU_WS_FWD_REMAT when remat = 1) or hstu_stu_layer_bwd
 * (HSTU_SLA_WS_BWD, or HSTU_STU_WS_BWD_REMAT when remat = 1); 256-byte
 * aligned, contents need not be initialised.  0 on invalid arguments. */
#define HSTU_STU_WS_FWD_FP8 2
#define HSTU_STU_WS_FWD_REMAT 3  /* forward with remat = 1: + x^, pre, U|V|Q|K, y scratch */
#define HSTU_STU_WS_BWD_REMAT 4  /* backward with remat = 1: + the recomputed tensors */
size_t hstu_stu_workspace_bytes(int which, int64_t total_tokens, int32_t B, int32_t H, int32_t d);

int hstu_stu_layer_fwd(const hstu_stu_layer_params* p, void* workspace, size_t workspace_bytes,
                       hstu_stream_t stream);
int hstu_stu_layer_bwd(const hstu_stu_layer_bwd_params* p, void* workspace,
                       size_t workspace_bytes, hstu_stream_t stream);

/* E4M3 copy of a weight W (bf16 [K][N], row stride ldw elements, the x W
 * convention of the layer) for the FP8 forward: wq[n][k] (row stride ldq
 * bytes, a multiple of 16) and scale[n] = max_k |W[k][n]| / 448 (1 for an
 * all-zero column), so that wq[n][k] * scale[n] ~ W[k][n] (round to nearest
 * even, saturating).  K and N multiples of 64.  Call it whenever W changes. */
int hstu_quant_weight_e4m3(const void* w, int64_t ldw, int32_t K, int32_t N, void* wq,
                           int64_t ldq, float* scale, hstu_stream_t stream);

/* Status of the last layer call that used `workspace` (syncs the stream). */
int hstu_stu_get_error(const void* workspace, hstu_stream_t stream);

/* Truncation.  new_offsets: device [B + 1], written by
 * hstu_jagged_truncate_offsets.  hstu_jagged_truncate copies `width` bf16
 * columns per row: scatter = 0 gathers the kept rows of `src` (full layout,
 * seq_offsets) into `dst` (truncated layout, T_out = new_offsets[B] rows);
 * scatter = 1 is its adjoint: `dst` (full layout, T_out = seq_offsets[B]
 * rows) receives the rows of `src` (truncated layout) and zeros for the
 * dropped rows.  Row strides in elements, multiples of 8; width a multiple
 * of 8. */
int hstu_jagged_truncate_offsets(const int32_t* seq_offsets, const int32_t* num_targets, int32_t B,
                                 int32_t contextual_len, int32_t tail, int32_t* new_offsets,
                                 hstu_stream_t stream);
/* Host-side form of the same rule, for sizing the truncated buffers before
 * any launch: host arrays lengths[B] and num_targets[B] (NULL = none) give
 * new_lengths[B] (host, may be NULL) and the return value T_out, the total
 * kept rows; HSTU_SLA_ERR_INVALID_ARG (negative) for a negative length or
 * num_targets outside [0, length].  Runs on the host only (no CUDA call). */
int64_t hstu_jagged_truncate_lengths(const int32_t* lengths, const int32_t* num_targets,
                                     int32_t B, int32_t contextual_len, int32_t tail,
                                     int32_t* new_lengths);
int hstu_jagged_truncate(const void* src, int64_t src_row_stride, const int32_t* seq_offsets,
                         const int32_t* new_offsets, const int32_t* num_targets, int32_t B,
                         int32_t contextual_len, int32_t tail, int32_t width, void* dst,
                         int64_t dst_row_stride, int64_t T_out, int32_t scatter,
                         hstu_stream_t stream);

/* The layer's GEMM, exposed for tests: D[m][n] = sum_k A[m][k] B[n][k] with
 * bf16 operands and fp32 accumulation.  An operand with *_mn_major = 0 is
 * stored K-major (row m of A / row n of B, K values contiguous); with 1, it
 * is stored with row k holding its M (or N) values.  N must be a multiple of
 * 256.  With fp8 = 1 both operands are E4M3, K-major, leading dimensions in
 * bytes (multiples of 16), and D[m][n] = a_scale[m] * b_scale[n] *
 * sum_k A[m][k] B[n][k] (not with HSTU_GEMM_RED_F32).  Epilogues: */
enum {
  HSTU_GEMM_STORE = 0,       /* out  = bf16(D) */
  HSTU_GEMM_BIAS_SILU = 1,   /* out2 = bf16(D + bias), out = bf16(SiLU(D + bias)) */
  HSTU_GEMM_BIAS_RESID = 2,  /* out  = bf16(D + bias + resid) */
  HSTU_GEMM_RED_F32 = 3      /* outf += D (fp32, split over K into `splits` parts) */
};
typedef struct {
  int32_t M, N, K;
  const void* a;
  int64_t lda;
  int32_t a_mn_major;
  const void* b;
  int64_t ldb;
  int32_t b_mn_major;
  int32_t epilogue;
  int32_t splits;
  const float* bias;   /* [N] */
  const void* resid;   /* bf16 [M][N] */
  int64_t ldr;
  void* out;           /* bf16 [M][N] */
  int64_t ldo;
  void* out2;          /* bf16 [M][N] */
  int64_t ldo2;
  float* outf;         /* fp32 [M][N] */
  int64_t ldf;
  int32_t fp8;
  const float* a_scale;  /* [M], fp8 = 1 only */
  const float* b_scale;  /* [N] */
} hstu_gemm_params;

/* workspace: >= 256 bytes, 256-byte aligned (a status word; read it with
 * hstu_sla_get_error). */
int hstu_gemm(const hstu_gemm_params* p, void* workspace, hstu_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_STU_H_ */
