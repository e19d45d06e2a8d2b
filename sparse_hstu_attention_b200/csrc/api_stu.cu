// C ABI of the STU layer (include/hstu_stu.h): host-side checks, workspace
// carving and the launch sequence of one layer's forward and backward.
#include <string.h>

#include "../../include/hstu_stu.h"
#include "stu_common.cuh"

using namespace hstu;

namespace {

constexpr size_t kHdr = sizeof(WsHeader);  // GEMM status word; the attention's workspace follows

bool al16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// need_out: the forward writes p->out; the backward does not read it.
int check_layer(const hstu_stu_layer_params* p, bool need_out) {
  if (p == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->total_tokens < 0 || p->max_seq_len < 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  if (p->d != 32 && p->d != 64 && p->d != 128) return HSTU_SLA_ERR_UNSUPPORTED;
  const int dm = p->H * p->d;
  if (dm != 256 && dm != 512 && dm != 1024) return HSTU_SLA_ERR_UNSUPPORTED;
  if (!(p->ln_eps >= 0.f)) return HSTU_SLA_ERR_INVALID_ARG;
  const void* ptrs[] = {p->ln1_w, p->ln1_b, p->w1, p->b1, p->ln2_w, p->ln2_b, p->w2, p->b2,
                        p->x,     p->av,    p->stats};
  for (const void* q : ptrs)
    if (!al16(q)) return HSTU_SLA_ERR_INVALID_ARG;
  if (need_out && !al16(p->out)) return HSTU_SLA_ERR_INVALID_ARG;
  if (p->remat != 0 && p->remat != 1) return HSTU_SLA_ERR_INVALID_ARG;
  if (p->remat) {  // Listing 1's save set: x, u, av, stats; the rest is scratch
    if (!al16(p->u)) return HSTU_SLA_ERR_INVALID_ARG;
    if (p->fp8) return HSTU_SLA_ERR_UNSUPPORTED;
  } else {
    const void* saved[] = {p->xn, p->pre, p->uvqk, p->y};
    for (const void* q : saved)
      if (!al16(q)) return HSTU_SLA_ERR_INVALID_ARG;
  }
  if (p->fp8 != 0 && p->fp8 != 1) return HSTU_SLA_ERR_INVALID_ARG;
  if (p->fp8 && need_out && (!al16(p->w1q) || !al16(p->w1s) || !al16(p->w2q) || !al16(p->w2s)))
    return HSTU_SLA_ERR_INVALID_ARG;
  return HSTU_SLA_OK;
}

int check_ws(const void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0 || bytes < need)
    return HSTU_SLA_ERR_WORKSPACE;
  return HSTU_SLA_OK;
}

// The layer's attention: Q, K, V are column blocks 2, 3, 1 of UVQK.
hstu_sla_fwd_params attn_params(const hstu_stu_layer_params* p) {
  hstu_sla_fwd_params f;
  memset(&f, 0, sizeof(f));
  const int dm = p->H * p->d;
  f.B = p->B;
  f.H = p->H;
  f.d = p->d;
  f.total_tokens = p->total_tokens;
  f.max_seq_len = p->max_seq_len;
  f.seq_offsets = p->seq_offsets;
  f.num_targets = p->num_targets;
  f.contextual_len = p->contextual_len;
  f.K1 = p->K1;
  f.K2 = p->K2;
  f.alpha = p->alpha;
  f.N = p->N;
  const bf16* u = static_cast<const bf16*>(p->uvqk);
  f.q = u + 2 * dm;
  f.k = u + 3 * dm;
  f.v = u + dm;
  f.q_row_stride = f.k_row_stride = f.v_row_stride = 4 * dm;
  f.out = p->av;
  f.out_row_stride = dm;
  return f;
}

// split-K factor of a weight-gradient GEMM (M x N output, K = tokens): about
// two tiles per SM, each split at least 8 blocks of 64 tokens.
int wgrad_splits(int M, int N, int64_t T) {
  const int tiles = (M / 128) * (N / 256);
  const int64_t kb = (T + 63) / 64;
  int s = (2 * device_sm_count() + tiles - 1) / tiles;
  if ((int64_t)s * 8 > kb) s = (int)(kb / 8);
  return s < 1 ? 1 : s;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? HSTU_SLA_OK : HSTU_SLA_ERR_CUDA; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

// FP8 forward scratch after the attention's workspace: E4M3 rows [T][d_model]
// (x^, then y) and their per-row scales [T].
size_t fp8_scratch_bytes(int64_t T, int dm) {
  return round256((size_t)T * dm) + round256((size_t)T * sizeof(float));
}

// Rematerialisation scratch after the attention's workspace: x^ [T][dm],
// pre and U|V|Q|K [T][4 dm] (bf16), y [T][dm], and the recomputed norms'
// statistics [4][T] (fp32; equal to the saved ones).
size_t remat_scratch_bytes(int64_t T, int dm) {
  const size_t r = (size_t)T * dm * sizeof(bf16);
  return 2 * round256(r) + 2 * round256(4 * r) + round256((size_t)4 * T * sizeof(float));
}

// Points x^, pre, uvqk, y and stats of `r` at the scratch.  `stats` stays
// the caller's unless `own_stats` (the backward's recomputation writes its
// statistics to the scratch, the saved ones are what the gradients read).
void carve_remat(hstu_stu_layer_params* r, void* scratch, float** recomputed_stats) {
  const int64_t T = r->total_tokens;
  const int dm = r->H * r->d;
  const size_t row = (size_t)T * dm * sizeof(bf16);
  char* c = static_cast<char*>(scratch);
  r->xn = c;
  c += round256(row);
  r->pre = c;
  c += round256(4 * row);
  r->uvqk = c;
  c += round256(4 * row);
  r->y = c;
  c += round256(row);
  *recomputed_stats = reinterpret_cast<float*>(c);
}

}  // namespace

extern "C" {

size_t hstu_stu_workspace_bytes(int which, int64_t total_tokens, int32_t B, int32_t H, int32_t d) {
  const bool f8 = which == HSTU_STU_WS_FWD_FP8;
  const bool rf = which == HSTU_STU_WS_FWD_REMAT, rb = which == HSTU_STU_WS_BWD_REMAT;
  const int attn = (f8 || rf) ? HSTU_SLA_WS_FWD : rb ? HSTU_SLA_WS_BWD : which;
  const size_t a = hstu_sla_workspace_bytes(attn, total_tokens, B, H, d);
  if (a == 0) return 0;
  return kHdr + round256(a) + (f8 ? fp8_scratch_bytes(total_tokens, H * d) : 0) +
         ((rf || rb) ? remat_scratch_bytes(total_tokens, H * d) : 0);
}

int hstu_stu_layer_fwd(const hstu_stu_layer_params* p, void* workspace, size_t workspace_bytes,
                       hstu_stream_t stream) {
  int e = check_layer(p, true);
  if (e) return e;
  const bool f8 = p->fp8 != 0;
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_stu_workspace_bytes(f8 ? HSTU_STU_WS_FWD_FP8
                                                : p->remat ? HSTU_STU_WS_FWD_REMAT
                                                           : HSTU_SLA_WS_FWD,
                                             p->total_tokens, p->B, p->H, p->d))))
    return e;
  // Listing 1's save set: x^, pre, U|V|Q|K and y go to scratch; U is copied
  // out for the backward at the end
  hstu_stu_layer_params remat_p;
  const hstu_stu_layer_params* caller = p;
  if (p->remat) {
    remat_p = *p;
    float* unused_stats = nullptr;
    carve_remat(&remat_p, static_cast<char*>(workspace) + kHdr +
                              round256(hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, p->total_tokens,
                                                                p->B, p->H, p->d)),
                &unused_stats);
    p = &remat_p;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* gh = static_cast<WsHeader*>(workspace);
  void* aws = static_cast<char*>(workspace) + kHdr;
  const int64_t T = p->total_tokens;
  const int dm = p->H * p->d;
  const size_t aws_bytes = hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, T, p->B, p->H, p->d);
  uint8_t* q8 = f8 ? static_cast<uint8_t*>(aws) + aws_bytes : nullptr;  // E4M3 rows
  float* q8s = f8 ? reinterpret_cast<float*>(q8 + round256((size_t)T * dm)) : nullptr;
  cudaError_t ce = cudaMemsetAsync(gh, 0, sizeof(WsHeader), st);
  if (ce != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  // x^ = LayerNorm(x)
  LnArgs l1;
  memset(&l1, 0, sizeof(l1));
  l1.T = T;
  l1.W = dm;
  l1.eps = p->ln_eps;
  l1.x = static_cast<const bf16*>(p->x);
  l1.ldx = dm;
  l1.gamma = p->ln1_w;
  l1.beta = p->ln1_b;
  l1.y = static_cast<bf16*>(p->xn);
  l1.ldy = dm;
  l1.mean = p->stats;
  l1.rstd = p->stats + T;
  l1.yq = q8;
  l1.ldyq = dm;
  l1.yscale = q8s;
  if ((ce = launch_ln_fwd(l1, false, st)) != cudaSuccess) return status_of(ce);
  // pre = x^ W1 + b1, UVQK = SiLU(pre)
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = (int)T;
  g.N = 4 * dm;
  g.K = dm;
  g.bias = p->b1;
  g.out = static_cast<bf16*>(p->uvqk);
  g.ldo = 4 * dm;
  g.out2 = static_cast<bf16*>(p->pre);
  g.ldo2 = 4 * dm;
  g.ws = gh;
  if (f8) {
    g.sa = q8s;
    g.sb = p->w1s;
    ce = launch_gemm({q8, dm, false, true}, {p->w1q, dm, false, true}, g, kEpiBiasSilu, st);
  } else {
    ce = launch_gemm({p->xn, dm, false}, {p->w1, 4 * dm, true}, g, kEpiBiasSilu, st);
  }
  if (ce != cudaSuccess) return status_of(ce);
  // A = SLA attention (Q, K, V)
  hstu_sla_fwd_params f = attn_params(p);
  if ((e = hstu_sla_fwd(&f, aws, workspace_bytes - kHdr, stream))) return e;
  // y = LayerNorm(A) * U
  LnArgs l2 = l1;
  l2.x = static_cast<const bf16*>(p->av);
  l2.u = static_cast<const bf16*>(p->uvqk);
  l2.ldu = 4 * dm;
  l2.gamma = p->ln2_w;
  l2.beta = p->ln2_b;
  l2.y = static_cast<bf16*>(p->y);
  l2.mean = p->stats + 2 * T;
  l2.rstd = p->stats + 3 * T;
  if ((ce = launch_ln_fwd(l2, true, st)) != cudaSuccess) return status_of(ce);
  // out = y W2 + b2 + x
  GemmArgs g2;
  memset(&g2, 0, sizeof(g2));
  g2.M = (int)T;
  g2.N = dm;
  g2.K = dm;
  g2.bias = p->b2;
  g2.resid = static_cast<const bf16*>(p->x);
  g2.ldr = dm;
  g2.out = static_cast<bf16*>(p->out);
  g2.ldo = dm;
  g2.ws = gh;
  if (f8) {
    g2.sa = q8s;
    g2.sb = p->w2s;
    ce = launch_gemm({q8, dm, false, true}, {p->w2q, dm, false, true}, g2, kEpiBiasResid, st);
  } else {
    ce = launch_gemm({p->y, dm, false}, {p->w2, dm, true}, g2, kEpiBiasResid, st);
  }
  if (ce == cudaSuccess && caller->remat && T > 0)  // the saved u: block 0 of U|V|Q|K
    ce = cudaMemcpy2DAsync(caller->u, (size_t)dm * sizeof(bf16), p->uvqk,
                           (size_t)4 * dm * sizeof(bf16), (size_t)dm * sizeof(bf16), (size_t)T,
                           cudaMemcpyDeviceToDevice, st);
  return status_of(ce);
}

int hstu_stu_layer_bwd(const hstu_stu_layer_bwd_params* p, void* workspace,
                       size_t workspace_bytes, hstu_stream_t stream) {
  if (p == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  const hstu_stu_layer_params* f = &p->fwd;
  int e = check_layer(f, false);
  if (e) return e;
  const void* ptrs[] = {p->dout,    p->dx,      p->dy,   p->dav,  p->dpre,    p->dxn,
                        p->d_ln1_w, p->d_ln1_b, p->d_w1, p->d_b1, p->d_ln2_w, p->d_ln2_b,
                        p->d_w2,    p->d_b2};
  for (const void* q : ptrs)
    if (!al16(q)) return HSTU_SLA_ERR_INVALID_ARG;
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_stu_workspace_bytes(f->remat ? HSTU_STU_WS_BWD_REMAT : HSTU_SLA_WS_BWD,
                                             f->total_tokens, f->B, f->H, f->d))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* gh = static_cast<WsHeader*>(workspace);
  void* aws = static_cast<char*>(workspace) + kHdr;
  const int64_t T = f->total_tokens;
  const int dm = f->H * f->d;
  const bf16* dout = static_cast<const bf16*>(p->dout);
  bf16* dpre = static_cast<bf16*>(p->dpre);
  cudaError_t ce = cudaMemsetAsync(gh, 0, sizeof(WsHeader), st);
  hstu_stu_layer_params remat_f;
  if (f->remat && ce == cudaSuccess) {
    // Listing 1: recompute x^ = LayerNorm(x), pre and U|V|Q|K = SiLU(x^ W1 +
    // b1) by the forward's own kernels (the same bits), and y = LayerNorm(av)
    // * u, into the scratch; the gradients below then read them as saved.
    // The recomputed statistics go to the scratch too (equal to the saved).
    remat_f = *f;
    float* rstats = nullptr;
    carve_remat(&remat_f, static_cast<char*>(workspace) + kHdr +
                              round256(hstu_sla_workspace_bytes(HSTU_SLA_WS_BWD, T, f->B, f->H,
                                                                f->d)),
                &rstats);
    LnArgs r1;
    memset(&r1, 0, sizeof(r1));
    r1.T = T;
    r1.W = dm;
    r1.eps = f->ln_eps;
    r1.x = static_cast<const bf16*>(f->x);
    r1.ldx = dm;
    r1.gamma = f->ln1_w;
    r1.beta = f->ln1_b;
    r1.y = static_cast<bf16*>(remat_f.xn);
    r1.ldy = dm;
    r1.mean = rstats;
    r1.rstd = rstats + T;
    ce = launch_ln_fwd(r1, false, st);
    GemmArgs rg;
    memset(&rg, 0, sizeof(rg));
    rg.M = (int)T;
    rg.N = 4 * dm;
    rg.K = dm;
    rg.bias = f->b1;
    rg.out = static_cast<bf16*>(remat_f.uvqk);
    rg.ldo = 4 * dm;
    rg.out2 = static_cast<bf16*>(remat_f.pre);
    rg.ldo2 = 4 * dm;
    rg.ws = gh;
    if (ce == cudaSuccess)
      ce = launch_gemm({remat_f.xn, dm, false}, {f->w1, 4 * dm, true}, rg, kEpiBiasSilu, st);
    LnArgs r2 = r1;
    r2.x = static_cast<const bf16*>(f->av);
    r2.u = static_cast<const bf16*>(f->u);
    r2.ldu = dm;
    r2.gamma = f->ln2_w;
    r2.beta = f->ln2_b;
    r2.y = static_cast<bf16*>(remat_f.y);
    r2.mean = rstats + 2 * T;
    r2.rstd = rstats + 3 * T;
    if (ce == cudaSuccess) ce = launch_ln_fwd(r2, true, st);
    f = &remat_f;
  }
  const struct { float* p; size_t n; } grads[] = {
      {p->d_ln1_w, (size_t)dm}, {p->d_ln1_b, (size_t)dm}, {p->d_w1, (size_t)dm * 4 * dm},
      {p->d_b1, (size_t)4 * dm}, {p->d_ln2_w, (size_t)dm}, {p->d_ln2_b, (size_t)dm},
      {p->d_w2, (size_t)dm * dm}, {p->d_b2, (size_t)dm}};
  for (const auto& gr : grads)
    if (ce == cudaSuccess) ce = cudaMemsetAsync(gr.p, 0, gr.n * sizeof(float), st);
  if (ce != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  // d b2 = colsum(dout);  d W2 = y^T dout
  if ((ce = launch_colsum(dout, dm, T, dm, p->d_b2, st)) != cudaSuccess) return status_of(ce);
  GemmArgs gw;
  memset(&gw, 0, sizeof(gw));
  gw.M = dm;
  gw.N = dm;
  gw.K = (int)T;
  gw.splits = wgrad_splits(dm, dm, T);
  gw.outf = p->d_w2;
  gw.ldf = dm;
  gw.ws = gh;
  if ((ce = launch_gemm({f->y, dm, true}, {p->dout, dm, true}, gw, kEpiRedF32, st)) !=
      cudaSuccess)
    return status_of(ce);
  // dy = dout W2^T
  GemmArgs gd;
  memset(&gd, 0, sizeof(gd));
  gd.M = (int)T;
  gd.N = dm;
  gd.K = dm;
  gd.out = static_cast<bf16*>(p->dy);
  gd.ldo = dm;
  gd.ws = gh;
  if ((ce = launch_gemm({p->dout, dm, false}, {f->w2, dm, false}, gd, kEpiStore, st)) !=
      cudaSuccess)
    return status_of(ce);
  // gated norm: dA, dU (times SiLU'(pre_U), into the U block of dpre), d ln2
  LnArgs l2;
  memset(&l2, 0, sizeof(l2));
  l2.T = T;
  l2.W = dm;
  l2.eps = f->ln_eps;
  l2.x = static_cast<const bf16*>(f->av);
  l2.ldx = dm;
  l2.u = static_cast<const bf16*>(f->uvqk);
  l2.ldu = 4 * dm;
  l2.gamma = f->ln2_w;
  l2.beta = f->ln2_b;
  l2.mean = f->stats + 2 * T;
  l2.rstd = f->stats + 3 * T;
  l2.dy = static_cast<const bf16*>(p->dy);
  l2.lddy = dm;
  l2.dx = static_cast<bf16*>(p->dav);
  l2.lddx = dm;
  l2.du = dpre;
  l2.lddu = 4 * dm;
  l2.pre_u = static_cast<const bf16*>(f->pre);
  l2.ldpu = 4 * dm;
  l2.dgamma = p->d_ln2_w;
  l2.dbeta = p->d_ln2_b;
  // d = 128 with an even number of heads up to 8: the attention backward's
  // last pass applies SiLU' to dQ, dK, dV and sums their bias gradients, the
  // gated norm sums dU's; no separate pass over dpre
  const bool fused = f->d == 128 && (f->H * 16) % 32 == 0 && 3 * f->H * 16 <= 384;
  if (fused) l2.dbias_u = p->d_b1;
  if ((ce = launch_ln_bwd(l2, true, st)) != cudaSuccess) return status_of(ce);
  // attention backward: dQ, dK, dV into blocks 2, 3, 1 of dpre
  hstu_sla_bwd_params ab;
  memset(&ab, 0, sizeof(ab));
  ab.fwd = attn_params(f);
  ab.dout = p->dav;
  ab.dout_row_stride = dm;
  ab.dq = dpre + 2 * dm;
  ab.dk = dpre + 3 * dm;
  ab.dv = dpre + dm;
  ab.dq_row_stride = ab.dk_row_stride = ab.dv_row_stride = 4 * dm;
  const bf16* pre = static_cast<const bf16*>(f->pre);
  if (fused) {
    const SiluFusion fz = {pre + 2 * dm, pre + 3 * dm, pre + dm, 4 * dm,
                           p->d_b1 + 2 * dm, p->d_b1 + 3 * dm, p->d_b1 + dm};
    if ((e = sla_bwd(&ab, aws, workspace_bytes - kHdr, st, &fz))) return e;
  } else {
    if ((e = hstu_sla_bwd(&ab, aws, workspace_bytes - kHdr, stream))) return e;
    // SiLU' on the V, Q, K blocks (U is done), d b1 = colsum(dpre)
    if ((ce = launch_silu_bwd_colsum(dpre, 4 * dm, pre, 4 * dm, T, 4 * dm, dm, p->d_b1, st)) !=
        cudaSuccess)
      return status_of(ce);
  }
  // d W1 = x^T dpre
  GemmArgs gw1 = gw;
  gw1.N = 4 * dm;
  gw1.splits = wgrad_splits(dm, 4 * dm, T);
  gw1.outf = p->d_w1;
  gw1.ldf = 4 * dm;
  if ((ce = launch_gemm({f->xn, dm, true}, {p->dpre, 4 * dm, true}, gw1, kEpiRedF32, st)) !=
      cudaSuccess)
    return status_of(ce);
  // d x^ = dpre W1^T
  GemmArgs gx = gd;
  gx.K = 4 * dm;
  gx.out = static_cast<bf16*>(p->dxn);
  if ((ce = launch_gemm({p->dpre, 4 * dm, false}, {f->w1, 4 * dm, false}, gx, kEpiStore, st)) !=
      cudaSuccess)
    return status_of(ce);
  // dx = dout + LayerNorm'(d x^)
  LnArgs l1;
  memset(&l1, 0, sizeof(l1));
  l1.T = T;
  l1.W = dm;
  l1.eps = f->ln_eps;
  l1.x = static_cast<const bf16*>(f->x);
  l1.ldx = dm;
  l1.gamma = f->ln1_w;
  l1.beta = f->ln1_b;
  l1.mean = f->stats;
  l1.rstd = f->stats + T;
  l1.dy = static_cast<const bf16*>(p->dxn);
  l1.lddy = dm;
  l1.resid_grad = dout;
  l1.ldr = dm;
  l1.dx = static_cast<bf16*>(p->dx);
  l1.lddx = dm;
  l1.dgamma = p->d_ln1_w;
  l1.dbeta = p->d_ln1_b;
  ce = launch_ln_bwd(l1, false, st);
  return status_of(ce);
}

int hstu_stu_get_error(const void* workspace, hstu_stream_t stream) {
  if (workspace == nullptr) return HSTU_SLA_ERR_WORKSPACE;
  const int g = hstu_sla_get_error(workspace, stream);
  if (g != HSTU_SLA_OK) return g;
  return hstu_sla_get_error(static_cast<const char*>(workspace) + kHdr, stream);
}

int hstu_jagged_truncate_offsets(const int32_t* seq_offsets, const int32_t* num_targets, int32_t B,
                                 int32_t contextual_len, int32_t tail, int32_t* new_offsets,
                                 hstu_stream_t stream) {
  if (seq_offsets == nullptr || new_offsets == nullptr || B < 1 || contextual_len < 0 || tail < 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  return status_of(launch_trunc_offsets(seq_offsets, num_targets, B, contextual_len, tail,
                                        new_offsets, reinterpret_cast<cudaStream_t>(stream)));
}

int64_t hstu_jagged_truncate_lengths(const int32_t* lengths, const int32_t* num_targets,
                                     int32_t B, int32_t contextual_len, int32_t tail,
                                     int32_t* new_lengths) {
  if (lengths == nullptr || B < 1 || contextual_len < 0 || tail < 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int b = 0; b < B; ++b) {
    const int nt = num_targets ? num_targets[b] : 0;
    if (lengths[b] < 0 || nt < 0 || nt > lengths[b]) return HSTU_SLA_ERR_INVALID_ARG;
  }
  for (int b = 0; b < B; ++b) {
    const int nt = num_targets ? num_targets[b] : 0;
    const int kept = lengths[b] - hstu::trunc_drop(lengths[b], nt, contextual_len, tail);
    if (new_lengths) new_lengths[b] = kept;
    total += kept;
  }
  return total;
}

int hstu_jagged_truncate(const void* src, int64_t src_row_stride, const int32_t* seq_offsets,
                         const int32_t* new_offsets, const int32_t* num_targets, int32_t B,
                         int32_t contextual_len, int32_t tail, int32_t width, void* dst,
                         int64_t dst_row_stride, int64_t T_out, int32_t scatter,
                         hstu_stream_t stream) {
  if (!al16(src) || !al16(dst) || seq_offsets == nullptr || new_offsets == nullptr || B < 1 ||
      contextual_len < 0 || tail < 0 || width <= 0 || width % 8 != 0 || T_out < 0 ||
      src_row_stride < width || dst_row_stride < width || src_row_stride % 8 != 0 ||
      dst_row_stride % 8 != 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  return status_of(launch_trunc_rows(static_cast<const bf16*>(src), src_row_stride, seq_offsets,
                                     new_offsets, num_targets, B, contextual_len, tail, width,
                                     static_cast<bf16*>(dst), dst_row_stride, T_out, scatter != 0,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int hstu_gemm(const hstu_gemm_params* p, void* workspace, hstu_stream_t stream) {
  if (p == nullptr || workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return HSTU_SLA_ERR_INVALID_ARG;
  if (p->M < 0 || p->N < 0 || p->K < 1 || p->N % 256 != 0 || p->epilogue < 0 ||
      p->epilogue > HSTU_GEMM_RED_F32 || !al16(p->a) || !al16(p->b) || p->lda % 8 != 0 ||
      p->ldb % 8 != 0 || (p->fp8 != 0 && p->fp8 != 1))
    return HSTU_SLA_ERR_INVALID_ARG;
  const bool f8 = p->fp8 != 0;
  if (f8 && (p->lda % 16 != 0 || p->ldb % 16 != 0 || !al16(p->a_scale) || !al16(p->b_scale)))
    return HSTU_SLA_ERR_INVALID_ARG;
  if (f8 && (p->a_mn_major || p->b_mn_major || p->epilogue == HSTU_GEMM_RED_F32))
    return HSTU_SLA_ERR_UNSUPPORTED;
  const bool red = p->epilogue == HSTU_GEMM_RED_F32;
  if (red ? !al16(p->outf) || p->ldf % 4 != 0 : !al16(p->out) || p->ldo % 8 != 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  if ((p->epilogue == HSTU_GEMM_BIAS_SILU || p->epilogue == HSTU_GEMM_BIAS_RESID) && !al16(p->bias))
    return HSTU_SLA_ERR_INVALID_ARG;
  if (p->epilogue == HSTU_GEMM_BIAS_SILU && (!al16(p->out2) || p->ldo2 % 8 != 0))
    return HSTU_SLA_ERR_INVALID_ARG;
  if (p->epilogue == HSTU_GEMM_BIAS_RESID && (!al16(p->resid) || p->ldr % 8 != 0))
    return HSTU_SLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = p->M;
  g.N = p->N;
  g.K = p->K;
  g.splits = p->splits;
  g.bias = p->bias;
  g.resid = static_cast<const bf16*>(p->resid);
  g.ldr = p->ldr;
  g.out = static_cast<bf16*>(p->out);
  g.ldo = p->ldo;
  g.out2 = static_cast<bf16*>(p->out2);
  g.ldo2 = p->ldo2;
  g.outf = p->outf;
  g.ldf = p->ldf;
  g.ws = static_cast<WsHeader*>(workspace);
  g.sa = p->a_scale;
  g.sb = p->b_scale;
  cudaError_t ce = cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st);
  if (ce == cudaSuccess)
    ce = launch_gemm({p->a, p->lda, p->a_mn_major != 0, f8},
                     {p->b, p->ldb, p->b_mn_major != 0, f8}, g, p->epilogue, st);
  if (ce == cudaErrorNotSupported) return HSTU_SLA_ERR_UNSUPPORTED;
  return status_of(ce);
}

int hstu_quant_weight_e4m3(const void* w, int64_t ldw, int32_t K, int32_t N, void* wq,
                           int64_t ldq, float* scale, hstu_stream_t stream) {
  if (!al16(w) || !al16(wq) || !al16(scale) || K < 0 || N < 0 || ldw < N || ldq < K)
    return HSTU_SLA_ERR_INVALID_ARG;
  if (K % 64 != 0 || N % 64 != 0 || ldq % 16 != 0) return HSTU_SLA_ERR_UNSUPPORTED;
  cudaError_t ce = launch_quant_wt(static_cast<const bf16*>(w), ldw, K, N,
                                   static_cast<uint8_t*>(wq), ldq, scale,
                                   reinterpret_cast<cudaStream_t>(stream));
  return status_of(ce);
}

}  // extern "C"
