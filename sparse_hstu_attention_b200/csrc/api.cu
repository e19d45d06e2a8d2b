// C ABI of the SLA HSTU attention library: host-side argument checks,
// workspace carving and kernel launches.  See include/hstu_sla.h.
#include <math.h>
#include <string.h>

#include "sla_common.cuh"

using namespace hstu;

namespace {

// 101: hstu_sla_fwd_params.candidates_only; 102: FP8 forward; 103: grouped calls;
// 104: relative attention bias
constexpr int kAbiVersion = 105;
static_assert(HSTU_SLA_MAX_GROUPS == kMaxGroups, "one grouped launch holds every group");

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_tensor(const void* p, int64_t rs, const hstu_sla_fwd_params* f) {
  if (p == nullptr && f->total_tokens == 0) return HSTU_SLA_OK;  // nothing is read or written
  if (p == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  if (!aligned16(p)) return HSTU_SLA_ERR_INVALID_ARG;
  if (rs < (int64_t)f->H * f->d || (rs % 8) != 0) return HSTU_SLA_ERR_INVALID_ARG;
  return HSTU_SLA_OK;
}

int check_common(const hstu_sla_fwd_params* f) {
  if (f == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  if (f->B < 1 || f->H < 1 || f->total_tokens < 0 || f->max_seq_len < 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  if (f->total_tokens > INT32_MAX) return HSTU_SLA_ERR_UNSUPPORTED;
  if (f->d != 32 && f->d != 64 && f->d != 128) return HSTU_SLA_ERR_UNSUPPORTED;
  if (f->K1 < 0 || f->K2 < 0 || f->contextual_len < 0) return HSTU_SLA_ERR_INVALID_ARG;
  if (!(f->N > 0.f) || !isfinite(f->N) || !isfinite(f->alpha)) return HSTU_SLA_ERR_INVALID_ARG;
  if (f->seq_offsets == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  if (f->rab_pos && (f->rab_pos_buckets < 1 || f->rab_pos_buckets > 32))
    return HSTU_SLA_ERR_INVALID_ARG;
  if (f->rab_time && (f->rab_time_buckets < 1 || f->rab_time_buckets > 32 || !f->timestamps))
    return HSTU_SLA_ERR_INVALID_ARG;
  int e;
  if ((e = check_tensor(f->q, f->q_row_stride, f))) return e;
  if ((e = check_tensor(f->k, f->k_row_stride, f))) return e;
  if ((e = check_tensor(f->v, f->v_row_stride, f))) return e;
  return HSTU_SLA_OK;
}

int check_ws(void* ws, size_t bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return HSTU_SLA_ERR_WORKSPACE;
  if (bytes < need) return HSTU_SLA_ERR_WORKSPACE;
  return HSTU_SLA_OK;
}

AttnArgs make_args(const hstu_sla_fwd_params* f, void* ws) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.offs = f->seq_offsets;
  a.nts = f->num_targets;
  a.ws = reinterpret_cast<WsHeader*>(ws);
  a.items = reinterpret_cast<const int2*>(static_cast<char*>(ws) + ws_items_offset());
  a.items2 = reinterpret_cast<const int2*>(static_cast<char*>(ws) +
                                           ws_items2_offset(f->total_tokens, f->B));
  a.B = f->B;
  a.H = f->H;
  a.K1 = f->K1;
  a.K2e = f->K2 > f->contextual_len ? f->K2 : f->contextual_len;
  a.max_seq_len = f->max_seq_len;
  a.T = f->total_tokens;
  a.alpha = f->alpha;
  a.inv_n = 1.0f / f->N;
  a.q = static_cast<const bf16*>(f->q);
  a.k = static_cast<const bf16*>(f->k);
  a.v = static_cast<const bf16*>(f->v);
  a.q_rs = f->q_row_stride;
  a.k_rs = f->k_row_stride;
  a.v_rs = f->v_row_stride;
  a.cand_only = f->candidates_only != 0;
  a.ts = f->timestamps;
  a.rab_pos = f->rab_pos;
  a.rab_time = f->rab_time;
  a.nbp = f->rab_pos ? f->rab_pos_buckets : 1;
  a.nbt = f->rab_time ? f->rab_time_buckets : 1;
  return a;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HSTU_SLA_OK : HSTU_SLA_ERR_CUDA; }

cudaError_t record(void* ev, cudaStream_t st) {
  return ev ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), st) : cudaSuccess;
}

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

// Launch order of a group's problems: larger windows (longer units) first.
void order_by_window(const hstu_sla_fwd_params* const* f, int G, int* order) {
  auto cost = [&](int g) {
    const int64_t m = f[g]->max_seq_len;
    const int64_t k2e = f[g]->K2 > f[g]->contextual_len ? f[g]->K2 : f[g]->contextual_len;
    return (f[g]->K1 < m ? f[g]->K1 : m) + (k2e < m ? k2e : m);
  };
  for (int g = 0; g < G; ++g) order[g] = g;
  for (int i = 1; i < G; ++i)  // insertion sort, stable
    for (int j = i; j > 0 && cost(order[j]) > cost(order[j - 1]); --j) {
      const int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
}

}  // namespace

extern "C" {

size_t hstu_sla_workspace_bytes(int which, int64_t total_tokens, int32_t B, int32_t H,
                                int32_t d) {
  if (total_tokens < 0 || B < 1 || H < 1 || d < 1) return 0;
  if (which == HSTU_SLA_WS_FWD) return ws_bytes(total_tokens, B);
  if (which == HSTU_SLA_WS_BWD) return ws_bwd_bytes(total_tokens, B, H, d);
  return 0;
}

int hstu_sla_fwd(const hstu_sla_fwd_params* p, void* workspace, size_t workspace_bytes,
                 hstu_stream_t stream) {
  int e = check_common(p);
  if (e) return e;
  if ((e = check_tensor(p->out, p->out_row_stride, p))) return e;
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, p->total_tokens, p->B, p->H, p->d))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a = make_args(p, workspace);
  a.out = static_cast<bf16*>(p->out);
  a.o_rs = p->out_row_stride;
  cudaError_t ce = launch_worklist(a, kFwdBM, 0, true, st);
  if (ce == cudaSuccess) ce = record(p->event_begin, st);
  if (ce == cudaSuccess) ce = launch_fwd_tc(a, p->d, st);
  if (ce == cudaSuccess) ce = record(p->event_end, st);
  return cuda_status(ce);
}

int hstu_sla_bwd(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                 hstu_stream_t stream) {
  return sla_bwd(p, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

int hstu_sla_bwd_prepare(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                         hstu_stream_t stream) {
  return sla_bwd_prepare(p, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t hstu_sla_grouped_workspace_bytes(int which, int32_t G, const int64_t* total_tokens,
                                        const int32_t* B, const int32_t* H, const int32_t* d) {
  if (G < 1 || G > HSTU_SLA_MAX_GROUPS || !total_tokens || !B || !H || !d) return 0;
  size_t n = sizeof(WsHeader);
  for (int g = 0; g < G; ++g) {
    const size_t b = hstu_sla_workspace_bytes(which, total_tokens[g], B[g], H[g], d[g]);
    if (b == 0) return 0;
    n += round256(b);
  }
  return n;
}

int hstu_sla_fwd_grouped(const hstu_sla_fwd_params* groups, int32_t G, void* workspace,
                         size_t workspace_bytes, hstu_stream_t stream) {
  if (groups == nullptr || G < 1 || G > HSTU_SLA_MAX_GROUPS) return HSTU_SLA_ERR_INVALID_ARG;
  int64_t T[HSTU_SLA_MAX_GROUPS];
  int32_t Bs[HSTU_SLA_MAX_GROUPS], Hs[HSTU_SLA_MAX_GROUPS], ds[HSTU_SLA_MAX_GROUPS];
  const hstu_sla_fwd_params* f[HSTU_SLA_MAX_GROUPS];
  int e;
  for (int g = 0; g < G; ++g) {
    f[g] = &groups[g];
    if ((e = check_common(f[g]))) return e;
    if ((e = check_tensor(f[g]->out, f[g]->out_row_stride, f[g]))) return e;
    if (f[g]->d != f[0]->d) return HSTU_SLA_ERR_UNSUPPORTED;
    T[g] = f[g]->total_tokens;
    Bs[g] = f[g]->B;
    Hs[g] = f[g]->H;
    ds[g] = f[g]->d;
  }
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_grouped_workspace_bytes(HSTU_SLA_WS_FWD, G, T, Bs, Hs, ds))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t ce = cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st);
  AttnArgs a[HSTU_SLA_MAX_GROUPS];
  char* w = static_cast<char*>(workspace) + sizeof(WsHeader);
  for (int g = 0; g < G && ce == cudaSuccess; ++g) {
    a[g] = make_args(f[g], w);
    a[g].out = static_cast<bf16*>(f[g]->out);
    a[g].o_rs = f[g]->out_row_stride;
    ce = launch_worklist(a[g], kFwdBM, 0, true, st);
    w += round256(hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, T[g], Bs[g], Hs[g], ds[g]));
  }
  int order[HSTU_SLA_MAX_GROUPS];
  order_by_window(f, G, order);
  GroupSet gs;
  memset(&gs, 0, sizeof(gs));
  for (int k = 0; k < G; ++k) gs.g[k] = a[order[k]];
  gs.common = static_cast<WsHeader*>(workspace);
  gs.G = G;
  if (ce == cudaSuccess) ce = record(f[0]->event_begin, st);
  if (ce == cudaSuccess) ce = launch_fwd_grouped(gs, f[0]->d, st);
  if (ce == cudaSuccess) ce = record(f[0]->event_end, st);
  return cuda_status(ce);
}

int hstu_sla_bwd_grouped(const hstu_sla_bwd_params* groups, int32_t G, void* workspace,
                         size_t workspace_bytes, hstu_stream_t stream) {
  if (groups == nullptr || G < 1 || G > HSTU_SLA_MAX_GROUPS) return HSTU_SLA_ERR_INVALID_ARG;
  int64_t T[HSTU_SLA_MAX_GROUPS];
  int32_t Bs[HSTU_SLA_MAX_GROUPS], Hs[HSTU_SLA_MAX_GROUPS], ds[HSTU_SLA_MAX_GROUPS];
  const hstu_sla_fwd_params* f[HSTU_SLA_MAX_GROUPS];
  int e;
  for (int g = 0; g < G; ++g) {
    const hstu_sla_bwd_params* p = &groups[g];
    f[g] = &p->fwd;
    if ((e = check_common(f[g]))) return e;
    if ((f[g]->rab_pos && !p->d_rab_pos) || (f[g]->rab_time && !p->d_rab_time))
      return HSTU_SLA_ERR_INVALID_ARG;
    if ((e = check_tensor(p->dout, p->dout_row_stride, f[g]))) return e;
    if ((e = check_tensor(p->dq, p->dq_row_stride, f[g]))) return e;
    if ((e = check_tensor(p->dk, p->dk_row_stride, f[g]))) return e;
    if ((e = check_tensor(p->dv, p->dv_row_stride, f[g]))) return e;
    if (f[g]->d != kFusedBwdD) return HSTU_SLA_ERR_UNSUPPORTED;
    T[g] = f[g]->total_tokens;
    Bs[g] = f[g]->B;
    Hs[g] = f[g]->H;
    ds[g] = f[g]->d;
  }
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_grouped_workspace_bytes(HSTU_SLA_WS_BWD, G, T, Bs, Hs, ds))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t ce = cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st);
  AttnArgs a[HSTU_SLA_MAX_GROUPS];
  char* w = static_cast<char*>(workspace) + sizeof(WsHeader);
  for (int g = 0; g < G && ce == cudaSuccess; ++g) {
    const hstu_sla_bwd_params* p = &groups[g];
    a[g] = make_args(f[g], w);
    a[g].cand_only = 0;
    a[g].dout = static_cast<const bf16*>(p->dout);
    a[g].dq = static_cast<bf16*>(p->dq);
    a[g].dk = static_cast<bf16*>(p->dk);
    a[g].dv = static_cast<bf16*>(p->dv);
    a[g].do_rs = p->dout_row_stride;
    a[g].dq_rs = p->dq_row_stride;
    a[g].dk_rs = p->dk_row_stride;
    a[g].dv_rs = p->dv_row_stride;
    a[g].dqacc = reinterpret_cast<float*>(w + ws_bytes(T[g], Bs[g]));
    a[g].d_rab_pos = f[g]->rab_pos ? p->d_rab_pos : nullptr;
    a[g].d_rab_time = f[g]->rab_time ? p->d_rab_time : nullptr;
    ce = launch_worklist(a[g], kKvBN, 1, true, st);
    w += round256(hstu_sla_workspace_bytes(HSTU_SLA_WS_BWD, T[g], Bs[g], Hs[g], ds[g]));
  }
  int order[HSTU_SLA_MAX_GROUPS];
  order_by_window(f, G, order);
  GroupSet gs;
  memset(&gs, 0, sizeof(gs));
  for (int k = 0; k < G; ++k) gs.g[k] = a[order[k]];
  gs.common = static_cast<WsHeader*>(workspace);
  gs.G = G;
  if (ce == cudaSuccess) ce = record(f[0]->event_begin, st);
  if (ce == cudaSuccess) ce = launch_bwd_fused_grouped(gs, st);
  if (ce == cudaSuccess) ce = record(f[0]->event_end, st);
  return cuda_status(ce);
}

int hstu_sla_count_pairs(const hstu_sla_fwd_params* p, int64_t* row_counts, int64_t* key_counts,
                         void* workspace, size_t workspace_bytes, hstu_stream_t stream) {
  int e = check_common(p);
  if (e) return e;
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_workspace_bytes(HSTU_SLA_WS_FWD, p->total_tokens, p->B, p->H, p->d))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a = make_args(p, workspace);
  cudaError_t ce = launch_worklist(a, kFwdBM, 0, true, st);
  if (ce == cudaSuccess)
    ce = launch_count_pairs(a, kFwdBM, kFwdBN, kKvBM, kKvBN, row_counts, key_counts, st);
  return cuda_status(ce);
}

int hstu_sla_get_error(const void* workspace, hstu_stream_t stream) {
  if (workspace == nullptr) return HSTU_SLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t status = 0;
  cudaError_t ce = cudaMemcpyAsync(&status, workspace, sizeof(status), cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  if (ce != cudaSuccess) return HSTU_SLA_ERR_CUDA;
  return status;
}

int hstu_sla_test_wait_timeout(const hstu_sla_bwd_params* p, int32_t which,
                               int64_t wait_limit_ns, void* workspace, size_t workspace_bytes,
                               hstu_stream_t stream) {
  if (p == nullptr || (which != 0 && which != 1) || wait_limit_ns <= 0)
    return HSTU_SLA_ERR_INVALID_ARG;
  const hstu_sla_fwd_params* f = &p->fwd;
  int e = check_common(f);
  if (e) return e;
  if (f->d != kFusedBwdD || f->rab_pos || f->rab_time || f->total_tokens == 0)
    return HSTU_SLA_ERR_UNSUPPORTED;
  if (which == 0) {
    if ((e = check_tensor(f->out, f->out_row_stride, f))) return e;
  } else {
    if ((e = check_tensor(p->dout, p->dout_row_stride, f))) return e;
    if ((e = check_tensor(p->dq, p->dq_row_stride, f))) return e;
    if ((e = check_tensor(p->dk, p->dk_row_stride, f))) return e;
    if ((e = check_tensor(p->dv, p->dv_row_stride, f))) return e;
  }
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_workspace_bytes(which ? HSTU_SLA_WS_BWD : HSTU_SLA_WS_FWD,
                                             f->total_tokens, f->B, f->H, f->d))))
    return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  AttnArgs a = make_args(f, workspace);
  a.wait_limit_ns = wait_limit_ns;
  GroupSet gs;
  memset(&gs, 0, sizeof(gs));
  gs.common = a.ws;
  gs.G = 1;
  gs.stall = 1;
  cudaError_t ce;
  if (which == 0) {
    a.out = static_cast<bf16*>(f->out);
    a.o_rs = f->out_row_stride;
    ce = launch_worklist(a, kFwdBM, 0, true, st);
    gs.g[0] = a;
    if (ce == cudaSuccess) ce = launch_fwd_grouped(gs, f->d, st);
  } else {
    a.cand_only = 0;
    a.dout = static_cast<const bf16*>(p->dout);
    a.dq = static_cast<bf16*>(p->dq);
    a.dk = static_cast<bf16*>(p->dk);
    a.dv = static_cast<bf16*>(p->dv);
    a.do_rs = p->dout_row_stride;
    a.dq_rs = p->dq_row_stride;
    a.dk_rs = p->dk_row_stride;
    a.dv_rs = p->dv_row_stride;
    a.dqacc = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                       ws_bytes(f->total_tokens, f->B));
    ce = launch_worklist(a, kKvBN, 1, true, st);
    gs.g[0] = a;
    if (ce == cudaSuccess) ce = launch_bwd_fused_grouped(gs, st);
  }
  return cuda_status(ce);
}

const char* hstu_sla_strerror(int code) {
  switch (code) {
    case HSTU_SLA_OK: return "ok";
    case HSTU_SLA_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or misalignment)";
    case HSTU_SLA_ERR_UNSUPPORTED: return "unsupported configuration (head_dim or device)";
    case HSTU_SLA_ERR_CUDA: return "CUDA runtime error";
    case HSTU_SLA_ERR_BAD_INPUT: return "invalid seq_offsets / num_targets detected on the device";
    case HSTU_SLA_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case HSTU_SLA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    default: return "unknown status";
  }
}

int hstu_sla_version(void) { return kAbiVersion; }

}  // extern "C"

namespace hstu {

// Validation and the launch arguments of a backward call (also used by its
// prepare step).
int bwd_args(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
             AttnArgs* out) {
  if (p == nullptr) return HSTU_SLA_ERR_INVALID_ARG;
  const hstu_sla_fwd_params* f = &p->fwd;
  int e = check_common(f);
  if (e) return e;
  if (p->prepared != 0 && p->prepared != 1) return HSTU_SLA_ERR_INVALID_ARG;
  if ((e = check_tensor(p->dout, p->dout_row_stride, f))) return e;
  if ((e = check_tensor(p->dq, p->dq_row_stride, f))) return e;
  if ((e = check_tensor(p->dk, p->dk_row_stride, f))) return e;
  if ((e = check_tensor(p->dv, p->dv_row_stride, f))) return e;
  if ((e = check_ws(workspace, workspace_bytes,
                    hstu_sla_workspace_bytes(HSTU_SLA_WS_BWD, f->total_tokens, f->B, f->H, f->d))))
    return e;
  AttnArgs a = make_args(f, workspace);
  a.cand_only = 0;  // the backward covers every row
  a.dout = static_cast<const bf16*>(p->dout);
  a.dq = static_cast<bf16*>(p->dq);
  a.dk = static_cast<bf16*>(p->dk);
  a.dv = static_cast<bf16*>(p->dv);
  a.do_rs = p->dout_row_stride;
  a.dq_rs = p->dq_row_stride;
  a.dk_rs = p->dk_row_stride;
  a.dv_rs = p->dv_row_stride;
  if (f->rab_pos || f->rab_time) {  // relative attention bias: one-pass kernel only
    if (f->d != kFusedBwdD) return HSTU_SLA_ERR_UNSUPPORTED;
    if ((f->rab_pos && !p->d_rab_pos) || (f->rab_time && !p->d_rab_time))
      return HSTU_SLA_ERR_INVALID_ARG;
    a.d_rab_pos = f->rab_pos ? p->d_rab_pos : nullptr;
    a.d_rab_time = f->rab_time ? p->d_rab_time : nullptr;
  }
  if (f->d == kFusedBwdD)  // the fp32 dQ workspace after the lists
    a.dqacc = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                       ws_bytes(f->total_tokens, f->B));
  *out = a;
  return HSTU_SLA_OK;
}

// Work lists (both passes' for head dims 32 / 64) and the clear of the dQ
// accumulator (head dim 128).
cudaError_t bwd_prepare(const AttnArgs& a, int d, cudaStream_t st) {
  if (d == kFusedBwdD) {
    cudaError_t ce = launch_worklist(a, kKvBN, 1, true, st);
    if (ce == cudaSuccess && a.T > 0)
      ce = cudaMemsetAsync(a.dqacc, 0, dq_workspace_bytes(a.T, a.H, d), st);
    return ce;
  }
  cudaError_t ce = launch_worklist(a, kQpBM, 0, true, st);
  if (ce == cudaSuccess) ce = launch_worklist(a, kKvBN, 1, false, st);
  return ce;
}

int sla_bwd_prepare(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                    cudaStream_t st) {
  AttnArgs a;
  const int e = bwd_args(p, workspace, workspace_bytes, &a);
  if (e) return e;
  return cuda_status(bwd_prepare(a, p->fwd.d, st));
}

int sla_bwd(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
            cudaStream_t st, const SiluFusion* fz) {
  AttnArgs a;
  int e = bwd_args(p, workspace, workspace_bytes, &a);
  if (e) return e;
  const hstu_sla_fwd_params* f = &p->fwd;
  cudaError_t ce;
  if (fz != nullptr) {  // the STU layer's SiLU' and bias-gradient fusion
    // silu_qkv_kernel: 3 H d / 8 threads, whole warps per block part
    const int ch = f->H * (f->d / 8);
    if (f->d != kFusedBwdD || ch % 32 != 0 || 3 * ch > 384) return HSTU_SLA_ERR_UNSUPPORTED;
    a.pre_q = fz->pre_q;
    a.pre_k = fz->pre_k;
    a.pre_v = fz->pre_v;
    a.pre_rs = fz->pre_rs;
    a.db_q = fz->db_q;
    a.db_k = fz->db_k;
    a.db_v = fz->db_v;
    a.db_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         ws_bytes(f->total_tokens, f->B) +
                                         dq_workspace_bytes(f->total_tokens, f->H, f->d));
  }
  // work lists (and the dQ clear), unless hstu_sla_bwd_prepare did them
  ce = p->prepared ? cudaSuccess : bwd_prepare(a, f->d, st);
  if (f->d == kFusedBwdD) {
    // one pass over key tiles; dQ through the fp32 workspace after the lists
    if (ce == cudaSuccess) ce = record(f->event_begin, st);
    if (ce == cudaSuccess) ce = launch_bwd_fused(a, st, /*cleared=*/true);
    if (ce == cudaSuccess) ce = record(f->event_end, st);
  } else {
    if (ce == cudaSuccess) ce = record(f->event_begin, st);
    if (ce == cudaSuccess) ce = launch_bwd_tc(a, f->d, /*kv_pass=*/true, st);
    if (ce == cudaSuccess) ce = launch_bwd_tc(a, f->d, /*kv_pass=*/false, st);
    if (ce == cudaSuccess) ce = record(f->event_end, st);
  }
  return cuda_status(ce);
}

}  // namespace hstu
