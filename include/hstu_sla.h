/*
 * hstu_sla.h -- C ABI of the B200 (sm_100a) SLA HSTU attention library.
 *
 * The operation is HSTU's pointwise-SiLU attention ("Bending the Scaling Law
 * Curve in Large-Scale Recommendation Systems", section 3, Eq. 3; HSTU notes
 * "Actions Speak Louder than Words", section 2.4, Eq. 2) under the
 * Semi-Local Attention mask (same paper, section 4.2.1, Eq. 7), over a jagged
 * batch.  Per sequence b of length L (contextual prefix first, num_targets
 * candidates last, Lh = L - num_targets history tokens) and per head:
 *
 *     out_i = (1/N) * sum_j M(i,j) * SiLU(alpha * q_i . k_j) * v_j
 *
 * with K2eff = max(K2, contextual_len) (TorchEasyRec "ULTRA HSTU" docs,
 * Semi-Local Attention bullet) and 0-based positions i, j in the sequence:
 *     history row i < Lh:   M = [j <= i] and ([i - j < K1] or [j < K2eff])
 *     candidate row i >= Lh: M = ([j < Lh] and ([Lh - j < K1] or [j < K2eff]))
 *                                or [j == i]
 * (candidates see the history and themselves, never each other: HSTU notes,
 * section 2.6, M-FALCON mask figure).  K1 and K2 are taken literally: K1 = 0
 * means no local window; "full causal" is K1 >= max length.
 *
 * The backward produces dq, dk, dv of  L = sum(out * dout)  (the attention
 * step of Listing 1's attention_backward(dattn, q, k, v)).
 *
 * Conventions for every entry point:
 *  - Pointers named "device" are CUDA device pointers; the caller owns every
 *    buffer (the library allocates nothing and keeps no state between calls).
 *  - Tensors are bf16 [T, H, d] with the H*d values of one token contiguous
 *    (head h at element offset h*d) and a per-token row stride in ELEMENTS,
 *    so q/k/v may be strided views into a fused projection buffer.  Row
 *    strides must be multiples of 8 elements and base pointers 16-byte
 *    aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  They return HSTU_SLA_OK or a negative code; no C++
 *    exception crosses the ABI.  Argument errors are detected on the host and
 *    nothing is launched.  Errors in the device-resident offsets/targets are
 *    detected on the device: the kernels then skip all work and the error is
 *    reported by hstu_sla_get_error().  Kernels never trap.
 *  - Supported head_dim d: 32, 64, 128.  max_seq_len bounds every length.
 */
#ifndef HSTU_SLA_H_
#define HSTU_SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* hstu_stream_t; /* identical to cudaStream_t */

enum {
  HSTU_SLA_OK = 0,
  HSTU_SLA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misalignment */
  HSTU_SLA_ERR_UNSUPPORTED = -2,  /* head_dim or device not supported */
  HSTU_SLA_ERR_CUDA = -3,         /* a CUDA runtime call failed */
  HSTU_SLA_ERR_BAD_INPUT = -4,    /* device-side check of offsets/targets failed */
  HSTU_SLA_ERR_WORKSPACE = -5,    /* workspace missing, too small or misaligned */
  HSTU_SLA_ERR_TIMEOUT = -6       /* a bounded device-side wait gave up */
};

/* Forward problem.  All integer fields are host values. */
typedef struct {
  int32_t B;                    /* number of sequences, >= 1 */
  int32_t H;                    /* heads, >= 1 */
  int32_t d;                    /* head_dim: 32, 64 or 128 */
  int64_t total_tokens;         /* T = seq_offsets[B] (host copy, for sizing) */
  int32_t max_seq_len;          /* >= every sequence length (device-checked) */
  const int32_t* seq_offsets;   /* device [B+1], offsets[0] = 0, non-decreasing */
  const int32_t* num_targets;   /* device [B], 0 <= num_targets[b] <= len_b; NULL = all 0 */
  int32_t contextual_len;       /* >= 0; K2eff = max(K2, contextual_len) */
  int32_t K1;                   /* local window (keys incl. self), >= 0 */
  int32_t K2;                   /* global prefix, >= 0 */
  float alpha;                  /* scale inside SiLU */
  float N;                      /* normaliser, > 0 */
  const void* q;                /* device bf16 [T, H, d]; the tensors may be NULL when T = 0 */
  const void* k;
  const void* v;
  int64_t q_row_stride;         /* elements between consecutive tokens (>= H*d) */
  int64_t k_row_stride;
  int64_t v_row_stride;
  void* out;                    /* device bf16 [T, H, d], written by hstu_sla_fwd */
  int64_t out_row_stride;
  /* Optional timing hooks: cudaEvent_t handles recorded on `stream` just
   * before and just after the main attention kernel (not the work-list or
   * conversion kernels).  NULL = not recorded. */
  void* event_begin;
  void* event_end;
  /* M-FALCON candidate scoring (HSTU notes, section 2.6): non-zero computes
   * only the query tiles that hold candidates (rows >= L - num_targets of
   * each sequence), reading every key's k and v (the cached history and the
   * candidates); out rows of other tiles are left untouched.  The rows of
   * the first candidate tile that precede the candidates are history rows
   * and are written too (with their correct values).  Ignored by the
   * backward. */
  int32_t candidates_only;
  /* Relative attention bias (optional; HSTU notes "Actions Speak Louder than
   * Words", section 2.4, Eq. 2, phi2(Q K^T + rab^{p,t})):
   *   x_ij = alpha q_i.k_j + rab_pos[h][bucket(dpos)] + rab_time[h][bucket(dt)]
   * with bucket(n) = min(floor(log2(n + 1)), buckets - 1), dpos = i - j for
   * a history row, Lh - j for a candidate row (0 to itself), and
   * dt = |timestamps[i] - timestamps[j]|.  A NULL table adds nothing;
   * rab_time needs timestamps.  Each table has 1..32 buckets per head.  The
   * backward needs d = 128.  In a grouped call each group has its own
   * tables and timestamps, or none. */
  const int32_t* timestamps;    /* device [T], any integer time unit, or NULL */
  const float* rab_pos;         /* device [H][rab_pos_buckets], or NULL */
  const float* rab_time;        /* device [H][rab_time_buckets], or NULL */
  int32_t rab_pos_buckets;
  int32_t rab_time_buckets;
} hstu_sla_fwd_params;

/* Backward problem: the forward problem plus dout and the three gradients. */
typedef struct {
  hstu_sla_fwd_params fwd;      /* fwd.out and fwd.out_row_stride are ignored */
  const void* dout;             /* device bf16 [T, H, d] */
  int64_t dout_row_stride;
  void* dq;                     /* device bf16 [T, H, d], written */
  void* dk;
  void* dv;
  int64_t dq_row_stride;
  int64_t dk_row_stride;
  int64_t dv_row_stride;
  /* With fwd.rab_pos / fwd.rab_time set: their gradients (device [H][buckets],
   * overwritten): d rab[h][b] = sum over visible pairs in bucket b of
   * dP_ij SiLU'(x_ij) / N.  Required for every table that is set. */
  float* d_rab_pos;
  float* d_rab_time;
  /* 1: hstu_sla_bwd_prepare already ran for this batch on this workspace
   * (work lists built, dQ accumulator cleared) and was ordered before this
   * call by the caller; the call then skips that work.  0: the call does it
   * itself. */
  int32_t prepared;
} hstu_sla_bwd_params;

#define HSTU_SLA_WS_FWD 0
#define HSTU_SLA_WS_BWD 1

/* Bytes of device workspace hstu_sla_fwd (which = HSTU_SLA_WS_FWD) or
 * hstu_sla_bwd (HSTU_SLA_WS_BWD) needs for a batch of total_tokens tokens in
 * B sequences: a status word and the device-built work lists, about
 * 16 * (total_tokens / 64 + B) bytes, plus, for the backward at d = 128, an
 * fp32 dQ accumulator of total_tokens * H * d * 4 bytes.  The workspace must
 * be 256-byte aligned; its contents need not be initialised.  Returns 0 on
 * invalid arguments. */
size_t hstu_sla_workspace_bytes(int which, int64_t total_tokens, int32_t B, int32_t H,
                                int32_t d);

/* Forward: writes p->out.  Enqueues a work-list kernel (validates offsets and
 * targets on the device, enumerates the non-empty query tiles) and the
 * attention kernel; nothing returns to the host. */
int hstu_sla_fwd(const hstu_sla_fwd_params* p, void* workspace, size_t workspace_bytes,
                 hstu_stream_t stream);

/* Backward: writes p->dq, p->dk, p->dv (bf16).  No atomics on dk/dv: each
 * key tile's dk/dv rows are accumulated on chip by one CTA.
 *  d = 128: one pass over key tiles.  Each (key tile, query tile) step also
 *           forms its dQ contribution on the tensor cores and adds it to the
 *           workspace's fp32 accumulator with fp32 atomic additions; a final
 *           kernel converts it to bf16 dq.  dk/dv are bitwise reproducible;
 *           dq is reproducible up to the order of fp32 additions.
 *  d = 32, 64: two passes, no atomics at all, bitwise reproducible: a
 *           key-tile pass for dk/dv and a query-tile pass that recomputes the
 *           scores for dq. */
int hstu_sla_bwd(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                 hstu_stream_t stream);

/* The part of hstu_sla_bwd that reads neither dout nor the forward's inputs:
 * the work lists of the batch (seq_offsets, num_targets, windows) and, for
 * head_dim 128, the clear of the fp32 dQ accumulator in `workspace`.  A
 * caller can issue it early on another stream, e.g. while the forward runs,
 * then call hstu_sla_bwd with p->prepared = 1 on its stream after an event
 * orders the two; the arguments and workspace must be the same, and nothing
 * may use the workspace in between.  Same validation and return codes as
 * hstu_sla_bwd; gradients and dout are not read. */
int hstu_sla_bwd_prepare(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                         hstu_stream_t stream);

/* Grouped calls: up to HSTU_SLA_MAX_GROUPS independent problems in ONE
 * launch of the attention kernel.  The use is the Mixture of Transducers
 * ("Bending the Scaling Law Curve in Large-Scale Recommendation Systems",
 * section 4.3; TorchEasyRec "ULTRA HSTU" docs, MoT): one transducer per
 * user-signal channel, each with its own sequences, SLA window (K1, K2,
 * contextual_len), N, alpha, heads and tensors.  The kernel's scheduler hands
 * out the units of all problems from one counter (the backward's prefix key
 * tiles of every problem first), so short channels fill the tail of long
 * ones.  Results equal G separate calls: the forward and dk / dv bitwise, dq
 * to fp32 summation order (as for one call).
 *   - groups[g] is read as for hstu_sla_fwd / hstu_sla_bwd; every group has
 *     the same d (the backward: d = 128).  candidates_only is per group.
 *   - workspace: hstu_sla_grouped_workspace_bytes(which, G, ...) bytes, 256-byte
 *     aligned: a 256-byte status header (read by hstu_sla_get_error; a
 *     device-side input error of any group is reported there), then each
 *     group's own workspace in the order given.
 *   - groups[0].event_begin / event_end (if set) bracket the attention kernel.
 *   - relative attention bias: per group, as for one call (the backward
 *     writes each group's d_rab_pos / d_rab_time).  If any group has a
 *     table, the launch runs the bias variant of the kernel for every group
 *     (a group without tables adds nothing but shares that kernel's cost).
 * Returns HSTU_SLA_ERR_INVALID_ARG for G outside [1, HSTU_SLA_MAX_GROUPS] or a
 * bad group (a backward group with a table but no gradient buffer for it),
 * HSTU_SLA_ERR_UNSUPPORTED for mixed d (or d != 128 backward). */
#define HSTU_SLA_MAX_GROUPS 4
size_t hstu_sla_grouped_workspace_bytes(int which, int32_t G, const int64_t* total_tokens,
                                        const int32_t* B, const int32_t* H, const int32_t* d);
int hstu_sla_fwd_grouped(const hstu_sla_fwd_params* groups, int32_t G, void* workspace,
                         size_t workspace_bytes, hstu_stream_t stream);
int hstu_sla_bwd_grouped(const hstu_sla_bwd_params* groups, int32_t G, void* workspace,
                         size_t workspace_bytes, hstu_stream_t stream);

/* Forward without a caller-provided workspace, for callers that may not
 * allocate device memory: inference engines and plugin hosts that plan all
 * device memory before running and forbid allocation inside their launch
 * path, and latency-critical loops that cannot afford cudaMalloc/cudaFree
 * (which may synchronise the device).  The cited papers have no counterpart: this is
 * an interface convenience, not part of the method.
 *
 * Same arguments, outputs and kernels as hstu_sla_fwd; the work lists and
 * status word go to a 2 MiB array in the library's own device memory, which
 * every GPU that loads the library keeps until the process exits.  Batches
 * need ceil(total_tokens / 64) + B <= 131,040 (about 8.3 million tokens);
 * larger ones return HSTU_SLA_ERR_WORKSPACE without launching anything.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress), so make that first call before any stream capture.
 *  - Every call on a device reuses the same array: calls that overlap on the
 *    GPU (other streams, other host threads) race and must be serialised by
 *    the caller.  Each call rewrites the status and work lists it reads, so
 *    nothing carries over from the previous call.
 *  - Device-detected input errors (corrupt seq_offsets / num_targets, a
 *    timed-out wait) leave out unwritten; hstu_sla_noalloc_get_error reads
 *    them.
 *  - The array's address is cached per device and context; after a device
 *    reset the next call looks it up again.
 * Allocates nothing: no cudaMalloc, no cudaFree. */
int hstu_sla_fwd_noalloc(const hstu_sla_fwd_params* p, hstu_stream_t stream);

/* Synchronises `stream` and returns the device-side status that the last
 * hstu_sla_fwd_noalloc call on the current device recorded in the library's
 * scratch array (HSTU_SLA_OK, HSTU_SLA_ERR_BAD_INPUT or HSTU_SLA_ERR_TIMEOUT),
 * or HSTU_SLA_ERR_CUDA.  Like the call itself, it reads the one shared array:
 * a call of another stream in between overwrites the status.  Allocates
 * nothing. */
int hstu_sla_noalloc_get_error(hstu_stream_t stream);

/* Test hook: the number of visible keys of every token as the forward
 * kernels enumerate them (row_counts, device int64 [T]) and the number of
 * query rows that see every token as a key, as the backward kernels
 * enumerate them (key_counts, device int64 [T]).  Either may be NULL.
 * Counts are per head (identical for all heads). */
int hstu_sla_count_pairs(const hstu_sla_fwd_params* p, int64_t* row_counts,
                         int64_t* key_counts, void* workspace, size_t workspace_bytes,
                         hstu_stream_t stream);

/* Synchronises `stream` and returns the device-side status recorded in
 * `workspace` by the last call that used it (HSTU_SLA_OK, HSTU_SLA_ERR_BAD_INPUT
 * or HSTU_SLA_ERR_TIMEOUT), or HSTU_SLA_ERR_CUDA.  The status is cleared by the
 * next hstu_sla_fwd / hstu_sla_bwd / hstu_sla_count_pairs call. */
int hstu_sla_get_error(const void* workspace, hstu_stream_t stream);

/* Test hook for the bounded-wait failure path (no counterpart in the cited
 * papers: it exists to show that a stalled kernel gives up instead of
 * hanging).  Runs the head_dim-128 forward (which = 0; p->fwd.out written) or
 * one-pass backward (which = 1) on the given inputs with a kernel
 * instantiation whose pointwise warps each withhold one hand-over arrive, so
 * the warp waiting for it runs into the limit: after wait_limit_ns (> 0)
 * the kernel records HSTU_SLA_ERR_TIMEOUT, every role stops, copies and
 * MMAs in flight drain, TMEM is released and the kernel returns.
 * hstu_sla_get_error(workspace) then reads HSTU_SLA_ERR_TIMEOUT; the outputs
 * are unspecified.  The production calls never take this instantiation, and
 * their limit stays 2 s.  Needs head_dim 128, no relative attention bias,
 * total_tokens > 0 (else HSTU_SLA_ERR_UNSUPPORTED); workspace as for the
 * chosen pass. */
int hstu_sla_test_wait_timeout(const hstu_sla_bwd_params* p, int32_t which,
                               int64_t wait_limit_ns, void* workspace, size_t workspace_bytes,
                               hstu_stream_t stream);

/* Static message for a status code. */
const char* hstu_sla_strerror(int code);

/* Library ABI version (major * 100 + minor). */
int hstu_sla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_SLA_H_ */
