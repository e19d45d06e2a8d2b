/*
 * Oracle for HSTU pointwise-SiLU attention under the Semi-Local Attention
 * (SLA) mask over jagged batches.  TEST INFRASTRUCTURE ONLY: the tests, the
 * package smoke check and the benchmark's CPU-baseline leg may call it; the
 * product path never does.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Plain, slow, obviously correct: every output element is an explicit sum over
 * ALL key positions j of the sequence, gated by the mask predicate below, in
 * fp64.  Inputs are the bf16-rounded values widened to double.
 *
 * What it follows:
 *   - Attention:  A = (phi2(Q K^T) (.) M) V with phi2 = SiLU and no softmax
 *     ("Bending the Scaling Law Curve in Large-Scale Recommendation Systems",
 *     section 3, Eq. 3; HSTU notes "Actions Speak Louder than Words",
 *     section 2.4, Eq. 2).  A scale alpha sits inside the SiLU and the sum is
 *     divided by a normaliser N.
 *   - Mask: causal; key j kept if it is inside the local window of K1 tokens
 *     or inside the global prefix of K2eff tokens ("Bending the Scaling Law
 *     Curve...", section 4.2.1, Eq. 7), with K2eff = max(K2, contextual_len)
 *     (TorchEasyRec "ULTRA HSTU" docs, Semi-Local Attention bullet).
 *   - Candidates: the trailing num_targets rows see the history and
 *     themselves, never each other (HSTU notes, section 2.6 and the M-FALCON
 *     mask figure of Q8).
 *
 * Readings taken where the cited sources are garbled or silent (flags select the
 * alternatives, for tests only):
 *   - Eq. 7's index form is garbled; the window is read as i - j < K1
 *     (K1 tokens including self).  ORACLE_INCLUSIVE_WINDOW selects the
 *     literal "<=" (K1 + 1 tokens).
 *   - A candidate row applies the window at the clamped position Lh (the
 *     first position after the history), so every candidate sees the same
 *     history.  ORACLE_UNCLAMPED_TARGETS applies it at the row's own index.
 *   - K1 = 0: no local window at all; a history row past the prefix sees
 *     nothing, not even itself.  Candidates still see themselves.
 *
 * Backward: with x_ij = alpha q_i.k_j, P_ij = M_ij SiLU(x_ij)/N and
 * dP_ij = dO_i.v_j:  dV_j = sum_i P_ij dO_i;  dS_ij = M_ij dP_ij SiLU'(x_ij)
 * alpha/N;  dQ_i = sum_j dS_ij k_j;  dK_j = sum_i dS_ij q_i   (the chain rule
 * on the forward above; Listing 1's attention_backward(dattn, q, k, v)).
 *
 * Relative attention bias (optional; HSTU notes "Actions Speak Louder than
 * Words", section 2.4, Eq. 2: phi2(Q K^T + rab^{p,t}) with a positional and a
 * temporal part; the relative time encoding as the talk notes
 * "基于昇腾 NPU 的生成式推荐 Scaling Law 落地实践" describe its usual
 * implementation, Fuxi section: difference of the two timestamps, bucketed,
 * looked up, added into the attention scores).  With it
 *   x_ij = alpha q_i.k_j + rab_pos[h][bucket(dpos)] + rab_time[h][bucket(dt)]
 * and everything above uses that x.  Readings (the sources fix none of them):
 *   - dpos = i - j for history rows; a candidate row measures from Lh, the
 *     position its window is applied at (Lh - j), and 0 to itself;
 *   - dt = |ts_i - ts_j| (integer timestamps);
 *   - bucket(n) = floor(log2(n + 1)), capped at the table size - 1;
 *   - one table row per head; a NULL table adds nothing.
 * Its gradient: d rab_*[h][b] = sum over visible pairs in bucket b of
 * dP_ij SiLU'(x_ij) / N (oracle_sla_bwd_drab).
 *
 * Layout: q, k, v, dout and all outputs are [T, H, d] row-major doubles;
 * seq_offsets is [B+1] with seq_offsets[0] = 0; num_targets is [B] or NULL;
 * timestamps [T]; rab tables [H][buckets].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_INCLUSIVE_WINDOW 1
#define ORACLE_UNCLAMPED_TARGETS 2

static int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

/* Mask predicate M(i, j) for one sequence of length L with nt candidates. */
int oracle_sla_visible(int64_t L, int64_t nt, int64_t contextual_len,
                       int64_t K1, int64_t K2, int64_t i, int64_t j, int flags) {
  if (i < 0 || j < 0 || i >= L || j >= L) return 0;
  int64_t Lh = L - nt;            /* history length (non-candidate tokens) */
  int64_t K2eff = max64(K2, contextual_len);
  int64_t pos;                    /* position at which the window is applied */
  if (i < Lh) {
    if (j > i) return 0;          /* causal */
    pos = i;
  } else {
    if (j == i) return 1;         /* a candidate sees itself */
    if (j >= Lh) return 0;        /* ... and no other candidate */
    pos = (flags & ORACLE_UNCLAMPED_TARGETS) ? i : Lh;
  }
  int in_window = (flags & ORACLE_INCLUSIVE_WINDOW) ? (pos - j <= K1) : (pos - j < K1);
  int in_prefix = j < K2eff;
  return in_window || in_prefix;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double silu(double x) { return x * sigmoid(x); }
static double dsilu(double x) { double s = sigmoid(x); return s * (1.0 + x * (1.0 - s)); }

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* Sequence index b with offsets[b] <= t < offsets[b+1] (offsets monotone). */
static int seq_of(const int64_t* offsets, int B, int64_t t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (offsets[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

typedef struct {
  int B, H, d;
  const int64_t* offsets;
  const int64_t* num_targets;
  int64_t contextual_len, K1, K2;
  double alpha, N;
  int flags;
  const int64_t* ts;      /* [T] timestamps, or NULL */
  const double* rab_pos;  /* [H][n_pos], or NULL */
  int64_t n_pos;
  const double* rab_time; /* [H][n_time], or NULL */
  int64_t n_time;
} oracle_cfg;

static int64_t nt_of(const oracle_cfg* c, int b) { return c->num_targets ? c->num_targets[b] : 0; }

/* floor(log2(n + 1)) for n >= 0, at most nb - 1: the number of times n + 1
 * can be halved before it reaches 1. */
int64_t oracle_rab_bucket(int64_t n, int64_t nb) {
  if (n < 0) n = 0;
  uint64_t x = (uint64_t)n + 1;
  int64_t b = 0;
  while (x > 1) {
    x >>= 1;
    ++b;
  }
  return b < nb - 1 ? b : nb - 1;
}

/* Position and time buckets of the pair (i, j) of the sequence starting at
 * token s0 (history length Lh). */
static void rab_buckets(const oracle_cfg* c, int64_t s0, int64_t Lh, int64_t i, int64_t j,
                        int64_t* bp, int64_t* bt) {
  int64_t dpos = i < Lh ? i - j : (j == i ? 0 : Lh - j);
  *bp = oracle_rab_bucket(dpos, c->n_pos);
  int64_t dt = 0;
  if (c->ts) {
    dt = c->ts[s0 + i] - c->ts[s0 + j];
    if (dt < 0) dt = -dt;
  }
  *bt = oracle_rab_bucket(dt, c->n_time);
}

/* The bias rab(i, j) of head h (0 without tables). */
static double rab_of(const oracle_cfg* c, int64_t s0, int64_t Lh, int h, int64_t i, int64_t j) {
  if (!c->rab_pos && !c->rab_time) return 0.0;
  int64_t bp, bt;
  rab_buckets(c, s0, Lh, i, j, &bp, &bt);
  double r = 0.0;
  if (c->rab_pos) r += c->rab_pos[h * c->n_pos + bp];
  if (c->rab_time) r += c->rab_time[h * c->n_time + bt];
  return r;
}

/* Number of visible keys of every token (the same for every head): [T]. */
void oracle_sla_row_counts(const oracle_cfg* c, int64_t* counts) {
  int64_t T = c->offsets[c->B];
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < T; ++t) {
    int b = seq_of(c->offsets, c->B, t);
    int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, i = t - s0, n = 0;
    for (int64_t j = 0; j < L; ++j)
      n += oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j, c->flags);
    counts[t] = n;
  }
}

/* Number of rows that see every token as a key (the same for every head): [T]. */
void oracle_sla_key_counts(const oracle_cfg* c, int64_t* counts) {
  int64_t T = c->offsets[c->B];
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < T; ++t) {
    int b = seq_of(c->offsets, c->B, t);
    int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, j = t - s0, n = 0;
    for (int64_t i = 0; i < L; ++i)
      n += oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j, c->flags);
    counts[t] = n;
  }
}

/* out[r, h, :] = (1/N) sum_j M(i,j) SiLU(alpha q_i.k_j) v_j for the tokens rows[r]. */
void oracle_sla_fwd_rows(const oracle_cfg* c, const double* q, const double* k,
                         const double* v, const int64_t* rows, int64_t n_rows,
                         double* out) {
  const int H = c->H, d = c->d;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int h = 0; h < H; ++h) {
      int64_t t = rows[r];
      int b = seq_of(c->offsets, c->B, t);
      int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, i = t - s0;
      const double* qi = q + (t * H + h) * d;
      double* o = out + (r * H + h) * d;
      for (int e = 0; e < d; ++e) o[e] = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        if (!oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j, c->flags))
          continue;
        const double* kj = k + ((s0 + j) * H + h) * d;
        const double* vj = v + ((s0 + j) * H + h) * d;
        double x = c->alpha * dot(qi, kj, d) + rab_of(c, s0, L - nt_of(c, b), h, i, j);
        double p = silu(x) / c->N;
        for (int e = 0; e < d; ++e) o[e] += p * vj[e];
      }
    }
  }
}

/* dq[r, h, :] = sum_j M(i,j) (alpha/N) SiLU'(alpha q_i.k_j) (dO_i.v_j) k_j. */
void oracle_sla_bwd_dq_rows(const oracle_cfg* c, const double* q, const double* k,
                            const double* v, const double* dout, const int64_t* rows,
                            int64_t n_rows, double* dq) {
  const int H = c->H, d = c->d;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int64_t r = 0; r < n_rows; ++r) {
    for (int h = 0; h < H; ++h) {
      int64_t t = rows[r];
      int b = seq_of(c->offsets, c->B, t);
      int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, i = t - s0;
      const double* qi = q + (t * H + h) * d;
      const double* doi = dout + (t * H + h) * d;
      double* g = dq + (r * H + h) * d;
      for (int e = 0; e < d; ++e) g[e] = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        if (!oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j, c->flags))
          continue;
        const double* kj = k + ((s0 + j) * H + h) * d;
        const double* vj = v + ((s0 + j) * H + h) * d;
        double x = c->alpha * dot(qi, kj, d) + rab_of(c, s0, L - nt_of(c, b), h, i, j);
        double ds = dot(doi, vj, d) * dsilu(x) * c->alpha / c->N;
        for (int e = 0; e < d; ++e) g[e] += ds * kj[e];
      }
    }
  }
}

/* For the tokens keys[r] taken as keys:
 *   dv[r, h, :] = sum_i M(i,j) SiLU(x_ij)/N dO_i
 *   dk[r, h, :] = sum_i M(i,j) (alpha/N) SiLU'(x_ij) (dO_i.v_j) q_i          */
void oracle_sla_bwd_dkv_keys(const oracle_cfg* c, const double* q, const double* k,
                             const double* v, const double* dout, const int64_t* keys,
                             int64_t n_keys, double* dk, double* dv) {
  const int H = c->H, d = c->d;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int64_t r = 0; r < n_keys; ++r) {
    for (int h = 0; h < H; ++h) {
      int64_t t = keys[r];
      int b = seq_of(c->offsets, c->B, t);
      int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, j = t - s0;
      const double* kj = k + (t * H + h) * d;
      const double* vj = v + (t * H + h) * d;
      double* gk = dk + (r * H + h) * d;
      double* gv = dv + (r * H + h) * d;
      for (int e = 0; e < d; ++e) { gk[e] = 0.0; gv[e] = 0.0; }
      for (int64_t i = 0; i < L; ++i) {
        if (!oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j, c->flags))
          continue;
        const double* qi = q + ((s0 + i) * H + h) * d;
        const double* doi = dout + ((s0 + i) * H + h) * d;
        double x = c->alpha * dot(qi, kj, d) + rab_of(c, s0, L - nt_of(c, b), h, i, j);
        double p = silu(x) / c->N;
        double ds = dot(doi, vj, d) * dsilu(x) * c->alpha / c->N;
        for (int e = 0; e < d; ++e) { gv[e] += p * doi[e]; gk[e] += ds * qi[e]; }
      }
    }
  }
}

/* Gradients of the bias tables (either may be NULL):
 *   d_pos[h][b]  = sum over visible (i, j) with position bucket b of
 *                  dP_ij SiLU'(x_ij) / N,   d_time likewise. */
void oracle_sla_bwd_drab(const oracle_cfg* c, const double* q, const double* k, const double* v,
                         const double* dout, double* d_pos, double* d_time) {
  const int H = c->H, d = c->d;
  if (d_pos) memset(d_pos, 0, sizeof(double) * H * c->n_pos);
  if (d_time) memset(d_time, 0, sizeof(double) * H * c->n_time);
#pragma omp parallel for schedule(dynamic, 1)
  for (int h = 0; h < H; ++h) {  /* each head owns its table rows */
    for (int b = 0; b < c->B; ++b) {
      int64_t s0 = c->offsets[b], L = c->offsets[b + 1] - s0, Lh = L - nt_of(c, b);
      for (int64_t i = 0; i < L; ++i) {
        const double* qi = q + ((s0 + i) * H + h) * d;
        const double* doi = dout + ((s0 + i) * H + h) * d;
        for (int64_t j = 0; j < L; ++j) {
          if (!oracle_sla_visible(L, nt_of(c, b), c->contextual_len, c->K1, c->K2, i, j,
                                  c->flags))
            continue;
          const double* kj = k + ((s0 + j) * H + h) * d;
          const double* vj = v + ((s0 + j) * H + h) * d;
          double x = c->alpha * dot(qi, kj, d) + rab_of(c, s0, Lh, h, i, j);
          double g = dot(doi, vj, d) * dsilu(x) / c->N;
          int64_t bp, bt;
          rab_buckets(c, s0, Lh, i, j, &bp, &bt);
          if (d_pos) d_pos[h * c->n_pos + bp] += g;
          if (d_time) d_time[h * c->n_time + bt] += g;
        }
      }
    }
  }
}
