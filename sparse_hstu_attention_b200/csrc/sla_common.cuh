// Shared device-side definitions of the SLA HSTU attention library: the
// kernel argument block, the workspace layout, the mask predicate and the
// tile enumeration that every kernel (work list, forward, backward, pair
// count) uses, so that all of them agree on which (query tile, key tile)
// pairs are non-empty.
//
// Mask ("Bending the Scaling Law Curve in Large-Scale Recommendation
// Systems", section 4.2.1, Eq. 7, read with a K1-token window that includes
// self; K2eff = max(K2, contextual_len) from the TorchEasyRec "ULTRA HSTU"
// docs; candidates as in the M-FALCON mask figure of the HSTU notes):
//   history row i < Lh:    j <= i  and (i - j < K1  or  j < K2eff)
//   candidate row i >= Lh: j == i  or (j < Lh and (Lh - j < K1 or j < K2eff))
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hstu_sla.h"

namespace hstu {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- workspace
// [0, 256)            WsHeader
// [256, ...)          int2 items[max_items]   list 0: (sequence, query tile)
// [align256, ...)     int2 items2[max_items]  list 1: (sequence, key tile),
//                                             prefix key tiles first
struct WsHeader {
  int32_t status;        // HSTU_SLA_OK or a negative code
  int32_t n_items;       // entries of list 0
  int32_t n_items2;      // entries of list 1
  int32_t n_items2_pre;  // leading entries of list 1 that hold prefix key tiles
  int32_t sched;         // dynamic scheduler counter over list 0 units
  int32_t sched2;        // dynamic scheduler counter over list 1 units
  int32_t pad0[2];
  int64_t wait_limit_ns; // bounded-wait limit of the launch's kernels (0: the default)
  int32_t pad[54];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kMinTile = 64;  // smallest tile any kernel enumerates with

// Tile shapes of the kernels the entry points launch (the pair-count hook
// walks the same enumeration).
constexpr int kFwdBM = 128, kFwdBN = 128;  // forward: query tile x key tile
constexpr int kKvBN = 128, kKvBM = 64;     // backward KV pass: key tile x streamed rows
constexpr int kQpBM = 128, kQpBN = 64;     // backward Q pass: query tile x streamed keys

__host__ __device__ inline int64_t max_items(int64_t T, int B) {
  return (T + kMinTile - 1) / kMinTile + B;
}
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline size_t ws_items_offset() { return sizeof(WsHeader); }
__host__ __device__ inline size_t ws_items2_offset(int64_t T, int B) {
  return align256(ws_items_offset() + sizeof(int2) * size_t(max_items(T, B)));
}
__host__ __device__ inline size_t ws_bytes(int64_t T, int B) {
  return align256(ws_items2_offset(T, B) + sizeof(int2) * size_t(max_items(T, B)));
}

// The one-pass backward (head_dim kFusedBwdD) accumulates dQ in fp32 [H, T, d]
// after the work lists; other head dims need no such buffer.
constexpr int kFusedBwdD = 128;
__host__ __device__ inline size_t dq_workspace_bytes(int64_t T, int H, int d) {
  return d == kFusedBwdD ? size_t(T) * size_t(H) * size_t(d) * sizeof(float) : 0;
}
// The STU layer's SiLU' pass after the one-pass backward (silu_qkv_kernel)
// runs kSiluBlocks blocks; each leaves its column sums of the Q, K, V blocks
// (the bias gradient's partial sums) after the dQ accumulator.
constexpr int kSiluBlocks = 1024;
__host__ __device__ inline size_t db_parts_bytes(int H, int d) {
  return d == kFusedBwdD ? size_t(kSiluBlocks) * 3 * size_t(H) * size_t(d) * sizeof(float) : 0;
}
__host__ __device__ inline size_t ws_bwd_bytes(int64_t T, int B, int H, int d) {
  return ws_bytes(T, B) + dq_workspace_bytes(T, H, d) + db_parts_bytes(H, d);
}

// ------------------------------------------------------------ kernel args
constexpr int kMaxGroups = 4;  // problems per grouped launch

struct AttnArgs {
  const int32_t* offs;   // [B+1]
  const int32_t* nts;    // [B] or null
  const int2* items;     // work list 0 (query tiles)
  const int2* items2;    // work list 1 (key tiles)
  WsHeader* ws;          // status / counts
  float* dqacc;          // fp32 dQ accumulator [H, T, d] (one-pass backward only)
  int B, H, K1, K2e, max_seq_len;
  int cand_only;         // forward work list: only query tiles holding candidates
  int64_t T;
  float alpha, inv_n;
  const bf16* q;
  const bf16* k;
  const bf16* v;
  const bf16* dout;
  bf16* out;
  bf16* dq;
  bf16* dk;
  bf16* dv;
  int64_t q_rs, k_rs, v_rs, do_rs, o_rs, dq_rs, dk_rs, dv_rs;
  // Optional (one-pass backward, set by the STU layer): q, k, v are SiLU
  // outputs of the pre-activations pre_q / pre_k / pre_v (row stride pre_rs);
  // the backward then leaves the pre-activation gradients dq * SiLU'(pre_q),
  // ... in dq, dk, dv and adds their column sums (the bias gradient) into
  // db_q / db_k / db_v ([H * d] each).  Null pre_q: plain dq, dk, dv.
  const bf16* pre_q;
  const bf16* pre_k;
  const bf16* pre_v;
  int64_t pre_rs;
  float* db_q;
  float* db_k;
  float* db_v;
  float* db_part;  // [kSiluBlocks][3 (q, k, v)][H * d] partial sums (workspace)
  // Relative attention bias (optional): per-head tables of nbp / nbt log2
  // buckets of the position and timestamp differences; their gradients.
  const int32_t* ts;
  const float* rab_pos;
  const float* rab_time;
  int nbp, nbt;
  float* d_rab_pos;
  float* d_rab_time;
  // Bounded-wait limit the work-list kernel records for the launch (0: the
  // kernels' default); only the wait-timeout test hook sets it.
  int64_t wait_limit_ns;
};

// Relative attention bias, with the tables held in registers: lane b of a
// warp holds half of bucket min(b, nb - 1) of this head's table (0 without
// one), so a bucket index needs no clamp to nb - 1 and the value goes
// straight into x / 2 = (alpha s + bias) / 2.  Every lane must take part.
__device__ __forceinline__ float rab_lane_table(const float* tab, int nb, int h, int lane) {
  return tab ? 0.5f * __ldg(tab + h * nb + (lane < nb ? lane : nb - 1)) : 0.f;
}

// The log bucket floor(log2(n + 1)) of a difference n >= 0, from u = n + 1
// modulo 2^32: the index of u's top bit, and -1 for u = 0 (n = 2^32 - 1).
// As a shuffle lane (low 5 bits) or after `& 31`, every n >= 2^31 - 1 lands
// in bucket 31, so the result equals the bucket of n capped at 2^31 - 1.
__device__ __forceinline__ int rab_log_bucket(uint32_t u) { return 31 - __clz(u); }

// u = |ti - tj| + 1 for two int32 timestamps: the exact difference as an
// unsigned 32-bit value.
__device__ __forceinline__ uint32_t rab_time_u(int32_t ti, int32_t tj) {
  return __sad(ti, tj, 1u);
}

// u = dpos + 1 of the pair (query i, key j) in a sequence with Lh history
// rows, where dpos = i - j for a history row and Lh - j for a candidate row
// (0 to itself), clamped below at 0.  Every visible pair has dpos >= 0, so
// one form serves both kinds of row: u = max(min(i, Lh) - j + 1, 1), which
// also gives a candidate's self pair dpos = 0 (invisible pairs' buckets are
// never used).  Callers split min(i, Lh) + 1 - j into a + b, one of them
// constant along their loop, for one fused add-max per pair.
__device__ __forceinline__ uint32_t rab_pos_u(int a, int b) {
  return (uint32_t)__viaddmax_s32(a, b, 1);
}

// Half the bias of a pair from its two buckets (shuffle lanes).
__device__ __forceinline__ float rab_half_bias(float tabp, float tabt, int bp, int bt) {
  return __shfl_sync(0xffffffffu, tabp, bp) + __shfl_sync(0xffffffffu, tabt, bt);
}

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int imax(int a, int b) { return a > b ? a : b; }

struct SeqGeom {
  int s0;  // first token of the sequence
  int L;   // length
  int Lh;  // history length (L - num_targets)
};

__device__ __forceinline__ SeqGeom seq_geom(const AttnArgs& a, int b) {
  SeqGeom g;
  g.s0 = a.offs[b];
  g.L = a.offs[b + 1] - g.s0;
  g.Lh = g.L - (a.nts ? a.nts[b] : 0);
  return g;
}

// Mask predicate for 0 <= i, j.
__host__ __device__ __forceinline__ bool sla_visible(int i, int j, int L, int Lh, int K1, int K2e) {
  if (i < Lh) return j <= i && (i - j < K1 || j < K2e);
  if (i >= L) return false;
  return j == i || (j < Lh && (Lh - j < K1 || j < K2e));
}

// The same predicate as three intervals per row, for inner loops:
// visible(j) = j < pre || (lo <= j && j < hi) || j == self.
struct RowMask {
  int pre, lo, hi, self;
  __host__ __device__ __forceinline__ bool operator()(int j) const {
    return j < pre || (j >= lo && j < hi) || j == self;
  }
};

__host__ __device__ __forceinline__ RowMask row_mask(int i, int L, int Lh, int K1, int K2e) {
  RowMask m;
  if (i < Lh) {
    m.pre = imin(K2e, i + 1);
    m.lo = imax(0, i - K1 + 1);
    m.hi = K1 > 0 ? i + 1 : 0;
    m.self = -1;
  } else if (i < L) {
    m.pre = imin(K2e, Lh);
    m.lo = imax(0, Lh - K1 + 1);
    m.hi = K1 > 0 ? Lh : 0;
    m.self = i;
  } else {
    m.pre = 0; m.lo = 0; m.hi = 0; m.self = -1;
  }
  return m;
}

// Bit e set iff position base + e lies in [lo, hi), for e in [0, 32).
__host__ __device__ __forceinline__ uint32_t range_bits(int lo, int hi, int base) {
  const int a = lo - base < 0 ? 0 : lo - base;
  const int b = hi - base > 32 ? 32 : hi - base;
  if (a >= b) return 0u;
  const uint32_t upto_b = b >= 32 ? 0xFFFFFFFFu : ((1u << b) - 1u);
  return upto_b & ~((1u << a) - 1u);
}

// Visibility of keys [base, base + 32) for one row / of rows [base, base + 32)
// for one key, one bit each: the interval forms above turned into a bitmask,
// so the per-element test in inner loops is a single bit test.
__host__ __device__ __forceinline__ uint32_t row_mask_bits(const RowMask& m, int base) {
  uint32_t bits = range_bits(0, m.pre, base) | range_bits(m.lo, m.hi, base);
  if (m.self >= base && m.self < base + 32) bits |= 1u << (m.self - base);
  return bits;
}

// Zero the bf16 halves of a packed pair whose bits (2e, 2e+1) of `bits` are clear.
__host__ __device__ __forceinline__ uint32_t mask_pair(uint32_t p2, uint32_t bits, int e) {
  const uint32_t lo = (bits >> (2 * e)) & 1u, hi = (bits >> (2 * e + 1)) & 1u;
  return p2 & ((0u - lo) & 0x0000FFFFu | (0u - hi) & 0xFFFF0000u);
}

// Up to three disjoint, increasing tile-index intervals [lo, hi).
struct Spans {
  int lo[3], hi[3], n;
  __host__ __device__ void clear() { n = 0; }
  // Pushes must come in non-decreasing order of lo; overlapping or touching
  // intervals merge.
  __host__ __device__ void push(int l, int h) {
    if (l >= h) return;
    if (n > 0 && l <= hi[n - 1]) {
      if (h > hi[n - 1]) hi[n - 1] = h;
      return;
    }
    lo[n] = l; hi[n] = h; ++n;
  }
  __host__ __device__ int count() const {
    int c = 0;
    for (int s = 0; s < n; ++s) c += hi[s] - lo[s];
    return c;
  }
  // Tile index of the n-th element (0 <= e < count()).
  __host__ __device__ int at(int e) const {
    for (int s = 0; s < n; ++s) {
      int w = hi[s] - lo[s];
      if (e < w) return lo[s] + e;
      e -= w;
    }
    return -1;
  }
};

// Key tiles (width BN) that hold a visible key for some row of the query
// rows [r0, r1) of one sequence: the global prefix, the local band (which for
// candidate rows is the band ending at Lh) and the candidates' own diagonal.
__host__ __device__ inline Spans q_tile_key_tiles(int r0, int r1, int Lh, int K1, int K2e,
                                                  int BN) {
  Spans s;
  s.clear();
  int hist_end = r1 < Lh ? r1 : Lh;        // prefix keys are history keys
  int pre_hi = K2e < hist_end ? K2e : hist_end;
  s.push(0, cdiv(pre_hi, BN));
  if (K1 > 0) {
    int blo, bhi;
    if (r0 < Lh) {
      blo = r0 - K1 + 1;
      bhi = r1 < Lh ? r1 : Lh;
    } else {
      blo = Lh - K1 + 1;
      bhi = Lh;
    }
    if (blo < 0) blo = 0;
    if (blo < bhi) s.push(blo / BN, cdiv(bhi, BN));
  }
  if (r1 > Lh) {
    int dlo = r0 > Lh ? r0 : Lh;
    s.push(dlo / BN, cdiv(r1, BN));
  }
  return s;
}

// Query tiles (height BM) that hold a row seeing some key of the key tile
// [j0, j1) of one sequence of length L.
__host__ __device__ inline Spans k_tile_q_tiles(int j0, int j1, int L, int Lh, int K1, int K2e,
                                                int BM) {
  Spans s;
  s.clear();
  int pre_end = K2e < Lh ? K2e : Lh;
  if (j0 < pre_end) {  // a prefix key of the history: every later row sees it
    s.push(j0 / BM, cdiv(L, BM));
    return s;
  }
  if (K1 > 0 && j0 < Lh) {
    int jh = j1 < Lh ? j1 : Lh;  // last history key + 1
    int rhi = jh - 1 + K1;       // history rows i <= j + K1 - 1
    if (rhi > Lh) rhi = Lh;
    s.push(j0 / BM, cdiv(rhi, BM));
    if (jh - 1 >= Lh - K1 + 1) s.push(Lh / BM, cdiv(L, BM));  // candidates' band
  }
  if (j1 > Lh) {  // candidate keys: only the candidate itself
    int dlo = j0 > Lh ? j0 : Lh;
    s.push(dlo / BM, cdiv(j1, BM));
  }
  return s;
}

// True if every (row, key) pair of rows [r0, r1) x keys [j0, j1) lies inside
// the sequence and is visible, so the mask need not be evaluated.  Callers pass
// the UNCLIPPED tile ends (r0 + BM, j0 + BN): a tile that runs past the
// sequence end is never full, so rows / keys past the end are always masked.
__host__ __device__ __forceinline__ bool tile_full(int r0, int r1, int j0, int j1, int Lh, int K1,
                                                   int K2e) {
  return r1 <= Lh && j1 <= r0 + 1 && (j1 <= K2e || j0 >= r1 - K1);
}

// The visible rows of key j as intervals, for inner loops of the key-major
// backward: visible(i) = (lo <= i < hi) || (tlo <= i < thi) || i == self.
struct KeyMask {
  int lo, hi, tlo, thi, self;
  __host__ __device__ __forceinline__ bool operator()(int i) const {
    return (i >= lo && i < hi) || (i >= tlo && i < thi) || i == self;
  }
};

__host__ __device__ __forceinline__ KeyMask key_mask(int j, int L, int Lh, int K1, int K2e) {
  KeyMask m;
  m.lo = m.hi = m.tlo = m.thi = 0;
  m.self = -1;
  if (j >= L || j < 0) return m;
  if (j >= Lh) {          // a candidate key: seen by that candidate only
    m.self = j;
  } else if (j < K2e) {   // a prefix key: every row from j on
    m.lo = j;
    m.hi = L;
  } else {                // history rows of its window; candidates if in theirs
    m.lo = j;
    m.hi = imin(j + K1, Lh);
    if (Lh - j < K1) {
      m.tlo = Lh;
      m.thi = L;
    }
  }
  return m;
}

__host__ __device__ __forceinline__ uint32_t key_mask_bits(const KeyMask& m, int base) {
  uint32_t bits = range_bits(m.lo, m.hi, base) | range_bits(m.tlo, m.thi, base);
  if (m.self >= base && m.self < base + 32) bits |= 1u << (m.self - base);
  return bits;
}

// One work unit as the producer warp decodes it once and hands it to the other
// roles through a shared-memory ring: the sequence geometry, the resident
// tile's rows [t0, t1) and the streamed tiles it meets, as up to three spans
// of tile indices.  nsteps = -1 marks the end of the CTA's schedule.
struct UnitRec {
  int h, s0, L, Lh, t0, t1, nsteps, nsp;
  int lo[3], hi[3];
  int grp;  // problem of the unit within its launch (0 unless grouped)
  int pad;
};
static_assert(sizeof(UnitRec) == 64, "unit record size");

__device__ __forceinline__ void unit_rec_fill(UnitRec* r, int h, int s0, int L, int Lh, int t0,
                                              int t1, const Spans& sp) {
  r->h = h; r->s0 = s0; r->L = L; r->Lh = Lh; r->t0 = t0; r->t1 = t1;
  r->grp = 0;
  r->nsteps = sp.count();
  r->nsp = sp.n;
  for (int s = 0; s < 3; ++s) {
    r->lo[s] = s < sp.n ? sp.lo[s] : 0;
    r->hi[s] = s < sp.n ? sp.hi[s] : 0;
  }
}

// Walks the streamed tiles of a unit record in order, one step at a time.
struct SpanCursor {
  int s, j, hi;
  __device__ __forceinline__ void begin(const UnitRec* r) {
    s = 0;
    j = r->lo[0];
    hi = r->hi[0];
  }
  __device__ __forceinline__ void next(const UnitRec* r) {
    if (++j == hi && s + 1 < r->nsp) {
      ++s;
      j = r->lo[s];
      hi = r->hi[s];
    }
  }
};

__device__ __forceinline__ void set_status(WsHeader* ws, int code) {
  atomicCAS(&ws->status, 0, code);
}

__device__ __forceinline__ int load_status(const WsHeader* ws) {
  return *((volatile const int32_t*)&ws->status);
}

// The launch's bounded-wait limit in ns (`dflt` unless the header sets one).
__device__ __forceinline__ uint64_t wait_limit(const WsHeader* ws, uint64_t dflt) {
  const int64_t v = *((volatile const int64_t*)&ws->wait_limit_ns);
  return v > 0 ? (uint64_t)v : dflt;
}

// ------------------------------------------------------------ host launchers
// (defined in the .cu files; return cudaError_t of the launch)
// list 0: (sequence, query tile of `tile` rows); list 1: (sequence, key tile
// of `tile` keys), prefix key tiles first.
// `first`: the call's first work list, which also resets the status word.
cudaError_t launch_worklist(const AttnArgs& a, int tile, int list, bool first, cudaStream_t st);
cudaError_t launch_count_pairs(const AttnArgs& a, int BMf, int BNf, int BMb, int BNb,
                               int64_t* row_counts, int64_t* key_counts, cudaStream_t st);
cudaError_t launch_fwd_tc(const AttnArgs& a, int d, cudaStream_t st);
// Several problems (same head_dim) in one launch of the forward / one-pass
// backward kernel: one schedule over every problem's units.  `common` holds
// the launch's status word and scheduler counters; each problem's work lists
// were built into its own workspace beforehand.
struct GroupSet {
  AttnArgs g[kMaxGroups];
  WsHeader* common;
  int G;
  // Wait-timeout test hook only: the launch takes the kernel instantiation
  // whose pointwise warps withhold their first hand-over arrive, so that the
  // role waiting for it runs into the bounded-wait limit.
  int stall;
  // The dQ accumulators were cleared beforehand (hstu_sla_bwd_prepare).
  int cleared;
};
cudaError_t launch_fwd_grouped(const GroupSet& gs, int d, cudaStream_t st);
// The backward entry point with the STU layer's SiLU' / bias-gradient fusion
// (AttnArgs::pre_q ...); fz = nullptr is hstu_sla_bwd.  Fusion needs
// d = kFusedBwdD and H * d / 8 dividing 256.
struct SiluFusion {
  const bf16* pre_q;
  const bf16* pre_k;
  const bf16* pre_v;
  int64_t pre_rs;
  float* db_q;
  float* db_k;
  float* db_v;
};
int sla_bwd(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
            cudaStream_t st, const SiluFusion* fz);
int sla_bwd_prepare(const hstu_sla_bwd_params* p, void* workspace, size_t workspace_bytes,
                    cudaStream_t st);
cudaError_t launch_bwd_fused_grouped(const GroupSet& gs, cudaStream_t st);
cudaError_t launch_bwd_tc(const AttnArgs& a, int d, bool kv_pass, cudaStream_t st);
// head_dim kFusedBwdD: zeroes a.dqacc, runs the one-pass backward, converts dq
cudaError_t launch_bwd_fused(const AttnArgs& a, cudaStream_t st, bool cleared = false);

}  // namespace hstu
