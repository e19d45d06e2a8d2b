// Work-list construction, device-side input validation and the pair-count
// test hook.
//
// The work list is built on the device from seq_offsets / num_targets, so a
// call never waits on the host.  Forward items are (sequence, query tile);
// backward items are (sequence, key tile) with the prefix key tiles first:
// a prefix key is seen by every later row of its sequence, so those items are
// the longest and start first (a longest-first order without a sort).
#include "sla_common.cuh"

namespace hstu {

namespace {

constexpr int kWlThreads = 1024;

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ int block_exclusive_scan(int v, int* out, int* smem) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (kWlThreads / 32) ? smem[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    smem[lane] = w;  // inclusive warp sums
  }
  __syncthreads();
  int base = warp > 0 ? smem[warp - 1] : 0;
  *out = base + x - v;
  int total = smem[kWlThreads / 32 - 1];
  __syncthreads();
  return total;
}

// One block.  list 0: items (b, query tile) in sequence order.  list 1:
// first every (b, key tile) whose key tile starts inside the history prefix
// [0, min(K2eff, Lh)), then all other key tiles.
__global__ void __launch_bounds__(kWlThreads) worklist_kernel(AttnArgs a, int tile, int list,
                                                             int first) {
  __shared__ int s_scan[32];
  __shared__ int s_bad;
  const int backward = list;
  int2* items = const_cast<int2*>(list ? a.items2 : a.items);
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  // validation of the device-resident offsets and targets
  for (int b = threadIdx.x; b <= a.B; b += blockDim.x) {
    int o = a.offs[b];
    bool bad = false;
    if (b == 0) bad |= (o != 0);
    if (b == a.B) bad |= ((int64_t)o != a.T);
    if (b < a.B) {
      int len = a.offs[b + 1] - o;
      int nt = a.nts ? a.nts[b] : 0;
      bad |= (len < 0) | (len > a.max_seq_len) | (nt < 0) | (nt > len);
    }
    if (bad) s_bad = 1;
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0) {
      a.ws->status = HSTU_SLA_ERR_BAD_INPUT;
      a.ws->n_items = 0;
      a.ws->n_items2 = 0;
      a.ws->n_items2_pre = 0;
      a.ws->sched = 0;
      a.ws->sched2 = 0;
    }
    return;
  }
  // pass 0 counts prefix items (backward) and writes them; pass 1 the rest.
  int written = 0, n_pre = 0;
  for (int pass = backward ? 0 : 1; pass < 2; ++pass) {
    for (int c0 = 0; c0 < a.B; c0 += kWlThreads) {
      int b = c0 + threadIdx.x;
      int cnt = 0, first = 0;
      if (b < a.B) {
        int L = a.offs[b + 1] - a.offs[b];
        int Lh = L - (a.nts ? a.nts[b] : 0);
        int ntile = cdiv(L, tile);
        int npre = 0;
        if (backward) {
          int pre_end = a.K2e < Lh ? a.K2e : Lh;
          npre = cdiv(pre_end, tile);
          if (npre > ntile) npre = ntile;
        }
        if (pass == 0) { cnt = npre; first = 0; }
        else { cnt = ntile - npre; first = npre; }
        if (!backward && a.cand_only) {  // from the tile of the first candidate on
          first = Lh < L ? Lh / tile : ntile;
          cnt = ntile - first;
        }
      }
      int off;
      int total = block_exclusive_scan(cnt, &off, s_scan);
      for (int e = 0; e < cnt; ++e) items[written + off + e] = make_int2(b, first + e);
      written += total;
    }
    if (pass == 0) n_pre = written;
  }
  if (threadIdx.x == 0) {
    if (first) {
      a.ws->status = HSTU_SLA_OK;
      a.ws->wait_limit_ns = a.wait_limit_ns;
    }
    if (list) {
      a.ws->n_items2 = written;
      a.ws->n_items2_pre = n_pre;
      a.ws->sched2 = 0;
    } else {
      a.ws->n_items = written;
      a.ws->sched = 0;
    }
  }
}

// Per token: number of visible keys found by walking the forward enumeration
// (row_counts), and number of rows that see it found by walking the backward
// enumeration (key_counts).
__global__ void count_pairs_kernel(AttnArgs a, int BMf, int BNf, int BMb, int BNb,
                                   int64_t* row_counts, int64_t* key_counts) {
  if (load_status(a.ws) != 0) return;
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= a.T) return;
  int lo = 0, hi = a.B - 1;  // sequence of token t
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (a.offs[mid] <= t) lo = mid; else hi = mid - 1;
  }
  SeqGeom g = seq_geom(a, lo);
  int p = int(t - g.s0);
  if (row_counts) {
    int r0 = (p / BMf) * BMf, r1 = imin(r0 + BMf, g.L);
    Spans s = q_tile_key_tiles(r0, r1, g.Lh, a.K1, a.K2e, BNf);
    int64_t n = 0;
    for (int e = 0; e < s.count(); ++e) {
      int kt = s.at(e);
      for (int j = kt * BNf; j < imin(kt * BNf + BNf, g.L); ++j)
        n += sla_visible(p, j, g.L, g.Lh, a.K1, a.K2e);
    }
    row_counts[t] = n;
  }
  if (key_counts) {
    int j0 = (p / BNb) * BNb, j1 = imin(j0 + BNb, g.L);
    Spans s = k_tile_q_tiles(j0, j1, g.L, g.Lh, a.K1, a.K2e, BMb);
    int64_t n = 0;
    for (int e = 0; e < s.count(); ++e) {
      int qt = s.at(e);
      for (int i = qt * BMb; i < imin(qt * BMb + BMb, g.L); ++i)
        n += sla_visible(i, p, g.L, g.Lh, a.K1, a.K2e);
    }
    key_counts[t] = n;
  }
}

}  // namespace

cudaError_t launch_worklist(const AttnArgs& a, int tile, int list, bool first, cudaStream_t st) {
  worklist_kernel<<<1, kWlThreads, 0, st>>>(a, tile, list, first ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_count_pairs(const AttnArgs& a, int BMf, int BNf, int BMb, int BNb,
                               int64_t* row_counts, int64_t* key_counts, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  int threads = 256;
  int64_t blocks = (a.T + threads - 1) / threads;
  count_pairs_kernel<<<(unsigned)blocks, threads, 0, st>>>(a, BMf, BNf, BMb, BNb, row_counts,
                                                           key_counts);
  return cudaGetLastError();
}

}  // namespace hstu
