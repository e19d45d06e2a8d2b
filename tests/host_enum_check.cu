// Host-side check of the library's tile enumeration (sla_common.cuh), built
// and run on the CPU by tests/test_enumeration_host.py.  For random sequence
// geometries it brute-forces the mask predicate and verifies, for every tile
// shape the kernels use (256-row units on CTA pairs included), that
//   - every visible (row, key) pair lies in an enumerated (query tile, key tile)
//     pair, from the query side (forward) and from the key side (backward);
//   - no enumerated (query tile, key tile) pair is empty, from either side;
//   - tile_full() on an unclipped tile is only true when every pair of the
//     tile lies inside the sequence and is visible;
//   - the per-row and per-key interval forms row_mask() / key_mask() and
//     their 32-bit bitmask forms equal the predicate.
// Prints "OK <cases>" or the first failure.
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "../sparse_hstu_attention_b200/csrc/sla_common.cuh"

using namespace hstu;

static bool vis(int i, int j, int L, int Lh, int K1, int K2e) {
  if (i < 0 || j < 0 || i >= L || j >= L) return false;
  return sla_visible(i, j, L, Lh, K1, K2e);
}

static int check(int L, int nt, int K1, int K2e, int BM, int BN) {
  const int Lh = L - nt;
  const int nq = cdiv(L, BM), nk = cdiv(L, BN);
  std::vector<char> qk(size_t(nq) * nk, 0), fwd(size_t(nq) * nk, 0), bwd(size_t(nq) * nk, 0);
  for (int i = 0; i < L; ++i) {
    RowMask m = row_mask(i, L, Lh, K1, K2e);
    for (int base = 0; base < L + 32; base += 16) {
      const uint32_t rb = row_mask_bits(m, base);
      const uint32_t kb = key_mask_bits(key_mask(i, L, Lh, K1, K2e), base);
      for (int e = 0; e < 32; ++e) {
        if (((rb >> e) & 1u) != (uint32_t)vis(i, base + e, L, Lh, K1, K2e)) { printf("row_mask_bits mismatch L=%d i=%d base=%d e=%d\n", L, i, base, e); return 1; }
        if (((kb >> e) & 1u) != (uint32_t)vis(base + e, i, L, Lh, K1, K2e)) { printf("key_mask_bits mismatch L=%d j=%d base=%d e=%d\n", L, i, base, e); return 1; }
      }
    }
    for (int j = 0; j < L; ++j) {
      bool v = vis(i, j, L, Lh, K1, K2e);
      if (v != key_mask(j, L, Lh, K1, K2e)(i)) { printf("key_mask mismatch L=%d nt=%d K1=%d K2e=%d i=%d j=%d\n", L, nt, K1, K2e, i, j); return 1; }
      if (v != m(j)) { printf("row_mask mismatch L=%d nt=%d K1=%d K2e=%d i=%d j=%d\n", L, nt, K1, K2e, i, j); return 1; }
      if (v) qk[size_t(i / BM) * nk + j / BN] = 1;
    }
  }
  for (int qt = 0; qt < nq; ++qt) {
    int r0 = qt * BM, r1 = r0 + BM < L ? r0 + BM : L;
    Spans s = q_tile_key_tiles(r0, r1, Lh, K1, K2e, BN);
    for (int e = 0; e < s.count(); ++e) {
      int kt = s.at(e);
      if (kt < 0 || kt >= nk) { printf("fwd tile out of range\n"); return 1; }
      if (fwd[size_t(qt) * nk + kt]) { printf("fwd tile twice\n"); return 1; }
      fwd[size_t(qt) * nk + kt] = 1;
      int j0 = kt * BN;
      // full means: the whole unclipped tile is inside the sequence and visible
      if (tile_full(r0, r0 + BM, j0, j0 + BN, Lh, K1, K2e))
        for (int i = r0; i < r0 + BM; ++i)
          for (int j = j0; j < j0 + BN; ++j)
            if (!vis(i, j, L, Lh, K1, K2e)) { printf("tile_full wrong L=%d nt=%d K1=%d K2e=%d r0=%d j0=%d BM=%d BN=%d\n", L, nt, K1, K2e, r0, j0, BM, BN); return 1; }
    }
  }
  for (int kt = 0; kt < nk; ++kt) {
    int j0 = kt * BN, j1 = j0 + BN < L ? j0 + BN : L;
    Spans s = k_tile_q_tiles(j0, j1, L, Lh, K1, K2e, BM);
    for (int e = 0; e < s.count(); ++e) {
      int qt = s.at(e);
      if (qt < 0 || qt >= nq) { printf("bwd tile out of range\n"); return 1; }
      if (bwd[size_t(qt) * nk + kt]) { printf("bwd tile twice\n"); return 1; }
      bwd[size_t(qt) * nk + kt] = 1;
    }
  }
  size_t extra_f = 0, extra_b = 0;
  for (size_t x = 0; x < qk.size(); ++x) {
    if (qk[x] && !fwd[x]) { printf("fwd misses a pair tile L=%d nt=%d K1=%d K2e=%d BM=%d BN=%d qt=%zu kt=%zu\n", L, nt, K1, K2e, BM, BN, x / nk, x % nk); return 1; }
    if (qk[x] && !bwd[x]) { printf("bwd misses a pair tile L=%d nt=%d K1=%d K2e=%d BM=%d BN=%d qt=%zu kt=%zu\n", L, nt, K1, K2e, BM, BN, x / nk, x % nk); return 1; }
    extra_f += fwd[x] && !qk[x];
    extra_b += bwd[x] && !qk[x];
  }
  if (extra_f || extra_b) {
    printf("empty tiles enumerated L=%d nt=%d K1=%d K2e=%d BM=%d BN=%d fwd=%zu bwd=%zu\n", L, nt, K1, K2e, BM, BN, extra_f, extra_b);
    return 1;
  }
  return 0;
}

int main(int argc, char** argv) {
  int n = argc > 1 ? atoi(argv[1]) : 3000;
  std::mt19937 rng(12345);
  int cases = 0;
  const int tiles[][2] = {{64, 64}, {128, 128}, {128, 64}, {64, 128}, {256, 64}, {64, 256}};
  for (int c = 0; c < n; ++c) {
    int L = 1 + rng() % 700;
    if (rng() % 6 == 0) L = 64 * (1 + rng() % 8) + (rng() % 2 ? 1 : 0);
    int nt = (rng() % 4 == 0) ? 0 : rng() % (L + 1);
    if (rng() % 8 == 0) nt = L;
    int K1 = rng() % 5 == 0 ? 0 : rng() % 400;
    if (rng() % 10 == 0) K1 = 1;
    if (rng() % 10 == 0) K1 = 100000;
    int K2e = rng() % 4 == 0 ? 0 : rng() % 300;
    for (auto& t : tiles) {
      if (check(L, nt, K1, K2e, t[0], t[1])) return 1;
      ++cases;
    }
  }
  printf("OK %d\n", cases);
  return 0;
}
