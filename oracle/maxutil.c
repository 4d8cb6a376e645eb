/*
 * Oracle (test infrastructure only): MaxUtil by exhaustive enumeration.
 *
 * "EasyBalance: Cross-Layer Load Balancing in Distributed MoE Inference",
 * §4.2 and §5.2: among the subsets S of the pending micro-batches with
 * |S| >= m, pick the one whose combined workload W = sum_{j in S} w_j has the
 * highest utilisation U(S) = sum_d W_d / (D max_d W_d).  Ties: larger |S|,
 * then the smaller bitmask of micro-batch ids.  A set without work has U = 0.
 *
 * This is the same definition as oracle/schedule.py's maxutil, in plain C so
 * that pending sets of 32 micro-batches (about 15 million admissible subsets
 * at m = 24) finish in seconds.  Two enumerations of it:
 *   oracle_maxutil_plain  every bitmask S over the n pending positions, in
 *                         increasing order, skipping |S| < m; W summed from
 *                         the member rows.  2^n masks: n <= 24 in practice.
 *   oracle_maxutil        every admissible S visited as its complement
 *                         C = P \ S with |C| <= n - m, C running over all
 *                         combinations in lexicographic order; W recomputed
 *                         from the totals minus the rows of C.  For large n
 *                         with m close to n (n = 32, m = 24).
 * They share nothing but the U comparison, so each pins the other.
 */
#include <stdint.h>
#include <string.h>

/* U(a) > U(b) for (sum, max) pairs, with U = 0 when max = 0. */
static int u_greater(int64_t sa, int64_t ma, int64_t sb, int64_t mb) {
  if (ma == 0 || mb == 0) return ma != 0 && mb == 0;
  return (__int128)sa * mb > (__int128)sb * ma;
}

static int u_equal(int64_t sa, int64_t ma, int64_t sb, int64_t mb) {
  if (ma == 0 || mb == 0) return ma == mb;
  return (__int128)sa * mb == (__int128)sb * ma;
}

/* w: n rows of D loads (row i belongs to micro-batch ids[i]); n <= 32, D <= 64. */
uint32_t oracle_maxutil(const int64_t* w, const int32_t* ids, int n, int D, int m) {
  uint32_t all = 0;
  for (int i = 0; i < n; ++i) all |= 1u << ids[i];
  if (n <= m) return all;
  int64_t total[64];
  for (int d = 0; d < D; ++d) {
    total[d] = 0;
    for (int i = 0; i < n; ++i) total[d] += w[i * D + d];
  }
  int have = 0, best_size = 0;
  int64_t best_sum = 0, best_max = 0;
  uint32_t best_mask = 0;
  int comb[33];
  for (int c = 0; c <= n - m; ++c) {
    for (int i = 0; i < c; ++i) comb[i] = i;  /* first combination of size c */
    for (;;) {
      uint32_t cmask = 0;
      for (int i = 0; i < c; ++i) cmask |= 1u << ids[comb[i]];
      int64_t sum = 0, mx = 0;
      for (int d = 0; d < D; ++d) {
        int64_t W = total[d];
        for (int i = 0; i < c; ++i) W -= w[comb[i] * D + d];
        sum += W;
        if (W > mx) mx = W;
      }
      const int size = n - c;
      const uint32_t mask = all & ~cmask;
      int better = !have;
      if (have) {
        if (u_greater(sum, mx, best_sum, best_max)) better = 1;
        else if (u_equal(sum, mx, best_sum, best_max))
          better = size > best_size || (size == best_size && mask < best_mask);
      }
      if (better) {
        have = 1;
        best_sum = sum;
        best_max = mx;
        best_size = size;
        best_mask = mask;
      }
      /* next combination in lexicographic order */
      int i = c - 1;
      while (i >= 0 && comb[i] == n - c + i) --i;
      if (i < 0) break;
      ++comb[i];
      for (int k = i + 1; k < c; ++k) comb[k] = comb[k - 1] + 1;
    }
  }
  return best_mask;
}

/* Forward enumeration: every mask over the n positions with at least m set
 * bits; W_d = sum of the member rows; the same order of candidates. */
uint32_t oracle_maxutil_plain(const int64_t* w, const int32_t* ids, int n, int D, int m) {
  uint32_t all = 0;
  for (int i = 0; i < n; ++i) all |= 1u << ids[i];
  if (n <= m) return all;
  int have = 0, best_size = 0;
  int64_t best_sum = 0, best_max = 0;
  uint32_t best_mask = 0;
  const uint64_t count = (uint64_t)1 << n;
  for (uint64_t s = 1; s < count; ++s) {
    int size = 0;
    uint32_t mask = 0;
    for (int i = 0; i < n; ++i)
      if ((s >> i) & 1u) {
        ++size;
        mask |= 1u << ids[i];
      }
    if (size < m) continue;
    int64_t sum = 0, mx = 0;
    for (int d = 0; d < D; ++d) {
      int64_t W = 0;
      for (int i = 0; i < n; ++i)
        if ((s >> i) & 1u) W += w[i * D + d];
      sum += W;
      if (W > mx) mx = W;
    }
    int better = !have;
    if (have) {
      if (u_greater(sum, mx, best_sum, best_max)) better = 1;
      else if (u_equal(sum, mx, best_sum, best_max))
        better = size > best_size || (size == best_size && mask < best_mask);
    }
    if (better) {
      have = 1;
      best_sum = sum;
      best_max = mx;
      best_size = size;
      best_mask = mask;
    }
  }
  return best_mask;
}
