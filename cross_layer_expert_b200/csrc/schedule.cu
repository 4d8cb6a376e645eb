// Loads, the RunSet scheduler, exact utilisation accounting and the segment
// plan of one step -- one CTA of 1024 threads, everything in shared memory.
//
// [EB] §2.3 Eq. (2) w_hat = max_d w_d, Eq. (3) u = sum sum w / (sum w_hat D);
// [EB] §4.2 Algorithm 1 and the minimum RunSet size m; [EB] §5.2 CumUtil
// (add j+1 iff U(S u {w_{j+1}}) > U(S)), MaxUtil (best U over the candidate
// subsets) and DiffPeak (add j+1 iff its peak device is new).
//
// U(S) = sum_d W_d / (D max_d W_d) is compared exactly:
//   U(A) > U(B)  <=>  sum_A * max_B > sum_B * max_A   (int64; D cancels),
// a set without work counts as U = 0.  MaxUtil ties go to the larger set,
// then to the smaller bitmask.  CumUtil and DiffPeak pad a short RunSet to m
// with the lowest skipped indices.
//
// MaxUtil enumerates the complements C of the pending set P with
// |C| <= |P| - m (so every candidate S = P \ C has |S| >= m).  Up to
// kWarpSearchMax candidates over at most 32 ranks, warp 0 searches them:
// with at most kMaskEnumMax pending micro-batches its lanes walk the
// complement bitmasks directly, above that they split the candidate ranks.
// Up to kBlockSearchMax candidates the scheduler's whole CTA splits them;
// above that a grid of kSearchCtas CTAs (k_maxutil_search) each searches a
// contiguous rank range and leaves its best candidate in a slot, and the
// scheduler reduces the slots.  A rank range is walked by unranking its
// first complement in colexicographic order and stepping on with Gosper's
// next-combination step.  The order on candidates is total, so no split
// changes the RunSet.
//
// The scheduler kernel runs once per step from a cold instruction cache;
// its time follows the size of the code it runs more than its arithmetic,
// so warp 0 does the serial parts with lane-parallel reductions, loops stay
// rolled, and the steps repeated per candidate or per segment are single
// out-of-line copies.
#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr int kThreads = 1024;

// Binomial coefficients C(a, b), 0 <= a, b <= 32, built at compile time
// (Pascal's rule) and placed in constant memory.
struct BinomTable {
  uint32_t v[33][33];
  constexpr BinomTable() : v() {
    for (int a = 0; a <= 32; ++a) {
      v[a][0] = 1;
      for (int b = 1; b <= 32; ++b) v[a][b] = a == 0 ? 0u : v[a - 1][b - 1] + v[a - 1][b];
    }
  }
};
__constant__ BinomTable kBinom = BinomTable();

// A MaxUtil candidate S = P \ C: (sum_d W_d, max_d W_d, |S|, C as a mask over
// positions in P).  size < 0 marks "no candidate".
struct Cand {
  long long sum, mx;
  int size;
  uint32_t cmask;
};

static_assert(sizeof(Cand) == kSearchSlotBytes, "search slot layout");

// Higher U first, then the larger set, then the smaller bitmask of
// micro-batch ids.  P lists ids in ascending order and C is a subset of P,
// so the RunSet's id mask is smaller exactly when its complement's position
// mask is larger.
__device__ __forceinline__ bool cand_better(const Cand& a, const Cand& b) {
  if (a.mx == 0 || b.mx == 0) {
    if (a.mx != b.mx) return a.mx != 0;  // a set with work beats one without
  } else {
    const long long l = a.sum * b.mx, r = b.sum * a.mx;
    if (l != r) return l > r;
  }
  if (a.size != b.size) return a.size > b.size;
  return a.cmask > b.cmask;
}

// a beats b, where either may be "no candidate"
__device__ __forceinline__ bool cand_wins(const Cand& a, const Cand& b) {
  return a.size >= 0 && (b.size < 0 || cand_better(a, b));
}

// Candidate counts up to this are searched by warp 0 alone; up to
// kMaskEnumMax pending micro-batches warp 0's lanes walk every complement
// bitmask directly instead of ranking the candidates.
constexpr unsigned long long kWarpSearchMax = 1024;
constexpr int kMaskEnumMax = 12;

// Row stride of the load rows in shared memory: odd, so threads reading the
// same rank of different micro-batches' rows hit different banks.
constexpr int kWStride = EB_MAX_D + 1;

// Candidate counts up to this are searched by the scheduler's own CTA.
constexpr unsigned long long kBlockSearchMax = 32768;

// Shared-memory workspace of the scheduler.
struct SchedSmem {
  int w[EB_MAX_M][kWStride];  // loads of pending micro-batches, by position in P
  long long wsum[EB_MAX_M];
  long long tot[EB_MAX_D];
  long long totsum;
  int P[EB_MAX_M];            // pending micro-batch ids, ascending
  int n;
  Cand red[kThreads / 32];
};

__device__ __forceinline__ uint64_t gosper_next(uint64_t v) {
  const uint64_t t = v | (v - 1);
  return (t + 1) | (((~t & (t + 1)) - 1) >> __ffsll((long long)v));
}

// The r-th c-subset of {0..n-1} in colexicographic order.
__device__ uint32_t unrank_colex(uint32_t r, int c, const uint32_t (*B)[33]) {
  uint32_t mask = 0;
  for (int i = c; i >= 1; --i) {
    int x = i - 1;
    while (B[x + 1][i] <= r) ++x;
    r -= B[x][i];
    mask |= 1u << x;
  }
  return mask;
}

__device__ Cand eval_complement(const SchedSmem& sm, int D, uint32_t cm) {
  long long mx = 0;
  long long sum = sm.totsum;
  for (uint32_t b = cm; b; b &= b - 1) sum -= sm.wsum[__ffs(b) - 1];
  for (int dd = 0; dd < D; ++dd) {
    long long Wd = sm.tot[dd];
    for (uint32_t b = cm; b; b &= b - 1) Wd -= sm.w[__ffs(b) - 1][dd];
    mx = Wd > mx ? Wd : mx;
  }
  return Cand{sum, mx, sm.n - __popc(cm), cm};
}

// RunSet id mask of a candidate.
__device__ uint32_t cand_runset(const SchedSmem& sm, const Cand& c) {
  uint32_t mask = 0;
  for (int i = 0; i < sm.n; ++i)
    if (!((c.cmask >> i) & 1u)) mask |= 1u << sm.P[i];
  return mask;
}

// Number of MaxUtil candidates of n pending micro-batches: complements of
// size 0 .. n - m.
__device__ unsigned long long candidate_count(int n, int m) {
  unsigned long long N = 0;
  for (int c = 0; c <= n - m; ++c) N += kBinom.v[n][c];
  return N;
}

// Loads and their sums stay below 2^31 (the configuration check bounds
// M * T * k), so a candidate crosses lanes as four 32-bit words.
__device__ Cand shfl_cand(const Cand& c, int off) {
  Cand o;
  o.sum = __shfl_xor_sync(0xffffffffu, (int)c.sum, off);
  o.mx = __shfl_xor_sync(0xffffffffu, (int)c.mx, off);
  o.size = __shfl_xor_sync(0xffffffffu, c.size, off);
  o.cmask = __shfl_xor_sync(0xffffffffu, c.cmask, off);
  return o;
}

// All lanes: the best of the warp's candidates, returned to every lane.
__device__ __noinline__ Cand warp_best(Cand best) {
#pragma unroll 1
  for (int off = 16; off; off >>= 1) {
    const Cand o = shfl_cand(best, off);
    if (cand_wins(o, best)) best = o;
  }
  return best;
}

// best := the better of best and the candidate S = P \ cm.
__device__ __noinline__ void consider(const SchedSmem& sm, int D, uint32_t cm, Cand& best) {
  const Cand cd = eval_complement(sm, D, cm);
  if (cand_wins(cd, best)) best = cd;
}

// All threads of the block: the best of every thread's `best` (threads
// without one pass size = -1).  Returns it to every thread.
__device__ Cand block_best(Cand best, Cand* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  best = warp_best(best);
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (warp == 0) {
    best = warp_best(lane < (int)(blockDim.x >> 5) ? red[lane] : Cand{0, 0, -1, 0});
    if (lane == 0) red[0] = best;
  }
  __syncthreads();
  best = red[0];
  __syncthreads();  // red may be reused
  return best;
}

// This thread's best candidate over the complement ranks [r_lo, r_hi)
// (sizes ascending, colexicographic order within a size), the range split
// evenly over `parts` searchers of which this is number `part`.
__device__ Cand search_ranks(const SchedSmem& sm, int D, unsigned long long r_lo,
                             unsigned long long r_hi, int part, int parts) {
  const int n = sm.n;
  const uint32_t (*B)[33] = kBinom.v;
  const unsigned long long N = r_hi > r_lo ? r_hi - r_lo : 0;
  const unsigned long long per = (N + parts - 1) / parts;
  unsigned long long r = r_lo + per * part;
  const unsigned long long r_end = r + per < r_hi ? r + per : r_hi;
  Cand best{0, 0, -1, 0};
  bool have = false;
  if (r < r_end) {
    int c = 0;
    unsigned long long q = r;
    while (q >= B[n][c]) {
      q -= B[n][c];
      ++c;
    }
    uint64_t cm = c == 0 ? 0 : unrank_colex((uint32_t)q, c, B);
    for (; r < r_end; ++r) {
      const Cand cd = eval_complement(sm, D, (uint32_t)cm);
      if (!have || cand_better(cd, best)) {
        best = cd;
        have = true;
      }
      if (++q == B[n][c]) {
        ++c;
        q = 0;
        cm = (c >= 64) ? 0 : ((1ull << c) - 1);
      } else {
        cm = gosper_next(cm);
      }
    }
  }
  return best;
}

// All threads of the block: MaxUtil over all complements of size <= n - m
// (up to kMaskEnumMax pending micro-batches each thread walks the bitmasks
// tid, tid + blockDim, ...; above, the candidate ranks are split).
__device__ uint32_t maxutil_block(SchedSmem& sm, int D, int m) {
  const int n = sm.n;
  Cand mine{0, 0, -1, 0};
  if (n <= kMaskEnumMax) {
    for (uint32_t cm = threadIdx.x; cm < (1u << n); cm += blockDim.x)
      if (__popc(cm) <= n - m) consider(sm, D, cm, mine);
  } else {
    mine = search_ranks(sm, D, 0, candidate_count(n, m), threadIdx.x, blockDim.x);
  }
  return cand_runset(sm, block_best(mine, sm.red));
}

// All threads of the block: the best of the search grid's slots.
__device__ uint32_t maxutil_slots(SchedSmem& sm, const Cand* __restrict__ slots, int n_slots) {
  Cand best{0, 0, -1, 0};
  for (int i = threadIdx.x; i < n_slots; i += blockDim.x) {
    const Cand c = slots[i];
    if (cand_wins(c, best)) best = c;
  }
  return cand_runset(sm, block_best(best, sm.red));
}

__device__ __forceinline__ long long warp_sum_ll(long long x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Warp 0: tot[d] = sum_i w_i[d], wsum[i] = sum_d w_i[d] and their total,
// lanes over ranks and over pending positions (n <= 32).
__device__ void warp_totals(SchedSmem& sm, int D) {
  const int lane = threadIdx.x & 31, n = sm.n;
  for (int dd = lane; dd < D; dd += 32) {
    long long t = 0;
    for (int i = 0; i < n; ++i) t += sm.w[i][dd];
    sm.tot[dd] = t;
  }
  long long ws = 0;
  if (lane < n) {
    for (int dd = 0; dd < D; ++dd) ws += sm.w[lane][dd];
    sm.wsum[lane] = ws;
  }
  ws = warp_sum_ll(ws);
  if (lane == 0) sm.totsum = ws;
  __syncwarp();
}

// All threads: the totals (warp 0), visible to the block.
__device__ void prepare_totals(SchedSmem& sm, int D) {
  if ((threadIdx.x >> 5) == 0) warp_totals(sm, D);
  __syncthreads();
}

// Warp 0: the RunSet (micro-batch ids) of a policy that needs no block-wide
// search, with the totals in place.  CumUtil walks the positions in order
// with the candidate's W_d spread over the lanes (d = lane, lane + 32); a
// step adds position i iff U(S u {i}) > U(S), compared exactly
// (nsum * mx > sum * nmx; a set without work has U = 0).  DiffPeak adds i
// iff its peak rank (lowest index of max_d w_i[d]) is the first occurrence
// of that rank among positions 0..i.  Both then pad to m with the lowest
// positions not taken.  MaxUtil splits the candidate ranks over the lanes.
// Warp 0, n <= kMaskEnumMax and D <= 32: MaxUtil over every complement
// bitmask with at most n - m bits, lane-strided; each candidate's W_d
// (d < D <= DMAX) is summed in registers, so a complement's rows are read
// with independent loads.
template <int DMAX>
__device__ __noinline__ Cand warp_maxutil_masks(const SchedSmem& sm, int D, int m) {
  const int lane = threadIdx.x & 31, n = sm.n, cmax = n - m;
  Cand best{0, 0, -1, 0};
  for (uint32_t cm = lane; cm < (1u << n); cm += 32) {
    if (__popc(cm) > cmax) continue;
    int W[DMAX];
    long long sum = sm.totsum;
#pragma unroll
    for (int d = 0; d < DMAX; ++d) W[d] = d < D ? (int)sm.tot[d] : 0;
    for (uint32_t b = cm; b; b &= b - 1) {
      const int i = __ffs(b) - 1;
      sum -= sm.wsum[i];
#pragma unroll
      for (int d = 0; d < DMAX; ++d)
        if (d < D) W[d] -= sm.w[i][d];
    }
    int mx = 0;
#pragma unroll
    for (int d = 0; d < DMAX; ++d) mx = W[d] > mx ? W[d] : mx;
    const Cand cd{sum, (long long)mx, n - __popc(cm), cm};
    if (cand_wins(cd, best)) best = cd;
  }
  return warp_best(best);
}

__device__ uint32_t warp_choose(SchedSmem& sm, int D, int m, int policy, uint32_t pending) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31, n = sm.n;
  if (policy == EB_SCHED_LOCKSTEP || n <= m) return pending;
  if (policy == EB_SCHED_MAXUTIL) {
    warp_totals(sm, D);
    Cand best{0, 0, -1, 0};
    if (n <= kMaskEnumMax && D <= 32) {
      best = D <= 8    ? warp_maxutil_masks<8>(sm, D, m)
             : D <= 16 ? warp_maxutil_masks<16>(sm, D, m)
                       : warp_maxutil_masks<32>(sm, D, m);
    } else {
      best = warp_best(search_ranks(sm, D, 0, candidate_count(n, m), lane, 32));
    }
    return cand_runset(sm, best);
  }
  uint32_t chosen;  // positions in P
  if (policy == EB_SCHED_DIFFPEAK) {
    int peak = -1 - lane;  // distinct keys for lanes without a position
    if (lane < n) {
      peak = 0;
      for (int dd = 1; dd < D; ++dd)
        if (sm.w[lane][dd] > sm.w[lane][peak]) peak = dd;
    }
    const unsigned same = __match_any_sync(kFull, peak);
    chosen = __ballot_sync(kFull, lane < n && (__ffs(same) - 1) == lane);
  } else {
    warp_totals(sm, D);
    const int d0 = lane, d1 = lane + 32;
    int W0 = d0 < D ? sm.w[0][d0] : 0, W1 = d1 < D ? sm.w[0][d1] : 0;
    long long sum = sm.wsum[0];
    long long mx = __reduce_max_sync(kFull, W0 > W1 ? W0 : W1);
    chosen = 1u;
    // the next row's loads are issued one step ahead
    int x0 = n > 1 && d0 < D ? sm.w[1][d0] : 0, x1 = n > 1 && d1 < D ? sm.w[1][d1] : 0;
    long long xs = n > 1 ? sm.wsum[1] : 0;
    for (int i = 1; i < n; ++i) {
      const int c0 = x0, c1 = x1;
      const long long cs = xs;
      if (i + 1 < n) {
        x0 = d0 < D ? sm.w[i + 1][d0] : 0;
        x1 = d1 < D ? sm.w[i + 1][d1] : 0;
        xs = sm.wsum[i + 1];
      }
      const int v0 = W0 + c0, v1 = W1 + c1;
      const long long nmx = __reduce_max_sync(kFull, v0 > v1 ? v0 : v1);
      const long long nsum = sum + cs;
      bool gain;
      if (nmx == 0 || mx == 0) gain = (nmx != 0 && mx == 0);
      else gain = nsum * mx > sum * nmx;
      if (gain) {
        chosen |= 1u << i;
        W0 = v0;
        W1 = v1;
        sum = nsum;
        mx = nmx;
      }
    }
  }
  const uint32_t posmask = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
  const int need = m - __popc(chosen);
  if (need > 0 && lane < n && !((chosen >> lane) & 1u) &&
      __popc(~chosen & posmask & ((1u << lane) - 1u)) < need)
    chosen |= 1u << lane;
  chosen = __reduce_or_sync(kFull, chosen);
  return __reduce_or_sync(kFull, (lane < n && ((chosen >> lane) & 1u)) ? 1u << sm.P[lane] : 0u);
}


// All threads, with sm.P, sm.n and the pending rows sm.w (by position) in
// place.  Returns the RunSet (micro-batch ids) to warp 0; the other threads'
// return value is unspecified.  slots: the MaxUtil search grid's results for
// this pending set (null: search here).  Only a large MaxUtil search, or
// one over more than 32 ranks, uses the whole block.
__device__ uint32_t choose_runset(SchedSmem& sm, int D, int m, int policy, uint32_t pending,
                                  const Cand* slots) {
  const int n = sm.n;
  if (policy == EB_SCHED_MAXUTIL && n > m &&
      (slots != nullptr || candidate_count(n, m) > kWarpSearchMax || D > 32)) {
    prepare_totals(sm, D);
    return slots ? maxutil_slots(sm, slots, kSearchCtas) : maxutil_block(sm, D, m);
  }
  if ((threadIdx.x >> 5) != 0) return 0u;
  return warp_choose(sm, D, m, policy, pending);
}

// Warp 0: the step's exact accounting -- sum_d W_d, max_d W_d of the RunSet
// and the sum over its members of their own peaks (Eq. (3) numerator and
// the scheduled and separate denominators / D).
__device__ void warp_account(const SchedSmem& sm, int D, uint32_t run, long long& sumW,
                             long long& maxW, long long& summax) {
  constexpr unsigned kFull = 0xffffffffu;
  const int lane = threadIdx.x & 31, n = sm.n;
  // positions in P of the RunSet's members
  const uint32_t rpos = __ballot_sync(kFull, lane < n && ((run >> sm.P[lane]) & 1u));
  unsigned s = 0;
  int mxw = 0;
  for (int dd = lane; dd < D; dd += 32) {
    int Wd = 0;
    for (uint32_t b = rpos; b; b &= b - 1) Wd += sm.w[__ffs(b) - 1][dd];
    s += (unsigned)Wd;
    mxw = Wd > mxw ? Wd : mxw;
  }
  unsigned own = 0;
  if ((rpos >> lane) & 1u) {
    int mx = 0;
    for (int dd = 0; dd < D; ++dd) mx = sm.w[lane][dd] > mx ? sm.w[lane][dd] : mx;
    own = (unsigned)mx;
  }
  sumW = __reduce_add_sync(kFull, s);
  maxW = __reduce_max_sync(kFull, mxw);
  summax = __reduce_add_sync(kFull, own);
}

// All threads: sm.P / sm.n from the pending mask, and the pending rows of
// sm.w (loaded by micro-batch id) moved to their positions (P ascending,
// so row p reads row P[p] >= p; every thread reads before any writes).
// Blocks of kThreads threads.
__device__ void compact_rows(SchedSmem& sm, uint32_t pending, int M, int D) {
  constexpr int kPer = (EB_MAX_M * EB_MAX_D) / 1024;
  const int tid = threadIdx.x;
  int val[kPer], dst[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int i = tid + q * kThreads;
    dst[q] = -1;
    if (i < M * D) {
      const int j = i / D, dd = i % D;
      if ((pending >> j) & 1u) {
        dst[q] = __popc(pending & ((1u << j) - 1u)) * kWStride + dd;
        val[q] = sm.w[j][dd];
      }
    }
  }
  if (tid < M && ((pending >> tid) & 1u)) sm.P[__popc(pending & ((1u << tid) - 1u))] = tid;
  if (tid == 0) sm.n = __popc(pending);
  __syncthreads();
#pragma unroll
  for (int q = 0; q < kPer; ++q)
    if (dst[q] >= 0) (&sm.w[0][0])[dst[q]] = val[q];
  __syncthreads();
}


// Expert counts of every micro-batch, kept in shared memory by the plan
// (M * E <= EB_MAX_M * EB_MAX_ETOT int32: 32 KiB).
constexpr int kPlanHistCache = EB_MAX_M * EB_MAX_ETOT;

constexpr int kSearchThreads = 256;

// The same search as search_ranks, for the grid: each thread keeps its
// current complement's W_d (d < D <= DMAX) in registers and updates it by
// the rows that enter or leave the complement between neighbours in
// Gosper's order (about two rows per step), instead of re-summing every
// member's row for every candidate.  W_d <= sum of all loads < 2^31.
template <int DMAX>
__device__ Cand search_ranks_inc(const SchedSmem& sm, int D, unsigned long long r_lo,
                                 unsigned long long r_hi) {
  const int n = sm.n;
  const uint32_t (*B)[33] = kBinom.v;
  const unsigned long long N = r_hi > r_lo ? r_hi - r_lo : 0;
  const unsigned long long per = (N + blockDim.x - 1) / blockDim.x;
  unsigned long long r = r_lo + per * threadIdx.x;
  const unsigned long long r_end = r + per < r_hi ? r + per : r_hi;
  Cand best{0, 0, -1, 0};
  if (r >= r_end) return best;
  int c = 0;
  unsigned long long q = r;
  while (q >= B[n][c]) {
    q -= B[n][c];
    ++c;
  }
  uint32_t cm = c == 0 ? 0u : unrank_colex((uint32_t)q, c, B);
  int W[DMAX];
  long long sum;
  auto load_full = [&]() {  // W and sum of the complement cm from scratch
    sum = sm.totsum;
#pragma unroll
    for (int d = 0; d < DMAX; ++d) W[d] = d < D ? (int)sm.tot[d] : 0;
    for (uint32_t b = cm; b; b &= b - 1) {
      const int i = __ffs(b) - 1;
      sum -= sm.wsum[i];
#pragma unroll
      for (int d = 0; d < DMAX; ++d)
        if (d < D) W[d] -= sm.w[i][d];
    }
  };
  load_full();
  bool have = false;
  for (;;) {
    int mx = 0;
#pragma unroll
    for (int d = 0; d < DMAX; ++d) mx = W[d] > mx ? W[d] : mx;
    const Cand cd{sum, (long long)mx, n - c, cm};
    if (!have || cand_better(cd, best)) {
      best = cd;
      have = true;
    }
    if (++r == r_end) break;
    if (++q == B[n][c]) {  // next size: its first combination, from scratch
      ++c;
      q = 0;
      cm = (1u << c) - 1u;
      load_full();
    } else {
      const uint32_t nx = (uint32_t)gosper_next(cm);
      for (uint32_t b = cm ^ nx; b; b &= b - 1) {
        const int i = __ffs(b) - 1;
        const int sgn = ((nx >> i) & 1u) ? -1 : 1;  // enters the complement: leaves S
        sum += sgn * sm.wsum[i];
#pragma unroll
        for (int d = 0; d < DMAX; ++d)
          if (d < D) W[d] += sgn * sm.w[i][d];
      }
      cm = nx;
    }
  }
  return best;
}

// MaxUtil search grid: CTA b searches complement ranks [N b / G, N (b+1) / G)
// of the pending set (N candidates, G = gridDim.x) and writes its best
// candidate (or "none") to slots[b].  The pending set and loads are the
// step state's (st != null; nothing is searched while a timed-out step
// awaits a reset) or the caller's (pending_arg, w).
template <int DMAX>
__global__ void __launch_bounds__(kSearchThreads) k_maxutil_search(int M, int D, int m,
                                                                   const State* __restrict__ st,
                                                                   uint32_t pending_arg,
                                                                   const int32_t* __restrict__ w,
                                                                   Cand* __restrict__ slots) {
  __shared__ SchedSmem sm;
  pdl_enter();
  const int tid = threadIdx.x;
  if (tid == 0) {
    const uint32_t pending =
        st ? (st->status == EB_ERR_TIMEOUT ? 0u : st->pending) : pending_arg;
    int n = 0;
    for (int j = 0; j < M; ++j)
      if ((pending >> j) & 1u) sm.P[n++] = j;
    sm.n = n;
  }
  __syncthreads();
  Cand best{0, 0, -1, 0};
  if (sm.n > m) {
    for (int i = tid; i < sm.n * D; i += blockDim.x) {
      const int p = i / D, dd = i % D;
      sm.w[p][dd] = w[sm.P[p] * D + dd];
    }
    __syncthreads();
    prepare_totals(sm, D);
    const unsigned long long N = candidate_count(sm.n, m), G = gridDim.x;
    best = search_ranks_inc<DMAX>(sm, D, N * blockIdx.x / G, N * (blockIdx.x + 1) / G);
  }
  best = block_best(best, sm.red);
  if (tid == 0) slots[blockIdx.x] = best;
}

// Work items of a segment of n rows: ceil(n / rows per item) * feature blocks.
__device__ __noinline__ int items_of(int n, int rn, int mb) { return (n + rn - 1) / rn * mb; }

// All threads: zero the counts and loads of the micro-batches routed at
// the next step (warp j clears row j).
__device__ void zero_next(const Dims& d, const CtxDev& c, uint32_t next) {
  const int lane = threadIdx.x & 31;
  for (int j = threadIdx.x >> 5; j < d.M; j += kThreads / 32)
    if ((next >> j) & 1u) {
      for (int e = lane; e < d.E; e += 32) c.hist[j * d.E + e] = 0;
      for (int r = lane; r < d.D; r += 32) c.w[j * d.D + r] = 0;
    }
}

// view: this step's StepView slot, written for the step's combine.
__global__ void __launch_bounds__(kThreads) k_schedule_step(Dims d, CtxDev c, Work wk, int rn1,
                                                             int rn2, int fm1, int fm2,
                                                             StepView* __restrict__ view) {
  __shared__ SchedSmem sm;
  // the step state lives in shared memory for the whole kernel
  __shared__ State ss;
  __shared__ int s_hist[kPlanHistCache];  // hist[j][e] of every micro-batch, by id
  State* st = &ss;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_enter();
  // 1. one round of global loads: the state, the loads w[j][:] of every
  //    micro-batch (by id) and, for the plan, the expert counts hist[j][:]
  //    accumulated by the routing kernel
  constexpr int kStateWords = sizeof(State) / sizeof(int);
  for (int i = tid; i < kStateWords; i += kThreads)
    reinterpret_cast<int*>(&ss)[i] = reinterpret_cast<const int*>(c.st)[i];
  for (int i = tid; i < d.M * d.D; i += kThreads) sm.w[i / d.D][i % d.D] = c.w[i];
  if (d.compute)
    for (int i = tid; i < d.M * d.E; i += kThreads) s_hist[i] = c.hist[i];
  __syncthreads();
  // the micro-batches routed for this step wrote their gates into the
  // buffers their gate_buf bits did not name: from now on those hold them
  if (tid == 0) {
    ss.gate_buf ^= ss.need_route;
    ss.sched_calls += 1u;
  }
  // the state goes back to global memory; then S and the launch count go to
  // the host's mapped words, S first (the host reads the count, then S)
  auto write_back = [&]() {
    __syncthreads();
    for (int i = tid; i < kStateWords; i += kThreads)
      reinterpret_cast<int*>(c.st)[i] = reinterpret_cast<const int*>(&ss)[i];
    if (tid == 0 && c.host_flag) {
      c.host_flag[0] = ss.pending;
      __threadfence_system();
      c.host_flag[1] = ss.sched_calls;
    }
  };
  auto finish_empty = [&]() {
    if (tid == 0) {
      view->n_run = 0;
      view->next = 0;
      st->pending = ss.status == EB_ERR_TIMEOUT ? 0u : st->pending;
      st->runset = 0;
      st->n_run = 0;
      st->need_route = 0;
      st->nseg = 0;
      st->items1 = 0;
      st->items2 = 0;
      st->rows = 0;
      for (int j = 0; j < d.M; ++j) st->step_layer[j] = -1;
    }
    write_back();
  };
  // A context whose status word holds EB_ERR_TIMEOUT (a bounded wait of an
  // earlier step expired, so its state may be partial) runs no further step
  // until eb_reset: the step does nothing and reports S as empty.  A step
  // with S empty (episode finished) does nothing either.
  const uint32_t pending = ss.pending;
  if (ss.status == EB_ERR_TIMEOUT || pending == 0u) {
    finish_empty();
    return;
  }
  // 2. pending set: positions in P and the pending rows of w by position
  compact_rows(sm, pending, d.M, d.D);
  // 3. RunSet (in warp 0)
  const uint32_t run = choose_runset(sm, d.D, d.m, d.policy, pending,
                                     static_cast<const Cand*>(c.search_slots));
  // 4. accounting, trace and Algorithm 1 bookkeeping (warp 0: lane j is
  //    micro-batch j, M <= 32)
  __shared__ int s_group_run[EB_MAX_M];  // group of RunSet member a
  if (warp == 0) {
    long long sumW, maxW, summax;
    warp_account(sm, d.D, run, sumW, maxW, summax);
    const int step = st->n_steps;
    const int j = lane;
    const bool inrun = j < d.M && ((run >> j) & 1u);
    const int lj = j < d.M ? st->layer[j] : 0;  // l_j before this step
    if (step < d.max_steps) {
      if (lane == 0) {
        c.trace[step * kTraceCols + 0] = run;
        c.trace[step * kTraceCols + 1] = sumW;
        c.trace[step * kTraceCols + 2] = maxW;
        c.trace[step * kTraceCols + 3] = summax;
        c.trace[step * kTraceCols + 4] = 0;
        c.trace[step * kTraceCols + 5] = 0;
      }
      if (j < d.M) c.trace_layers[step * d.M + j] = inrun ? lj : -1;
    }
    const int nl = lj + (inrun ? 1 : 0);
    const uint32_t still = __ballot_sync(0xffffffffu, j < d.M && nl < d.L);
    // segment groups: the distinct layers of the RunSet, ascending; lane j's
    // group is the number of distinct RunSet layers below l_j
    const unsigned same = __match_any_sync(0xffffffffu, inrun ? lj : -1 - lane);
    const bool leader = inrun && (__ffs(same) - 1) == lane;
    const uint32_t leaders = __ballot_sync(0xffffffffu, leader);
    int g = 0;
    for (uint32_t b = leaders; b; b &= b - 1) {
      const int li = __shfl_sync(0xffffffffu, lj, __ffs(b) - 1);
      g += li < lj;
    }
    __syncwarp();  // every lane has read n_steps and l_j before they change
    if (j < d.M) {
      st->step_layer[j] = inrun ? lj : -1;
      st->layer[j] = nl;
    }
    if (inrun) {
      const int a = __popc(run & ((1u << j) - 1u));
      st->run_list[a] = j;
      st->group_of[j] = g;
      s_group_run[a] = g;
      view->run_list[a] = j;
    }
    if (leader) st->group_layer[g] = lj;
    if (lane == 0) {
      view->n_run = __popc(run);
      view->gate_buf = ss.gate_buf;
      view->next = 0;
      st->num += sumW;
      st->den += (long long)d.D * maxW;
      st->den_sep += (long long)d.D * summax;
      st->n_steps = step + 1;
      st->n_run = __popc(run);
      st->runset = run;
      st->pending = still;
      st->need_route = run & still;
      st->n_groups = __popc(leaders);
      st->nseg = __popc(leaders) * d.Etot;
    }
  }
  __syncthreads();
  if (!d.compute) {
    zero_next(d, c, st->need_route);
    write_back();
    return;
  }
  // 5. segment plan, one warp per segment group (G <= 32 warps).  Lane l of
  //    warp g holds the segments (g, e) for e in [l Q, (l + 1) Q), Q =
  //    ceil(Et / 32).  The warp walks the group's members in RunSet order:
  //    prior[j][e] is the running count before member j and the final count
  //    is the segment's rows.  Items per segment follow, a warp scan gives
  //    the offsets inside the group's row, and after one barrier a scan of
  //    the G row totals gives each row's base.  The kernel runs once per
  //    step from a cold instruction cache, so its loops stay rolled: code
  //    size, not arithmetic, sets the time of this single-CTA kernel.
  const int G = st->n_groups, nr = st->n_run, Et = d.Etot, nseg = G * Et;
  const int mb1 = d.F / fm1, mb2 = d.H / fm2;
  constexpr int kQ = EB_MAX_ETOT / 32;
  const int Q = (Et + 31) / 32, e0 = lane * Q;
  __shared__ int4 s_rowtot[EB_MAX_M];  // rows, items1, items2, non-empty segments of each group
  int cnt[kQ];
  int3 mine = make_int3(0, 0, 0);  // this lane's sums of rows, items1, items2
  if (warp < G) {
#pragma unroll 1
    for (int q = 0; q < Q; ++q) cnt[q] = 0;
    for (int a = 0; a < nr; ++a) {
      if (s_group_run[a] != warp) continue;  // warp-uniform
      const int j = st->run_list[a];
      const int* hj = s_hist + j * d.E;
      int32_t* pj = wk.prior + j * Et;
#pragma unroll 1
      for (int q = 0; q < Q; ++q) {
        const int e = e0 + q;
        if (e < Et) {
          pj[e] = cnt[q];
          cnt[q] += e < d.E ? hj[e] : d.T;  // a shared expert takes every token
        }
      }
    }
    int nonempty = 0;
#pragma unroll 1
    for (int q = 0; q < Q; ++q) {
      const int e = e0 + q;
      if (e < Et) {
        mine.x += cnt[q];
        mine.y += items_of(cnt[q], rn1, mb1);
        mine.z += items_of(cnt[q], rn2, mb2);
        nonempty += cnt[q] > 0;
        wk.seg_wid[warp * Et + e] = st->group_layer[warp] * Et + e;
      }
    }
    // inclusive warp scan of the lanes' sums; lane 31 holds the row's totals
    int3 inc = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, inc.x, off);
      const int y = __shfl_up_sync(0xffffffffu, inc.y, off);
      const int z = __shfl_up_sync(0xffffffffu, inc.z, off);
      if (lane >= off) {
        inc.x += x;
        inc.y += y;
        inc.z += z;
      }
    }
    nonempty = __reduce_add_sync(0xffffffffu, nonempty);
    if (lane == 31) s_rowtot[warp] = make_int4(inc.x, inc.y, inc.z, nonempty);
    mine = make_int3(inc.x - mine.x, inc.y - mine.y, inc.z - mine.z);  // exclusive
  }
  __syncthreads();
  if (warp < G) {
    // base of row g: the totals of rows 0..g-1 (lane r holds row r's)
    int4 t = lane < G ? s_rowtot[lane] : make_int4(0, 0, 0, 0);
    int4 inc = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, inc.x, off);
      const int y = __shfl_up_sync(0xffffffffu, inc.y, off);
      const int z = __shfl_up_sync(0xffffffffu, inc.z, off);
      const int w = __shfl_up_sync(0xffffffffu, inc.w, off);
      if (lane >= off) {
        inc.x += x;
        inc.y += y;
        inc.z += z;
        inc.w += w;
      }
    }
    const int bx = __shfl_sync(0xffffffffu, inc.x - t.x, warp);
    const int by = __shfl_sync(0xffffffffu, inc.y - t.y, warp);
    const int bz = __shfl_sync(0xffffffffu, inc.z - t.z, warp);
    int3 acc3 = make_int3(bx + mine.x, by + mine.y, bz + mine.z);
#pragma unroll 1
    for (int q = 0; q < Q; ++q) {
      const int e = e0 + q;
      if (e < Et) {
        const int i = warp * Et + e;
        wk.seg_rows[i] = acc3.x;
        wk.seg_items1[i] = acc3.y;
        wk.seg_items2[i] = acc3.z;
        acc3.x += cnt[q];
        acc3.y += items_of(cnt[q], rn1, mb1);
        acc3.z += items_of(cnt[q], rn2, mb2);
      }
    }
    if (warp == 0) {
      // every row's totals: lane G - 1's inclusive sums
      const int rows = __shfl_sync(0xffffffffu, inc.x, G - 1);
      const int it1 = __shfl_sync(0xffffffffu, inc.y, G - 1);
      const int it2 = __shfl_sync(0xffffffffu, inc.z, G - 1);
      const int ne = __shfl_sync(0xffffffffu, inc.w, G - 1);
      if (lane == 0) {
        wk.seg_rows[nseg] = rows;
        wk.seg_items1[nseg] = it1;
        wk.seg_items2[nseg] = it2;
        st->rows = rows;
        st->items1 = it1;
        st->items2 = it2;
        wk.gemm_next[0] = 0;
        wk.gemm_next[1] = 0;
        const int step = st->n_steps - 1;  // the row written above
        if (step < d.max_steps) {
          c.trace[step * kTraceCols + 4] = rows;
          c.trace[step * kTraceCols + 5] = ne;
        }
      }
    }
  }
  // the micro-batches routed at the next step start from zero counts (the
  // counts of this step were read into shared memory above)
  zero_next(d, c, st->need_route);
  write_back();
}

__global__ void __launch_bounds__(kThreads) k_schedule_once(const int32_t* __restrict__ w,
                                                             uint32_t pending, int M, int D,
                                                             int m, int policy,
                                                             uint32_t* __restrict__ runset_out,
                                                             long long* __restrict__ stats,
                                                             const Cand* __restrict__ slots) {
  __shared__ SchedSmem sm;
  const int tid = threadIdx.x;
  if (pending == 0u) {
    if (tid == 0) {
      *runset_out = 0;
      if (stats) stats[0] = stats[1] = stats[2] = 0;
    }
    return;
  }
  for (int i = tid; i < M * D; i += kThreads) sm.w[i / D][i % D] = w[i];
  __syncthreads();
  compact_rows(sm, pending, M, D);
  const uint32_t run = choose_runset(sm, D, m, policy, pending, slots);
  if ((tid >> 5) == 0) {
    long long sumW, maxW, summax;
    warp_account(sm, D, run, sumW, maxW, summax);
    if (tid == 0) {
      *runset_out = run;
      if (stats) {
        stats[0] = sumW;
        stats[1] = maxW;
        stats[2] = summax;
      }
    }
  }
}

__global__ void k_loads(const int32_t* __restrict__ hist, int M, int E, int D,
                        const int32_t* __restrict__ expert_rank, int32_t* __restrict__ w,
                        int32_t* __restrict__ status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * D) return;
  const int j = i / D, dd = i % D;
  int s = 0;
  if (expert_rank) {  // custom placement: the experts whose rank is dd
    for (int e = 0; e < E; ++e) {
      const int r = expert_rank[e];
      if (r == dd) s += hist[j * E + e];
      else if ((r < 0 || r >= D) && dd == 0 && status) atomicExch(status, EB_ERR_INVALID_ARG);
    }
  } else {
    const int per = E / D;
    for (int e = dd * per; e < (dd + 1) * per; ++e) s += hist[j * E + e];
  }
  w[i] = s;
}

__global__ void k_reset(Dims d, CtxDev c) {
  pdl_enter();
  State* st = c.st;
  for (int i = threadIdx.x; i < d.M * d.E; i += blockDim.x) c.hist[i] = 0;
  for (int i = threadIdx.x; i < d.M * d.D; i += blockDim.x) c.w[i] = 0;
  // a routing launch cut short may have left tickets behind
  for (int i = threadIdx.x; i < d.M; i += blockDim.x) c.tickets[i] = 0;
  if (threadIdx.x != 0) return;
  const uint32_t all = d.M >= 32 ? 0xffffffffu : ((1u << d.M) - 1u);
  for (int j = 0; j < EB_MAX_M; ++j) {
    st->layer[j] = 0;
    st->step_layer[j] = -1;
    st->run_list[j] = 0;
    st->group_of[j] = 0;
    st->group_layer[j] = 0;
  }
  st->pending = d.L > 0 ? all : 0u;
  st->need_route = st->pending;
  st->runset = 0;
  st->n_run = 0;
  st->n_groups = 0;
  st->n_steps = 0;
  st->status = EB_OK;
  st->gate_buf = 0;
  st->nseg = 0;
  st->items1 = st->items2 = 0;
  st->rows = 0;
  st->num = st->den = st->den_sep = 0;
}

}  // namespace

unsigned long long maxutil_candidates(int n, int m) {
  if (n <= m) return 1;
  unsigned long long total = 0, b = 1;  // b = C(n, c)
  for (int c = 0; c <= n - m; ++c) {
    total += b;
    b = b * (unsigned long long)(n - c) / (unsigned long long)(c + 1);
  }
  return total;
}

bool maxutil_uses_grid(int n, int m) { return maxutil_candidates(n, m) > kBlockSearchMax; }

cudaError_t launch_schedule_step(const Dims& d, const CtxDev& c, const Work& w, int rn1, int rn2,
                                 int fm1, int fm2, int slot, cudaStream_t s) {
  if (c.search_slots) {
    auto go = [&](auto kernel) {
      return launch_pdl(kernel, dim3(kSearchCtas), dim3(kSearchThreads), 0, s, 1, d.M, d.D, d.m,
                        (const State*)c.st, 0u, (const int32_t*)c.w,
                        static_cast<Cand*>(c.search_slots));
    };
    const cudaError_t e = d.D <= 8    ? go(k_maxutil_search<8>)
                          : d.D <= 16 ? go(k_maxutil_search<16>)
                          : d.D <= 32 ? go(k_maxutil_search<32>)
                                      : go(k_maxutil_search<64>);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(k_schedule_step, dim3(1), dim3(kThreads), 0, s, 1, d, c, w, rn1, rn2, fm1, fm2,
                    w.views + slot);
}

cudaError_t launch_schedule_once(const int32_t* w, uint32_t pending, int M, int D, int m,
                                 int policy, uint32_t* runset, long long* stats, void* slots,
                                 cudaStream_t s) {
  if (slots) {
    auto go = [&](auto kernel) {
      kernel<<<kSearchCtas, kSearchThreads, 0, s>>>(M, D, m, nullptr, pending, w,
                                                     static_cast<Cand*>(slots));
    };
    if (D <= 8) go(k_maxutil_search<8>);
    else if (D <= 16) go(k_maxutil_search<16>);
    else if (D <= 32) go(k_maxutil_search<32>);
    else go(k_maxutil_search<64>);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  k_schedule_once<<<1, kThreads, 0, s>>>(w, pending, M, D, m, policy, runset, stats,
                                         static_cast<const Cand*>(slots));
  return cudaGetLastError();
}

cudaError_t launch_loads(const int32_t* hist, int M, int E, int D, const int32_t* expert_rank,
                         int32_t* w, int32_t* status, cudaStream_t s) {
  const int n = M * D;
  if (n == 0) return cudaSuccess;
  k_loads<<<(n + 255) / 256, 256, 0, s>>>(hist, M, E, D, expert_rank, w, status);
  return cudaGetLastError();
}

__global__ void k_set_status(State* st, int status) {
  pdl_enter();
  st->status = status;
}

cudaError_t launch_set_status(State* st, int status, cudaStream_t s) {
  return launch_pdl(k_set_status, dim3(1), dim3(1), 0, s, 1, st, status);
}

cudaError_t launch_reset(const Dims& d, const CtxDev& c, cudaStream_t s) {
  return launch_pdl(k_reset, dim3(1), dim3(1024), 0, s, 1, d, c);
}

}  // namespace eb
