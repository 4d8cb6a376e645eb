// Loads, the RunSet scheduler, exact utilisation accounting and the segment
// plan of one step -- one CTA, everything in shared memory.
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
// |C| <= |P| - m (so every candidate S = P \ C has |S| >= m): the threads
// split the candidate ranks, unrank a first complement in colexicographic
// order and walk on with Gosper's next-combination step.  Up to
// kBlockSearchMax candidates the scheduler's own CTA searches them; above
// that a grid of kSearchCtas CTAs (k_maxutil_search) each searches a
// contiguous rank range and leaves its best candidate in a slot, and the
// scheduler reduces the slots.  The order on candidates is total, so the
// split never changes the RunSet.
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
  uint32_t result;
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

__device__ Cand shfl_cand(const Cand& c, int off) {
  Cand o;
  o.sum = __shfl_xor_sync(0xffffffffu, c.sum, off);
  o.mx = __shfl_xor_sync(0xffffffffu, c.mx, off);
  o.size = __shfl_xor_sync(0xffffffffu, c.size, off);
  o.cmask = __shfl_xor_sync(0xffffffffu, c.cmask, off);
  return o;
}

// All threads of the block: the best of every thread's `best` (threads
// without one pass size = -1).  Returns it to every thread.
__device__ Cand block_best(Cand best, Cand* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int off = 16; off; off >>= 1) {
    const Cand o = shfl_cand(best, off);
    if (cand_wins(o, best)) best = o;
  }
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (warp == 0) {
    best = lane < (int)(blockDim.x >> 5) ? red[lane] : Cand{0, 0, -1, 0};
    for (int off = 16; off; off >>= 1) {
      const Cand o = shfl_cand(best, off);
      if (cand_wins(o, best)) best = o;
    }
    if (lane == 0) red[0] = best;
  }
  __syncthreads();
  best = red[0];
  __syncthreads();  // red may be reused
  return best;
}

// This thread's best candidate over the complement ranks [r_lo, r_hi)
// (sizes ascending, colexicographic order within a size), the range split
// evenly over the block's threads.
__device__ Cand search_ranks(const SchedSmem& sm, int D, int m, unsigned long long r_lo,
                             unsigned long long r_hi) {
  const int n = sm.n;
  const uint32_t (*B)[33] = kBinom.v;
  const unsigned long long N = r_hi > r_lo ? r_hi - r_lo : 0;
  const unsigned long long per = (N + blockDim.x - 1) / blockDim.x;
  unsigned long long r = r_lo + per * threadIdx.x;
  const unsigned long long r_end = r + per < r_hi ? r + per : r_hi;
  Cand best{0, 0, -1, 0};
  bool have = false;
  (void)m;
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

// All threads of the block: MaxUtil over all complements of size <= n - m.
__device__ uint32_t maxutil_block(SchedSmem& sm, int D, int m) {
  const Cand best = block_best(search_ranks(sm, D, m, 0, candidate_count(sm.n, m)), sm.red);
  return cand_runset(sm, best);
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

// Thread 0 only: CumUtil (policy 0) or DiffPeak (policy 3), padded to m.
__device__ uint32_t scan_policy(const SchedSmem& sm, int D, int m, int policy) {
  const int n = sm.n;
  long long W[EB_MAX_D];
  for (int dd = 0; dd < D; ++dd) W[dd] = sm.w[0][dd];
  long long sum = sm.wsum[0], mx = 0;
  for (int dd = 0; dd < D; ++dd) mx = W[dd] > mx ? W[dd] : mx;
  uint32_t chosen = 1u;  // positions in P
  unsigned long long peaks = 0;
  auto peak_of = [&](int i) {
    int best = 0;
    for (int dd = 1; dd < D; ++dd)
      if (sm.w[i][dd] > sm.w[i][best]) best = dd;
    return best;
  };
  if (policy == EB_SCHED_DIFFPEAK) peaks = 1ull << peak_of(0);
  for (int i = 1; i < n; ++i) {
    if (policy == EB_SCHED_DIFFPEAK) {
      const int p = peak_of(i);
      if (!((peaks >> p) & 1ull)) {
        peaks |= 1ull << p;
        chosen |= 1u << i;
      }
      continue;
    }
    long long nmx = 0;
    for (int dd = 0; dd < D; ++dd) {
      const long long v = W[dd] + sm.w[i][dd];
      nmx = v > nmx ? v : nmx;
    }
    const long long nsum = sum + sm.wsum[i];
    // U(S u {i}) > U(S) <=> nsum * mx > sum * nmx; a set without work has U = 0
    bool gain;
    if (nmx == 0 || mx == 0) gain = (nmx != 0 && mx == 0);
    else gain = nsum * mx > sum * nmx;
    if (gain) {
      chosen |= 1u << i;
      for (int dd = 0; dd < D; ++dd) W[dd] += sm.w[i][dd];
      sum = nsum;
      mx = nmx;
    }
  }
  for (int i = 0; i < n && __popc(chosen) < m; ++i) chosen |= 1u << i;
  uint32_t mask = 0;
  for (int i = 0; i < n; ++i)
    if ((chosen >> i) & 1u) mask |= 1u << sm.P[i];
  return mask;
}

// All threads: loads w[j][:] of the pending set must be in sm.w (by position);
// returns the RunSet mask (over micro-batch ids).  slots: the MaxUtil search
// grid's results for this pending set (null: search here).
__device__ void prepare_totals(SchedSmem& sm, int D) {
  const int tid = threadIdx.x;
  for (int dd = tid; dd < D; dd += blockDim.x) {
    long long t = 0;
    for (int i = 0; i < sm.n; ++i) t += sm.w[i][dd];
    sm.tot[dd] = t;
  }
  for (int i = tid; i < sm.n; i += blockDim.x) {
    long long t = 0;
    for (int dd = 0; dd < D; ++dd) t += sm.w[i][dd];
    sm.wsum[i] = t;
  }
  __syncthreads();
  if (tid == 0) {
    long long ts = 0;
    for (int i = 0; i < sm.n; ++i) ts += sm.wsum[i];
    sm.totsum = ts;
  }
  __syncthreads();
}

__device__ uint32_t choose_runset(SchedSmem& sm, int D, int m, int policy, uint32_t pending,
                                  const Cand* slots = nullptr) {
  prepare_totals(sm, D);
  if (policy == EB_SCHED_LOCKSTEP || sm.n <= m) return pending;
  if (policy == EB_SCHED_MAXUTIL)
    return slots ? maxutil_slots(sm, slots, kSearchCtas) : maxutil_block(sm, D, m);
  if (threadIdx.x == 0) sm.result = scan_policy(sm, D, m, policy);
  __syncthreads();
  return sm.result;
}


struct PlanSmem {
  int3 tmp3[33];
};

// Expert counts of the RunSet's micro-batches kept in shared memory by the
// plan when nr * E fits (32 KiB).
constexpr int kPlanHistCache = 8192;

// Exclusive block-wide scan of per-thread int3 values: returns this thread's
// offsets; tmp[32] receives the block totals.  All threads must call it.
__device__ int3 block_exclusive_scan3(int3 v, int3* tmp /* >= 33 */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int3 incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int yx = __shfl_up_sync(0xffffffffu, incl.x, off);
    const int yy = __shfl_up_sync(0xffffffffu, incl.y, off);
    const int yz = __shfl_up_sync(0xffffffffu, incl.z, off);
    if (lane >= off) {
      incl.x += yx;
      incl.y += yy;
      incl.z += yz;
    }
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int3 x = lane < nw ? tmp[lane] : make_int3(0, 0, 0);
    int3 xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int yx = __shfl_up_sync(0xffffffffu, xi.x, off);
      const int yy = __shfl_up_sync(0xffffffffu, xi.y, off);
      const int yz = __shfl_up_sync(0xffffffffu, xi.z, off);
      if (lane >= off) {
        xi.x += yx;
        xi.y += yy;
        xi.z += yz;
      }
    }
    if (lane < nw) tmp[lane] = make_int3(xi.x - x.x, xi.y - x.y, xi.z - x.z);
    if (lane == 31) tmp[32] = xi;
  }
  __syncthreads();
  const int3 w = tmp[warp];
  return make_int3(w.x + incl.x - v.x, w.y + incl.y - v.y, w.z + incl.z - v.z);
}

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

__global__ void __launch_bounds__(kThreads) k_schedule_step(Dims d, CtxDev c, Work wk, int rn1,
                                                             int rn2, int fm1, int fm2) {
  __shared__ SchedSmem sm;
  __shared__ PlanSmem pl;
  // the step state lives in shared memory for the whole kernel (thread 0's
  // bookkeeping would otherwise be a chain of dependent global loads)
  __shared__ State ss;
  State* st = &ss;
  const int tid = threadIdx.x;
  pdl_enter();
  constexpr int kStateWords = sizeof(State) / sizeof(int);
  for (int i = tid; i < kStateWords; i += blockDim.x)
    reinterpret_cast<int*>(&ss)[i] = reinterpret_cast<const int*>(c.st)[i];
  __syncthreads();
  auto write_back = [&]() {
    __syncthreads();
    for (int i = tid; i < kStateWords; i += blockDim.x)
      reinterpret_cast<int*>(c.st)[i] = reinterpret_cast<const int*>(&ss)[i];
  };
  // A context whose status word holds EB_ERR_TIMEOUT (a bounded wait of an
  // earlier step expired, so its state may be partial) runs no further step
  // until eb_reset: the step does nothing and reports S as empty.
  if (ss.status == EB_ERR_TIMEOUT) {
    if (tid == 0) {
      st->pending = 0;
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
    return;
  }
  // 1. hist[j][:] and w[j][:] of the micro-batches routed for this step were
  //    accumulated by the routing kernel
  // 2. pending set
  const uint32_t pending = st->pending;
  if (tid == 0) {
    int n = 0;
    for (int j = 0; j < d.M; ++j)
      if ((pending >> j) & 1u) sm.P[n++] = j;
    sm.n = n;
  }
  __syncthreads();
  if (sm.n == 0) {  // episode finished: this step does nothing
    if (tid == 0) {
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
    return;
  }
  for (int i = tid; i < sm.n * d.D; i += blockDim.x) {
    const int p = i / d.D, dd = i % d.D;
    sm.w[p][dd] = c.w[sm.P[p] * d.D + dd];
  }
  __syncthreads();
  // 3. RunSet
  const uint32_t run = choose_runset(sm, d.D, d.m, d.policy, pending,
                                     static_cast<const Cand*>(c.search_slots));
  // 4. accounting, trace and Algorithm 1 bookkeeping (thread 0)
  if (tid == 0) {
    long long sumW = 0, maxW = 0, summax = 0;
    for (int dd = 0; dd < d.D; ++dd) {
      long long Wd = 0;
      for (int p = 0; p < sm.n; ++p)
        if ((run >> sm.P[p]) & 1u) Wd += sm.w[p][dd];
      sumW += Wd;
      maxW = Wd > maxW ? Wd : maxW;
    }
    for (int p = 0; p < sm.n; ++p)
      if ((run >> sm.P[p]) & 1u) {
        long long mx = 0;
        for (int dd = 0; dd < d.D; ++dd) mx = sm.w[p][dd] > mx ? sm.w[p][dd] : mx;
        summax += mx;
      }
    st->num += sumW;
    st->den += (long long)d.D * maxW;
    st->den_sep += (long long)d.D * summax;
    const int step = st->n_steps;
    if (step < d.max_steps) {
      c.trace[step * kTraceCols + 0] = run;
      c.trace[step * kTraceCols + 1] = sumW;
      c.trace[step * kTraceCols + 2] = maxW;
      c.trace[step * kTraceCols + 3] = summax;
      c.trace[step * kTraceCols + 4] = 0;
      c.trace[step * kTraceCols + 5] = 0;
      for (int j = 0; j < d.M; ++j)
        c.trace_layers[step * d.M + j] = ((run >> j) & 1u) ? st->layer[j] : -1;
    }
    st->n_steps = step + 1;
    int nr = 0;
    uint32_t still = 0;
    for (int j = 0; j < d.M; ++j) {
      if ((run >> j) & 1u) {
        st->step_layer[j] = st->layer[j];
        st->run_list[nr++] = j;
        st->layer[j] += 1;
      } else {
        st->step_layer[j] = -1;
      }
      if (st->layer[j] < d.L) still |= 1u << j;
    }
    st->n_run = nr;
    st->runset = run;
    st->pending = still;
    st->need_route = run & still;
    // segment groups: distinct layers of the RunSet, ascending
    int G = 0;
    for (int a = 0; a < nr; ++a) {
      const int l = st->step_layer[st->run_list[a]];
      bool seen = false;
      for (int g = 0; g < G; ++g) seen |= (st->group_layer[g] == l);
      if (!seen) {
        int g = G++;
        while (g > 0 && st->group_layer[g - 1] > l) {
          st->group_layer[g] = st->group_layer[g - 1];
          --g;
        }
        st->group_layer[g] = l;
      }
    }
    for (int a = 0; a < nr; ++a) {
      const int j = st->run_list[a];
      for (int g = 0; g < G; ++g)
        if (st->group_layer[g] == st->step_layer[j]) st->group_of[j] = g;
    }
    st->n_groups = G;
    st->nseg = G * d.Etot;
  }
  if (!d.compute) {
    __syncthreads();
    const uint32_t next = st->need_route;
    for (int i = tid; i < d.M * d.E; i += blockDim.x)
      if ((next >> (i / d.E)) & 1u) c.hist[i] = 0;
    for (int i = tid; i < d.M * d.D; i += blockDim.x)
      if ((next >> (i / d.D)) & 1u) c.w[i] = 0;
    write_back();
    return;
  }
  __syncthreads();
  // 5. segment plan: rows of (group, expert) are counted into seg_rows and
  //    scanned in place; GEMM work items per segment likewise.  The RunSet's
  //    expert counts are staged in shared memory when they fit (the counts
  //    and the prior table below read them several times).
  const int G = st->n_groups, nr = st->n_run, Et = d.Etot, nseg = G * Et;
  const int mb1 = d.F / fm1, mb2 = d.H / fm2;
  __shared__ int s_nonempty;
  __shared__ int s_hist[kPlanHistCache];
  const bool cached = nr * d.E <= kPlanHistCache;
  if (tid == 0) s_nonempty = 0;
  if (cached)
    for (int i = tid; i < nr * d.E; i += blockDim.x)
      s_hist[i] = c.hist[st->run_list[i / d.E] * d.E + i % d.E];
  __syncthreads();
  // counts of RunSet member a (position in run_list) for expert e
  auto count_of = [&](int a, int e) -> int {
    if (e >= d.E) return d.T;  // shared expert: every token
    return cached ? s_hist[a * d.E + e] : c.hist[st->run_list[a] * d.E + e];
  };
  int my_nonempty = 0;
  int3 local = make_int3(0, 0, 0);  // this thread's sums of rows, items1, items2
  const int per = (nseg + blockDim.x - 1) / blockDim.x;
  const int sb = tid * per, se = min(nseg, sb + per);
  for (int i = sb; i < se; ++i) {
    const int g = i / Et, e = i % Et;
    int cnt = 0;
    for (int a = 0; a < nr; ++a)
      if (st->group_of[st->run_list[a]] == g) cnt += count_of(a, e);
    my_nonempty += cnt > 0;
    const int i1 = (cnt + rn1 - 1) / rn1 * mb1, i2 = (cnt + rn2 - 1) / rn2 * mb2;
    wk.seg_rows[i] = cnt;
    wk.seg_items1[i] = i1;
    wk.seg_items2[i] = i2;
    wk.seg_wid[i] = st->group_layer[g] * Et + e;
    local.x += cnt;
    local.y += i1;
    local.z += i2;
  }
  if (my_nonempty) atomicAdd(&s_nonempty, my_nonempty);
  // one block-wide exclusive scan of the three running sums
  const int3 base = block_exclusive_scan3(local, pl.tmp3);
  int3 acc3 = base;
  for (int i = sb; i < se; ++i) {
    const int a = wk.seg_rows[i], b = wk.seg_items1[i], cc = wk.seg_items2[i];
    wk.seg_rows[i] = acc3.x;
    wk.seg_items1[i] = acc3.y;
    wk.seg_items2[i] = acc3.z;
    acc3.x += a;
    acc3.y += b;
    acc3.z += cc;
  }
  const int rows = pl.tmp3[32].x, it1 = pl.tmp3[32].y, it2 = pl.tmp3[32].z;
  if (tid == 0) {
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
      c.trace[step * kTraceCols + 5] = s_nonempty;
    }
  }
  __syncthreads();
  // rows of (j's segment, expert) taken by earlier micro-batches of its group;
  // the permute kernel adds the earlier chunks of j itself
  for (int i = tid; i < nr * Et; i += blockDim.x) {
    const int a = i / Et, e = i % Et;
    const int j = st->run_list[a], g = st->group_of[j];
    int prior = 0;
    for (int b = 0; b < a; ++b)
      if (st->group_of[st->run_list[b]] == g) prior += count_of(b, e);
    wk.prior[j * Et + e] = prior;
  }
  __syncthreads();
  // the micro-batches routed at the next step start from zero counts
  const uint32_t next = st->need_route;
  for (int i = tid; i < d.M * d.E; i += blockDim.x)
    if ((next >> (i / d.E)) & 1u) c.hist[i] = 0;
  for (int i = tid; i < d.M * d.D; i += blockDim.x)
    if ((next >> (i / d.D)) & 1u) c.w[i] = 0;
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
  if (tid == 0) {
    int n = 0;
    for (int j = 0; j < M; ++j)
      if ((pending >> j) & 1u) sm.P[n++] = j;
    sm.n = n;
  }
  __syncthreads();
  if (sm.n == 0) {
    if (tid == 0) {
      *runset_out = 0;
      if (stats) stats[0] = stats[1] = stats[2] = 0;
    }
    return;
  }
  for (int i = tid; i < sm.n * D; i += blockDim.x) {
    const int p = i / D, dd = i % D;
    sm.w[p][dd] = w[sm.P[p] * D + dd];
  }
  __syncthreads();
  const uint32_t run = choose_runset(sm, D, m, policy, pending, slots);
  if (tid == 0) {
    *runset_out = run;
    if (stats) {
      long long sumW = 0, maxW = 0, summax = 0;
      for (int dd = 0; dd < D; ++dd) {
        long long Wd = 0;
        for (int p = 0; p < sm.n; ++p)
          if ((run >> sm.P[p]) & 1u) Wd += sm.w[p][dd];
        sumW += Wd;
        maxW = Wd > maxW ? Wd : maxW;
      }
      for (int p = 0; p < sm.n; ++p)
        if ((run >> sm.P[p]) & 1u) {
          long long mx = 0;
          for (int dd = 0; dd < D; ++dd) mx = sm.w[p][dd] > mx ? sm.w[p][dd] : mx;
          summax += mx;
        }
      stats[0] = sumW;
      stats[1] = maxW;
      stats[2] = summax;
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
                                 int fm1, int fm2, cudaStream_t s) {
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
  return launch_pdl(k_schedule_step, dim3(1), dim3(kThreads), 0, s, 1, d, c, w, rn1, rn2, fm1, fm2);
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
