// Routing: softmax top-k with renormalised gates and per-expert token counts.
//
// [EB] §2.1: W_l, I_l = topk(G(h'_l)) -- each token picks its top-k experts and
// weighs them.  The counts T_e per expert are what a rank's load is built
// from ([SysLB] §1: L_r = sum_{e in E_r} T_e).
//
// A warp routes token rows: the E logits are read coalesced (lane i holds
// experts i, i+32, ...) and mapped to order-preserving integer keys, and each
// lane sorts its experts by key, descending (a stable sort, so equal keys
// keep their ascending expert order).  The k winners then come out of k
// rounds over the lanes' heads: a hardware max-reduction of the head keys,
// after which the lane holding the maximum pops its head and marks the
// round.  A lane's winners are thus a prefix of its sorted list, and the
// rounds it marked are their slots.  When two lanes hold equal maxima in a
// round, both pop and the warp counts more than k pops; such a row is
// selected again with the exact order (logit descending, expert index
// ascending): among the lanes holding the maximum, a min-reduction of their
// head indices names the one that pops.  Two rows are routed together, their
// rounds interleaved.  Each lane then writes its own winners: the gates
// exp(l_s - l_max) / sum_{s'} exp(l_s' - l_max) are formed from the winners
// alone when renormalised (the full softmax denominator cancels), l_max being
// the first round's maximum.  Counts go to shared-memory atomics (integers,
// so the result is exact and order-free), are written once per
// (micro-batch, chunk) and are added to the micro-batch's histogram and rank
// loads with one global atomic per (chunk, expert) and (chunk, rank).
#include <math.h>

#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
  return x;
}

// Order-preserving map of a finite float (or -inf) to uint32 (-0 is folded
// into +0 first, so equal floats map to equal keys).  Every such key is at
// least order_key(-inf) = 0x007fffff, so 0 is free to mark padding.
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float order_key maps to this key.
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One round over the lanes' heads h[0]: returns the warp maximum; every lane
// holding it pops its head and sets `bit` in `won`.
template <int VPL>
__device__ __forceinline__ uint32_t pop_max(uint32_t (&h)[VPL], uint32_t& won, uint32_t bit) {
  const uint32_t m = __reduce_max_sync(kFull, h[0]);
  if (h[0] == m) {
    won |= bit;
#pragma unroll
    for (int i = 0; i + 1 < VPL; ++i) h[i] = h[i + 1];
    h[VPL - 1] = 0u;
  }
  return m;
}

// Sorted position -> expert of a lane: byte i of the packed words is the
// slot q (expert q * 32 + lane) at sorted position i.
template <int VPL>
struct Perm {
  static constexpr int kW = (VPL + 3) / 4;
  uint32_t w[kW];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int q = 0; q < kW; ++q) w[q] = 0x03020100u + 0x04040404u * (uint32_t)q;
  }
  // exchanges positions b - 1 and b (b a constant once unrolled)
  __device__ __forceinline__ void swap(int b) {
    if ((b & 3) != 0) {
      const int q = b >> 2, j = b & 3;
      const uint32_t sel = (0x3210u & ~(0xffu << (4 * (j - 1)))) |
                           ((uint32_t)j << (4 * (j - 1))) | ((uint32_t)(j - 1) << (4 * j));
      w[q] = __byte_perm(w[q], 0u, sel);
    } else if (kW > 1) {  // byte 3 of one word and byte 0 of the next
      const int q = (b >> 2) - 1, q1 = min(q + 1, kW - 1);
      const uint32_t lo = __byte_perm(w[q], w[q1], 0x4210u);
      const uint32_t hi = __byte_perm(w[q], w[q1], 0x7653u);
      w[q] = lo;
      w[q1] = hi;
    }
  }
  // drops position 0 (the others move down by one)
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int q = 0; q + 1 < kW; ++q) w[q] = __funnelshift_r(w[q], w[q + 1], 8);
    w[kW - 1] >>= 8;
  }
  __device__ __forceinline__ int slot(int i) const { return (w[i >> 2] >> (8 * (i & 3))) & 0xff; }
};

// The k rounds under the exact order: among the lanes whose head holds the
// maximum key, the one with the smallest expert index pops.
template <int VPL>
__device__ __forceinline__ uint32_t exact_rounds(const uint32_t (&key)[VPL], const Perm<VPL>& perm,
                                                 int lane, int k) {
  uint32_t h[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) h[i] = key[i];
  Perm<VPL> p = perm;
  uint32_t won = 0u;
  for (int s = 0; s < k; ++s) {
    const uint32_t m = __reduce_max_sync(kFull, h[0]);
    const uint32_t hid = h[0] == m ? (uint32_t)(p.slot(0) * 32 + lane) : 0xffffffffu;
    const uint32_t me = __reduce_min_sync(kFull, hid);
    if (hid == me) {
      won |= 1u << s;
#pragma unroll
      for (int i = 0; i + 1 < VPL; ++i) h[i] = h[i + 1];
      h[VPL - 1] = 0u;
      p.pop();
    }
  }
  return won;
}

// Routes R token rows with the calling warp, their rounds interleaved so the
// rows' dependency chains overlap, and writes slot s of row r to
// idx_out[r][s], gate_out[r][s], counting its expert in hist_s.  x[r][i] is
// the logit of expert i * 32 + lane of row r (0 where that is not below E);
// FULL: E == 32 * VPL.  A row with valid[r] false is skipped.  With emask
// set, each winner also sets bit tl[r] (the row's token within its 64-token
// chunk) of its expert's 64-bit mask emask[2e], emask[2e + 1].
template <int VPL, int R, bool FULL>
__device__ __forceinline__ void route_rows(const float (&x)[R][VPL], const bool (&valid)[R], int E,
                                           int k, int renorm, int lane,
                                           int32_t* const (&idx_out)[R],
                                           float* const (&gate_out)[R], int* hist_s,
                                           uint32_t* emask, const int (&tl)[R],
                                           bool& nonfinite) {
  uint32_t key[R][VPL];
  Perm<VPL> perm[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float z = 0.f;  // becomes NaN once a logit is infinite or NaN
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      z = fmaf(x[r][i], 0.f, z);
      key[r][i] = order_key(x[r][i]);
    }
    if (__any_sync(kFull, z != 0.f)) {
      // selection stays among real experts, a non-finite logit ranking as
      // -inf; the call reports the error
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (!isfinite(x[r][i])) {
          nonfinite = true;
          key[r][i] = order_key(-INFINITY);
        }
    }
    if (!FULL) {
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (i * 32 + lane >= E) key[r][i] = 0u;  // padding ranks below every real expert
    }
    perm[r].init();
  }
  // stable sort, key descending: equal keys stay in ascending expert order
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int a = 0; a + 1 < VPL; ++a)
#pragma unroll
      for (int b = VPL - 1; b > a; --b) {
        const uint32_t hi = key[r][b - 1], lo = key[r][b];
        key[r][b - 1] = max(hi, lo);
        key[r][b] = min(hi, lo);
        if (lo > hi) perm[r].swap(b);
      }
  uint32_t h[R][VPL], won[R], top[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) h[r][i] = key[r][i];
    won[r] = 0u;
    top[r] = pop_max<VPL>(h[r], won[r], 1u);
  }
#pragma unroll 2
  for (int s = 1; s < k; ++s) {
    const uint32_t bit = 1u << s;
#pragma unroll
    for (int r = 0; r < R; ++r) pop_max<VPL>(h[r], won[r], bit);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (!valid[r]) continue;
    // equal maxima in two lanes made both pop: select the row again exactly
    if (__reduce_add_sync(kFull, (unsigned)__popc(won[r])) != (unsigned)k)
      won[r] = exact_rounds<VPL>(key[r], perm[r], lane, k);
    const float vmax = key_value(top[r]);
    const int c = __popc(won[r]);
    // the most winners any lane holds: the loops below stop there
    const int cmax = (int)__reduce_max_sync(kFull, (unsigned)c);
    float ex[VPL];
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      ex[i] = 0.f;
      if (renorm ? (i < cmax && i < c) : (key[r][i] != 0u)) {
        ex[i] = expf(key_value(key[r][i]) - vmax);
        sum += ex[i];
      }
    }
    const float inv = __frcp_rn(warp_sum(sum));
    uint32_t rest = won[r];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (i >= cmax) break;
      if (i < c) {
        const int s = __ffs(rest) - 1;
        rest &= rest - 1u;
        const int e = perm[r].slot(i) * 32 + lane;
        idx_out[r][s] = e;
        gate_out[r][s] = ex[i] * inv;
        atomicAdd(&hist_s[e], 1);
        if (emask) atomicOr(&emask[2 * e + (tl[r] >> 5)], 1u << (tl[r] & 31));
      }
    }
  }
}

// Logits of rows t + r * W (r < R) that lie below t1; lane i holds experts
// i, i + 32, ...
template <int VPL, int R>
__device__ __forceinline__ void load_rows(const float* __restrict__ logits, int t, int t1, int E,
                                          int W, int lane, float (&x)[R][VPL]) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int tr = t + r * W;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = i * 32 + lane;
      x[r][i] = (tr < t1 && e < E) ? __ldg(logits + (size_t)tr * E + e) : 0.f;
    }
  }
}

// Tokens [t0, t1) of a block of rows: warp w routes tokens w, w + W, ...
// (W warps) R at a time, R = 2 while two rows' registers fit (VPL <= 4).
// The next R rows' logits are loaded while the current ones are routed.
template <int VPL, bool FULL>
__device__ __forceinline__ void route_chunk_t(const float* __restrict__ logits, int t0, int t1,
                                              int E, int k, int renorm,
                                              int32_t* __restrict__ idx,
                                              float* __restrict__ gate, int* hist_s,
                                              uint32_t* emask, bool& nonfinite) {
  constexpr int R = VPL <= 4 ? 2 : 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, W = blockDim.x >> 5;
  float next[R][VPL];
  int t = t0 + warp;
  if (t < t1) load_rows<VPL, R>(logits, t, t1, E, W, lane, next);
  for (; t < t1; t += R * W) {
    float x[R][VPL];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int i = 0; i < VPL; ++i) x[r][i] = next[r][i];
    if (t + R * W < t1) load_rows<VPL, R>(logits, t + R * W, t1, E, W, lane, next);
    bool valid[R];
    int32_t* io[R];
    float* go[R];
    int tl[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int tr = t + r * W;
      valid[r] = tr < t1;
      const size_t q = (size_t)(valid[r] ? tr : t);
      io[r] = idx + q * k;
      go[r] = gate + q * k;
      tl[r] = (valid[r] ? tr : t) - t0;
    }
    route_rows<VPL, R, FULL>(x, valid, E, k, renorm, lane, io, go, hist_s, emask, tl, nonfinite);
  }
}

template <int VPL>
__device__ void route_chunk(const float* __restrict__ logits, int t0, int t1, int E, int k,
                            int renorm, int32_t* __restrict__ idx, float* __restrict__ gate,
                            int* hist_s, uint32_t* emask, bool& nonfinite) {
  if (E == 32 * VPL)
    route_chunk_t<VPL, true>(logits, t0, t1, E, k, renorm, idx, gate, hist_s, emask, nonfinite);
  else
    route_chunk_t<VPL, false>(logits, t0, t1, E, k, renorm, idx, gate, hist_s, emask, nonfinite);
}

constexpr int kRankWarps = 8;  // warps of a 256-thread routing CTA
static_assert(kChunk <= 64, "a chunk's tokens fit one 64-bit mask per expert");

// Step path: CTA (c, j) routes chunk c of micro-batch j at its layer l_j if j
// is in need_route; its counts land in chunk_hist[j][c][:] and are added
// (integer atomics: exact, order-free) to the micro-batch's histogram
// hist[j][:] and rank loads w[j][:], which the previous step zeroed.  The
// loads fold the counts by the context's expert placement: contiguous
// blocks of E/D experts, or emap[e] if one was set.
//
// With `rank` set (expert arithmetic on), the CTA also ranks its chunk's
// (token, slot) pairs among those with the same expert, in (token, slot)
// order, into rank[j][t][s]; and the last of micro-batch j's NC CTAs to
// finish (a ticket taken after every CTA's counts are visible) writes the
// chunk offsets cbase[j][c][e] = sum over c' < c of chunk_hist[j][c'][e].
// rank + cbase is the pair's place among micro-batch j's pairs of its
// expert; none of it depends on the schedule, so the row copy of the step
// that runs j only adds the segment's base and the rows of earlier RunSet
// members (see k_permute_bulk).
//
// early: launched right after the previous step's GEMM 2 (whose persistent
// CTAs are all resident), which reads nothing routing writes -- the gates go
// to the buffer the micro-batch's gate_buf bit does not name, while the
// previous step's combine reads the other.  The CTA then routes first and
// waits for GEMM 2 only at its end, so the step's combine and everything
// after it still start after GEMM 2.  The state it reads was written by the
// previous scheduler step, which completed before GEMM 2 started.
template <int VPL>
__global__ void __launch_bounds__(256, 4) k_route_step(Dims d, State* __restrict__ st,
                                                     const float* __restrict__ logits,
                                                     int32_t* __restrict__ idx,
                                                     float* __restrict__ gate,
                                                     int32_t* __restrict__ chunk_hist,
                                                     int32_t* __restrict__ hist,
                                                     int32_t* __restrict__ wload,
                                                     const int32_t* __restrict__ emap,
                                                     long long mb_stride, long long layer_stride,
                                                     int32_t* __restrict__ rank,
                                                     int32_t* __restrict__ cbase,
                                                     int32_t* __restrict__ tickets, int early) {
  if (early) pdl_trigger();
  else pdl_enter();
  const int c = blockIdx.x, j = blockIdx.y;
  // nothing routes while a timed-out step awaits eb_reset
  if (!((st->need_route >> j) & 1u) || st->status == EB_ERR_TIMEOUT) {
    if (early) pdl_wait();
    return;
  }
  const int l = st->layer[j];
  // the gate buffer j's current routing does not use
  float* gate_j = gate + (size_t)(((st->gate_buf >> j) & 1u) ^ 1u) * ((size_t)d.M * d.T * d.k);
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int w_s[EB_MAX_D];
  __shared__ int bad;
  __shared__ uint32_t emask[2 * EB_MAX_ETOT];  // tokens of the chunk that chose each expert
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) hist_s[e] = 0;
  for (int r = threadIdx.x; r < d.D; r += blockDim.x) w_s[r] = 0;
  if (rank)
    for (int i = threadIdx.x; i < 2 * d.E; i += blockDim.x) emask[i] = 0u;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  // rows of micro-batch j at layer l: the caller's logits [M, L, T, E], or
  // the router's scores of this step (see launch_route_step)
  const float* blk = logits + (size_t)j * mb_stride + (size_t)l * layer_stride;
  const int t0 = c * kChunk, t1 = min(d.T, t0 + kChunk);
  bool nonfinite = false;
  route_chunk<VPL>(blk, t0, t1, d.E, d.k, d.renorm, idx + (size_t)j * d.T * d.k,
                   gate_j + (size_t)j * d.T * d.k, hist_s, rank ? emask : nullptr, nonfinite);
  if (nonfinite) bad = 1;
  __syncthreads();
  int32_t* out = chunk_hist + ((size_t)j * d.NC + c) * d.E;
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) {
    out[e] = hist_s[e];
    if (hist_s[e]) atomicAdd(&hist[j * d.E + e], hist_s[e]);
  }
  if (emap) {  // custom placement (ranks validated on the host)
    for (int e = threadIdx.x; e < d.E; e += blockDim.x)
      if (hist_s[e]) atomicAdd(&w_s[emap[e]], hist_s[e]);
    __syncthreads();
    for (int r = threadIdx.x; r < d.D; r += blockDim.x)
      if (w_s[r]) atomicAdd(&wload[j * d.D + r], w_s[r]);
  } else {
    const int per = d.E / d.D;
    for (int r = threadIdx.x; r < d.D; r += blockDim.x) {
      int sum = 0;
      for (int e = r * per; e < (r + 1) * per; ++e) sum += hist_s[e];
      if (sum) atomicAdd(&wload[j * d.D + r], sum);
    }
  }
  if (threadIdx.x == 0 && bad) atomicCAS(&st->status, EB_OK, EB_ERR_NONFINITE);
  if (rank) {
    // a token's k experts are distinct, so the place of (t, s) among the
    // chunk's pairs of its expert is the number of earlier tokens of the
    // chunk whose mask bit that expert has
    const size_t base = (size_t)j * d.T + t0;
    const int32_t* ex = idx + base * d.k;
    int32_t* rk = rank + base * d.k;
    for (int p = threadIdx.x; p < (t1 - t0) * d.k; p += blockDim.x) {
      const int t = p / d.k, e = ex[p];
      const uint32_t lo = emask[2 * e], below = (1u << (t & 31)) - 1u;
      rk[p] = t < 32 ? __popc(lo & below) : __popc(lo) + __popc(emask[2 * e + 1] & below);
    }
    __shared__ int scratch[kRankWarps][EB_MAX_ETOT];
    // every thread's counts of this chunk are visible before the ticket
    __threadfence();
    __shared__ int last;
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&tickets[j], 1) == d.NC - 1;
    __syncthreads();
    if (last) {
      // warp w sums its range of chunks per expert (lanes over experts,
      // loads coalesced), the ranges' totals are scanned in shared memory,
      // and each warp writes its range's offsets
      __threadfence();
      const int32_t* ch = chunk_hist + (size_t)j * d.NC * d.E;
      int32_t* cb = cbase + (size_t)j * d.NC * d.E;
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
      const int per = (d.NC + kRankWarps - 1) / kRankWarps;
      const int c0 = min(d.NC, warp * per), c1 = min(d.NC, c0 + per);
      for (int e = lane; e < d.E; e += 32) {
        int sum = 0;
#pragma unroll 8
        for (int cc = c0; cc < c1; ++cc) sum += __ldcg(ch + (size_t)cc * d.E + e);
        scratch[warp][e] = sum;
      }
      __syncthreads();
      for (int e = lane; e < d.E; e += 32) {
        int run = 0;
        for (int w = 0; w < warp; ++w) run += scratch[w][e];
#pragma unroll 8
        for (int cc = c0; cc < c1; ++cc) {
          cb[(size_t)cc * d.E + e] = run;
          run += __ldcg(ch + (size_t)cc * d.E + e);
        }
      }
      if (threadIdx.x == 0) tickets[j] = 0;
    }
  }
  if (early) pdl_wait();
}

// Stand-alone path: rows [c*kChunk, ...) of an [n, E] block; counts summed
// into hist[E] with one global atomic per (CTA, expert) with a non-zero count.
template <int VPL>
__global__ void __launch_bounds__(256, 4) k_route_rows(const float* __restrict__ logits, int n, int E,
                                                     int k, int renorm, int32_t* __restrict__ idx,
                                                     float* __restrict__ gate,
                                                     int32_t* __restrict__ hist,
                                                     int32_t* __restrict__ status) {
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int bad;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_s[e] = 0;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kChunk, t1 = min(n, t0 + kChunk);
  bool nonfinite = false;
  route_chunk<VPL>(logits, t0, t1, E, k, renorm, idx, gate, hist_s, nullptr, nonfinite);
  if (nonfinite) bad = 1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist_s[e]) atomicAdd(&hist[e], hist_s[e]);
  if (threadIdx.x == 0 && bad && status) atomicExch(status, EB_ERR_NONFINITE);
}

int vpl_for(int E) { return E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : 8; }

}  // namespace

cudaError_t launch_route_step(const Dims& d, const CtxDev& c, const Work& w, const float* logits,
                              long long mb_stride, long long layer_stride, bool early,
                              cudaStream_t s) {
  dim3 grid(d.NC, d.M);
  // 256-thread CTAs, four per SM: a warp routes a chunk's rows R at a time
  // while the next ones load, and beside GEMM 2's CTAs (one per SM, most of
  // its registers and shared memory) an early launch still finds room
  const dim3 block(256);
  const int32_t* emap = c.use_emap ? c.emap : nullptr;
  const int ea = early ? 1 : 0;
  cudaError_t e;
  switch (vpl_for(d.E)) {
    case 1: e = launch_pdl(k_route_step<1>, dim3(grid), block, 0, s, 1, d, c.st, logits, w.idx, w.gate, w.chunk_hist, c.hist, c.w, emap, mb_stride, layer_stride, w.rank, w.cbase, c.tickets, ea); break;
    case 2: e = launch_pdl(k_route_step<2>, dim3(grid), block, 0, s, 1, d, c.st, logits, w.idx, w.gate, w.chunk_hist, c.hist, c.w, emap, mb_stride, layer_stride, w.rank, w.cbase, c.tickets, ea); break;
    case 4: e = launch_pdl(k_route_step<4>, dim3(grid), block, 0, s, 1, d, c.st, logits, w.idx, w.gate, w.chunk_hist, c.hist, c.w, emap, mb_stride, layer_stride, w.rank, w.cbase, c.tickets, ea); break;
    default: e = launch_pdl(k_route_step<8>, dim3(grid), block, 0, s, 1, d, c.st, logits, w.idx, w.gate, w.chunk_hist, c.hist, c.w, emap, mb_stride, layer_stride, w.rank, w.cbase, c.tickets, ea); break;
  }
  return e;
}

cudaError_t launch_route_rows(const float* logits, int n, int E, int k, int renorm, int32_t* idx,
                              float* gate, int32_t* hist, int32_t* status, cudaStream_t s) {
  if (cuda_error_pending()) return cudaErrorUnknown;
  cudaError_t err = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)E, s);
  if (err != cudaSuccess || n == 0) return err;
  dim3 grid((n + kChunk - 1) / kChunk);
  switch (vpl_for(E)) {
    case 1: k_route_rows<1><<<grid, 256, 0, s>>>(logits, n, E, k, renorm, idx, gate, hist, status); break;
    case 2: k_route_rows<2><<<grid, 256, 0, s>>>(logits, n, E, k, renorm, idx, gate, hist, status); break;
    case 4: k_route_rows<4><<<grid, 256, 0, s>>>(logits, n, E, k, renorm, idx, gate, hist, status); break;
    default: k_route_rows<8><<<grid, 256, 0, s>>>(logits, n, E, k, renorm, idx, gate, hist, status); break;
  }
  return cudaGetLastError();
}

}  // namespace eb

// ---------------------------------------------------------------------------
// Routing + loads for callers that cannot allocate device memory.
//
// The step path keeps its per-(micro-batch, chunk, expert) counts in the
// caller's workspace.  Some callers cannot provide one: a serving process
// whose device memory is fixed once at start-up (a pre-reserved pool, or an
// allocator that refuses new cudaMalloc after warm-up), or a caller that must
// not call cudaMalloc / cudaFree because they can synchronise the device and
// stall work on other streams.  eb_route_loads_static serves them: the counts
// live in the file-scope array below, which every GPU that loads this library
// holds (4 MiB) until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

namespace eb {
namespace {

constexpr long long kStaticCountInts = 1ll << 20;  // 4 MiB of int32 counts
static __device__ __align__(256) int32_t g_static_counts[kStaticCountInts];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
struct StaticAddr {
  void* ctx;     // CUDA context the address belongs to
  int32_t* ptr;  // device address of g_static_counts in that context
};
StaticAddr g_static_addr[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// cuCtxGetCurrent through the runtime's driver entry-point query (no link
// against the driver library); null if unavailable.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

void* current_ctx() {
  void* c = nullptr;
  CtxGetCurrentFn fn = ctx_get_current();
  if (!fn || fn(&c) != 0) return nullptr;
  return c;
}

// Device address of g_static_counts on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress (with the device current) and cached together with the
// CUDA context it belongs to.  When the current context is not the cached
// one -- the first call on a device, or after cudaDeviceReset() tore the
// primary context down and the module was loaded again -- it is looked up
// afresh, so a stale address is never launched with.
cudaError_t static_counts_ptr(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticAddr& a = g_static_addr[dev];
  void* ctx = current_ctx();
  if (!a.ptr || !ctx || ctx != a.ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_counts);  // also makes the primary context current
    if (e != cudaSuccess) return e;
    a.ptr = static_cast<int32_t*>(p);
    a.ctx = current_ctx();
  }
  *out = a.ptr;
  return cudaSuccess;
}

// CTA (c, j): chunk c of micro-batch j of logits [n_mb, T, E]; writes every
// count of its (j, c) row, so nothing in the scratch needs to start at zero.
template <int VPL>
__global__ void __launch_bounds__(256, 4) k_route_counts_static(const float* __restrict__ logits,
                                                              int T, int E, int k, int renorm, int NC,
                                                              int32_t* __restrict__ idx,
                                                              float* __restrict__ gate,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ status) {
  const int c = blockIdx.x, j = blockIdx.y;
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int bad;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_s[e] = 0;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int t0 = c * kChunk, t1 = min(T, t0 + kChunk);
  bool nonfinite = false;
  route_chunk<VPL>(logits + (size_t)j * T * E, t0, t1, E, k, renorm, idx + (size_t)j * T * k,
                   gate + (size_t)j * T * k, hist_s, nullptr, nonfinite);
  if (nonfinite) bad = 1;
  __syncthreads();
  int32_t* out = counts + ((size_t)j * NC + c) * E;
  for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = hist_s[e];
  if (threadIdx.x == 0 && bad && status) atomicExch(status, EB_ERR_NONFINITE);
}

// w[j][d] = sum over chunks and over the contiguous expert block of rank d.
__global__ void k_fold_static(const int32_t* __restrict__ counts, int n_mb, int NC, int E, int D,
                              int32_t* __restrict__ w) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_mb * D) return;
  const int j = i / D, dd = i % D, per = E / D;
  int s = 0;
  for (int ch = 0; ch < NC; ++ch) {
    const int32_t* row = counts + ((size_t)j * NC + ch) * E;
    for (int e = dd * per; e < (dd + 1) * per; ++e) s += row[e];
  }
  w[i] = s;
}

}  // namespace
}  // namespace eb

extern "C" eb_status eb_route_loads_static(const float* logits, int n_mb, int T, int E, int k,
                                           int renorm, int D, int32_t* idx, float* gate,
                                           int32_t* w, int32_t* status_dev, void* stream) {
  using namespace eb;
  if (n_mb < 1 || T < 1 || E < 1 || k < 1 || k > E || D < 1 || E % D != 0)
    return EB_ERR_INVALID_ARG;
  if (!logits || !idx || !gate || !w) return EB_ERR_INVALID_ARG;
  if (E > EB_MAX_ETOT || k > EB_MAX_K || n_mb > 65535) return EB_ERR_UNSUPPORTED;
  const int NC = (T + kChunk - 1) / kChunk;
  if ((long long)n_mb * NC * E > kStaticCountInts) return EB_ERR_TOO_LARGE;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  int32_t* counts = nullptr;
  if (static_counts_ptr(&counts) != cudaSuccess) return EB_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  dim3 grid(NC, n_mb);
  switch (vpl_for(E)) {
    case 1: k_route_counts_static<1><<<grid, 256, 0, s>>>(logits, T, E, k, renorm, NC, idx, gate, counts, status_dev); break;
    case 2: k_route_counts_static<2><<<grid, 256, 0, s>>>(logits, T, E, k, renorm, NC, idx, gate, counts, status_dev); break;
    case 4: k_route_counts_static<4><<<grid, 256, 0, s>>>(logits, T, E, k, renorm, NC, idx, gate, counts, status_dev); break;
    default: k_route_counts_static<8><<<grid, 256, 0, s>>>(logits, T, E, k, renorm, NC, idx, gate, counts, status_dev); break;
  }
  if (cudaGetLastError() != cudaSuccess) return EB_ERR_CUDA;
  const int n = n_mb * D;
  k_fold_static<<<(n + 255) / 256, 256, 0, s>>>(counts, n_mb, NC, E, D, w);
  return cudaGetLastError() == cudaSuccess ? EB_OK : EB_ERR_CUDA;
}
