// Token permutation into (layer, expert) segments and the gated combine.
//
// [EB] §2.2 (expert parallelism): tokens are dispatched to the experts that
// process them and the expert outputs come back to be aggregated by the
// weighted sum of Eq. (1).  On one GPU the "dispatch" is a permutation of the
// RunSet's token rows into contiguous segments, one per (layer, expert) --
// micro-batches at the same layer share a segment --, and the "combine" is
//   out[j,t] = (h[j,t] +) sum_{s<k} gate[j,t,s] * y[j,t,s]
//              (+ sum over shared experts of y[j,t,k+s'])
// summed in slot order in fp32 and rounded once to the storage type.
// [EB-read] §2.1: scheduling may change neither the expert set, the gates nor
// the aggregation order -- the slot order here is fixed.
//
// The permutation: routing already ranked every (token, slot) pair among its
// micro-batch's pairs of the same expert (none of which depends on the
// schedule); the row copy adds the step's segment bases, writes each row's
// position and its inverse, the (token, slot) of every row, and moves the
// rows.  When GEMM 1 gathers the rows from the hidden states itself, there is
// no copy, and k_positions computes the positions from the routing counts
// in a pass of its own.  GEMM 2 writes
// each row's output at its (token, slot) position, so the combine reads a
// token's k + n_shared outputs from one contiguous run.  The copy and the combine are HBM-bound and
// persistent: a grid of resident CTAs sized to the SM count works through
// the RunSet's tokens, one warp per token row with 16-byte vector loads and
// stores, so the work spreads evenly over the SMs whatever the RunSet size
// (no partial last wave).  The copy strides over the tokens; the combine's
// CTAs claim them from a counter, since some of them may start late beside
// the next step's scheduler.  Each row is read once and written k + n_shared
// times (permute), or k + n_shared rows are read and one written (combine).
#include <cuda_bf16.h>

#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kPermThreads = 256;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

constexpr int kPosThreads = 512;

// CTA (c, j): chunk c of RunSet micro-batch j.  Row of (t, s) = base of
// (j, c, expert) + number of earlier (t', s') of this chunk with the same
// expert, so rows follow (micro-batch, token, slot) order inside a segment.
// The base is the segment's first row + the rows of earlier RunSet members
// of the segment (prior) + this micro-batch's rows in chunks 0..c-1.  Every
// load that does not depend on the step state (the chunk's routing indices,
// prior, the earlier chunks' counts) is issued before the state is read.
__global__ void __launch_bounds__(kPosThreads) k_positions(Dims d, const State* __restrict__ st,
                                                           const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ chunk_hist,
                                                           const int32_t* __restrict__ seg_rows,
                                                           const int32_t* __restrict__ prior,
                                                           int32_t* __restrict__ pos,
                                                           int32_t* __restrict__ rowslot) {
  constexpr int kWarps = kPosThreads / 32;
  pdl_enter();
  const int c = blockIdx.x, j = blockIdx.y;
  __shared__ int cnt[kWarps][EB_MAX_ETOT];
  __shared__ int running[EB_MAX_ETOT];
  __shared__ int bj[EB_MAX_ETOT];  // first row of (j, this chunk, expert)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = c * kChunk, nt = min(kChunk, d.T - t0);
  const int k = d.k, kk = d.kk, E = d.E, Et = d.Etot;
  const int npairs = nt * k;
  const int32_t* idx_c = idx + ((size_t)j * d.T + t0) * k;
  int32_t* pos_c = pos + ((size_t)j * d.T + t0) * kk;
  // state-independent loads: the first round's expert, and for expert
  // e = tid % Et the counts of chunks part, part + parts, ... below c
  // (parts = threads per expert) plus, in part 0, prior
  int e_next = tid < npairs ? __ldg(idx_c + tid) : -1;
  const int parts = kPosThreads / Et, part = tid / Et, pe = tid % Et;
  int partial = 0;
  if (part < parts) {
    if (pe < E) {
      const int32_t* ch = chunk_hist + (size_t)j * d.NC * E + pe;
      int cc = part;
      for (; cc + 7 * parts < c; cc += 8 * parts) {  // eight independent loads in flight
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(ch + (size_t)(cc + u * parts) * E);
#pragma unroll
        for (int u = 0; u < 8; ++u) partial += v[u];
      }
      for (; cc < c; cc += parts) partial += __ldg(ch + (size_t)cc * E);
    } else if (part == 0) {
      partial = c * kChunk;  // shared expert: every token of the earlier chunks
    }
    if (part == 0) partial += __ldg(prior + j * Et + pe);
  }
  for (int i = tid; i < kWarps * E; i += kPosThreads) cnt[i / E][i % E] = 0;
  for (int e = tid; e < E; e += kPosThreads) running[e] = 0;
  if (!((st->runset >> j) & 1u)) return;
  const int g = st->group_of[j];
  if (part == 0) bj[pe] = partial + seg_rows[g * Et + pe];
  __syncthreads();
  if (part > 0 && part < parts && partial) atomicAdd(&bj[pe], partial);
  for (int r0 = 0; r0 < npairs; r0 += kPosThreads) {
    const int p = r0 + tid;
    const int e = e_next;
    const unsigned peers = __match_any_sync(kFull, e);
    const int rank = __popc(peers & lanemask_lt());
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] = __popc(peers);
    if (p + kPosThreads < npairs) e_next = idx_c[p + kPosThreads];
    else e_next = -1;
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPosThreads) {
      int run = running[ee];
      for (int w = 0; w < kWarps; ++w) {
        const int t = cnt[w][ee];
        cnt[w][ee] = run;
        run += t;
      }
      running[ee] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int row = bj[e] + cnt[warp][e] + rank;
      pos_c[(p / k) * kk + p % k] = row;
      rowslot[row] = (j * d.T + t0 + p / k) * kk + p % k;
    }
    if (r0 + kPosThreads < npairs) {
      __syncthreads();
      for (int i = tid; i < kWarps * E; i += kPosThreads) cnt[i / E][i % E] = 0;
      __syncthreads();
    }
  }
  for (int i = tid; i < nt * d.n_shared; i += kPosThreads) {
    const int t = i / d.n_shared, s = i % d.n_shared;
    pos_c[t * kk + k + s] = bj[E + s] + t;
    rowslot[bj[E + s] + t] = (j * d.T + t0 + t) * kk + k + s;
  }
}

// Token u of the RunSet (members in ascending order, T tokens each).
__device__ __forceinline__ size_t runset_token(const State* st, int T, int u) {
  return (size_t)st->run_list[u / T] * T + (u % T);
}

// What the row copy needs to place the rows itself (engines other than the
// gathering one, which keep k_positions): routing's per-pair ranks and chunk
// offsets, the step's segment bases and prior rows; the positions it writes.
struct Place {
  const int32_t* idx;       // [M][T][k]
  const int32_t* rank;      // [M][T][k]: place among the chunk's pairs of the expert
  const int32_t* cbase;     // [M][NC][E]: pairs of the expert in the earlier chunks
  const int32_t* seg_rows;  // first row of each (group, expert) segment
  const int32_t* prior;     // [M][Etot]: rows of the segment taken by earlier RunSet members
  int32_t* pos;             // [M][T][kk]: row of each (token, slot), written here
  int32_t* rowslot;         // [Rcap]: (token, slot) of each row, written here
  long long Rcap;
};

// Row of slot s (< k + n_shared) of token t of RunSet member j, recorded in
// pos and rowslot: the segment's first row, the rows of earlier RunSet
// members in it, and the pair's place among j's pairs of that expert in
// (token, slot) order -- the rows k_positions computes, in the same order.
// A row outside [0, Rcap) (inconsistent inputs) is returned as -1 and
// nothing is stored for it.
__device__ __forceinline__ int place_row(const Dims& d, const State* st, const Place& pl, int j,
                                         int t, int s) {
  const size_t tok = (size_t)j * d.T + t;
  int e, r;
  if (s < d.k) {
    e = __ldg(pl.idx + tok * d.k + s);
    r = __ldg(pl.rank + tok * d.k + s) +
        __ldg(pl.cbase + ((size_t)j * d.NC + t / kChunk) * d.E + e);
  } else {  // shared expert: every token of j has one pair
    e = d.E + (s - d.k);
    r = t;
  }
  const int row = __ldg(pl.seg_rows + st->group_of[j] * d.Etot + e) +
                  __ldg(pl.prior + j * d.Etot + e) + r;
  if (row < 0 || (long long)row >= pl.Rcap) return -1;
  pl.pos[tok * d.kk + s] = row;
  pl.rowslot[row] = (int)(tok * d.kk + s);
  return row;
}

// Persistent copy: warp w moves tokens w, w + W, ... (W = warps in the grid),
// two at a time: both rows' 16-byte vectors are loaded into registers (8 per
// lane per token) before the k + n_shared stores of each.
template <typename T>
__global__ void __launch_bounds__(kPermThreads) k_permute_copy(Dims d, const State* __restrict__ st,
                                                               Place pl,
                                                               const T* __restrict__ hidden,
                                                               T* __restrict__ A) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int W = (int)(gridDim.x * (kPermThreads / 32));
  const int wid = (int)(blockIdx.x * (kPermThreads / 32) + (threadIdx.x >> 5));
  const int units = st->n_run * d.T;
  const int kk = d.kk;
  const int nvec = d.H * (int)sizeof(T) / 16;
  constexpr int kU = 8;
  for (int u = wid; u < units; u += 2 * W) {
    const int u2 = u + W;
    const bool two = u2 < units;
    const size_t tok0 = runset_token(st, d.T, u), tok1 = runset_token(st, d.T, two ? u2 : u);
    // slot rows of both tokens, one per lane
    const int row0 = lane < kk ? place_row(d, st, pl, st->run_list[u / d.T], u % d.T, lane) : 0;
    const int row1 =
        two && lane < kk ? place_row(d, st, pl, st->run_list[u2 / d.T], u2 % d.T, lane) : 0;
    const uint4* src0 = reinterpret_cast<const uint4*>(hidden + tok0 * d.H);
    const uint4* src1 = reinterpret_cast<const uint4*>(hidden + tok1 * d.H);
    for (int base = 0; base < nvec; base += 32 * kU) {
      uint4 v0[kU], v1[kU];
#pragma unroll
      for (int q = 0; q < kU; ++q) {
        const int v = base + q * 32 + lane;
        if (v < nvec) {
          v0[q] = __ldg(src0 + v);
          if (two) v1[q] = __ldg(src1 + v);
        }
      }
      for (int s = 0; s < kk; ++s) {
        const int r0 = __shfl_sync(kFull, row0, s);
        const int r1 = __shfl_sync(kFull, row1, s);
        if (r0 >= 0) {
          uint4* dst0 = reinterpret_cast<uint4*>(A + (size_t)r0 * d.H);
#pragma unroll
          for (int q = 0; q < kU; ++q) {
            const int v = base + q * 32 + lane;
            if (v < nvec) dst0[v] = v0[q];
          }
        }
        if (two && r1 >= 0) {
          uint4* dst1 = reinterpret_cast<uint4*>(A + (size_t)r1 * d.H);
#pragma unroll
          for (int q = 0; q < kU; ++q) {
            const int v = base + q * 32 + lane;
            if (v < nvec) dst1[v] = v1[q];
          }
        }
      }
    }
  }
}

// ---- the copy by the TMA engine ----
// Rows of up to kBulkMaxRowBytes are copied with bulk copies: a warp's lane 0
// loads a token's row into one of its kBulkSlots shared-memory slots
// (cp.async.bulk, completion on an mbarrier), then lanes s < k + n_shared
// each store it to the row of slot s (cp.async.bulk to global, one bulk
// group per lane per token).  Before a slot is loaded again, every lane's
// stores that read it (kBulkSlots tokens back) must have read it.  The copy engine
// moves the bytes; the warps only issue.
constexpr int kBulkWarps = 8;
constexpr int kBulkSlots = 3;
constexpr int kBulkMaxRowBytes = 8192;
static_assert(kBulkWarps * kBulkSlots * kBulkMaxRowBytes <= 227 * 1024,
              "the row slots of a CTA fit its shared memory");
constexpr unsigned long long kBulkWaitNs = 4000000000ull;  // 4 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier; false after kBulkWaitNs.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity) {
  if (bar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (bar_try(bar, parity)) return true;
    if ((it & 63) == 0 && global_ns() - t0 > kBulkWaitNs) return false;
  }
}

template <typename T>
__global__ void __launch_bounds__(32 * kBulkWarps) k_permute_bulk(Dims d, State* __restrict__ st,
                                                                  Place pl,
                                                                  const T* __restrict__ hidden,
                                                                  T* __restrict__ A) {
  pdl_enter();
  extern __shared__ __align__(128) uint8_t bulk_rows[];
  __shared__ __align__(8) uint64_t bars[kBulkWarps][kBulkSlots];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = (int)(gridDim.x * kBulkWarps);
  const int wid = (int)(blockIdx.x * kBulkWarps) + warp;
  const int units = st->n_run * d.T;
  const int kk = d.kk;
  const uint32_t bytes = (uint32_t)(d.H * sizeof(T));
  if (lane == 0) {
    for (int sl = 0; sl < kBulkSlots; ++sl)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[warp][sl])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  uint32_t phases = 0;  // bit sl: parity of slot sl's next completion
  int it = 0;
  int row = 0;  // this lane's row of the current token (placed one token ahead)
  for (int u = wid; u < units; u += W, ++it) {
    const int sl = it % kBulkSlots;
    uint8_t* buf = bulk_rows + (size_t)(warp * kBulkSlots + sl) * bytes;
    const uint32_t bar = smem_u32(&bars[warp][sl]);
    // the stores issued from this slot two tokens ago have read it
    if (lane < kk) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kBulkSlots - 1) : "memory");
    __syncwarp();
    const int j = st->run_list[u / d.T], t = u % d.T;
    const size_t tok = (size_t)j * d.T + t;
    if (lane == 0) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(smem_u32(buf)), "l"(hidden + tok * d.H), "r"(bytes), "r"(bar)
          : "memory");
    }
    if (it == 0 && lane < kk) row = place_row(d, st, pl, j, t, lane);
    // the next token's rows are placed while this token's row loads
    int row_next = 0;
    const int un = u + W;
    if (un < units && lane < kk) row_next = place_row(d, st, pl, st->run_list[un / d.T], un % d.T, lane);
    const bool ok = bar_wait(bar, (phases >> sl) & 1u);
    phases ^= 1u << sl;
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) {
        atomicCAS(&st->status, EB_OK, EB_ERR_TIMEOUT);
        bar_wait(bar, (phases >> sl) & 1u ^ 1u);  // give the load in flight one more bounded wait
      }
      break;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (lane < kk && row >= 0) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                   ::"l"(A + (size_t)row * d.H), "r"(smem_u32(buf)), "r"(bytes)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    row = row_next;
  }
  // every store has completed (its writes are performed) before the CTA exits
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, int v, float* out) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p) + v);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  }
  __device__ static void load_plain(const float* p, int v, float* out) {
    const float4 x = reinterpret_cast<const float4*>(p)[v];
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
  }
  __device__ static void unpack(const uint4& x, float* out) {
    out[0] = __uint_as_float(x.x); out[1] = __uint_as_float(x.y);
    out[2] = __uint_as_float(x.z); out[3] = __uint_as_float(x.w);
  }
  __device__ static void store(float* p, int v, const float* in) {
    reinterpret_cast<float4*>(p)[v] = make_float4(in[0], in[1], in[2], in[3]);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, int v, float* out) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(p) + v);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ static void load_plain(const __nv_bfloat16* p, int v, float* out) {
    const uint4 x = reinterpret_cast<const uint4*>(p)[v];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ static void unpack(const uint4& x, float* out) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, int v, const float* in) {
    uint4 x;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
    reinterpret_cast<uint4*>(p)[v] = x;
  }
};

constexpr int kCombineThreads = 256;

// Tokens a combine CTA claims at a time (two per warp).
constexpr int kCombineClaim = 2 * (kCombineThreads / 32);

// Persistent: each CTA claims kCombineClaim consecutive tokens of the RunSet
// at a time from the step view's counter, and warp w combines the claim's
// tokens w and w + 8.  Claiming keeps a CTA that starts late (beside the
// next step's scheduler) from holding the others up.  The step view (not
// the live state, which the next step's scheduler may be rewriting) gives
// the RunSet and the gate buffers.
template <typename T>
__global__ void __launch_bounds__(kCombineThreads, 3) k_combine(Dims d, StepView* __restrict__ view,
                                                             const float* __restrict__ gate,
                                                             const int32_t* __restrict__ pos,
                                                             const T* __restrict__ y, T* hidden,
                                                             int early) {
  if (early) pdl_trigger();
  else pdl_enter();
  __shared__ int s_claim;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int units = view->n_run * d.T;
  const uint32_t gate_buf = view->gate_buf;
  const int k = d.k, kk = d.kk;
  constexpr int VE = Vec<T>::n;
  const int nvec = d.H / VE;
  for (;;) {
    __syncthreads();  // every warp has read the previous claim
    if (threadIdx.x == 0) s_claim = atomicAdd(&view->next, kCombineClaim);
    __syncthreads();
    const int base = s_claim;
    if (base >= units) break;
  for (int u = base + warp; u < min(base + kCombineClaim, units); u += kCombineThreads / 32) {
    const size_t tok = (size_t)view->run_list[u / d.T] * d.T + (u % d.T);
    // the token's expert outputs sit at its slots (tok * kk + s); gates, one
    // per lane
    const int my_row = lane < kk ? (int)(tok * kk + lane) : 0;
    const float my_gate = lane < k ? __ldg(gates_of(gate, gate_buf, d, (long long)tok) + lane) : 0.f;
    T* out = hidden + tok * d.H;
    // two 16-byte vectors per lane per pass, slots loaded four at a time
    // (registers for three CTAs per SM)
    for (int v0 = lane; v0 < nvec; v0 += 64) {
      const int v1 = v0 + 32;
      const bool has1 = v1 < nvec;
      float acc0[VE], acc1[VE];
      if (d.residual) {
        Vec<T>::load_plain(out, v0, acc0);
        if (has1) Vec<T>::load_plain(out, v1, acc1);
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) acc0[i] = acc1[i] = 0.f;
      }
      for (int s0 = 0; s0 < kk; s0 += 4) {
        uint4 r0[4], r1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = __shfl_sync(kFull, my_row, (s0 + q) & 31);
          if (s0 + q < kk) {
            const uint4* yrow = reinterpret_cast<const uint4*>(y + (size_t)row * d.H);
            r0[q] = __ldg(yrow + v0);
            if (has1) r1[q] = __ldg(yrow + v1);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int s = s0 + q;
          const float g = __shfl_sync(kFull, my_gate, s & 31);
          if (s >= kk) break;
          float y0[VE], y1[VE];
          Vec<T>::unpack(r0[q], y0);
          if (has1) Vec<T>::unpack(r1[q], y1);
          if (s < k) {
#pragma unroll
            for (int i = 0; i < VE; ++i) {
              acc0[i] = fmaf(g, y0[i], acc0[i]);
              if (has1) acc1[i] = fmaf(g, y1[i], acc1[i]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < VE; ++i) {
              acc0[i] += y0[i];
              if (has1) acc1[i] += y1[i];
            }
          }
        }
      }
      Vec<T>::store(out, v0, acc0);
      if (has1) Vec<T>::store(out, v1, acc1);
    }
  }
  }
  if (early) pdl_wait();
}

}  // namespace

// Resident CTAs of a persistent kernel: its blocks per SM (by registers and
// shared memory) times the SM count, queried on the first launch and kept in
// the caller's `cache`.
int persistent_grid(const void* kernel, int threads, int& cache) {
  if (cache == 0) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) == cudaSuccess &&
        sms > 0 && per_sm > 0)
      cache = sms * per_sm;
    else
      cache = 148;
  }
  return cache;
}

int g_grid_copy_bf16 = 0, g_grid_copy_f32 = 0, g_grid_comb_bf16 = 0, g_grid_comb_f32 = 0;

cudaError_t launch_positions(const Dims& d, const CtxDev& c, const Work& w, cudaStream_t s) {
  return launch_pdl(k_positions, dim3(d.NC, d.M), dim3(kPosThreads), 0, s, 1, d, c.st,
                    (const int32_t*)w.idx, (const int32_t*)w.chunk_hist,
                    (const int32_t*)w.seg_rows, (const int32_t*)w.prior, w.pos, w.rowslot);
}

int g_grid_bulk_bf16 = 0, g_grid_bulk_f32 = 0;

Place place_of(const Work& w) {
  return Place{w.idx, w.rank, w.cbase, w.seg_rows, w.prior, w.pos, w.rowslot, w.Rcap};
}

template <typename T>
cudaError_t launch_permute_bulk(const Dims& d, const CtxDev& c, const Work& w, const void* hidden,
                                int& grid_cache, cudaStream_t s) {
  const size_t smem = (size_t)kBulkWarps * kBulkSlots * d.H * sizeof(T);
  if (grid_cache == 0) {
    cudaError_t e = cudaFuncSetAttribute(k_permute_bulk<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kBulkWarps * kBulkSlots * kBulkMaxRowBytes));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_permute_bulk<T>,
                                                      32 * kBulkWarps, smem) == cudaSuccess &&
        sms > 0 && per_sm > 0)
      grid_cache = sms * per_sm;
    else
      grid_cache = 148;
  }
  return launch_pdl(k_permute_bulk<T>, dim3(grid_cache), dim3(32 * kBulkWarps), smem, s, 1, d,
                    c.st, place_of(w), static_cast<const T*>(hidden), static_cast<T*>(w.A));
}

cudaError_t launch_permute_copy(const Dims& d, const CtxDev& c, const Work& w, const void* hidden,
                                cudaStream_t s) {
  // rows that fit two shared-memory slots per warp go through the copy engine
  if ((size_t)d.H * (d.dtype == EB_DTYPE_BF16 ? 2 : 4) <= (size_t)kBulkMaxRowBytes)
    return d.dtype == EB_DTYPE_BF16
               ? launch_permute_bulk<__nv_bfloat16>(d, c, w, hidden, g_grid_bulk_bf16, s)
               : launch_permute_bulk<float>(d, c, w, hidden, g_grid_bulk_f32, s);
  if (d.dtype == EB_DTYPE_BF16)
    return launch_pdl(k_permute_copy<__nv_bfloat16>,
                      dim3(persistent_grid((const void*)k_permute_copy<__nv_bfloat16>, kPermThreads,
                                           g_grid_copy_bf16)),
                      dim3(kPermThreads), 0, s, 1, d, c.st, place_of(w),
                      static_cast<const __nv_bfloat16*>(hidden), static_cast<__nv_bfloat16*>(w.A));
  return launch_pdl(k_permute_copy<float>,
                    dim3(persistent_grid((const void*)k_permute_copy<float>, kPermThreads,
                                         g_grid_copy_f32)),
                    dim3(kPermThreads), 0, s, 1, d, c.st, place_of(w), static_cast<const float*>(hidden),
                    static_cast<float*>(w.A));
}

cudaError_t launch_combine(const Dims& d, const Work& w, void* hidden, int slot, bool early,
                           cudaStream_t s) {
  StepView* view = w.views + slot;
  const int ea = early ? 1 : 0;
  if (d.dtype == EB_DTYPE_BF16)
    return launch_pdl(k_combine<__nv_bfloat16>,
                      dim3(persistent_grid((const void*)k_combine<__nv_bfloat16>, kCombineThreads,
                                           g_grid_comb_bf16)),
                      dim3(kCombineThreads), 0, s, 1, d, view, (const float*)w.gate,
                      (const int32_t*)w.pos, static_cast<const __nv_bfloat16*>(w.y),
                      static_cast<__nv_bfloat16*>(hidden), ea);
  return launch_pdl(k_combine<float>,
                    dim3(persistent_grid((const void*)k_combine<float>, kCombineThreads,
                                         g_grid_comb_f32)),
                    dim3(kCombineThreads), 0, s, 1, d, view, (const float*)w.gate,
                    (const int32_t*)w.pos, static_cast<const float*>(w.y),
                    static_cast<float*>(hidden), ea);
}

}  // namespace eb
