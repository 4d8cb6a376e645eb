// Routing: softmax top-k with renormalised gates and per-expert token counts.
//
// [EB] §2.1: W_l, I_l = topk(G(h'_l)) -- each token picks its top-k experts and
// weighs them.  The counts T_e per expert are what a rank's load is built
// from ([SysLB] §1: L_r = sum_{e in E_r} T_e).
//
// One CTA routes one 64-token chunk.  Its threads first copy the chunk's
// logits into shared memory with coalesced 16-byte loads (rows padded to an
// odd stride, so that threads reading the same expert of different tokens
// hit different banks).  Then one thread routes one token on its own: it
// walks the E logits keeping its k best in registers, sorted under the order
// (logit descending, expert index ascending) -- each logit becomes a 64-bit
// key (an order-preserving integer image of the float, then the complement
// of the expert index), so the order is a plain integer compare -- and forms
// the gates from the winners (softmax restricted to the top-k and
// renormalised: the full softmax denominator cancels; without
// renormalisation the thread sums exp over all E).  No thread waits on
// another while routing.  Counts go to shared-memory atomics (integers, so
// the result is exact and order-free) and are written once per
// (micro-batch, chunk): no global atomics and no zeroing pass in the step
// path.
#include <math.h>

#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr int kRouteThreads = 256;

// Order-preserving map of a finite float to uint32 (-0 is folded into +0
// first, so equal floats map to equal keys); never 0 for a real value.
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint64_t key) {
  const uint32_t k = (uint32_t)(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ int key_expert(uint64_t key) {
  return (int)(0xffffffffu - (uint32_t)key);
}

// Shared-memory row stride (floats) of a chunk of E logits: odd.
__host__ __device__ __forceinline__ int row_stride(int E) { return E | 1; }

// Bytes of dynamic shared memory of a routing CTA.
__host__ __device__ __forceinline__ size_t route_smem_bytes(int E) {
  return sizeof(float) * (size_t)kChunk * row_stride(E);
}

// Copies rows [t0, t1) of an [*, E] float32 block into shared memory (all
// threads; 16-byte loads when E is a multiple of 4 and the block is aligned).
__device__ __forceinline__ void load_chunk(const float* __restrict__ rows, int t0, int t1, int E,
                                           float* sm) {
  const int st = row_stride(E), n = (t1 - t0) * E;
  const float* src = rows + (size_t)t0 * E;
  if ((E & 3) == 0 && ((uintptr_t)src & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    for (int v = threadIdx.x; v < n / 4; v += blockDim.x) {
      const float4 x = __ldg(s4 + v);
      const int i = 4 * v, r = i / E, c = i % E;  // E % 4 == 0: one row per vector
      float* d = sm + r * st + c;
      d[0] = x.x;
      d[1] = x.y;
      d[2] = x.z;
      d[3] = x.w;
    }
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) sm[(i / E) * st + i % E] = __ldg(src + i);
  }
}

// Routes one token from its shared-memory row: writes its k indices and
// gates (slot order: descending logit, then ascending expert) and counts
// them in hist_s.  KMAX >= k is the register capacity of the top-k list.
template <int KMAX>
__device__ __forceinline__ void route_token(const float* row, int E, int k, int renorm,
                                            int32_t* __restrict__ idx, float* __restrict__ gate,
                                            int* hist_s, bool& nonfinite) {
  uint64_t top[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) top[i] = 0;  // below every real key
  uint64_t kth = 0;                            // the k-th best so far
  for (int e = 0; e < E; ++e) {
    float x = row[e];
    if (!isfinite(x)) {
      nonfinite = true;
      x = -INFINITY;  // selection stays among real experts; the call reports the error
    }
    uint64_t cur = ((uint64_t)order_key(x) << 32) | (0xffffffffu - (uint32_t)e);
    if (cur <= kth) continue;
    // insert into the sorted list: the larger key stays, the smaller moves
    // on down; what falls off the end is dropped
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      const uint64_t hi = cur > top[i] ? cur : top[i];
      const uint64_t lo = cur > top[i] ? top[i] : cur;
      if (i < k) {
        top[i] = hi;
        cur = lo;
      }
    }
    // the k-th best is the smallest of the first k (a minimum rather than
    // top[k - 1], which would index the register list at run time)
    kth = ~0ull;
#pragma unroll
    for (int i = 0; i < KMAX; ++i)
      if (i < k) kth = top[i] < kth ? top[i] : kth;
  }
  const float vmax = key_value(top[0]);
  float ex[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) ex[i] = i < k ? expf(key_value(top[i]) - vmax) : 0.f;
  float denom;
  if (renorm) {
    // pairwise sum of the k terms (a tree keeps the rounding error at
    // log2(k) additions)
    float t[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) t[i] = ex[i];
#pragma unroll
    for (int w = KMAX / 2; w >= 1; w /= 2)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] += t[i + w];
    denom = t[0];
  } else {
    // softmax over all E: eight interleaved partial sums, then a tree
    float part[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) part[i] = 0.f;
    for (int e0 = 0; e0 < E; e0 += 8)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (e0 + i < E) {
          const float x = row[e0 + i];
          part[i] += expf((isfinite(x) ? x : -INFINITY) - vmax);
        }
#pragma unroll
    for (int w = 4; w >= 1; w /= 2)
#pragma unroll
      for (int i = 0; i < w; ++i) part[i] += part[i + w];
    denom = part[0];
  }
#pragma unroll
  for (int i = 0; i < KMAX; ++i)
    if (i < k) {
      const int e = key_expert(top[i]);
      idx[i] = e;
      gate[i] = ex[i] / denom;
      atomicAdd(&hist_s[e], 1);
    }
}

template <int KMAX>
__device__ __forceinline__ void route_rows_in_smem(const float* sm, int t0, int t1, int E, int k,
                                                   int renorm, int32_t* __restrict__ idx,
                                                   float* __restrict__ gate, int* hist_s,
                                                   bool& nonfinite) {
  const int t = t0 + (int)threadIdx.x;
  if (t < t1)
    route_token<KMAX>(sm + threadIdx.x * row_stride(E), E, k, renorm, idx + (size_t)t * k,
                      gate + (size_t)t * k, hist_s, nonfinite);
}

// Step path: CTA (c, j) routes chunk c of micro-batch j at its layer l_j if j
// is in need_route; its counts land in chunk_hist[j][c][:] and are added
// (integer atomics: exact, order-free) to the micro-batch's histogram
// hist[j][:] and rank loads w[j][:], which the previous step zeroed.  The
// loads fold the counts by the context's expert placement: contiguous
// blocks of E/D experts, or emap[e] if one was set.
template <int KMAX>
__global__ void __launch_bounds__(kRouteThreads) k_route_step(Dims d, State* __restrict__ st,
                                                     const float* __restrict__ logits,
                                                     int32_t* __restrict__ idx,
                                                     float* __restrict__ gate,
                                                     int32_t* __restrict__ chunk_hist,
                                                     int32_t* __restrict__ hist,
                                                     int32_t* __restrict__ wload,
                                                     const int32_t* __restrict__ emap,
                                                     long long mb_stride, long long layer_stride) {
  pdl_enter();
  const int c = blockIdx.x, j = blockIdx.y;
  // nothing routes while a timed-out step awaits eb_reset
  if (!((st->need_route >> j) & 1u) || st->status == EB_ERR_TIMEOUT) return;
  const int l = st->layer[j];
  extern __shared__ float rows_s[];
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int w_s[EB_MAX_D];
  __shared__ int bad;
  for (int e = threadIdx.x; e < d.E; e += blockDim.x) hist_s[e] = 0;
  for (int r = threadIdx.x; r < d.D; r += blockDim.x) w_s[r] = 0;
  if (threadIdx.x == 0) bad = 0;
  // rows of micro-batch j at layer l: the caller's logits [M, L, T, E], or
  // the router's scores of this step (see launch_route_step)
  const float* blk = logits + (size_t)j * mb_stride + (size_t)l * layer_stride;
  const int t0 = c * kChunk, t1 = min(d.T, t0 + kChunk);
  load_chunk(blk, t0, t1, d.E, rows_s);
  __syncthreads();
  bool nonfinite = false;
  route_rows_in_smem<KMAX>(rows_s, t0, t1, d.E, d.k, d.renorm, idx + (size_t)j * d.T * d.k,
                           gate + (size_t)j * d.T * d.k, hist_s, nonfinite);
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
}

// Stand-alone path: rows [c*kChunk, ...) of an [n, E] block; counts summed
// into hist[E] with one global atomic per (CTA, expert) with a non-zero count.
template <int KMAX>
__global__ void __launch_bounds__(kRouteThreads) k_route_rows(const float* __restrict__ logits,
                                                              int n, int E, int k, int renorm,
                                                              int32_t* __restrict__ idx,
                                                              float* __restrict__ gate,
                                                              int32_t* __restrict__ hist,
                                                              int32_t* __restrict__ status) {
  extern __shared__ float rows_s[];
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int bad;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_s[e] = 0;
  if (threadIdx.x == 0) bad = 0;
  const int t0 = blockIdx.x * kChunk, t1 = min(n, t0 + kChunk);
  load_chunk(logits, t0, t1, E, rows_s);
  __syncthreads();
  bool nonfinite = false;
  route_rows_in_smem<KMAX>(rows_s, t0, t1, E, k, renorm, idx, gate, hist_s, nonfinite);
  if (nonfinite) bad = 1;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist_s[e]) atomicAdd(&hist[e], hist_s[e]);
  if (threadIdx.x == 0 && bad && status) atomicExch(status, EB_ERR_NONFINITE);
}

int kmax_for(int k) { return k <= 8 ? 8 : k <= 16 ? 16 : 32; }

// Dynamic shared memory above the default 48 KiB (E > 187) needs the
// kernel's attribute raised once.
template <typename K>
cudaError_t allow_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

cudaError_t launch_route_step(const Dims& d, const CtxDev& c, const Work& w, const float* logits,
                              long long mb_stride, long long layer_stride, cudaStream_t s) {
  dim3 grid(d.NC, d.M);
  const int32_t* emap = c.use_emap ? c.emap : nullptr;
  const size_t smem = route_smem_bytes(d.E);
  auto go = [&](auto kernel) {
    cudaError_t e = allow_smem(kernel, smem);
    if (e == cudaSuccess)
      e = launch_pdl(kernel, grid, dim3(kRouteThreads), smem, s, 1, d, c.st, logits, w.idx, w.gate,
                     w.chunk_hist, c.hist, c.w, emap, mb_stride, layer_stride);
    return e;
  };
  switch (kmax_for(d.k)) {
    case 8: return go(k_route_step<8>);
    case 16: return go(k_route_step<16>);
    default: return go(k_route_step<32>);
  }
}

cudaError_t launch_route_rows(const float* logits, int n, int E, int k, int renorm, int32_t* idx,
                              float* gate, int32_t* hist, int32_t* status, cudaStream_t s) {
  if (cuda_error_pending()) return cudaErrorUnknown;
  cudaError_t err = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)E, s);
  if (err != cudaSuccess || n == 0) return err;
  const dim3 grid((n + kChunk - 1) / kChunk);
  const size_t smem = route_smem_bytes(E);
  auto go = [&](auto kernel) {
    cudaError_t e = allow_smem(kernel, smem);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kRouteThreads, smem, s>>>(logits, n, E, k, renorm, idx, gate, hist, status);
    return cudaGetLastError();
  };
  switch (kmax_for(k)) {
    case 8: return go(k_route_rows<8>);
    case 16: return go(k_route_rows<16>);
    default: return go(k_route_rows<32>);
  }
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
template <int KMAX>
__global__ void __launch_bounds__(kRouteThreads) k_route_counts_static(const float* __restrict__ logits,
                                                              int T, int E, int k, int renorm, int NC,
                                                              int32_t* __restrict__ idx,
                                                              float* __restrict__ gate,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ status) {
  const int c = blockIdx.x, j = blockIdx.y;
  extern __shared__ float rows_s[];
  __shared__ int hist_s[EB_MAX_ETOT];
  __shared__ int bad;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist_s[e] = 0;
  if (threadIdx.x == 0) bad = 0;
  const int t0 = c * kChunk, t1 = min(T, t0 + kChunk);
  load_chunk(logits + (size_t)j * T * E, t0, t1, E, rows_s);
  __syncthreads();
  bool nonfinite = false;
  route_rows_in_smem<KMAX>(rows_s, t0, t1, E, k, renorm, idx + (size_t)j * T * k,
                           gate + (size_t)j * T * k, hist_s, nonfinite);
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
  const size_t smem = route_smem_bytes(E);
  auto go = [&](auto kernel) {
    if (allow_smem(kernel, smem) != cudaSuccess) return false;
    kernel<<<grid, kRouteThreads, smem, s>>>(logits, T, E, k, renorm, NC, idx, gate, counts,
                                             status_dev);
    return cudaGetLastError() == cudaSuccess;
  };
  const bool launched = kmax_for(k) == 8 ? go(k_route_counts_static<8>)
                        : kmax_for(k) == 16 ? go(k_route_counts_static<16>)
                                            : go(k_route_counts_static<32>);
  if (!launched) return EB_ERR_CUDA;
  const int n = n_mb * D;
  k_fold_static<<<(n + 255) / 256, 256, 0, s>>>(counts, n_mb, NC, E, D, w);
  return cudaGetLastError() == cudaSuccess ? EB_OK : EB_ERR_CUDA;
}
