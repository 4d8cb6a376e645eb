// Token permutation into (layer, expert) segments and the gated combine.
//
// [EB] §2.2 (expert parallelism): tokens are dispatched to the experts that
// process them and the expert outputs come back to be aggregated by the
// weighted sum of Eq. (1).  On one GPU the "dispatch" is a permutation of the
// RunSet's token rows into contiguous segments, one per (layer, expert) --
// micro-batches at the same layer share a segment --, and the "combine" is
//   out[j,t] = (h[j,t] +) sum_{s<k} gate[j,t,s] * y[pos(j,t,s)]
//              (+ sum over shared experts of y[pos(j,t,k+s')])
// summed in slot order in fp32 and rounded once to the storage type.
// [EB-read] §2.1: scheduling may change neither the expert set, the gates nor
// the aggregation order -- the slot order here is fixed.
//
// Both kernels are HBM-bound copies: one warp per token row, 16-byte vector
// loads and stores, each row read once and written (permute) k + n_shared
// times or k + n_shared rows read and one written (combine).
#include <cuda_bf16.h>

#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kPermThreads = 256;
constexpr int kMaxSlots = EB_MAX_K;  // k + n_shared <= 32 (one lane per slot in the combine)

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// CTA (c, j): chunk c of RunSet micro-batch j.  Row of (t, s) = base of
// (j, c, expert) + number of earlier (t', s') of this chunk with the same
// expert, so rows follow (micro-batch, token, slot) order inside a segment.
// Each chunk's ranks are computed by kPermSplit CTAs (cheap, identical); each
// copies a quarter of the chunk's tokens, so the HBM-bound copy has 4x the CTAs.
constexpr int kPermSplit = 4;

template <typename T>
__global__ void __launch_bounds__(kPermThreads) k_permute(Dims d, const State* __restrict__ st,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ chunk_hist,
                                                          const int32_t* __restrict__ seg_rows,
                                                          const int32_t* __restrict__ prior,
                                                          int32_t* __restrict__ pos,
                                                          const T* __restrict__ hidden,
                                                          T* __restrict__ A) {
  const int c = blockIdx.x / kPermSplit, part = blockIdx.x % kPermSplit, j = blockIdx.y;
  if (!((st->runset >> j) & 1u)) return;
  __shared__ int cnt[kPermThreads / 32][EB_MAX_ETOT];
  __shared__ int running[EB_MAX_ETOT];
  __shared__ int dest[kChunk * kMaxSlots];
  __shared__ int bj[EB_MAX_ETOT];  // first row of (j, this chunk, expert)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = c * kChunk, nt = min(kChunk, d.T - t0);
  const int k = d.k, kk = d.kk, E = d.E, Et = d.Etot;
  const int g = st->group_of[j];
  for (int e = tid; e < Et; e += kPermThreads) {
    int b = seg_rows[g * Et + e] + prior[j * Et + e];
    if (e < E) {
      const int32_t* ch = chunk_hist + (size_t)j * d.NC * E + e;
      int cc = 0;
      for (; cc + 8 <= c; cc += 8) {  // eight independent loads in flight
        int part[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) part[u] = __ldg(ch + (size_t)(cc + u) * E);
#pragma unroll
        for (int u = 0; u < 8; ++u) b += part[u];
      }
      for (; cc < c; ++cc) b += __ldg(ch + (size_t)cc * E);
    } else {
      b += c * kChunk;
    }
    bj[e] = b;
  }
  for (int e = tid; e < E; e += kPermThreads) running[e] = 0;
  const int npairs = nt * k;
  const int32_t* idx_c = idx + ((size_t)j * d.T + t0) * k;
  for (int r0 = 0; r0 < npairs; r0 += kPermThreads) {
    for (int i = tid; i < (kPermThreads / 32) * E; i += kPermThreads) cnt[i / E][i % E] = 0;
    __syncthreads();
    const int p = r0 + tid;
    const int e = p < npairs ? idx_c[p] : -1;
    const unsigned peers = __match_any_sync(kFull, e);
    const int rank = __popc(peers & lanemask_lt());
    if (e >= 0 && lane == __ffs(peers) - 1) cnt[warp][e] = __popc(peers);
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPermThreads) {
      int run = running[ee];
      for (int w = 0; w < kPermThreads / 32; ++w) {
        const int t = cnt[w][ee];
        cnt[w][ee] = run;
        run += t;
      }
      running[ee] = run;
    }
    __syncthreads();
    if (e >= 0) {
      const int t = p / k, s = p % k;
      const int row = bj[e] + cnt[warp][e] + rank;
      dest[t * kk + s] = row;
      if (part == 0) pos[((size_t)j * d.T + t0 + t) * kk + s] = row;
    }
    __syncthreads();
  }
  for (int i = tid; i < nt * d.n_shared; i += kPermThreads) {
    const int t = i / d.n_shared, s = i % d.n_shared;
    const int row = bj[E + s] + t;
    dest[t * kk + k + s] = row;
    if (part == 0) pos[((size_t)j * d.T + t0 + t) * kk + k + s] = row;
  }
  __syncthreads();
  const int nvec = d.H * (int)sizeof(T) / 16;
  const int per = (nt + kPermSplit - 1) / kPermSplit;
  const int ta = part * per, tb = min(nt, ta + per);
  // each warp copies two tokens at a time: both rows' 16-byte vectors are
  // loaded into registers (8 per lane per token) before any store is issued
  constexpr int kU = 8;
  for (int t = ta + warp; t < tb; t += 2 * (kPermThreads / 32)) {
    const int t2 = t + kPermThreads / 32;
    const bool two = t2 < tb;
    const uint4* src0 = reinterpret_cast<const uint4*>(hidden + ((size_t)j * d.T + t0 + t) * d.H);
    const uint4* src1 = reinterpret_cast<const uint4*>(hidden + ((size_t)j * d.T + t0 + (two ? t2 : t)) * d.H);
    for (int base = 0; base < nvec; base += 32 * kU) {
      uint4 v0[kU], v1[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int v = base + u * 32 + lane;
        if (v < nvec) {
          v0[u] = __ldg(src0 + v);
          if (two) v1[u] = __ldg(src1 + v);
        }
      }
      for (int s = 0; s < kk; ++s) {
        uint4* dst0 = reinterpret_cast<uint4*>(A + (size_t)dest[t * kk + s] * d.H);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int v = base + u * 32 + lane;
          if (v < nvec) dst0[v] = v0[u];
        }
        if (two) {
          uint4* dst1 = reinterpret_cast<uint4*>(A + (size_t)dest[t2 * kk + s] * d.H);
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int v = base + u * 32 + lane;
            if (v < nvec) dst1[v] = v1[u];
          }
        }
      }
    }
  }
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

constexpr int kCombineTokens = 8;  // one warp per token

template <typename T>
__global__ void __launch_bounds__(256) k_combine(Dims d, const State* __restrict__ st,
                                                  const float* __restrict__ gate,
                                                  const int32_t* __restrict__ pos,
                                                  const T* __restrict__ y, T* hidden) {
  const int j = blockIdx.y;
  if (!((st->runset >> j) & 1u)) return;
  __shared__ int s_row[kCombineTokens][kMaxSlots];
  __shared__ float s_gate[kCombineTokens][kMaxSlots];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * kCombineTokens + warp;
  if (t >= d.T) return;
  const int k = d.k, kk = d.kk;
  constexpr int VE = Vec<T>::n;
  const int nvec = d.H / VE;
  const size_t tok = (size_t)j * d.T + t;
  if (lane < kk) s_row[warp][lane] = pos[tok * kk + lane];
  if (lane < k) s_gate[warp][lane] = gate[tok * k + lane];
  __syncwarp();
  T* out = hidden + tok * d.H;
  // two 16-byte vectors per lane per pass: 2 * kk loads in flight
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
    for (int s0 = 0; s0 < kk; s0 += 8) {
      uint4 r0[8], r1[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (s0 + u < kk) {
          const uint4* yrow = reinterpret_cast<const uint4*>(y + (size_t)s_row[warp][s0 + u] * d.H);
          r0[u] = __ldg(yrow + v0);
          if (has1) r1[u] = __ldg(yrow + v1);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s0 + u;
        if (s >= kk) break;
        float y0[VE], y1[VE];
        Vec<T>::unpack(r0[u], y0);
        if (has1) Vec<T>::unpack(r1[u], y1);
        if (s < k) {
          const float g = s_gate[warp][s];
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

}  // namespace

cudaError_t launch_permute(const Dims& d, const CtxDev& c, const Work& w, const void* hidden,
                           cudaStream_t s) {
  dim3 grid(d.NC * kPermSplit, d.M);
  if (d.dtype == EB_DTYPE_BF16)
    k_permute<__nv_bfloat16><<<grid, kPermThreads, 0, s>>>(
        d, c.st, w.idx, w.chunk_hist, w.seg_rows, w.prior, w.pos,
        static_cast<const __nv_bfloat16*>(hidden), static_cast<__nv_bfloat16*>(w.A));
  else
    k_permute<float><<<grid, kPermThreads, 0, s>>>(d, c.st, w.idx, w.chunk_hist, w.seg_rows,
                                                   w.prior, w.pos, static_cast<const float*>(hidden),
                                                   static_cast<float*>(w.A));
  return cudaGetLastError();
}

cudaError_t launch_combine(const Dims& d, const CtxDev& c, const Work& w, void* hidden,
                           cudaStream_t s) {
  dim3 grid((d.T + kCombineTokens - 1) / kCombineTokens, d.M);
  if (d.dtype == EB_DTYPE_BF16)
    k_combine<__nv_bfloat16><<<grid, 256, 0, s>>>(d, c.st, w.gate, w.pos,
                                                  static_cast<const __nv_bfloat16*>(w.y),
                                                  static_cast<__nv_bfloat16*>(hidden));
  else
    k_combine<float><<<grid, 256, 0, s>>>(d, c.st, w.gate, w.pos, static_cast<const float*>(w.y),
                                          static_cast<float*>(hidden));
  return cudaGetLastError();
}

}  // namespace eb
