// Grouped expert GEMMs on the CUDA cores (fp32 FFMA), one launch per GEMM
// over every (layer, expert) segment of the step.
//
// Expert FFN of [EB] Eq. (1), read as SwiGLU:
//   act = silu(A W_gate^T) * (A W_up^T),   y = act W_down^T.
// This engine serves fp32 stacks (a tensor-core path would round to tf32) and
// any shape as a cross-check of the tensor-core engine.  Work items are
// (segment, 64-feature block, 64-row chunk), listed by the step's plan; a
// persistent grid walks them.  Accumulation runs over k in ascending order in
// fp32, so a row's result does not depend on which segment or chunk holds it.
#include <cuda_bf16.h>

#include "eb_internal.cuh"

namespace eb {
namespace {

constexpr int BM = kSimtRows;  // token rows per item
constexpr int BN = kSimtFeat;  // output features per item
constexpr int BK = 32;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float v, float* p) { *p = v; }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* p) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ int find_segment(const int32_t* items, int nseg, int item) {
  int lo = 0, hi = nseg;  // items[lo] <= item < items[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (items[mid] <= item) lo = mid;
    else hi = mid;
  }
  return lo;
}

// GATEUP: X = A [R][H], W = w_gateup, out = act [R][F] (SwiGLU epilogue).
// DOWN:   X = act [R][F], W = w_down,  out = y [M*T*kk][H], row r stored at
//         its (token, slot) position rowslot[r].
template <typename T, bool GATEUP>
__global__ void __launch_bounds__(256) k_gemm_simt(Dims d, const State* __restrict__ st,
                                                   const int32_t* __restrict__ seg_rows,
                                                   const int32_t* __restrict__ seg_wid,
                                                   const int32_t* __restrict__ seg_items,
                                                   const T* __restrict__ X,
                                                   const T* __restrict__ W,
                                                   const int32_t* __restrict__ rowslot,
                                                   T* __restrict__ out) {
  pdl_enter();
  const int nseg = st->nseg;
  if (nseg == 0 || st->runset == 0) return;
  const int total = seg_items[nseg];
  const int K = GATEUP ? d.H : d.F;
  const int NOUT = GATEUP ? d.F : d.H;
  const int wstride = GATEUP ? 2 * d.F : d.H;  // weight rows per expert
  __shared__ float Xs[BK][BM + 1];
  __shared__ float Gs[BK][BN + 1];
  __shared__ float Us[GATEUP ? BK : 1][BN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    const int s = find_segment(seg_items, nseg, item);
    const int local = item - seg_items[s];
    const int r_beg = seg_rows[s], cnt = seg_rows[s + 1] - r_beg;
    const int nch = (cnt + BM - 1) / BM;
    const int chunk = local % nch, mb = local / nch;
    const int r0 = r_beg + chunk * BM, nr = min(BM, cnt - chunk * BM);
    const int f0 = mb * BN;
    const T* wg = W + ((size_t)seg_wid[s] * wstride + f0) * K;
    const T* wu = wg + (size_t)d.F * K;  // GATEUP only
    float accg[4][4] = {}, accu[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += BK) {
      __syncthreads();
      for (int i = tid; i < BM * BK; i += 256) {
        const int r = i / BK, kk = i % BK;
        Xs[kk][r] = (r < nr && k0 + kk < K) ? to_f(X[(size_t)(r0 + r) * K + k0 + kk]) : 0.f;
      }
      for (int i = tid; i < BN * BK; i += 256) {
        const int f = i / BK, kk = i % BK;
        const bool ok = f0 + f < NOUT && k0 + kk < K;
        Gs[kk][f] = ok ? to_f(wg[(size_t)f * K + k0 + kk]) : 0.f;
        if (GATEUP) Us[kk][f] = ok ? to_f(wu[(size_t)f * K + k0 + kk]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < BK; ++kk) {
        float xr[4], gr[4], ur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xr[i] = Xs[kk][ty * 4 + i];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gr[i] = Gs[kk][tx * 4 + i];
          if (GATEUP) ur[i] = Us[kk][tx * 4 + i];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            accg[a][b] = fmaf(xr[a], gr[b], accg[a][b]);
            if (GATEUP) accu[a][b] = fmaf(xr[a], ur[b], accu[a][b]);
          }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = ty * 4 + a;
      if (r >= nr) continue;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int f = f0 + tx * 4 + b;
        if (f >= NOUT) continue;
        float v = accg[a][b];
        if (GATEUP) v = v / (1.f + expf(-v)) * accu[a][b];
        // GEMM 2 stores each row at its (token, slot) position
        const size_t orow = GATEUP ? (size_t)(r0 + r) : (size_t)__ldg(rowslot + r0 + r);
        from_f(v, out + orow * NOUT + f);
      }
    }
  }
}

template <typename T>
cudaError_t run(const Dims& d, const CtxDev& c, const Work& w, const void* wgu, const void* wdn,
                cudaStream_t s, int which) {
  const int grid = 148 * 4;
  if (which == 1)
    return launch_pdl(k_gemm_simt<T, true>, dim3(grid), dim3(256), 0, s, 1, d, c.st,
                      (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                      (const int32_t*)w.seg_items1, static_cast<const T*>(w.A),
                      static_cast<const T*>(wgu), (const int32_t*)w.rowslot, static_cast<T*>(w.act));
  return launch_pdl(k_gemm_simt<T, false>, dim3(grid), dim3(256), 0, s, 1, d, c.st,
                    (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                    (const int32_t*)w.seg_items2, static_cast<const T*>(w.act),
                    static_cast<const T*>(wdn), (const int32_t*)w.rowslot, static_cast<T*>(w.y));
}

}  // namespace

cudaError_t launch_gemm_simt(const Dims& d, const CtxDev& c, const Work& w, const void* w_gateup,
                             const void* w_down, cudaStream_t s, int which) {
  if (d.dtype == EB_DTYPE_BF16) return run<__nv_bfloat16>(d, c, w, w_gateup, w_down, s, which);
  return run<float>(d, c, w, w_gateup, w_down, s, which);
}

}  // namespace eb
