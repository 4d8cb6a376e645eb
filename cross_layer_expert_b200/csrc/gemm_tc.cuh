// Host-side interface of the tcgen05 grouped expert GEMMs.
#pragma once

#include <cuda.h>

#include "eb_internal.cuh"

namespace eb {

// TMA descriptors of the four bf16 operands (128-byte swizzle, 64-element K
// boxes of 128 rows).
struct TcMaps {
  CUtensorMap w_gateup;  // [L*Etot*2F rows, H cols]
  CUtensorMap w_down;    // [L*Etot*H rows, F cols]
  CUtensorMap A;         // [Rcap rows, H cols]
  CUtensorMap act;       // [Rcap rows, F cols]
  CUtensorMap A32;       // same buffers, boxes of 32 rows (token-major engines)
  CUtensorMap act32;
};

// Encodes the maps for these buffers; returns cudaErrorInvalidValue if the
// driver rejects a map (alignment, strides).
cudaError_t make_tc_maps(const Dims& d, const Work& w, const void* w_gateup, const void* w_down,
                         TcMaps* maps);
// Opts the kernels into their dynamic shared memory (once per device).
cudaError_t gemm_tc_prepare();
int gemm_tc_smem_bytes(bool gateup);
// Token-major engine: 128 token rows x 256 weight rows per MMA (GEMM 1: 128
// features of gate and up; GEMM 2: 256 features).
// x_rows (GEMM 1 only, may be null): the hidden states [M*T, H]; when given,
// token rows are gathered from them through the row map instead of being
// read from the permuted copy.
// combine_into (GEMM 2 only, may be null): the hidden states [M*T, H]; when
// given, GEMM 2 also combines every RunSet token into them (the step needs no
// combine kernel) using the arrival counters c.arrive, which must be zero
// before the launch and are zero again after it.
cudaError_t launch_gemm_tm(const Dims& d, const CtxDev& c, const Work& w, const TcMaps& maps,
                           int grid, cudaStream_t s, int which, const void* x_rows,
                           void* combine_into);
// Router projection (float32 scores = h W_r^T): maps of the hidden rows
// [rows, H] (boxes of 128 rows) and of the routers [layers * E, H] (boxes of
// E rows), and the launch: n_mb blocks of T rows; st == nullptr routes one
// block at layer 0, else the micro-batches in st->need_route at their layer;
// row t of micro-batch j at layer l lands at out + j mb_stride + l
// layer_stride + t E.
cudaError_t make_router_maps(const void* hidden, long long rows, int H, const void* w_router,
                             int layers, int E, CUtensorMap* map_h, CUtensorMap* map_r);
cudaError_t launch_router(const CUtensorMap& map_h, const CUtensorMap& map_r, int T, int H, int E,
                          int n_mb, const State* st, float* out, long long mb_stride,
                          long long layer_stride, int* status, cudaStream_t s);
// Runs the GEMM's bounded mbarrier wait on a barrier nothing arrives on.
cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* status, cudaStream_t s);
// GEMM `which` (1: gate/up + SwiGLU, 2: down) of a step; grid = persistent
// CTAs (one per SM).
cudaError_t launch_gemm_tc(const Dims& d, const CtxDev& c, const Work& w, const TcMaps& maps,
                           int grid, cudaStream_t s, int which);

}  // namespace eb
