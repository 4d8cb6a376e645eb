// Internal declarations shared by the CUDA sources of the cross-layer MoE
// step library.  Citations: [EB] = "EasyBalance: Cross-Layer Load Balancing in
// Distributed MoE Inference" (Wu, Gao, Li, Wu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/eb.h"

namespace eb {

// Tokens handled by one routing / permute / combine CTA.  The per-chunk
// expert counts written by routing give every (micro-batch, chunk, expert) a
// fixed base row, so the permutation is deterministic.
constexpr int kChunk = 64;

// Sizes of GEMM work items: token rows per item and output features per item.
// The tcgen05 tiles are 128 features x kTcRows1 tokens (gate/up GEMM) and
// 128 features x kTcRows2 tokens (down GEMM); the SIMT tile is 64 x 64.
#ifndef EB_TC_ROWS1
#define EB_TC_ROWS1 128
#endif
#ifndef EB_TC_ROWS2
#define EB_TC_ROWS2 256
#endif
constexpr int kTcRows1 = EB_TC_ROWS1;
constexpr int kTcRows2 = EB_TC_ROWS2;
constexpr int kTcFeat = 128;
// Token-major tiles: 128 tokens x (128 gate/up features | 256 down features).
constexpr int kTmRows = 128;
constexpr int kTmFeat1 = 128;
constexpr int kTmFeat2 = 256;
constexpr int kSimtRows = 64;
constexpr int kSimtFeat = 64;

// Columns of a trace row: RunSet mask, sum_d W_d, max_d W_d, sum_j max_d w_j,
// permuted rows R, non-empty (layer, expert) segments.
constexpr int kTraceCols = 6;

// Exact per-step and per-episode accounting lives in this device struct.
struct State {
  int32_t layer[EB_MAX_M];       // l_j: next layer of micro-batch j
  int32_t step_layer[EB_MAX_M];  // layer micro-batch j runs at in this step, -1 if not run
  int32_t run_list[EB_MAX_M];    // RunSet members, ascending
  int32_t group_of[EB_MAX_M];    // segment group (one per distinct layer) of each micro-batch
  int32_t group_layer[EB_MAX_M]; // layer of each group, ascending
  uint32_t pending;              // S: micro-batches with l_j < L
  uint32_t need_route;           // micro-batches whose logits at l_j must be routed
  uint32_t runset;               // RunSet of the current step
  int32_t n_run;
  int32_t n_groups;
  int32_t n_steps;   // steps with a non-empty RunSet since reset
  int32_t status;    // first device-side error (EB_OK if none)
  int32_t nseg;      // segments of this step: n_groups * (E + n_shared)
  int32_t items1;    // work items of the gate/up GEMM
  int32_t items2;    // work items of the down GEMM
  int32_t rows;      // permuted rows of this step
  uint32_t gate_buf; // bit j: which of the two gate buffers holds j's current routing
  uint32_t sched_calls;  // scheduler launches since the context was created (eb_reset keeps it)
  long long num, den, den_sep;  // utilisation accumulators (Eq. (3))
};

// What a step's combine reads of the step state.  The step's scheduler
// writes it into one of two slots (by step parity), so the next step's
// scheduler may run while this step's combine still reads it.
struct StepView {
  int32_t n_run;
  uint32_t gate_buf;  // State::gate_buf of the step
  int32_t next;       // the combine's next unclaimed token (zeroed by the scheduler)
  int32_t pad;
  int32_t run_list[EB_MAX_M];
};

// Plain-old-data copy of the configuration used by kernels.
struct Dims {
  int L, E, k, H, F, D, M, T, n_shared, Etot, renorm, dtype, policy, m, residual, compute;
  int NC;     // routing chunks per micro-batch: ceil(T / kChunk)
  int kk;     // slots per token including shared experts: k + n_shared
  int max_steps;
};

// Pointers into the caller's workspace.
struct Work {
  int32_t* idx;        // [M][T][k]
  float* gate;         // [2][M][T][k]: two buffers, State::gate_buf picks one per micro-batch
  int32_t* chunk_hist; // [M][NC][E]: counts of each 64-token chunk
  int32_t* rank;       // [M][T][k]: place of (j, t, s) among its chunk's pairs of its expert
                       // (expert arithmetic on; else null)
  int32_t* cbase;      // [M][NC][E]: pairs of expert e in micro-batch j's chunks before c
  int32_t* prior;      // [M][Etot]: rows of (j's segment, expert) taken by earlier RunSet members
  int32_t* pos;        // [M][T][kk]: row of (j, t, slot)
  int32_t* rowslot;    // [Rcap]: slot (j * T + t) * kk + s of each permuted row
  int32_t* seg_rows;   // [M*Etot + 1]
  int32_t* seg_wid;    // [M*Etot]: layer * Etot + expert
  int32_t* seg_items1; // [M*Etot + 1]
  int32_t* seg_items2; // [M*Etot + 1]
  int32_t* gemm_next;  // [2]: next dynamically claimed item of GEMM 1 / GEMM 2 (zeroed by the plan)
  StepView* views;     // [2]: the combine's view of a step, by step parity
  float* scores;       // [M][T][E]: router scores of the step (router mode)
  void* A;             // [Rcap][H] permuted tokens
  void* act;           // [Rcap][F] SwiGLU activations
  void* y;             // [M*T*kk][H] expert outputs, at each row's (token, slot) position
  long long Rcap;
};

// Device state owned by a context.
struct CtxDev {
  State* st;
  int32_t* hist;        // [M][E]: counts of micro-batch j at layer l_j (accumulated by routing)
  int32_t* w;           // [M][D]: loads of micro-batch j at layer l_j (accumulated by routing)
  long long* trace;     // [max_steps][kTraceCols]
  int32_t* trace_layers;  // [max_steps][M]
  int32_t* emap;        // [E]: rank of each expert (a custom placement)
  int use_emap;         // 0: contiguous map, experts [d E/D, (d+1) E/D) on rank d
  int32_t* tickets;     // [M]: routing CTAs of micro-batch j done with their chunk (the last
                        // one writes the chunk offsets and resets it)
  int32_t* arrive;      // [M*T][H/256]: fused-combine arrival counts (engine TMC), else null
  size_t arrive_bytes;
  void* search_slots;   // [kSearchCtas] MaxUtil search results (MaxUtil with a large
                        // candidate count), else null
  // mapped pinned host words {S after the step, scheduler launches so far}
  // that each scheduler launch writes, so that the host learns of the
  // episode's end without a copy in the stream between the kernels; or null
  volatile uint32_t* host_flag;
};

// ---- programmatic dependent launch ----
// Every kernel of a step is launched with programmatic stream serialisation
// allowed, so it can be scheduled while the previous kernel of the stream
// drains.  Each one calls pdl_wait() before it reads anything (griddepcontrol
// .wait returns once the previous grid has completed and its writes are
// visible; without a programmatic dependency it returns at once) and then
// pdl_trigger(), which lets the next kernel be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

// Launch with programmatic dependent launch allowed (and, cluster > 1, with
// that cluster size along x).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, int cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// A launch error that something else left pending is not this library's:
// every entry point checks cudaPeekAtLastError() right before its first
// launch and, if an error is pending, returns EB_ERR_CUDA without launching
// and without clearing it.  The cudaGetLastError() after its own launches
// then reports only errors of those launches.
inline bool cuda_error_pending() { return cudaPeekAtLastError() != cudaSuccess; }

// Gates of token tok = j T + t of the current step.  Routing writes a
// micro-batch's gates into the buffer its gate_buf bit does not name, and
// the scheduler flips the bits of the micro-batches it routed, so the
// routing of step i + 1 can run while step i's combine still reads step i's
// gates.
__device__ __forceinline__ const float* gates_of(const float* gate, uint32_t gate_buf,
                                                 const Dims& d, long long tok) {
  const int j = (int)(tok / d.T);
  return gate + (size_t)((gate_buf >> j) & 1u) * ((size_t)d.M * d.T * d.k) + (size_t)tok * d.k;
}

// ---- launchers (all asynchronous on `s`) ----
// Micro-batch j's rows at layer l start at logits + j * mb_stride + l *
// layer_stride (elements): (L T E, T E) for the caller's [M, L, T, E] logits,
// (T E, 0) for router scores of the step kept as [M, T, E].
// early: the launch follows a kernel of the previous step that does not
// read what routing writes (the persistent GEMM 2); the routing runs before
// waiting for it, in smaller CTAs that fit beside it, and waits at its end.
cudaError_t launch_route_step(const Dims& d, const CtxDev& c, const Work& w, const float* logits,
                              long long mb_stride, long long layer_stride, bool early,
                              cudaStream_t s);
cudaError_t launch_route_rows(const float* logits, int n, int E, int k, int renorm, int32_t* idx,
                              float* gate, int32_t* hist, int32_t* status, cudaStream_t s);
// rn1 / rn2: token rows per work item of GEMM 1 / GEMM 2; fm1 / fm2:
// output features per item.  With c.search_slots set, the MaxUtil search
// grid runs first (two launches).
// slot: the StepView slot of this step (its parity).
cudaError_t launch_schedule_step(const Dims& d, const CtxDev& c, const Work& w, int rn1, int rn2,
                                 int fm1, int fm2, int slot, cudaStream_t s);
// slots: kSearchCtas * kSearchSlotBytes of device scratch for the MaxUtil
// search grid, or null to search in the scheduler's CTA.
cudaError_t launch_schedule_once(const int32_t* w, uint32_t pending, int M, int D, int m,
                                 int policy, uint32_t* runset, long long* stats, void* slots,
                                 cudaStream_t s);
// expert_rank: device [E] placement, or nullptr for the contiguous map;
// status (device, may be nullptr) gets EB_ERR_INVALID_ARG for a rank outside
// [0, D) (that expert's count is then dropped).
cudaError_t launch_loads(const int32_t* hist, int M, int E, int D, const int32_t* expert_rank,
                         int32_t* w, int32_t* status, cudaStream_t s);
cudaError_t launch_reset(const Dims& d, const CtxDev& c, cudaStream_t s);
// Records `status` in the step state's status word (stream-ordered).
cudaError_t launch_set_status(State* st, int status, cudaStream_t s);
// Rows of every (token, slot) of the RunSet (pos) and the (token, slot) of
// every row (rowslot).
cudaError_t launch_positions(const Dims& d, const CtxDev& c, const Work& w, cudaStream_t s);
// The permuted copy A of the RunSet's token rows (after launch_positions).
cudaError_t launch_permute_copy(const Dims& d, const CtxDev& c, const Work& w, const void* hidden,
                                cudaStream_t s);
// slot: the StepView slot of the step being combined.  early: launched
// after the next step's scheduler, which it does not depend on; it combines
// first and waits for the scheduler only at its end.
cudaError_t launch_combine(const Dims& d, const Work& w, void* hidden, int slot, bool early,
                           cudaStream_t s);
// GEMM `which` (1: gate/up + SwiGLU, 2: down) on the CUDA cores.
cudaError_t launch_gemm_simt(const Dims& d, const CtxDev& c, const Work& w, const void* w_gateup,
                             const void* w_down, cudaStream_t s, int which);

// MaxUtil enumerates complements of size <= |S| - m; this caps the candidate
// count a single step may need (sum_{c <= M-m} C(M, c)).
constexpr unsigned long long kMaxUtilCandidateCap = 1ull << 25;
unsigned long long maxutil_candidates(int n, int m);
// Above a candidate count that one CTA searches quickly, MaxUtil runs a
// search grid of kSearchCtas CTAs first; each leaves its best candidate in
// a slot of kSearchSlotBytes bytes, which the scheduler then reduces.
constexpr int kSearchCtas = 296;
constexpr size_t kSearchSlotBytes = 24;
bool maxutil_uses_grid(int n, int m);

}  // namespace eb
