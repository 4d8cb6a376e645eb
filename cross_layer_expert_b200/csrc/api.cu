// The C ABI of include/eb.h: argument checks, the context and its device
// state, the workspace layout and the step / episode drivers.
//
// [EB] = "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
// Inference"; Algorithm 1 in its §4.2 is the loop eb_episode runs.
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <thread>
#include <vector>

#include "eb_internal.cuh"
#include "gemm_tc.cuh"

using namespace eb;

struct eb_ctx {
  eb_config cfg;
  Dims d;
  CtxDev dev;
  void* dev_alloc = nullptr;
  int device = 0;
  int num_sms = 148;
  bool use_tc = false;
  int eng1 = EB_GEMM_SIMT, eng2 = EB_GEMM_SIMT;  // engine of GEMM 1 / GEMM 2
  // router mode: scores projected from the hidden states (eb_set_router)
  const void* w_router = nullptr;
  float* router_out = nullptr;  // optional caller buffer [M, L, T, E] for the scores
  CUtensorMap router_map_h, router_map_r;
  const void* router_keys[2] = {nullptr, nullptr};
  cudaStream_t last_stream = nullptr;
  // set once the host has seen EB_ERR_TIMEOUT in the status word; steps are
  // refused until eb_reset
  bool timed_out = false;
  // the previous step already enqueued this step's routing (eb_episode)
  bool routed_ahead = false;
  // the previous step's combine is enqueued by this step, beside its
  // scheduler (eb_episode); it writes deferred_hidden
  bool combine_deferred = false;
  void* deferred_hidden = nullptr;
  // steps enqueued since create; its parity picks the step's StepView slot
  long long seq = 0;
  // the GEMMs' state for eb_expert_ffn (the step state stays untouched)
  State* ffn_st = nullptr;
  uint32_t* host_pending = nullptr;  // pinned ring for eb_episode's completion checks
  cudaEvent_t events[8] = {};
  // mapped pinned words the scheduler writes, {S, scheduler launches}; the
  // host polls them instead (null: the copies and events above are used)
  volatile uint32_t* host_flag = nullptr;
  uint32_t sched_launched = 0;  // scheduler launches enqueued since create
  // cached TMA maps (rebuilt when a pointer changes)
  TcMaps maps;
  const void* map_keys[3] = {nullptr, nullptr, nullptr};
  // kernel launches enqueued since create, and optional per-kernel event timing
  long long launches = 0;
  bool prof = false;
  struct Mark {
    int kernel;
    cudaEvent_t a, b;
  };
  std::vector<Mark> marks;
  std::vector<cudaEvent_t> pool;
};

namespace {

constexpr size_t kAlign = 256;
constexpr int kLookahead = 4;  // steps enqueued ahead of the host's completion check

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool use_tc_for(const eb_config& c) {
  if (c.dtype != EB_DTYPE_BF16) return false;
  return c.gemm != EB_GEMM_SIMT;
}

// Engine of each GEMM.  AUTO takes the token-major engine for every GEMM
// whose tile shape fits (GEMM 1: F a multiple of 128; GEMM 2: H a multiple of
// 256) and the weight-major engine otherwise; an explicit choice that does not
// fit one GEMM runs that GEMM on the weight-major engine.
void choose_engines(const eb_config& c, bool use_tc, int* g1, int* g2) {
  *g1 = *g2 = EB_GEMM_SIMT;
  if (!use_tc) return;
  const int want = c.gemm == EB_GEMM_AUTO ? EB_GEMM_TM : c.gemm;
  auto fits = [&](int eng, int which) {
    const int nout = which == 1 ? c.F : c.H;
    switch (eng) {
      case EB_GEMM_TC: return true;
      case EB_GEMM_TM: return nout % (which == 1 ? kTmFeat1 : kTmFeat2) == 0;
      case EB_GEMM_TMG: return which == 1 && nout % kTmFeat1 == 0;
      case EB_GEMM_TMC: return which == 2 && nout % kTmFeat2 == 0;
      default: return false;
    }
  };
  // TMC fuses the combine into GEMM 2; its GEMM 1 is the token-major one
  const int want1 = want == EB_GEMM_TMC ? EB_GEMM_TM : want;
  *g1 = fits(want1, 1) ? want1 : EB_GEMM_TC;
  // TMG gathers GEMM 1's input; its GEMM 2 is the token-major one
  const int want2 = want == EB_GEMM_TMG ? EB_GEMM_TM : want;
  *g2 = fits(want2, 2) ? want2 : EB_GEMM_TC;
}

// Token rows and output features of one work item of `eng` for GEMM `which`.
void engine_tiles(int eng, int which, int* rows, int* feats) {
  switch (eng) {
    case EB_GEMM_TC:
      *rows = which == 1 ? kTcRows1 : kTcRows2;
      *feats = kTcFeat;
      return;
    case EB_GEMM_TM:
    case EB_GEMM_TMG:
    case EB_GEMM_TMC:
      *rows = kTmRows;
      *feats = which == 1 ? kTmFeat1 : kTmFeat2;
      return;
    default:
      *rows = kSimtRows;
      *feats = kSimtFeat;
  }
}

Dims make_dims(const eb_config& c) {
  Dims d;
  d.L = c.L; d.E = c.E; d.k = c.k; d.H = c.H; d.F = c.F; d.D = c.D; d.M = c.M; d.T = c.T;
  d.n_shared = c.n_shared; d.Etot = c.E + c.n_shared; d.renorm = c.renorm; d.dtype = c.dtype;
  d.policy = c.policy; d.m = c.m; d.residual = c.residual; d.compute = c.compute;
  d.NC = (c.T + kChunk - 1) / kChunk;
  d.kk = c.k + c.n_shared;
  d.max_steps = c.M * c.L;
  return d;
}

size_t elem_size(int dtype) { return dtype == EB_DTYPE_BF16 ? 2 : 4; }

// Offsets of the workspace buffers; returns the total size.
size_t layout(const eb_config& c, char* base, Work* w) {
  const Dims d = make_dims(c);
  const size_t M = c.M, T = c.T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return base ? (void*)(base + o) : nullptr;
  };
  Work x{};
  x.idx = (int32_t*)take(sizeof(int32_t) * M * T * c.k);
  x.gate = (float*)take(sizeof(float) * 2 * M * T * c.k);
  x.chunk_hist = (int32_t*)take(sizeof(int32_t) * M * d.NC * c.E);
  if (c.compute) {
    x.rank = (int32_t*)take(sizeof(int32_t) * M * T * c.k);
    x.cbase = (int32_t*)take(sizeof(int32_t) * M * d.NC * c.E);
  }
  x.views = (StepView*)take(sizeof(StepView) * 2);
  const size_t nseg = M * (size_t)d.Etot;
  if (c.compute) {
    x.prior = (int32_t*)take(sizeof(int32_t) * M * d.Etot);
    x.pos = (int32_t*)take(sizeof(int32_t) * M * T * d.kk);
    x.rowslot = (int32_t*)take(sizeof(int32_t) * M * T * d.kk);
    x.seg_rows = (int32_t*)take(sizeof(int32_t) * (nseg + 1));
    x.seg_wid = (int32_t*)take(sizeof(int32_t) * nseg);
    x.seg_items1 = (int32_t*)take(sizeof(int32_t) * (nseg + 1));
    x.seg_items2 = (int32_t*)take(sizeof(int32_t) * (nseg + 1));
    x.gemm_next = (int32_t*)take(sizeof(int32_t) * 2);
    x.scores = (float*)take(sizeof(float) * M * T * c.E);
    x.Rcap = (long long)(M * T * d.kk);
    const size_t es = elem_size(c.dtype);
    x.A = take(es * (size_t)x.Rcap * c.H);
    x.act = take(es * (size_t)x.Rcap * c.F);
    x.y = take(es * (size_t)x.Rcap * c.H);
  }
  if (w) *w = x;
  return off;
}

eb_status cuda_status(cudaError_t e) { return e == cudaSuccess ? EB_OK : EB_ERR_CUDA; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

cudaEvent_t take_event(eb_ctx* x) {
  if (!x->pool.empty()) {
    cudaEvent_t e = x->pool.back();
    x->pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Launches one stage, counting it and (when profiling) bracketing it with
// events on its stream.
template <typename F>
cudaError_t timed(eb_ctx* x, int kernel, int n_launch, cudaStream_t s, F&& launch) {
  if (!x->prof) {
    x->launches += n_launch;
    return launch();
  }
  eb_ctx::Mark mk{kernel, take_event(x), take_event(x)};
  cudaEventRecord(mk.a, s);
  const cudaError_t e = launch();
  cudaEventRecord(mk.b, s);
  x->marks.push_back(mk);
  x->launches += n_launch;
  return e;
}

// p[i] = i for i < n (the identity row map of eb_expert_ffn).
__global__ void k_iota(int32_t* p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = i;
}

cudaError_t launch_iota(int32_t* p, int n, cudaStream_t s) {
  k_iota<<<(n + 255) / 256, 256, 0, s>>>(p, n);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

const char* eb_status_string(eb_status s) {
  switch (s) {
    case EB_OK: return "ok";
    case EB_ERR_INVALID_ARG: return "invalid argument";
    case EB_ERR_UNSUPPORTED: return "unsupported shape or option";
    case EB_ERR_NONFINITE: return "non-finite router logit";
    case EB_ERR_CUDA: return "CUDA runtime error";
    case EB_ERR_TIMEOUT: return "bounded device wait expired";
    case EB_ERR_WORKSPACE: return "workspace too small";
    case EB_ERR_TOO_LARGE: return "exceeds the fixed scratch capacity of a no-allocation call";
    default: return "unknown status";
  }
}

eb_status eb_config_check(const eb_config* c) {
  if (!c) return EB_ERR_INVALID_ARG;
  if (c->L < 1 || c->E < 1 || c->k < 1 || c->D < 1 || c->M < 1 || c->T < 1 || c->m < 1)
    return EB_ERR_INVALID_ARG;
  if (c->k > c->E || c->m > c->M || c->n_shared < 0) return EB_ERR_INVALID_ARG;
  if (c->E % c->D != 0) return EB_ERR_INVALID_ARG;
  if (c->policy < EB_SCHED_CUMUTIL || c->policy > EB_SCHED_DIFFPEAK) return EB_ERR_INVALID_ARG;
  if (c->dtype != EB_DTYPE_F32 && c->dtype != EB_DTYPE_BF16) return EB_ERR_INVALID_ARG;
  if (c->gemm < EB_GEMM_AUTO || c->gemm > EB_GEMM_TMC || c->gemm == 3 || c->gemm == 5)
    return EB_ERR_INVALID_ARG;  // 3 and 5 were retired engines
  if (c->M > EB_MAX_M || c->D > EB_MAX_D || c->E + c->n_shared > EB_MAX_ETOT ||
      c->k + c->n_shared > EB_MAX_K)
    return EB_ERR_UNSUPPORTED;
  if ((long long)c->M * c->L * c->T * c->E > (1ll << 40)) return EB_ERR_UNSUPPORTED;
  // a RunSet's rank loads sum at most M T k token slots: int32 throughout
  if ((long long)c->M * c->T * c->k > (1ll << 31) - 1) return EB_ERR_UNSUPPORTED;
  if (c->policy == EB_SCHED_MAXUTIL && maxutil_candidates(c->M, c->m) > kMaxUtilCandidateCap)
    return EB_ERR_UNSUPPORTED;
  if (c->compute) {
    if (c->H < 1 || c->F < 1) return EB_ERR_INVALID_ARG;
    const int vec = c->dtype == EB_DTYPE_BF16 ? 8 : 4;  // 16-byte rows
    if (c->H % vec != 0) return EB_ERR_UNSUPPORTED;
    if ((long long)c->M * c->T * (c->k + c->n_shared) > (1ll << 31) - 1) return EB_ERR_UNSUPPORTED;
    const bool forced_tc = c->gemm != EB_GEMM_AUTO && c->gemm != EB_GEMM_SIMT;
    if (c->dtype == EB_DTYPE_F32 && forced_tc) return EB_ERR_UNSUPPORTED;
    if (use_tc_for(*c) && (c->H % 128 != 0 || c->F % 128 != 0)) {
      if (forced_tc) return EB_ERR_UNSUPPORTED;
    }
  }
  return EB_OK;
}

eb_status eb_workspace_size(const eb_config* c, size_t* bytes) {
  const eb_status s = eb_config_check(c);
  if (s != EB_OK) return s;
  if (!bytes) return EB_ERR_INVALID_ARG;
  *bytes = layout(*c, nullptr, nullptr);
  return EB_OK;
}

eb_status eb_create(const eb_config* c, eb_ctx** out) {
  const eb_status s = eb_config_check(c);
  if (s != EB_OK) return s;
  if (!out) return EB_ERR_INVALID_ARG;
  eb_ctx* x = new eb_ctx();
  x->cfg = *c;
  x->d = make_dims(*c);
  // the tensor-core engine needs 128-row feature tiles; otherwise SIMT
  x->use_tc = use_tc_for(*c) && c->H % 128 == 0 && c->F % 128 == 0;
  cudaError_t e = cudaGetDevice(&x->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&x->num_sms, cudaDevAttrMultiProcessorCount, x->device);
  if (e == cudaSuccess) choose_engines(*c, x->use_tc, &x->eng1, &x->eng2);
  const size_t n_state = align_up(sizeof(State));
  const size_t n_hist = align_up(sizeof(int32_t) * c->M * c->E);
  const size_t n_w = align_up(sizeof(int32_t) * c->M * c->D);
  const size_t n_trace = align_up(sizeof(long long) * kTraceCols * x->d.max_steps);
  const size_t n_tl = align_up(sizeof(int32_t) * c->M * (size_t)x->d.max_steps);
  const size_t n_map = align_up(sizeof(int32_t) * c->E);
  const size_t n_tickets = align_up(sizeof(int32_t) * c->M);
  // arrival counters of the fused combine, one per (token, 256-feature block)
  const size_t n_arrive =
      x->eng2 == EB_GEMM_TMC ? align_up(sizeof(int32_t) * (size_t)c->M * c->T * (c->H / kTmFeat2)) : 0;
  // MaxUtil search grid results, when one CTA would search too many subsets
  const bool grid_search = c->policy == EB_SCHED_MAXUTIL && maxutil_uses_grid(c->M, c->m);
  const size_t n_slots = grid_search ? align_up(kSearchCtas * kSearchSlotBytes) : 0;
  const size_t n_all =
      n_state + n_hist + n_w + n_trace + n_tl + n_map + n_arrive + n_slots + n_state + n_tickets;
  char* p = nullptr;
  if (e == cudaSuccess) e = cudaMalloc(&p, n_all);
  if (e == cudaSuccess) e = cudaMemset(p, 0, n_all);
  if (e == cudaSuccess) {
    x->dev_alloc = p;
    x->dev.st = (State*)p;
    x->dev.hist = (int32_t*)(p + n_state);
    x->dev.w = (int32_t*)(p + n_state + n_hist);
    x->dev.trace = (long long*)(p + n_state + n_hist + n_w);
    x->dev.trace_layers = (int32_t*)(p + n_state + n_hist + n_w + n_trace);
    x->dev.emap = (int32_t*)(p + n_state + n_hist + n_w + n_trace + n_tl);
    x->dev.use_emap = 0;
    x->dev.arrive = n_arrive ? (int32_t*)(p + n_state + n_hist + n_w + n_trace + n_tl + n_map) : nullptr;
    x->dev.arrive_bytes = n_arrive;
    x->dev.search_slots =
        n_slots ? (void*)(p + n_state + n_hist + n_w + n_trace + n_tl + n_map + n_arrive) : nullptr;
    x->ffn_st = (State*)(p + n_state + n_hist + n_w + n_trace + n_tl + n_map + n_arrive + n_slots);
    x->dev.tickets =
        (int32_t*)(p + n_state + n_hist + n_w + n_trace + n_tl + n_map + n_arrive + n_slots + n_state);
    e = cudaHostAlloc(&x->host_pending, sizeof(uint32_t) * kLookahead, cudaHostAllocDefault);
  }
  if (e == cudaSuccess) {
    void* hf = nullptr;
    void* hd = nullptr;
    if (cudaHostAlloc(&hf, 64, cudaHostAllocMapped) == cudaSuccess) {
      memset(hf, 0, 64);
      if (cudaHostGetDevicePointer(&hd, hf, 0) == cudaSuccess) {
        x->host_flag = static_cast<volatile uint32_t*>(hf);
        x->dev.host_flag = static_cast<volatile uint32_t*>(hd);
      } else {
        cudaFreeHost(hf);
      }
    }
    (void)cudaGetLastError();  // without mapped memory eb_episode copies instead
  }
  for (int i = 0; e == cudaSuccess && i < kLookahead; ++i)
    e = cudaEventCreateWithFlags(&x->events[i], cudaEventDisableTiming);
  if (e == cudaSuccess && x->use_tc) e = gemm_tc_prepare();
  if (e == cudaSuccess) e = launch_reset(x->d, x->dev, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    eb_destroy(x);
    return EB_ERR_CUDA;
  }
  *out = x;
  return EB_OK;
}

eb_status eb_destroy(eb_ctx* x) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (x->last_stream) cudaStreamSynchronize(x->last_stream);
  for (int i = 0; i < kLookahead; ++i)
    if (x->events[i]) cudaEventDestroy(x->events[i]);
  for (auto& mk : x->marks) {
    cudaEventDestroy(mk.a);
    cudaEventDestroy(mk.b);
  }
  for (auto e : x->pool) cudaEventDestroy(e);
  if (x->host_pending) cudaFreeHost(x->host_pending);
  if (x->host_flag) cudaFreeHost(const_cast<uint32_t*>(x->host_flag));
  if (x->dev_alloc) cudaFree(x->dev_alloc);
  delete x;
  return EB_OK;
}

eb_status eb_reset(eb_ctx* x, void* stream) {
  if (!x) return EB_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  x->last_stream = s;
  x->launches += 1;
  x->timed_out = false;
  x->routed_ahead = false;
  x->combine_deferred = false;
  cudaError_t e = launch_reset(x->d, x->dev, s);
  // the fused combine leaves its counters at zero; a step that gave up on a
  // bounded wait may not have, so a reset clears them
  if (e == cudaSuccess && x->dev.arrive)
    e = cudaMemsetAsync(x->dev.arrive, 0, x->dev.arrive_bytes, s);
  return cuda_status(e);
}

eb_status eb_set_expert_map(eb_ctx* x, const int32_t* expert_rank) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (!expert_rank) {
    x->dev.use_emap = 0;
    return EB_OK;
  }
  for (int e = 0; e < x->cfg.E; ++e)
    if (expert_rank[e] < 0 || expert_rank[e] >= x->cfg.D) return EB_ERR_INVALID_ARG;
  // synchronous: no step of this context may be in flight
  const cudaError_t err = cudaMemcpy(x->dev.emap, expert_rank, sizeof(int32_t) * x->cfg.E,
                                     cudaMemcpyHostToDevice);
  if (err != cudaSuccess) return EB_ERR_CUDA;
  x->dev.use_emap = 1;
  return EB_OK;
}

eb_status eb_set_router(eb_ctx* x, const void* w_router, float* scores) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (w_router) {
    const eb_config& c = x->cfg;
    if (!c.compute || c.dtype != EB_DTYPE_BF16 || c.E % 16 != 0 || c.E > 256 || c.H % 64 != 0)
      return EB_ERR_UNSUPPORTED;
    if (((uintptr_t)w_router & 15u) != 0) return EB_ERR_INVALID_ARG;
    if (gemm_tc_prepare() != cudaSuccess) return EB_ERR_CUDA;
  }
  if (scores && ((uintptr_t)scores & 15u) != 0) return EB_ERR_INVALID_ARG;
  x->w_router = w_router;
  x->router_out = w_router ? scores : nullptr;
  x->router_keys[1] = nullptr;
  return EB_OK;
}

static cudaError_t launch_engine(eb_ctx* x, int eng, const Work& w, const void* wgu,
                                 const void* wdn, const void* hidden, cudaStream_t s, int which) {
  switch (eng) {
    case EB_GEMM_TC: return launch_gemm_tc(x->d, x->dev, w, x->maps, x->num_sms, s, which);
    case EB_GEMM_TM:
      return launch_gemm_tm(x->d, x->dev, w, x->maps, x->num_sms, s, which, nullptr, nullptr);
    case EB_GEMM_TMG:
      return launch_gemm_tm(x->d, x->dev, w, x->maps, x->num_sms, s, which,
                            which == 1 ? hidden : nullptr, nullptr);
    case EB_GEMM_TMC:  // GEMM 2 only (GEMM 1 of TMC is TM)
      return launch_gemm_tm(x->d, x->dev, w, x->maps, x->num_sms, s, which, nullptr,
                            const_cast<void*>(hidden));
    default: return launch_gemm_simt(x->d, x->dev, w, wgu, wdn, s, which);
  }
}

// route_next: the caller enqueues the next step with the same logits
// (eb_episode), so this step may route it ahead: after GEMM 2, whose
// persistent CTAs it runs beside, and before the combine.
static eb_status enqueue_step(eb_ctx* x, const float* logits, void* hidden, const void* wgu,
                              const void* wdn, void* workspace, size_t ws_bytes,
                              cudaStream_t s, bool route_next) {
  const eb_config& c = x->cfg;
  if (x->timed_out) return EB_ERR_TIMEOUT;
  if ((!logits && !x->w_router) || !workspace) return EB_ERR_INVALID_ARG;
  if (x->w_router && !hidden) return EB_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & (kAlign - 1)) != 0) return EB_ERR_INVALID_ARG;
  if (c.compute && (!hidden || !wgu || !wdn)) return EB_ERR_INVALID_ARG;
  if (c.compute && (!aligned16(hidden) || !aligned16(wgu) || !aligned16(wdn)))
    return EB_ERR_INVALID_ARG;
  Work w;
  const size_t need = layout(c, (char*)workspace, &w);
  if (ws_bytes < need) return EB_ERR_WORKSPACE;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  x->last_stream = s;
  const bool tc = c.compute && x->use_tc;
  if (tc && (x->map_keys[0] != wgu || x->map_keys[1] != wdn || x->map_keys[2] != workspace)) {
    if (make_tc_maps(x->d, w, wgu, wdn, &x->maps) != cudaSuccess) return EB_ERR_UNSUPPORTED;
    x->map_keys[0] = wgu;
    x->map_keys[1] = wdn;
    x->map_keys[2] = workspace;
  }
  // GEMM 1 on the gathering engine reads its token rows from `hidden` itself
  // (no permuted copy)
  const bool gather = c.compute && x->eng1 == EB_GEMM_TMG;

  const int g1 = c.compute ? x->eng1 : EB_GEMM_SIMT, g2 = c.compute ? x->eng2 : EB_GEMM_SIMT;
  int rn1, fm1, rn2, fm2;
  engine_tiles(g1, 1, &rn1, &fm1);
  engine_tiles(g2, 2, &rn2, &fm2);
  cudaError_t e = cudaSuccess;
  if (x->w_router) {  // project this step's router scores from the hidden states
    if (x->router_keys[0] != hidden || x->router_keys[1] != x->w_router) {
      if (make_router_maps(hidden, (long long)c.M * c.T, c.H, x->w_router, c.L, c.E,
                           &x->router_map_h, &x->router_map_r) != cudaSuccess)
        return EB_ERR_UNSUPPORTED;
      x->router_keys[0] = hidden;
      x->router_keys[1] = x->w_router;
    }
  }
  // where routing reads each micro-batch's rows: the caller's logits, the
  // caller's score buffer (router mode) or the workspace (router mode)
  const long long TE = (long long)c.T * c.E;
  const float* rsrc = logits;
  long long mbs = (long long)c.L * TE, ls = TE;
  if (x->w_router) {
    float* dst = x->router_out ? x->router_out : w.scores;
    if (!x->router_out) {
      mbs = TE;
      ls = 0;
    }
    rsrc = dst;
    e = timed(x, 7, 1, s, [&] {
      return launch_router(x->router_map_h, x->router_map_r, c.T, c.H, c.E, c.M, x->dev.st, dst,
                           mbs, ls, &x->dev.st->status, s);
    });
  }
  if (e == cudaSuccess && !x->routed_ahead)
    e = timed(x, 0, 1, s,
              [&] { return launch_route_step(x->d, x->dev, w, rsrc, mbs, ls, false, s); });
  x->routed_ahead = false;
  const int slot = (int)(x->seq & 1);
  x->seq += 1;
  if (e == cudaSuccess) {
    e = timed(x, 1, x->dev.search_slots ? 2 : 1, s,
              [&] { return launch_schedule_step(x->d, x->dev, w, rn1, rn2, fm1, fm2, slot, s); });
    if (e == cudaSuccess) x->sched_launched += 1u;
  }
  // the previous step's combine runs beside this step's scheduler: it reads
  // the previous step's view, outputs and gates, none of which the scheduler
  // writes, and the row copy (or the positions pass) after it waits for both
  if (e == cudaSuccess && x->combine_deferred) {
    x->combine_deferred = false;
    e = timed(x, 5, 1, s, [&] {
      return launch_combine(x->d, w, x->deferred_hidden, slot ^ 1, true, s);
    });
  }
  if (c.compute) {
    // the gathering engine reads the rows' positions in GEMM 1; otherwise
    // the row copy places the rows itself, from the ranks routing wrote
    if (e == cudaSuccess && gather)
      e = timed(x, 6, 1, s, [&] { return launch_positions(x->d, x->dev, w, s); });
    if (e == cudaSuccess && !gather)
      e = timed(x, 2, 1, s, [&] { return launch_permute_copy(x->d, x->dev, w, hidden, s); });
    if (e == cudaSuccess) {
      e = timed(x, 3, 1, s, [&] { return launch_engine(x, g1, w, wgu, wdn, hidden, s, 1); });
      if (e == cudaSuccess)
        e = timed(x, 4, 1, s, [&] { return launch_engine(x, g2, w, wgu, wdn, hidden, s, 2); });
    }
    // the next step's routing reads the caller's logits and this step's
    // state only, so it runs beside GEMM 2 (router mode projects the scores
    // from the hidden states this step's combine writes, so it does not)
    if (e == cudaSuccess && route_next && !x->w_router && g2 != EB_GEMM_SIMT) {
      e = timed(x, 0, 1, s,
                [&] { return launch_route_step(x->d, x->dev, w, rsrc, mbs, ls, true, s); });
      x->routed_ahead = e == cudaSuccess;
    }
    // the fused engine combines inside GEMM 2; after routing ahead the
    // combine waits for the next step, to run beside its scheduler
    if (e == cudaSuccess && g2 != EB_GEMM_TMC) {
      if (x->routed_ahead) {
        x->combine_deferred = true;
        x->deferred_hidden = hidden;
      } else {
        e = timed(x, 5, 1, s, [&] { return launch_combine(x->d, w, hidden, slot, false, s); });
      }
    }
  }
  return cuda_status(e);
}

// The combine a step deferred to the next one, when no next step follows.
static eb_status flush_combine(eb_ctx* x, void* workspace, cudaStream_t s) {
  if (!x->combine_deferred) return EB_OK;
  x->combine_deferred = false;
  Work w;
  layout(x->cfg, (char*)workspace, &w);
  const int slot = (int)((x->seq - 1) & 1);
  return cuda_status(timed(x, 5, 1, s, [&] {
    return launch_combine(x->d, w, x->deferred_hidden, slot, false, s);
  }));
}

eb_status eb_moe_step(eb_ctx* x, const float* logits, void* hidden, const void* wgu,
                      const void* wdn, void* workspace, size_t ws_bytes, void* stream,
                      uint32_t* runset_host) {
  if (!x) return EB_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const eb_status st = enqueue_step(x, logits, hidden, wgu, wdn, workspace, ws_bytes, s, false);
  if (st != EB_OK) return st;
  if (runset_host) {
    cudaError_t e = cudaMemcpyAsync(runset_host, &x->dev.st->runset, sizeof(uint32_t),
                                    cudaMemcpyDeviceToHost, s);
    int status = EB_OK;
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(&status, &x->dev.st->status, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return EB_ERR_CUDA;
    if (status == EB_ERR_TIMEOUT) {
      x->timed_out = true;
      return EB_ERR_TIMEOUT;
    }
  }
  return EB_OK;
}

// Waits until the scheduler launch numbered `target` (counting from the
// context's creation) has written the host's mapped words, and returns S as
// of that step or later (S only shrinks, and an empty S is all the caller
// tests).  If the stream runs dry first (a launch that never ran, e.g. after
// an error), S is read from the device state instead.
static eb_status wait_scheduler(eb_ctx* x, cudaStream_t s, uint32_t target, uint32_t* pending) {
  for (unsigned it = 1;; ++it) {
    if ((int32_t)(x->host_flag[1] - target) >= 0) {
      std::atomic_thread_fence(std::memory_order_acquire);
      *pending = x->host_flag[0];
      return EB_OK;
    }
    if ((it & 15u) == 0u) {
      const cudaError_t q = cudaStreamQuery(s);
      if (q == cudaSuccess) {
        if ((int32_t)(x->host_flag[1] - target) >= 0) continue;
        uint32_t p = 0;
        if (cudaMemcpy(&p, &x->dev.st->pending, sizeof(p), cudaMemcpyDeviceToHost) != cudaSuccess)
          return EB_ERR_CUDA;
        *pending = p;
        return EB_OK;
      }
      if (q != cudaErrorNotReady) return EB_ERR_CUDA;
    }
    std::this_thread::yield();
  }
}

eb_status eb_episode(eb_ctx* x, const float* logits, void* hidden, const void* wgu,
                     const void* wdn, void* workspace, size_t ws_bytes, void* stream,
                     int* n_steps) {
  if (!x) return EB_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  eb_status st = eb_reset(x, stream);
  if (st != EB_OK) return st;
  const int max_steps = x->d.max_steps;
  const uint32_t base = x->sched_launched;
  for (int i = 0; i < max_steps; ++i) {
    st = enqueue_step(x, logits, hidden, wgu, wdn, workspace, ws_bytes, s, true);
    if (st != EB_OK) return st;
    if (x->host_flag) {
      // the scheduler of the step enqueued kLookahead - 1 steps ago has told
      // the host S; nothing but kernels sits in the stream
      const int chk = i - (kLookahead - 1);
      if (chk >= 0) {
        uint32_t pending = 0;
        st = wait_scheduler(x, s, base + (uint32_t)chk + 1u, &pending);
        if (st != EB_OK) return st;
        if (pending == 0) break;
      }
      continue;
    }
    const int slot = i % kLookahead;
    cudaError_t e = cudaMemcpyAsync(&x->host_pending[slot], &x->dev.st->pending, sizeof(uint32_t),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaEventRecord(x->events[slot], s);
    if (e != cudaSuccess) return EB_ERR_CUDA;
    // check the step enqueued kLookahead - 1 steps ago; the GPU keeps working
    const int chk = i - (kLookahead - 1);
    if (chk >= 0) {
      const int cs = chk % kLookahead;
      if (cudaEventSynchronize(x->events[cs]) != cudaSuccess) return EB_ERR_CUDA;
      if (x->host_pending[cs] == 0) break;
    }
  }
  st = flush_combine(x, workspace, s);
  if (st != EB_OK) return st;
  if (cudaStreamSynchronize(s) != cudaSuccess) return EB_ERR_CUDA;
  int steps = 0, status = EB_OK;
  if (cudaMemcpy(&steps, &x->dev.st->n_steps, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(&status, &x->dev.st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EB_ERR_CUDA;
  if (n_steps) *n_steps = steps;
  if (status == EB_ERR_TIMEOUT) {
    x->timed_out = true;
    return EB_ERR_TIMEOUT;
  }
  return EB_OK;
}

eb_status eb_utilization(eb_ctx* x, int64_t* num, int64_t* den, int64_t* den_sep) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (x->last_stream && cudaStreamSynchronize(x->last_stream) != cudaSuccess) return EB_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return EB_ERR_CUDA;
  State h;
  if (cudaMemcpy(&h, x->dev.st, sizeof(State), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EB_ERR_CUDA;
  if (num) *num = h.num;
  if (den) *den = h.den;
  if (den_sep) *den_sep = h.den_sep;
  return EB_OK;
}

eb_status eb_trace(eb_ctx* x, int64_t* rows, int32_t* layers, int max_steps, int* n_steps) {
  if (!x || max_steps < 0 || (max_steps > 0 && !rows)) return EB_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return EB_ERR_CUDA;
  State h;
  if (cudaMemcpy(&h, x->dev.st, sizeof(State), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EB_ERR_CUDA;
  const int n = h.n_steps < x->d.max_steps ? h.n_steps : x->d.max_steps;
  const int cp = n < max_steps ? n : max_steps;
  if (cp > 0) {
    if (cudaMemcpy(rows, x->dev.trace, sizeof(long long) * kTraceCols * cp, cudaMemcpyDeviceToHost) !=
        cudaSuccess)
      return EB_ERR_CUDA;
    if (layers && cudaMemcpy(layers, x->dev.trace_layers, sizeof(int32_t) * x->d.M * cp,
                             cudaMemcpyDeviceToHost) != cudaSuccess)
      return EB_ERR_CUDA;
  }
  if (n_steps) *n_steps = h.n_steps;
  return EB_OK;
}

eb_status eb_profile(eb_ctx* x, int enable) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (x->last_stream && cudaStreamSynchronize(x->last_stream) != cudaSuccess) return EB_ERR_CUDA;
  for (auto& mk : x->marks) {
    x->pool.push_back(mk.a);
    x->pool.push_back(mk.b);
  }
  x->marks.clear();
  x->prof = enable != 0;
  return EB_OK;
}

eb_status eb_profile_read(eb_ctx* x, double* ms, int64_t* launches) {
  if (!x || !ms || !launches) return EB_ERR_INVALID_ARG;
  for (int i = 0; i < EB_PROF_KERNELS; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  for (auto& mk : x->marks) {
    if (cudaEventSynchronize(mk.b) != cudaSuccess) return EB_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, mk.a, mk.b) != cudaSuccess) return EB_ERR_CUDA;
    ms[mk.kernel] += t;
    launches[mk.kernel] += 1;
    x->pool.push_back(mk.a);
    x->pool.push_back(mk.b);
  }
  x->marks.clear();
  return EB_OK;
}

eb_status eb_launch_count(eb_ctx* x, int64_t* n) {
  if (!x || !n) return EB_ERR_INVALID_ARG;
  *n = x->launches;
  return EB_OK;
}

eb_status eb_engines(const eb_ctx* x, int* gemm1, int* gemm2) {
  if (!x || !gemm1 || !gemm2) return EB_ERR_INVALID_ARG;
  *gemm1 = x->eng1;
  *gemm2 = x->eng2;
  return EB_OK;
}

eb_status eb_sync_status(eb_ctx* x) {
  if (!x) return EB_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return EB_ERR_CUDA;
  int status = 0;
  if (cudaMemcpy(&status, &x->dev.st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EB_ERR_CUDA;
  if (status == EB_ERR_TIMEOUT) x->timed_out = true;
  return status;
}

eb_status eb_inject_status(eb_ctx* x, eb_status status, void* stream) {
  if (!x || status > 0 || status < EB_ERR_TOO_LARGE) return EB_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  x->last_stream = s;
  cudaError_t e = launch_set_status(x->dev.st, status, s);
  // the partial arrival counts a fused GEMM 2 that gave up part-way leaves
  if (e == cudaSuccess && status == EB_ERR_TIMEOUT && x->dev.arrive)
    e = cudaMemsetAsync(x->dev.arrive, 1, x->dev.arrive_bytes, s);
  return cuda_status(e);
}

eb_status eb_selftest_timeout(int64_t limit_ns, int32_t* status_dev, void* stream) {
  if (!status_dev || limit_ns < 1000 || limit_ns > 2000000000ll) return EB_ERR_INVALID_ARG;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  return cuda_status(launch_selftest_wait((unsigned long long)limit_ns, status_dev,
                                          (cudaStream_t)stream));
}

eb_status eb_route(const float* logits, int n, int E, int k, int renorm, int32_t* idx, float* gate,
                   int32_t* hist, int32_t* status_dev, void* stream) {
  if (n < 0 || E < 1 || k < 1 || k > E) return EB_ERR_INVALID_ARG;
  if (E > EB_MAX_ETOT || k > EB_MAX_K) return EB_ERR_UNSUPPORTED;
  if (!hist || (n > 0 && (!logits || !idx || !gate))) return EB_ERR_INVALID_ARG;
  return cuda_status(launch_route_rows(logits, n, E, k, renorm, idx, gate, hist, status_dev,
                                       (cudaStream_t)stream));
}

eb_status eb_loads(const int32_t* hist, int M, int E, int D, int32_t* w, void* stream) {
  if (M < 0 || E < 1 || D < 1 || E % D != 0) return EB_ERR_INVALID_ARG;
  if (M > 0 && (!hist || !w)) return EB_ERR_INVALID_ARG;
  if (M == 0) return EB_OK;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  return cuda_status(launch_loads(hist, M, E, D, nullptr, w, nullptr, (cudaStream_t)stream));
}

eb_status eb_router(const void* hidden, int n, int H, const void* w_router, int E, float* scores,
                    int32_t* status_dev, void* stream) {
  if (n < 0 || H < 1 || E < 1 || (n > 0 && (!hidden || !w_router || !scores)))
    return EB_ERR_INVALID_ARG;
  if (E % 16 != 0 || E > 256 || H % 64 != 0) return EB_ERR_UNSUPPORTED;
  if (((uintptr_t)hidden & 15u) != 0 || ((uintptr_t)w_router & 15u) != 0 ||
      ((uintptr_t)scores & 15u) != 0)
    return EB_ERR_INVALID_ARG;
  if (n == 0) return EB_OK;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  if (gemm_tc_prepare() != cudaSuccess) return EB_ERR_CUDA;
  CUtensorMap mh, mr;
  if (make_router_maps(hidden, n, H, w_router, 1, E, &mh, &mr) != cudaSuccess)
    return EB_ERR_UNSUPPORTED;
  return cuda_status(launch_router(mh, mr, n, H, E, 1, nullptr, scores, 0, 0, status_dev,
                                   (cudaStream_t)stream));
}

eb_status eb_loads_mapped(const int32_t* hist, int M, int E, int D, const int32_t* expert_rank,
                          int32_t* w, int32_t* status_dev, void* stream) {
  if (M < 0 || E < 1 || D < 1 || !expert_rank) return EB_ERR_INVALID_ARG;
  if (M > 0 && (!hist || !w)) return EB_ERR_INVALID_ARG;
  if (M == 0) return EB_OK;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  return cuda_status(
      launch_loads(hist, M, E, D, expert_rank, w, status_dev, (cudaStream_t)stream));
}

eb_status eb_expert_ffn(eb_ctx* x, const void* rows, int R, const int32_t* seg_off,
                        const int32_t* seg_layer, const int32_t* seg_expert, int nseg, void* out,
                        const void* wgu, const void* wdn, void* workspace, size_t ws_bytes,
                        void* stream) {
  if (!x) return EB_ERR_INVALID_ARG;
  const eb_config& c = x->cfg;
  if (!c.compute) return EB_ERR_UNSUPPORTED;
  if (R < 0 || nseg < 0 || !wgu || !wdn || !workspace) return EB_ERR_INVALID_ARG;
  if (R > 0 && (!rows || !out)) return EB_ERR_INVALID_ARG;
  if (nseg > 0 && (!seg_off || !seg_layer || !seg_expert)) return EB_ERR_INVALID_ARG;
  if (((uintptr_t)workspace & (kAlign - 1)) != 0) return EB_ERR_INVALID_ARG;
  if (!aligned16(wgu) || !aligned16(wdn) || (R > 0 && (!aligned16(rows) || !aligned16(out))))
    return EB_ERR_INVALID_ARG;
  Work w;
  const size_t need = layout(c, (char*)workspace, &w);
  if (ws_bytes < need) return EB_ERR_WORKSPACE;
  const int Et = c.E + c.n_shared;
  if ((long long)R > w.Rcap || nseg > c.M * Et) return EB_ERR_UNSUPPORTED;
  // the segment table: offsets ascending from 0 to R, (layer, expert) in range
  if (nseg == 0 ? R != 0 : (seg_off[0] != 0 || seg_off[nseg] != R)) return EB_ERR_INVALID_ARG;
  for (int i = 0; i < nseg; ++i)
    if (seg_off[i + 1] < seg_off[i] || seg_layer[i] < 0 || seg_layer[i] >= c.L ||
        seg_expert[i] < 0 || seg_expert[i] >= Et)
      return EB_ERR_INVALID_ARG;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  if (R == 0) return EB_OK;
  cudaStream_t s = (cudaStream_t)stream;
  x->last_stream = s;
  // the engines of the step, without the gather (GEMM 1 reads the rows as
  // given) and without the fused combine (there is no combine here)
  const int g1 = !x->use_tc ? EB_GEMM_SIMT : x->eng1 == EB_GEMM_TMG ? EB_GEMM_TM : x->eng1;
  const int g2 = !x->use_tc ? EB_GEMM_SIMT : x->eng2 == EB_GEMM_TMC ? EB_GEMM_TM : x->eng2;
  int rn1, fm1, rn2, fm2;
  engine_tiles(g1, 1, &rn1, &fm1);
  engine_tiles(g2, 2, &rn2, &fm2);
  // the plan, built here: rows, (layer, expert) and work items per segment
  std::vector<int32_t> plan(4 * (size_t)(nseg + 1), 0);
  int32_t* p_rows = plan.data();
  int32_t* p_wid = p_rows + (nseg + 1);
  int32_t* p_it1 = p_wid + (nseg + 1);
  int32_t* p_it2 = p_it1 + (nseg + 1);
  const int mb1 = c.F / fm1, mb2 = c.H / fm2;
  for (int i = 0; i <= nseg; ++i) {
    p_rows[i] = seg_off[i];
    if (i == nseg) break;
    const int n = seg_off[i + 1] - seg_off[i];
    p_wid[i] = seg_layer[i] * Et + seg_expert[i];
    p_it1[i + 1] = p_it1[i] + (n + rn1 - 1) / rn1 * mb1;
    p_it2[i + 1] = p_it2[i] + (n + rn2 - 1) / rn2 * mb2;
  }
  State fs{};
  fs.nseg = nseg;
  fs.runset = 1u;
  fs.rows = R;
  fs.items1 = p_it1[nseg];
  fs.items2 = p_it2[nseg];
  // the GEMMs read the rows as given and write each output row in place:
  // row r's (token, slot) is r
  Work wf = w;
  wf.A = const_cast<void*>(rows);
  wf.y = out;
  wf.Rcap = R;
  CtxDev cf = x->dev;
  cf.st = x->ffn_st;
  cf.arrive = nullptr;
  cudaError_t e = cudaMemcpyAsync(w.seg_rows, p_rows, sizeof(int32_t) * (nseg + 1),
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(w.seg_wid, p_wid, sizeof(int32_t) * nseg, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(w.seg_items1, p_it1, sizeof(int32_t) * (nseg + 1), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(w.seg_items2, p_it2, sizeof(int32_t) * (nseg + 1), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(x->ffn_st, &fs, sizeof(State), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.gemm_next, 0, sizeof(int32_t) * 2, s);
  if (e == cudaSuccess) e = launch_iota(w.rowslot, R, s);
  // (the host buffers above are pageable: each copy has read its source
  // before it returns)
  TcMaps maps;
  if (e == cudaSuccess && x->use_tc && make_tc_maps(x->d, wf, wgu, wdn, &maps) != cudaSuccess)
    return EB_ERR_UNSUPPORTED;
  auto run = [&](int eng, int which) -> cudaError_t {
    switch (eng) {
      case EB_GEMM_TC: return launch_gemm_tc(x->d, cf, wf, maps, x->num_sms, s, which);
      case EB_GEMM_TM:
        return launch_gemm_tm(x->d, cf, wf, maps, x->num_sms, s, which, nullptr, nullptr);
      default: return launch_gemm_simt(x->d, cf, wf, wgu, wdn, s, which);
    }
  };
  if (e == cudaSuccess) e = timed(x, 3, 1, s, [&] { return run(g1, 1); });
  if (e == cudaSuccess) e = timed(x, 4, 1, s, [&] { return run(g2, 2); });
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return EB_ERR_CUDA;
  int status = EB_OK;
  if (cudaMemcpy(&status, &x->ffn_st->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EB_ERR_CUDA;
  return status == EB_OK ? EB_OK : (eb_status)status;
}

eb_status eb_schedule(const int32_t* w, uint32_t pending_mask, int M, int D, int m, int policy,
                      uint32_t* runset_mask, int64_t* step_stats, void* stream) {
  if (M < 1 || D < 1 || m < 1 || m > M || !w || !runset_mask) return EB_ERR_INVALID_ARG;
  if (policy < EB_SCHED_CUMUTIL || policy > EB_SCHED_DIFFPEAK) return EB_ERR_INVALID_ARG;
  if (M > EB_MAX_M || D > EB_MAX_D) return EB_ERR_UNSUPPORTED;
  if (M < 32 && (pending_mask >> M) != 0) return EB_ERR_INVALID_ARG;
  if (policy == EB_SCHED_MAXUTIL && maxutil_candidates(__builtin_popcount(pending_mask), m) >
                                        kMaxUtilCandidateCap)
    return EB_ERR_UNSUPPORTED;
  if (cuda_error_pending()) return EB_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // a large MaxUtil search runs on a grid whose per-CTA results need a few KB
  // of scratch: stream-ordered, freed on the same stream
  void* slots = nullptr;
  if (policy == EB_SCHED_MAXUTIL && maxutil_uses_grid(__builtin_popcount(pending_mask), m) &&
      cudaMallocAsync(&slots, kSearchCtas * kSearchSlotBytes, s) != cudaSuccess)
    return EB_ERR_CUDA;
  cudaError_t e = launch_schedule_once(w, pending_mask, M, D, m, policy, runset_mask,
                                       (long long*)step_stats, slots, s);
  if (slots) {
    const cudaError_t f = cudaFreeAsync(slots, s);
    if (e == cudaSuccess) e = f;
  }
  return cuda_status(e);
}

}  // extern "C"
