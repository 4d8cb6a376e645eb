/*
 * eb.h -- C ABI of the B200 cross-layer MoE step (EasyBalance).
 *
 * The library runs one EasyBalance step on one GPU for M micro-batches that
 * each sit at their own MoE layer, with D expert-parallel ranks simulated on
 * the device.  Cited sources:
 *   [EB]      "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
 *             Inference" (Wu, Gao, Li, Wu).
 *   [EB-read] deep-read page "EasyBalance：分布式 MoE 推理的跨层负载均衡".
 *   [SysLB]   page "系统侧负载均衡：EPLB、LPLB、UltraEP 与 MoonEP".
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers unless a parameter says "host".
 *     They are owned by the caller; the library never frees them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it unless stated.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned as a negative eb_status; nothing runs in that case.
 *   - Errors the device detects (a non-finite router logit, an expired
 *     bounded wait) are recorded in the context's status word and returned by
 *     eb_sync_status().  After EB_ERR_TIMEOUT the context's state may be
 *     partial, so it runs no further step until eb_reset (see eb_moe_step).
 *   - A CUDA error that something else left pending (cudaPeekAtLastError)
 *     makes a call return EB_ERR_CUDA before it launches anything; the error
 *     stays pending for its owner.
 *   - There is no CPU fallback: a shape the kernels do not support returns
 *     EB_ERR_UNSUPPORTED.
 *   - A context is not thread-safe; its calls must be ordered on one stream.
 *   - All integer outputs (indices, histograms, loads, RunSets, utilisation
 *     numerators and denominators) are exact.
 */
#ifndef EB_H
#define EB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int eb_status;
#define EB_OK 0
#define EB_ERR_INVALID_ARG (-1) /* null pointer, size out of range, m > M ... */
#define EB_ERR_UNSUPPORTED (-2) /* valid but outside the kernels' limits     */
#define EB_ERR_NONFINITE (-3)   /* a NaN or Inf router logit was seen        */
#define EB_ERR_CUDA (-4)        /* a CUDA runtime call failed                */
#define EB_ERR_TIMEOUT (-5)     /* a bounded device-side wait expired        */
#define EB_ERR_WORKSPACE (-6)   /* workspace smaller than eb_workspace_size  */
#define EB_ERR_TOO_LARGE (-7)   /* beyond the fixed capacity of a no-allocation call */

/* RunSet policies, [EB] §4.2 and §5.2. */
#define EB_SCHED_CUMUTIL 0  /* O(n) scan: add j iff U(S+{j}) > U(S)          */
#define EB_SCHED_MAXUTIL 1  /* argmax U(S) over all S with |S| >= m          */
#define EB_SCHED_LOCKSTEP 2 /* every pending micro-batch: layer-by-layer     */
#define EB_SCHED_DIFFPEAK 3 /* add j iff its peak device is not yet taken    */

/* storage type of hidden states, expert weights and intermediates */
#define EB_DTYPE_F32 0
#define EB_DTYPE_BF16 1

/* expert GEMM engine (all tensor-core engines use tcgen05 with TMA-fed
 * operands and TMEM accumulators, and need bf16 with H and F multiples of 128).
 *   AUTO  bf16: TM for each GEMM it fits, else TC; f32: SIMT.
 *   TC    one SM per tile; weight rows are the MMA's M side (128 features),
 *         tokens its N side.
 *   SIMT  CUDA cores (any shape, f32 or bf16).
 *   TM    token-major, one SM: 128 tokens x 256 weight rows per MMA (gate/up:
 *         128 features of each; down: 256 features); work items are claimed
 *         dynamically, so CTAs finish together whatever the segment sizes.
 *   TMG   as TM, but GEMM 1 reads its token rows straight from `hidden`
 *         (extra warps copy each row into the operand tile with 16-byte
 *         cp.async) instead of from a permuted copy, which is then not
 *         written.
 *   TMC   as TM, with the combine fused into GEMM 2: each token is combined
 *         into `hidden` by the GEMM 2 drain that stores its last expert
 *         output row, and the step launches no combine kernel.  Bit-identical
 *         to TM.  The context then holds M*T*H/256 int32 arrival counters.
 * TM and TMC need F a multiple of 128 (gate/up) and H a multiple of 256
 * (down); a GEMM they do not fit runs on TC (and TMC's step then runs the
 * combine kernel).  Values 3 and 5 (two-SM engines, measured slower than TM)
 * are retired and rejected as EB_ERR_INVALID_ARG. */
#define EB_GEMM_AUTO 0
#define EB_GEMM_TC 1
#define EB_GEMM_SIMT 2
#define EB_GEMM_TM 4
#define EB_GEMM_TMG 6
#define EB_GEMM_TMC 7

/* Compile-time limits of the library. */
#define EB_MAX_M 32   /* micro-batches (RunSets are 32-bit masks)        */
#define EB_MAX_D 64   /* virtual ranks                                   */
#define EB_MAX_ETOT 256 /* routed + shared experts per layer            */
#define EB_MAX_K 32   /* experts per token                               */

typedef struct eb_config {
  int L;        /* MoE layers (l_max)                                    */
  int E;        /* routed experts per layer                              */
  int k;        /* experts per token, 1 <= k <= min(E, EB_MAX_K)         */
  int H;        /* hidden size                                           */
  int F;        /* expert FFN width (SwiGLU inner size)                  */
  int D;        /* virtual EP ranks; E % D == 0; rank d holds experts
                   [d E/D, (d+1) E/D)  ([EB] §5 Models: even mapping)     */
  int M;        /* micro-batches, 1..EB_MAX_M                            */
  int T;        /* tokens per micro-batch, >= 1; M * T * k < 2^31      */
  int n_shared; /* always-on shared experts per layer (gate 1.0, not
                   counted in the workloads w)                           */
  int renorm;   /* 1: gates renormalised over the top-k                  */
  int dtype;    /* EB_DTYPE_*                                            */
  int policy;   /* EB_SCHED_*                                            */
  int m;        /* minimum RunSet size, 1..M ([EB] §4.2)                 */
  int residual; /* 1: h_{l+1} = h_l + MoE_l(h_l); 0: h_{l+1} = MoE_l(h_l) */
  int compute;  /* 1: full step; 0: routing + scheduling only            */
  int gemm;     /* EB_GEMM_*                                             */
} eb_config;

typedef struct eb_ctx eb_ctx;

/* Human-readable name of a status code (static string). */
const char* eb_status_string(eb_status s);

/* Checks a configuration without touching the GPU. */
eb_status eb_config_check(const eb_config* cfg);

/* Bytes of device workspace eb_moe_step needs for `cfg` (host only).  The
 * caller allocates it (256-byte aligned) and keeps it, unchanged, for a whole
 * episode: it carries the routed indices and gates of deferred micro-batches
 * from one step to the next. */
eb_status eb_workspace_size(const eb_config* cfg, size_t* bytes);

/* Creates a context on the current CUDA device.  The context owns a small
 * device state (per-micro-batch layers l_j, the pending set S, histograms,
 * loads, the exact utilisation accumulators and the per-step trace). */
eb_status eb_create(const eb_config* cfg, eb_ctx** out);
eb_status eb_destroy(eb_ctx* ctx);

/* Algorithm 1 initialisation ([EB] §4.2): l_j = 0 for all j, S_0 = all
 * micro-batches, RunSet_0 = all (every micro-batch routes at step 1), and
 * zeroed accumulators and trace.  With EB_GEMM_TMC it also zeroes the fused
 * combine's arrival counters, which a step that gave up on a bounded wait
 * (EB_ERR_TIMEOUT) may have left non-zero: after such an error, reset before
 * the next step.  Enqueued on `stream`. */
eb_status eb_reset(eb_ctx* ctx, void* stream);

/* Router mode ([EB] §2.1, W_l, I_l = topk(G(h'_l)) with a linear scorer):
 * w_router (DEVICE, bf16 [L, E, H], 16-byte aligned, caller-owned) makes
 * every step project the routing scores itself -- scores = h W_r[l]^T in
 * float32 for each micro-batch that routes, from its current hidden state
 * and the router of its layer -- instead of reading the caller's logits,
 * so the chain becomes data-dependent; eb_moe_step / eb_episode may then
 * get logits = NULL.  scores (optional DEVICE float32 [M, L, T, E], 16-byte
 * aligned, caller-owned) receives every step's scores at (j, l_j), where the
 * routing then reads them; with scores = NULL they stay in the workspace.
 * w_router = NULL returns to caller-given logits.  Needs compute, bf16, E a
 * multiple of 16 (at most 256) and H a multiple of 64 (EB_ERR_UNSUPPORTED
 * otherwise). */
eb_status eb_set_router(eb_ctx* ctx, const void* w_router, float* scores);

/* Expert placement used to fold expert counts into rank loads.  By default
 * rank d holds experts [d E/D, (d+1) E/D) ([EB] §5 Models, "evenly
 * distributed").  expert_rank (HOST array of cfg.E int32, each in
 * [0, cfg.D)) replaces it by any placement -- e.g. one a load balancer such
 * as EPLB chose, which [EB] §5.3 treats as orthogonal to scheduling; NULL
 * restores the contiguous map.  Copied synchronously into the context (call
 * it with none of the context's steps in flight); takes effect from the next
 * routing.  EB_ERR_INVALID_ARG for a rank outside [0, D). */
eb_status eb_set_expert_map(eb_ctx* ctx, const int32_t* expert_rank);

/*
 * One EasyBalance step, [EB] §4.2 Algorithm 1 loop body, entirely on device:
 *   1. route the micro-batches of the previous RunSet at their layer l_j:
 *      softmax top-k of the fp32 logits, renormalised gates ([EB] §2.1);
 *      per-expert counts T_e folded into w_j over the contiguous map, or
 *      the placement set by eb_set_expert_map ([SysLB] §1; [EB] §2.3);
 *   2. RunSet = Schedule(S, m) with cfg.policy; exact int64 utilisation
 *      accumulators ([EB] Eq. (2), (3)); trace row;
 *   3. permute the RunSet's tokens into segments keyed (layer, expert)
 *      -- micro-batches at the same layer share a segment --, one grouped
 *      SwiGLU expert GEMM over all segments (experts of different layers in
 *      one launch), and the gated combine in slot order ([EB] Eq. (1)),
 *      written back into `hidden`;
 *   4. l_j += 1 for the RunSet; finished micro-batches leave S.
 * Once S is empty a step does nothing.
 *
 * After a step that gave up on a bounded wait (status EB_ERR_TIMEOUT) the
 * context refuses to step until eb_reset: on the device every later step
 * does nothing and reports S as empty; once the host has seen the status
 * (eb_sync_status, eb_episode, or a step with runset_host) eb_moe_step
 * returns EB_ERR_TIMEOUT at once.  With runset_host the call also returns
 * EB_ERR_TIMEOUT when the status word holds it after the step.
 *
 * logits    [M, L, T, E] float32: the router logits of micro-batch j at
 *           layer l; only the blocks (j, l_j) of routed micro-batches are read.
 * hidden    [M, T, H] cfg.dtype, updated in place for RunSet micro-batches.
 * w_gateup  [L, E + n_shared, 2F, H] cfg.dtype, row-major; rows 0..F-1 of an
 *           expert are its gate projection, rows F..2F-1 its up projection.
 *           Must be 16-byte aligned.
 * w_down    [L, E + n_shared, H, F] cfg.dtype.  Must be 16-byte aligned.
 * workspace at least eb_workspace_size() bytes, 256-byte aligned.
 * runset_host  optional host pointer: if non-NULL the call waits for the step
 *           and stores its RunSet bitmask (bit j = micro-batch j; 0 = nothing
 *           ran because S was empty).
 * With cfg.compute == 0 only steps 1, 2 and 4 run (hidden and weights may be
 * NULL).
 */
eb_status eb_moe_step(eb_ctx* ctx, const float* logits, void* hidden, const void* w_gateup,
                      const void* w_down, void* workspace, size_t workspace_bytes, void* stream,
                      uint32_t* runset_host);

/* The expert computation of expert parallelism ([EB] §2.2: between the
 * dispatch and combine all-to-alls, a rank runs its experts' FFNs on the
 * token rows it received): rows [R, H] (cfg.dtype, DEVICE, 16-byte aligned,
 * caller-owned) are grouped into nseg segments, segment i being rows
 * [seg_off[i], seg_off[i+1]) for expert seg_expert[i] (0..E+n_shared-1) of
 * layer seg_layer[i] (HOST int32 arrays; seg_off has nseg + 1 entries,
 * ascending from 0 to R; segments may come in any order and repeat an
 * expert).  out [R, H] (cfg.dtype, DEVICE, 16-byte aligned) receives
 * W_down (silu(W_gate x) * (W_up x)) of every row x, in the same order, with
 * the step's arithmetic (bf16 activation, fp32 accumulation, one rounding of
 * each output).  The step's GEMM engines run it (the gathering and
 * fused-combine engines as their plain token-major form); it uses the
 * context's workspace, so no step of the context may be in flight, and it
 * leaves the step state untouched.  Synchronous.  Needs cfg.compute;
 * R <= M * T * (k + n_shared) and nseg <= M * (E + n_shared)
 * (EB_ERR_UNSUPPORTED otherwise); EB_ERR_INVALID_ARG for a malformed segment
 * table; EB_ERR_TIMEOUT if a bounded device wait expired. */
eb_status eb_expert_ffn(eb_ctx* ctx, const void* rows, int R, const int32_t* seg_off,
                        const int32_t* seg_layer, const int32_t* seg_expert, int nseg, void* out,
                        const void* w_gateup, const void* w_down, void* workspace,
                        size_t workspace_bytes, void* stream);

/* A whole episode: eb_reset, then eb_moe_step until S is empty.  Steps are
 * enqueued a few ahead of the host's completion check, so the GPU never waits
 * for the host; steps enqueued after S became empty do nothing.  The check
 * reads S from pinned host memory that each scheduler launch writes (the
 * calling thread polls it, yielding), so nothing but kernels is enqueued
 * between the steps; without mapped host memory it falls back to a copy and
 * an event per step.  Returns the
 * number of steps that ran in *n_steps (host).  Waits for completion; returns
 * EB_ERR_TIMEOUT if a bounded device wait expired during the episode.
 * Because every step reads the same logits, consecutive steps overlap (same
 * results, bit for bit, as eb_moe_step step by step; without router mode
 * and with a tensor-core GEMM 2):
 *   - step i+1's routing runs beside step i's GEMM 2, into the second of the
 *     workspace's two gate buffers;
 *   - step i's combine runs beside step i+1's scheduler.
 * An episode that returns an error leaves the context mid-step: call
 * eb_reset before stepping it again. */
eb_status eb_episode(eb_ctx* ctx, const float* logits, void* hidden, const void* w_gateup,
                     const void* w_down, void* workspace, size_t workspace_bytes, void* stream,
                     int* n_steps);

/* Exact utilisation totals of the steps run since eb_reset (waits for the
 * context's work):
 *   num     = sum over steps of sum_d W_d            (work done)
 *   den     = D * sum over steps of max_d W_d         ([EB] Eq. (3) denominator)
 *   den_sep = D * sum over executed (j, l) of max_d w_{j,l}
 *             (each micro-batch run on its own: the "maximum workload" of
 *             [EB] Fig. 6).
 * u = num / den; the no-combination baseline is num / den_sep. */
eb_status eb_utilization(eb_ctx* ctx, int64_t* num, int64_t* den, int64_t* den_sep);

/* Per-step trace since eb_reset (waits).  Host arrays: rows [max_steps][6]
 * int64 = (RunSet mask, sum_d W_d, max_d W_d, sum_{j in RunSet} max_d w_j,
 * permuted token rows R of the step, non-empty (layer, expert) segments);
 * layers [max_steps][M] int32 = layer at which micro-batch j ran in that step,
 * or -1.  *n_steps receives the number of steps recorded (may exceed
 * max_steps; only max_steps rows are written).  layers may be NULL. */
eb_status eb_trace(eb_ctx* ctx, int64_t* rows, int32_t* layers, int max_steps, int* n_steps);

/* Measurement support.  eb_profile(ctx, 1) brackets every kernel the context
 * enqueues with CUDA events on the launching stream (eb_profile(ctx, 0) stops;
 * both drop earlier marks).  eb_profile_read waits for them and returns, per
 * kernel, the summed milliseconds and the number of launches since, then
 * clears the marks.  Kernel order: route (with the rows' ranks within their
 * chunk and the chunk offsets), schedule+plan, permute (the row copy, which
 * also places the rows), GEMM 1 (gate/up + SwiGLU), GEMM 2 (down), combine,
 * positions (the rows of every token slot, computed in a pass of its own
 * only for the gathering GEMM 1, which has no row copy), router projection
 * (router mode).
 * eb_launch_count returns the kernels the context has enqueued since
 * eb_create.  eb_engines returns the EB_GEMM_* engine that runs GEMM 1 and
 * GEMM 2 (after AUTO and the shape fallbacks above are resolved; SIMT for
 * f32); with EB_GEMM_TMC as GEMM 2 the step launches no combine kernel and
 * the combine's time is in GEMM 2's.  Host only: EB_ERR_INVALID_ARG for a
 * null argument. */
#define EB_PROF_KERNELS 8
eb_status eb_profile(eb_ctx* ctx, int enable);
eb_status eb_profile_read(eb_ctx* ctx, double* ms, int64_t* launches);
eb_status eb_launch_count(eb_ctx* ctx, int64_t* n);
eb_status eb_engines(const eb_ctx* ctx, int* gemm1, int* gemm2);

/* Failure-detection self-test (the pages describe no failure handling).  Every
 * device-side wait of the tensor-core GEMMs is bounded; when one expires the
 * kernel records EB_ERR_TIMEOUT, finishes its own copies, frees its TMEM and
 * returns instead of hanging.  This call runs that same bounded wait on a
 * barrier nothing ever arrives on, with a limit of limit_ns nanoseconds
 * (1e3..2e9), and leaves EB_ERR_TIMEOUT in the device int32 *status_dev. */
eb_status eb_selftest_timeout(int64_t limit_ns, int32_t* status_dev, void* stream);

/* Waits for the context's work and returns the device-side status. */
eb_status eb_sync_status(eb_ctx* ctx);

/* Failure-injection hook for tests (the pages describe no failure handling):
 * records `status` (EB_OK or one of the EB_ERR_* codes) in the context's
 * device status word, stream-ordered, as a failing kernel would.  With
 * EB_ERR_TIMEOUT and the fused-combine engine (EB_GEMM_TMC) it also leaves
 * every arrival counter non-zero, the partial counts a GEMM 2 that gave up
 * part-way can leave, so a test can check that the context refuses to step
 * and that eb_reset restores it.  Nothing on the GPU waits, traps or faults.
 * EB_ERR_INVALID_ARG for an unknown code. */
eb_status eb_inject_status(eb_ctx* ctx, eb_status status, void* stream);

/* ---------------------------------------------------------------------------
 * Stand-alone stages (stateless; device pointers; async on `stream`).
 * ------------------------------------------------------------------------ */

/* Router top-k over n independent token rows, [EB] §2.1 topk(G(h')):
 * logits [n, E] float32 -> idx [n, k] int32 (descending logit; equal logits
 * to the lower expert index), gate [n, k] float32 (softmax probabilities of
 * the selected experts, renormalised to sum 1 if renorm), hist [E] int32
 * (tokens per expert, T_e of [SysLB] §1; overwritten).  status_dev is an
 * optional device int32: if non-NULL it is set to EB_ERR_NONFINITE when a
 * NaN or Inf logit is seen (and left unchanged otherwise). */
eb_status eb_route(const float* logits, int n, int E, int k, int renorm, int32_t* idx, float* gate,
                   int32_t* hist, int32_t* status_dev, void* stream);

/* Virtual-rank loads under the contiguous map: w[j][d] = sum of hist[j][e]
 * over e in [d E/D, (d+1) E/D).  hist [M, E] int32 -> w [M, D] int32. */
eb_status eb_loads(const int32_t* hist, int M, int E, int D, int32_t* w, void* stream);

/* Router scores for n token rows: scores [n, E] float32 = hidden [n, H] bf16
 * times w_router [E, H] bf16 transposed (float32 accumulation on the tensor
 * cores).  DEVICE pointers, 16-byte aligned.  E a multiple of 16 (<= 256), H a
 * multiple of 64, else EB_ERR_UNSUPPORTED.  status_dev (optional device
 * int32) gets EB_ERR_TIMEOUT if a bounded device wait expires. */
eb_status eb_router(const void* hidden, int n, int H, const void* w_router, int E, float* scores,
                    int32_t* status_dev, void* stream);

/* Virtual-rank loads under an arbitrary placement: w[j][d] = sum of
 * hist[j][e] over the experts e with expert_rank[e] == d.  expert_rank is a
 * DEVICE array of E int32; E need not be a multiple of D.  An entry outside
 * [0, D) drops that expert's counts and sets *status_dev (optional device
 * int32) to EB_ERR_INVALID_ARG. */
eb_status eb_loads_mapped(const int32_t* hist, int M, int E, int D, const int32_t* expert_rank,
                          int32_t* w, int32_t* status_dev, void* stream);

/* RunSet = Schedule(S, m) for one step ([EB] §4.2, §5.2).
 * w [M, D] int32 loads; pending_mask: bit j set = j in S.
 * runset_mask (device uint32) receives the RunSet bitmask; step_stats
 * (device int64[3], may be NULL) receives (sum_d W_d, max_d W_d,
 * sum_{j in RunSet} max_d w_j).  If |S| <= m the RunSet is S. */
eb_status eb_schedule(const int32_t* w, uint32_t pending_mask, int M, int D, int m, int policy,
                      uint32_t* runset_mask, int64_t* step_stats, void* stream);

/* ---------------------------------------------------------------------------
 * No-allocation routing + loads.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- a serving
 * process whose memory is fixed at start-up (a pre-reserved pool, or an
 * allocator that refuses cudaMalloc after warm-up), or a caller that must
 * not call cudaMalloc / cudaFree because they can synchronise the device.
 *
 * Routes n_mb independent micro-batches (as eb_route does for each) and folds
 * their expert counts into virtual-rank loads (as eb_loads does):
 *   logits [n_mb, T, E] float32 -> idx [n_mb, T, k] int32,
 *   gate [n_mb, T, k] float32, w [n_mb, D] int32 (contiguous map).
 * status_dev: optional device int32, set to EB_ERR_NONFINITE on a NaN/Inf.
 * The caller passes inputs and outputs; the intermediate per-(micro-batch,
 * 64-token chunk, expert) counts live in a file-scope device array of
 * 2^20 int32 (4 MiB) that every GPU loading the library holds until exit.
 * n_mb * ceil(T / 64) * E above 2^20 returns EB_ERR_TOO_LARGE before any
 * launch.  The call allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).  Its first call on a device looks the array's device
 * address up (cudaGetSymbolAddress) and caches it with the CUDA context it
 * belongs to: make that first call before any stream capture.  If the
 * context changes (cudaDeviceReset() ends the primary context; the next
 * call runs in a new one), the next call looks the address up again, and
 * that call too should come before any stream capture.  Every call shares the one array: calls that
 * overlap on the GPU (other streams, other threads) race on it, so order
 * them on one stream.  Each call writes every count it reads, so stale
 * contents from an earlier call never leak into a result.
 * ------------------------------------------------------------------------ */
eb_status eb_route_loads_static(const float* logits, int n_mb, int T, int E, int k, int renorm,
                                int D, int32_t* idx, float* gate, int32_t* w, int32_t* status_dev,
                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EB_H */
