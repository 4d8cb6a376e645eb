// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a):
// one persistent launch per GEMM over every (layer, expert) segment of the
// step, so experts of different layers share a launch.
//
// Expert FFN of [EB] Eq. (1), read as SwiGLU:
//   GEMM 1:  act = bf16( silu(A W_gate^T) * (A W_up^T) )   (fp32 accumulation)
//   GEMM 2:  y   = bf16( act W_down^T )
//
// Layout ("swap AB"): the 128 weight rows of an output-feature block are the
// MMA's M side and the segment's token rows its N side (N = the chunk's row
// count rounded up to 16, at most 128), so a segment of a few dozen rows costs
// a narrow MMA instead of a half-empty 128-row tile.  D[f, r] accumulates in
// TMEM; lane f of the accumulator belongs to epilogue thread f.
//
// Work item = (segment, 128-feature block, 128-row chunk), chunks innermost,
// so CTAs that run side by side read the same weight tile (L2 reuse).  Roles
// per CTA (192 threads): warp 0 issues TMA loads into a ring of shared-memory
// stages, warp 1 allocates TMEM and one thread issues the MMAs, warps 2-5 drain
// the accumulator (double buffered, so the drain overlaps the next item).
// Operands are K-major with the 128-byte swizzle in both TMA and the MMA
// descriptors.  Every mbarrier wait is bounded: on expiry the CTA records
// EB_ERR_TIMEOUT in the step's status word, waits (bounded) for its own copies
// and MMAs in flight, frees its TMEM and returns.
#include <cuda.h>

#include <atomic>
#include <cuda_bf16.h>

#include "eb_internal.cuh"
#include "gemm_tc.cuh"

namespace eb {
namespace {

constexpr int kBM = 128;        // weight rows (features) per MMA tile
constexpr int kBK = 64;         // K elements per stage: 128 bytes of bf16 = one swizzle row
constexpr int kTileBytes = kBM * kBK * 2;  // 16 KiB
#ifndef EB_EPI_WARPS
#define EB_EPI_WARPS 8
#endif
constexpr int kEpiWarps = EB_EPI_WARPS;    // 4 or 8: warps draining TMEM
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
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

// Bounded wait for the phase of parity `parity` to complete.  Returns false
// (and raises the CTA's abort flag) if it does not within the limit, or if
// another role of the CTA has aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicCAS(status, EB_OK, EB_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// K-major operand, 128-byte swizzle: rows of 128 B, 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address (16 B units)
  d |= (uint64_t)1 << 16;                     // leading byte offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;           // stride byte offset: next 8-row atom
  d |= (uint64_t)1 << 46;                     // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                     // SWIZZLE_128B
  return d;
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 columns of 32-bit accumulator -> 32 registers per thread,
// issued without waiting (tmem_wait() makes the registers valid).
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  tmem_ld32_issue(taddr, r);
  tmem_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 32-column loads in flight together, one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t taddr0, uint32_t taddr1, float* v0,
                                            float* v1) {
  uint32_t r0[32], r1[32];
  tmem_ld32_issue(taddr0, r0);
  tmem_ld32_issue(taddr1, r1);
  tmem_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v0[i] = __uint_as_float(r0[i]);
    v1[i] = __uint_as_float(r1[i]);
  }
}

__device__ __forceinline__ int find_segment(const int32_t* items, int nseg, int item) {
  int lo = 0, hi = nseg;  // items[lo] <= item < items[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (items[mid] <= item) lo = mid;
    else hi = mid;
  }
  return lo;
}

struct Item {
  int r0;     // first token row of the chunk
  int n;      // token rows in the chunk (1..128)
  int f0;     // first output feature of the block
  int wrow;   // first weight row (gate rows for GEMM 1)
};

template <bool GATEUP>
struct Cfg;

template <bool GATEUP>
__device__ __forceinline__ Item decode(const Dims& d, const int32_t* seg_rows,
                                       const int32_t* seg_wid, const int32_t* seg_items,
                                       int nseg, int item) {
  constexpr int kBN = Cfg<GATEUP>::kBN;
  const int s = find_segment(seg_items, nseg, item);
  const int local = item - seg_items[s];
  const int rb = seg_rows[s], cnt = seg_rows[s + 1] - rb;
  const int nch = (cnt + kBN - 1) / kBN;
  const int chunk = local % nch, mb = local / nch;
  Item it;
  it.r0 = rb + chunk * kBN;
  it.n = min(kBN, cnt - chunk * kBN);
  it.f0 = mb * kBM;
  it.wrow = seg_wid[s] * (GATEUP ? 2 * d.F : d.H) + it.f0;
  return it;
}

template <bool GATEUP>
struct Cfg {
  static constexpr int kBN = GATEUP ? kTcRows1 : kTcRows2;  // token rows per item (max MMA N)
  static constexpr int kXBytes = kBN * kBK * 2;              // 16 or 32 KiB
  static constexpr int kStageBytes = (GATEUP ? 2 : 1) * kTileBytes + kXBytes;
  static constexpr int kStages = (196608 / kStageBytes) < 8 ? (196608 / kStageBytes) : 8;
  static constexpr int kAccCols = (GATEUP ? 2 : 1) * kBN;  // TMEM columns per accumulator
  static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;  // double buffer if it fits
  static constexpr int kTmemCols = kAccBufs * kAccCols;     // 256 or 512
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /* barriers */ + 1024 /* align */;
};

// GATEUP: map_w = w_gateup [L*Etot*2F, H], map_x = A [Rcap, H], out = act [Rcap, F]
// DOWN:   map_w = w_down   [L*Etot*H, F],  map_x = act [Rcap, F], out = y [Rcap, H]
template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
              Dims d, State* __restrict__ st, const int32_t* __restrict__ seg_rows,
              const int32_t* __restrict__ seg_wid, const int32_t* __restrict__ seg_items,
              const int32_t* __restrict__ rowslot, __nv_bfloat16* __restrict__ out) {
  pdl_enter();
  using C = Cfg<GATEUP>;
  constexpr int kBN = C::kBN;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;                      // [kStages]
  uint64_t* empty = bars + C::kStages;        // [kStages]
  uint64_t* tfull = bars + 2 * C::kStages;    // [2]
  uint64_t* tempty = tfull + 2;               // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nseg = st->nseg;
  const int total = (nseg > 0 && st->runset != 0) ? seg_items[nseg] : 0;
  if (total == 0) return;  // uniform across the CTA: nothing to do this step
  const int K = GATEUP ? d.H : d.F;
  const int nk = K / kBK;
  const int NOUT = GATEUP ? d.F : d.H;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 32 * kEpiWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // per stage: armed at least once / parity of last arm
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const Item it = decode<GATEUP>(d, seg_rows, seg_wid, seg_items, nseg, item);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, &st->status)) {
            ok = false;
            break;
          }
          uint8_t* sb = stage_base + stage * C::kStageBytes;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, C::kStageBytes);
          tma_load_2d(smem_u32(sb), &map_w, kb * kBK, it.wrow, fb);
          if (GATEUP) tma_load_2d(smem_u32(sb + kTileBytes), &map_w, kb * kBK, it.wrow + d.F, fb);
          tma_load_2d(smem_u32(sb + (GATEUP ? 2 : 1) * kTileBytes), &map_x, kb * kBK, it.r0, fb);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {  // let our own copies land before the CTA's shared memory goes away
        for (int s = 0; s < C::kStages; ++s)
          if ((armed >> s) & 1u) {
            const unsigned long long t0 = global_ns();
            while (!mbar_try(smem_u32(&full[s]), (armed_par >> s) & 1u) &&
                   global_ns() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t last_bar = 0, last_par = 0;
      bool ok = true, issued = false;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const Item it = decode<GATEUP>(d, seg_rows, seg_wid, seg_items, nseg, item);
        const int N = ((it.n + 15) / 16) * 16;
        const uint32_t idesc = idesc_bf16(kBM, N);
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, abort_flag, &st->status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_gate = tmem + acc * C::kAccCols;
        const uint32_t d_up = d_gate + kBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, &st->status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(stage_base + stage * C::kStageBytes);
          const uint32_t sx = sb + (GATEUP ? 2 : 1) * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks) {
            const uint32_t koff = ks * 32;  // 16 bf16 = 32 bytes along K
            const uint32_t acc_flag = (kb | ks) != 0;
            mma_bf16(d_gate, sdesc(sb + koff), sdesc(sx + koff), idesc, acc_flag);
            if (GATEUP) mma_bf16(d_up, sdesc(sb + kTileBytes + koff), sdesc(sx + koff), idesc, acc_flag);
          }
          mma_commit(smem_u32(&empty[stage]));
          last_bar = smem_u32(&empty[stage]);
          last_par = phase;
          issued = true;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull[acc]));
        last_bar = smem_u32(&tfull[acc]);
        last_par = acc_phase;
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok && issued) {  // MMAs still reading shared memory / writing TMEM
        const unsigned long long t0 = global_ns();
        while (!mbar_try(last_bar, last_par) && global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int frow = q * 32 + lane;    // feature row of this thread within the tile
    const int cgrp = (warp - 2) >> 2;  // with 8 warps, two warps split a quarter's columns
    constexpr int kColStep = 32 * (kEpiWarps / 4);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const Item it = decode<GATEUP>(d, seg_rows, seg_wid, seg_items, nseg, item);
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, &st->status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + acc * C::kAccCols;
      __nv_bfloat16* orow = out + (size_t)it.r0 * NOUT + it.f0 + frow;
      for (int cb = cgrp * 32; cb < it.n; cb += kColStep) {
        float g[32];
        tmem_ld32(tbase + cb, g);
        if (GATEUP) {
          float u[32];
          tmem_ld32(tbase + kBN + cb, u);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (cb + i < it.n) {
              const float a = g[i] / (1.f + expf(-g[i])) * u[i];
              orow[(size_t)(cb + i) * NOUT] = __float2bfloat16_rn(a);
            }
          }
        } else {  // y rows at their (token, slot) positions
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (cb + i < it.n)
              out[(size_t)__ldg(rowslot + it.r0 + cb + i) * NOUT + (orow - out) % NOUT] =
                  __float2bfloat16_rn(g[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::kTmemCols));
  }
}

// Failure-detection self-test: waits, with the GEMM's bounded wait, on an
// mbarrier nothing ever arrives on; the wait expires after limit_ns and
// leaves EB_ERR_TIMEOUT in *status.  Nothing faults and the context stays
// usable.
__global__ void k_selftest_wait(unsigned long long limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0 && mbar_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns))
    atomicExch(status, EB_OK);  // not reached: nothing arrives on the barrier
}


// ---------------------------------------------------------------------------
// Token-major variant.  Tokens are the MMA's M side (128 per accumulator) and
// 256 weight rows its N side (GEMM 1: the gate and up rows of one 128-feature
// block; GEMM 2: 256 output features), so every MMA is 128 x 256 x 16 -- large
// enough to run at the tensor pipe's rate with operands read fresh from
// shared memory -- and a token's accumulator row holds its 256 outputs, so
// the drain writes contiguous 16-byte chunks.
//
// One work item is one 128-token chunk of a segment against one weight tile.
// Only the chunk's own token rows are loaded (32-row boxes); the rest of the
// 128-row operand is stale shared memory whose products land in accumulator
// rows that are never stored.  Items are claimed dynamically from a
// step-wide counter, so CTAs finish together whatever the segment sizes.
// ---------------------------------------------------------------------------

// Segment plan (row offsets, expert ids, item offsets) of up to kSegCache
// segments is copied into shared memory at kernel start, so the per-item
// decode (a binary search over item offsets) runs on shared memory instead
// of dependent global loads; larger plans are read from global memory.
constexpr int kSegCache = 1536;
constexpr int kSegCacheBytes = ((3 * 4 * (kSegCache + 1)) + 127) / 128 * 128;

struct SegView {
  const int32_t* rows;
  const int32_t* wid;
  const int32_t* items;
};

__device__ __forceinline__ SegView cache_segments(uint8_t* buf, int nseg, const int32_t* seg_rows,
                                                  const int32_t* seg_wid,
                                                  const int32_t* seg_items) {
  if (nseg > kSegCache) return {seg_rows, seg_wid, seg_items};
  int32_t* r = reinterpret_cast<int32_t*>(buf);
  int32_t* w = r + kSegCache + 1;
  int32_t* it = w + kSegCache + 1;
  for (int i = threadIdx.x; i <= nseg; i += blockDim.x) {
    r[i] = seg_rows[i];
    it[i] = seg_items[i];
    if (i < nseg) w[i] = seg_wid[i];
  }
  return {r, w, it};
}

constexpr int kGatherWarps = 4;  // row-gathering warps of the gathering GEMM 1 (one thread per row)
// The fused combine (GEMM 2, engine TMC): the drain hands every completed
// (token, 256-feature block) to kCombineWarps extra warps through a ring of
// kCombineQueue entries in shared memory, so the drain never waits on the
// combine's loads.
constexpr int kCombineWarps = 8;
constexpr int kCombineQueue = 512;
constexpr int kCombineBytes = (kCombineQueue + 4) * 4;
constexpr int kGatherDepth = 2;  // k-blocks a gathering thread keeps in flight before signalling
constexpr int kTmBox = 32;                    // token rows per TMA box
constexpr int kTmBoxBytes = kTmBox * kBK * 2;  // 4 KiB

template <bool GATEUP>
struct CfgTM {
  static constexpr int kRows = kTmRows;  // token rows per item (MMA M)
  static constexpr int kN = 256;         // weight rows per item (MMA N)
  static constexpr int kFeat = GATEUP ? kTmFeat1 : kTmFeat2;  // output features per item
  static constexpr int kABytes = kRows * kBK * 2;   // 16 KiB token tile
  static constexpr int kBBytes = kN * kBK * 2;      // 32 KiB weight tile
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 196608 / kStageBytes;  // 4
  static constexpr int kAccCols = kN;
  static constexpr int kAccBufs = 2;
  static constexpr int kTmemCols = kAccBufs * kAccCols;  // 512
  static constexpr int kQueue = 8;  // claimed items queued for the MMA issuer and the drain
  static constexpr int kSmemBytes =
      kStages * kStageBytes + 1024 + kSegCacheBytes + (GATEUP ? 0 : kCombineBytes) + 1024;
  static_assert(kRows == 128 && kFeat * (GATEUP ? 2 : 1) == kN, "token-major tile shape");
  static_assert(kGatherDepth >= 1 && kGatherDepth < kStages, "a gathering thread signals a stage before it reuses it");
  static_assert(32 * kGatherWarps == kRows, "one gathering thread per token row");
  static_assert((2 * kStages + 4 + 2 * kQueue) * 8 + 8 + 4 * kQueue <= 1024, "barrier region");
};

template <bool GATEUP>
__device__ __forceinline__ Item decode_tm(const Dims& d, const int32_t* seg_rows,
                                          const int32_t* seg_wid, const int32_t* seg_items,
                                          int nseg, int item) {
  using C = CfgTM<GATEUP>;
  const int s = find_segment(seg_items, nseg, item);
  const int local = item - seg_items[s];
  const int rb = seg_rows[s], cnt = seg_rows[s + 1] - rb;
  // The feature blocks of one chunk are consecutive items: the CTAs running
  // side by side share that chunk's token rows (read from DRAM once), and a
  // segment's weight tiles stay in L2 across its chunks.  (With the chunks
  // of one feature block consecutive instead, a long segment's token rows
  // came back from DRAM once per feature block: 3.4x the DRAM reads of
  // GEMM 1 at 8192 tokens per micro-batch.)
  const int nfb = (GATEUP ? d.F : d.H) / C::kFeat;
  const int chunk = local / nfb, mb = local % nfb;
  Item it;
  it.r0 = rb + chunk * C::kRows;
  it.n = min(C::kRows, cnt - chunk * C::kRows);
  it.f0 = mb * C::kFeat;
  it.wrow = seg_wid[s] * (GATEUP ? 2 * d.F : d.H) + it.f0;
  return it;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One token's combine over 256 features, by one warp (lane: features
// f + 8 lane .. + 7): h (if residual) + sum over slots s of gate_s y_s (shared
// slots s >= k with weight 1), in slot order, rounded once to bf16 into
// hidden.  The same arithmetic, element for element, as the stand-alone
// combine kernel, so the fused and unfused steps agree bit for bit.  The
// token's y rows were stored by other CTAs of this launch: they are read
// through L2 (ld.global.cg), after the acquiring fence of the caller.
__device__ __forceinline__ void combine_token(const Dims& d, const State* st, int tok, int f,
                                              int lane, const float* __restrict__ gate,
                                              const __nv_bfloat16* y, __nv_bfloat16* hidden) {
  const int k = d.k, kk = d.kk;
  const float my_gate = lane < k ? __ldg(gates_of(gate, st->gate_buf, d, tok) + lane) : 0.f;
  uint4* hp = reinterpret_cast<uint4*>(hidden + (size_t)tok * d.H + f + 8 * lane);
  float acc[8];
  if (d.residual) {
    const uint4 h = __ldcg(hp);
    const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&h);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __bfloat1622float2(hb[i]);
      acc[2 * i] = v.x;
      acc[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  }
  const __nv_bfloat16* yt = y + (size_t)tok * kk * d.H + f + 8 * lane;
  for (int s0 = 0; s0 < kk; s0 += 4) {
    uint4 r[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (s0 + q < kk) r[q] = __ldcg(reinterpret_cast<const uint4*>(yt + (size_t)(s0 + q) * d.H));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = s0 + q;
      const float g = __shfl_sync(0xffffffffu, my_gate, s & 31);
      if (s >= kk) break;
      const __nv_bfloat162* yb = reinterpret_cast<const __nv_bfloat162*>(&r[q]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(yb[i]);
        if (s < k) {
          acc[2 * i] = fmaf(g, v.x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(g, v.y, acc[2 * i + 1]);
        } else {
          acc[2 * i] += v.x;
          acc[2 * i + 1] += v.y;
        }
      }
    }
  }
  *hp = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// map_x: token rows [Rcap, K] in boxes of 32 rows; map_w: weights in boxes
// of 128 rows.  GATEUP: out = act [Rcap, F]; else out = y [Rcap, H].
// next_item: the step's claim counter (zero before the launch).
// GATHER (GEMM 1 only): the token rows are not read from a permuted copy;
// kGatherWarps extra warps copy each chunk row straight from the hidden
// states xsrc [M*T, H], through rowslot (permuted row -> (token, slot)), into
// the swizzled operand tile with 16-byte cp.async copies.  GEMM 2 stores each
// output row at its (token, slot) position rowslot[row].
// COMBINE (GEMM 2 only): the combine runs in the drain.  Each drain thread
// that has stored its share of a row of y counts it in arrive[token][feature
// block] (after a fence); the thread that brings the count to kk * kGroups
// (every slot of the token, every column group) resets it to zero and its
// warp combines the token's 256 features of that block into hidden.
// Nothing waits: a token is combined by whichever drain finishes it last.
template <bool GATEUP, bool GATHER, bool COMBINE>
__global__ void __launch_bounds__(GATHER    ? kThreads + 32 * kGatherWarps
                                  : COMBINE ? kThreads + 32 * kCombineWarps
                                            : kThreads,
                                  1)
    k_gemm_tm(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
              Dims d, State* __restrict__ st, const int32_t* __restrict__ seg_rows,
              const int32_t* __restrict__ seg_wid, const int32_t* __restrict__ seg_items,
              int32_t* __restrict__ next_item, const int32_t* __restrict__ rowslot,
              const __nv_bfloat16* __restrict__ xsrc, __nv_bfloat16* out,
              int32_t* __restrict__ arrive, const float* __restrict__ gate,
              __nv_bfloat16* hidden) {
  static_assert(!COMBINE || (!GATEUP && !GATHER), "the combine follows GEMM 2");
  pdl_enter();
  using C = CfgTM<GATEUP>;
  constexpr int Q = C::kQueue;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;                      // [kStages] k-block landed
  uint64_t* empty = bars + C::kStages;        // [kStages] k-block consumed by the MMAs
  uint64_t* tfull = bars + 2 * C::kStages;    // [2] accumulator complete
  uint64_t* tempty = tfull + 2;               // [2] accumulator drained
  uint64_t* iready = tempty + 2;              // [Q] item queue entry written
  uint64_t* ifree = iready + Q;               // [Q] entry read by the MMA issuer and the drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ifree + Q);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* iq = const_cast<int*>(abort_flag) + 1;  // [Q] claimed items, -1 ends the sequence
  uint8_t* seg_buf = reinterpret_cast<uint8_t*>(bars) + 1024;
  // fused combine: ring of (token, feature block) entries (-1: empty), then
  // the push and pop counters and the count of drain warps that finished
  volatile int* cq = reinterpret_cast<volatile int*>(seg_buf + kSegCacheBytes);
  int* cq_ctl = const_cast<int*>(cq) + kCombineQueue;  // [0] pushed [1] popped [2] drains done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nseg = st->nseg;
  const int total = (nseg > 0 && st->runset != 0) ? seg_items[nseg] : 0;
  if (total == 0) return;
  const int K = GATEUP ? d.H : d.F;
  const int nk = K / kBK;
  const int NOUT = GATEUP ? d.F : d.H;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      // GATHER: the weight copies' arrival plus one per gathering thread
      mbar_init(smem_u32(&full[i]), GATHER ? 1 + 32 * kGatherWarps : 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), kEpiWarps);
    }
    for (int i = 0; i < Q; ++i) {
      mbar_init(smem_u32(&iready[i]), 1);
      mbar_init(smem_u32(&ifree[i]), kEpiWarps + 1 + (GATHER ? kGatherWarps : 0));
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (COMBINE) {
    for (int i = threadIdx.x; i < kCombineQueue; i += blockDim.x) cq[i] = -1;
    if (threadIdx.x < 3) cq_ctl[threadIdx.x] = 0;
  }
  const SegView sv = cache_segments(seg_buf, nseg, seg_rows, seg_wid, seg_items);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // A CTA's first item is blockIdx.x; each further one is gridDim.x plus
    // the next value of the claim counter, claimed when the current item
    // starts and decoded once its last k-block is issued (both off the
    // k-block path).  Claimed items go to the MMA issuer and the drain
    // through a queue in shared memory.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool ok = true;
      int item = (int)blockIdx.x < total ? (int)blockIdx.x : -1;
      Item it = decode_tm<GATEUP>(d, sv.rows, sv.wid, sv.items, nseg, item < 0 ? 0 : item);
      for (int u = 0; ok; ++u) {
        const int qs = u % Q;
        if (u >= Q && !mbar_wait(smem_u32(&ifree[qs]), (uint32_t)(((u / Q) - 1) & 1), abort_flag,
                                 &st->status)) {
          ok = false;
          break;
        }
        iq[qs] = item;
        mbar_arrive(smem_u32(&iready[qs]));  // releases iq[qs]
        if (item < 0) break;
        const int claim = atomicAdd(next_item, 1);  // used after the k-loop
        const int nbox = GATHER ? 0 : (it.n + kTmBox - 1) / kTmBox;
        const uint32_t tx = (uint32_t)(nbox * kTmBoxBytes + C::kBBytes);
        // weight rows of the 256-row N tile: GATEUP gate rows then up rows of
        // the feature block; else 256 consecutive output rows
        const int w0 = it.wrow, w1 = GATEUP ? it.wrow + d.F : it.wrow + 128;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, &st->status)) {
            ok = false;
            break;
          }
          uint8_t* sb = stage_base + stage * C::kStageBytes;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, tx);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(smem_u32(sb + b * kTmBoxBytes), &map_x, kb * kBK, it.r0 + b * kTmBox, fb);
          tma_load_2d(smem_u32(sb + C::kABytes), &map_w, kb * kBK, w0, fb);
          tma_load_2d(smem_u32(sb + C::kABytes + C::kBBytes / 2), &map_w, kb * kBK, w1, fb);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        const int nxt = (int)gridDim.x + claim;
        item = nxt < total ? nxt : -1;
        if (item >= 0) it = decode_tm<GATEUP>(d, sv.rows, sv.wid, sv.items, nseg, item);
      }
      if (!ok) {  // let every issued copy land before the CTA exits
        for (int s2 = 0; s2 < C::kStages; ++s2)
          if ((armed >> s2) & 1u) {
            const unsigned long long t0 = global_ns();
            while (!mbar_try(smem_u32(&full[s2]), (armed_par >> s2) & 1u) &&
                   global_ns() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t last_bar = 0, last_par = 0;
      bool ok = true, issued = false;
      const uint32_t idesc = idesc_bf16(C::kRows, C::kN);
      for (int u = 0; ok; ++u) {
        const int qs = u % Q;
        if (!mbar_wait(smem_u32(&iready[qs]), (uint32_t)((u / Q) & 1), abort_flag, &st->status)) {
          ok = false;
          break;
        }
        const int item = iq[qs];
        mbar_arrive(smem_u32(&ifree[qs]));
        if (item < 0) break;
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, abort_flag, &st->status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem + acc * C::kAccCols;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, &st->status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * C::kStageBytes);
          const uint32_t sb = sa + C::kABytes;
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks) {
            const uint32_t koff = ks * 32;
            mma_bf16(dcol, sdesc(sa + koff), sdesc(sb + koff), idesc, (kb | ks) != 0);
          }
          mma_commit(smem_u32(&empty[stage]));
          last_bar = smem_u32(&empty[stage]);
          last_par = phase;
          issued = true;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull[acc]));
        last_bar = smem_u32(&tfull[acc]);
        last_par = acc_phase;
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok && issued) {
        const unsigned long long t0 = global_ns();
        while (!mbar_try(last_bar, last_par) && global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (GATHER && warp >= 2 + kEpiWarps) {
    // ------------------------------------------------------------ row gather
    // Thread g copies chunk row g (128 bytes of K per k-block, eight 16-byte
    // cp.async) to its swizzled place in the stage's token tile.  A stage's
    // copies are signalled kGatherDepth - 1 stages later: the thread waits for
    // its own copies (cp.async.wait_group), makes them visible to the tensor
    // core's proxy and arrives on the stage's full barrier.
    const int g = threadIdx.x - 32 * (2 + kEpiWarps);
    const uint32_t row_off = (uint32_t)((g >> 3) * 1024 + (g & 7) * 128);
    int stage = 0, pending = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto signal_oldest = [&](int depth_left) {
      if (depth_left == 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
      else asm volatile("cp.async.wait_group %0;" ::"n"(kGatherDepth - 1) : "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // unsignalled stages: stage - pending .. stage - 1 (stage already advanced)
      const int old = (stage - pending + 4 * C::kStages) % C::kStages;
      mbar_arrive(smem_u32(&full[old]));
      --pending;
    };
    for (int u = 0; ok; ++u) {
      const int qs = u % Q;
      if (!mbar_wait(smem_u32(&iready[qs]), (uint32_t)((u / Q) & 1), abort_flag, &st->status)) break;
      const int item = iq[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ifree[qs]));
      if (item < 0) break;
      const Item it = decode_tm<GATEUP>(d, sv.rows, sv.wid, sv.items, nseg, item);
      const bool active = g < it.n;
      const char* src =
          reinterpret_cast<const char*>(xsrc + (size_t)(active ? __ldg(rowslot + it.r0 + g) / d.kk : 0) * d.H);
      for (int kb = 0; kb < nk; ++kb) {
        int good = 1;
        if (lane == 0) good = mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, &st->status);
        if (!__shfl_sync(0xffffffffu, good, 0)) {
          ok = false;
          break;
        }
        if (active) {
          const uint32_t dst = smem_u32(stage_base + stage * C::kStageBytes) + row_off;
          const char* s0 = src + kb * kBK * 2;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + ((c ^ (g & 7)) << 4)),
                         "l"(s0 + 16 * c)
                         : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        ++pending;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (pending == kGatherDepth) signal_oldest(1);
      }
    }
    while (pending > 0) {  // the last stages (or, on an abort, let the copies land)
      if (ok) signal_oldest(0);
      else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        pending = 0;
      }
    }
  } else if (COMBINE && warp >= 2 + kEpiWarps) {
    // ------------------------------------------------------------ combine
    // Each warp pops (token, feature block) entries in order and combines
    // that block of the token into hidden.  It stops once every drain warp
    // has finished and the ring holds nothing more.
    const unsigned long long t_begin = global_ns();
    for (;;) {
      int slot = 0;
      if (lane == 0) slot = atomicAdd(&cq_ctl[1], 1);
      slot = __shfl_sync(0xffffffffu, slot, 0);
      int v = -1;
      if (lane == 0) {
        const unsigned long long t0 = global_ns();
        for (uint32_t it_ = 1;; ++it_) {
          v = cq[slot % kCombineQueue];
          if (v >= 0) {
            cq[slot % kCombineQueue] = -1;  // frees the entry for the push kCombineQueue later
            break;
          }
          // every push happens before its drain warp counts itself done, so
          // with all drains done the pushed count is final
          if (*(volatile int*)&cq_ctl[2] == kEpiWarps && *(volatile int*)&cq_ctl[0] <= slot) break;
          if ((it_ & 255) == 0 && (*abort_flag || global_ns() - t0 > kWaitLimitNs)) {
            if (!*abort_flag) {
              *abort_flag = 1;
              atomicCAS(&st->status, EB_OK, EB_ERR_TIMEOUT);
            }
            break;
          }
        }
      }
      v = __shfl_sync(0xffffffffu, v, 0);
      if (v < 0) break;
      __threadfence();  // the arrivals the drain counted before the reads of y
      const int nfb = d.H / C::kFeat;
      combine_token(d, st, v / nfb, (v % nfb) * C::kFeat, lane, gate, out, hidden);
    }
    (void)t_begin;
  } else {
    // ------------------------------------------------------------ drain
    // warp w reads TMEM lanes (tokens) 32 (w % 4) .. +31; with 8 warps two
    // warps share a lane quarter and split its 32-column blocks.
    const int q = warp & 3;
    const int cgrp = (warp - 2) >> 2;
    constexpr int kGroups = kEpiWarps / 4;
    constexpr int kBlocks = C::kFeat / 32;  // 32-feature blocks of an item's output
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = 0;; ++u) {
      const int qs = u % Q;
      if (!mbar_wait(smem_u32(&iready[qs]), (uint32_t)((u / Q) & 1), abort_flag, &st->status)) break;
      const int item = iq[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ifree[qs]));
      if (item < 0) break;
      const Item it = decode_tm<GATEUP>(d, sv.rows, sv.wid, sv.items, nseg, item);
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, &st->status)) break;
      tc_fence_after();
      const int row = q * 32 + lane;  // token row within the item
      const bool live = row < it.n;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + acc * C::kAccCols;
      // GEMM 2 stores each row at its (token, slot) position
      const int orow_idx = GATEUP ? it.r0 + row : (live ? __ldg(rowslot + it.r0 + row) : 0);
      __nv_bfloat16* orow = out + (size_t)orow_idx * NOUT + it.f0;
      // a lane quarter past the chunk's last token has nothing to drain
      const int b_end = q * 32 < it.n ? kBlocks : 0;
      for (int b = cgrp; b < b_end; b += kGroups) {
        float g[32];
        uint32_t packed[16];
        if (GATEUP) {
          float uu[32];
          tmem_ld32x2(tbase + b * 32, tbase + 128 + b * 32, g, uu);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = g[2 * i] / (1.f + expf(-g[2 * i])) * uu[2 * i];
            const float a1 = g[2 * i + 1] / (1.f + expf(-g[2 * i + 1])) * uu[2 * i + 1];
            packed[i] = pack_bf16x2(a0, a1);
          }
        } else {
          tmem_ld32(tbase + b * 32, g);
#pragma unroll
          for (int i = 0; i < 16; ++i) packed[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
        }
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + b * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1;
      }
      if constexpr (COMBINE) {
        // the accumulator is released; count this thread's stored share
        int tok = 0;
        bool last = false;
        if (live) {
          tok = orow_idx / d.kk;
          int32_t* cnt = arrive + (size_t)tok * (d.H / C::kFeat) + it.f0 / C::kFeat;
          __threadfence();  // the stores of y above before the count
          last = atomicAdd(cnt, 1) == d.kk * kGroups - 1;
          if (last) *cnt = 0;  // no other arrival on it in this launch
        }
        if (last) {  // hand the block to the combine warps
          __threadfence();  // every counted share before the hand-over
          const int slot = atomicAdd(&cq_ctl[0], 1);
          const unsigned long long t0 = global_ns();
          for (uint32_t it_ = 1; cq[slot % kCombineQueue] >= 0; ++it_)  // ring full: wait
            if ((it_ & 255) == 0 && (*abort_flag || global_ns() - t0 > kWaitLimitNs)) {
              if (!*abort_flag) {
                *abort_flag = 1;
                atomicCAS(&st->status, EB_OK, EB_ERR_TIMEOUT);
              }
              break;
            }
          cq[slot % kCombineQueue] = tok * (d.H / C::kFeat) + it.f0 / C::kFeat;
        }
      }
    }
    if constexpr (COMBINE) {  // this drain warp pushes nothing more
      __syncwarp();
      __threadfence_block();
      if (lane == 0) atomicAdd(&cq_ctl[2], 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"((uint32_t)C::kTmemCols));
  }
}


// ---------------------------------------------------------------------------
// Router projection: scores = h W_r^T in float32 for the micro-batches that
// route this step, each with the router of its current layer ([EB] §2.1:
// W_l, I_l = topk(G(h'_l)), with a linear scorer).  One CTA per (micro-batch,
// 128-token chunk): 128 tokens are the MMA's M side, the E router rows its N
// side (E a multiple of 16, at most 256), K = H in 64-element k-blocks fed by
// TMA through a 4-stage ring; the accumulator (128 lanes x E columns) is
// drained to [token][expert] float32 rows.
// ---------------------------------------------------------------------------

constexpr int kRouterThreads = 192;  // producer, MMA issuer, 4 drain warps
constexpr int kRouterStages = 4;
constexpr int kRouterABytes = 128 * kBK * 2;                 // 16 KiB
constexpr int kRouterStageBytes = kRouterABytes + 256 * kBK * 2;  // room for E = 256
constexpr int kRouterSmemBytes = kRouterStages * kRouterStageBytes + 1024 + 1024;

// map_h: hidden rows [rows, H] in boxes of 128 rows; map_r: router rows
// [layers * E, H] in boxes of E rows.  st == nullptr: stand-alone call, one
// block of T rows at layer 0; else the micro-batches in st->need_route at
// st->layer[j].  Row t of micro-batch j at layer l goes to out + j * mb_stride
// + l * layer_stride + t * E.
__global__ void __launch_bounds__(kRouterThreads, 1)
    k_router(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_r,
             int T, int H, int E, const State* __restrict__ st, float* __restrict__ out,
             long long mb_stride, long long layer_stride, int* __restrict__ status) {
  pdl_enter();
  const int c = blockIdx.x, j = blockIdx.y;
  int l = 0;
  if (st) {
    if (!((st->need_route >> j) & 1u)) return;
    l = st->layer[j];
  }
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRouterStages * kRouterStageBytes);
  uint64_t* full = bars;                  // [kRouterStages]
  uint64_t* empty = bars + kRouterStages;  // [kRouterStages]
  uint64_t* done = bars + 2 * kRouterStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = H / kBK;
  const uint32_t tmem_cols = E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
  int dummy = 0;
  int* stat = status ? status : &dummy;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRouterStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row0 = j * T + c * 128;  // first hidden row of the chunk
  const uint32_t tx = (uint32_t)(kRouterABytes + E * kBK * 2);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, stat)) {
          ok = false;
          break;
        }
        uint8_t* sb = smem + stage * kRouterStageBytes;
        const uint32_t fb = smem_u32(&full[stage]);
        mbar_expect_tx(fb, tx);
        tma_load_2d(smem_u32(sb), &map_h, kb * kBK, row0, fb);
        tma_load_2d(smem_u32(sb + kRouterABytes), &map_r, kb * kBK, l * E, fb);
        armed |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kRouterStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {
        for (int s2 = 0; s2 < kRouterStages; ++s2)
          if ((armed >> s2) & 1u) {
            const unsigned long long t0 = global_ns();
            while (!mbar_try(smem_u32(&full[s2]), (armed_par >> s2) & 1u) &&
                   global_ns() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      uint32_t last_bar = 0, last_par = 0;
      const uint32_t idesc = idesc_bf16(128, E);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, stat)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * kRouterStageBytes);
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          mma_bf16(tmem, sdesc(sa + ks * 32), sdesc(sa + kRouterABytes + ks * 32), idesc,
                   (kb | ks) != 0);
        mma_commit(smem_u32(&empty[stage]));
        last_bar = smem_u32(&empty[stage]);
        last_par = phase;
        issued = true;
        if (++stage == kRouterStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok) mma_commit(smem_u32(done));
      else if (issued) {
        const unsigned long long t0 = global_ns();
        while (!mbar_try(last_bar, last_par) && global_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // drain: warp w reads TMEM lanes 32 (w % 4) .. +31 = tokens of the chunk
    const int q = warp & 3;
    if (mbar_wait(smem_u32(done), 0, abort_flag, stat)) {
      tc_fence_after();
      const int t = c * 128 + q * 32 + lane;
      float* orow = out + (size_t)j * mb_stride + (size_t)l * layer_stride + (size_t)t * E;
      for (int cb = 0; cb < E; cb += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + cb, v);
        if (t < T) {
          const int n = min(32, E - cb);  // E is a multiple of 16
          for (int i = 0; i < n; i += 4)
            *reinterpret_cast<float4*>(orow + cb + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(tmem_cols));
  }
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* status, cudaStream_t s) {
  k_selftest_wait<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

int gemm_tc_smem_bytes(bool gateup) {
  return gateup ? Cfg<true>::kSmemBytes : Cfg<false>::kSmemBytes;
}

cudaError_t gemm_tc_prepare() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<true>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<false>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tm<true, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgTM<true>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tm<true, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgTM<true>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tm<false, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgTM<false>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_tm<false, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CfgTM<false>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_router, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kRouterSmemBytes);
  return e;
}

cudaError_t launch_gemm_tm(const Dims& d, const CtxDev& c, const Work& w, const TcMaps& maps,
                           int grid, cudaStream_t s, int which, const void* x_rows, void* combine_into) {
  const bool gather = x_rows != nullptr;
  const int32_t* rowslot = w.rowslot;
  const __nv_bfloat16* none = nullptr;
  int32_t* no_count = nullptr;
  const float* no_gate = nullptr;
  __nv_bfloat16* no_hidden = nullptr;
  if (which == 1 && gather)
    return launch_pdl(k_gemm_tm<true, true, false>, dim3(grid), dim3(kThreads + 32 * kGatherWarps),
                      CfgTM<true>::kSmemBytes, s, 1, maps.w_gateup, maps.w_gateup, d, c.st,
                      (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                      (const int32_t*)w.seg_items1, w.gemm_next, rowslot,
                      static_cast<const __nv_bfloat16*>(x_rows), static_cast<__nv_bfloat16*>(w.act),
                      no_count, no_gate, no_hidden);
  if (which == 1)
    return launch_pdl(k_gemm_tm<true, false, false>, dim3(grid), dim3(kThreads),
                      CfgTM<true>::kSmemBytes, s, 1, maps.w_gateup, maps.A32, d, c.st,
                      (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                      (const int32_t*)w.seg_items1, w.gemm_next, rowslot, none,
                      static_cast<__nv_bfloat16*>(w.act), no_count, no_gate, no_hidden);
  if (combine_into)
    return launch_pdl(k_gemm_tm<false, false, true>, dim3(grid), dim3(kThreads + 32 * kCombineWarps),
                      CfgTM<false>::kSmemBytes, s, 1, maps.w_down, maps.act32, d, c.st,
                      (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                      (const int32_t*)w.seg_items2, w.gemm_next + 1, rowslot, none,
                      static_cast<__nv_bfloat16*>(w.y), c.arrive, (const float*)w.gate,
                      static_cast<__nv_bfloat16*>(combine_into));
  return launch_pdl(k_gemm_tm<false, false, false>, dim3(grid), dim3(kThreads),
                    CfgTM<false>::kSmemBytes, s, 1, maps.w_down, maps.act32, d, c.st,
                    (const int32_t*)w.seg_rows, (const int32_t*)w.seg_wid,
                    (const int32_t*)w.seg_items2, w.gemm_next + 1, rowslot, none,
                    static_cast<__nv_bfloat16*>(w.y), no_count, no_gate, no_hidden);
}

cudaError_t launch_router(const CUtensorMap& map_h, const CUtensorMap& map_r, int T, int H, int E,
                          int n_mb, const State* st, float* out, long long mb_stride,
                          long long layer_stride, int* status, cudaStream_t s) {
  return launch_pdl(k_router, dim3((T + 127) / 128, n_mb), dim3(kRouterThreads),
                    (size_t)kRouterSmemBytes, s, 1, map_h, map_r, T, H, E, st, out, mb_stride,
                    layer_stride, status);
}

cudaError_t launch_gemm_tc(const Dims& d, const CtxDev& c, const Work& w, const TcMaps& maps,
                           int grid, cudaStream_t s, int which) {
  if (which == 1)
    return launch_pdl(k_gemm_tc<true>, dim3(grid), dim3(kThreads), Cfg<true>::kSmemBytes, s, 1,
                      maps.w_gateup, maps.A, d, c.st, (const int32_t*)w.seg_rows,
                      (const int32_t*)w.seg_wid, (const int32_t*)w.seg_items1,
                      (const int32_t*)w.rowslot, static_cast<__nv_bfloat16*>(w.act));
  return launch_pdl(k_gemm_tc<false>, dim3(grid), dim3(kThreads), Cfg<false>::kSmemBytes, s, 1,
                    maps.w_down, maps.act, d, c.st, (const int32_t*)w.seg_rows,
                    (const int32_t*)w.seg_wid, (const int32_t*)w.seg_items2,
                    (const int32_t*)w.rowslot, static_cast<__nv_bfloat16*>(w.y));
}

}  // namespace eb

namespace eb {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in boxes of 64 columns x box_rows rows.
cudaError_t encode(CUtensorMap* map, const void* base, unsigned long long rows, int cols,
                   int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t make_tc_maps(const Dims& d, const Work& w, const void* w_gateup, const void* w_down,
                         TcMaps* maps) {
  const unsigned long long experts = (unsigned long long)d.L * d.Etot;
  cudaError_t e = encode(&maps->w_gateup, w_gateup, experts * 2 * d.F, d.H, kBM);
  if (e == cudaSuccess) e = encode(&maps->w_down, w_down, experts * d.H, d.F, kBM);
  if (e == cudaSuccess) e = encode(&maps->A, w.A, (unsigned long long)w.Rcap, d.H, kTcRows1);
  if (e == cudaSuccess) e = encode(&maps->act, w.act, (unsigned long long)w.Rcap, d.F, kTcRows2);
  if (e == cudaSuccess) e = encode(&maps->A32, w.A, (unsigned long long)w.Rcap, d.H, kTmBox);
  if (e == cudaSuccess) e = encode(&maps->act32, w.act, (unsigned long long)w.Rcap, d.F, kTmBox);
  return e;
}

cudaError_t make_router_maps(const void* hidden, long long rows, int H, const void* w_router,
                             int layers, int E, CUtensorMap* map_h, CUtensorMap* map_r) {
  cudaError_t e = encode(map_h, hidden, (unsigned long long)rows, H, 128);
  if (e == cudaSuccess) e = encode(map_r, w_router, (unsigned long long)layers * E, H, E);
  return e;
}

}  // namespace eb
