"""Benchmark of the cross-layer MoE step (EasyBalance) on B200.

A bench "step" is one whole episode of Algorithm 1 on the Qwen3-30B-A3B-shaped
workload (48 MoE layers, 128 experts, top-8, hidden 2048, expert FFN 768,
D = 8 virtual ranks, M = 8 micro-batches x 1024 tokens): from reset until every
micro-batch has passed all 48 layers, each scheduler step running routing,
loads, the RunSet choice, permutation, the two grouped expert GEMMs and the
combine.  Throughput counts token-layer passes: M * T * L per episode (the
model-level rate, M * T tokens per episode, is printed beside it).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --sweep [--impl reference]   # routing + scheduling sweep, D x M

N > 1 (launched with torchrun) runs one independent replica per GPU: the path
has no exchange step on one GPU ("replicas only"); value = all ranks' tokens /
the slowest rank's time.  --impl reference times the CPU oracle (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cross-layer MoE step tokens/s at Qwen3-30B shape (1 B200); under-util 1−u"
UNIT = "token-layer passes/s"
POLICY_NAMES = {0: "cumutil", 1: "maxutil", 2: "lockstep", 3: "diffpeak"}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="qwen3_bf16")
    p.add_argument("--policy", default="maxutil", choices=list(POLICY_NAMES.values()))
    p.add_argument("--gemm", type=int, default=0,
                   help="expert-GEMM engine (include/eb.h EB_GEMM_*; 0: the library's default)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-under-util", action="store_true")
    p.add_argument("--no-router-mode", action="store_true",
                   help="skip the extra router-mode episode timing")
    p.add_argument("--no-policy-times", action="store_true",
                   help="skip timing an episode of every scheduling policy")
    p.add_argument("--layers", type=int, default=0,
                   help="override the workload's MoE layer count (small profiling cases)")
    p.add_argument("--sweep", action="store_true",
                   help="instead of the step benchmark: the routing + scheduling sweep at the "
                        "Qwen3-30B shape (D in 8..64, M in 4..32), 1-u per policy and the "
                        "routing / scheduler kernel time per step (one GPU, one JSON line)")
    p.add_argument("--sweep-episodes", type=int, default=4,
                   help="episodes per sweep point (the workload defines 43, about 2048 "
                        "lock-step steps; each episode's logits are drawn on the host)")
    p.add_argument("--sweep-episodes-m32", type=int, default=0,
                   help="episodes of the MaxUtil points at M = 32, whose exhaustive search "
                        "covers about 15.3M subsets per step (0: skip those points)")
    return p.parse_args()


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of every rank's x (all ranks call it, in the same order)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_config(wl, args, world: int) -> dict:
    """The workload description both arms print (same keys and values)."""
    weights = wl.L * wl.E_tot * 3 * wl.F * wl.H * (2 if wl.dtype == "bf16" else 4)
    return {"workload": f"{wl.name}: Qwen3-30B-A3B shape L={wl.L} E={wl.E} k={wl.k} "
                        f"H={wl.H} F={wl.F} D={wl.D} M={wl.M} T={wl.T}",
            "policy": args.policy, "m": wl.m_default, "step": "one Algorithm-1 episode",
            "tokens_per_step": wl.M * wl.T * wl.L, "model_tokens_per_step": wl.M * wl.T,
            "l2": (f"inputs larger than L2: {weights / 1e9:.0f} GB of expert weights resident; "
                   "each scheduler step streams the weights of every (layer, expert) it touches "
                   "(per-episode GEMM bytes in `kernels`)"),
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


def job_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (replicas do equal work, so weak scaling)."""
    return units_per_rank * world / (ms_max / 1e3)


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: int):
        self.gpu = gpu
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, sustained, source): the pool's
    measured figures when present, else the profiling recipe's fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0),
                d.get("bf16_tflops_sustained", 1400.0), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def ncu_traffic(name: str, alg_bytes_per_launch: float):
    """Per-launch DRAM bytes (read + write) of a kernel, from the committed
    ncu summary profiles/traffic.json: the measured DRAM bytes per algorithmic
    byte of captured launches, times this run's algorithmic bytes per launch.
    None when there is no summary for the kernel or its source file changed
    since the counters were taken (the summary records the file's SHA-256)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            e = json.load(f).get(name)
        if not e:
            return None
        with open(os.path.join(ROOT, e["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != e["source_sha256"]:
                return None
        return int(e["dram_bytes_per_alg_byte"] * alg_bytes_per_launch)
    except Exception:
        return None


# ------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local):
    import numpy as np
    import torch

    import cross_layer_expert_b200 as eb
    import synth
    from cross_layer_expert_b200 import build

    if rank == 0 or not os.path.exists(build.LIB):
        build.build()
    barrier(world)
    eb.load()
    wl = synth.get(args.workload)
    if args.layers:
        wl = wl.replace(L=args.layers)
    policy = {v: k for k, v in POLICY_NAMES.items()}[args.policy]
    dev = torch.device("cuda", torch.cuda.current_device())
    logits_np = synth.logits(wl)
    logits = torch.from_numpy(logits_np).to(dev)
    h0 = synth.hidden_torch(wl).to(dev)
    wgu, wdn = synth.weights_torch(wl, device=dev)
    torch.cuda.synchronize()

    def cfg_for(pol, compute=1):
        return eb.make_config(L=wl.L, E=wl.E, k=wl.k, H=wl.H, F=wl.F, D=wl.D, M=wl.M, T=wl.T,
                              n_shared=wl.n_shared, dtype=eb.DTYPE_BF16, policy=pol,
                              m=wl.m_default, compute=compute, gemm=args.gemm)

    # exact under-utilisation of every policy (routing + scheduling only)
    under = {}
    for pol, name in ([] if args.no_under_util else POLICY_NAMES.items()):
        c = eb.Context(cfg_for(pol, compute=0))
        c.eb_episode(logits, None, None, None)
        num, den, den_sep = c.eb_utilization()
        under[name] = round(1 - num / den, 6)
        under["separate"] = round(1 - num / den_sep, 6)
        c.close()

    ctx = eb.Context(cfg_for(policy))
    hidden = torch.empty_like(h0)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        hidden.copy_(h0)
        ctx.eb_episode(logits, hidden, wgu, wdn)
    assert ctx.eb_sync_status() == eb.EB_OK
    rows, _ = ctx.eb_trace()
    n_steps = rows.shape[0]
    # algorithmic bytes of one episode, per kernel (bf16 = 2 bytes)
    b = 2
    R = rows[:, 4].astype(np.int64)
    P_touch = rows[:, 5].astype(np.int64)
    alg = {
        "gemm_gateup": int((P_touch * 2 * wl.F * wl.H * b + R * (wl.H + wl.F) * b).sum()),
        "gemm_down": int((P_touch * wl.H * wl.F * b + R * (wl.F + wl.H) * b).sum()),
        # the RunSet's rows in, every permuted row out; per row the copy also
        # reads its pair's expert and rank and writes its position and the
        # row's (token, slot)
        "permute": int(sum(bin(int(m)).count("1") for m in rows[:, 0]) * wl.T * wl.H * b
                       + (R * (wl.H * b + 16)).sum()),
        "combine": int((R * (wl.H * b + 8)).sum()
                       + 2 * sum(bin(int(m)).count("1") for m in rows[:, 0]) * wl.T * wl.H * b),
        # every (micro-batch, layer) is routed once: fp32 logits in, indices,
        # gates and in-chunk ranks out, one count row per 64-token chunk
        # (written, then read back with the chunk offsets written)
        "route": int(wl.M * wl.L * (wl.T * (4 * wl.E + 12 * wl.k) + -(-wl.T // 64) * 12 * wl.E)),
        # indices in, the row of every (token, slot) and the token of every row out
        "positions": int((R * (4 + 4 + 4)).sum()),
    }
    # useful FLOPs of the expert GEMMs (rows x 2 H F per output pair)
    flops = {"gemm_gateup": int((R * 4 * wl.H * wl.F).sum()),
             "gemm_down": int((R * 2 * wl.H * wl.F).sum())}
    fused = ctx.eb_engines()[1] == eb.GEMM_TMC
    if fused:
        # GEMM 2 also combines: its bytes are the down GEMM's and the
        # combine's, less the combine re-reading y (y stays on chip or in L2
        # as far as the design goes)
        alg["gemm_down"] += alg.pop("combine") - int((R * wl.H * b).sum())

    # the headline: whole episodes, nothing between the kernels
    clocks = ClockSampler(local)
    launches0 = ctx.eb_launch_count()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        hidden.copy_(h0)
        ctx.eb_episode(logits, hidden, wgu, wdn)
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_stop)
    launches = ctx.eb_launch_count() - launches0
    assert ctx.eb_sync_status() == eb.EB_OK
    ms_max = max_over_ranks(ms_total, world)
    value = job_throughput(wl.M * wl.T * wl.L * args.steps, ms_max, world)

    # per-kernel times: a separate pass with CUDA events around every kernel
    k_prof = max(2, args.steps // 2)
    ctx.eb_profile(True)
    for _ in range(k_prof):
        hidden.copy_(h0)
        ctx.eb_episode(logits, hidden, wgu, wdn)
    prof = ctx.eb_profile_read()
    ctx.eb_profile(False)
    hbm, tf_burst, tf_sust, peak_src = measured_peaks()

    def floor_bound(k):
        """The binding roofline of kernel k: whichever of its bytes at the HBM
        peak and its useful FLOPs at the sustained tensor peak takes longer."""
        if k in flops and flops[k] / (tf_sust * 1e12) > alg[k] / (hbm * 1e9):
            return "tensor"
        return "hbm"

    kern = max((k for k in ("gemm_gateup", "gemm_down", "permute", "combine") if k in alg),
               key=lambda k: prof[k][0])
    kms, kl = prof[kern]
    alg_launch = alg[kern] * k_prof / max(1, kl)
    bound = floor_bound(kern)
    if bound == "tensor":
        achieved = flops[kern] * k_prof / (kms / 1e3) / 1e12
        roof = {"kernel": kern, "bound": "tensor", "achieved": round(achieved, 1), "peak": tf_sust,
                "unit": "TFLOP/s", "frac": round(achieved / tf_sust, 4),
                "peak_source": (peak_src + " dense bf16, sustained (the kernel runs inside a "
                                "long step)"),
                "flops_per_launch": int(flops[kern] * k_prof / max(1, kl)),
                "hbm_frac": round(alg[kern] * k_prof / (kms / 1e3) / 1e9 / hbm, 4)}
    else:
        achieved = alg[kern] * k_prof / (kms / 1e3) / 1e9
        roof = {"kernel": kern, "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(achieved / hbm, 4),
                "peak_source": (peak_src + " HBM copy bandwidth" if peak_src == "measured"
                                else "fallback 6650 GB/s")}
    roof.update({"traffic": ncu_traffic(kern, alg_launch), "alg_bytes_per_launch": int(alg_launch),
                 "avg_launch_ms": round(kms / max(1, kl), 5), "of": peak_src})
    kernels = {k: {"ms_per_episode": round(v[0] / k_prof, 4), "launches": v[1]}
               for k, v in prof.items()}
    for k in ("route", "positions", "permute", "gemm_gateup", "gemm_down", "combine"):
        if k in alg and prof[k][0] > 0:
            kernels[k]["GB_per_episode"] = round(alg[k] / 1e9, 3)
            kernels[k]["GBps"] = round(alg[k] * k_prof / (prof[k][0] / 1e3) / 1e9, 1)
            kernels[k]["frac_of_hbm"] = round(kernels[k]["GBps"] / hbm, 4)
            if k in flops:
                tfs = flops[k] * k_prof / (prof[k][0] / 1e3) / 1e12
                kernels[k]["useful_TFLOPs"] = round(tfs, 1)
                kernels[k]["frac_of_tensor_sustained"] = round(tfs / tf_sust, 4)
                kernels[k]["bound"] = floor_bound(k)
    kernels["note"] = ("per-kernel times from a separate pass with CUDA events around every "
                       "kernel; the headline pass has none")

    # every policy's episode time and GEMM weight bytes on the same inputs
    # ([EB] Table 3 / Fig. 2 compare policies by time): on one GPU a step
    # streams the weights of every (layer, expert) its RunSet touches, so the
    # schedule with the best 1 - u may move more bytes
    policy_ms = {}
    if not args.no_policy_times:
        for pol, name in POLICY_NAMES.items():
            pc = ctx if pol == policy else eb.Context(cfg_for(pol))
            hidden.copy_(h0)
            pc.eb_episode(logits, hidden, wgu, wdn)
            prow, _ = pc.eb_trace()
            reps = max(1, args.steps // 3)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                hidden.copy_(h0)
                pc.eb_episode(logits, hidden, wgu, wdn)
            e1.record(stream)
            torch.cuda.synchronize()
            ms_p = max_over_ranks(e0.elapsed_time(e1) / reps, world)
            num, den, _ = pc.eb_utilization()
            pt = prow[:, 5].astype(np.int64)
            policy_ms[name] = {"ms_per_episode": round(ms_p, 3), "scheduler_steps": int(prow.shape[0]),
                               "gemm_weight_GB": round(float((pt * 3 * wl.F * wl.H * b).sum()) / 1e9, 2),
                               "under_util": round(1 - num / den, 6)}
            if pc is not ctx:
                pc.close()

    # end to end: host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        lg_host = torch.from_numpy(logits_np).pin_memory()
        h_host = h0.cpu().pin_memory()
        out_host = torch.empty_like(h_host).pin_memory()
        lg_dev = torch.empty_like(logits)
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        k_e2e = max(1, args.steps // 2)
        for _ in range(k_e2e):
            lg_dev.copy_(lg_host, non_blocking=True)
            hidden.copy_(h_host, non_blocking=True)
            ctx.eb_episode(lg_dev, hidden, wgu, wdn)
            out_host.copy_(hidden, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": round(job_throughput(wl.M * wl.T * wl.L * k_e2e, ms_e2e, world), 1),
               "unit": UNIT,
               "h2d_bytes_per_step": int(lg_host.numel() * 4 + h_host.numel() * h_host.element_size()),
               "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
               "steps": k_e2e,
               "model_tokens_per_s": round(job_throughput(wl.M * wl.T * k_e2e, ms_e2e, world), 1)}
    ctx.close()

    # router mode (the routing scores projected from the hidden states on the
    # device, a data-dependent chain): episode time and the projection's share
    router_mode = None
    if not args.no_router_mode:
        w_router = synth.router_torch(wl, device=dev)
        rctx = eb.Context(cfg_for(policy))
        rctx.eb_set_router(w_router)
        for _ in range(2):
            hidden.copy_(h0)
            rctx.eb_episode(None, hidden, wgu, wdn)
        barrier(world)
        torch.cuda.synchronize()
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        k_r = max(1, args.steps // 2)
        r0.record(stream)
        for _ in range(k_r):
            hidden.copy_(h0)
            n_r = rctx.eb_episode(None, hidden, wgu, wdn)
        r1.record(stream)
        torch.cuda.synchronize()
        assert rctx.eb_sync_status() == eb.EB_OK
        ms_r = max_over_ranks(r0.elapsed_time(r1), world)
        rctx.eb_profile(True)
        hidden.copy_(h0)
        rctx.eb_episode(None, hidden, wgu, wdn)
        rprof = rctx.eb_profile_read()
        rctx.close()
        del w_router
        router_mode = {"value": round(job_throughput(wl.M * wl.T * wl.L * k_r, ms_r, world), 1),
                       "unit": UNIT, "ms_per_step": round(ms_r / k_r, 3), "scheduler_steps": n_r,
                       "router_ms_per_episode": round(rprof["router"][0], 4),
                       "router_tflops": round(2.0 * wl.M * wl.T * wl.L * wl.E * wl.H
                                              / (rprof["router"][0] / 1e3) / 1e12, 2)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, policy, logits_np, h0, wgu, wdn)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "model_tokens_per_s": round(value / wl.L, 1),
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": ("synthetic (seeded routing skew: " + wl.profile + "; random-init weights "
                     + ("N(0, 1/(3 fan_in))" if wl.w_init == "fan_in" else f"N(0, {wl.w_std}^2)") + ")"),
            "workload_layers": wl.L,
            "config": bench_config(wl, args, world), "scheduler_steps": n_steps,
            "e2e": e2e, "gpu_launches": int(launches), "roofline": roof,
            "cpu_baseline": cpu, "clocks": clk, "under_util": under, "kernels": kernels,
            "policy_ms": policy_ms, "router_mode": router_mode,
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ oracle

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def episode_loads(wl, logits_np):
    """Loads of every (micro-batch, layer) through the oracle (not timed)."""
    import numpy as np
    import oracle
    return np.stack([np.stack([oracle.loads(oracle.histogram(oracle.route(logits_np[j, l], wl.k)[0],
                                                             wl.E), wl.D) for l in range(wl.L)])
                     for j in range(wl.M)])


def oracle_sample(wl, policy, logits_np, h0_np, fetch_expert, n_tokens: int, route_tokens: int,
                  full_loads, ffn_layers: int):
    """Times the oracle on a bounded sample; returns (seconds per token-layer, detail).

    The expert weights the sampled tokens need are fetched before the clock
    starts (fetch_expert(l, e) -> float32 arrays); the oracle's own float64
    conversion and arithmetic are timed.
    """
    import numpy as np
    import oracle
    from oracle import moe as omoe

    t0 = time.perf_counter()
    for l in range(wl.L):
        idx, _ = oracle.route(logits_np[0, l, :route_tokens], wl.k)
        oracle.loads(oracle.histogram(idx, wl.E), wl.D)
    t_route = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.run_episode(full_loads, policy, wl.m_default)
    t_sched = time.perf_counter() - t0
    toks = [(j % wl.M, (j * 131) % wl.T) for j in range(n_tokens)]
    need = set()
    for l in range(ffn_layers):
        rows = np.stack([logits_np[j, l, t] for j, t in toks])
        need |= {(l, int(e)) for e in oracle.route(rows, wl.k)[0].reshape(-1)}
        need |= {(l, wl.E + s) for s in range(wl.n_shared)}
    weights = {key: fetch_expert(*key) for key in sorted(need)}
    t0 = time.perf_counter()
    omoe.forward_tokens(np.stack([h0_np[j, t] for j, t in toks]), lambda j, l: logits_np[j, l],
                        toks, ffn_layers, wl.E, wl.k, wl.n_shared, wl.dtype,
                        lambda l, e: weights[(l, e)])
    t_ffn = time.perf_counter() - t0
    per_tl = (t_route / (route_tokens * wl.L) + t_sched / (wl.M * wl.T * wl.L)
              + t_ffn / (n_tokens * ffn_layers))
    detail = (f"oracle on a bounded sample: routing+loads of {route_tokens} tokens x {wl.L} layers "
              f"({t_route:.2f}s), the full-episode schedule ({t_sched:.2f}s), expert FFN + combine "
              f"of {n_tokens} token(s) through {ffn_layers} layers ({t_ffn:.2f}s); time per "
              f"token-layer = sum of the three per-unit costs, extrapolated to the workload")
    return per_tl, detail, t_route + t_sched + t_ffn


def make_fetch(wgu, wdn, F):
    def fetch(l, e):
        gu = wgu[l, e].float().cpu().numpy()
        return gu[:F], gu[F:], wdn[l, e].float().cpu().numpy()
    return fetch


def cpu_baseline(wl, policy, logits_np, h0, wgu, wdn, n_tokens=4, ffn_layers=8):
    import numpy as np
    h0_np = h0.float().cpu().numpy().astype(np.float64)
    per_tl, detail, _ = oracle_sample(wl, policy, logits_np, h0_np, make_fetch(wgu, wdn, wl.F),
                                      n_tokens, 256, episode_loads(wl, logits_np), ffn_layers)
    return {"value": round(1.0 / per_tl, 2), "unit": UNIT, "cores": _blas_threads(),
            "kind": "oracle", "sample": detail + " (expert weights copied from the device)"}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import synth
    wl = synth.get(args.workload)
    policy = {v: k for k, v in POLICY_NAMES.items()}[args.policy]
    logits_np = synth.logits(wl)
    h0_np = synth.hidden(wl).astype(np.float64)
    if wl.dtype == "bf16":
        h0_np = torch.from_numpy(synth.hidden(wl)).to(torch.bfloat16).double().numpy()
    sg, sd = ((3.0 * wl.H) ** -0.5, (3.0 * wl.F) ** -0.5) if wl.w_init == "fan_in" else (wl.w_std,) * 2

    def fetch(l, e):  # one expert's weights drawn on the host
        g = torch.Generator().manual_seed((wl.seed * 7919 + l * 1009 + e) & 0x7FFFFFFF)
        gu = (torch.randn((2 * wl.F, wl.H), generator=g) * sg).to(torch.bfloat16).float().numpy()
        dn = (torch.randn((wl.H, wl.F), generator=g) * sd).to(torch.bfloat16).float().numpy()
        return gu[:wl.F], gu[wl.F:], dn

    times, sample_s, detail = [], [], ""
    full_loads = episode_loads(wl, logits_np)
    for i in range(args.warmup + args.steps):
        per_tl, detail, sec = oracle_sample(wl, policy, logits_np, h0_np, fetch, 1, 64, full_loads, 4)
        if i >= args.warmup:
            times.append(per_tl)
            sample_s.append(sec)
    per_tl = statistics.median(times)
    value = 1.0 / per_tl
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            # one step of the workload (a whole episode) is far beyond a
            # bounded CPU run: each timed step is a sample, and the step time
            # below is extrapolated from the sample's per-unit costs
            "ms_per_step": round(per_tl * wl.M * wl.T * wl.L * 1e3, 1),
            "ms_per_step_extrapolated": True,
            "sample_s_per_step": round(statistics.median(sample_s), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(wl, args, 1),
            "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": _blas_threads(),
                             "kind": "oracle", "sample": detail + " (host-drawn weights)"},
            "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SWEEP_M = (4, 8, 16, 32)
SWEEP_D = (8, 16, 32, 64)
SWEEP_NOTE = ("routing + scheduling only, Qwen3-30B shape: L=48 E=128 k=8 T=256, "
              "13 task profiles switching every 16 lock-step steps")


def sweep_jobs(args):
    """(M, D, policy, episodes) of the routing + scheduling sweep, in order.
    1 - u of a point pools its episodes: numerators and denominators are
    summed over them."""
    jobs = []
    for M in SWEEP_M:
        for D in SWEEP_D:
            for pol in POLICY_NAMES:
                n = args.sweep_episodes_m32 if (M == 32 and pol == 1) else args.sweep_episodes
                if n > 0:
                    jobs.append((M, D, pol, n))
    return jobs


def sweep_line(M, D, pol, n_ep, num, den, den_sep, steps, extra):
    line = {"M": M, "D": D, "policy": POLICY_NAMES[pol], "episodes": n_ep, "steps": steps,
            "under_util": round(1 - num / den, 6), "separate": round(1 - num / den_sep, 6),
            "num": num, "den": den, "den_sep": den_sep}
    line.update(extra)
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """The sweep on the GPU: for every (M, D) and policy, the exact 1 - u over
    the point's episodes, the no-balancing 1 - u (every micro-batch run
    separately) and the CUDA-event time per launch of the routing and
    scheduler kernels.  One JSON line per point, as it completes."""
    import torch

    import cross_layer_expert_b200 as eb
    import synth
    from cross_layer_expert_b200 import build

    build.build()
    eb.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    print(json.dumps({"sweep": SWEEP_NOTE, "impl": "ours", "gpu": torch.cuda.get_device_name(dev),
                      "unit_time": "step_us: whole steps (routing + scheduling; the host's "
                                   "per-episode completion checks included), CUDA events "
                                   "around the episodes; route_us / "
                                   "schedule_us: each kernel alone, CUDA events around every "
                                   "launch (launch gaps included)"}),
          flush=True)
    t0 = time.time()
    cache_M, episodes = None, []
    for M, D, pol, n_ep in sweep_jobs(args):
        base = synth.get("sweep", M=M)
        if cache_M != M:
            episodes = [torch.from_numpy(synth.logits(base, episode=r)).to(dev)
                        for r in range(max(args.sweep_episodes, args.sweep_episodes_m32))]
            cache_M = M
        wl = base.replace(D=D)
        ctx = eb.Context(eb.make_config(L=wl.L, E=wl.E, k=wl.k, H=wl.H, F=wl.F, D=wl.D, M=wl.M,
                                        T=wl.T, dtype=eb.DTYPE_BF16, policy=pol,
                                        m=wl.m_default, compute=0))
        ctx.eb_episode(episodes[0], None, None, None)  # warm-up
        # whole steps, no events between the kernels
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = 0
        e0.record(stream)
        for lg in episodes[:n_ep]:
            steps += ctx.eb_episode(lg, None, None, None)
        e1.record(stream)
        torch.cuda.synchronize()
        step_us = 1e3 * e0.elapsed_time(e1) / max(1, steps)
        # each kernel alone (events around every launch), and the exact
        # utilisation of every episode (the same episodes again)
        num = den = den_sep = 0
        ctx.eb_profile(True)
        for lg in episodes[:n_ep]:
            ctx.eb_episode(lg, None, None, None)
            a, b, c = ctx.eb_utilization()
            num, den, den_sep = num + a, den + b, den_sep + c
        prof = ctx.eb_profile_read()
        ctx.eb_profile(False)
        assert ctx.eb_sync_status() == eb.EB_OK
        ctx.close()
        rt, sc = prof["route"], prof["schedule"]
        sweep_line(M, D, pol, n_ep, num, den, den_sep, steps,
                   {"step_us": round(step_us, 2),
                    "route_us": round(1e3 * rt[0] / max(1, rt[1]), 2),
                    "schedule_us": round(1e3 * sc[0] / max(1, sc[1]), 2)})
    print(json.dumps({"sweep_done": True, "wall_s": round(time.time() - t0, 1)}), flush=True)


def _oracle_sweep_job(job):
    """One sweep point on the host with the oracle (a worker of a spawn pool)."""
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    from oracle import native
    M, D, pol, n_ep = job
    wl = synth.get("sweep", M=M, D=D)
    t = time.time()
    num = den = den_sep = steps = 0
    for r in range(n_ep):
        hist = oracle.route_all(synth.logits(wl, episode=r), wl.k, D)[2]
        ep = oracle.run_episode(oracle.loads(hist, D), pol, wl.m_default,
                                maxutil_impl=native.maxutil if M > 12 else None)
        num, den, den_sep = num + ep["num"], den + ep["den"], den_sep + ep["den_sep"]
        steps += len(ep["steps"])
    return job, (num, den, den_sep, steps, time.time() - t)


def run_reference_sweep(args):
    """The same sweep with the CPU oracle (routing, loads and Algorithm 1 in
    float64 / exact integers; the exhaustive MaxUtil in plain C), one point
    per worker of a spawn pool over the host's cores."""
    import multiprocessing as mproc
    cores = os.cpu_count() or 1
    print(json.dumps({"sweep": SWEEP_NOTE, "impl": "reference", "kind": "oracle", "cores": cores,
                      "unit_time": "s of one core per point"}), flush=True)
    from oracle import native
    native.build()
    t0 = time.time()
    # the heaviest points first, so the pool's tail is short
    jobs = sorted(sweep_jobs(args), key=lambda j: (j[0] == 32 and j[2] == 1, j[1]), reverse=True)
    with mproc.get_context("spawn").Pool(cores) as pool:
        for (M, D, pol, n_ep), (num, den, den_sep, steps, sec) in pool.imap_unordered(
                _oracle_sweep_job, jobs):
            sweep_line(M, D, pol, n_ep, num, den, den_sep, steps, {"oracle_s": round(sec, 2)})
    print(json.dumps({"sweep_done": True, "wall_s": round(time.time() - t0, 1)}), flush=True)


def main():
    args = parse()
    if args.sweep:
        (run_reference_sweep if args.impl == "reference" else run_sweep)(args)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
