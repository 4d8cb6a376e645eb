"""Seeded synthetic workloads for the cross-layer MoE step.

This module only draws random numbers: router logits with a per-layer expert
skew, initial hidden states and expert weights.  It holds none of the method's
arithmetic (no routing, no load folding, no scheduling, no expert math), so the
CPU oracle under ``oracle/`` and the CUDA library can both take their inputs
from it without sharing any code of the method.

Workload shapes follow the models the EasyBalance paper evaluates
("EasyBalance: Cross-Layer Load Balancing in Distributed MoE Inference",
§5 Models): Qwen3-30B-A3B (48 MoE layers, 128 experts, top-8, hidden 2048,
expert FFN 768) and Moonlight-16B-A3B (26 MoE layers, 64 routed + 2 shared
experts, top-6, hidden 2048, expert FFN 1408).  The paper measures on
LongBench's 13 tasks with trained weights; neither is available here, so
seeded Dirichlet / Zipf "task profiles" stand in for the tasks' routing skew
(the paper's Fig. 7 shows the skew is task- and layer-dependent) and weights
are random (below).

Logit recipes (noise is always N(0,1) per (micro-batch, layer, token, expert)):

* ``zipf_perm``      bias_l[e] = -s * ln(1 + perm_l[e]), one seeded expert
                     permutation per layer.
* ``dirichlet_layer`` bias_l[e] = ln max(pi_l[e], 1e-9), pi_l ~ Dir(alpha).
* ``task_profiles``  13 profiles; pi_{p,l} ~ Dir(alpha) per (profile, layer);
                     micro-batch j draws its profile p_j uniformly.
* ``sweep_profiles`` 13 profiles with alpha_p = 0.1 + 0.9 p / 12; for episode r
                     and layer l every micro-batch uses profile
                     floor((r L + l) / 16) mod 13 (the profile switches every
                     16 lock-step layer positions).
* ``zipf_rotating``  bias_l[e] = -s * ln(1 + rank_l[e]) where rank_l is one
                     seeded permutation rolled by floor(l / 4) * (E / D)
                     positions: the hot set moves by one virtual rank every
                     4 layers.

Router weights (for stacks whose logits are projected from the hidden state):
row e of layer l is N(0, (s_{l,e} / sqrt(H))^2) with s_{l,e} = 0.5 + 2.5
pi_{l,e} / max_e pi_{l,e} and pi_l ~ Dir(alpha) per layer, so experts with
larger rows win more often -- a per-layer routing skew -- while the scores
stay O(1) for hidden states of unit scale.

Weights: ``w_init="normal"`` draws N(0, w_std^2) (the stated N(0, 0.02) of
the tiny and Moonlight-shaped stacks); ``w_init="fan_in"`` draws
N(0, 1 / (3 fan_in)) per matrix -- the variance of a linear layer's default
initialisation -- for stacks whose description says only "random-init
weights" (Qwen3-shaped ones).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

BASE_SEED = 20260808

# stream tags keep the draws of different tensors independent
_TAG_LOGITS, _TAG_HIDDEN, _TAG_WEIGHTS, _TAG_PROFILE, _TAG_PROFILE_PICK, _TAG_ROUTER = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one synthetic cross-layer MoE workload."""
    name: str
    L: int            # MoE layers
    E: int            # routed experts per layer
    k: int            # experts per token (top-k)
    H: int            # hidden size
    F: int            # expert FFN width (SwiGLU inner size)
    D: int            # virtual EP ranks
    M: int            # micro-batches
    T: int            # tokens per micro-batch
    n_shared: int = 0  # always-on shared experts per layer (gate 1.0)
    dtype: str = "bf16"  # storage type of hidden states and weights
    m: int = 0        # minimum RunSet size (0: round(0.75 M))
    profile: str = "task_profiles"
    alpha: float = 0.2
    zipf_s: float = 1.2
    n_profiles: int = 13
    compute: bool = True  # False: routing and scheduling only (no expert FFN)
    w_init: str = "normal"  # "normal": N(0, w_std^2); "fan_in": N(0, 1/(3 fan_in))
    w_std: float = 0.02
    seed: int = BASE_SEED

    @property
    def m_default(self) -> int:
        return self.m if self.m > 0 else max(1, int(round(0.75 * self.M)))

    @property
    def E_tot(self) -> int:
        return self.E + self.n_shared

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # tiny fp32 stack: brute force over all 2^4 micro-batch subsets is cheap
    "tiny_f32": Workload("tiny_f32", L=4, E=16, k=2, H=128, F=256, D=4, M=4, T=64,
                         dtype="f32", m=3, profile="zipf_perm", zipf_s=1.2),
    # Moonlight-16B-A3B shape
    "moonlight_bf16": Workload("moonlight_bf16", L=26, E=64, k=6, H=2048, F=1408, D=8,
                               M=8, T=512, n_shared=2, profile="dirichlet_layer",
                               alpha=0.3),
    # Moonlight-16B-A3B shape with weights scaled by fan-in (N(0, 1/(3 fan_in))),
    # so that the full 26-layer chain stays finite in bf16
    "moonlight_fanin_bf16": Workload("moonlight_fanin_bf16", L=26, E=64, k=6, H=2048, F=1408,
                                     D=8, M=8, T=512, n_shared=2, profile="dirichlet_layer",
                                     alpha=0.3, w_init="fan_in"),
    # Qwen3-30B-A3B shape: the throughput workload
    "qwen3_bf16": Workload("qwen3_bf16", L=48, E=128, k=8, H=2048, F=768, D=8, M=8,
                           T=1024, profile="task_profiles", alpha=0.2, w_init="fan_in"),
    # routing + scheduling only sweep at the Qwen3-30B shape (D and M vary)
    "sweep": Workload("sweep", L=48, E=128, k=8, H=2048, F=768, D=8, M=8, T=256,
                      profile="sweep_profiles", compute=False),
    # long-context prefill at the Qwen3-30B shape
    "longctx_bf16": Workload("longctx_bf16", L=48, E=128, k=8, H=2048, F=768, D=8,
                             M=8, T=8192, profile="zipf_rotating", zipf_s=1.5, w_init="fan_in"),
    # small cases the oracle finishes in seconds; several GEMM tiles and a
    # ragged token tail (T not a multiple of 64 or 128)
    "small_bf16": Workload("small_bf16", L=6, E=16, k=4, H=256, F=384, D=4, M=4,
                           T=200, profile="task_profiles", alpha=0.3),
    "small_shared_bf16": Workload("small_shared_bf16", L=5, E=12, k=3, H=256, F=256,
                                  D=3, M=5, T=77, n_shared=2, profile="dirichlet_layer",
                                  alpha=0.3),
}


def get(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(x) & 0xFFFFFFFF for x in key])


def _profile_pis(w: Workload, alphas) -> np.ndarray:
    """Dirichlet expert-popularity vectors [n_profiles, L, E]."""
    out = np.empty((len(alphas), w.L, w.E), dtype=np.float64)
    for p, a in enumerate(alphas):
        for l in range(w.L):
            out[p, l] = _rng(w.seed, _TAG_PROFILE, p, l).dirichlet(np.full(w.E, a))
    return out


def logit_bias(w: Workload, episode: int = 0) -> np.ndarray:
    """Per-(micro-batch, layer, expert) logit bias [M, L, E] (float64)."""
    M, L, E = w.M, w.L, w.E
    bias = np.empty((M, L, E), dtype=np.float64)
    if w.profile == "zipf_perm":
        for l in range(L):
            perm = _rng(w.seed, _TAG_PROFILE, 0, l).permutation(E)
            bias[:, l, :] = -w.zipf_s * np.log1p(perm.astype(np.float64))
    elif w.profile == "dirichlet_layer":
        pis = _profile_pis(w, [w.alpha])[0]
        bias[:] = np.log(np.maximum(pis, 1e-9))[None]
    elif w.profile == "task_profiles":
        pis = _profile_pis(w, [w.alpha] * w.n_profiles)
        pick = _rng(w.seed, _TAG_PROFILE_PICK, episode).integers(0, w.n_profiles, size=M)
        for j in range(M):
            bias[j] = np.log(np.maximum(pis[pick[j]], 1e-9))
    elif w.profile == "sweep_profiles":
        alphas = [0.1 + 0.9 * p / 12.0 for p in range(w.n_profiles)]
        pis = _profile_pis(w, alphas)
        for l in range(L):
            p = ((episode * L + l) // 16) % w.n_profiles
            bias[:, l, :] = np.log(np.maximum(pis[p, l], 1e-9))[None]
    elif w.profile == "zipf_rotating":
        perm = _rng(w.seed, _TAG_PROFILE, 0, 0).permutation(E)
        for l in range(L):
            rank = np.roll(perm, (l // 4) * (E // w.D))
            bias[:, l, :] = -w.zipf_s * np.log1p(rank.astype(np.float64))
    else:
        raise ValueError(f"unknown profile {w.profile!r}")
    return bias


def logits(w: Workload, episode: int = 0, mbs: Optional[range] = None,
           layers: Optional[range] = None) -> np.ndarray:
    """Router logits [M, L, T, E] float32 (optionally a sub-block of them).

    Each (micro-batch, layer) block is drawn from its own stream, so any
    sub-block can be regenerated alone.
    """
    bias = logit_bias(w, episode)
    mbs = range(w.M) if mbs is None else mbs
    layers = range(w.L) if layers is None else layers
    out = np.empty((len(mbs), len(layers), w.T, w.E), dtype=np.float32)
    for a, j in enumerate(mbs):
        for b, l in enumerate(layers):
            noise = _rng(w.seed, _TAG_LOGITS, episode, j, l).standard_normal(
                (w.T, w.E), dtype=np.float32)
            out[a, b] = (noise + bias[j, l].astype(np.float32)[None, :])
    return out


def hidden(w: Workload, episode: int = 0, scale: float = 1.0) -> np.ndarray:
    """Initial hidden states h_0 [M, T, H] float32 drawn from N(0, scale^2).

    For bf16 workloads the caller converts to bfloat16 (the stored input).
    """
    out = np.empty((w.M, w.T, w.H), dtype=np.float32)
    for j in range(w.M):
        out[j] = _rng(w.seed, _TAG_HIDDEN, episode, j).standard_normal((w.T, w.H),
                                                                      dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def hidden_torch(w: Workload, episode: int = 0, scale: float = 1.0):
    """h_0 as a torch CPU tensor in the workload's storage type."""
    import torch
    t = torch.from_numpy(hidden(w, episode, scale))
    return t.to(torch.bfloat16) if w.dtype == "bf16" else t


def weights_torch(w: Workload, device="cpu"):
    """Expert weights as torch tensors on `device` (see the module docstring
    for the two initialisations).

    Returns (w_gateup [L, E_tot, 2F, H], w_down [L, E_tot, H, F]).  Along the
    2F axis the first F rows are the gate projection and the next F the up
    projection.  Experts E..E_tot-1 of each layer are the shared experts.
    Each layer is drawn from its own generator seeded by (seed, layer), so the
    same device type reproduces the same values.
    """
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Et = w.E_tot
    if w.w_init == "fan_in":
        std_gu, std_dn = (3.0 * w.H) ** -0.5, (3.0 * w.F) ** -0.5
    else:
        std_gu = std_dn = w.w_std
    gu = torch.empty((w.L, Et, 2 * w.F, w.H), dtype=dt, device=device)
    dn = torch.empty((w.L, Et, w.H, w.F), dtype=dt, device=device)
    for l in range(w.L):
        g = torch.Generator(device=device)
        g.manual_seed((w.seed * 1000003 + _TAG_WEIGHTS * 7919 + l) & 0x7FFFFFFFFFFF)
        gu[l] = (torch.randn((Et, 2 * w.F, w.H), generator=g, device=device,
                             dtype=torch.float32) * std_gu).to(dt)
        dn[l] = (torch.randn((Et, w.H, w.F), generator=g, device=device,
                             dtype=torch.float32) * std_dn).to(dt)
    return gu, dn


def router_torch(w: Workload, device="cpu"):
    """Router weights [L, E, H] in the workload's storage type (see the module
    docstring); each layer from its own generator seeded by (seed, layer)."""
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    pis = _profile_pis(w, [w.alpha])[0]  # [L, E]
    out = torch.empty((w.L, w.E, w.H), dtype=dt, device=device)
    for l in range(w.L):
        s = 0.5 + 2.5 * pis[l] / pis[l].max()
        g = torch.Generator(device=device)
        g.manual_seed((w.seed * 1000003 + _TAG_ROUTER * 7919 + l) & 0x7FFFFFFFFFFF)
        rows = torch.randn((w.E, w.H), generator=g, device=device, dtype=torch.float32)
        scale = torch.tensor(s / np.sqrt(w.H), dtype=torch.float32, device=device)[:, None]
        out[l] = (rows * scale).to(dt)
    return out
