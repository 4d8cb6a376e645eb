"""Oracle: SwiGLU experts, the gated combine and whole-stack token trajectories.

Test infrastructure only (parity checks, the smoke check, and the CPU
baseline and reference arm of the benchmark); nothing in the library's
product path calls it.

[EB] is the paper "EasyBalance: Cross-Layer Load Balancing in Distributed MoE
Inference".  All arithmetic is float64; values are rounded to the storage type
("bf16" or "f32") at the points where the library stores a tensor: the SwiGLU
activation, each expert output and the layer output.
"""
from __future__ import annotations

from typing import Callable, Sequence, Tuple

import numpy as np

from .routing import route


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even).

    bfloat16 keeps 8 significant bits: with x = f * 2^e, 0.5 <= |f| < 1, the
    result is rint(f * 2^8) * 2^(e-8).  Below the smallest normal (2^-126) the
    spacing stays 2^-133.  np.rint rounds halfway cases to even.
    """
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)
    e = np.maximum(e, -125)
    return np.ldexp(np.rint(np.ldexp(x, -e + 8)), e - 8)


def round_storage(x, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def silu(z) -> np.ndarray:
    """silu(z) = z / (1 + e^-z)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(x, w_gate, w_up, w_down, dtype: str) -> np.ndarray:
    """expert_i(x) of [EB] Eq. (1), read as the SwiGLU FFN of the evaluated
    models: y = W_down (silu(W_gate x) * (W_up x)).

    x [n, H], w_gate / w_up [F, H], w_down [H, F]; the activation and the output
    are rounded to the storage type.
    """
    x = np.asarray(x, dtype=np.float64)
    g = x @ np.asarray(w_gate, dtype=np.float64).T
    u = x @ np.asarray(w_up, dtype=np.float64).T
    a = round_storage(silu(g) * u, dtype)
    return round_storage(a @ np.asarray(w_down, dtype=np.float64).T, dtype)


ExpertGetter = Callable[[int, int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def moe_layer(h, idx, gate, layer: int, get_expert: ExpertGetter, E: int,
              n_shared: int, dtype: str, residual: bool = True) -> np.ndarray:
    """One MoE layer for a block of tokens.

    [EB] Eq. (1): MLP(h') = sum_{i in I_l} W_{l,i} * expert_i(h'), and §2.1
    h_{l+1} = h'_l + MLP(h'_l).  Shared experts (always on, weight 1.0) are
    added after the routed slots.  The sum runs over slots in order
    s = 0..k-1 (routed) then the shared experts, and is rounded once.

    h [n, H] storage values; idx/gate [n, k]; get_expert(l, e) returns
    (w_gate [F,H], w_up [F,H], w_down [H,F]) of expert e (e >= E: shared).
    """
    h = np.asarray(h, dtype=np.float64)
    idx = np.asarray(idx)
    n, k = idx.shape
    y = np.zeros((n, k, h.shape[1]), dtype=np.float64)
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        wg, wu, wd = get_expert(layer, int(e))
        y[rows, slots] = expert_ffn(h[rows], wg, wu, wd, dtype)
    acc = h.copy() if residual else np.zeros_like(h)
    for s in range(k):
        acc = acc + np.asarray(gate, dtype=np.float64)[:, s:s + 1] * y[:, s]
    for s in range(n_shared):
        wg, wu, wd = get_expert(layer, E + s)
        acc = acc + expert_ffn(h, wg, wu, wd, dtype)
    return round_storage(acc, dtype)


def array_expert_getter(w_gateup, w_down, F: int) -> ExpertGetter:
    """Expert getter over full weight arrays [L, E_tot, 2F, H] / [L, E_tot, H, F]
    (the first F rows of 2F are the gate projection, the next F the up one)."""
    def get(l, e):
        gu = np.asarray(w_gateup[l, e], dtype=np.float64)
        return gu[:F], gu[F:], np.asarray(w_down[l, e], dtype=np.float64)
    return get


def forward_tokens(h0, logits_fn: Callable[[int, int], np.ndarray], tokens: Sequence[Tuple[int, int]],
                   L: int, E: int, k: int, n_shared: int, dtype: str,
                   get_expert: ExpertGetter, renorm: bool = True,
                   residual: bool = True) -> np.ndarray:
    """Final hidden state of the given tokens after all L MoE layers.

    A token's trajectory h_0 -> h_1 -> ... -> h_L depends only on its own
    hidden state, its own router logits and the weights ([EB] Eq. (1); the
    attention module is taken as the identity).  Scheduling moves only *when*
    each (micro-batch, layer) runs ([EB] §4.1 and [EB-read] §2.1: scheduling
    changes neither I_l, W_{l,i} nor the aggregation), so the expected output
    of every schedule is this schedule-free layer-by-layer pass.

    h0: [n_tokens, H] storage values of the tokens; logits_fn(j, l) returns the
    [T, E] logits of micro-batch j at layer l; tokens lists (j, t).
    """
    h = np.asarray(h0, dtype=np.float64).copy()
    tokens = list(tokens)
    for l in range(L):
        rows = []
        for (j, t) in tokens:
            rows.append(np.asarray(logits_fn(j, l))[t])
        idx, gate = route(np.stack(rows).astype(np.float32), k, renorm)
        h = moe_layer(h, idx, gate, l, get_expert, E, n_shared, dtype, residual)
    return h
