"""Expert parallelism over several GPUs: the host-side plan of one step.

[EB] §2.2 ("Expert Parallelism"): the experts of every MoE layer are spread
over the ranks, and each step moves every routed token to the rank of its
expert and back (the all-to-alls of Algorithm 1's Attn_RouteDispatch and
MoECompute_Combine, [EB] §4.2).  On one GPU the library simulates D ranks in
device memory; this module is the plan for R real GPUs, one process each,
with D = R.

Partition:
  * experts -- rank r owns experts [r E/R, (r+1) E/R) of every layer, the
    contiguous map of [EB] §5 ("evenly distributed"), now on real devices;
  * tokens  -- each micro-batch's T tokens are split into R contiguous shards,
    rank r routes and holds shard r (data-parallel attention and routing).

One step:
  1. every rank routes its shard of the micro-batches that route this step
     (``eb_route`` on its GPU) and counts tokens per expert: hist_r [M, E];
  2. one all-reduce (sum) of the int32 counts gives every rank the same
     hist [M, E] -- integer sums, so exact and independent of the order;
  3. every rank folds hist into loads w [M, R] and runs the same
     deterministic scheduler (``eb_loads``, ``eb_schedule``): all ranks reach
     the same RunSet with no further message;
  4. dispatch: each (token, slot) row of a RunSet micro-batch goes to the
     rank owning its expert (one all-to-all of row counts, then of rows);
  5. the owner runs its experts' SwiGLU FFN on the rows it received;
  6. combine: the outputs return along the reverse all-to-all, and the
     token's rank sums them in slot order.

Everything here is plumbing over ``torch.distributed``: the all-reduce of
counts, the all-to-alls of counts and rows, the agreement check, and the
grouping of received rows into (layer, expert) segments.  The routing,
scheduling and expert arithmetic are the callers' -- on a GPU the library's
kernels: ``eb_route`` / the step's routing, ``eb_loads``, ``eb_schedule``,
and for step 5 ``eb_expert_ffn`` over the segments ``segment_rows`` builds.
"""
from __future__ import annotations

from typing import Callable, List, Sequence, Tuple

import numpy as np


def token_shard(T: int, rank: int, world: int) -> Tuple[int, int]:
    """Token range [t0, t1) of a micro-batch that `rank` routes: contiguous
    shards whose sizes differ by at most one."""
    base, extra = divmod(T, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def expert_owner(E: int, world: int) -> np.ndarray:
    """Rank owning each expert under the contiguous map (E a multiple of world)."""
    if E % world:
        raise ValueError("E must be a multiple of the number of ranks")
    return np.repeat(np.arange(world, dtype=np.int64), E // world)


def allreduce_counts(hist_local, group=None):
    """Sum of every rank's expert counts (int32 tensor [M, E] or [E]); returns
    a new tensor, identical on every rank."""
    import torch.distributed as dist
    out = hist_local.clone()
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def same_on_all_ranks(value: int, group=None) -> bool:
    """True when every rank passes the same integer (e.g. a RunSet mask)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    mine = torch.tensor([int(value)], dtype=torch.int64)
    got = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(got, mine, group=group)
    return all(int(g.item()) == int(value) for g in got)


def schedule_step(route_counts: Callable[[int, int], np.ndarray], pending: Sequence[int],
                  layer: Sequence[int], need_route: Sequence[int], hist_cache: dict,
                  fold: Callable[[np.ndarray], np.ndarray],
                  choose: Callable[[List[int], dict], List[int]], group=None) -> List[int]:
    """Steps 1-3 on this rank.

    route_counts(j, l) -> int counts [E] of this rank's shard of micro-batch
    j at layer l; hist_cache holds the all-reduced counts of micro-batches
    routed in earlier steps and still waiting (keyed by j); fold(hist [E]) ->
    loads [R]; choose(pending, {j: loads}) -> RunSet.  Returns the RunSet,
    checked to be the same on every rank."""
    import torch
    need = sorted(need_route)
    if need:
        local = np.stack([np.asarray(route_counts(j, layer[j]), dtype=np.int64) for j in need])
        total = allreduce_counts(torch.from_numpy(local.astype(np.int32)), group).numpy()
        for a, j in enumerate(need):
            hist_cache[j] = total[a].astype(np.int64)
    w = {j: [int(x) for x in fold(hist_cache[j])] for j in sorted(pending)}
    run = sorted(choose(sorted(pending), w))
    mask = sum(1 << j for j in run)
    if not same_on_all_ranks(mask, group):
        raise RuntimeError("ranks disagree on the RunSet")
    return run


def exchange(rows, dest, world: int, group=None):
    """One all-to-all of rows: rows [n, ...] (a torch tensor) go to rank
    dest[i] (dest sorted ascending is not required).  Returns (received rows,
    received counts per source rank, the order in which this rank's rows were
    sent), so that ``exchange_back`` can return results to where they came
    from."""
    import torch
    import torch.distributed as dist
    dest = np.asarray(dest, dtype=np.int64)
    order = np.argsort(dest, kind="stable")
    send_counts = np.bincount(dest, minlength=world).astype(np.int64)
    sc = torch.from_numpy(send_counts)
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    recv_counts = rc.numpy().astype(np.int64)
    send = rows[torch.from_numpy(order)].contiguous()
    recv = rows.new_empty((int(recv_counts.sum()),) + tuple(rows.shape[1:]))
    dist.all_to_all_single(recv, send, output_split_sizes=recv_counts.tolist(),
                           input_split_sizes=send_counts.tolist(), group=group)
    return recv, recv_counts, order, send_counts


def exchange_back(results, recv_counts, order, send_counts, group=None):
    """The reverse all-to-all of ``exchange``: results [sum(recv_counts), ...]
    in received order return to their source ranks, and come back in the
    original order of the rows this rank sent."""
    import torch
    import torch.distributed as dist
    back = results.new_empty((int(np.sum(send_counts)),) + tuple(results.shape[1:]))
    dist.all_to_all_single(back, results.contiguous(),
                           output_split_sizes=[int(x) for x in send_counts],
                           input_split_sizes=[int(x) for x in recv_counts], group=group)
    out = torch.empty_like(back)
    out[torch.from_numpy(np.asarray(order))] = back
    return out


def segment_rows(layer, expert):
    """Groups received rows by (layer, expert) for the expert FFN of step 5.

    layer, expert: int arrays [n] of each received row.  Returns (order,
    seg_off, seg_layer, seg_expert): rows[order] lists the rows segment by
    segment (segments ascending by (layer, expert), rows of a segment in
    received order), segment i being rows seg_off[i] .. seg_off[i+1] of that
    list.  The FFN's output row q belongs to received row order[q]."""
    layer = np.asarray(layer, dtype=np.int64)
    expert = np.asarray(expert, dtype=np.int64)
    if len(layer) == 0:
        empty = np.zeros(0, dtype=np.int64)
        return empty, np.zeros(1, dtype=np.int64), empty, empty
    order = np.lexsort((np.arange(len(layer)), expert, layer))
    key = np.stack([layer[order], expert[order]], 1)
    starts = [0] + [q for q in range(1, len(order)) if (key[q] != key[q - 1]).any()]
    seg_off = np.array(starts + [len(order)], dtype=np.int64)
    return order, seg_off, key[starts, 0], key[starts, 1]

