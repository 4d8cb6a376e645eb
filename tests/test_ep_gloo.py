"""Expert parallelism over real ranks, host plumbing on CPU: two gloo ranks
run the plan of ``cross_layer_expert_b200.ep`` ([EB] §2.2) for whole
Algorithm-1 episodes.

Each rank routes only its token shard (the oracle's routing stands in for
``eb_route`` on the rank's GPU), the ranks all-reduce their expert counts,
and each runs the scheduler on the summed counts (the oracle's scheduler
stands in for ``eb_schedule``).  Checked: every rank reaches the same RunSet
at every step, and it equals the single-process oracle episode over all
tokens; the dispatch all-to-all delivers to each rank exactly the (token,
slot) rows of its experts, and the combine all-to-all returns every row to
where it came from.  Nothing here needs a GPU.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, policy):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    from cross_layer_expert_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.get("small_bf16").replace(D=world)
        logits = synth.logits(wl)
        t0, t1 = ep.token_shard(wl.T, rank, world)
        owner = ep.expert_owner(wl.E, world)

        def route_counts(j, l):  # this rank's shard only
            idx, _ = oracle.route(logits[j, l, t0:t1], wl.k)
            return oracle.histogram(idx, wl.E)

        def fold(h):
            return oracle.loads(h, world)

        def choose(pending, w):
            return oracle.schedule.schedule(policy, pending, w, wl.m_default)

        layer = [0] * wl.M
        pending = list(range(wl.M))
        need = list(range(wl.M))
        cache, steps = {}, []
        while pending:
            run = ep.schedule_step(route_counts, pending, layer, need, cache, fold, choose)
            steps.append({"runset": run, "layers": {j: layer[j] for j in run}})
            for j in run:
                layer[j] += 1
            pending = [j for j in range(wl.M) if layer[j] < wl.L]
            need = [j for j in run if layer[j] < wl.L]

        # dispatch and combine of one step's rows: micro-batch 0 at layer 0
        idx, _ = oracle.route(logits[0, 0, t0:t1], wl.k)
        tok = np.repeat(np.arange(t0, t1), wl.k)
        slot = np.tile(np.arange(wl.k), t1 - t0)
        expert = idx.reshape(-1)
        payload = torch.from_numpy(np.stack([tok, slot, expert, np.full_like(tok, rank)], 1))
        recv, recv_counts, order, send_counts = ep.exchange(payload, owner[expert], world)
        got = sorted(map(tuple, recv[:, :3].tolist()))
        # step 5's grouping of the received rows (all at layer 0 here) into
        # (layer, expert) segments for the expert FFN
        seg_order, seg_off, seg_layer, seg_expert = ep.segment_rows(
            np.zeros(recv.shape[0], dtype=np.int64), recv[:, 2].numpy())
        grouped = recv[:, 2].numpy()[seg_order]
        seg_ok = (bool(np.all(seg_layer == 0)) and bool(np.all(np.diff(seg_expert) > 0)) and
                  all(bool(np.all(grouped[seg_off[i]:seg_off[i + 1]] == seg_expert[i]))
                      for i in range(len(seg_expert))) and int(seg_off[-1]) == recv.shape[0])
        # the rows returned carry a mark of the rank that served them
        served = recv.clone()
        served[:, 3] = rank
        back = ep.exchange_back(served, recv_counts, order, send_counts)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"steps": [{"runset": s["runset"], "layers": {str(k): v for k, v in s["layers"].items()}}
                                 for s in steps],
                       "received": got, "recv_owner_ok": bool(np.all(owner[recv[:, 2].numpy()] == rank)),
                       "back_rows_ok": bool(torch.equal(back[:, :3], payload[:, :3])),
                       "back_served_by_owner": bool(np.all(back[:, 3].numpy() == owner[expert])),
                       "segments_ok": seg_ok}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("policy", [0, 1])
def test_ep_two_ranks_agree_with_single_process_oracle(tmp_path, policy):
    import oracle
    import synth
    from cross_layer_expert_b200 import ep
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), policy), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    wl = synth.get("small_bf16").replace(D=world)
    logits = synth.logits(wl)
    ref = oracle.run_episode(oracle.route_all(logits, wl.k, world)[3], policy, wl.m_default)
    for r in res:
        assert len(r["steps"]) == len(ref["steps"])
        for got, want in zip(r["steps"], ref["steps"]):
            assert got["runset"] == want["runset"]
            assert {int(k): v for k, v in got["layers"].items()} == want["layers"]
        assert r["recv_owner_ok"] and r["back_rows_ok"] and r["back_served_by_owner"]
        assert r["segments_ok"]
    # every (token, slot) of micro-batch 0 at layer 0 lands on its expert's owner exactly once
    idx, _ = oracle.route(logits[0, 0], wl.k)
    owner = ep.expert_owner(wl.E, world)
    want = {r: [] for r in range(world)}
    for t in range(wl.T):
        for s in range(wl.k):
            want[int(owner[idx[t, s]])].append((t, s, int(idx[t, s])))
    for r in range(world):
        assert [tuple(x) for x in res[r]["received"]] == sorted(want[r])


def test_segment_rows():
    from cross_layer_expert_b200 import ep
    order, off, lay, ex = ep.segment_rows([1, 0, 1, 0, 0], [3, 2, 3, 5, 2])
    assert order.tolist() == [1, 4, 3, 0, 2]
    assert off.tolist() == [0, 2, 3, 5] and lay.tolist() == [0, 0, 1] and ex.tolist() == [2, 5, 3]
    order, off, lay, ex = ep.segment_rows([], [])
    assert len(order) == 0 and off.tolist() == [0] and len(lay) == 0 and len(ex) == 0


def test_token_shards_and_owner_map():
    from cross_layer_expert_b200 import ep
    for T, world in [(200, 2), (77, 4), (5, 8), (1024, 8)]:
        spans = [ep.token_shard(T, r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        sizes = [b - a for a, b in spans]
        assert max(sizes) - min(sizes) <= 1
    assert ep.expert_owner(16, 4).tolist() == [0] * 4 + [1] * 4 + [2] * 4 + [3] * 4
    with pytest.raises(ValueError):
        ep.expert_owner(10, 4)
