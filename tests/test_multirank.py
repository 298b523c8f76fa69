"""The multi-GPU path on CPU: two gloo ranks shard users by LPT, agree on the
plan, cover every user exactly once, and their per-shard results (fp64 oracle)
equal the whole batch's, so no data-path collective is needed. The max over
ranks used for timing is checked too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W
from oracle import rest_oracle as O
from shared_prefix_behavior_b200 import shard as S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _small_ragged():
    w = W.small_workload("f32", lengths=(40, 7, 23, 31, 12, 3), d=32, n_heads=4, n_layers=1, l_switch=0,
                         requests=[(0, 40, 3), (0, 11, 2), (1, 7, 1), (2, 23, 4), (3, 31, 2), (3, 5, 1),
                                   (4, 12, 2), (5, 3, 1)])
    return w, W.make_inputs(w, 61)


def _costs(w, inp):
    return S.user_costs(inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"], inp["cu_cands"], w.d, w.n_layers,
                        w.d_ff, w.K)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, inp = _small_ragged()
        plan = S.partition_users(_costs(w, inp), world)
        mine = plan[rank]
        rows, cu, ru, rc, cc, cand_rows, _ = S.shard_arrays(inp["cu_seqlens"], inp["req_user"], inp["req_cutoff"],
                                                            inp["cu_cands"], mine)
        sub = dict(inp, x=inp["x"][rows], ts=inp["ts"][rows], cu_seqlens=cu, req_user=ru, req_cutoff=rc,
                   cu_cands=cc, z=inp["z"][cand_rows])
        Hs, ys = O.rank_request(sub)
        # every rank must hold the same plan
        plans = [None] * world
        dist.all_gather_object(plans, plan)
        # timing reduction used by bench.py: max over ranks
        t = torch.tensor([float(rank + 1)])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), rows=rows, cand_rows=cand_rows, H=Hs, y=ys,
                 same=np.array([all(p == plan for p in plans)]), tmax=t.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_users_without_a_collective(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    w, inp = _small_ragged()
    H_all, y_all = O.rank_request(inp)
    seen_rows, seen_cands = [], []
    for r in range(world):
        res = np.load(tmp_path / f"rank{r}.npz")
        assert bool(res["same"][0])
        assert float(res["tmax"][0]) == float(world)
        np.testing.assert_allclose(res["H"], H_all[res["rows"]], rtol=0, atol=1e-12)
        np.testing.assert_allclose(res["y"], y_all[res["cand_rows"]], rtol=0, atol=1e-12)
        seen_rows += list(res["rows"])
        seen_cands += list(res["cand_rows"])
    assert sorted(seen_rows) == list(range(w.total_tokens))
    assert sorted(seen_cands) == list(range(w.total_cands))


def test_lpt_partition_is_balanced_and_deterministic():
    rng = np.random.default_rng(0)
    costs = rng.lognormal(0, 1, size=200)
    for world in (1, 2, 3, 8):
        plan = S.partition_users(costs, world)
        assert sorted(u for p in plan for u in p) == list(range(200))
        loads = [costs[p].sum() for p in plan]
        # LPT guarantee: max load <= (4/3 - 1/(3m)) OPT <= that bound of the mean lower bound or the largest item
        lower = max(costs.sum() / world, costs.max())
        assert max(loads) <= (4 / 3) * lower + 1e-9
        assert plan == S.partition_users(costs, world)


def test_user_costs_grow_with_length_and_candidates():
    c = S.user_costs([0, 10, 30, 60], [0, 1, 2, 2], [10, 20, 30, 15], [0, 1, 1, 5, 6], d=32, n_layers=1, d_ff=64)
    assert c[0] < c[1] < c[2]
    with pytest.raises(ValueError):
        S.partition_users([1.0], 0)
