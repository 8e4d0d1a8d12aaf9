"""The multi-rank logic of bench.py on CPU (gloo, world size 2): each rank
draws its own token batch while the weights are identical on every rank, the
timed duration is the max over ranks, and the reported value counts the
tokens of all ranks.  The data path has no collective: ranks are replicas."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from fine_grained_moe_fp32_b200.workloads import make_inputs, small_config

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_setup()
        assert (w, r, lr) == (world, rank, rank)
        cfg = small_config(T=16, d=128, E=8, k=2, I=64)
        x = make_inputs(cfg, seed=bench.shard_seed(0, rank), weights=False)["x"]
        w1 = make_inputs(cfg, seed=0)["w1"]
        xs = [torch.empty_like(x) for _ in range(world)]
        ws = [torch.empty_like(w1) for _ in range(world)]
        dist.all_gather(xs, x)
        dist.all_gather(ws, w1)
        ms = bench.max_over_ranks(10.0 + rank, world, "cpu")
        out[rank] = {"x_differs": not torch.equal(xs[0], xs[1]),
                     "w_same": torch.equal(ws[0], ws[1]), "ms": ms}
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_on_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        assert res[r]["x_differs"] and res[r]["w_same"]
        assert res[r]["ms"] == 11.0          # max over ranks, same on every rank


def test_whole_job_value_counts_all_ranks():
    import bench
    # 2 ranks x 128 tokens x 10 steps in 5 ms (slowest rank) = 512k tokens/s
    assert bench.whole_job_value(2, 128, 10, 5.0) == pytest.approx(512000.0)
    assert bench.whole_job_value(1, 128, 10, 5.0) == pytest.approx(256000.0)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def _loads_worker(rank, world, port, out):
    """Each rank routes its own tokens; the bias step of the replicas uses the
    loads summed over the group (fine_grained_moe_fp32_b200.moe.global_loads)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import numpy as np
    import bench
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200.workloads import make_inputs, small_config
    from oracle import moe_oracle as O

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T = 24 + 8 * rank                       # ranks may hold different batch sizes
        cfg = small_config(T=T, d=128, E=8, k=2, I=64)
        inp = make_inputs(cfg, seed=bench.shard_seed(0, rank))
        wts = make_inputs(cfg, seed=0)          # same router weights on every rank
        idx = O.route(inp["x"], wts["w_gate"], wts["bias"], cfg.k)["idx"]
        counts = torch.as_tensor(np.bincount(idx.ravel(), minlength=cfg.E), dtype=torch.int32)
        c_all, T_all = M.global_loads(counts, T, group=dist.group.WORLD)
        sizes = [None] * world
        dist.all_gather_object(sizes, idx.tolist())
        whole = np.concatenate([np.asarray(s) for s in sizes])
        out[rank] = {"T_all": T_all, "c_all": c_all.tolist(),
                     "c_whole": np.bincount(whole.ravel(), minlength=cfg.E).tolist(),
                     "T_whole": whole.shape[0],
                     "step": O.bias_update(wts["bias"], c_all.numpy(), 1e-3, T_all, cfg.k).tolist(),
                     "step_whole": O.bias_update(wts["bias"], np.bincount(whole.ravel(),
                                                 minlength=cfg.E), 1e-3, whole.shape[0],
                                                 cfg.k).tolist()}
    finally:
        dist.destroy_process_group()


def test_two_rank_bias_step_uses_global_loads_on_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_loads_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        assert res[r]["T_all"] == res[r]["T_whole"] == 24 + 32
        assert res[r]["c_all"] == res[r]["c_whole"]
        assert res[r]["step"] == res[r]["step_whole"]
    assert res[0]["step"] == res[1]["step"]      # every replica takes the same step


def _grads_worker(rank, world, port, out):
    """Every replica's weight gradients are summed; dx stays per replica."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from fine_grained_moe_fp32_b200 import moe as M

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = {name: torch.full((3, 4), float(rank + 1)) for name in M.WEIGHT_GRADS}
        g["dx"] = torch.full((2, 4), float(rank + 1))
        M.allreduce_grads(g)
        out[rank] = {"weights": [float(g[n].max()) for n in M.WEIGHT_GRADS] +
                     [float(g[n].min()) for n in M.WEIGHT_GRADS],
                     "dx": float(g["dx"].max())}
    finally:
        dist.destroy_process_group()


def test_two_rank_weight_gradient_allreduce_on_gloo():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_grads_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for r in range(world):
        assert all(v == 3.0 for v in res[r]["weights"])   # 1 + 2 on every rank
        assert res[r]["dx"] == float(r + 1)


def _ep_exchange_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from fine_grained_moe_fp32_b200 import ep_dist

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # fake handles: byte 0 names the owner's allocation; "x_recv" and
        # "y_recv" share one allocation (one handle, two offsets), as the
        # caching allocator may arrange; the fake opener's base shows the owner
        local = {"x_recv": (bytes([rank]) * 64, 16 * rank, 1000 + rank),
                 "y_recv": (bytes([rank]) * 64, 16 * rank + 4096, 1100 + rank),
                 "counts": (bytes([rank + 100]) * 64, 8, 2000 + rank)}
        calls = []

        def opener(h):
            calls.append(h[0])
            return 5000 + 100 * h[0]

        addrs, opened = ep_dist.exchange_pointers(local, opener=opener)
        out[rank] = {"addrs": addrs, "opened": opened, "calls": calls}
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ep_pointer_exchange_on_gloo(world):
    """Every rank gets every buffer's address in rank order: its own as it
    is, a peer's as the base of that peer's allocation (opened once per
    distinct handle) plus the buffer's offset."""
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_ep_exchange_worker, args=(world, port, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    for r in range(world):
        a = res[r]["addrs"]
        for s in range(world):
            if s == r:
                assert (a["x_recv"][s], a["y_recv"][s], a["counts"][s]) == \
                    (1000 + r, 1100 + r, 2000 + r)
            else:
                assert a["x_recv"][s] == 5000 + 100 * s + 16 * s
                assert a["y_recv"][s] == 5000 + 100 * s + 16 * s + 4096
                assert a["counts"][s] == 5000 + 100 * (s + 100) + 8
        peers = [s for s in range(world) if s != r]
        assert sorted(res[r]["calls"]) == sorted(peers + [s + 100 for s in peers])
        assert len(res[r]["opened"]) == 2 * (world - 1)
