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
    with mp.Manager() as mgr:
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
