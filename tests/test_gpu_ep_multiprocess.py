"""Expert parallelism across processes (ep_dist.EPGroup): W processes share
the one GPU of this machine, each a rank of a gloo group, and reach each
other's receive buffers through CUDA IPC.  The barriers are on the host after
a stream synchronisation, so no kernel ever waits on another process.  Each
rank's output must equal, bit for bit, the same rank's output from the
single-process emulation (moe.EPRanks) on the same inputs: the same kernels
on the same bytes, only the buffers now live in other processes."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from fine_grained_moe_fp32_b200 import ep_dist
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200.workloads import TINY, make_inputs

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    res = {"rank": rank}
    try:
        inp = make_inputs(TINY, device="cuda")
        xs = [inp["x"]] + [make_inputs(TINY, device="cuda", seed=1000 + r, weights=False)["x"]
                           for r in range(1, world)]
        g = ep_dist.EPGroup(inp, TINY.T)
        y1 = g(xs[rank]).clone()
        y2 = g(xs[rank]).clone()            # buffers reused: same answer
        torch.cuda.synchronize()
        res["status"] = M.device_status()
        ys = M.EPRanks(inp, world, TINY.T)(xs)
        torch.cuda.synchronize()
        res["equal_emulation"] = bool(torch.equal(y1.view(torch.int16), ys[rank].view(torch.int16)))
        res["equal_repeat"] = bool(torch.equal(y1.view(torch.int16), y2.view(torch.int16)))
        res["recv_rows"] = int(g.views["recv_offsets"][-1])
        g.close()
    finally:
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_processes_match_the_emulation_bit_for_bit(world, tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.terminate()
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    from fine_grained_moe_fp32_b200 import moe as M
    for r in res:
        assert r["status"] == M.MOE_OK
        assert r["equal_emulation"] and r["equal_repeat"]
        assert r["recv_rows"] > 0
