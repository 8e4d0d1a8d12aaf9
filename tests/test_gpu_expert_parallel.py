"""Parity of the expert-parallel path (moe_ep_route / _dispatch / _experts /
_combine) with the fp64 oracle, on W ranks emulated by one process on one
GPU (each rank's calls are the ones a multi-GPU rank makes; its peers'
buffers are buffers of the same device).

Bit-exact: the routing (as moe_route), the receive layout of every rank
(segment starts and counts, and the receive row of every pair, against the
oracle's layout run on the GPU's own routing), and the rows the dispatch
writes (a byte copy; padding rows zero).  With one rank the whole layer must
equal moe_forward bit for bit (same kernels on the same rows).  The output
of every rank is checked against the oracle forward of its own tokens with
the bounds of the single-GPU forward tests."""
import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import (CONFIGS, MoEConfig, make_inputs, small_config, DECODE, TINY)
from oracle import moe_oracle as O
import parity_utils as PU

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ranks(cfg, W, T=None, device=DEV, bias=None):
    """Shared weights (seed 0) and one token batch per rank (rank r: seed 1000 + r)."""
    inp = make_inputs(cfg, T=T, device=device)
    if bias is not None:
        inp["bias"] = bias.to(device)
    xs = [inp["x"]] + [make_inputs(cfg, T=T, device=device, seed=1000 + r, weights=False)["x"]
                       for r in range(1, W)]
    return inp, [x.contiguous() for x in xs]


def _run(inp, xs, W, align=16):
    ep = M.EPRanks(inp, W, xs[0].shape[0], align)
    for b in ep.x_recv + ep.y_recv:          # stale bytes the dispatch must not leave behind
        b.fill_(float("nan"))
    ys = ep(xs)
    torch.cuda.synchronize()
    return ep, ys, M.device_status()


def _check_layout(ep, xs, align):
    """Layout and dispatched rows of every rank, bit for bit."""
    cfg, W = ep.cfg, ep.world
    El = cfg.E // W
    idx = [v["topk_idx"].cpu().numpy() for v in ep.views]
    L = O.ep_layout(idx, cfg.E, align)
    for r in range(W):
        v = ep.views[r]
        np.testing.assert_array_equal(v["recv_offsets"].cpu().numpy(), L["recv_offsets"][r])
        np.testing.assert_array_equal(v["recv_counts"].cpu().numpy(), L["recv_counts"][r])
        np.testing.assert_array_equal(v["remote_row"].cpu().numpy(), L["row"][r])
        n = int(L["recv_offsets"][r, El])
        assert n <= ep.recv_cap
        src = np.array([s for s, _ in L["src_of_row"][r]], dtype=np.int64)
        tok = np.array([t for _, t in L["src_of_row"][r]], dtype=np.int64)
        want = torch.zeros((n, cfg.d), dtype=torch.bfloat16, device=DEV)
        for s in range(W):
            rows = np.nonzero(src == s)[0]
            if rows.size:
                want[torch.as_tensor(rows, device=DEV)] = xs[s][torch.as_tensor(tok[rows],
                                                                               device=DEV)]
        got = ep.x_recv[r][:n]
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), f"rank {r} rows"
    return L


def _check_outputs(inp, xs, ys, ep, spec):
    cfg = inp["cfg"]
    host = PU.np_inputs(inp)
    for r, (x, y) in enumerate(zip(xs, ys)):
        inp_r = dict(host, x=x.cpu(), T=x.shape[0])
        idx = ep.views[r]["topk_idx"].cpu().numpy()
        ref = O.forward(inp_r, align=ep.align, idx=None)
        ties = PU.check_routing(idx, ref["keys"], ref["idx"], cfg.k)
        PU.check_probs(ep.views[r]["probs"], ref["probs"])
        if ties:
            ref = O.forward(inp_r, align=ep.align, idx=idx)
        routed_abs = O.unpermute_sum(np.abs(ref["y_perm"]), ref["row_of"], ref["w"],
                                     x.shape[0], cfg.k)
        PU.check_output(y, ref["y"], f"y of rank {r}", spec=spec, routed_abs=routed_abs)


def test_ep_one_rank_is_moe_forward_bit_for_bit():
    """One rank: the receive buffer is the permutation's x_perm and the layer
    output is moe_forward's, bit for bit."""
    inp, xs = _ranks(TINY, 1)
    ep, ys, st = _run(inp, xs, 1)
    assert st == M.MOE_OK
    layer = M.MoELayer(inp)
    y = layer(xs[0])
    torch.cuda.synchronize()
    v = M.workspace_views(layer.dims(xs[0].shape[0]), layer.workspace(xs[0].shape[0]))
    n = int(v["offsets"][-1])
    assert torch.equal(ep.views[0]["recv_offsets"], v["offsets"])
    assert torch.equal(ep.x_recv[0][:n].view(torch.int16), v["x_perm"][:n].view(torch.int16))
    assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))


EP_CASES = [
    ("tiny_W2", TINY, 2, None, 16),
    ("tiny_W4", TINY, 4, None, 16),
    ("tiny_W8", TINY, 8, None, 16),
    ("tiny_W4_align128", TINY, 4, None, 128),
    ("E16_T77_W4_ragged", small_config(T=77, d=256, E=16, k=4, I=128), 4, None, 16),
    ("E16_T40_W16_one_expert_per_rank", small_config(T=40, d=256, E=16, k=4, I=128), 16,
     None, 16),
    ("E32_k1_T300_W2_no_shared", MoEConfig("k1", T=300, d=256, E=32, k=1, S=0, I=128,
                                           bias="normal0.05"), 2, None, 16),
]


@pytest.mark.parametrize("name,cfg,W,T,align", EP_CASES, ids=[c[0] for c in EP_CASES])
def test_ep_parity_small(name, cfg, W, T, align):
    inp, xs = _ranks(cfg, W, T)
    ep, ys, st = _run(inp, xs, W, align)
    assert st == M.MOE_OK
    _check_layout(ep, xs, align)
    _check_outputs(inp, xs, ys, ep, spec=cfg in CONFIGS.values())


def test_ep_all_pairs_to_one_owner_fills_its_buffer():
    """A bias that makes every token of every rank pick experts 0..3, all on
    rank 0: rank 0 receives all W*T*k pairs (its capacity less the padding
    slack), the other ranks nothing."""
    cfg = small_config(T=64, d=256, E=16, k=4, I=128)
    bias = torch.zeros(16)
    bias[:4] = 10.0
    inp, xs = _ranks(cfg, 4, bias=bias)
    ep, ys, st = _run(inp, xs, 4)
    assert st == M.MOE_OK
    L = _check_layout(ep, xs, 16)
    assert L["recv_counts"][0].sum() == 4 * 64 * 4
    assert all(L["recv_counts"][r].sum() == 0 for r in range(1, 4))
    assert int(L["recv_offsets"][0, -1]) <= ep.recv_cap
    _check_outputs(inp, xs, ys, ep, spec=False)


def test_ep_empty_batches():
    cfg = small_config(T=0, d=256, E=16, k=4, I=128)
    inp, xs = _ranks(cfg, 4)
    ep, ys, st = _run(inp, xs, 4)
    assert st == M.MOE_OK
    for v in ep.views:
        assert int(v["recv_offsets"][-1]) == 0
    assert all(y.shape == (0, 256) for y in ys)


def test_ep_rejected_count_table_sends_nothing():
    """Rank 1 is handed a count table whose own entry is rank 0's counts: its
    plan rejects the table (it disagrees with rank 1's own counts), so rank 1
    sends and receives nothing and the status word reports INVALID_ARG."""
    cfg = small_config(T=64, d=256, E=16, k=4, I=128)
    inp, xs = _ranks(cfg, 2)
    ep = M.EPRanks(inp, 2, 64)
    ep.route(xs)
    bad = M.pointer_array([ep.views[0]["counts"], ep.views[0]["counts"]], DEV)
    torch.cuda.synchronize()
    assert not torch.equal(ep.views[0]["counts"], ep.views[1]["counts"])
    M.ep_dispatch(ep.dm, 2, 1, xs[1], bad, ep.x_recv_of, ep.ws[1])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_ERR_INVALID_ARG
    v = ep.views[1]
    assert (v["remote_row"] == -1).all() and (v["dst_row"] == -1).all()
    assert (v["recv_counts"] == 0).all() and (v["recv_offsets"] == 0).all()
    assert M.device_status() == M.MOE_OK


def test_ep_deterministic():
    inp, xs = _ranks(TINY, 4)
    ep = M.EPRanks(inp, 4, xs[0].shape[0])
    a = [y.clone() for y in ep(xs)]
    b = ep(xs)
    torch.cuda.synchronize()
    for u, w in zip(a, b):
        assert torch.equal(u.view(torch.int16), w.view(torch.int16))


def test_ep_full_size_decode_8_ranks():
    """The decode workload (T=128 per rank, d=5120, I=1408, 128 experts) on 8
    emulated ranks of 16 experts: every rank's layout and dispatched rows bit
    for bit, the output on a seeded sample of every rank's tokens against the
    per-token oracle, and against the single-GPU layer on the same tokens."""
    cfg = DECODE
    W = 8
    inp, xs = _ranks(cfg, W)
    ep, ys, st = _run(inp, xs, W)
    assert st == M.MOE_OK
    _check_layout(ep, xs, 16)
    host = PU.np_inputs(inp)
    layer = M.MoELayer(inp)
    rng = np.random.default_rng(8)
    for r in range(W):
        idx = ep.views[r]["topk_idx"].cpu().numpy()
        rt = O.route(xs[r].cpu(), host["w_gate"], host["bias"], cfg.k)
        PU.check_routing(idx, rt["keys"], rt["idx"], cfg.k)
        toks = np.sort(rng.choice(cfg.T, size=4, replace=False))
        ref = O.forward_tokens(dict(host, x=xs[r].cpu()), toks, idx=idx[toks])
        PU.check_output(ys[r][torch.as_tensor(toks, device=DEV)], ref["y"], f"y rank {r}")
        y1 = layer(xs[r])
        torch.cuda.synchronize()
        PU.check_output(ys[r], y1.double().cpu().numpy(), f"y rank {r} vs one GPU")
