"""Parity of the load-balancing calls (moe_balance_stats, moe_bias_update)
with the fp64 oracle on the GPU's own routing of seeded workloads: small
configurations in full, the full-size skewed prefill and fwd+bwd workloads on
their whole routing; the bias step bit for bit; and the edge cases (one-token
sequences, a single sequence, ragged chunks, an empty batch, out-of-range ids,
the in-place step, run-to-run determinism).

Tolerances: f is a count times E/(k L), so with the same selection it must
equal the oracle's value rounded to fp32.  P and the loss are fp64 sums of the
router probabilities rounded once: against the oracle fed with the GPU's own
probabilities they agree to one fp32 ulp (2^-23 relative); against the
oracle's own probabilities they inherit the 1e-5 relative bound of the
probabilities (sums of positive terms keep the relative bound)."""
import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import (MoEConfig, make_inputs, small_config, FWD_BWD, PREFILL_SKEWED, TINY)
from oracle import moe_oracle as O
import parity_utils as PU

pytestmark = pytest.mark.gpu

ALPHA = 1e-4
GAMMA = 1e-3
ULP32 = 2.0 ** -23


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-30)


def _routed(cfg, T=None, train=False):
    inp = make_inputs(cfg, T=T, device="cuda")
    layer = M.MoELayer(inp)
    if train:
        layer.forward_train(inp["x"])
    else:
        layer(inp["x"])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    ws = layer.train_workspace(inp["T"]) if train else layer.workspace(inp["T"])
    return inp, layer, M.workspace_views(layer.dims(inp["T"]), ws)


def _check_stats(inp, layer, v, seq_len, train=False):
    cfg, T = inp["cfg"], inp["T"]
    st = layer.balance_stats(T, seq_len, ALPHA, train=train)
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    idx = v["topk_idx"].cpu().numpy()
    r = O.route(inp["x"].cpu(), inp["w_gate"].cpu(), inp["bias"].cpu(), cfg.k)
    PU.check_routing(idx, r["keys"], r["idx"], cfg.k)
    ref = O.balance_stats(r["probs"], idx, cfg.E, cfg.k, seq_len, ALPHA)
    own = O.balance_stats(v["probs"].cpu().numpy(), idx, cfg.E, cfg.k, seq_len, ALPHA)
    f, P = st["f"].cpu().numpy(), st["P"].cpu().numpy()
    loss = float(st["loss"].item())
    np.testing.assert_array_equal(f, ref["f"].astype(np.float32))
    assert _rel(P, own["P"]).max() <= ULP32, f"P vs own probs {_rel(P, own['P']).max():.3e}"
    assert _rel(P, ref["P"]).max() <= PU.PROB_RTOL, f"P {_rel(P, ref['P']).max():.3e}"
    assert _rel(loss, own["loss"]) <= ULP32
    assert _rel(loss, ref["loss"]) <= PU.PROB_RTOL
    return st, ref


def _check_bias(inp, layer, v, gamma=GAMMA, train=False):
    cfg, T = inp["cfg"], inp["T"]
    out = torch.empty_like(layer.bias)
    layer.bias_step(T, gamma, out=out, train=train)
    torch.cuda.synchronize()
    counts = v["counts"].cpu().numpy()
    np.testing.assert_array_equal(
        counts, np.bincount(v["topk_idx"].cpu().numpy().ravel(), minlength=cfg.E))
    want = O.bias_update(layer.bias.cpu().numpy(), counts, float(np.float32(gamma)), T, cfg.k)
    want = want.astype(np.float32)
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.int32), want.view(np.int32)), \
        f"bias step differs at {np.nonzero(got != want)[0][:8]}"
    return got


SMALL = [
    ("tiny_L64", TINY, None, 64),
    ("tiny_L1", TINY, None, 1),
    ("tiny_L256_one_seq", TINY, None, 256),
    ("E16_T300_L100_ragged_chunks", small_config(T=300, d=256, E=16, k=4, I=128), None, 100),
    ("E8_k1_T77_L7", MoEConfig("e8k1", T=77, d=128, E=8, k=1, S=1, I=64, bias="uniform0.01"),
     None, 7),
    ("E128_k8_T129_L43", MoEConfig("k8", T=129, d=384, E=128, k=8, S=2, I=64, bias="normal0.05"),
     None, 43),
]


@pytest.mark.parametrize("name,cfg,T,seq_len", SMALL, ids=[c[0] for c in SMALL])
def test_balance_small(name, cfg, T, seq_len):
    inp, layer, v = _routed(cfg, T)
    st, ref = _check_stats(inp, layer, v, seq_len)
    if seq_len == 1:   # a one-token sequence: f = E/k on its chosen experts, P = its probs
        idx = v["topk_idx"].cpu().numpy()
        for t in range(0, inp["T"], 37):
            nz = np.nonzero(st["f"][t].cpu().numpy())[0]
            assert sorted(nz) == sorted(idx[t])
    _check_bias(inp, layer, v)


def test_balance_full_size_skewed_prefill():
    """T=16384 skewed routing (most pairs on a few experts, many experts
    empty) in 4 sequences of 4096 tokens."""
    inp, layer, v = _routed(PREFILL_SKEWED)
    st, ref = _check_stats(inp, layer, v, 4096)
    assert (st["f"].cpu().numpy() == 0).any()          # empty experts inside a sequence
    _check_bias(inp, layer, v)


def test_balance_full_size_fwd_bwd_workload():
    """The fwd+bwd workload (T=8192, one 8192-token sequence) after
    moe_forward_train, reading the training workspace."""
    inp, layer, v = _routed(FWD_BWD, train=True)
    _check_stats(inp, layer, v, 8192, train=True)
    _check_bias(inp, layer, v, train=True)


def test_balance_empty_batch():
    cfg = small_config(T=0, d=256, E=16, k=4, I=128)
    dm = M.dims_of(cfg, T=0)
    loss = torch.full((1,), 7.0, device="cuda")
    e = torch.empty((0, 16), device="cuda")
    M.balance_stats(dm, 16, torch.empty((0, 16), device="cuda"),
                    torch.empty((0, 4), dtype=torch.int32, device="cuda"), ALPHA, e, e.clone(),
                    loss, M.alloc_workspace(M.balance_workspace_size(dm, 16)))
    torch.cuda.synchronize()
    assert loss.item() == 0.0
    bias = torch.linspace(-1, 1, 16, device="cuda")
    out = torch.empty_like(bias)
    M.bias_update(dm, torch.zeros(16, dtype=torch.int32, device="cuda"), GAMMA, bias, out)
    assert torch.equal(out, bias)                       # no load, no step


def test_balance_bad_ids_flagged_and_skipped():
    cfg = small_config(T=64, d=256, E=16, k=4, I=128)
    dm = M.dims_of(cfg, T=64)
    g = torch.Generator().manual_seed(3)
    idx = torch.randint(0, 16, (64, 4), generator=g, dtype=torch.int32)
    probs = torch.softmax(torch.randn((64, 16), generator=g), 1)
    bad = idx.clone()
    bad[5, 2], bad[40, 0] = -1, 16
    f = torch.empty((2, 16), device="cuda")
    P = torch.empty((2, 16), device="cuda")
    loss = torch.empty(1, device="cuda")
    M.balance_stats(dm, 32, probs.cuda(), bad.cuda(), ALPHA, f, P, loss,
                    M.alloc_workspace(M.balance_workspace_size(dm, 32)))
    assert M.device_status() == M.MOE_ERR_INVALID_ARG
    counts = np.zeros((2, 16), np.int64)
    for t in range(64):
        for j in range(4):
            e = int(bad[t, j])
            if 0 <= e < 16:
                counts[t // 32, e] += 1
    np.testing.assert_array_equal(f.cpu().numpy(),
                                  (16 * counts / (4 * 32)).astype(np.float32))
    assert M.device_status() == M.MOE_OK               # the status word was cleared


def test_bias_update_in_place_and_determinism():
    inp, layer, v = _routed(TINY)
    T = inp["T"]
    a = layer.balance_stats(T, 64, ALPHA, train=False)
    b = layer.balance_stats(T, 64, ALPHA, train=False)
    for key in ("f", "P", "loss"):
        assert torch.equal(a[key].view(torch.int32), b[key].view(torch.int32))
    want = _check_bias(inp, layer, v)
    before = layer.bias.clone()
    layer.bias_step(T, GAMMA, train=False)                 # in place (bias_out == bias_in)
    torch.cuda.synchronize()
    assert np.array_equal(layer.bias.cpu().numpy().view(np.int32), want.view(np.int32))
    assert not torch.equal(layer.bias, before)
