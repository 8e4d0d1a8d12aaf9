"""Pins of the fp64 oracle against facts that do not come from the oracle:
hand-derived closed forms (tests/golden), brute force over all expert subsets,
textbook constants and identities, library routines for special cases, the
invariants the pages fix, and finite differences for the backward."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200.workloads import MoEConfig, make_inputs, small_config
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(v):
    if isinstance(v, str):
        if "/" in v:
            a, b = v.split("/")
            return float(a) / float(b)
        neg = v.startswith("-")
        v = v.lstrip("-")
        assert v.startswith("ln")
        r = math.log(float(v[2:]))
        return -r if neg else r
    if isinstance(v, list):
        return [_val(u) for u in v]
    return float(v)


def _hand_inputs():
    with open(os.path.join(GOLDEN, "moe_hand_example.json")) as f:
        g = json.load(f)
    cfg = MoEConfig("hand", T=g["T"], d=g["d"], E=g["E"], k=g["k"], S=g["S"], I=g["I"])
    inp = {"cfg": cfg}
    for key in ("x", "w_gate", "bias", "w1", "w3", "w2", "ws1", "ws3", "ws2"):
        inp[key] = np.array(_val(g[key]), dtype=np.float64)
    return g, inp


# ---------------------------------------------------------------- golden

def test_hand_example_forward():
    g, inp = _hand_inputs()
    f = O.forward(inp, align=g["align"])
    ex = g["expected"]
    np.testing.assert_allclose(f["probs"], np.array(_val(ex["probs"])), rtol=1e-14)
    assert f["idx"].tolist() == ex["idx"]
    np.testing.assert_allclose(f["w"], np.array(_val(ex["w"])), rtol=1e-14)
    assert f["counts"].tolist() == ex["counts"]
    assert f["offsets"].tolist() == ex["offsets"]
    assert f["row_of"].tolist() == ex["row_of"]
    assert f["token_of_row"].tolist() == ex["token_of_row"]
    np.testing.assert_allclose(f["y"], np.array(ex["y"]), rtol=1e-13, atol=1e-15)


def test_hand_example_per_token_path():
    g, inp = _hand_inputs()
    f = O.forward_tokens(inp, [0, 1])
    np.testing.assert_allclose(f["y"], np.array(g["expected"]["y"]), rtol=1e-13)


@pytest.mark.parametrize("case", [0, 1])
def test_permute_golden(case):
    with open(os.path.join(GOLDEN, "permute_small.json")) as f:
        g = json.load(f)
    c = g["cases"][case]
    pm = O.permute(np.array(g["idx"]), g["E"], c["align"])
    assert pm["counts"].tolist() == c["counts"]
    assert pm["offsets"].tolist() == c["offsets"]
    assert pm["row_of"].tolist() == c["row_of"]
    assert pm["token_of_row"].tolist() == c["token_of_row"]


# ---------------------------------------------------------------- softmax

def test_softmax_closed_forms():
    z = np.array([[0.0, math.log(2), math.log(3), 0.0],
                  [5.0, 5.0, 5.0, 5.0],
                  [1000.0, 0.0, -1000.0, 1000.0]])
    p = O.softmax(z)
    np.testing.assert_allclose(p[0], [1 / 7, 2 / 7, 3 / 7, 1 / 7], rtol=1e-14)
    np.testing.assert_allclose(p[1], [0.25] * 4, rtol=1e-15)
    np.testing.assert_allclose(p[2], [0.5, 0.0, 0.0, 0.5], atol=1e-300)
    # shift invariance and normalisation on random rows
    rng = np.random.default_rng(1)
    zr = rng.normal(size=(50, 128)) * 3
    np.testing.assert_allclose(O.softmax(zr), O.softmax(zr + 7.25), rtol=1e-12)
    np.testing.assert_allclose(O.softmax(zr).sum(1), 1.0, rtol=1e-14)
    # ratio p_a / p_b = exp(z_a - z_b)
    pr = O.softmax(zr)
    np.testing.assert_allclose(pr[:, 3] / pr[:, 7], np.exp(zr[:, 3] - zr[:, 7]), rtol=1e-12)


def test_gate_logits_brute_force():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 5))
    wg = rng.normal(size=(4, 5))
    z = O.gate_logits(x, wg)
    for t in range(3):
        for e in range(4):
            assert abs(z[t, e] - sum(x[t, i] * wg[e, i] for i in range(5))) < 1e-12


# ---------------------------------------------------------------- top-k

def _dominant_subset(keys, k):
    """Brute force: the unique k-subset S with key_i > key_j, or equal keys and
    i < j, for every i in S and j outside S."""
    E = len(keys)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [j for j in range(E) if j not in S]
        if all(keys[i] > keys[j] or (keys[i] == keys[j] and i < j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("E,k", [(8, 2), (10, 3), (7, 6)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # values on a coarse grid so that exact ties are frequent
    keys = rng.integers(0, 5, size=(16, E)).astype(np.float64) * 0.25
    idx = O.select_topk(keys, k)
    for t in range(16):
        assert set(idx[t].tolist()) == _dominant_subset(keys[t].tolist(), k)
        # order: descending key, equal keys by ascending id
        kk = [(-keys[t, i], i) for i in idx[t]]
        assert kk == sorted(kk)
        # the chosen set maximises the sum of keys
        best = max(sum(keys[t, list(S)]) for S in itertools.combinations(range(E), k))
        assert abs(keys[t, idx[t]].sum() - best) < 1e-12


def test_topk_tie_lower_id_first():
    keys = np.array([[0.5, 0.7, 0.7, 0.1, 0.7]])
    assert O.select_topk(keys, 2).tolist() == [[1, 2]]
    assert O.select_topk(keys, 3).tolist() == [[1, 2, 4]]


def test_bias_is_selection_only():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(32, 16))
    wg = rng.normal(size=(8, 16)) * 0.3
    b = np.zeros(8)
    b[5] = 10.0                     # expert 5 always wins selection
    r = O.route(x, wg, b, 3)
    assert (r["idx"][:, 0] == 5).all()
    p = O.softmax(x @ wg.T)
    psel = np.take_along_axis(p, r["idx"], 1)
    np.testing.assert_allclose(r["w"], psel / psel.sum(1, keepdims=True), rtol=1e-14)
    # a constant added to every bias changes nothing
    r2 = O.route(x, wg, b + 0.125, 3)
    assert (r2["idx"] == r["idx"]).all()
    np.testing.assert_allclose(r2["w"], r["w"], rtol=1e-15)


# ---------------------------------------------------------------- SwiGLU

def test_silu_constants_and_identities():
    assert O.silu(np.array([0.0]))[0] == 0.0
    # sigma(1) = 1 / (1 + 1/e), a textbook constant
    assert abs(O.silu(np.array([1.0]))[0] - 0.7310585786300049) < 1e-16
    g = np.linspace(-30, 30, 601)
    # silu(-g) = silu(g) - g
    np.testing.assert_allclose(O.silu(-g), O.silu(g) - g, atol=1e-12)
    np.testing.assert_allclose(O.silu(np.array([60.0])), [60.0], rtol=1e-15)
    assert abs(O.silu(np.array([-60.0]))[0]) < 1e-20
    # the library's SiLU
    np.testing.assert_allclose(O.silu(g), torch.nn.functional.silu(torch.tensor(g)).numpy(),
                               rtol=1e-14, atol=1e-300)


def test_silu_grad_central_difference():
    g = np.linspace(-8, 8, 97)
    h = 1e-6
    fd = (O.silu(g + h) - O.silu(g - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_grad(g), fd, atol=1e-8)


def _dense_ffn_torch(x, w1, w3, w2):
    x, w1, w3, w2 = (torch.as_tensor(np.asarray(a, dtype=np.float64)) for a in (x, w1, w3, w2))
    F = torch.nn.functional
    return (F.silu(F.linear(x, w1)) * F.linear(x, w3)).matmul(w2.T).numpy()


def _identical_expert_inputs(shared_equal: bool):
    cfg = small_config(T=40, d=64, E=8, k=3, S=2, I=32)
    inp = make_inputs(cfg)
    inp = {k: (v.double().numpy() if torch.is_tensor(v) else v) for k, v in inp.items()}
    for name in ("w1", "w3", "w2"):
        inp[name] = np.broadcast_to(inp[name][0], inp[name].shape).copy()
    for name in ("ws1", "ws3", "ws2"):
        src = inp[name.replace("s", "")][0]
        inp[name] = (np.broadcast_to(src, inp[name].shape).copy() if shared_equal
                     else np.zeros_like(inp[name]))
    return inp


def test_identical_experts_reduce_to_dense_swiglu():
    inp = _identical_expert_inputs(shared_equal=False)
    f = O.forward(inp)
    F = _dense_ffn_torch(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    np.testing.assert_allclose(f["w"].sum(1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(f["y"], F, rtol=1e-10, atol=1e-12)


def test_identical_experts_and_shared_give_three_times_dense():
    inp = _identical_expert_inputs(shared_equal=True)
    f = O.forward(inp)
    F = _dense_ffn_torch(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    np.testing.assert_allclose(f["y"], 3 * F, rtol=1e-10, atol=1e-12)


def test_single_expert_is_textbook_ffn():
    cfg = MoEConfig("e1", T=10, d=32, E=1, k=1, S=1, I=16)
    inp = make_inputs(cfg)
    inp = {k: (v.double().numpy() if torch.is_tensor(v) else v) for k, v in inp.items()}
    f = O.forward(inp, align=4)
    F0 = _dense_ffn_torch(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    Fs = _dense_ffn_torch(inp["x"], inp["ws1"][0], inp["ws3"][0], inp["ws2"][0])
    assert (f["w"] == 1.0).all()
    np.testing.assert_allclose(f["y"], F0 + Fs, rtol=1e-10, atol=1e-12)


def test_dense_swiglu_is_textbook_ffn_and_one_expert_layer():
    """The dense layer equals torch's textbook SwiGLU FFN, and equals the MoE
    layer reduced to one routed expert (k = 1, weight 1) with no shared one."""
    cfg = MoEConfig("e1s0", T=12, d=32, E=1, k=1, S=0, I=24)
    inp = make_inputs(cfg)
    inp = {k: (v.double().numpy() if torch.is_tensor(v) else v) for k, v in inp.items()}
    y = O.dense_swiglu(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0])
    np.testing.assert_allclose(
        y, _dense_ffn_torch(inp["x"], inp["w1"][0], inp["w3"][0], inp["w2"][0]),
        rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(y, O.forward(inp, align=4)["y"], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- whole layer

def test_dense_mask_brute_force_tiny_config():
    """All experts on all tokens, combined through a one-hot weight matrix."""
    inp = make_inputs(0, T=48)
    f = O.forward(inp)
    x = inp["x"].double().numpy()
    E = inp["cfg"].E
    mask = np.zeros((48, E))
    for t in range(48):
        for j in range(inp["cfg"].k):
            mask[t, f["idx"][t, j]] = f["w"][t, j]
    y = np.zeros_like(x)
    for s in range(inp["cfg"].S):
        y += _dense_ffn_torch(x, inp["ws1"][s].double(), inp["ws3"][s].double(),
                              inp["ws2"][s].double())
    for e in range(E):
        if mask[:, e].any():
            y += mask[:, e:e + 1] * _dense_ffn_torch(x, inp["w1"][e].double(),
                                                     inp["w3"][e].double(),
                                                     inp["w2"][e].double())
    np.testing.assert_allclose(f["y"], y, rtol=1e-10, atol=1e-12)


@pytest.fixture(scope="module")
def tiny_forward():
    inp = make_inputs(0)
    return inp, O.forward(inp, align=16)


def test_routing_invariants_tiny_config(tiny_forward):
    inp, f = tiny_forward
    cfg = inp["cfg"]
    T = inp["T"]
    idx = f["idx"]
    assert idx.shape == (T, cfg.k)
    for t in range(T):
        assert len(set(idx[t].tolist())) == cfg.k          # k distinct experts
    assert ((idx >= 0) & (idx < cfg.E)).all()
    assert f["counts"].sum() == T * cfg.k                   # nothing dropped
    assert (f["w"] >= 0).all()
    np.testing.assert_allclose(f["w"].sum(1), 1.0, rtol=1e-14)


def test_permutation_invariants_tiny_config(tiny_forward):
    inp, f = tiny_forward
    cfg = inp["cfg"]
    T, k, E = inp["T"], cfg.k, cfg.E
    off, cnt = f["offsets"], f["counts"]
    assert (off % 16 == 0).all()
    assert (np.diff(off) >= cnt).all() and (np.diff(off) - cnt < 16).all()
    row_of = f["row_of"].reshape(T, k)
    tor = f["token_of_row"]
    assert len(set(f["row_of"].tolist())) == T * k                    # injective
    assert ((tor >= 0).sum()) == T * k
    for t in range(T):
        for j in range(k):
            r = row_of[t, j]
            e = f["idx"][t, j]
            assert off[e] <= r < off[e] + cnt[e]
            assert tor[r] == t
    for e in range(E):                                                # ascending tokens
        seg = tor[off[e]:off[e] + cnt[e]]
        assert (np.diff(seg) > 0).all()
        assert (tor[off[e] + cnt[e]:off[e + 1]] == -1).all()
    # permute then un-permute is the identity on x
    x = inp["x"].double().numpy()
    xp = O.gather_rows(x, tor)
    assert (xp[tor < 0] == 0).all()
    for j in range(k):
        np.testing.assert_array_equal(xp[row_of[:, j]], x)
    for j in range(k):
        onehot = np.zeros((T, k))
        onehot[:, j] = 1.0
        np.testing.assert_array_equal(O.unpermute_sum(xp, f["row_of"], onehot, T, k), x)


def test_per_token_path_matches_segment_path(tiny_forward):
    inp, f = tiny_forward
    toks = [0, 5, 17, 100, 255]
    ft = O.forward_tokens(inp, toks)
    np.testing.assert_allclose(ft["y"], f["y"][toks], rtol=1e-10, atol=1e-13)
    assert (ft["idx"] == f["idx"][toks]).all()


@pytest.mark.parametrize("align", [1, 16, 128])
def test_output_independent_of_align(align):
    inp = make_inputs(small_config(T=24, d=64, E=8, k=3, I=32))
    y16 = O.forward(inp, align=16)["y"]
    np.testing.assert_allclose(O.forward(inp, align=align)["y"], y16, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- backward

def _fd_inputs():
    cfg = MoEConfig("fd", T=4, d=16, E=8, k=2, S=2, I=8, bias="uniform0.01", grad=True)
    inp = make_inputs(cfg, seed=7)
    out = {"cfg": cfg}
    for key, v in inp.items():
        if torch.is_tensor(v):
            out[key] = v.double().numpy().copy()
    # larger weights so that every term is well above round-off
    for key in ("w1", "w3", "w2", "ws1", "ws3", "ws2"):
        out[key] *= 10.0
    out["w_gate"] *= 10.0
    return out


@pytest.mark.parametrize("name,grad", [("x", "dx"), ("w_gate", "dw_gate"), ("w1", "dw1"),
                                       ("w3", "dw3"), ("w2", "dw2"), ("ws1", "dws1"),
                                       ("ws3", "dws3"), ("ws2", "dws2")])
def test_backward_finite_differences(name, grad):
    inp = _fd_inputs()
    dy = inp["dy"]
    fwd = O.forward(inp)
    g = O.backward(inp, dy, fwd)[grad]
    rng = np.random.default_rng(11)
    flat = inp[name].reshape(-1)
    picks = rng.choice(flat.size, size=min(flat.size, 48), replace=False)
    h = 1e-6
    for i in picks:
        old = flat[i]
        flat[i] = old + h
        fp = O.forward(inp)
        flat[i] = old - h
        fm = O.forward(inp)
        flat[i] = old
        assert (fp["idx"] == fwd["idx"]).all() and (fm["idx"] == fwd["idx"]).all()
        fd = (np.sum(fp["y"] * dy) - np.sum(fm["y"] * dy)) / (2 * h)
        assert abs(g.reshape(-1)[i] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, i, g.reshape(-1)[i], fd)


def test_backward_bias_gets_no_gradient():
    """The bias only moves the selection key, so with the selection fixed the
    loss does not depend on it."""
    inp = _fd_inputs()
    dy = inp["dy"]
    y0 = O.forward(inp)
    inp["bias"] = inp["bias"] + 1e-7
    y1 = O.forward(inp)
    assert (y0["idx"] == y1["idx"]).all()
    assert np.sum(y0["y"] * dy) == np.sum(y1["y"] * dy)


# ------------------------------------------------------------------ load balancing

def test_balance_hand_example():
    """Worked example with exact fractions (golden/balance_hand_example.json)."""
    with open(os.path.join(GOLDEN, "balance_hand_example.json")) as f:
        g = json.load(f)
    probs = np.array(_val(g["probs"]))
    idx = np.array(g["idx"])
    r = O.balance_stats(probs, idx, g["E"], g["k"], g["seq_len"], _val(g["alpha"]))
    np.testing.assert_array_equal(r["counts"], g["counts"])
    np.testing.assert_allclose(r["f"], _val(g["f"]), rtol=1e-15, atol=0)
    np.testing.assert_allclose(r["P"], _val(g["P"]), rtol=1e-15, atol=0)
    np.testing.assert_allclose((r["f"] * r["P"]).sum(1), _val(g["sum_fP"]), rtol=1e-15)
    assert r["loss"] == pytest.approx(_val(g["loss"]), rel=1e-15)
    nb = O.bias_update(_val(g["bias"]), g["batch_counts"], _val(g["gamma"]), T=len(idx), k=g["k"])
    np.testing.assert_array_equal(nb, _val(g["bias_next"]))


def _balanced_seq(E, k, L):
    """Every expert gets exactly k*L/E pairs; uniform probabilities."""
    idx = np.array([[(k * t + j) % E for j in range(k)] for t in range(L)])
    return np.full((L, E), 1.0 / E), idx


def _collapsed_seq(E, k, L):
    """Every token picks experts 0..k-1 and puts all its mass on them."""
    p = np.zeros((L, E))
    p[:, :k] = 1.0 / k
    return p, np.tile(np.arange(k), (L, 1))


def test_balance_closed_forms():
    """Perfect balance gives f = 1, P = 1/E and loss = alpha; full collapse
    onto k experts gives f = E/k there, P = 1/k and loss = alpha * E / k; two
    such sequences give the mean of the two."""
    E, k, L, alpha = 8, 2, 16, 0.3
    pb, ib = _balanced_seq(E, k, L)
    r = O.balance_stats(pb, ib, E, k, L, alpha)
    np.testing.assert_allclose(r["f"], 1.0, rtol=1e-15)
    np.testing.assert_allclose(r["P"], 1.0 / E, rtol=1e-15)
    assert r["loss"] == pytest.approx(alpha, rel=1e-14)
    pc, ic = _collapsed_seq(E, k, L)
    r = O.balance_stats(pc, ic, E, k, L, alpha)
    np.testing.assert_allclose(r["f"][0, :k], E / k, rtol=1e-15)
    assert not r["f"][0, k:].any() and not r["P"][0, k:].any()
    assert r["loss"] == pytest.approx(alpha * E / k, rel=1e-14)
    r = O.balance_stats(np.concatenate([pb, pc]), np.concatenate([ib, ic]), E, k, L, alpha)
    assert r["loss"] == pytest.approx(alpha * (1 + E / k) / 2, rel=1e-14)


def test_balance_invariants_random_routing():
    """On a random softmax / top-k routing: sum_e f = E and sum_e P = 1 per
    sequence; the loss does not change when tokens are reordered inside a
    sequence or when the experts are relabelled (probabilities and ids
    permuted together), and it does change when only the ids are shuffled."""
    rng = np.random.default_rng(5)
    E, k, L, n = 16, 4, 24, 3
    p = O.softmax(rng.normal(size=(n * L, E)) * 2)
    idx = np.argsort(-p - rng.uniform(0, 0.05, size=p.shape), axis=1)[:, :k]
    r = O.balance_stats(p, idx, E, k, L, 1.0)
    np.testing.assert_allclose(r["f"].sum(1), E, rtol=1e-14)
    np.testing.assert_allclose(r["P"].sum(1), 1.0, rtol=1e-14)
    assert r["counts"].sum() == n * L * k
    perm_t = np.concatenate([s * L + rng.permutation(L) for s in range(n)])
    r2 = O.balance_stats(p[perm_t], idx[perm_t], E, k, L, 1.0)
    assert r2["loss"] == pytest.approx(r["loss"], rel=1e-13)
    relabel = rng.permutation(E)            # expert e becomes relabel[e]
    p3 = np.empty_like(p)
    p3[:, relabel] = p
    r3 = O.balance_stats(p3, relabel[idx], E, k, L, 1.0)
    assert r3["loss"] == pytest.approx(r["loss"], rel=1e-13)
    np.testing.assert_allclose(r3["f"][:, relabel], r["f"], rtol=1e-15)
    r4 = O.balance_stats(p, (idx + 1) % E, E, k, L, 1.0)
    assert abs(r4["loss"] - r["loss"]) > 1e-3 * r["loss"]


def test_bias_update_direction_and_fixed_point():
    """Overloaded experts move down by gamma, underloaded up by gamma, experts
    exactly at the mean load keep their bias bit for bit (also -0.0); a batch
    with every expert at the mean is a fixed point."""
    T, k, E, gamma = 32, 4, 8, 1e-3
    mean = T * k // E
    counts = np.array([mean + 3, mean - 1, mean, mean, mean + 1, mean - 2, mean, mean - 1])
    assert counts.sum() == T * k
    bias = np.array([0.5, -0.25, -0.0, 1e-3, 0.0, 0.0, 2.0, -1.0])
    nb = O.bias_update(bias, counts, gamma, T, k)
    np.testing.assert_array_equal(np.sign(nb - bias), [-1, 1, 0, 0, -1, 1, 0, 1])
    np.testing.assert_allclose(np.abs(nb - bias)[nb != bias], gamma, rtol=1e-12)
    assert np.signbit(nb[2])
    np.testing.assert_array_equal(O.bias_update(bias, np.full(E, mean), gamma, T, k), bias)


# ---- expert-parallel layout ------------------------------------------------

def test_ep_layout_hand_example():
    """W = 2 ranks, E = 4 experts (rank 0 owns 0-1, rank 1 owns 2-3), k = 2,
    align = 2.  Rank 0 routes t0 -> {0, 1}, t1 -> {1, 3}; rank 1 routes
    t0 -> {3, 0}, t1 -> {1, 2}.  Worked by hand: rank 0's expert 0 gets
    (s0 t0), (s1 t0) = rows 0-1; expert 1 gets (s0 t0), (s0 t1), (s1 t1) =
    rows 2-4 and one padding row 5.  Rank 1's expert 2 gets (s1 t1) = row 0 and
    padding row 1; expert 3 gets (s0 t1), (s1 t0) = rows 2-3."""
    L = O.ep_layout([np.array([[0, 1], [1, 3]]), np.array([[3, 0], [1, 2]])], 4, 2)
    assert L["recv_offsets"].tolist() == [[0, 2, 6], [0, 2, 4]]
    assert L["recv_counts"].tolist() == [[2, 3], [1, 2]]
    assert L["owner"][0].tolist() == [0, 0, 0, 1] and L["row"][0].tolist() == [0, 2, 3, 2]
    assert L["owner"][1].tolist() == [1, 0, 0, 1] and L["row"][1].tolist() == [3, 1, 4, 0]
    assert L["src_of_row"][0] == [(0, 0), (1, 0), (0, 0), (0, 1), (1, 1), (-1, -1)]
    assert L["src_of_row"][1] == [(1, 1), (-1, -1), (0, 1), (1, 0)]


@pytest.mark.parametrize("align", [1, 16])
def test_ep_layout_one_rank_is_the_permutation(align):
    """With one rank the exchange is the identity: the receive layout is the
    permutation's own segment layout."""
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(16)[:4] for _ in range(37)])
    L = O.ep_layout([idx], 16, align)
    P = O.permute(idx, 16, align)
    assert L["recv_offsets"][0].tolist() == P["offsets"].tolist()
    assert L["recv_counts"][0].tolist() == P["counts"].tolist()
    assert L["row"][0].tolist() == P["row_of"].tolist()
    assert (L["owner"][0] == 0).all()
    tor = [t for (_, t) in L["src_of_row"][0]]
    assert tor == P["token_of_row"][:len(tor)].tolist()


@pytest.mark.parametrize("W,E,k,align", [(2, 16, 4, 16), (4, 32, 3, 4), (8, 8, 2, 16)])
def test_ep_layout_invariants_random_routing(W, E, k, align):
    """Every pair lands exactly once, on the rank that owns its expert, inside
    that expert's segment; segments are padded multiples of align and hold
    the pairs by ascending (source rank, token); the ranks' loads add up."""
    rng = np.random.default_rng(W * 100 + E)
    T = [int(rng.integers(0, 40)) for _ in range(W)]
    idx = [np.stack([rng.permutation(E)[:k] for _ in range(t)]) if t else
           np.zeros((0, k), np.int64) for t in T]
    L = O.ep_layout(idx, E, align)
    El = E // W
    taken = [set() for _ in range(W)]
    for s in range(W):
        for p in range(T[s] * k):
            e = int(idx[s].reshape(-1)[p])
            r, row = int(L["owner"][s][p]), int(L["row"][s][p])
            assert r == e // El
            le = e - r * El
            assert L["recv_offsets"][r, le] <= row < L["recv_offsets"][r, le] + L["recv_counts"][r, le]
            assert row not in taken[r]
            taken[r].add(row)
            assert L["src_of_row"][r][row] == (s, p // k)
    for r in range(W):
        off, cnt = L["recv_offsets"][r], L["recv_counts"][r]
        assert off[0] == 0 and (np.diff(off) % align == 0).all()
        assert (np.diff(off) >= cnt).all() and (np.diff(off) - cnt < align).all()
        assert len(taken[r]) == cnt.sum()
        for le in range(El):
            seg = L["src_of_row"][r][off[le]:off[le] + cnt[le]]
            assert seg == sorted(seg)                       # (source, token) ascending
            assert all(s < 0 for s, _ in L["src_of_row"][r][off[le] + cnt[le]:off[le + 1]])
    total = sum(int(L["recv_counts"][r].sum()) for r in range(W))
    assert total == sum(T) * k


def test_ep_recv_rows_gathers_the_source_tokens():
    rng = np.random.default_rng(9)
    x = [rng.standard_normal((5, 8)), rng.standard_normal((3, 8))]
    idx = [np.array([[0, 1], [2, 3], [1, 2], [0, 3], [3, 1]]), np.array([[2, 0], [1, 3], [0, 2]])]
    L = O.ep_layout(idx, 4, 4)
    for r in range(2):
        rows = O.ep_recv_rows(x, L, r)
        for i, (s, t) in enumerate(L["src_of_row"][r]):
            np.testing.assert_array_equal(rows[i], x[s][t] if s >= 0 else np.zeros(8))


@pytest.mark.parametrize("W,align", [(1, 16), (2, 4), (4, 16)])
def test_ep_exchange_reproduces_the_layer_output(W, align):
    """Every rank routes its own tokens; the rows move to their owners by the
    layout, each owner runs its experts segment by segment, and each rank
    reads its pairs' outputs back by (owner, row) and combines them with its
    shared experts: the result is forward() of that rank's tokens."""
    cfg = small_config(T=11, d=32, E=8, k=2, S=1, I=16)
    base = make_inputs(cfg)
    host = {n: (v.double().numpy() if torch.is_tensor(v) else v) for n, v in base.items()}
    xs = [host["x"]] + [make_inputs(cfg, seed=300 + r, weights=False)["x"].double().numpy()
                        for r in range(1, W)]
    routes = [O.route(x, host["w_gate"], host["bias"], cfg.k) for x in xs]
    L = O.ep_layout([r["idx"] for r in routes], cfg.E, align)
    El = cfg.E // W
    outs = []
    for r in range(W):
        rows = O.ep_recv_rows(xs, L, r)
        o = np.zeros_like(rows)
        for le in range(El):
            a, b = int(L["recv_offsets"][r, le]), int(L["recv_offsets"][r, le + 1])
            e = r * El + le
            if b > a:
                o[a:b] = O.swiglu_expert(rows[a:b], host["w1"][e], host["w3"][e], host["w2"][e])[0]
        outs.append(o)
    for s, x in enumerate(xs):
        y = O.swiglu_expert(x, host["ws1"][0], host["ws3"][0], host["ws2"][0])[0]
        for p in range(x.shape[0] * cfg.k):
            t, j = divmod(p, cfg.k)
            y[t] += routes[s]["w"][t, j] * outs[L["owner"][s][p]][L["row"][s][p]]
        want = O.forward(dict(host, x=x, T=x.shape[0]), align=align)["y"]
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_bf16_emulation_without_rounding_is_the_oracle_backward():
    """The backward tests' emulation of the bf16 MMA operands, with the
    rounding switched off, must give the oracle's routed weight gradients
    (it restates them from the forward's intermediates, not through
    swiglu_expert_backward); with bf16 rounding it must differ."""
    import bf16_emulation as EM
    cfg = small_config(T=40, d=64, E=8, k=2, I=64)
    inp = make_inputs(cfg)
    inp["dy"] = torch.randn((40, 64), generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    f = O.forward(inp)
    b = O.backward(inp, inp["dy"], f)
    ex = list(range(cfg.E))
    exact = EM.routed_weight_grads(inp, f, b, ex, rnd=lambda a: np.asarray(a, dtype=np.float64))
    rounded = EM.routed_weight_grads(inp, f, b, ex)
    for name in ("dw1", "dw3", "dw2"):
        for e in ex:
            np.testing.assert_allclose(exact[name][e], b[name][e], rtol=0, atol=1e-12)
        assert max(np.abs(rounded[name][e] - b[name][e]).max() for e in ex) > 0
