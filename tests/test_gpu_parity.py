"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Each step of the layer is checked on its own (route, permute, grouped SwiGLU,
combine) and the fused moe_forward end to end, on seeded inputs of the
workload configurations: the tiny configuration in full, ragged and edge-case
shapes that span several tiles and a tail, and the full-size configurations
on the full routing plus sampled output tokens."""
import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import (CONFIGS, MoEConfig, make_inputs, small_config, DECODE, PREFILL_BALANCED, PREFILL_SKEWED, TINY)
from oracle import moe_oracle as O
import parity_utils as PU

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _gpu(inp):
    return {k: (v.to(DEV).contiguous() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _route(dm, g):
    T, E, k = dm.T, dm.E, dm.k
    probs = torch.empty((T, E), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    ws = M.alloc_workspace(M.route_workspace_size(dm))
    M.route(dm, g["x"], g["w_gate"], g["bias"], probs, idx, w, ws)
    return probs, idx, w


def _permute(dm, idx, x):
    cap = M.capacity(dm)
    out = {
        "counts": torch.empty(dm.E, dtype=torch.int32, device=DEV),
        "offsets": torch.empty(dm.E + 1, dtype=torch.int32, device=DEV),
        "row_of": torch.empty(dm.T * dm.k, dtype=torch.int32, device=DEV),
        "token_of_row": torch.full((cap,), 7, dtype=torch.int32, device=DEV),
        "x_perm": torch.full((cap, dm.d), float("nan"), dtype=torch.bfloat16, device=DEV),
    }
    ws = M.alloc_workspace(M.permute_workspace_size(dm))
    M.permute(dm, idx, x, out["counts"], out["offsets"], out["row_of"], out["token_of_row"],
              out["x_perm"], ws)
    return out


def _check_permutation(dm, pm, idx_gpu, x):
    ref = O.permute(idx_gpu.cpu().numpy(), dm.E, dm.align)
    np.testing.assert_array_equal(pm["counts"].cpu().numpy(), ref["counts"])
    np.testing.assert_array_equal(pm["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(pm["row_of"].cpu().numpy(), ref["row_of"])
    np.testing.assert_array_equal(pm["token_of_row"].cpu().numpy(), ref["token_of_row"])
    used = int(ref["offsets"][-1])
    got = pm["x_perm"][:used].cpu()
    want = torch.zeros((used, dm.d), dtype=torch.bfloat16)
    tor = torch.as_tensor(ref["token_of_row"][:used])
    valid = tor >= 0
    want[valid] = x.cpu()[tor[valid]]
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), "x_perm not bit-exact"
    return ref


# ------------------------------------------------------------------ router

ROUTE_CASES = [
    ("tiny_full", TINY, None),
    ("small_E16_ragged", small_config(T=300, d=256, E=16, k=4, I=128), None),
    ("E8_k1", MoEConfig("e8k1", T=77, d=128, E=8, k=1, S=1, I=64, bias="uniform0.01"), None),
    ("E128_k8", MoEConfig("k8", T=129, d=384, E=128, k=8, S=2, I=64, bias="normal0.05"), None),
    ("decode_full", DECODE, None),
    # 46 and 18 split partials: the top-k sums them with 4 and 2 warps per token
    ("d5120_T300_46_splits", DECODE, 300),
    ("d5120_T1024_18_splits", PREFILL_BALANCED, 1024),
    ("skewed_zipf_slice", PREFILL_SKEWED, 2048),
]


@pytest.mark.parametrize("name,cfg,T", ROUTE_CASES, ids=[c[0] for c in ROUTE_CASES])
def test_route_parity(name, cfg, T):
    inp = make_inputs(cfg, T=T, weights=False)
    g = _gpu(inp)
    dm = M.dims_of(cfg, T=inp["T"])
    probs, idx, w = _route(dm, g)
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    r = O.route(inp["x"], inp["w_gate"], inp["bias"], cfg.k)
    PU.check_probs(probs, r["probs"])
    ties = PU.check_routing(idx.cpu().numpy(), r["keys"], r["idx"], cfg.k)
    assert ties <= max(1, inp["T"] // 500)
    # weights: the oracle's probabilities of the GPU's choice, renormalised
    p_sel = np.take_along_axis(r["probs"], idx.cpu().numpy().astype(np.int64), 1)
    w_ref = p_sel / p_sel.sum(1, keepdims=True)
    err = np.abs(w.cpu().double().numpy() - w_ref) / w_ref
    assert err.max() <= PU.PROB_RTOL


def test_route_exact_ties_lower_id_first():
    """All logits equal and zero bias: every key ties, so the chosen experts
    are 0..k-1 in that order and the weights are 1/k."""
    cfg = small_config(T=40, d=128, E=32, k=6, I=64)
    dm = M.dims_of(cfg)
    g = {"x": torch.ones((40, 128), dtype=torch.bfloat16, device=DEV),
         "w_gate": torch.zeros((32, 128), dtype=torch.float32, device=DEV),
         "bias": torch.zeros(32, dtype=torch.float32, device=DEV)}
    probs, idx, w = _route(dm, g)
    assert (idx.cpu() == torch.arange(6, dtype=torch.int32)).all()
    assert torch.allclose(w.cpu(), torch.full((40, 6), 1 / 6), rtol=1e-6)
    assert torch.allclose(probs.cpu(), torch.full((40, 32), 1 / 32), rtol=1e-6)


# ------------------------------------------------------------------ permute

@pytest.mark.parametrize("align", [16, 128])
@pytest.mark.parametrize("pattern", ["routed", "all_one_expert", "ragged_random"])
def test_permute_parity(align, pattern):
    T, d, E, k = 1000, 256, 128, 6
    dm = M.dims(T, d, E, k, 64, 0, align)
    gen = torch.Generator().manual_seed(5)
    x = torch.randn((T, d), generator=gen).to(torch.bfloat16)
    if pattern == "routed":
        inp = make_inputs(0, T=T, weights=False)
        idx = O.route(inp["x"], inp["w_gate"], inp["bias"], k)["idx"]
        idx = torch.as_tensor(idx, dtype=torch.int32)
    elif pattern == "all_one_expert":
        idx = torch.stack([torch.full((T,), e, dtype=torch.int32) for e in (7, 0, 127, 3, 9, 64)], 1)
    else:
        idx = torch.stack([torch.randperm(E, generator=gen)[:k] for _ in range(T)]).to(torch.int32)
    pm = _permute(dm, idx.to(DEV), x.to(DEV))
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    _check_permutation(dm, pm, idx, x)


def test_permute_empty_batch():
    dm = M.dims(0, 256, 16, 4, 64, 0, 16)
    pm = _permute(dm, torch.empty((0, 4), dtype=torch.int32, device=DEV),
                  torch.empty((0, 256), dtype=torch.bfloat16, device=DEV))
    torch.cuda.synchronize()
    assert (pm["counts"].cpu() == 0).all() and (pm["offsets"].cpu() == 0).all()
    assert (pm["token_of_row"].cpu() == -1).all()


def test_permute_flags_bad_expert_ids():
    dm = M.dims(64, 128, 16, 2, 64, 0, 16)
    idx = torch.zeros((64, 2), dtype=torch.int32)
    idx[:, 1] = 1
    idx[5, 1] = 16          # out of range: skipped and flagged
    idx[9, 1] = 0           # repeated within a token: flagged
    x = torch.zeros((64, 128), dtype=torch.bfloat16)
    _permute(dm, idx.to(DEV), x.to(DEV))
    assert M.device_status() == M.MOE_ERR_INVALID_ARG
    assert M.device_status() == M.MOE_OK   # cleared by the read


# ------------------------------------------------------------------ grouped GEMMs

GEMM_CASES = [
    ("tiny_full", TINY, None, 16),
    ("tiny_align128", TINY, None, 128),
    ("small_ragged", small_config(T=333, d=256, E=16, k=4, I=192), None, 16),
    ("decode_full", DECODE, None, 16),
    ("pair_prefill_T700", small_config(T=700, d=512, E=16, k=4, I=256), None, 16),
]


def _grouped(dm, x_perm, offsets, g):
    cap = M.capacity(dm)
    h = torch.full((cap, dm.I), float("nan"), dtype=torch.bfloat16, device=DEV)
    y = torch.full((cap, dm.d), float("nan"), dtype=torch.float32, device=DEV)
    M.grouped_swiglu(dm, x_perm, offsets, g["w1"], g["w3"], g["w2"], h, y)
    return h, y


@pytest.mark.parametrize("name,cfg,T,align", GEMM_CASES, ids=[c[0] for c in GEMM_CASES])
def test_grouped_swiglu_parity(name, cfg, T, align):
    inp = make_inputs(cfg, T=T)
    g = _gpu(inp)
    dm = M.dims_of(cfg, T=inp["T"], align=align)
    _, idx, _ = _route(dm, g)
    pm = _permute(dm, idx, g["x"])
    h, y = _grouped(dm, pm["x_perm"], pm["offsets"], g)
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    off = pm["offsets"].cpu().numpy()
    xp = pm["x_perm"]
    # every expert when the shape is small; a spread of experts otherwise
    experts = range(cfg.E) if cfg.d * cfg.I <= 512 * 256 else range(0, cfg.E, 9)
    for e in experts:
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        xe = xp[a:b].cpu()
        o_ref, h_ref, _, _ = O.swiglu_expert(xe, inp["w1"][e], inp["w3"][e], inp["w2"][e])
        PU.check_bf16_elementwise(h[a:b], h_ref, f"h_perm expert {e}")
        # the down GEMM (fp32 out) against the oracle fed with the GPU's own bf16 h
        hg, w2 = PU.to_np(h[a:b]), inp["w2"][e].double().numpy()
        PU.check_fp32_sum(y[a:b], hg @ w2.T, np.abs(hg) @ np.abs(w2).T, f"y_perm expert {e}")


# ------------------------------------------------------------------ combine

def test_combine_parity():
    T, d, E, k = 300, 256, 16, 4
    dm = M.dims(T, d, E, k, 64, 2, 16)
    cap = M.capacity(dm)
    gen = torch.Generator().manual_seed(3)
    y_perm = torch.randn((cap, d), generator=gen)
    rows = torch.randperm(cap, generator=gen)[:T * k].to(torch.int32)
    w = torch.rand((T, k), generator=gen)
    w = w / w.sum(1, keepdim=True)
    y_sh = torch.randn((T, d), generator=gen)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    M.combine(dm, y_perm.to(DEV), rows.to(DEV), w.to(DEV), y_sh.to(DEV), y)
    ref = y_sh.double().numpy() + O.unpermute_sum(y_perm, rows.numpy(), w, T, k)
    # one rounding of an fp32 sum: elementwise bf16 bound
    PU.check_bf16_elementwise(y, ref, "combine")
    y2 = torch.empty_like(y)
    M.combine(dm, y_perm.to(DEV), rows.to(DEV), w.to(DEV), None, y2)
    PU.check_bf16_elementwise(y2, O.unpermute_sum(y_perm, rows.numpy(), w, T, k), "combine S=0")


# ------------------------------------------------------------------ fused forward

def _forward(inp, align=16):
    g = _gpu(inp)
    layer = M.MoELayer(g, align=align)
    y = layer(g["x"])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    return y, M.workspace_views(layer.dims(inp["T"]), layer.workspace(inp["T"]))


FWD_CASES = [
    ("tiny_full", TINY, None, 16),
    ("tiny_align128", TINY, None, 128),
    ("small_ragged_T333", small_config(T=333, d=256, E=16, k=4, I=192), None, 16),
    ("single_token", small_config(T=1, d=256, E=16, k=4, I=128), None, 16),
    ("pair_prefill_T700", small_config(T=700, d=512, E=16, k=4, I=256), None, 16),
    ("pair_prefill_align128", small_config(T=700, d=512, E=16, k=4, I=256), None, 128),
    ("no_shared", MoEConfig("noshared", T=200, d=256, E=32, k=6, S=0, I=128,
                            bias="uniform0.01"), None, 16),
    ("one_shared_k8", MoEConfig("s1k8", T=130, d=384, E=64, k=8, S=1, I=256,
                                bias="normal0.05"), None, 16),
]


@pytest.mark.parametrize("name,cfg,T,align", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_forward_parity_small(name, cfg, T, align):
    inp = make_inputs(cfg, T=T)
    y, v = _forward(inp, align)
    ref = O.forward(PU.np_inputs(inp), align=align, idx=None)
    ties = PU.check_routing(v["topk_idx"].cpu().numpy(), ref["keys"], ref["idx"], cfg.k)
    PU.check_probs(v["probs"], ref["probs"])
    if ties:
        ref = O.forward(PU.np_inputs(inp), align=align, idx=v["topk_idx"].cpu().numpy())
    _check_permutation(M.dims_of(cfg, T=inp["T"], align=align),
                       {k: v[k] for k in ("counts", "offsets", "row_of", "token_of_row", "x_perm")},
                       v["topk_idx"].cpu(), inp["x"])
    spec = cfg in CONFIGS.values()
    if cfg.S > 0:
        PU.check_bf16_elementwise(v["h_shared"], ref["h_shared"], "h_shared")
        PU.check_output(v["y_shared"], ref["y_shared"], "y_shared", spec=spec)
    routed_abs = O.unpermute_sum(np.abs(ref["y_perm"]), ref["row_of"], ref["w"], inp["T"], cfg.k)
    PU.check_output(y, ref["y"], spec=spec, routed_abs=routed_abs)


def test_forward_empty_batch():
    cfg = small_config(T=0, d=256, E=16, k=4, I=128)
    inp = make_inputs(cfg)
    g = _gpu(inp)
    layer = M.MoELayer(g)
    y = layer(g["x"])
    torch.cuda.synchronize()
    assert y.shape == (0, 256)
    assert M.device_status() == M.MOE_OK


def test_forward_deterministic():
    inp = make_inputs(0)
    g = _gpu(inp)
    layer = M.MoELayer(g)
    y1 = layer(g["x"]).clone()
    y2 = layer(g["x"]).clone()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# ------------------------------------------------------------------ full-size configurations

@pytest.mark.parametrize("cfg,n_sample,seed",
                         [(DECODE, 128, 1), (PREFILL_BALANCED, 1024, 2),
                          (PREFILL_SKEWED, 1024, 3)],
                         ids=["decode", "prefill_balanced", "prefill_skewed"])
def test_forward_full_size_sampled(cfg, n_sample, seed):
    """The full configuration on the device: the whole routing and permutation
    are compared; the output on a seeded sample of tokens (per-token oracle;
    every token of the decode batch, 1024 of a prefill batch)."""
    inp = make_inputs(cfg, device=DEV)
    layer = M.MoELayer(inp)
    y = layer(inp["x"])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    v = M.workspace_views(layer.dims(cfg.T), layer.workspace(cfg.T))
    host = PU.np_inputs(inp)
    r = O.route(host["x"], host["w_gate"], host["bias"], cfg.k)
    idx_gpu = v["topk_idx"].cpu().numpy()
    PU.check_routing(idx_gpu, r["keys"], r["idx"], cfg.k)
    PU.check_probs(v["probs"], r["probs"])
    pm = O.permute(idx_gpu, cfg.E, 16)
    np.testing.assert_array_equal(v["offsets"].cpu().numpy(), pm["offsets"])
    np.testing.assert_array_equal(v["row_of"].cpu().numpy(), pm["row_of"])
    np.testing.assert_array_equal(v["token_of_row"].cpu().numpy(), pm["token_of_row"])
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(cfg.T, size=n_sample, replace=False))
    ref = O.forward_tokens(host, toks, idx=idx_gpu[toks])
    PU.check_output(y[torch.as_tensor(toks, device=DEV)], ref["y"], "y (sampled)")


@pytest.mark.parametrize("cfg", [DECODE, PREFILL_BALANCED, PREFILL_SKEWED],
                         ids=["decode", "prefill_balanced", "prefill_skewed"])
def test_forward_full_size_every_segment(cfg):
    """Every tile of both grouped GEMMs at the full configuration (one-CTA
    kernels at decode, CTA pairs at prefill): h_perm and y_perm of every
    non-empty expert segment, and the shared experts' h and fp32 y, each
    against the oracle's SwiGLU expert fed the GPU's own permuted rows (for
    the down projection, the GPU's own bf16 h: exactly what that GEMM read).
    Segment rows beyond a segment's tokens (padding) must be exactly zero."""
    inp = make_inputs(cfg, device=DEV)
    layer = M.MoELayer(inp)
    layer(inp["x"])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    v = M.workspace_views(layer.dims(cfg.T), layer.workspace(cfg.T))
    off = v["offsets"].cpu().numpy()
    counts = v["counts"].cpu().numpy()
    done = 0
    for e in range(cfg.E):
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        xe = v["x_perm"][a:b]
        _, h_ref, _, _ = O.swiglu_expert(xe, inp["w1"][e], inp["w3"][e], inp["w2"][e])
        PU.check_bf16_elementwise(v["h_perm"][a:b], h_ref, f"h_perm expert {e}")
        w2 = inp["w2"][e].double().cpu().numpy()
        hg = PU.to_np(v["h_perm"][a:b])
        PU.check_fp32_sum(v["y_perm"][a:b], hg @ w2.T, np.abs(hg) @ np.abs(w2).T,
                          f"y_perm expert {e}")
        pad = slice(a + int(counts[e]), b)
        assert not v["h_perm"][pad].any() and not v["y_perm"][pad].any(), f"padding of {e}"
        done += 1
    assert done == int((counts > 0).sum())
    S, I = cfg.S, cfg.I
    h_sh = v["h_shared"]
    y_ref = np.zeros((cfg.T, cfg.d))
    y_abs = np.zeros((cfg.T, cfg.d))
    for s_ in range(S):
        _, h_ref, _, _ = O.swiglu_expert(inp["x"], inp["ws1"][s_], inp["ws3"][s_], inp["ws2"][s_])
        hs = h_sh[:, s_ * I:(s_ + 1) * I]
        PU.check_bf16_elementwise(hs, h_ref, f"h_shared expert {s_}")
        w2 = inp["ws2"][s_].double().cpu().numpy()
        hg = PU.to_np(hs)
        y_ref += hg @ w2.T
        y_abs += np.abs(hg) @ np.abs(w2).T
    PU.check_fp32_sum(v["y_shared"], y_ref, y_abs, "y_shared")


@pytest.mark.parametrize("cfg,T", [(small_config(T=700, d=512, E=16, k=4, I=256), None),
                                   (PREFILL_BALANCED, None), (DECODE, None), (TINY, None)],
                         ids=["pair_prefill_T700", "prefill_balanced", "decode", "tiny"])
def test_fused_forward_equals_the_step_calls(cfg, T):
    """moe_forward runs the shared experts' GEMMs on a side stream (beside
    the permutation at prefill sizes, beside the router and the permutation
    on half of the SMs at decode sizes) and launches the routed GEMMs alone;
    the result must be bit-identical to the public step calls (moe_route,
    moe_permute, moe_grouped_swiglu, moe_combine) on the same batch, whose
    grouped-GEMM call runs the routed experts in one launch per projection.
    The combine is fed the fused call's fp32 shared output."""
    inp = make_inputs(cfg, T=T, device=DEV)
    g = _gpu(inp)
    layer = M.MoELayer(g)
    y = layer(g["x"]).clone()
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    dm = M.dims_of(cfg, T=inp["T"])
    v = M.workspace_views(dm, layer.workspace(inp["T"]))
    probs, idx, w = _route(dm, g)
    pm = _permute(dm, idx, g["x"])
    h, yp = _grouped(dm, pm["x_perm"], pm["offsets"], g)
    y2 = torch.empty_like(y)
    M.combine(dm, yp, pm["row_of"], w, v["y_shared"], y2)
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    eq = lambda a, b: torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a.view(torch.int16),  # noqa: E731
                                  b.view(torch.int32) if b.dtype == torch.float32 else b.view(torch.int16))
    assert eq(probs, v["probs"]) and torch.equal(idx, v["topk_idx"]) and eq(w, v["topk_w"])
    for name in ("counts", "offsets", "row_of"):
        assert torch.equal(pm[name], v[name]), name
    used = int(pm["offsets"][-1])
    assert eq(pm["x_perm"][:used], v["x_perm"][:used])
    assert eq(h[:used], v["h_perm"][:used]) and eq(yp[:used], v["y_perm"][:used])
    assert eq(y2, y)
