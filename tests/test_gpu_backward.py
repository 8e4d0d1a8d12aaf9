"""Parity of the backward (moe_forward_train + moe_backward through the C ABI)
with the fp64 oracle: the combine, renormalisation and softmax backward
(dx, dWg), the expert dgrad/wgrad grouped GEMMs with the SwiGLU backward
(dW1, dW3, dW2 and the shared experts' gradients).  The routing choice is
held fixed; where the GPU took a tie the other way, the oracle is run with
the GPU's selection.  The full-size fwd+bwd workload is checked on a
256-token slice (its weights, 256 of its tokens) with a sample of experts."""
import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import (CONFIGS, MoEConfig, make_inputs, small_config, FWD_BWD, TINY)
from oracle import moe_oracle as O
import parity_utils as PU
import bf16_emulation as EM

pytestmark = pytest.mark.gpu


def _dy(T, d, seed=11):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((T, d), generator=g).to(torch.bfloat16)


GRAD_NAMES = ("dx", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2")


def _run(inp, align=16):
    """forward_train, then the backward twice on the same workspace: bf16
    outputs (moe_backward) and fp32 outputs (moe_backward_f32)."""
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    layer = M.MoELayer(g, align=align)
    y_inf = layer(g["x"]).clone()
    y = layer.forward_train(g["x"])
    T = inp["T"]
    grads = layer.backward(g["x"], g["dy"], layer.alloc_grads(T, torch.bfloat16))
    grads32 = layer.backward(g["x"], g["dy"], layer.alloc_grads(T, torch.float32))
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    idx = M.workspace_views(layer.dims(T), layer.train_workspace(T))["topk_idx"]
    return y_inf, y, grads, grads32, idx.cpu().numpy()


def _oracle(inp, idx_gpu, experts=None):
    host = PU.np_inputs(inp)
    f = O.forward(host)
    if (f["idx"] != idx_gpu).any():
        PU.check_routing(idx_gpu, f["keys"], f["idx"], inp["cfg"].k)
        f = O.forward(host, idx=idx_gpu)
    return f, O.backward(host, host["dy"], f, experts=experts)


def _check_bf16_is_rounding(grads, grads32):
    """moe_backward's outputs are exactly the bf16 roundings (to nearest even)
    of moe_backward_f32's, and both give the same fp32 dw_gate."""
    assert torch.equal(grads["dw_gate"], grads32["dw_gate"]), "dw_gate differs between calls"
    for name in GRAD_NAMES:
        a, b = grads[name], grads32[name]
        assert torch.equal(a.view(torch.int16), b.to(torch.bfloat16).view(torch.int16)), (
            f"{name}: bf16 output is not the rounding of the fp32 output")


def _check_all(inp, y_inf, y, grads, grads32, f, b, experts=None, spec=True):
    """Every gradient is checked; all failures are reported together with
    each tensor's max error / rms.

    spec (the workload configurations): the fp32 dx, dw_gate and shared
    experts' weight gradients within 2e-2 rms of the oracle.  The routed
    experts' weight gradients keep the arithmetic's bound, and only after a
    CPU emulation of the bf16 MMA operands (everything else exact) on the same
    inputs shows that it misses 2e-2 rms itself.  Off-spec shapes: every
    gradient within the arithmetic's bound."""
    assert torch.equal(y.view(torch.int16), y_inf.view(torch.int16)), "training forward differs"
    _check_bf16_is_rounding(grads, grads32)
    ex = list(range(inp["cfg"].E) if experts is None else experts)
    off, I = f["offsets"], inp["cfg"].I
    xp, hp, dyp, dgu = f["x_perm"], f["h_perm"], b["dy_perm"], b["dgu_perm"]

    def seg(a, e):
        return np.abs(a[int(off[e]):int(off[e + 1])])

    # magnitude sums of the routed weight-gradient products (oracle values)
    abs_sums = {"dw1": np.stack([seg(dgu, e)[:, :I].T @ seg(xp, e) for e in ex]),
                "dw3": np.stack([seg(dgu, e)[:, I:].T @ seg(xp, e) for e in ex]),
                "dw2": np.stack([seg(dyp, e).T @ seg(hp, e) for e in ex])}
    kappa = {"dw1": 5, "dw3": 5, "dw2": 3}
    emul = EM.routed_weight_grads(PU.np_inputs(inp), f, b, ex)
    report, failed = [], []

    def run(fn):
        try:
            fn()
        except AssertionError as e:
            failed.append(str(e))

    def check_y():
        routed_abs = O.unpermute_sum(np.abs(f["y_perm"]), f["row_of"], f["w"], inp["T"],
                                     inp["cfg"].k)
        r = PU.check_output(y, f["y"], "y", spec=spec, routed_abs=routed_abs)
        report.append(f"y {r:.4f} (bf16 floor {PU.bf16_floor(f['y']):.4f})")
    run(check_y)
    names = ["dx", "dw_gate"] + (["dws1", "dws3", "dws2"] if inp["cfg"].S > 0 else [])
    for name in names:
        def one(name=name):
            got, ref = grads32[name], b[name]
            if spec:
                r = PU.check_spec(got, ref, name)
            else:
                r = PU.check_grad(got, ref, name, rounded_output=False)
            line = f"{name} {r:.4f}"
            if name != "dw_gate":
                line += f" (bf16 output {PU.rel_err(grads[name], ref):.4f}, " \
                        f"floor {PU.bf16_floor(ref):.4f})"
            report.append(line)
        run(one)
    for name in ("dw1", "dw3", "dw2"):
        def routed(name=name):
            got = np.stack([PU.to_np(grads32[name][e]) for e in ex])
            ref = np.stack([b[name][e] for e in ex])
            em = np.stack([emul[name][e] for e in ex])
            r_em = PU.rel_err(em, ref)
            if spec and r_em <= PU.Y_RMS_FRAC:
                # bf16 operands can meet the bound here: so must the GPU
                r = PU.check_spec(got, ref, name)
            else:
                r = PU.check_grad(got, ref, name, abs_sums[name], kappa[name],
                                  rounded_output=False)
            report.append(f"{name} {r:.4f} (bf16-operand emulation {r_em:.4f}, "
                          f"gpu vs emulation {PU.rel_err(got, em, PU.rms(ref)):.4f}; "
                          f"bf16 output {PU.rel_err(np.stack([PU.to_np(grads[name][e]) for e in ex]), ref):.4f})")
        run(routed)
    print("max err / rms:", ", ".join(report))
    assert not failed, "; ".join(failed)


CASES = [
    ("tiny_full", TINY, None),
    ("small_E16_T200", small_config(T=200, d=256, E=16, k=4, I=128), None),
    ("E32_S1_k8_T97", MoEConfig("s1k8", T=97, d=384, E=32, k=8, S=1, I=256, bias="normal0.05"),
     None),
    # ~256 rows per expert: several token tiles per dgrad, several K chunks per wgrad
    ("E8_k2_T1024_long_segments", small_config(T=1024, d=256, E=8, k=2, I=128), None),
    # ~512 rows per expert: weight gradients with the A panel resident (<= 512
    # rows) and with 512-row panels reloaded per N tile (longer segments)
    ("E4_k1_T2048_panels_over_512", small_config(T=2048, d=256, E=4, k=1, I=128), None),
    # hidden size past 8192: every 16-byte vector of a token's row, not a fixed count per thread
    ("E8_k2_T64_d8448_wide_rows", small_config(T=64, d=8448, E=8, k=2, I=128), None),
]


@pytest.mark.parametrize("name,cfg,T", CASES, ids=[c[0] for c in CASES])
def test_backward_parity_small(name, cfg, T):
    inp = make_inputs(cfg, T=T)
    inp["dy"] = _dy(inp["T"], cfg.d)
    y_inf, y, grads, grads32, idx = _run(inp)
    f, b = _oracle(inp, idx)
    _check_all(inp, y_inf, y, grads, grads32, f, b, spec=cfg in CONFIGS.values())
    # experts that received no token have exactly zero gradient
    counts = np.bincount(idx.ravel(), minlength=cfg.E)
    for e in np.nonzero(counts == 0)[0]:
        assert not grads["dw1"][e].any() and not grads["dw2"][e].any()


@pytest.mark.parametrize("T", [256, 1024], ids=["T256_one_cta", "T1024_cta_pairs"])
def test_backward_full_size_slice(T):
    """The fwd+bwd workload's layer (d=5120, E=128, I=1408, 2 shared) on its
    first T tokens (256: the one-CTA GEMMs for decode-sized segments; 1024:
    the paired-CTA GEMMs of prefill-sized batches): dx, dWg and the shared
    experts' gradients in full, the routed experts' gradients on a seeded
    sample of experts."""
    cfg = FWD_BWD
    inp = make_inputs(cfg, T=T, device="cuda")
    y_inf, y, grads, grads32, idx = _run(inp)
    rng = np.random.default_rng(4)
    experts = sorted(set(rng.choice(cfg.E, size=6, replace=False).tolist()) | {int(idx[0, 0])})
    f, b = _oracle(inp, idx, experts=experts)
    _check_all(inp, y_inf, y, grads, grads32, f, b, experts=experts, spec=True)


def test_backward_empty_batch():
    cfg = small_config(T=0, d=256, E=16, k=4, I=128)
    inp = make_inputs(cfg)
    inp["dy"] = torch.empty((0, 256), dtype=torch.bfloat16)
    y_inf, y, grads, grads32, idx = _run(inp)
    for gr in (grads, grads32):
        assert not gr["dw_gate"].any()
        assert not gr["dw1"].any() and not gr["dws2"].any() and not gr["dws1"].any()


def test_backward_kernels_on_their_own_inputs():
    """Each backward grouped GEMM against fp64 math fed with the GPU's own
    bf16 inputs from the workspace (isolates one kernel at a time):
    dGU from dy_perm, w2, g, u; dx_perm from dGU, w1, w3; dW2 from dy_perm and
    h_perm; dW1 / dW3 from dGU and x_perm; the same for the shared experts."""
    cfg = small_config(T=200, d=256, E=16, k=4, I=128)
    inp = make_inputs(cfg)
    inp["dy"] = _dy(200, 256)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    layer = M.MoELayer(g)
    layer.forward_train(g["x"])
    grads = layer.backward(g["x"], g["dy"])
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    v = M.train_workspace_views(layer.dims(200), layer.train_workspace(200))
    f64 = lambda t: t.double().cpu().numpy()  # noqa: E731
    off = v["offsets"].cpu().numpy()
    I, S = cfg.I, cfg.S
    w1, w3, w2 = f64(g["w1"]), f64(g["w3"]), f64(g["w2"])
    fails = []

    def chk(got, ref, what):
        try:
            PU.check_bf16_elementwise(got, ref, what)
        except AssertionError as e:
            fails.append(str(e)[:200])

    dyp, gp, up, dgu, hp, xp = (f64(v[n]) for n in ("dy_perm", "g_perm", "u_perm", "dgu_perm",
                                                     "h_perm", "x_perm"))
    for e in range(cfg.E):
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        dh = dyp[a:b] @ w2[e]
        sg = 1 / (1 + np.exp(-gp[a:b]))
        dg = dh * up[a:b] * sg * (1 + gp[a:b] * (1 - sg))
        du = dh * gp[a:b] * sg
        chk(v["dgu_perm"][a:b], np.concatenate([dg, du], 1), f"dGU expert {e}")
        dxp = dgu[a:b, :I] @ w1[e] + dgu[a:b, I:] @ w3[e]
        chk(v["dx_perm"][a:b], dxp, f"dx_perm expert {e}")
        chk(grads["dw2"][e], dyp[a:b].T @ hp[a:b], f"dW2 expert {e}")
        chk(grads["dw1"][e], dgu[a:b, :I].T @ xp[a:b], f"dW1 expert {e}")
        chk(grads["dw3"][e], dgu[a:b, I:].T @ xp[a:b], f"dW3 expert {e}")
    dy, x = f64(g["dy"]), f64(g["x"])
    gs, us, dgus, hs = (f64(v[n]) for n in ("g_shared", "u_shared", "dgu_shared", "h_shared"))
    ws1, ws3, ws2 = f64(g["ws1"]), f64(g["ws3"]), f64(g["ws2"])
    dh = np.concatenate([dy @ ws2[s] for s in range(S)], 1)
    sg = 1 / (1 + np.exp(-gs))
    chk(v["dgu_shared"], np.concatenate([dh * us * sg * (1 + gs * (1 - sg)), dh * gs * sg], 1),
        "dGU shared")
    SI = S * I
    for s in range(S):
        chk(grads["dws2"][s], dy.T @ hs[:, s * I:(s + 1) * I], f"dWs2 {s}")
        chk(grads["dws1"][s], dgus[:, s * I:(s + 1) * I].T @ x, f"dWs1 {s}")
        chk(grads["dws3"][s], dgus[:, SI + s * I:SI + (s + 1) * I].T @ x, f"dWs3 {s}")
    assert not fails, "\n".join(fails[:12]) + f"\n({len(fails)} failures)"
