"""Runtime behaviour on the GPU: bounded waits that run out report a timeout
and leave the context usable; the phase-event measurement hook."""
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


def _layer(T=200):
    inp = make_inputs(0, T=T)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    return g, M.MoELayer(g)


def test_bounded_wait_times_out_and_recovers():
    """A 1 ns wait limit makes the GEMM pipelines give up at their first
    unready barrier; the kernels record MOE_ERR_TIMEOUT, drain their copies,
    free tensor memory and return.  With the default limit restored the
    same call is correct again."""
    g, layer = _layer()
    y_ok = layer(g["x"]).clone()
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    try:
        M.set_wait_limit_ns(1)
        layer(g["x"])
        assert M.device_status() == M.MOE_ERR_TIMEOUT
    finally:
        M.set_wait_limit_ns(0)
    y = layer(g["x"])
    assert M.device_status() == M.MOE_OK
    assert torch.equal(y.view(torch.int16), y_ok.view(torch.int16))


def test_phase_events_cover_the_step():
    g, layer = _layer()
    layer(g["x"])
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    M.set_phase_events(ev)
    try:
        outer[0].record()
        layer(g["x"])
        outer[1].record()
    finally:
        M.set_phase_events(None)
    torch.cuda.synchronize()
    parts = [ev[i].elapsed_time(ev[i + 1]) for i in range(5)]
    assert all(p >= 0 for p in parts)
    assert sum(parts) <= outer[0].elapsed_time(outer[1]) * 1.01 + 0.05


@pytest.mark.parametrize("name,T", [("TINY", None), ("DECODE", None), ("PREFILL_BALANCED", 1024)],
                         ids=["tiny", "decode", "prefill_T1024_cta_pairs"])
def test_forward_captures_into_a_cuda_graph(name, T):
    """moe_forward issues only stream work (no host sync, no allocation), so it
    can be captured once and replayed: every replay gives the eager result bit
    for bit, and a replay follows new input values written in place."""
    import torch
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200 import workloads as W
    cfg = getattr(W, name)
    make_inputs = W.make_inputs
    inp = make_inputs(cfg, device="cuda", T=T)
    layer = M.MoELayer(inp)
    x = inp["x"].clone()
    y = torch.empty((x.shape[0], cfg.d), dtype=torch.bfloat16, device="cuda")
    eager = layer(x).clone()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        layer(x, y, stream=st)          # warm-up on the capture stream
        st.synchronize()
        with torch.cuda.graph(g, stream=st):
            layer(x, y, stream=st)
    torch.cuda.current_stream().wait_stream(st)
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), eager.view(torch.int16))
    x2 = make_inputs(cfg, device="cuda", T=T, seed=5, weights=False)["x"]
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    assert torch.equal(y.view(torch.int16), layer(x2).view(torch.int16))


def test_out_of_range_row_is_skipped_and_flagged_by_the_checks_build():
    """moe_combine given a row index past the permuted buffer for one pair:
    that pair contributes nothing in both builds (the kernel's own range
    test skips it); the MOE_CHECKS build also records MOE_ERR_BOUNDS, the
    normal build records nothing.  Every other token is unaffected."""
    T, d, E, k = 8, 256, 16, 2
    dm = M.dims(T, d, E, k, 64, 0, 16)
    cap = M.capacity(dm)
    gen = torch.Generator().manual_seed(9)
    y_perm = torch.randn((cap, d), generator=gen).cuda()
    rows = torch.arange(T * k, dtype=torch.int32)
    w = torch.full((T, k), 0.5)
    bad = rows.clone()
    bad[3] = cap + 5                  # token 1, slot 1
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    y_ok = torch.empty_like(y)
    M.combine(dm, y_perm, rows.cuda(), w.cuda(), None, y_ok)
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    M.combine(dm, y_perm, bad.cuda(), w.cuda(), None, y)
    status = M.device_status()
    assert status == (M.MOE_ERR_BOUNDS if M.CHECKS else M.MOE_OK)
    assert M.device_status() == M.MOE_OK        # cleared by the read
    keep = [t for t in range(T) if t != 1]
    assert torch.equal(y[keep].view(torch.int16), y_ok[keep].view(torch.int16))
    want = (0.5 * y_perm[2].float()).to(torch.bfloat16)   # token 1's first slot alone
    assert torch.equal(y[1].view(torch.int16), want.view(torch.int16))
