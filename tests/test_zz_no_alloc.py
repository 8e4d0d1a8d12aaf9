"""moe_route_noalloc, the router entry point for callers that cannot
allocate device memory when they route (a plugin hook handed a stream and
buffers but no allocator, or a serving loop that forbids allocation after
warm-up): its output must match moe_route's, called through the C ABI, on two
calls in a row that share the library's built-in scratch."""
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import make_inputs, PREFILL_BALANCED, TINY

pytestmark = pytest.mark.gpu


def _outputs(dm, dev="cuda"):
    return (torch.full((dm.T, dm.E), float("nan"), dtype=torch.float32, device=dev),
            torch.full((dm.T, dm.k), -7, dtype=torch.int32, device=dev),
            torch.full((dm.T, dm.k), float("nan"), dtype=torch.float32, device=dev))


def _with_workspace(dm, g):
    probs, idx, w = _outputs(dm)
    ws = M.alloc_workspace(M.route_workspace_size(dm))
    M.route(dm, g["x"], g["w_gate"], g["bias"], probs, idx, w, ws)
    return probs, idx, w


def _no_alloc(dm, g):
    probs, idx, w = _outputs(dm)
    M.route_noalloc(dm, g["x"], g["w_gate"], g["bias"], probs, idx, w)
    return probs, idx, w


def test_no_alloc_route_matches_moe_route_on_two_calls():
    cases = [(PREFILL_BALANCED, 4096, 0), (TINY, 256, 3)]   # big call first, then a small one
    for cfg, T, seed in cases:
        inp = make_inputs(cfg, T=T, seed=seed, weights=False)
        g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
        dm = M.dims_of(cfg, T=T)
        ref = _with_workspace(dm, g)
        got = _no_alloc(dm, g)
        torch.cuda.synchronize()
        assert M.device_status() == M.MOE_OK
        # the same kernels on the same partial-logit layout: bit-identical
        for a, b in zip(got, ref):
            assert torch.equal(a, b)

