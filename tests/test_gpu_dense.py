"""Parity of moe_dense_swiglu (the first layer's dense SwiGLU FFN, run on the
grouped GEMM kernels as one group of every token) with the fp64 oracle: small
shapes in full (the decode-sized one-CTA kernels, the paired-CTA kernels, a
ragged token count, the one-CTA prefill kernel when I is not a multiple of
128), the full-size layer (d = 5120, I = 11264) on sampled tokens, and an
empty batch.  The bound per element is one bf16 rounding of |y| plus
1e-2 rms (h is stored in bf16, sums run in fp32)."""
import numpy as np
import pytest
import torch

from fine_grained_moe_fp32_b200 import moe as M
from fine_grained_moe_fp32_b200.workloads import DENSE_I, make_dense_inputs
from oracle import moe_oracle as O
import parity_utils as PU

pytestmark = pytest.mark.gpu


def _run(inp):
    dm = M.dense_dims(inp["T"], inp["d"], inp["I"])
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    y = torch.full((inp["T"], inp["d"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.dense_swiglu(dm, g["x"], g["w1"], g["w3"], g["w2"], y,
                   M.alloc_workspace(M.dense_workspace_size(dm)))
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
    return y


CASES = [
    ("T1_decode_path", 1, 256, 128),
    ("T20_decode_path", 20, 512, 256),
    ("T37_pairs_ragged", 37, 256, 256),
    ("T300_pairs", 300, 512, 384),
    ("T200_one_cta_I192", 200, 256, 192),
    # too few tiles for the SM pairs: the gate/up GEMM (2 K splits: fp32 g and
    # u partials summed before the SwiGLU) and the down GEMM are split over K
    # (T300_pairs: the gate/up GEMM alone)
    ("T128_down_split_4", 128, 512, 1024),
    ("T300_down_split_ragged", 300, 512, 1408),
]


@pytest.mark.parametrize("name,T,d,I", CASES, ids=[c[0] for c in CASES])
def test_dense_small(name, T, d, I):
    inp = make_dense_inputs(T, d, I)
    y = _run(inp)
    ref = O.dense_swiglu(inp["x"], inp["w1"], inp["w3"], inp["w2"])
    PU.check_output(y, ref, f"dense y ({name})", spec=False)


def test_dense_full_size_sampled():
    """d = 5120, I = 11264 (the MoE layer's activated width), T = 4096 on the
    device; the output checked on a seeded sample of tokens."""
    inp = make_dense_inputs(4096, 5120, DENSE_I, device="cuda")
    y = _run(inp)
    toks = np.sort(np.random.default_rng(7).choice(4096, size=16, replace=False))
    idx = torch.as_tensor(toks, device="cuda")
    ref = O.dense_swiglu(inp["x"][idx].cpu(), inp["w1"].cpu(), inp["w3"].cpu(), inp["w2"].cpu())
    PU.check_output(y[idx], ref, "dense y (sampled)", spec=False)


def test_dense_full_size_T128_down_split():
    """d = 5120, I = 11264 at T = 128: the gate/up GEMM's 88 tiles (5 K
    splits) and the down GEMM's 20 tiles (7 K splits) are split over K (fp32
    partials summed in a fixed order, one rounding each); every token
    against the oracle."""
    inp = make_dense_inputs(128, 5120, DENSE_I, device="cuda")
    y = _run(inp)
    ref = O.dense_swiglu(inp["x"].cpu(), inp["w1"].cpu(), inp["w3"].cpu(), inp["w2"].cpu())
    PU.check_output(y, ref, "dense y (T=128)", spec=False)


def test_dense_empty_batch():
    dm = M.dense_dims(0, 256, 128)
    e = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    M.dense_swiglu(dm, e, w, w, w.T.contiguous(), e.clone(), M.alloc_workspace(1))
    torch.cuda.synchronize()
    assert M.device_status() == M.MOE_OK
