"""bench.py's own bookkeeping, on CPU: the kernel launches it claims per step
follow the library's launch sequence.  The dense FFN's count depends on
which of its GEMMs the library splits over K; that decision is read back
from the library itself (a split GEMM's fp32 partials make the workspace
larger than h alone) and compared with bench.py's count."""
import ctypes
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from fine_grained_moe_fp32_b200 import moe as M  # noqa: E402
from fine_grained_moe_fp32_b200.workloads import CONFIGS  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    return M.load()


def test_forward_launch_counts():
    # decode: router GEMM + top-k, one-CTA permutation index + row copy,
    # shared gate/up + down on the side stream, routed gate/up + down, combine
    dec = CONFIGS[1]
    assert bench.forward_kernels(dec.T, bench.shared_on_side_stream(dec, dec.T, False)) == 9
    # prefill: count / scan / scatter + row copy
    pre = CONFIGS[2]
    assert bench.forward_kernels(pre.T, bench.shared_on_side_stream(pre, pre.T, False)) == 11
    # training forward: one stream, the shared experts inside the routed launches
    tr = CONFIGS[4]
    assert not bench.shared_on_side_stream(tr, tr.T, True)
    assert bench.forward_kernels(tr.T) == 9


@pytest.mark.parametrize("T,d,I", [(128, 5120, 11264), (256, 5120, 11264), (4096, 5120, 11264),
                                   (128, 512, 1024), (300, 512, 384), (300, 512, 1408),
                                   (37, 256, 256), (20, 512, 256)])
def test_dense_launch_count_matches_the_library_split(lib, T, d, I):
    need = lib.moe_dense_workspace_size(ctypes.byref(M.dense_dims(T=T, d=d, I=I)))
    h = T * I * 2
    split_any = need > h + 4096          # partials beyond h (and its alignment)
    n = bench.dense_kernels(T, d, I)
    assert n in (3, 4, 5)
    assert (n > 3) == split_any, (T, d, I, n, need, h)
