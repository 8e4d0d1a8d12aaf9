"""The C ABI library loads and exports every symbol include/moe_b200.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from fine_grained_moe_fp32_b200 import build as B
from fine_grained_moe_fp32_b200 import moe as M

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "moe_b200.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(M.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_is_sm100a_build():
    out = B.ARCH
    assert "arch=compute_100a,code=sm_100a" in out


def test_capacity_and_sizes(lib):
    dm = M.dims(T=4096, d=5120, E=128, k=6, I=1408, n_shared=2, align=16)
    assert M.capacity(dm) == 4096 * 6 + 128 * 15
    L = M.forward_layout(dm)
    assert L["total"] == M.workspace_size(dm)
    offs = [L[n] for n in ("route_partials", "probs", "topk_idx", "topk_w", "counts", "offsets",
                           "row_of", "token_of_row", "permute_scratch", "x_perm", "h_perm",
                           "y_perm", "h_shared", "y_shared")]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    cap = M.capacity(dm)
    assert L["h_perm"] - L["x_perm"] >= cap * 5120 * 2
    assert L["total"] - L["y_shared"] >= 4096 * 5120 * 4
    assert M.route_workspace_size(dm) > 0
    assert M.permute_workspace_size(dm) == 2 * 16 * 128 * 4


@pytest.mark.parametrize("field,value,status", [
    ("d", 100, M.MOE_ERR_UNSUPPORTED_SHAPE),
    ("I", 96, M.MOE_ERR_UNSUPPORTED_SHAPE),
    ("E", 129, M.MOE_ERR_UNSUPPORTED_SHAPE),
    ("k", 9, M.MOE_ERR_UNSUPPORTED_SHAPE),
    ("align", 8, M.MOE_ERR_UNSUPPORTED_SHAPE),
    ("T", -1, M.MOE_ERR_INVALID_ARG),
    ("E", 0, M.MOE_ERR_INVALID_ARG),
])
def test_bad_dims_rejected_on_host(lib, field, value, status):
    dm = M.dims(T=64, d=256, E=16, k=4, I=128, n_shared=2, align=16)
    setattr(dm, field, value)
    rc = lib.moe_forward(ctypes.byref(dm), None, None, None, None, None, None, None, None, None,
                         None, None, 0, None)
    assert rc == status
    assert lib.moe_workspace_size(ctypes.byref(dm)) == 0


def test_null_pointers_and_workspace_rejected_on_host(lib):
    dm = M.dims(T=64, d=256, E=16, k=4, I=128, n_shared=2, align=16)
    rc = lib.moe_forward(ctypes.byref(dm), None, None, None, None, None, None, None, None, None,
                         None, None, 0, None)
    assert rc == M.MOE_ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check fails first
    rc = lib.moe_forward(ctypes.byref(dm), fake, fake, None, fake, fake, fake, fake, fake, fake,
                         fake, fake, 16, None)
    assert rc == M.MOE_ERR_WORKSPACE
    rc = lib.moe_route(ctypes.byref(dm), fake, fake, None, None, fake, fake, None, 0, None)
    assert rc == M.MOE_ERR_WORKSPACE
    misaligned = ctypes.c_void_p((1 << 20) + 2)
    rc = lib.moe_route(ctypes.byref(dm), misaligned, fake, None, None, fake, fake, fake,
                       1 << 30, None)
    assert rc == M.MOE_ERR_INVALID_ARG


def test_balance_calls_rejected_on_host(lib):
    dm = M.dims(T=64, d=256, E=16, k=4, I=128, n_shared=2, align=16)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails first
    assert lib.moe_balance_workspace_size(ctypes.byref(dm), 48) == 0   # 64 tokens % 48
    assert lib.moe_balance_workspace_size(ctypes.byref(dm), 0) == 0
    n = lib.moe_balance_workspace_size(ctypes.byref(dm), 16)           # 4 sequences
    assert n >= 4 * 16 * (8 + 4) + 4 * 8
    rc = lib.moe_balance_stats(ctypes.byref(dm), 48, fake, fake, 1.0, fake, fake, fake, fake,
                               1 << 20, None)
    assert rc == M.MOE_ERR_INVALID_ARG
    rc = lib.moe_balance_stats(ctypes.byref(dm), 16, fake, fake, 1.0, fake, fake, fake, fake,
                               16, None)
    assert rc == M.MOE_ERR_WORKSPACE
    rc = lib.moe_balance_stats(ctypes.byref(dm), 16, None, fake, 1.0, fake, fake, fake, fake,
                               1 << 20, None)
    assert rc == M.MOE_ERR_INVALID_ARG
    misaligned = ctypes.c_void_p((1 << 20) + 8)
    rc = lib.moe_balance_stats(ctypes.byref(dm), 16, fake, fake, 1.0, fake, fake, fake,
                               misaligned, 1 << 20, None)
    assert rc == M.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(ctypes.byref(dm), None, 0.1, fake, fake, None) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(ctypes.byref(dm), fake, 0.1, fake, None, None) == \
        M.MOE_ERR_INVALID_ARG


def test_dense_calls_rejected_on_host(lib):
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails first
    bad_d = M.dense_dims(T=16, d=200, I=128)
    assert lib.moe_dense_workspace_size(ctypes.byref(bad_d)) == 0
    assert lib.moe_dense_swiglu(ctypes.byref(bad_d), fake, fake, fake, fake, fake, fake, 1 << 30,
                                None) == M.MOE_ERR_UNSUPPORTED_SHAPE
    dm = M.dense_dims(T=16, d=256, I=128)
    need = lib.moe_dense_workspace_size(ctypes.byref(dm))
    assert need >= 16 * 128 * 2
    assert lib.moe_dense_swiglu(ctypes.byref(dm), None, fake, fake, fake, fake, fake, need,
                                None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_dense_swiglu(ctypes.byref(dm), fake, fake, fake, fake, fake, fake, 64,
                                None) == M.MOE_ERR_WORKSPACE


def test_dense_workspace_holds_the_split_k_partials(lib):
    """At T = 128 (d = 5120, I = 11264) both dense GEMMs have too few pair
    tiles for 74 SM pairs and are split over K: 5 splits of fp32 g and u
    partials for gate/up, 7 of fp32 y partials for down, sharing one region
    after h.  The workspace must hold h and the larger of the two; at T =
    4096 nothing is split and the workspace is h alone (plus alignment)."""
    def need(T):
        return lib.moe_dense_workspace_size(ctypes.byref(M.dense_dims(T=T, d=5120, I=11264)))
    T, d, I = 128, 5120, 11264
    h = T * I * 2
    up, down = 5 * 2 * T * I * 4, 7 * T * d * 4
    assert need(T) >= h + max(up, down)
    assert need(T) < h + max(up, down) + 4096
    assert 4096 * I * 2 <= need(4096) < 4096 * I * 2 + 4096


def test_expert_parallel_sizes_and_rejects_on_host(lib):
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: every call below fails first
    dm = M.dims(T=128, d=5120, E=128, k=6, I=1408, n_shared=2, align=16)
    assert M.ep_recv_capacity(dm, 8) == 8 * 128 * 6 + 16 * 15
    assert M.ep_recv_capacity(dm, 1) == M.capacity(dm)
    for bad_world in (0, -1, 3, 129):
        assert M.ep_recv_capacity(dm, bad_world) == 0
        assert M.ep_workspace_size(dm, bad_world) == 0
    L = M.ep_layout(dm, 8)
    offs = [L[n] for n, _ in M.MoeEpLayout._fields_ if n != "total"]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L["total"] == M.ep_workspace_size(dm, 8)
    assert L["h_shared"] - L["h_recv"] >= M.ep_recv_capacity(dm, 8) * 1408 * 2
    need = L["total"]
    P = ctypes.byref(dm)
    assert lib.moe_ep_route(P, 3, fake, fake, None, fake, need, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_route(P, 8, fake, fake, None, fake, 64, None) == M.MOE_ERR_WORKSPACE
    assert lib.moe_ep_route(P, 8, None, fake, None, fake, need, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_dispatch(P, 8, 8, fake, fake, fake, fake, need, None) == \
        M.MOE_ERR_INVALID_ARG                                       # rank out of range
    assert lib.moe_ep_dispatch(P, 8, 0, fake, None, fake, fake, need, None) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_experts(P, 8, fake, None, fake, fake, fake, fake, fake, fake, fake, fake,
                              need, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_experts(P, 8, fake, fake, fake, fake, fake, None, fake, fake, fake, fake,
                              need, None) == M.MOE_ERR_INVALID_ARG   # S = 2 without ws1
    assert lib.moe_ep_combine(P, 8, None, fake, fake, need, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_combine(P, 8, fake, fake, ctypes.c_void_p((1 << 20) + 64), need,
                              None) == M.MOE_ERR_WORKSPACE


def test_ipc_calls_rejected_on_host(lib):
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_uint64(0)
    ptr = ctypes.c_void_p(0)
    assert lib.moe_ipc_export(None, h, ctypes.byref(off)) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_export(ctypes.c_void_p(1 << 20), None, ctypes.byref(off)) == \
        M.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_open(None, 0, ctypes.byref(ptr)) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_open(h, 0, None) == M.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_close(None, 0) == M.MOE_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        M.ipc_open(b"short", 0)


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert M.status_string(s) != "unknown status"


def test_no_alloc_route_rejects_shapes_beyond_its_scratch(lib):
    """The size check of moe_route_noalloc comes before any pointer is used or
    any CUDA call is made: one split of T * E fp32 partial logits above the
    built-in 16 MiB is rejected, one that fits is not rejected for size."""
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced
    over = M.dims(T=32769, d=5120, E=128, k=6, I=1408, n_shared=2, align=16)
    assert 32769 * 128 * 4 > (16 << 20)
    assert lib.moe_route_noalloc(ctypes.byref(over), fake, fake, None, None, fake, fake,
                                 None) == M.MOE_ERR_WORKSPACE
    assert M.route_workspace_size(M.dims(T=32768, d=5120, E=128, k=6, I=1408, n_shared=2,
                                         align=16)) <= (16 << 20)


def test_guard_zone_bookkeeping(monkeypatch):
    """The checks build's canary bookkeeping (host side, on a CPU tensor): a
    fresh workspace holds the canary everywhere; writing into a region leaves
    its guards intact; writing into a guard zone is reported."""
    monkeypatch.setattr(M, "CHECKS", True)
    monkeypatch.setattr(M, "GUARD_BYTES", 256)
    monkeypatch.setattr(M, "_guarded", [])
    layout = {"a": 0, "b": 1024, "c": 2048, "total": 4096}
    ws = M.guard_layout(M.alloc_workspace(4096, "cpu"), layout)
    assert bool((ws == M.CANARY).all())
    ws[0:700] = 1                     # region a (its guard is [768, 1024))
    ws[1024:1700] = 2                 # region b
    assert M.check_guards() == []
    ws[1800] = 0                      # region b's guard
    ws[4095] = 0                      # the trailing guard
    bad = M.check_guards()
    assert (4096, 1792, 2048) in bad and (4096, 3840, 4096) in bad
    del ws
    assert M.check_guards() == []     # a freed workspace is forgotten
