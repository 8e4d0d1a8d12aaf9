"""ctypes binding of libmoe_b200.so (the C ABI in include/moe_b200.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch tensors are used for device memory and the current stream.
There is no CPU fallback: if the library is missing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_CHECKS=1 in the environment selects the bounds-checking build of the
# library (device bounds checks recorded as MOE_ERR_BOUNDS, a guard zone
# after every workspace region); it is built by `build --checks`.
CHECKS = os.environ.get("MOE_CHECKS", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libmoe_b200_checks.so" if CHECKS else "libmoe_b200.so")
GUARD_BYTES = 256 if CHECKS else 0

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_TIMEOUT = -5
MOE_ERR_BOUNDS = -6

# every symbol declared in include/moe_b200.h
EXPORTED = (
    "moe_capacity", "moe_status_string", "moe_route_workspace_size", "moe_route",
    "moe_permute_workspace_size", "moe_permute", "moe_grouped_swiglu", "moe_combine",
    "moe_workspace_size", "moe_forward_layout", "moe_forward", "moe_get_last_device_status",
    "moe_set_wait_limit_ns", "moe_set_phase_events", "moe_route_noalloc",
    "moe_train_workspace_size", "moe_train_layout_of", "moe_forward_train", "moe_backward",
    "moe_backward_f32",
    "moe_balance_workspace_size", "moe_balance_stats", "moe_bias_update",
    "moe_dense_workspace_size", "moe_dense_swiglu",
    "moe_ep_recv_capacity", "moe_ep_workspace_size", "moe_ep_layout_of", "moe_ep_route",
    "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine",
    "moe_ipc_export", "moe_ipc_open", "moe_ipc_close",
)


class MoeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("I", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("align", ctypes.c_int)]


class MoeWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "route_partials", "probs", "topk_idx", "topk_w", "counts", "offsets", "row_of",
        "token_of_row", "permute_scratch", "x_perm", "h_perm", "y_perm", "h_shared",
        "y_shared", "total")]


class MoeTrainLayout(ctypes.Structure):
    _fields_ = [("fwd", MoeWsLayout)] + [(n, ctypes.c_size_t) for n in (
        "g_perm", "u_perm", "g_shared", "u_shared", "dy_perm", "dw", "dz", "dgu_perm",
        "dgu_shared", "dx_perm", "dx_shared", "dx_router", "dwg_partials", "total")]


class MoeEpLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "route_partials", "probs", "topk_idx", "topk_w", "counts", "offsets", "row_of",
        "token_of_row", "permute_scratch", "dst_row", "recv_offsets", "recv_counts",
        "remote_row", "h_recv", "h_shared", "y_shared", "total")]


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m fine_grained_moe_fp32_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, Z, V = ctypes.POINTER(MoeDims), ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "moe_capacity": (ctypes.c_int64, [P]),
        "moe_status_string": (ctypes.c_char_p, [I]),
        "moe_route_workspace_size": (Z, [P]),
        "moe_route": (I, [P, V, V, V, V, V, V, V, Z, V]),
        "moe_permute_workspace_size": (Z, [P]),
        "moe_permute": (I, [P, V, V, V, V, V, V, V, V, Z, V]),
        "moe_grouped_swiglu": (I, [P, V, V, V, V, V, V, V, V]),
        "moe_combine": (I, [P, V, V, V, V, V, V]),
        "moe_workspace_size": (Z, [P]),
        "moe_forward_layout": (I, [P, ctypes.POINTER(MoeWsLayout)]),
        "moe_forward": (I, [P, V, V, V, V, V, V, V, V, V, V, V, Z, V]),
        "moe_get_last_device_status": (I, [V]),
        "moe_set_wait_limit_ns": (I, [ctypes.c_uint64]),
        "moe_set_phase_events": (I, [ctypes.POINTER(ctypes.c_void_p), I]),
        "moe_route_noalloc": (I, [P, V, V, V, V, V, V, V]),
        "moe_train_workspace_size": (Z, [P]),
        "moe_train_layout_of": (I, [P, ctypes.POINTER(MoeTrainLayout)]),
        "moe_forward_train": (I, [P, V, V, V, V, V, V, V, V, V, V, V, Z, V]),
        "moe_backward": (I, [P, V, V, V, V, V, V, V, V, V, V, Z, V, V, V, V, V, V, V, V, V]),
        "moe_backward_f32": (I, [P, V, V, V, V, V, V, V, V, V, V, Z, V, V, V, V, V, V, V, V, V]),
        "moe_balance_workspace_size": (Z, [P, I]),
        "moe_balance_stats": (I, [P, I, V, V, ctypes.c_float, V, V, V, V, Z, V]),
        "moe_bias_update": (I, [P, V, ctypes.c_float, V, V, V]),
        "moe_dense_workspace_size": (Z, [P]),
        "moe_dense_swiglu": (I, [P, V, V, V, V, V, V, Z, V]),
        "moe_ep_recv_capacity": (ctypes.c_int64, [P, I]),
        "moe_ep_workspace_size": (Z, [P, I]),
        "moe_ep_layout_of": (I, [P, I, ctypes.POINTER(MoeEpLayout)]),
        "moe_ep_route": (I, [P, I, V, V, V, V, Z, V]),
        "moe_ep_dispatch": (I, [P, I, I, V, V, V, V, Z, V]),
        "moe_ep_experts": (I, [P, I, V, V, V, V, V, V, V, V, V, V, Z, V]),
        "moe_ep_combine": (I, [P, I, V, V, V, Z, V]),
        "moe_ipc_export": (I, [V, V, ctypes.POINTER(ctypes.c_uint64)]),
        "moe_ipc_open": (I, [V, ctypes.c_uint64, ctypes.POINTER(ctypes.c_void_p)]),
        "moe_ipc_close": (I, [V, ctypes.c_uint64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load().moe_status_string(status).decode()
    except RuntimeError:
        return "unknown"


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoEError(rc, what)


def dims(T, d, E, k, I, n_shared, align=16) -> MoeDims:
    return MoeDims(int(T), int(d), int(E), int(k), int(I), int(n_shared), int(align))


def dims_of(cfg, T=None, align=16) -> MoeDims:
    return dims(cfg.T if T is None else T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, align)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t, dtype, shape, name):
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def capacity(dm: MoeDims) -> int:
    return int(load().moe_capacity(ctypes.byref(dm)))


def workspace_size(dm: MoeDims) -> int:
    return int(load().moe_workspace_size(ctypes.byref(dm)))


def route_workspace_size(dm: MoeDims) -> int:
    return int(load().moe_route_workspace_size(ctypes.byref(dm)))


def permute_workspace_size(dm: MoeDims) -> int:
    return int(load().moe_permute_workspace_size(ctypes.byref(dm)))


def forward_layout(dm: MoeDims) -> dict:
    L = MoeWsLayout()
    _check(load().moe_forward_layout(ctypes.byref(dm), ctypes.byref(L)), "moe_forward_layout")
    return {n: getattr(L, n) for n, _ in MoeWsLayout._fields_}


CANARY = 0xA5  # checks build: the byte every workspace starts filled with
_guarded = []  # checks build: (weak reference to a workspace, [(start, end) guard bytes])


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A uint8 device buffer of at least nbytes (torch's allocator aligns to 512 B).
    Checks build: filled with CANARY (so a region read before it is written
    shows up as a parity failure) and registered with its trailing guard
    zone, which the library never writes."""
    ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)
    if CHECKS:
        import weakref
        ws.fill_(CANARY)
        n = int(nbytes)
        _guarded.append((weakref.ref(ws), [(n - GUARD_BYTES, n)] if n >= GUARD_BYTES else []))
    return ws


def guard_layout(ws: torch.Tensor, layout: dict) -> torch.Tensor:
    """Checks build: register the guard zone in front of every region of a
    workspace layout (the 256 bytes before each offset: the previous
    region's guard).  A no-op otherwise."""
    if CHECKS:
        import weakref
        offs = sorted({v for k, v in _flatten(layout).items() if v > 0})
        _guarded.append((weakref.ref(ws), [(o - GUARD_BYTES, o) for o in offs]))
    return ws


def _flatten(layout: dict) -> dict:
    out = {}
    for k, v in layout.items():
        if isinstance(v, dict):
            out.update({f"{k}.{kk}": vv for kk, vv in _flatten(v).items()})
        else:
            out[k] = int(v)
    return out


def check_guards() -> list:
    """Checks build: every registered guard zone of every live workspace
    still holds CANARY.  Returns a list of (workspace bytes, start, end) that
    do not (empty when all are intact); forgets workspaces that are gone."""
    bad, keep = [], []
    for ref, ranges in _guarded:
        ws = ref()
        if ws is None:
            continue
        keep.append((ref, ranges))
        for a, b in ranges:
            if a < 0 or b > ws.numel():
                bad.append((ws.numel(), a, b))
            elif not bool((ws[a:b] == CANARY).all()):
                bad.append((ws.numel(), a, b))
    _guarded[:] = keep
    return bad


# ------------------------------------------------------------------ calls

def route(dm, x, w_gate, bias, probs, topk_idx, topk_w, workspace, stream=None):
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(w_gate, torch.float32, (dm.E, dm.d), "w_gate")
    _expect(bias, torch.float32, (dm.E,), "bias")
    _expect(probs, torch.float32, (dm.T, dm.E), "probs")
    _expect(topk_idx, torch.int32, (dm.T, dm.k), "topk_idx")
    _expect(topk_w, torch.float32, (dm.T, dm.k), "topk_w")
    rc = load().moe_route(ctypes.byref(dm), _ptr(x), _ptr(w_gate), _ptr(bias), _ptr(probs),
                          _ptr(topk_idx), _ptr(topk_w), _ptr(workspace),
                          workspace.numel() if workspace is not None else 0, _stream(stream))
    _check(rc, "moe_route")


def route_noalloc(dm, x, w_gate, bias, probs, topk_idx, topk_w, stream=None):
    """moe_route for callers that cannot allocate device memory: the scratch
    is a fixed 16 MiB array inside the library (see include/moe_b200.h)."""
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(w_gate, torch.float32, (dm.E, dm.d), "w_gate")
    _expect(bias, torch.float32, (dm.E,), "bias")
    _expect(probs, torch.float32, (dm.T, dm.E), "probs")
    _expect(topk_idx, torch.int32, (dm.T, dm.k), "topk_idx")
    _expect(topk_w, torch.float32, (dm.T, dm.k), "topk_w")
    rc = load().moe_route_noalloc(ctypes.byref(dm), _ptr(x), _ptr(w_gate), _ptr(bias),
                                  _ptr(probs), _ptr(topk_idx), _ptr(topk_w), _stream(stream))
    _check(rc, "moe_route_noalloc")


def permute(dm, topk_idx, x, counts, offsets, row_of, token_of_row, x_perm, workspace,
            stream=None):
    cap = capacity(dm)
    _expect(topk_idx, torch.int32, (dm.T, dm.k), "topk_idx")
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(counts, torch.int32, (dm.E,), "counts")
    _expect(offsets, torch.int32, (dm.E + 1,), "offsets")
    _expect(row_of, torch.int32, (dm.T * dm.k,), "row_of")
    _expect(token_of_row, torch.int32, (cap,), "token_of_row")
    _expect(x_perm, torch.bfloat16, (cap, dm.d), "x_perm")
    rc = load().moe_permute(ctypes.byref(dm), _ptr(topk_idx), _ptr(x), _ptr(counts),
                            _ptr(offsets), _ptr(row_of), _ptr(token_of_row), _ptr(x_perm),
                            _ptr(workspace), workspace.numel() if workspace is not None else 0,
                            _stream(stream))
    _check(rc, "moe_permute")


def grouped_swiglu(dm, x_perm, offsets, w1, w3, w2, h_perm, y_perm, stream=None):
    cap = capacity(dm)
    _expect(x_perm, torch.bfloat16, (cap, dm.d), "x_perm")
    _expect(offsets, torch.int32, (dm.E + 1,), "offsets")
    _expect(w1, torch.bfloat16, (dm.E, dm.I, dm.d), "w1")
    _expect(w3, torch.bfloat16, (dm.E, dm.I, dm.d), "w3")
    _expect(w2, torch.bfloat16, (dm.E, dm.d, dm.I), "w2")
    _expect(h_perm, torch.bfloat16, (cap, dm.I), "h_perm")
    _expect(y_perm, torch.float32, (cap, dm.d), "y_perm")
    rc = load().moe_grouped_swiglu(ctypes.byref(dm), _ptr(x_perm), _ptr(offsets), _ptr(w1),
                                   _ptr(w3), _ptr(w2), _ptr(h_perm), _ptr(y_perm),
                                   _stream(stream))
    _check(rc, "moe_grouped_swiglu")


def combine(dm, y_perm, row_of, topk_w, y_shared, y, stream=None):
    cap = capacity(dm)
    _expect(y_perm, torch.float32, (cap, dm.d), "y_perm")
    _expect(row_of, torch.int32, (dm.T * dm.k,), "row_of")
    _expect(topk_w, torch.float32, (dm.T, dm.k), "topk_w")
    _expect(y_shared, torch.float32, (dm.T, dm.d), "y_shared")
    _expect(y, torch.bfloat16, (dm.T, dm.d), "y")
    rc = load().moe_combine(ctypes.byref(dm), _ptr(y_perm), _ptr(row_of), _ptr(topk_w),
                            _ptr(y_shared), _ptr(y), _stream(stream))
    _check(rc, "moe_combine")


def forward(dm, x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace, stream=None):
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(w_gate, torch.float32, (dm.E, dm.d), "w_gate")
    _expect(bias, torch.float32, (dm.E,), "bias")
    _expect(w1, torch.bfloat16, (dm.E, dm.I, dm.d), "w1")
    _expect(w3, torch.bfloat16, (dm.E, dm.I, dm.d), "w3")
    _expect(w2, torch.bfloat16, (dm.E, dm.d, dm.I), "w2")
    if dm.n_shared > 0:
        _expect(ws1, torch.bfloat16, (dm.n_shared, dm.I, dm.d), "ws1")
        _expect(ws3, torch.bfloat16, (dm.n_shared, dm.I, dm.d), "ws3")
        _expect(ws2, torch.bfloat16, (dm.n_shared, dm.d, dm.I), "ws2")
    _expect(y, torch.bfloat16, (dm.T, dm.d), "y")
    rc = load().moe_forward(ctypes.byref(dm), _ptr(x), _ptr(w_gate), _ptr(bias), _ptr(w1),
                            _ptr(w3), _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(y),
                            _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_forward")


def train_workspace_size(dm: MoeDims) -> int:
    return int(load().moe_train_workspace_size(ctypes.byref(dm)))


def train_layout(dm: MoeDims) -> dict:
    L = MoeTrainLayout()
    _check(load().moe_train_layout_of(ctypes.byref(dm), ctypes.byref(L)), "moe_train_layout_of")
    out = {n: getattr(L, n) for n, _ in MoeTrainLayout._fields_ if n != "fwd"}
    out["fwd"] = {n: getattr(L.fwd, n) for n, _ in MoeWsLayout._fields_}
    return out


def forward_train(dm, x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2, y, workspace, stream=None):
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(y, torch.bfloat16, (dm.T, dm.d), "y")
    rc = load().moe_forward_train(ctypes.byref(dm), _ptr(x), _ptr(w_gate), _ptr(bias), _ptr(w1),
                                  _ptr(w3), _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(y),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "moe_forward_train")


def backward(dm, x, w_gate, w1, w3, w2, ws1, ws3, ws2, dy, workspace, grads: dict, stream=None):
    """grads: dict with preallocated dx, dw_gate, dw1, dw3, dw2, dws1, dws3, dws2.
    dx and the expert weight gradients are all bf16 (moe_backward) or all fp32
    (moe_backward_f32); dw_gate is fp32 either way."""
    dt = grads["dw1"].dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise TypeError(f"dw1: expected bf16 or fp32, got {dt}")
    _expect(dy, torch.bfloat16, (dm.T, dm.d), "dy")
    _expect(grads["dx"], dt, (dm.T, dm.d), "dx")
    _expect(grads["dw_gate"], torch.float32, (dm.E, dm.d), "dw_gate")
    _expect(grads["dw1"], dt, (dm.E, dm.I, dm.d), "dw1")
    _expect(grads["dw3"], dt, (dm.E, dm.I, dm.d), "dw3")
    _expect(grads["dw2"], dt, (dm.E, dm.d, dm.I), "dw2")
    for n, shape in (("dws1", (dm.n_shared, dm.I, dm.d)), ("dws3", (dm.n_shared, dm.I, dm.d)),
                     ("dws2", (dm.n_shared, dm.d, dm.I))):
        if grads.get(n) is not None:
            _expect(grads[n], dt, shape, n)
    g = grads
    fn = load().moe_backward_f32 if dt == torch.float32 else load().moe_backward
    rc = fn(ctypes.byref(dm), _ptr(x), _ptr(w_gate), _ptr(w1), _ptr(w3),
            _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2), _ptr(dy), _ptr(workspace),
            workspace.numel(), _ptr(g["dx"]), _ptr(g["dw_gate"]), _ptr(g["dw1"]),
            _ptr(g["dw3"]), _ptr(g["dw2"]), _ptr(g.get("dws1")),
            _ptr(g.get("dws3")), _ptr(g.get("dws2")), _stream(stream))
    _check(rc, "moe_backward_f32" if dt == torch.float32 else "moe_backward")


def dense_dims(T, d, I) -> MoeDims:
    """Dims of the dense FFN (E, k, n_shared are not used by it)."""
    return dims(T, d, 1, 1, I, 0)


def dense_workspace_size(dm: MoeDims) -> int:
    return int(load().moe_dense_workspace_size(ctypes.byref(dm)))


def dense_swiglu(dm, x, w1, w3, w2, y, workspace, stream=None):
    """y = (silu(x w1^T) * (x w3^T)) w2^T: the first layer's dense SwiGLU FFN."""
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _expect(w1, torch.bfloat16, (dm.I, dm.d), "w1")
    _expect(w3, torch.bfloat16, (dm.I, dm.d), "w3")
    _expect(w2, torch.bfloat16, (dm.d, dm.I), "w2")
    _expect(y, torch.bfloat16, (dm.T, dm.d), "y")
    rc = load().moe_dense_swiglu(ctypes.byref(dm), _ptr(x), _ptr(w1), _ptr(w3), _ptr(w2),
                                 _ptr(y), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_dense_swiglu")


def balance_workspace_size(dm: MoeDims, seq_len: int) -> int:
    return int(load().moe_balance_workspace_size(ctypes.byref(dm), int(seq_len)))


def balance_stats(dm, seq_len, probs, topk_idx, alpha, f, P, loss, workspace, stream=None):
    """Sequence-wise balance statistics f, P [T/seq_len, E] and the loss [1]."""
    n_seq = dm.T // seq_len if seq_len > 0 else 0
    _expect(probs, torch.float32, (dm.T, dm.E), "probs")
    _expect(topk_idx, torch.int32, (dm.T, dm.k), "topk_idx")
    _expect(f, torch.float32, (n_seq, dm.E), "f")
    _expect(P, torch.float32, (n_seq, dm.E), "P")
    _expect(loss, torch.float32, (1,), "loss")
    rc = load().moe_balance_stats(ctypes.byref(dm), int(seq_len), _ptr(probs), _ptr(topk_idx),
                                  float(alpha), _ptr(f), _ptr(P), _ptr(loss), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "moe_balance_stats")


def bias_update(dm, counts, gamma, bias_in, bias_out, stream=None):
    """One auxiliary-loss-free bias step (bias_out may be bias_in)."""
    _expect(counts, torch.int32, (dm.E,), "counts")
    _expect(bias_in, torch.float32, (dm.E,), "bias_in")
    _expect(bias_out, torch.float32, (dm.E,), "bias_out")
    rc = load().moe_bias_update(ctypes.byref(dm), _ptr(counts), float(gamma), _ptr(bias_in),
                                _ptr(bias_out), _stream(stream))
    _check(rc, "moe_bias_update")


# ------------------------------------------------------------ expert parallel

def ep_recv_capacity(dm: MoeDims, world: int) -> int:
    return int(load().moe_ep_recv_capacity(ctypes.byref(dm), int(world)))


def ep_workspace_size(dm: MoeDims, world: int) -> int:
    return int(load().moe_ep_workspace_size(ctypes.byref(dm), int(world)))


def ep_layout(dm: MoeDims, world: int) -> dict:
    L = MoeEpLayout()
    _check(load().moe_ep_layout_of(ctypes.byref(dm), int(world), ctypes.byref(L)),
           "moe_ep_layout_of")
    return {n: getattr(L, n) for n, _ in MoeEpLayout._fields_}


def pointer_array(tensors, device) -> torch.Tensor:
    """A device array of the tensors' device addresses (int64), the form the
    expert-parallel calls take for per-rank buffers."""
    for t in tensors:
        _ptr(t)
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def ep_route(dm, world, x, w_gate, bias, workspace, stream=None):
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _check(load().moe_ep_route(ctypes.byref(dm), int(world), _ptr(x), _ptr(w_gate), _ptr(bias),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_ep_route")


def ep_dispatch(dm, world, rank, x, counts_of, x_recv, workspace, stream=None):
    """counts_of, x_recv: pointer_array() of every rank's counts / receive buffer."""
    _expect(x, torch.bfloat16, (dm.T, dm.d), "x")
    _check(load().moe_ep_dispatch(ctypes.byref(dm), int(world), int(rank), _ptr(x),
                                  _ptr(counts_of), _ptr(x_recv), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "moe_ep_dispatch")


def ep_experts(dm, world, x, x_recv, w1, w3, w2, ws1, ws3, ws2, y_recv, workspace, stream=None):
    El, rc = dm.E // world, ep_recv_capacity(dm, world)
    _expect(x_recv, torch.bfloat16, (rc, dm.d), "x_recv")
    _expect(y_recv, torch.float32, (rc, dm.d), "y_recv")
    _expect(w1, torch.bfloat16, (El, dm.I, dm.d), "w1")
    _expect(w2, torch.bfloat16, (El, dm.d, dm.I), "w2")
    _check(load().moe_ep_experts(ctypes.byref(dm), int(world), _ptr(x), _ptr(x_recv), _ptr(w1),
                                 _ptr(w3), _ptr(w2), _ptr(ws1), _ptr(ws3), _ptr(ws2),
                                 _ptr(y_recv), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "moe_ep_experts")


def ep_combine(dm, world, y_recv, y, workspace, stream=None):
    """y_recv: pointer_array() of every rank's expert-output buffer."""
    _expect(y, torch.bfloat16, (dm.T, dm.d), "y")
    _check(load().moe_ep_combine(ctypes.byref(dm), int(world), _ptr(y_recv), _ptr(y),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_ep_combine")


def ipc_export(t: torch.Tensor) -> tuple[bytes, int]:
    """CUDA IPC handle (64 bytes) of the allocation holding tensor t, and t's
    byte offset inside it."""
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_uint64(0)
    _check(load().moe_ipc_export(_ptr(t), h, ctypes.byref(off)), "moe_ipc_export")
    return h.raw, int(off.value)


def ipc_open(handle: bytes, offset: int) -> int:
    """Device address, in this process, of another process's exported tensor."""
    if len(handle) != 64:
        raise ValueError("an IPC handle is 64 bytes")
    p = ctypes.c_void_p(0)
    _check(load().moe_ipc_open(handle, ctypes.c_uint64(offset), ctypes.byref(p)), "moe_ipc_open")
    return int(p.value)


def ipc_close(ptr: int, offset: int) -> None:
    _check(load().moe_ipc_close(ctypes.c_void_p(ptr), ctypes.c_uint64(offset)), "moe_ipc_close")


def ep_workspace_views(dm: MoeDims, world: int, ws: torch.Tensor) -> dict:
    """Typed views of one rank's expert-parallel workspace."""
    L = ep_layout(dm, world)
    T, E, k, I = dm.T, dm.E, dm.k, dm.I
    El, rc = E // world, ep_recv_capacity(dm, world)

    def view(off, n, dtype, shape):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).view(*shape)

    i32 = torch.int32
    return {
        "probs": view(L["probs"], T * E, torch.float32, (T, E)),
        "topk_idx": view(L["topk_idx"], T * k, i32, (T, k)),
        "topk_w": view(L["topk_w"], T * k, torch.float32, (T, k)),
        "counts": view(L["counts"], E, i32, (E,)),
        "offsets": view(L["offsets"], E + 1, i32, (E + 1,)),
        "row_of": view(L["row_of"], T * k, i32, (T * k,)),
        "dst_row": view(L["dst_row"], E, i32, (E,)),
        "recv_offsets": view(L["recv_offsets"], El + 1, i32, (El + 1,)),
        "recv_counts": view(L["recv_counts"], El, i32, (El,)),
        "remote_row": view(L["remote_row"], T * k, i32, (T * k,)),
        "h_recv": view(L["h_recv"], rc * I, torch.bfloat16, (rc, I)),
    }


class EPRanks:
    """Expert parallelism over ``world`` ranks emulated by one process on one
    device: rank r owns experts [r E/W, (r+1) E/W) (its weight slices are
    views of the full tensors) and its own receive buffers; the cross-rank
    arguments are arrays of this device's buffers instead of peer pointers.
    Each step issues, rank after rank, the same calls a rank of a multi-GPU
    job makes, with stream order standing in for the barriers between the
    phases, so no kernel ever waits on another."""

    def __init__(self, inputs: dict, world: int, T: int, align: int = 16, device="cuda"):
        cfg = inputs["cfg"]
        if cfg.E % world:
            raise ValueError("the routed experts must split evenly over the ranks")
        self.cfg, self.world, self.T, self.align = cfg, int(world), int(T), align
        self.device = torch.device(device)
        to = lambda t: t.to(self.device).contiguous()  # noqa: E731
        self.w_gate, self.bias = to(inputs["w_gate"]), to(inputs["bias"])
        w1, w3, w2 = to(inputs["w1"]), to(inputs["w3"]), to(inputs["w2"])
        self.ws1, self.ws3, self.ws2 = to(inputs["ws1"]), to(inputs["ws3"]), to(inputs["ws2"])
        El = cfg.E // world
        self.experts = [(w1[r * El:(r + 1) * El], w3[r * El:(r + 1) * El],
                         w2[r * El:(r + 1) * El]) for r in range(world)]
        self.dm = dims(T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, align)
        self.recv_cap = ep_recv_capacity(self.dm, world)
        nbytes = ep_workspace_size(self.dm, world)
        self.ws = [guard_layout(alloc_workspace(nbytes, self.device), ep_layout(self.dm, world))
                   for _ in range(world)]
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.x_recv = [torch.empty((self.recv_cap, cfg.d), **bf) for _ in range(world)]
        self.y_recv = [torch.empty((self.recv_cap, cfg.d), dtype=torch.float32, device=self.device)
                       for _ in range(world)]
        self.views = [ep_workspace_views(self.dm, world, w) for w in self.ws]
        self.counts_of = pointer_array([v["counts"] for v in self.views], self.device)
        self.x_recv_of = pointer_array(self.x_recv, self.device)
        self.y_recv_of = pointer_array(self.y_recv, self.device)

    def route(self, xs, stream=None):
        for r in range(self.world):
            ep_route(self.dm, self.world, xs[r], self.w_gate, self.bias, self.ws[r], stream)

    def dispatch(self, xs, stream=None):
        for r in range(self.world):
            ep_dispatch(self.dm, self.world, r, xs[r], self.counts_of, self.x_recv_of, self.ws[r],
                        stream)

    def experts_step(self, xs, stream=None):
        for r in range(self.world):
            w1, w3, w2 = self.experts[r]
            ep_experts(self.dm, self.world, xs[r], self.x_recv[r], w1, w3, w2, self.ws1,
                       self.ws3, self.ws2, self.y_recv[r], self.ws[r], stream)

    def combine(self, ys, stream=None):
        for r in range(self.world):
            ep_combine(self.dm, self.world, self.y_recv_of, ys[r], self.ws[r], stream)

    def __call__(self, xs, ys=None, stream=None):
        """xs: the ranks' token batches ([T, d] bf16 each); returns their y."""
        if len(xs) != self.world:
            raise ValueError(f"expected {self.world} token batches")
        if ys is None:
            ys = [torch.empty((self.T, self.cfg.d), dtype=torch.bfloat16, device=self.device)
                  for _ in range(self.world)]
        self.route(xs, stream)
        self.dispatch(xs, stream)
        self.experts_step(xs, stream)
        self.combine(ys, stream)
        return ys


def device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(load().moe_get_last_device_status(_stream(stream)))


def set_wait_limit_ns(ns: int) -> None:
    load().moe_set_wait_limit_ns(int(ns))


PHASES = ("router", "permute", "gemm_gate_up_swiglu", "gemm_down", "combine")
BWD_PHASES = ("combine_router_bwd", "dgrad_down_swiglu_bwd", "wgrad_w2", "dgrad_up",
              "wgrad_w1_w3", "gate_gemms_unpermute")


def set_phase_events(events) -> None:
    """Record torch.cuda.Event objects between the kernels of moe_forward
    (6 events: before the router, then after each of the 5 phases) and, with
    13 events, of moe_backward too (before it, then after each of its 6
    phases); None turns the hook off.  An entry may be None: that point is
    not recorded (timing one phase needs only its two bounding events)."""
    if events is None:
        _check(load().moe_set_phase_events(None, 0), "moe_set_phase_events")
        return
    for e in events:
        if e is not None and e.cuda_event == 0:   # torch creates the event on first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    _check(load().moe_set_phase_events(arr, len(events)), "moe_set_phase_events")


# ------------------------------------------------------------------ helpers

def workspace_views(dm: MoeDims, ws: torch.Tensor) -> dict:
    """Typed views of the intermediates moe_forward leaves in its workspace."""
    L = forward_layout(dm)
    cap = capacity(dm)
    T, d, E, k, I, S = dm.T, dm.d, dm.E, dm.k, dm.I, dm.n_shared

    def view(off, n, dtype, shape):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).view(*shape)

    return {
        "probs": view(L["probs"], T * E, torch.float32, (T, E)),
        "topk_idx": view(L["topk_idx"], T * k, torch.int32, (T, k)),
        "topk_w": view(L["topk_w"], T * k, torch.float32, (T, k)),
        "counts": view(L["counts"], E, torch.int32, (E,)),
        "offsets": view(L["offsets"], E + 1, torch.int32, (E + 1,)),
        "row_of": view(L["row_of"], T * k, torch.int32, (T * k,)),
        "token_of_row": view(L["token_of_row"], cap, torch.int32, (cap,)),
        "x_perm": view(L["x_perm"], cap * d, torch.bfloat16, (cap, d)),
        "h_perm": view(L["h_perm"], cap * I, torch.bfloat16, (cap, I)),
        "y_perm": view(L["y_perm"], cap * d, torch.float32, (cap, d)),
        "h_shared": view(L["h_shared"], T * S * I, torch.bfloat16, (T, S * I)),
        "y_shared": view(L["y_shared"], T * d, torch.float32, (T, d)),
    }


def train_workspace_views(dm: MoeDims, ws: torch.Tensor) -> dict:
    """Typed views of what moe_forward_train / moe_backward leave in the
    training workspace (the forward views plus the backward intermediates)."""
    v = workspace_views(dm, ws)
    L = train_layout(dm)
    cap = capacity(dm)
    T, d, E, k, I, S = dm.T, dm.d, dm.E, dm.k, dm.I, dm.n_shared

    def view(off, n, dtype, shape):
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).view(*shape)

    bf, f32 = torch.bfloat16, torch.float32
    v.update({
        "g_perm": view(L["g_perm"], cap * I, f32, (cap, I)),
        "u_perm": view(L["u_perm"], cap * I, f32, (cap, I)),
        "g_shared": view(L["g_shared"], T * S * I, f32, (T, S * I)),
        "u_shared": view(L["u_shared"], T * S * I, f32, (T, S * I)),
        "dy_perm": view(L["dy_perm"], cap * d, bf, (cap, d)),
        "dw": view(L["dw"], T * k, f32, (T, k)),
        "dz": view(L["dz"], T * E, f32, (T, E)),
        "dgu_perm": view(L["dgu_perm"], cap * 2 * I, bf, (cap, 2 * I)),
        "dgu_shared": view(L["dgu_shared"], T * 2 * S * I, bf, (T, 2 * S * I)),
        "dx_perm": view(L["dx_perm"], cap * d, f32, (cap, d)),
        "dx_shared": view(L["dx_shared"], T * d, f32, (T, d)),
        "dx_router": view(L["dx_router"], T * d, f32, (T, d)),
    })
    return v


def global_loads(counts: torch.Tensor, T: int, group=None):
    """Per-expert loads and token count of the whole data-parallel batch: the
    sum over the ranks of ``group`` (unchanged when there is no group)."""
    if group is None:
        return counts, int(T)
    import torch.distributed as dist
    c = counts.clone()
    n = torch.tensor([int(T)], dtype=torch.int64, device=counts.device)
    dist.all_reduce(c, group=group)
    dist.all_reduce(n, group=group)
    return c, int(n.item())


WEIGHT_GRADS = ("dw_gate", "dw1", "dw3", "dw2", "dws1", "dws3", "dws2")


def allreduce_grads(grads: dict, group=None) -> dict:
    """Data-parallel training: sum the weight gradients of every replica in
    place (the input gradient dx stays per replica).  One collective per
    tensor, in a fixed order on every rank; the caller scales by 1/world if
    it wants the mean."""
    import torch.distributed as dist
    for name in WEIGHT_GRADS:
        t = grads.get(name)
        if t is not None and t.numel() > 0:
            dist.all_reduce(t, group=group)
    return grads


class MoELayer:
    """The layer with its weights resident on one device; ``__call__`` runs
    moe_forward into a reusable workspace."""

    def __init__(self, inputs: dict, align: int = 16, device="cuda"):
        cfg = inputs["cfg"]
        self.cfg = cfg
        self.align = align
        self.device = torch.device(device)
        to = lambda t: t.to(self.device).contiguous()  # noqa: E731
        self.w_gate = to(inputs["w_gate"])
        self.bias = to(inputs["bias"])
        self.w1, self.w3, self.w2 = to(inputs["w1"]), to(inputs["w3"]), to(inputs["w2"])
        self.ws1, self.ws3, self.ws2 = to(inputs["ws1"]), to(inputs["ws3"]), to(inputs["ws2"])
        self._ws = None
        self._ws_T = -1

    def dims(self, T: int) -> MoeDims:
        c = self.cfg
        return dims(T, c.d, c.E, c.k, c.I, c.S, self.align)

    def workspace(self, T: int) -> torch.Tensor:
        if self._ws is None or self._ws_T != T:
            self._ws = guard_layout(alloc_workspace(workspace_size(self.dims(T)), self.device),
                                    forward_layout(self.dims(T)))
            self._ws_T = T
        return self._ws

    def train_workspace(self, T: int) -> torch.Tensor:
        if getattr(self, "_tws", None) is None or self._tws_T != T:
            self._tws = guard_layout(
                alloc_workspace(train_workspace_size(self.dims(T)), self.device),
                train_layout(self.dims(T)))
            self._tws_T = T
        return self._tws

    def forward_train(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None):
        """Forward that keeps what the backward needs in the training workspace."""
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=self.device)
        forward_train(self.dims(T), x, self.w_gate, self.bias, self.w1, self.w3, self.w2,
                      self.ws1, self.ws3, self.ws2, y, self.train_workspace(T), stream)
        return y

    def alloc_grads(self, T: int, dtype=torch.bfloat16) -> dict:
        """Gradient buffers: dx and the expert weight gradients in ``dtype``
        (bf16 or fp32), the gate's gradient in fp32."""
        c, dev = self.cfg, self.device
        bf = dict(dtype=dtype, device=dev)
        return {"dx": torch.empty((T, c.d), **bf),
                "dw_gate": torch.empty((c.E, c.d), dtype=torch.float32, device=dev),
                "dw1": torch.empty((c.E, c.I, c.d), **bf), "dw3": torch.empty((c.E, c.I, c.d), **bf),
                "dw2": torch.empty((c.E, c.d, c.I), **bf),
                "dws1": torch.empty((c.S, c.I, c.d), **bf), "dws3": torch.empty((c.S, c.I, c.d), **bf),
                "dws2": torch.empty((c.S, c.d, c.I), **bf)}

    def backward(self, x: torch.Tensor, dy: torch.Tensor, grads: dict | None = None, stream=None):
        """Gradients after forward_train on the same x (routing held fixed)."""
        T = x.shape[0]
        grads = self.alloc_grads(T) if grads is None else grads
        backward(self.dims(T), x, self.w_gate, self.w1, self.w3, self.w2, self.ws1, self.ws3,
                 self.ws2, dy, self.train_workspace(T), grads, stream)
        return grads

    def _routing_views(self, T: int, train: bool) -> dict:
        ws = self.train_workspace(T) if train else self.workspace(T)
        return workspace_views(self.dims(T), ws)

    def balance_stats(self, T: int, seq_len: int, alpha: float, train: bool = True,
                      out: dict | None = None, stream=None) -> dict:
        """Sequence-wise balance statistics of the last forward over T tokens
        (forward_train when ``train``, else __call__): f, P and the loss."""
        dm = self.dims(T)
        v = self._routing_views(T, train)
        n_seq = T // seq_len
        if out is None:
            f32 = dict(dtype=torch.float32, device=self.device)
            out = {"f": torch.empty((n_seq, self.cfg.E), **f32),
                   "P": torch.empty((n_seq, self.cfg.E), **f32),
                   "loss": torch.empty(1, **f32)}
        key = (T, seq_len)
        if getattr(self, "_bal_key", None) != key:
            self._bal_ws = alloc_workspace(balance_workspace_size(dm, seq_len), self.device)
            self._bal_key = key
        balance_stats(dm, seq_len, v["probs"], v["topk_idx"], alpha, out["f"], out["P"],
                      out["loss"], self._bal_ws, stream)
        return out

    def bias_step(self, T: int, gamma: float, out: torch.Tensor | None = None, train: bool = True,
                  group=None, stream=None) -> torch.Tensor:
        """One auxiliary-loss-free bias step from the expert counts of the last
        forward over T tokens; writes into ``out`` (default: the layer's bias).
        With a torch.distributed ``group`` of data-parallel replicas the loads
        and token counts are summed over the group first, so every replica
        takes the same step as one replica holding the whole batch would."""
        out = self.bias if out is None else out
        counts, T_all = global_loads(self._routing_views(T, train)["counts"], T, group)
        bias_update(self.dims(T_all), counts, gamma, self.bias, out, stream)
        return out

    def __call__(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None):
        T = x.shape[0]
        dm = self.dims(T)
        if y is None:
            y = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=self.device)
        forward(dm, x, self.w_gate, self.bias, self.w1, self.w3, self.w2, self.ws1, self.ws3,
                self.ws2, y, self.workspace(T), stream)
        return y
