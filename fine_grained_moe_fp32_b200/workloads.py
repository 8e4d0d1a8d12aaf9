"""Seeded synthetic workloads for the dots.llm1 fine-grained MoE FFN layer.

This module only draws random numbers; it holds none of the layer's arithmetic.
Both the fp64 oracle and the CUDA path take their inputs from here, so the two
sides always see the same bytes.

Layer shape (dots.llm1 Technical Report, Method; "MoE Architecture
Specifications" block on the xugj520.cn overview page): hidden size 5120,
128 routed experts of which 6 are active per token, 2 shared experts.  The
expert intermediate size (1408) is not printed on the pages; it and the value
distributions below are the workload recipe this library is measured on.

Tensors (row-major, weights in ``[out, in]`` order):

=========  ==================  ======  ==========================================
name       shape               dtype   distribution
=========  ==================  ======  ==========================================
x          [T, d]              bf16    N(0, 1)
w_gate     [E, d]              fp32    N(0, 0.02^2)
bias       [E]                 fp32    see ``bias`` of the config
w1, w3     [E, I, d]           bf16    N(0, 0.02^2)  (gate / up projections)
w2         [E, d, I]           bf16    N(0, 0.02^2)  (down projection)
ws1, ws3   [S, I, d]           bf16    N(0, 0.02^2)  (shared experts)
ws2        [S, d, I]           bf16    N(0, 0.02^2)
dy         [T, d]              bf16    N(0, 1)       (only when ``grad``)
=========  ==================  ======  ==========================================

The skewed-load workload adds a per-expert logit offset ``ln(r^-1.2)`` (Zipf
weights with s = 1.2 over ranks r = 1..E, assigned to experts by a seeded
random permutation).  The layer has no logit-offset input, so the offset is
realised inside the inputs: feature 0 of every token is set to 1.0 and
``w_gate[e, 0]`` to the offset of expert e, which adds exactly the offset to
logit e.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int = 128
    k: int = 6
    S: int = 2
    I: int = 1408
    bias: str = "zero"        # "zero" | "uniform0.01" | "normal0.05"
    zipf: bool = False        # per-expert Zipf(1.2) logit offsets
    grad: bool = False        # also draw an upstream gradient dy

    @property
    def n_experts_active(self) -> int:
        return self.k + self.S


CONFIGS = {
    0: MoEConfig("tiny_T256_d512_I128", T=256, d=512, I=128, bias="uniform0.01"),
    1: MoEConfig("decode_T128_d5120_I1408", T=128, d=5120),
    2: MoEConfig("prefill_balanced_T4096_d5120_I1408", T=4096, d=5120),
    3: MoEConfig("prefill_skewed_T16384_d5120_I1408", T=16384, d=5120,
                 bias="normal0.05", zipf=True),
    4: MoEConfig("fwd_bwd_T8192_d5120_I1408", T=8192, d=5120, grad=True),
}

TINY = CONFIGS[0]
DECODE = CONFIGS[1]
PREFILL_BALANCED = CONFIGS[2]
PREFILL_SKEWED = CONFIGS[3]
FWD_BWD = CONFIGS[4]

# one independent stream per tensor, so shrinking T leaves the weights alone
_STREAM = {"x": 1, "w_gate": 2, "bias": 3, "w1": 4, "w3": 5, "w2": 6,
           "ws1": 7, "ws3": 8, "ws2": 9, "dy": 10, "zipf_perm": 11,
           "dense_w1": 12, "dense_w3": 13, "dense_w2": 14}

# The first layer's dense SwiGLU FFN: its intermediate size is not on the
# pages; the MoE layer's activated width (6 routed + 2 shared experts of 1408)
# is used, so both layers cost the same per token.
DENSE_I = 8 * 1408


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + _STREAM[name])
    return g


def _normal(shape, std, seed, name, device, dtype):
    g = _gen(seed, name, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_offsets(E: int, seed: int = 0, s: float = 1.2) -> torch.Tensor:
    """ln of Zipf(s) weights r^-s (r = 1..E), permuted over experts (fp32, CPU)."""
    g = _gen(seed, "zipf_perm", "cpu")
    perm = torch.randperm(E, generator=g)
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    offs = (-s * torch.log(ranks))[perm]
    return offs.to(torch.float32)


def make_inputs(cfg: MoEConfig | int, device="cpu", seed: int = 0,
                T: int | None = None, weights: bool = True) -> dict:
    """Draw the workload's tensors on ``device``.

    ``T`` overrides the token count (the weights do not depend on it).
    ``weights=False`` skips the expert weight tensors (router-only tests).
    The same (seed, device type) always gives the same values.
    """
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    T = cfg.T if T is None else T
    d, E, I, S = cfg.d, cfg.E, cfg.I, cfg.S
    dev = torch.device(device)
    out = {"cfg": cfg, "T": T}
    out["x"] = _normal((T, d), 1.0, seed, "x", dev, torch.bfloat16)
    out["w_gate"] = _normal((E, d), 0.02, seed, "w_gate", dev, torch.float32)
    if cfg.bias == "zero":
        out["bias"] = torch.zeros(E, device=dev, dtype=torch.float32)
    elif cfg.bias == "uniform0.01":
        g = _gen(seed, "bias", dev)
        u = torch.rand((E,), generator=g, device=dev, dtype=torch.float32)
        out["bias"] = (u * 0.02 - 0.01)
    elif cfg.bias == "normal0.05":
        out["bias"] = _normal((E,), 0.05, seed, "bias", dev, torch.float32)
    else:
        raise ValueError(cfg.bias)
    if cfg.zipf:
        out["x"][:, 0] = 1.0
        out["w_gate"][:, 0] = zipf_offsets(E, seed).to(dev)
    if weights:
        out["w1"] = _normal((E, I, d), 0.02, seed, "w1", dev, torch.bfloat16)
        out["w3"] = _normal((E, I, d), 0.02, seed, "w3", dev, torch.bfloat16)
        out["w2"] = _normal((E, d, I), 0.02, seed, "w2", dev, torch.bfloat16)
        out["ws1"] = _normal((S, I, d), 0.02, seed, "ws1", dev, torch.bfloat16)
        out["ws3"] = _normal((S, I, d), 0.02, seed, "ws3", dev, torch.bfloat16)
        out["ws2"] = _normal((S, d, I), 0.02, seed, "ws2", dev, torch.bfloat16)
    if cfg.grad:
        out["dy"] = _normal((T, d), 1.0, seed, "dy", dev, torch.bfloat16)
    return out


def make_dense_inputs(T: int, d: int = 5120, I: int = DENSE_I, device="cpu",
                      seed: int = 0) -> dict:
    """Tokens and weights of the dense SwiGLU FFN: x N(0,1) bf16 [T, d];
    w1, w3 [I, d] and w2 [d, I] N(0, 0.02) bf16.  x is the same draw as the
    MoE workloads' x for the same (seed, T, d)."""
    dev = torch.device(device)
    return {"T": T, "d": d, "I": I,
            "x": _normal((T, d), 1.0, seed, "x", dev, torch.bfloat16),
            "w1": _normal((I, d), 0.02, seed, "dense_w1", dev, torch.bfloat16),
            "w3": _normal((I, d), 0.02, seed, "dense_w3", dev, torch.bfloat16),
            "w2": _normal((d, I), 0.02, seed, "dense_w2", dev, torch.bfloat16)}


def small_config(T=64, d=256, E=16, k=4, S=2, I=128, bias="uniform0.01") -> MoEConfig:
    """A shape for quick tests (any T/d/E/k/S/I the kernels accept)."""
    return MoEConfig(f"small_T{T}_d{d}_E{E}_k{k}_I{I}", T=T, d=d, E=E, k=k, S=S,
                     I=I, bias=bias)


def zipf_log_range(E: int = 128, s: float = 1.2) -> tuple[float, float]:
    """Range of the Zipf logit offsets, for documentation checks."""
    return (-s * math.log(E), 0.0)
