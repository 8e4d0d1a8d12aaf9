"""CPU emulation of the bf16 storage points that the tensor-core backward
cannot avoid, used to show where the 2e-2 * rms bound is out of reach of any
implementation that feeds bf16 operands to the MMAs.

The backward's grouped GEMMs take bf16 operands (tcgen05 kind::f16): the
weight gradients of a routed expert are
    dW2 = dY_perm^T H,   dW1 = dG^T X_perm,   dW3 = dU^T X_perm
where dY_perm = w * dy (one bf16 rounding), H = silu(g) * u (one rounding,
it is the forward down GEMM's operand too), and dG / dU come from
dH = dY_perm W2 with the SwiGLU backward (one rounding each).  Everything
else is taken exact (fp64) here, including the fp32 accumulation, g and u.
Test infrastructure only; it uses the oracle's exact intermediates.
"""
import numpy as np
import torch

from oracle import moe_oracle as O


def bf16(a):
    """Round every element to the nearest bf16 (ties to even), as float64."""
    return torch.tensor(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def routed_weight_grads(inp, fwd, bwd, experts, rnd=bf16):
    """{name: {expert: array}} of the routed weight gradients computed from
    operands rounded by ``rnd`` (bf16 by default; exact arithmetic otherwise)."""
    off = fwd["offsets"]
    xp = fwd["x_perm"]
    dyp = rnd(bwd["dy_perm"])
    hp = rnd(fwd["h_perm"])
    out = {"dw1": {}, "dw3": {}, "dw2": {}}
    for e in experts:
        a, b = int(off[e]), int(off[e + 1])
        w1 = O._f64(inp["w1"][e])
        w3 = O._f64(inp["w3"][e])
        w2 = O._f64(inp["w2"][e])
        if a == b:
            out["dw1"][e] = np.zeros(w1.shape)
            out["dw3"][e] = np.zeros(w3.shape)
            out["dw2"][e] = np.zeros(w2.shape)
            continue
        x = xp[a:b]
        g = x @ w1.T
        u = x @ w3.T
        dh = dyp[a:b] @ w2
        dg = rnd(dh * u * O.silu_grad(g))
        du = rnd(dh * O.silu(g))
        out["dw1"][e] = dg.T @ x
        out["dw3"][e] = du.T @ x
        out["dw2"][e] = dyp[a:b].T @ hp[a:b]
    return out
