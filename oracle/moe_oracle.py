"""fp64 CPU oracle for the dots.llm1 fine-grained MoE FFN layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The library itself never calls it
and has no CPU fallback.  It shares no code with the CUDA path; the only thing
the two sides share is the seeded input generator.

It is the plain definition of what the layer computes, written in numpy float64
from the exact bf16 / fp32 input values, with no blocking or fusion.  Sources
(pages about dots.llm1; the numbers in brackets are the sections cited):

* "dots.llm1 Technical Report" (bud-325.pages.dev), Method: every MoE layer has
  128 routed experts with the top 6 chosen per token, plus 2 shared experts
  that are always on (8 active in total); the gate projection runs in FP32;
  balancing uses the auxiliary-loss-free per-expert bias; no token is dropped.
  Key claims / Method, systems paragraph: the grouped GEMM pads each expert's
  token segment to a multiple of the MMA tile.
* "dots.llm1: the first MoE large language model open-sourced by Little Red
  Book" (kdjingpai.com), Model Architecture Features: 6 routed + 2 shared
  experts per token, SwiGLU experts, load balancing by dynamic bias terms.
* aibase.com news item on dots.llm1, architecture paragraph: each expert is a
  two-layer feed-forward network with the SwiGLU activation.

Readings where the pages are silent (each is listed with its reason in the
design notes of this repository):

* score function: softmax over the E fp32 logits;
* the bias enters the selection key only (key = p + b); the weights of the
  chosen experts are their unbiased probabilities renormalised to sum to 1;
* equal keys: the lower expert id ranks first;
* SwiGLU: h = silu(W1 x) * (W3 x), out = W2 h, no biases, silu(g) = g / (1 + e^-g);
* shared experts enter with weight 1;
* inside an expert's segment rows follow ascending token id; a segment holds
  ceil(count / align) * align rows and padding rows are zero with token -1.

Parity pins: every function here is pinned by tests under ``tests/`` (closed
forms, brute force over all expert subsets, a hand-derived worked example,
invariants the pages fix, finite differences for the backward).
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    """torch tensor (any dtype, any device) or array -> float64 numpy array."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def _rows(a, rows) -> np.ndarray:
    """a[rows] as float64, for a torch tensor or an array."""
    if hasattr(a, "detach"):
        import torch
        return _f64(a[torch.as_tensor(np.asarray(rows), device=a.device)])
    return _f64(np.asarray(a)[np.asarray(rows)])


# --------------------------------------------------------------------------
# Routing (Technical Report, Method: FP32 gate, aux-loss-free bias, top-6)
# --------------------------------------------------------------------------

def gate_logits(x, w_gate) -> np.ndarray:
    """z[t, e] = sum_i x[t, i] * w_gate[e, i]  (the gate projection)."""
    return _f64(x) @ _f64(w_gate).T


def softmax(z) -> np.ndarray:
    """p = exp(z - max z) / sum exp(z - max z), per row."""
    z = _f64(z)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def select_topk(keys, k: int) -> np.ndarray:
    """Ids of the k largest keys per row, by descending key; equal keys rank
    the lower expert id first."""
    keys = _f64(keys)
    T, E = keys.shape
    ids = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids, -keys), axis=-1)        # primary -key, then id
    return order[:, :k].astype(np.int64)


def route(x, w_gate, bias, k: int, idx=None) -> dict:
    """Gate, softmax, bias-adjusted top-k selection and renormalised weights.

    Returns probs [T,E], keys [T,E] (= probs + bias), idx [T,k] (descending key)
    and w [T,k] (probs of the chosen experts divided by their sum).  A given
    ``idx`` replaces the selection (used where two keys tie within rounding and
    either choice is correct); the weights still follow from the probs.
    """
    z = gate_logits(x, w_gate)
    p = softmax(z)
    keys = p + _f64(bias)[None, :]
    idx = select_topk(keys, k) if idx is None else np.asarray(idx, dtype=np.int64)
    p_sel = np.take_along_axis(p, idx, axis=-1)
    w = p_sel / p_sel.sum(axis=-1, keepdims=True)
    return {"logits": z, "probs": p, "keys": keys, "idx": idx, "w": w}


# --------------------------------------------------------------------------
# Permutation into tile-padded per-expert segments (Technical Report, systems
# paragraph of Method: segments padded to MMA tile multiples)
# --------------------------------------------------------------------------

def capacity(T: int, k: int, E: int, align: int) -> int:
    """Largest number of segment rows any routing can need."""
    return T * k + E * (align - 1)


def permute(idx, E: int, align: int) -> dict:
    """Counting sort of the (token, slot) pairs by expert.

    counts[e]      number of pairs routed to e
    offsets[e]     first row of segment e; offsets[e+1] - offsets[e] is
                   counts[e] rounded up to a multiple of align
    row_of[t*k+j]  row of pair (t, j); rows of a segment follow ascending t
    token_of_row   token of each row, -1 for padding (length = capacity)
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        padded = -(-counts[e] // align) * align
        offsets[e + 1] = offsets[e] + padded
    fill = offsets[:-1].copy()
    row_of = np.zeros(T * k, dtype=np.int64)
    token_of_row = np.full(capacity(T, k, E, align), -1, dtype=np.int64)
    for t in range(T):                       # ascending token id
        for j in range(k):
            e = idx[t, j]
            row_of[t * k + j] = fill[e]
            token_of_row[fill[e]] = t
            fill[e] += 1
    return {"counts": counts, "offsets": offsets, "row_of": row_of,
            "token_of_row": token_of_row}


def gather_rows(x, token_of_row) -> np.ndarray:
    """x_perm[r] = x[token_of_row[r]], zero rows where token_of_row is -1."""
    x = _f64(x)
    tor = np.asarray(token_of_row)
    out = np.zeros((len(tor), x.shape[1]))
    valid = tor >= 0
    out[valid] = x[tor[valid]]
    return out


def unpermute_sum(rows, row_of, w, T: int, k: int) -> np.ndarray:
    """out[t] = sum_j w[t, j] * rows[row_of[t*k + j]], j in ascending order."""
    rows = _f64(rows)
    w = _f64(w)
    out = np.zeros((T, rows.shape[1]))
    for j in range(k):
        out += w[:, j:j + 1] * rows[np.asarray(row_of).reshape(T, k)[:, j]]
    return out


# --------------------------------------------------------------------------
# SwiGLU experts (Model Architecture Features; aibase architecture paragraph)
# --------------------------------------------------------------------------

def silu(g):
    g = _f64(g)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def swiglu_expert(xr, w1, w3, w2):
    """One expert on rows xr: g = xr W1^T, u = xr W3^T, h = silu(g) * u,
    out = h W2^T.  Returns (out, h, g, u)."""
    xr = _f64(xr)
    g = xr @ _f64(w1).T
    u = xr @ _f64(w3).T
    h = silu(g) * u
    return h @ _f64(w2).T, h, g, u


def dense_swiglu(x, w1, w3, w2) -> np.ndarray:
    """The dense SwiGLU FFN of the model's first layer (Technical Report,
    Method: layer 1 is a dense SwiGLU FFN, the other layers MoE):
    y = (silu(x W1^T) * (x W3^T)) W2^T on every token."""
    return swiglu_expert(x, w1, w3, w2)[0]


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------

def forward(inp: dict, align: int = 16, idx=None) -> dict:
    """The MoE FFN forward in the pages' order: route, permute into padded
    segments, one SwiGLU per segment, shared experts on every token, weighted
    combine back to token order.

    ``inp`` holds x, w_gate, bias, w1, w3, w2, ws1, ws3, ws2 (torch or numpy)
    and the config (for k).  ``idx`` optionally fixes the selection.
    """
    cfg = inp["cfg"]
    k, E = cfg.k, cfg.E
    x = _f64(inp["x"])
    T = x.shape[0]
    r = route(x, inp["w_gate"], inp["bias"], k, idx)
    pm = permute(r["idx"], E, align)
    x_perm = gather_rows(x, pm["token_of_row"])
    off = pm["offsets"]
    w1, w3, w2 = inp["w1"], inp["w3"], inp["w2"]
    I = w1.shape[1]
    d = x.shape[1]
    h_perm = np.zeros((len(x_perm), I))
    y_perm = np.zeros((len(x_perm), d))
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        o, h, _, _ = swiglu_expert(x_perm[a:b], w1[e], w3[e], w2[e])
        h_perm[a:b] = h
        y_perm[a:b] = o
    S = inp["ws1"].shape[0]
    y_shared = np.zeros((T, d))
    h_shared = []
    for s in range(S):
        o, h, _, _ = swiglu_expert(x, inp["ws1"][s], inp["ws3"][s], inp["ws2"][s])
        y_shared += o
        h_shared.append(h)
    y = y_shared + unpermute_sum(y_perm, pm["row_of"], r["w"], T, k)
    return {**r, **pm, "x_perm": x_perm, "h_perm": h_perm, "y_perm": y_perm,
            "h_shared": (np.concatenate(h_shared, axis=1) if h_shared else np.zeros((T, 0))),
            "y_shared": y_shared,
            "y": y}


def forward_tokens(inp: dict, tokens, idx=None) -> dict:
    """The layer output for a subset of tokens, without the permutation:
    y_t = sum_s F_s(x_t) + sum_j w_tj F_{e_tj}(x_t), with F_e the SwiGLU expert
    e.  Each expert is applied to the sampled tokens that chose it.  Used for
    sampled parity at sizes the full oracle cannot run.  ``idx`` optionally
    fixes the selection of these tokens."""
    cfg = inp["cfg"]
    tokens = np.asarray(tokens, dtype=np.int64)
    xt = _rows(inp["x"], tokens)
    r = route(xt, inp["w_gate"], inp["bias"], cfg.k, idx)
    ys = np.zeros_like(xt)
    for s in range(inp["ws1"].shape[0]):
        o, _, _, _ = swiglu_expert(xt, inp["ws1"][s], inp["ws3"][s], inp["ws2"][s])
        ys += o
    for e in np.unique(r["idx"]):
        n, j = np.nonzero(r["idx"] == e)
        o, _, _, _ = swiglu_expert(xt[n], inp["w1"][int(e)], inp["w3"][int(e)], inp["w2"][int(e)])
        ys[n] += r["w"][n, j][:, None] * o
    return {**r, "tokens": tokens, "y": ys}


# --------------------------------------------------------------------------
# Backward (Technical Report, Results: the grouped GEMM is also measured in
# the backward pass).  Selection is held fixed; the bias gets no gradient
# because it only enters the selection key.
# --------------------------------------------------------------------------

def silu_grad(g):
    """d silu / dg = s (1 + g (1 - s)) with s = 1 / (1 + e^-g)."""
    g = _f64(g)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def swiglu_expert_backward(xr, w1, w3, w2, dout, with_pre=False):
    """Gradients of out = W2 (silu(W1 x) * W3 x) for rows xr given dout.
    Returns dx, dW1, dW3, dW2 (and dg, du, the gradients at the gate and up
    pre-activations, when with_pre)."""
    xr, w1, w3, w2, dout = map(_f64, (xr, w1, w3, w2, dout))
    g = xr @ w1.T
    u = xr @ w3.T
    sg = silu(g)
    h = sg * u
    dW2 = dout.T @ h
    dh = dout @ w2
    dg = dh * u * silu_grad(g)
    du = dh * sg
    dW1 = dg.T @ xr
    dW3 = du.T @ xr
    dx = dg @ w1 + du @ w3
    if with_pre:
        return dx, dW1, dW3, dW2, dg, du
    return dx, dW1, dW3, dW2


def backward(inp: dict, dy, fwd: dict | None = None, experts=None) -> dict:
    """Gradients of sum(y * dy) for the whole layer, with the routing choice of
    the forward held fixed.

    combine:   d y_perm[row(t,j)] = w[t,j] dy[t];  dw[t,j] = <dy[t], y_perm[row(t,j)]>
    renorm:    dp_sel = (dw - sum_i w_i dw_i) / sum_sel p
    softmax:   dz = p * (dp - <p, dp>)  (dp is zero off the chosen experts)
    gate:      dWg = dz^T x,  dx += dz Wg
    experts:   swiglu_expert_backward per segment and for each shared expert

    ``experts`` (optional) limits which routed experts' weight gradients are
    kept (returned as dicts expert -> array); every expert still contributes
    to dx.  At full size the dense [E, I, d] float64 gradients would not fit.
    """
    cfg = inp["cfg"]
    k, E = cfg.k, cfg.E
    if fwd is None:
        fwd = forward(inp)
    x = _f64(inp["x"])
    dy = _f64(dy)
    T, d = x.shape
    w = fwd["w"]
    idx = fwd["idx"]
    p = fwd["probs"]
    row_of = fwd["row_of"].reshape(T, k)
    y_perm = fwd["y_perm"]
    # combine backward
    dw = np.zeros((T, k))
    dy_perm = np.zeros_like(y_perm)
    for j in range(k):
        rows = row_of[:, j]
        dw[:, j] = np.sum(dy * y_perm[rows], axis=1)
        dy_perm[rows] = w[:, j:j + 1] * dy
    # experts
    x_perm = fwd["x_perm"]
    off = fwd["offsets"]
    dx_perm = np.zeros_like(x_perm)
    keep = range(E) if experts is None else [int(e) for e in experts]
    if experts is None:
        dW1 = np.zeros(inp["w1"].shape)
        dW3 = np.zeros(inp["w3"].shape)
        dW2 = np.zeros(inp["w2"].shape)
    else:
        dW1 = {e: np.zeros(inp["w1"].shape[1:]) for e in keep}
        dW3 = {e: np.zeros(inp["w3"].shape[1:]) for e in keep}
        dW2 = {e: np.zeros(inp["w2"].shape[1:]) for e in keep}
    I = inp["w1"].shape[1]
    dgu_perm = np.zeros((len(x_perm), 2 * I))
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if a == b:
            continue
        dxe, g1, g3, g2, dg, du = swiglu_expert_backward(x_perm[a:b], inp["w1"][e],
                                                         inp["w3"][e], inp["w2"][e],
                                                         dy_perm[a:b], with_pre=True)
        dx_perm[a:b] = dxe
        dgu_perm[a:b, :I], dgu_perm[a:b, I:] = dg, du
        if e in keep:
            dW1[e], dW3[e], dW2[e] = g1, g3, g2
    S = inp["ws1"].shape[0]
    dWs1 = np.zeros(inp["ws1"].shape)
    dWs3 = np.zeros(inp["ws3"].shape)
    dWs2 = np.zeros(inp["ws2"].shape)
    dx = np.zeros((T, d))
    dg_sh, du_sh = [], []
    for s in range(S):
        dxs, g1, g3, g2, dg, du = swiglu_expert_backward(x, inp["ws1"][s], inp["ws3"][s],
                                                         inp["ws2"][s], dy, with_pre=True)
        dx += dxs
        dWs1[s], dWs3[s], dWs2[s] = g1, g3, g2
        dg_sh.append(dg)
        du_sh.append(du)
    for j in range(k):                       # un-permute: gather-sum
        dx += dx_perm[row_of[:, j]]
    # renormalisation and softmax backward, then the gate projection
    p_sel = np.take_along_axis(p, idx, axis=-1)
    ssum = p_sel.sum(axis=1, keepdims=True)
    dp_sel = (dw - np.sum(w * dw, axis=1, keepdims=True)) / ssum
    dp = np.zeros_like(p)
    np.put_along_axis(dp, idx, dp_sel, axis=1)
    dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    wg = _f64(inp["w_gate"])
    dWg = dz.T @ x
    dx += dz @ wg
    dgu_shared = np.concatenate(dg_sh + du_sh, axis=1) if S else np.zeros((T, 0))
    return {"dx": dx, "dw_gate": dWg, "dw1": dW1, "dw3": dW3, "dw2": dW2,
            "dws1": dWs1, "dws3": dWs3, "dws2": dWs2, "dw": dw, "dz": dz,
            "dy_perm": dy_perm, "dx_perm": dx_perm, "dgu_perm": dgu_perm,
            "dgu_shared": dgu_shared}


# --------------------------------------------------------------------------
# Load balancing, training side (Technical Report, Method: the DeepSeek
# auxiliary-loss-free bias update, complemented by a sequence-wise balance
# loss against extreme imbalance inside one sequence).  The pages name both
# mechanisms but give no formula; the forms below are the published DeepSeek
# ones the report points to (the reading is listed in the design notes).
# --------------------------------------------------------------------------

def balance_stats(probs, idx, E: int, k: int, seq_len: int, alpha: float) -> dict:
    """Sequence-wise balance statistics and loss.

    The T tokens are T / seq_len consecutive sequences of seq_len tokens.  For
    sequence s and expert e:

      f[s, e] = E / (k * seq_len) * (number of (token, slot) pairs of s routed to e)
      P[s, e] = (1 / seq_len) * sum over the tokens t of s of probs[t, e]

    (softmax probabilities already sum to 1 per token, so they are their own
    normalised affinities), and

      loss = alpha / n_seq * sum_s sum_e f[s, e] * P[s, e]

    i.e. the mean over sequences of alpha * sum_e f * P.  Returns f, P
    [n_seq, E], the per-sequence selection counts and the loss.
    """
    p = _f64(probs)
    idx = np.asarray(idx, dtype=np.int64)
    T = idx.shape[0]
    assert seq_len > 0 and T % seq_len == 0, "T must be a whole number of sequences"
    n_seq = T // seq_len
    f = np.zeros((n_seq, E))
    P = np.zeros((n_seq, E))
    counts = np.zeros((n_seq, E), dtype=np.int64)
    for s in range(n_seq):
        t0, t1 = s * seq_len, (s + 1) * seq_len
        for t in range(t0, t1):
            for j in range(k):
                counts[s, idx[t, j]] += 1
        f[s] = E * counts[s] / (k * seq_len)
        P[s] = p[t0:t1].sum(axis=0) / seq_len
    loss = alpha * float(np.sum(f * P)) / n_seq if n_seq else 0.0
    return {"f": f, "P": P, "counts": counts, "loss": loss}


def bias_update(bias, counts, gamma: float, T: int, k: int) -> np.ndarray:
    """Auxiliary-loss-free bias step: an expert that received more than the
    mean load T*k/E of the batch has its bias lowered by gamma, one that
    received less has it raised by gamma, one exactly at the mean keeps it.
    ``counts`` are the batch's per-expert pair counts (summed over all
    data-parallel replicas when there are several)."""
    b = _f64(bias)
    c = np.asarray(counts, dtype=np.int64)
    E = b.shape[0]
    excess = E * c - T * k                 # E * (count - mean), exact integers
    step = -np.sign(excess).astype(np.float64)
    return np.where(step == 0, b, b + gamma * step)


# --------------------------------------------------------------------------
# Expert parallelism (Technical Report, Method / Key claims, systems
# paragraph: the MoE all-to-all between ranks, overlapped with the grouped
# GEMMs; "How dots.llm1's 14B MoE Architecture Matches 72B LLM Performance",
# Computational Infrastructure Innovations: all-to-all expert communication).
# The pages name the exchange but not its layout.  The reading used here:
# rank r of W owns the experts [r E/W, (r+1) E/W); every rank routes its own
# tokens; on the owner, expert e's segment holds the (token, slot) pairs of e
# from every rank, ordered by source rank and then by the source's own
# segment order (ascending token id), padded to `align` rows.  The layer's
# output is unchanged by the exchange: each rank's y is forward() of its own
# tokens.
# --------------------------------------------------------------------------

def ep_layout(idx_per_rank, E: int, align: int) -> dict:
    """Receive layout of the dispatch among W = len(idx_per_rank) ranks.

    idx_per_rank[s] is the [T_s, k] expert choice of rank s.  Returns

      recv_offsets[r]  [E/W + 1]  first row of each local expert's segment on
                                  rank r (segment le holds expert r E/W + le)
      recv_counts[r]   [E/W]      pairs rank r receives for each local expert
      owner[s], row[s] [T_s * k]  rank and receive row of pair (t, j) of rank s
                                  at index t*k + j
      src_of_row[r]    list of (source rank, token) per receive row of rank r,
                       (-1, -1) for padding rows

    Built by walking the pairs in the order the layout defines, one row at a
    time.
    """
    W = len(idx_per_rank)
    assert W > 0 and E % W == 0, "the experts must split evenly over the ranks"
    El = E // W
    idx = [np.asarray(a, dtype=np.int64) for a in idx_per_rank]
    owner = [np.full(a.size, -1, dtype=np.int64) for a in idx]
    row = [np.full(a.size, -1, dtype=np.int64) for a in idx]
    recv_offsets = np.zeros((W, El + 1), dtype=np.int64)
    recv_counts = np.zeros((W, El), dtype=np.int64)
    src_of_row = []
    for r in range(W):
        rows = []
        for le in range(El):
            e = r * El + le
            recv_offsets[r, le] = len(rows)
            for s in range(W):
                T_s, k = idx[s].shape
                for t in range(T_s):
                    for j in range(k):
                        if idx[s][t, j] == e:
                            owner[s][t * k + j] = r
                            row[s][t * k + j] = len(rows)
                            rows.append((s, t))
            recv_counts[r, le] = len(rows) - recv_offsets[r, le]
            while (len(rows) - recv_offsets[r, le]) % align:
                rows.append((-1, -1))
        recv_offsets[r, El] = len(rows)
        src_of_row.append(rows)
    return {"recv_offsets": recv_offsets, "recv_counts": recv_counts, "owner": owner,
            "row": row, "src_of_row": src_of_row}


def ep_recv_rows(x_per_rank, layout: dict, r: int) -> np.ndarray:
    """Rows rank r holds after the dispatch: x of the source token of each
    receive row, zero rows for padding."""
    rows = layout["src_of_row"][r]
    d = _f64(x_per_rank[0][:1]).shape[1]
    out = np.zeros((len(rows), d))
    for i, (s, t) in enumerate(rows):
        if s >= 0:
            out[i] = _f64(x_per_rank[s][t:t + 1])[0]
    return out
