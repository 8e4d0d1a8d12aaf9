"""Property-based pins of the oracle's index work (hypothesis, CPU): for
random routings of random shapes, the permutation and the expert-parallel
receive layout keep the invariants the pages fix (every pair routed once, no
token dropped, segments padded to the tile multiple and holding one expert,
rows in ascending token order) and agree with each other where they must."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import moe_oracle as O


@st.composite
def routings(draw, max_ranks=1):
    E = draw(st.integers(1, 12))
    k = draw(st.integers(1, min(E, 4)))
    W = draw(st.sampled_from([w for w in range(1, max_ranks + 1) if E % w == 0]))
    align = draw(st.sampled_from([1, 2, 4, 16]))
    idx = []
    for _ in range(W):
        T = draw(st.integers(0, 24))
        rows = [draw(st.permutations(range(E)))[:k] for _ in range(T)]
        idx.append(np.array(rows, dtype=np.int64).reshape(T, k))
    return E, k, W, align, idx


@settings(max_examples=80, deadline=None)
@given(routings())
def test_permutation_invariants(case):
    E, k, _, align, (idx,) = case
    T = idx.shape[0]
    P = O.permute(idx, E, align)
    counts, off, row_of, tor = P["counts"], P["offsets"], P["row_of"], P["token_of_row"]
    assert counts.sum() == T * k                                    # no token dropped
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    seg = np.diff(off)
    assert off[0] == 0 and (seg % align == 0).all() and (seg >= counts).all()
    assert (seg - counts < align).all()                             # the least padding
    assert off[-1] <= O.capacity(T, k, E, align)
    assert len(set(row_of.tolist())) == T * k                       # rows distinct
    for t in range(T):
        for j in range(k):
            e, r = idx[t, j], row_of[t * k + j]
            assert off[e] <= r < off[e] + counts[e] and tor[r] == t
    for e in range(E):                                              # ascending tokens
        toks = tor[off[e]:off[e] + counts[e]]
        assert (np.diff(toks) > 0).all()
        assert (tor[off[e] + counts[e]:off[e + 1]] == -1).all()


@settings(max_examples=60, deadline=None)
@given(routings(max_ranks=6))
def test_ep_layout_invariants(case):
    E, k, W, align, idx = case
    L = O.ep_layout(idx, E, align)
    El = E // W
    total = sum(a.shape[0] for a in idx) * k
    assert sum(int(L["recv_counts"][r].sum()) for r in range(W)) == total
    for r in range(W):
        off, cnt = L["recv_offsets"][r], L["recv_counts"][r]
        assert off[0] == 0 and (np.diff(off) % align == 0).all()
        assert (np.diff(off) - cnt >= 0).all() and (np.diff(off) - cnt < align).all()
        assert len(L["src_of_row"][r]) == off[-1]
    for s, a in enumerate(idx):
        for p in range(a.size):
            e = int(a.reshape(-1)[p])
            r, row = int(L["owner"][s][p]), int(L["row"][s][p])
            le = e - r * El
            assert r == e // El
            assert L["recv_offsets"][r, le] <= row < L["recv_offsets"][r, le] + \
                L["recv_counts"][r, le]
            assert L["src_of_row"][r][row] == (s, p // k)
    if W == 1:   # one rank: the layout is the permutation's
        P = O.permute(idx[0], E, align)
        np.testing.assert_array_equal(L["recv_offsets"][0], P["offsets"])
        np.testing.assert_array_equal(L["row"][0], P["row_of"])
