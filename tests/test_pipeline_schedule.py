"""The interleaved-1F1B schedule with the MoE all-to-all overlapped
(pipeline_schedule.py), on CPU: its structure (every pass once, forward
before backward, the published warm-up counts, one more warm-up forward in
the overlapped variant), deadlock freedom and peak activation memory under
the cross-stage dependencies, the all-to-all hidden in the steady phase, and
an execution by real processes (gloo ranks exchanging activations and
gradients point to point) whose weight gradients equal a sequential pass."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fine_grained_moe_fp32_b200 import pipeline_schedule as S

SHAPES = [(1, 1, 3), (2, 1, 4), (4, 1, 8), (2, 2, 4), (4, 2, 8), (4, 3, 12), (8, 2, 16), (3, 2, 9)]


@pytest.mark.parametrize("P,V,M", SHAPES)
@pytest.mark.parametrize("overlap", [False, True])
def test_every_pass_once_and_forward_before_backward(P, V, M, overlap):
    stages = S.interleaved_1f1b(P, V, M, overlap)
    for r, steps in enumerate(stages):
        ops = [op for step in steps for op in step]
        want = {(k, m, v) for k in "FB" for m in range(M) for v in range(V)}
        assert sorted(ops) == sorted(want)
        at = {op: i for i, step in enumerate(steps) for op in step}
        for m in range(M):
            for v in range(V):
                assert at[("F", m, v)] < at[("B", m, v)]
        if overlap:
            for step in steps:
                if len(step) == 2:   # a pair: one forward, one backward, two microbatches
                    (kf, mf, _), (kb, mb, _) = step
                    assert (kf, kb) == ("F", "B") and mf != mb


def test_published_warmup_counts_and_the_extra_forward():
    """Plain: W = 2 (P-1-r) + (V-1) P warm-up forwards (capped at M V), so
    W + 1 forwards have run when the first backward runs; overlapped: one
    warm-up forward more, so W + 2 (the last with the first backward, in one
    paired step), capped at M V."""
    def forwards_until_first_backward(steps):
        n = 0
        for st in steps:
            n += sum(o[0] == "F" for o in st)
            if any(o[0] == "B" for o in st):
                return n
        return n

    for P, V, M in SHAPES:
        plain = S.interleaved_1f1b(P, V, M, False)
        ovl = S.interleaved_1f1b(P, V, M, True)
        for r in range(P):
            w = min(M * V, 2 * (P - 1 - r) + (V - 1) * P)
            assert S.warmup_forwards(P, V, M, r) == w
            assert forwards_until_first_backward(plain[r]) == min(M * V, w + 1)
            assert forwards_until_first_backward(ovl[r]) == min(M * V, w + 2)


def test_plain_order_by_hand_p2_v2():
    """P = 2, V = 2, M = 2 worked by hand.  Stage 0: W = 2*1 + 1*2 = 4
    forwards (m0 c0, m1 c0, m0 c1, m1 c1), then the backwards chunk 1 first
    (m0 c1, m1 c1, m0 c0, m1 c0).  Stage 1: W = 2 forwards, then F m0 c1,
    B m0 c1, F m1 c1, B m1 c1, then B m0 c0, B m1 c0."""
    st = S.interleaved_1f1b(2, 2, 2, False)
    flat = [[op for step in s for op in step] for s in st]
    assert flat[0] == [("F", 0, 0), ("F", 1, 0), ("F", 0, 1), ("F", 1, 1),
                       ("B", 0, 1), ("B", 1, 1), ("B", 0, 0), ("B", 1, 0)]
    assert flat[1] == [("F", 0, 0), ("F", 1, 0), ("F", 0, 1), ("B", 0, 1), ("F", 1, 1),
                       ("B", 1, 1), ("B", 0, 0), ("B", 1, 0)]


def test_dependencies_producer_consumer_inverse():
    for P, V, _ in SHAPES:
        for r in range(P):
            for kind in "FB":
                for v in range(V):
                    op = (kind, 0, v)
                    c = S.consumer(op, P, V, r)
                    if c is not None:
                        assert S.producer(c[1], P, V, c[0]) == (r, op)


@pytest.mark.parametrize("P,V,M", SHAPES)
def test_no_deadlock_and_no_extra_activation_memory(P, V, M):
    plain = S.simulate(S.interleaved_1f1b(P, V, M, False), P, V, 1.0, 2.0, 0.0)
    ovl = S.simulate(S.interleaved_1f1b(P, V, M, True), P, V, 1.0, 2.0, 0.0)
    assert ovl.peak_in_flight == plain.peak_in_flight
    # the plain schedule holds W_r + 1 chunk activations at most (capped at M V)
    for r in range(P):
        assert plain.peak_in_flight[r] == min(M * V, 2 * (P - 1 - r) + (V - 1) * P + 1)


@pytest.mark.parametrize("P,V,M", [(4, 1, 8), (4, 2, 8), (8, 2, 16)])
def test_alltoall_hidden_in_the_steady_phase(P, V, M):
    """Without communication both schedules take the same time; with an
    all-to-all per pass the overlapped one is shorter, and when the
    all-to-all fits under the paired compute (2 a <= f + b) every steady
    step costs only its compute."""
    f, b = 1.0, 2.0
    t0 = [S.simulate(S.interleaved_1f1b(P, V, M, o), P, V, f, b, 0.0).makespan
          for o in (False, True)]
    assert t0[0] == t0[1]
    for a in (0.5, 1.0, 1.5):
        plain = S.simulate(S.interleaved_1f1b(P, V, M, False), P, V, f, b, a)
        ovl = S.simulate(S.interleaved_1f1b(P, V, M, True), P, V, f, b, a)
        assert ovl.makespan < plain.makespan
        paired = sum(len(st) == 2 for st in S.interleaved_1f1b(P, V, M, True)[0])
        single = len(S.interleaved_1f1b(P, V, M, True)[0]) - paired
        busy0 = paired * max(f + b, 2 * a) + sum(
            (f if st[0][0] == "F" else b) + a
            for st in S.interleaved_1f1b(P, V, M, True)[0] if len(st) == 1)
        assert ovl.busy[0] == pytest.approx(busy0)
        assert single > 0 and paired > 0


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        S.interleaved_1f1b(2, 1, 3)
    with pytest.raises(ValueError):
        S.interleaved_1f1b(0, 1, 2)


# ---------------------------------------------------------------- execution

H, N = 6, 3   # feature width and rows of a microbatch


def _layer_weights(L):
    rng = np.random.default_rng(11)
    return [rng.standard_normal((H, H)) * 0.4 for _ in range(L)]


def _inputs(M):
    rng = np.random.default_rng(12)
    return [rng.standard_normal((N, H)) for _ in range(M)]


def _sequential_grads(L, M):
    """Layer l: y = tanh(x W_l); loss of a microbatch = sum(y_L^2) / 2."""
    W = _layer_weights(L)
    dW = [np.zeros((H, H)) for _ in range(L)]
    for x in _inputs(M):
        acts = []
        for l in range(L):
            y = np.tanh(x @ W[l])
            acts.append((x, y))
            x = y
        dy = x
        for l in reversed(range(L)):
            xin, y = acts[l]
            dz = dy * (1.0 - y * y)
            dW[l] += xin.T @ dz
            dy = dz @ W[l].T
    return dW


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _stage_worker(r, P, V, M, overlap, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=r, world_size=P)
    try:
        L = P * V
        W = _layer_weights(L)
        X = _inputs(M)
        dW = {v: np.zeros((H, H)) for v in range(V)}
        saved = {}
        pending = []

        def tag(kind, m, v, src):
            return ((m * V + v) * 2 + (kind == "B")) * P + src

        def recv(src_stage, src_op):
            buf = torch.empty((N, H), dtype=torch.float64)
            dist.recv(buf, src=src_stage, tag=tag(*src_op, src_stage))
            return buf.numpy()

        def send(arr, dst_stage, op):
            pending.append(dist.isend(torch.from_numpy(np.ascontiguousarray(arr)),
                                      dst=dst_stage, tag=tag(*op, r)))

        for step in S.interleaved_1f1b(P, V, M, overlap)[r]:
            for op in step:   # a pair runs its forward, then its backward
                kind, m, v = op
                l = v * P + r
                src = S.producer(op, P, V, r)
                dst = S.consumer(op, P, V, r)
                if kind == "F":
                    x = X[m] if src is None else recv(*src)
                    y = np.tanh(x @ W[l])
                    saved[(m, v)] = (x, y)
                    if dst is not None:
                        send(y, dst[0], op)
                else:
                    xin, y = saved.pop((m, v))
                    dy = y if src[0] == r and src[1][0] == "F" else recv(*src)
                    dz = dy * (1.0 - y * y)
                    dW[v] += xin.T @ dz
                    if dst is not None:
                        send(dz @ W[l].T, dst[0], op)
        for p in pending:
            p.wait()
        out[r] = {v: dW[v].tolist() for v in range(V)}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("P,V,overlap", [(2, 2, True), (3, 2, True), (3, 1, False),
                                         (2, 2, False)])
def test_processes_running_the_schedule_reproduce_sequential_gradients(P, V, overlap):
    M = 2 * P
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_stage_worker, args=(P, V, M, overlap, port, out), nprocs=P,
                           join=True, start_method="spawn")
        res = dict(out)
    ref = _sequential_grads(P * V, M)
    for r in range(P):
        for v in range(V):
            np.testing.assert_allclose(np.array(res[r][v]), ref[v * P + r], rtol=1e-13,
                                       atol=1e-13)
