"""Pipeline schedule of the training step: interleaved 1F1B with the MoE
all-to-all overlapped (dots.llm1 Technical Report, Method / Key claims,
systems paragraph, and "How dots.llm1's 14B MoE Architecture Matches 72B LLM
Performance", Computational Infrastructure Innovations).  What the pages fix:
in the steady state the expert all-to-all is hidden behind the math of
another pass; the price is a single additional warm-up pass; the activation
footprint stays that of the plain schedule.

The pages give those properties, not the schedule.  The reading built here:

* P pipeline stages, V model chunks per stage (chunk v of stage r is the
  layer block v*P + r, so a microbatch visits stages 0..P-1 V times), M
  microbatches, M a multiple of P;
* plain interleaved 1F1B (the published order): stage r first runs
  W_r = min(M*V, 2*(P-1-r) + (V-1)*P) forward passes, then alternates one
  forward and one backward, then runs the remaining backward passes.  Its
  k-th forward processes microbatch (k // (P*V))*P + k % P on chunk
  (k // P) % V; its k-th backward the same microbatch on chunk
  V-1-(k // P) % V;
* the overlapped variant: one more warm-up forward (W_r + 1 when one is
  left), then every steady step runs a forward and a backward of two
  different microbatches together, so the all-to-all of each runs while the
  other computes; the cool-down backward passes run alone.  Counting a paired
  step as allocating and freeing one microbatch's activations together, its
  peak number of microbatches in flight equals the plain schedule's.

A schedule is a list per stage of steps; a step is a tuple of ops, an op a
tuple (kind, microbatch, chunk) with kind "F" or "B".  ``simulate`` runs the
steps against the cross-stage dependencies with given durations.
"""
from __future__ import annotations

import dataclasses


def _fwd(k: int, P: int, V: int) -> tuple[str, int, int]:
    return ("F", (k // (P * V)) * P + k % P, (k // P) % V)


def _bwd(k: int, P: int, V: int) -> tuple[str, int, int]:
    return ("B", (k // (P * V)) * P + k % P, V - 1 - (k // P) % V)


def warmup_forwards(P: int, V: int, M: int, r: int) -> int:
    """Forward passes stage r runs before its first backward (plain order)."""
    return min(M * V, 2 * (P - 1 - r) + (V - 1) * P)


def interleaved_1f1b(P: int, V: int, M: int, overlap: bool = False) -> list[list[tuple]]:
    """Per-stage step lists of the plain (``overlap=False``) or the
    all-to-all-overlapped interleaved 1F1B schedule."""
    if P < 1 or V < 1 or M < 1 or M % P:
        raise ValueError("need P, V, M >= 1 with M a multiple of P")
    total = M * V
    stages = []
    for r in range(P):
        w = warmup_forwards(P, V, M, r)
        if overlap:
            w = min(total, w + 1)
        steps = [(_fwd(k, P, V),) for k in range(w)]
        for i in range(total - w):
            f, b = _fwd(w + i, P, V), _bwd(i, P, V)
            steps.append((f, b) if overlap else (f,))
            if not overlap:
                steps.append((b,))
        steps += [(_bwd(k, P, V),) for k in range(total - w, total)]
        stages.append(steps)
    return stages


def producer(op: tuple, P: int, V: int, r: int):
    """(stage, op) whose output op (kind, m, v) on stage r consumes, or None.

    A forward of chunk v on stage r takes the activation of the same chunk on
    stage r-1, or of chunk v-1 on the last stage when r = 0; a backward takes
    the gradient of the same chunk on stage r+1, or of chunk v+1 on stage 0
    when r = P-1; the last layer's backward starts from its own forward."""
    kind, m, v = op
    if kind == "F":
        if r > 0:
            return r - 1, ("F", m, v)
        return (P - 1, ("F", m, v - 1)) if v > 0 else None
    if r < P - 1:
        return r + 1, ("B", m, v)
    return (0, ("B", m, v + 1)) if v < V - 1 else (r, ("F", m, v))


def consumer(op: tuple, P: int, V: int, r: int):
    """(stage, op) that consumes the output of op on stage r, or None (the
    last layer's forward feeds its own backward; the first layer's backward
    ends the microbatch)."""
    kind, m, v = op
    if kind == "F":
        if r < P - 1:
            return r + 1, ("F", m, v)
        return (0, ("F", m, v + 1)) if v < V - 1 else None
    if r > 0:
        return r - 1, ("B", m, v)
    return (P - 1, ("B", m, v - 1)) if v > 0 else None


@dataclasses.dataclass
class SimResult:
    makespan: float
    finish: dict            # (stage, op) -> finish time
    peak_in_flight: list    # per stage: most chunk activations held between steps
    busy: list              # per stage: time spent in steps


def simulate(stages: list, P: int, V: int, f: float = 1.0, b: float = 2.0,
             a2a: float = 0.0) -> SimResult:
    """Run the schedule with compute times f (forward) and b (backward) per
    chunk and an all-to-all of a2a per pass.  A single op costs its compute
    plus its all-to-all; a paired step costs max(f + b, 2 a2a), its two
    all-to-alls hidden behind the other's compute.  Each stage runs its steps
    in order; a step starts once the stage is free and every op's producer
    has finished.  Raises if the schedule deadlocks."""
    finish = {}
    pos = [0] * P
    free_at = [0.0] * P
    busy = [0.0] * P
    live = [0] * P
    peak = [0] * P
    remaining = sum(len(s) for s in stages)
    while remaining:
        progressed = False
        for r in range(P):
            while pos[r] < len(stages[r]):
                step = stages[r][pos[r]]
                ready = free_at[r]
                ok = True
                for op in step:
                    src = producer(op, P, V, r)
                    if src is None:
                        continue
                    if src not in finish:
                        ok = False
                        break
                    ready = max(ready, finish[src])
                if not ok:
                    break
                if len(step) == 1:
                    dur = (f if step[0][0] == "F" else b) + a2a
                else:
                    dur = max(f + b, 2 * a2a)
                end = ready + dur
                for op in step:
                    finish[(r, op)] = end
                free_at[r] = end
                busy[r] += dur
                nf = sum(op[0] == "F" for op in step)
                live[r] += nf - (len(step) - nf)   # a pair allocates and frees together
                peak[r] = max(peak[r], live[r])
                pos[r] += 1
                remaining -= 1
                progressed = True
        if not progressed:
            raise RuntimeError(f"schedule deadlocks at steps {pos}")
    return SimResult(max(free_at), finish, peak, busy)
