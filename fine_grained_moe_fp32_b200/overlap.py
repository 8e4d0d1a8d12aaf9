"""Overlapped execution on one GPU: the MoE all-to-all of one microbatch under
another microbatch's grouped GEMMs, and the paired forward/backward steps of
the overlapped 1F1B schedule.

dots.llm1 Technical Report, Method / Key claims (systems paragraph): the
expert all-to-all is hidden behind computation; in the interleaved 1F1B
schedule the steady state runs a forward and a backward of two different
microbatches together.  Both are realised here with CUDA streams and events
around the library's calls (every step still runs in the library's kernels):

* ``EPOverlap`` splits each emulated rank's batch into microbatches, each
  with its own ``moe.EPRanks`` state (workspace, receive buffers), and issues
  every microbatch's route -> dispatch -> experts -> combine chain on its own
  stream.  The chains share nothing but the read-only weights, so the
  scheduler may run one chain's memory-bound dispatch and combine kernels on
  the SMs next to the other chain's tensor-core GEMMs.  ``serial`` issues the
  same calls on one stream, one microbatch after the other: the results are
  bit-identical (the kernels are deterministic and the chains independent).

* ``PipelineStage`` executes one stage's step list from
  ``pipeline_schedule.interleaved_1f1b`` with the layer's training calls.  A
  step of two ops (a forward and a backward of different microbatches) issues
  the forward on one stream and the backward on the other; every step ends
  with both streams joined (the step boundary, where a multi-stage pipeline
  exchanges activations and gradients).  Each microbatch in flight owns a
  training workspace from a pool; a backward returns its workspace once its
  kernels are done (an event orders the next forward that takes it).
"""
from __future__ import annotations

import torch

from . import moe as M


def split_sizes(T: int, n: int) -> list[int]:
    """n microbatch sizes summing to T, the first ones one token larger."""
    if n < 1 or T < n:
        raise ValueError("need 1 <= n <= T")
    return [T // n + (1 if i < T % n else 0) for i in range(n)]


class EPOverlap:
    """Expert parallelism over ``world`` emulated ranks with each rank's T
    tokens split into ``n_micro`` microbatches on their own streams."""

    def __init__(self, inputs: dict, world: int, T: int, n_micro: int = 2, align: int = 16,
                 device="cuda"):
        self.device = torch.device(device)
        self.sizes = split_sizes(T, n_micro)
        self.world, self.T, self.d = int(world), int(T), inputs["cfg"].d
        self.parts = [M.EPRanks(inputs, world, t, align, self.device) for t in self.sizes]
        self.streams = [torch.cuda.Stream(self.device) for _ in self.sizes]
        self.starts = [sum(self.sizes[:i]) for i in range(len(self.sizes))]

    def _slices(self, ts, i):
        a, n = self.starts[i], self.sizes[i]
        return [t[a:a + n] for t in ts]

    def _alloc(self, ys):
        if ys is None:
            ys = [torch.empty((self.T, self.d), dtype=torch.bfloat16, device=self.device)
                  for _ in range(self.world)]
        return ys

    def __call__(self, xs, ys=None, events=None):
        """Overlapped step.  xs, ys: the ranks' [T, d] batches.  ``events``
        (optional): per microbatch a list of 5 timing events recorded on its
        stream before route and after route, dispatch, experts and combine."""
        ys = self._alloc(ys)
        cur = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(cur)
        for i, (ep, st) in enumerate(zip(self.parts, self.streams)):
            st.wait_event(start)
            xi, yi = self._slices(xs, i), self._slices(ys, i)
            ev = events[i] if events is not None else None
            with torch.cuda.stream(st):
                if ev is not None:
                    ev[0].record(st)
                ep.route(xi, st)
                if ev is not None:
                    ev[1].record(st)
                ep.dispatch(xi, st)
                if ev is not None:
                    ev[2].record(st)
                ep.experts_step(xi, st)
                if ev is not None:
                    ev[3].record(st)
                ep.combine(yi, st)
                if ev is not None:
                    ev[4].record(st)
        for st in self.streams:   # the caller's stream sees every microbatch done
            done = torch.cuda.Event()
            done.record(st)
            cur.wait_event(done)
        return ys

    def serial(self, xs, ys=None):
        """The same calls on the current stream, microbatch after microbatch."""
        ys = self._alloc(ys)
        for i, ep in enumerate(self.parts):
            ep(self._slices(xs, i), self._slices(ys, i))
        return ys


class PipelineStage:
    """One pipeline stage of the MoE layer on this GPU, driven by a step list
    of ``pipeline_schedule.interleaved_1f1b``.  ``layers[v]`` is the layer of
    model chunk v (one layer per chunk); every microbatch has T tokens.  The
    chunks of a microbatch chain: chunk v > 0 takes chunk v-1's output, and
    chunk v < V-1's backward takes chunk v+1's dx as its upstream gradient,
    which must then be bf16 (``grad_dtype``)."""

    def __init__(self, layers, T: int, grad_dtype=torch.float32):
        self.layers = list(layers)
        self.T = int(T)
        self.grad_dtype = grad_dtype
        if len(self.layers) > 1 and grad_dtype != torch.bfloat16:
            raise ValueError("chained chunks pass dx on as a bf16 upstream gradient")
        dev = self.layers[0].device
        self.device = dev
        self.fwd_stream = torch.cuda.Stream(dev)
        self.bwd_stream = torch.cuda.Stream(dev)
        self._free = []   # (workspace, event after its last use)
        nbytes = M.train_workspace_size(self.layers[0].dims(T))
        self._nbytes = nbytes

    def _take(self, st):
        if self._free:
            ws, ev = self._free.pop()
            st.wait_event(ev)
            return ws
        return M.guard_layout(M.alloc_workspace(self._nbytes, self.device),
                              M.train_layout(self.layers[0].dims(self.T)))

    def run(self, steps, xs, dys, grads=None, ys=None):
        """Execute ``steps`` (a stage's list from interleaved_1f1b).  xs[m],
        dys[m]: microbatch m's tokens and upstream gradient; ``grads`` maps
        (m, chunk) to a gradient dict (allocated when missing).  Returns
        (ys, grads) with ys keyed by (m, chunk)."""
        grads = {} if grads is None else grads
        ys = {} if ys is None else ys
        live = {}   # (m, chunk) -> training workspace
        cur = torch.cuda.current_stream(self.device)
        boundary = torch.cuda.Event()
        boundary.record(cur)
        T = self.T
        for step in steps:
            for st in (self.fwd_stream, self.bwd_stream):
                st.wait_event(boundary)
            for kind, m, v in step:
                layer = self.layers[v]
                dm = layer.dims(T)
                if kind == "F":
                    st = self.fwd_stream
                    with torch.cuda.stream(st):
                        ws = self._take(st)
                        y = ys.get((m, v))
                        if y is None:
                            y = torch.empty((T, layer.cfg.d), dtype=torch.bfloat16,
                                            device=self.device)
                            ys[(m, v)] = y
                        x = xs[m] if v == 0 else ys[(m, v - 1)]
                        M.forward_train(dm, x, layer.w_gate, layer.bias, layer.w1, layer.w3,
                                        layer.w2, layer.ws1, layer.ws3, layer.ws2, y, ws, st)
                    live[(m, v)] = ws
                elif kind == "B":
                    st = self.bwd_stream
                    ws = live.pop((m, v))
                    g = grads.get((m, v))
                    with torch.cuda.stream(st):
                        if g is None:
                            g = layer.alloc_grads(T, self.grad_dtype)
                            grads[(m, v)] = g
                        x = xs[m] if v == 0 else ys[(m, v - 1)]
                        dy = dys[m] if v == len(self.layers) - 1 else grads[(m, v + 1)]["dx"]
                        M.backward(dm, x, layer.w_gate, layer.w1, layer.w3, layer.w2,
                                   layer.ws1, layer.ws3, layer.ws2, dy, ws, g, st)
                        done = torch.cuda.Event()
                        done.record(st)
                    self._free.append((ws, done))
                else:
                    raise ValueError(f"unknown op {kind}")
            boundary = torch.cuda.Event()
            join = torch.cuda.Event()
            join.record(self.bwd_stream)
            self.fwd_stream.wait_event(join)
            boundary.record(self.fwd_stream)
        if live:
            raise ValueError(f"forwards without a backward: {sorted(live)}")
        cur.wait_event(boundary)
        return ys, grads

    def sequential(self, steps, xs, dys, grads=None, ys=None):
        """The same ops in the schedule's order on the current stream, one at
        a time (the reference the overlapped run must equal)."""
        flat = [[op] for step in steps for op in sorted(step, key=lambda o: o[0] != "F")]
        cur = torch.cuda.current_stream(self.device)
        saved = (self.fwd_stream, self.bwd_stream)
        self.fwd_stream = self.bwd_stream = cur
        try:
            return self.run(flat, xs, dys, grads, ys)
        finally:
            self.fwd_stream, self.bwd_stream = saved
