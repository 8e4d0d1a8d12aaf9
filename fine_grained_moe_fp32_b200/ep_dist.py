"""Expert parallelism across processes: one process per GPU, the ranks of a
torch.distributed group (dots.llm1 Technical Report, Method / Key claims,
systems paragraph: the MoE all-to-all between ranks; "How dots.llm1's 14B MoE
Architecture Matches 72B LLM Performance", Computational Infrastructure
Innovations).

Every rank holds the weights of its E/W routed experts and of the shared
experts, routes its own T tokens, and lets the other ranks reach three of its
device buffers through CUDA IPC: its per-expert counts, its receive buffer
and its expert-output buffer.  A step is the library's four expert-parallel
calls with a barrier between each two of them:

    route  | dispatch (stores into the owners' receive buffers) |
    experts (grouped GEMMs over the own receive buffer)       | combine
    (reads each pair's output from its owner's buffer)

The barrier is on the device for an NCCL group (a one-element all-reduce on
the current stream: ordered after this rank's kernels and before its next
ones, no host wait) and a stream synchronisation plus a host barrier for
other backends.  The library itself never waits on another rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe as M


def exchange_pointers(local: dict, group=None, opener=None) -> tuple[dict, list]:
    """Rank-ordered device addresses of every rank's exported buffers.

    ``local`` maps a buffer name to (IPC handle, offset, own address).  The
    handles travel with one all_gather_object.  A peer's allocation is opened
    once per distinct handle with ``opener(handle)`` (default: CUDA IPC at
    offset 0) and a buffer's address is that base plus its offset; this
    rank's own buffers are used as they are.  (The caching allocator may put
    two buffers in one allocation: they then share a handle.)  Returns
    {name: [address on rank 0, 1, ...]} and the bases this rank opened, to
    close later."""
    opener = (lambda h: M.ipc_open(h, 0)) if opener is None else opener
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    mine = {name: (h, off) for name, (h, off, _) in local.items()}
    everyone = [None] * world
    dist.all_gather_object(everyone, mine, group=group)
    bases = {}
    addrs = {}
    for name, (_, _, own) in local.items():
        row = []
        for s in range(world):
            if s == rank:
                row.append(int(own))
                continue
            h, off = everyone[s][name]
            if h not in bases:
                bases[h] = int(opener(h))
            row.append(bases[h] + int(off))
        addrs[name] = row
    return addrs, list(bases.values())


class EPGroup:
    """One rank of an expert-parallel MoE layer.

    ``inputs`` holds the layer's tensors (as drawn by workloads.make_inputs);
    the routed expert weights may be the full [E, ...] tensors (this rank
    keeps views of its slice) or already this rank's [E/W, ...] slice.  Every
    rank must use the same T.  Call ``close()`` before the process group is
    destroyed."""

    def __init__(self, inputs: dict, T: int, group=None, align: int = 16, device=None):
        cfg = inputs["cfg"]
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if cfg.E % self.world:
            raise ValueError("the routed experts must split evenly over the ranks")
        self.cfg, self.T, self.align = cfg, int(T), align
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        El = cfg.E // self.world
        to = lambda t: t.to(self.device).contiguous()  # noqa: E731

        def local(w):
            w = to(w)
            if w.shape[0] == cfg.E:
                return w[self.rank * El:(self.rank + 1) * El]
            if w.shape[0] != El:
                raise ValueError(f"expert weights with {w.shape[0]} experts")
            return w

        self.w_gate, self.bias = to(inputs["w_gate"]), to(inputs["bias"])
        self.w1, self.w3, self.w2 = local(inputs["w1"]), local(inputs["w3"]), local(inputs["w2"])
        self.ws1, self.ws3, self.ws2 = to(inputs["ws1"]), to(inputs["ws3"]), to(inputs["ws2"])
        self.dm = M.dims(T, cfg.d, cfg.E, cfg.k, cfg.I, cfg.S, align)
        self.recv_cap = M.ep_recv_capacity(self.dm, self.world)
        self.ws = M.guard_layout(M.alloc_workspace(M.ep_workspace_size(self.dm, self.world),
                                                   self.device), M.ep_layout(self.dm, self.world))
        self.views = M.ep_workspace_views(self.dm, self.world, self.ws)
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.x_recv = torch.empty((self.recv_cap, cfg.d), **bf)
        self.y_recv = torch.empty((self.recv_cap, cfg.d), dtype=torch.float32, device=self.device)
        bufs = {"counts": self.views["counts"], "x_recv": self.x_recv, "y_recv": self.y_recv}
        local_h = {n: (*M.ipc_export(t), t.data_ptr()) for n, t in bufs.items()}
        addrs, self._opened = exchange_pointers(local_h, group)
        as_dev = lambda a: torch.tensor(a, dtype=torch.int64, device=self.device)  # noqa: E731
        self.counts_of = as_dev(addrs["counts"])
        self.x_recv_of = as_dev(addrs["x_recv"])
        self.y_recv_of = as_dev(addrs["y_recv"])
        self._nccl = dist.get_backend(group) == "nccl"
        self._token = torch.zeros(1, device=self.device)

    def barrier(self):
        if self._nccl:
            dist.all_reduce(self._token, group=self.group)
        else:
            torch.cuda.current_stream(self.device).synchronize()
            dist.barrier(group=self.group)

    def __call__(self, x: torch.Tensor, y: torch.Tensor | None = None):
        if y is None:
            y = torch.empty((self.T, self.cfg.d), dtype=torch.bfloat16, device=self.device)
        W = self.world
        M.ep_route(self.dm, W, x, self.w_gate, self.bias, self.ws)
        self.barrier()                      # every rank's counts are written
        M.ep_dispatch(self.dm, W, self.rank, x, self.counts_of, self.x_recv_of, self.ws)
        self.barrier()                      # every receive buffer is complete
        M.ep_experts(self.dm, W, x, self.x_recv, self.w1, self.w3, self.w2, self.ws1, self.ws3,
                     self.ws2, self.y_recv, self.ws)
        self.barrier()                      # every owner's outputs are complete
        M.ep_combine(self.dm, W, self.y_recv_of, y, self.ws)
        return y

    def close(self):
        """Unmap the peers' buffers (after every rank's last step)."""
        torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)      # no peer still reads this rank's buffers
        for base in self._opened:
            M.ipc_close(base, 0)
        self._opened = []
