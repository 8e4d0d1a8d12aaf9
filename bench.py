#!/usr/bin/env python
"""Benchmark of the dots.llm1 MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one moe_forward (router, permutation, grouped SwiGLU GEMMs with the
shared experts, combine) over one batch of T synthetic tokens.  The default
workload is the decode-sized layer (T=128, d=5120, 128 experts top-6 + 2
shared, I=1408), whose throughput is bound by streaming the expert weights
from HBM.  Under torchrun every rank runs its own batch with replicated
weights and no collective on the data path (data-parallel replicas, weak
scaling); the timed region is bracketed by a barrier and synchronisation on
both sides and the time is the max over ranks.

Prints ONE JSON line on rank 0.  `--impl reference` times the fp64 CPU oracle
on host cores on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from fine_grained_moe_fp32_b200.workloads import CONFIGS, make_inputs  # noqa: E402

METRIC = "MoE-layer tokens/s (bf16, d=5120, 128E top-6 + 2 shared) and % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
def forward_kernels(T: int, side: bool = False) -> int:
    """Launches of one moe_forward: router GEMM + top-k, the permutation (one
    index kernel + row copy for a batch of at most 256 tokens, else count,
    scan, scatter + row copy), the two grouped GEMMs, the combine; with
    ``side`` the shared experts' two GEMMs launched on the side stream."""
    return 2 + (2 if T <= 256 else 4) + 2 + 1 + (2 if side else 0)


def dense_kernels(T: int, d: int, I: int, num_sms: int = 148) -> int:
    """Launches of one moe_dense_swiglu: the offsets kernel, the two GEMMs,
    and for each GEMM split over K (the library's rule: at most two waves of
    pair tiles, 15 % or more fewer waves x K chunks) the kernel that sums
    its partials."""
    def splits(base, kit):
        pairs = num_sms // 2
        if base > 2 * pairs or kit < 4:
            return 1
        unsplit = -(-base // pairs) * kit
        best, best_cost = 1, unsplit
        for sp in range(2, min(8, kit // 2) + 1):
            if -(-kit // sp) * (sp - 1) >= kit:
                continue
            cost = -(-(base * sp) // pairs) * -(-kit // sp)
            if cost < best_cost:
                best, best_cost = sp, cost
        return best if best_cost * 100 <= unsplit * 85 else 1
    n = 3
    if T > 24 and d % 256 == 0 and I % 128 == 0:  # CTA-pair GEMMs
        n += splits(-(-T // 256) * (I // 128), d // 128) > 1
        n += splits(-(-T // 256) * (d // 256), I // 128) > 1
    return n
BWD_KERNELS = 11      # combine/router bwd (3), 4 grouped GEMMs (dW1 and dW3 in one), 2 gate GEMMs + split sum, un-permute
BALANCE_KERNELS = 4   # balance partial sums, per-sequence f/P, loss, bias step
# training-side balancing of the fwd+bwd step: sequences of the 8K pretraining
# context (Technical Report, Results: 8K extended to 32K later); the loss
# coefficient and the bias step size are not on the pages (DeepSeek-V3 values)
BALANCE_SEQ = 8192
BALANCE_ALPHA = 1e-4
BALANCE_GAMMA = 1e-3


# ---------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# the kernel, its PTX helpers, and the entry point that decides what one
# launch covers (a change to any of them invalidates a traffic capture)
GEMM_SOURCES = ("fine_grained_moe_fp32_b200/csrc/grouped_gemm.cu",
                "fine_grained_moe_fp32_b200/csrc/ptx_sm100.cuh",
                "fine_grained_moe_fp32_b200/csrc/moe_api.cu")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from a committed ncu summary
    (profiles/<kernel>__<workload>.txt: 'traffic_bytes_per_launch: N' and the
    'kernel_source_hash' of the kernel it was captured on).  None when there
    is no capture or the kernel has changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.txt")
    fields = {}
    try:
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
    except OSError:
        return None
    if fields.get("kernel_source_hash") != kernel_source_hash():
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons of one GPU, sampled in the
    background while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 50):
        self.rows = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, RuntimeError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r for t, r in self.rows if t0 - 0.06 <= t <= t1 + 0.06] or [r for _, r in self.rows]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, T: int, steps: int, ms_max: float) -> float:
    """Tokens per second of the whole job: every rank's tokens over the
    slowest rank's time."""
    return world * T * steps / (ms_max / 1e3)


def shard_seed(seed: int, rank: int) -> int:
    """Each rank draws its own token batch; the weights are replicated."""
    return seed + 7919 * rank


def train_gemm_flops(cfg, T):
    """Algorithmic flops of each grouped-GEMM phase of one fwd+bwd step."""
    d, I, S, k = cfg.d, cfg.I, cfg.S, cfg.k
    rows = T * k
    up = 2 * (rows * 2 * I + T * 2 * S * I) * d      # gate/up shaped
    down = 2 * (rows * I + T * S * I) * d            # down shaped
    return {"gemm_gate_up_swiglu": up, "gemm_down": down, "dgrad_down_swiglu_bwd": down,
            "wgrad_w2": down, "dgrad_up": up, "wgrad_w1_w3": up}


def shared_on_side_stream(cfg, T, train):
    """The inference forward runs the shared experts' GEMMs on the library's
    side stream (beside the router and the permutation), so the gate/up and
    down phases timed on the caller's stream hold the routed experts' GEMMs
    only."""
    return (not train) and cfg.S > 0 and T > 0


def gemm_units(cfg, T, counts, routed_only=False):
    """Algorithmic work of the two grouped GEMMs for one step (padding not
    counted): bytes that must move and flops that must be done; with
    ``routed_only`` the routed experts' launches alone."""
    d, I, S, k = cfg.d, cfg.I, cfg.S, cfg.k
    touched = int((counts > 0).sum())
    rows = T * k
    if routed_only:
        S = 0
    g1_bytes = (touched + S) * 2 * I * d * 2 + (rows + (T if S else 0)) * d * 2 \
        + (rows + T * S) * I * 2
    g2_bytes = (touched + S) * d * I * 2 + (rows + T * S) * I * 2 + rows * d * 4 \
        + (T * d * 4 if S else 0)
    g1_flops = 2 * (rows * 2 * I + T * 2 * S * I) * d
    g2_flops = 2 * (rows * I + T * S * I) * d
    return {"touched_experts": touched, "gemm_gate_up_swiglu": (g1_bytes, g1_flops),
            "gemm_down": (g2_bytes, g2_flops)}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        if n:
            return n
    except Exception:  # pragma: no cover
        pass
    return os.cpu_count() or 1


def oracle_sample(inp, n_tokens, seed=0):
    """Time the fp64 oracle on a seeded sample of the batch's tokens: the
    forward (per-token path), or for a training workload the forward, the
    backward (input gradients, router and all experts; weight gradients not
    kept), the balance statistics and the bias step of the sampled tokens."""
    from oracle import moe_oracle as O
    host = {k: (v.detach().cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(inp["T"], size=min(n_tokens, inp["T"]), replace=False))
    t0 = time.perf_counter()
    if inp["cfg"].grad:
        sub = dict(host)
        idx = torch.as_tensor(toks)
        sub["x"], sub["dy"], sub["T"] = host["x"][idx], host["dy"][idx], len(toks)
        f = O.forward(sub)
        O.backward(sub, sub["dy"], f, experts=[])
        cfg = inp["cfg"]
        O.balance_stats(f["probs"], f["idx"], cfg.E, cfg.k, len(toks), BALANCE_ALPHA)
        O.bias_update(host["bias"], np.bincount(f["idx"].ravel(), minlength=cfg.E),
                      BALANCE_GAMMA, len(toks), cfg.k)
    else:
        O.forward_tokens(host, toks)
    return len(toks), time.perf_counter() - t0


# ---------------------------------------------------------------- arms

def workload(args):
    """The configuration, optionally shrunk for profiler captures: fewer
    experts / tokens with the same per-expert shape, or a narrower expert
    hidden size I (the router's shape T x d x E is then unchanged)."""
    cfg = CONFIGS[args.config]
    if args.experts or args.tokens or args.inter:
        E = args.experts or cfg.E
        T = args.tokens or cfg.T
        I = args.inter or cfg.I
        name = f"{cfg.name}__E{E}_T{T}" + (f"_I{I}" if args.inter else "")
        cfg = dataclasses.replace(cfg, E=E, T=T, I=I, name=name)
    return cfg


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    cfg = workload(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, device=dev)
    host = {k: (v.detach().cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    from oracle import moe_oracle as O
    touched = len(np.unique(O.route(host["x"], host["w_gate"], host["bias"], cfg.k)["idx"]))
    n = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample(host, n, seed=1)
    times = []
    for s in range(args.steps):
        nt, dt = oracle_sample(host, n, seed=100 + s)
        times.append(dt)
    total = sum(times)
    value = nt * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, args.gpus, args.align, touched),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(),
                         "kind": "oracle",
                         "sample": f"{nt} seeded tokens of the T={cfg.T} batch per step, "
                                   "fp64 numpy oracle (per-token path)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}   # B200 spec sheet, dense bf16
EXTRA_CONFIGS = (2, 3, 4)   # measured beside the headline decode line, same K and W


def layer_units(cfg, T, counts, train):
    """Algorithmic work of one whole step of the layer: the bytes it must move
    (every touched routed expert's and the shared experts' weights, the fp32
    gate, tokens in and out) and the tensor-core flops (3 contractions of
    2*d*I per expert row; the backward doubles them)."""
    d, I, S, k, E = cfg.d, cfg.I, cfg.S, cfg.k, cfg.E
    touched = int((counts > 0).sum())
    bytes_ = (touched + S) * 3 * d * I * 2 + E * d * 4 + 2 * T * d * 2
    flops = 2 * 3 * d * I * (T * k + T * S) * (3 if train else 1)
    return bytes_, flops


def config_dict(cfg, world, align, touched):
    c = {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
         "S": cfg.S, "I": cfg.I, "align": align, "router": "fp32",
         "parallelism": f"dp{world} (replicas, no collective)",
         "l2": "inputs larger than L2: the step streams the expert weights "
               f"({(touched + cfg.S) * 3 * cfg.I * cfg.d * 2 / 1e9:.2f} GB)"}
    if cfg.grad:
        c["step"] = ("forward (training, keeps g/u) + backward + sequence-wise balance "
                     f"statistics (seq_len {math.gcd(cfg.T, BALANCE_SEQ)}) + bias step"
                     + (" + weight-gradient all-reduce and summed expert loads (NCCL)"
                        if world > 1 else ""))
        if world > 1:
            c["parallelism"] = f"dp{world} (weight gradients all-reduced)"
    return c


def measure(cfg, args, dev, world, rank, local):
    """Time one workload on this rank's GPU: W warm-up steps, an untimed pass
    with every phase bracketed by events, K timed steps (device-resident
    inputs), K end-to-end steps through the public API with host copies.
    Returns plain numbers only, so every device tensor is freed on return."""
    from fine_grained_moe_fp32_b200 import moe as M
    T = cfg.T
    inp = make_inputs(cfg, device=dev, seed=0, weights=True)
    if world > 1:  # own token batch per rank
        inp["x"] = make_inputs(cfg, device=dev, seed=shard_seed(0, rank), weights=False)["x"]
    layer = M.MoELayer(inp, align=args.align, device=dev)
    x = inp["x"]
    y = torch.empty((T, cfg.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    train = cfg.grad
    if train:
        dy = inp["dy"]
        grads = layer.alloc_grads(T)
        seq_len = math.gcd(T, BALANCE_SEQ)
        f32 = dict(dtype=torch.float32, device=dev)
        bal = {"f": torch.empty((T // seq_len, cfg.E), **f32),
               "P": torch.empty((T // seq_len, cfg.E), **f32), "loss": torch.empty(1, **f32)}
        bias_next = torch.empty_like(layer.bias)

        group = torch.distributed.group.WORLD if world > 1 else None

        def step(xin, yout, evs=None, dyin=None, dxout=None):
            layer.forward_train(xin, yout)
            g = grads if dxout is None else dict(grads, dx=dxout)
            layer.backward(xin, dy if dyin is None else dyin, g)
            if world > 1:   # data parallel: sum the weight gradients of all replicas
                M.allreduce_grads(g, group)
            if evs is not None:
                evs[0].record(stream)
            layer.balance_stats(T, seq_len, BALANCE_ALPHA, out=bal)
            layer.bias_step(T, BALANCE_GAMMA, out=bias_next, group=group)
            if evs is not None:
                evs[1].record(stream)
    else:
        def step(xin, yout, evs=None, dyin=None, dxout=None):
            layer(xin, yout)
    n_events = 13 if train else 6

    for _ in range(args.warmup):
        step(x, y)
    torch.cuda.synchronize(dev)
    st = M.device_status()
    if st != M.MOE_OK:
        raise SystemExit(f"{cfg.name}: device status after warm-up: {M.status_string(st)}")
    views = M.workspace_views(layer.dims(T), layer.train_workspace(T) if train
                              else layer.workspace(T))
    counts = views["counts"].cpu().numpy()

    # ---- per-phase breakdown: an untimed pass with every phase bracketed
    n_phase = min(args.steps, 20)
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
           for _ in range(n_phase)]
    bal_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
              for _ in range(n_phase)] if train else [None] * n_phase
    for s in range(n_phase):
        M.set_phase_events(pev[s])
        step(x, y, bal_ev[s])
    torch.cuda.synchronize(dev)
    M.set_phase_events(None)
    phase_ms = {}
    bracket = {}  # phase -> (event before, event after) in the hook's list
    for i, name in enumerate(M.PHASES):
        bracket[name] = (i, i + 1)
    for i, name in enumerate(M.BWD_PHASES if train else ()):
        bracket[name] = (6 + i, 7 + i)
    for name, (a, b) in bracket.items():
        phase_ms[name] = statistics.mean(pev[s][a].elapsed_time(pev[s][b])
                                         for s in range(n_phase))
    if train:
        phase_ms["balance_stats_bias_step"] = statistics.mean(
            bal_ev[s][0].elapsed_time(bal_ev[s][1]) for s in range(n_phase))
    split = shared_on_side_stream(cfg, T, train)
    units = gemm_units(cfg, T, counts, routed_only=split)
    if train:
        tflops = train_gemm_flops(cfg, T)
        dom = max(tflops, key=lambda n: phase_ms[n])
    else:
        dom = max(("gemm_gate_up_swiglu", "gemm_down"), key=lambda n: phase_ms[n])

    # ---- device-resident timed region: only the dominant kernel's two
    # bounding events are recorded, so the hook costs the step nothing else
    ia, ib = bracket[dom]
    ev = []
    for _ in range(args.steps):
        row = [None] * n_events
        row[ia] = torch.cuda.Event(enable_timing=True)
        row[ib] = torch.cuda.Event(enable_timing=True)
        ev.append(row)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    time.sleep(0.15)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    start.record(stream)
    for s in range(args.steps):
        M.set_phase_events(ev[s])
        step(x, y)
    end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    M.set_phase_events(None)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(t0, t1)
    st = M.device_status()
    if st != M.MOE_OK:
        raise SystemExit(f"{cfg.name}: device status after timing: {M.status_string(st)}")
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world, dev)
    value = whole_job_value(world, T, args.steps, ms)
    dom_ms = statistics.mean(ev[s][ia].elapsed_time(ev[s][ib]) for s in range(args.steps))

    # ---- end to end through the public API: every step copies its inputs
    # from pinned host memory and reads its result back.  The copies run on
    # their own streams with double-buffered device tensors, so step i's
    # copies overlap the neighbouring steps' compute (as a serving loop
    # would); each step still moves all of its bytes inside the timed region.
    h2d_st = torch.cuda.Stream(dev)
    d2h_st = torch.cuda.Stream(dev)
    x_host = x.cpu().pin_memory()
    out_host = [torch.empty((T, cfg.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_buf = [torch.empty_like(x) for _ in range(2)]
    y_buf = [torch.empty_like(y) for _ in range(2)]
    if train:
        dy_host = dy.cpu().pin_memory()
        dy_buf = [torch.empty_like(dy) for _ in range(2)]
        dx_buf = [torch.empty_like(grads["dx"]) for _ in range(2)]
    in_ready = [torch.cuda.Event() for _ in range(2)]   # inputs of buffer b on the device
    computed = [torch.cuda.Event() for _ in range(2)]   # the step using buffer b is done
    out_read = [torch.cuda.Event() for _ in range(2)]   # result of buffer b read back

    def e2e_step(i):
        b = i & 1
        h2d_st.wait_event(computed[b])   # the step that last used buffer b has finished
        with torch.cuda.stream(h2d_st):
            x_buf[b].copy_(x_host, non_blocking=True)
            if train:
                dy_buf[b].copy_(dy_host, non_blocking=True)
        in_ready[b].record(h2d_st)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_read[b])   # its previous result has been read out
        if train:
            step(x_buf[b], y_buf[b], dyin=dy_buf[b], dxout=dx_buf[b])
        else:
            step(x_buf[b], y_buf[b])
        computed[b].record(stream)
        d2h_st.wait_event(computed[b])
        with torch.cuda.stream(d2h_st):
            out_host[b].copy_(dx_buf[b] if train else y_buf[b], non_blocking=True)
        out_read[b].record(d2h_st)

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_st.wait_event(e0)
    d2h_st.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(out_read[0])
    stream.wait_event(out_read[1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_value(world, T, args.steps, e2e_ms)

    # ---- roofline of the dominant kernel (its duration from the timed region)
    peaks, peak_src = load_peaks()
    if train:
        bytes_, flops = 0, tflops[dom]
    else:
        bytes_, flops = units[dom]
    dur_s = dom_ms / 1e3
    hbm_bound = (not train) and T * cfg.k <= 24 * cfg.E
    if hbm_bound:
        achieved = bytes_ / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = flops / dur_s / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak}
    roof["kernel"] = dom + (" (routed experts; the shared experts' GEMMs run on a side stream)"
                            if split else "")
    roof["kernel_ms"] = dom_ms
    roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if hbm_bound else 'bf16_tflops'})"
    roof["traffic"] = load_traffic(dom, cfg.name)
    roof["algorithmic_per_launch"] = bytes_ if hbm_bound else flops
    # ---- the whole step against the same two ceilings (measured and nominal)
    lbytes, lflops = layer_units(cfg, T, counts, train)
    step_s = ms / args.steps / 1e3   # every rank does one step's work in this time
    key = "hbm_gbs" if hbm_bound else "bf16_tflops"
    lach = (lbytes / step_s / 1e9) if hbm_bound else (lflops / step_s / 1e12)
    roof["layer"] = {"bound": "hbm" if hbm_bound else "tensor", "achieved": lach,
                     "unit": "GB/s" if hbm_bound else "TFLOP/s",
                     "algorithmic_per_step": lbytes if hbm_bound else lflops,
                     "frac_measured": lach / peaks[key],
                     "frac_nominal": lach / NOMINAL_PEAKS[key],
                     "nominal_peak": NOMINAL_PEAKS[key]}
    res = {"value": value, "ms_per_step": ms / args.steps, "roofline": roof,
           "phases_ms": {k: round(v, 4) for k, v in phase_ms.items()}, "clocks": clocks,
           "e2e": {"value": e2e_value, "unit": "tokens/s",
                   "h2d_bytes_per_step": T * cfg.d * 2 * (2 if train else 1),
                   "d2h_bytes_per_step": T * cfg.d * 2},
           "gpu_launches": (forward_kernels(T, shared_on_side_stream(cfg, T, train))
                            + (BWD_KERNELS + BALANCE_KERNELS if train else 0)) * args.steps,
           "config": config_dict(cfg, world, args.align, gemm_units(cfg, T, counts)["touched_experts"]),
           "n_phase": n_phase}
    if train:
        res["train_tflop_per_step"] = sum(train_gemm_flops(cfg, T).values()) / 1e12
    return res


def cpu_baseline_full(cfg):
    """The fp64 oracle on a whole batch of the workload (every token, the
    oracle's own permutation path), timed on this host's cores."""
    from oracle import moe_oracle as O
    inp = make_inputs(cfg, device="cpu")
    host = {k: (v.detach() if torch.is_tensor(v) else v) for k, v in inp.items()}
    t0 = time.perf_counter()
    O.forward(host)
    return cfg.T, time.perf_counter() - t0


def run_ours(args):
    world, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    cfg = workload(args)
    r = measure(cfg, args, dev, world, rank, local)
    line = {
        "metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights; random-init layer)",
        "config": r["config"],
        "roofline": r["roofline"],
        "phases_ms": r["phases_ms"],
        "phases_ms_source": f"untimed pass of {r['n_phase']} steps with every phase bracketed "
                            "by events; the timed region brackets only the roofline kernel",
        "clocks": r["clocks"], "e2e": r["e2e"], "gpu_launches": r["gpu_launches"],
    }
    if "train_tflop_per_step" in r:
        line["train_tflop_per_step"] = r["train_tflop_per_step"]
    shrunk = bool(args.experts or args.tokens or args.inter)
    if world == 1 and args.config == 1 and not shrunk and not args.no_extra_configs:
        # the prefill and training workloads, each timed like the headline
        extra = {}
        for c in EXTRA_CONFIGS:
            torch.cuda.empty_cache()
            rc = measure(CONFIGS[c], args, dev, world, rank, local)
            rc.pop("n_phase")
            extra[CONFIGS[c].name] = {"tokens_per_s": rc.pop("value"), **rc}
            line["gpu_launches"] += rc["gpu_launches"]
        line["configs"] = extra
        line["configs_note"] = ("the prefill and fwd+bwd workloads, each timed like the "
                                f"headline ({args.warmup} warm-up, {args.steps} timed steps, "
                                "CUDA events, clocks sampled); gpu_launches above counts "
                                "their launches too")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if cfg.T <= 256 and not cfg.grad:
            n, dt = cpu_baseline_full(cfg)
            n0, dt0 = cpu_baseline_full(CONFIGS[0])
            line["cpu_baseline"] = {
                "value": n / dt, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                "sample": f"the whole T={n} batch of {cfg.name} through the fp64 numpy oracle "
                          f"(route, permute, 128 experts, shared, combine): {dt:.1f} s",
                "tiny_full": {"workload": CONFIGS[0].name, "value": n0 / dt0,
                              "unit": "tokens/s", "seconds": dt0}}
        else:
            inp = make_inputs(cfg, device=dev)
            n, dt = oracle_sample(inp, args.cpu_tokens)
            line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": cpu_threads(),
                                    "kind": "oracle",
                                    "sample": f"{n} seeded tokens of the T={cfg.T} batch, fp64 "
                                              f"numpy oracle ({'forward + backward' if cfg.grad else 'forward'}"
                                              f"), {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


DENSE_METRIC = "dense SwiGLU FFN tokens/s (bf16, d=5120, I=11264) and % of roofline"


def run_dense(args):
    """The first layer's dense SwiGLU FFN (moe_dense_swiglu) on the workload's
    token count: device-resident timing, roofline, pipelined end-to-end copies."""
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200.workloads import DENSE_I, make_dense_inputs
    world, rank, local = dist_setup()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    T = args.tokens or CONFIGS[args.config].T
    d = CONFIGS[args.config].d
    I = args.inter or DENSE_I
    inp = make_dense_inputs(T, d, I, device=dev, seed=shard_seed(0, rank) if world > 1 else 0)
    dm = M.dense_dims(T, d, I)
    ws = M.alloc_workspace(M.dense_workspace_size(dm), dev)
    x, w1, w3, w2 = inp["x"], inp["w1"], inp["w3"], inp["w2"]
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(xin, yout):
        M.dense_swiglu(dm, xin, w1, w3, w2, yout, ws)

    for _ in range(args.warmup):
        step(x, y)
    torch.cuda.synchronize(dev)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after warm-up")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    time.sleep(0.15)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    start.record(stream)
    for _ in range(args.steps):
        step(x, y)
    end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(t0, t1)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after timing")
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    value = whole_job_value(world, T, args.steps, ms)

    # end to end: x in from pinned memory, y back, on copy streams (double-buffered)
    h2d_st, d2h_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_host = x.cpu().pin_memory()
    y_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xb = [torch.empty_like(x) for _ in range(2)]
    yb = [torch.empty_like(y) for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i & 1
        h2d_st.wait_event(done[b])
        with torch.cuda.stream(h2d_st):
            xb[b].copy_(x_host, non_blocking=True)
        ready[b].record(h2d_st)
        stream.wait_event(ready[b])
        stream.wait_event(read[b])
        step(xb[b], yb[b])
        done[b].record(stream)
        d2h_st.wait_event(done[b])
        with torch.cuda.stream(d2h_st):
            y_host[b].copy_(yb[b], non_blocking=True)
        read[b].record(d2h_st)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_st.wait_event(e0)
    d2h_st.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(read[0])
    stream.wait_event(read[1])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = whole_job_value(world, T, args.steps, max_over_ranks(e0.elapsed_time(e1), world, dev))

    peaks, peak_src = load_peaks()
    dur_s = ms / args.steps / 1e3
    flops = 2.0 * T * d * I * 3
    bytes_ = 3.0 * I * d * 2 + 2.0 * T * d * 2 + T * I * 2 * 2
    # bound by whichever floor is longer: streaming the weights or the flops
    hbm_bound = bytes_ / (peaks["hbm_gbs"] * 1e9) >= flops / (peaks["bf16_tflops"] * 1e12)
    if hbm_bound:
        ach = bytes_ / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"]}
    else:
        ach = flops / dur_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"]}
    roof.update({"kernel": "dense step (gate/up + down grouped GEMMs as one group)",
                 "peak_source": peak_src, "traffic": None,
                 "algorithmic_per_launch": bytes_ if hbm_bound else flops})
    if rank == 0:
        print(json.dumps({
            "metric": DENSE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights)",
            "config": {"workload": f"dense_swiglu_T{T}_d{d}_I{I}", "T": T, "d": d, "I": I,
                       "parallelism": f"dp{world} (replicas, no collective)"},
            "roofline": roof, "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * d * 2,
                    "d2h_bytes_per_step": T * d * 2},
            "gpu_launches": dense_kernels(T, d, I) * args.steps}), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def ep_kernels(T: int) -> int:
    """Launches of one emulated rank's expert-parallel step: router GEMM +
    top-k, the permutation index (one kernel for at most 256 tokens, else
    count, scan, scatter), the layout plan, the dispatch, the two grouped
    GEMMs, the combine."""
    return 2 + (1 if T <= 256 else 3) + 2 + 2 + 1


def run_ep(args):
    """Expert parallelism over --ep W ranks emulated on one GPU: each step
    runs every rank's route, dispatch, expert GEMMs and combine (the calls a
    rank of a multi-GPU job makes) on this device, stream order standing in
    for the barriers.  Every rank routes its own batch of the workload's T
    tokens; the value counts all W*T tokens."""
    from fine_grained_moe_fp32_b200 import moe as M
    world, rank, local = dist_setup()
    if world > 1:
        raise SystemExit("--ep emulates the ranks on one GPU; run it without torchrun")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = workload(args)
    W, T = args.ep, cfg.T
    inp = make_inputs(cfg, device=dev)
    xs = [inp["x"]] + [make_inputs(cfg, device=dev, seed=1000 + r, weights=False)["x"]
                       for r in range(1, W)]
    ep = M.EPRanks(inp, W, T, args.align, dev)
    ys = [torch.empty((T, cfg.d), dtype=torch.bfloat16, device=dev) for _ in range(W)]
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        ep(xs, ys)
    torch.cuda.synchronize(dev)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after warm-up")

    # phase pass (untimed): events between the four phases of every step
    names = ("route", "dispatch", "experts", "combine")
    n_phase = min(args.steps, 20)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_phase)]
    for i in range(n_phase):
        ev[i][0].record(stream)
        ep.route(xs)
        ev[i][1].record(stream)
        ep.dispatch(xs)
        ev[i][2].record(stream)
        ep.experts_step(xs)
        ev[i][3].record(stream)
        ep.combine(ys)
        ev[i][4].record(stream)
    torch.cuda.synchronize(dev)
    phase_ms = {n: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n_phase))
                for j, n in enumerate(names)}

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    time.sleep(0.15)
    torch.cuda.synchronize(dev)
    t0 = time.time()
    start.record(stream)
    for _ in range(args.steps):
        ep(xs, ys)
    end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    clocks = sampler.stop(t0, t1)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after timing")
    ms = start.elapsed_time(end)
    value = W * T * args.steps / (ms / 1e3)

    # end to end through the same calls: every rank's x in from pinned host
    # memory and its y back, inside the timed region
    x_host = [x.cpu().pin_memory() for x in xs]
    y_host = [torch.empty((T, cfg.d), dtype=torch.bfloat16).pin_memory() for _ in range(W)]
    xb = [torch.empty_like(x) for x in xs]
    for _ in range(args.warmup):
        for r in range(W):
            xb[r].copy_(x_host[r], non_blocking=True)
        ep(xb, ys)
        for r in range(W):
            y_host[r].copy_(ys[r], non_blocking=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        for r in range(W):
            xb[r].copy_(x_host[r], non_blocking=True)
        ep(xb, ys)
        for r in range(W):
            y_host[r].copy_(ys[r], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = W * T * args.steps / (e0.elapsed_time(e1) / 1e3)

    # algorithmic work per phase, from the routing of the last step
    d, I, S, k = cfg.d, cfg.I, cfg.S, cfg.k
    El = cfg.E // W
    recv = [v["recv_counts"].cpu().numpy().astype(np.int64) for v in ep.views]
    pad = [int(v["recv_offsets"][-1]) - int(c.sum()) for v, c in zip(ep.views, recv)]
    exp_bytes = exp_flops = 0
    for c in recv:
        rows, touched = int(c.sum()), int((c > 0).sum())
        exp_bytes += ((touched + S) * 3 * I * d * 2 + (rows + T) * d * 2
                      + 2 * (rows + T * S) * I * 2 + rows * d * 2 + T * d * 4)
        exp_flops += 2 * (rows * 3 * I + T * 3 * S * I) * d
    disp_bytes = W * T * d * 2 + W * T * k * d * 2 + sum(pad) * d * 2
    comb_bytes = W * (T * k * d * 2 + T * d * (4 if S else 0) + T * d * 2)
    peaks, peak_src = load_peaks()
    # bound by whichever floor is longer: streaming the bytes or the flops
    hbm_bound = exp_bytes / (peaks["hbm_gbs"] * 1e9) >= exp_flops / (peaks["bf16_tflops"] * 1e12)
    dur_s = phase_ms["experts"] / 1e3
    if hbm_bound:
        ach = exp_bytes / dur_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"]}
    else:
        ach = exp_flops / dur_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"]}
    roof.update({"kernel": f"expert GEMMs of all {W} ranks (2 grouped GEMMs per rank)",
                 "peak_source": f"{peak_src} ({'hbm_gbs' if hbm_bound else 'bf16_tflops'})",
                 "traffic": None, "algorithmic_per_launch": exp_bytes if hbm_bound else exp_flops,
                 "duration_source": "phase pass (events around the expert GEMMs of all ranks)"})
    phases = {n: {"ms": round(phase_ms[n], 4)} for n in names}
    phases["dispatch"]["GB/s"] = round(disp_bytes / (phase_ms["dispatch"] / 1e3) / 1e9, 1)
    phases["combine"]["GB/s"] = round(comb_bytes / (phase_ms["combine"] / 1e3) / 1e9, 1)
    line = {
        "metric": METRIC + f"; expert parallel over {W} ranks emulated on one GPU",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) tokens per rank, N(0,0.02) weights; random-init layer)",
        "config": {"workload": f"ep{W}_emulated_{cfg.name}", "ranks": W, "T_per_rank": T,
                   "d": d, "E": cfg.E, "experts_per_rank": El, "k": k, "S": S, "I": I,
                   "align": args.align, "recv_capacity_rows": ep.recv_cap,
                   "parallelism": f"ep{W} emulated (one process, one GPU)",
                   "l2": "inputs larger than L2: the step streams the expert weights"},
        "roofline": roof, "phases": phases, "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": W * T * d * 2,
                "d2h_bytes_per_step": W * T * d * 2},
        "gpu_launches": W * ep_kernels(T) * args.steps,
    }
    if args.micro > 1:
        line["overlap"] = ep_overlap_measurement(args, inp, xs, W, T, dev, stream, phase_ms)
    if not args.no_cpu_baseline:
        n, secs = oracle_sample(inp, args.cpu_tokens)
        line["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s", "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": f"{n} seeded tokens of rank 0's batch, fp64 numpy "
                                          f"oracle (forward; the exchange does not change it), "
                                          f"{secs:.1f} s"}
    print(json.dumps(line), flush=True)
    return 0


def ep_overlap_measurement(args, inp, xs, W, T, dev, stream, phase_ms):
    """The expert-parallel step with every rank's batch split into
    --micro microbatches, each chain (route, dispatch, experts, combine) on
    its own stream: timed against the same calls issued microbatch after
    microbatch, with a per-microbatch phase timeline of one untimed step."""
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200.overlap import EPOverlap
    ov = EPOverlap(inp, W, T, args.micro, args.align, dev)
    ys = [torch.empty((T, inp["cfg"].d), dtype=torch.bfloat16, device=dev) for _ in range(W)]
    for _ in range(args.warmup):
        ov(xs, ys)
        ov.serial(xs, ys)
    torch.cuda.synchronize(dev)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.steps):
            fn(xs, ys)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    ovl_ms = timed(ov)
    ser_ms = timed(ov.serial)
    # timeline of one overlapped step: every microbatch's phase boundaries
    t0 = torch.cuda.Event(enable_timing=True)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in ov.sizes]
    t0.record(stream)
    ov(xs, ys, events=evs)
    torch.cuda.synchronize(dev)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after the overlapped steps")
    names = ("route", "dispatch", "experts", "combine")
    timeline = [{n: [round(t0.elapsed_time(e[i]), 4), round(t0.elapsed_time(e[i + 1]), 4)]
                 for i, n in enumerate(names)} for e in evs]
    # phase sum of the microbatched work: each microbatch's own phases, timed
    # one after the other (untimed pass, events between phases)
    sum_micro = 0.0
    for i, ep in enumerate(ov.parts):
        xi = ov._slices(xs, i)
        yi = ov._slices(ys, i)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        e[0].record(stream)
        ep.route(xi)
        e[1].record(stream)
        ep.dispatch(xi)
        e[2].record(stream)
        ep.experts_step(xi)
        e[3].record(stream)
        ep.combine(yi)
        e[4].record(stream)
        torch.cuda.synchronize(dev)
        sum_micro += e[0].elapsed_time(e[4])
    return {"microbatches": ov.sizes, "overlapped_ms_per_step": ovl_ms,
            "serial_ms_per_step": ser_ms, "sum_of_microbatch_phases_ms": sum_micro,
            "sum_of_unsplit_phases_ms": sum(phase_ms.values()),
            "hidden_fraction_vs_serial": 1.0 - ovl_ms / ser_ms,
            "timeline_ms": timeline,
            "note": "each microbatch's route -> dispatch -> experts -> combine on its own "
                    "stream; serial = the same calls one microbatch after the other"}


def run_paired(args):
    """One pipeline stage executing the overlapped interleaved-1F1B step
    list (one warm-up forward, then a forward of microbatch m+1 and the
    backward of microbatch m together on two streams, then the last
    backward) at the workload's microbatch size, timed against the same
    passes run one at a time."""
    from fine_grained_moe_fp32_b200 import moe as M
    from fine_grained_moe_fp32_b200.overlap import PipelineStage
    from fine_grained_moe_fp32_b200.pipeline_schedule import interleaved_1f1b
    world, rank, local = dist_setup()
    if world > 1:
        raise SystemExit("--paired runs one pipeline stage on one GPU; run it without torchrun")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = workload(args)
    if not cfg.grad:
        cfg = dataclasses.replace(CONFIGS[4], T=cfg.T, name=CONFIGS[4].name)
    T, Mn = cfg.T, max(2, args.micro)
    inp = make_inputs(cfg, device=dev)
    layer = M.MoELayer(inp, align=args.align, device=dev)
    xs = [inp["x"]] + [make_inputs(cfg, device=dev, seed=1000 + m, weights=False)["x"]
                       for m in range(1, Mn)]
    dys = [inp["dy"]] + [make_inputs(cfg, device=dev, seed=2000 + m, weights=False)["dy"]
                         for m in range(1, Mn)]
    steps = interleaved_1f1b(1, 1, Mn, overlap=True)[0]
    stage = PipelineStage([layer], T, grad_dtype=torch.bfloat16)
    # one gradient buffer set: the backwards run one after the other on their stream
    g = layer.alloc_grads(T)
    grads = {(m, 0): g for m in range(Mn)}
    ys = {(m, 0): torch.empty((T, cfg.d), dtype=torch.bfloat16, device=dev) for m in range(Mn)}
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        stage.run(steps, xs, dys, grads, ys)
        stage.sequential(steps, xs, dys, grads, ys)
    torch.cuda.synchronize(dev)

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(args.steps):
            fn(steps, xs, dys, grads, ys)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    sampler = ClockSampler(local)
    time.sleep(0.15)
    t0 = time.time()
    ovl = timed(stage.run)
    t1 = time.time()
    clocks = sampler.stop(t0, t1)
    seq = timed(stage.sequential)
    if M.device_status() != M.MOE_OK:
        raise SystemExit("device status after the paired steps")
    flops = sum(train_gemm_flops(cfg, T).values()) * Mn
    peaks, peak_src = load_peaks()
    ach = flops / (ovl / 1e3) / 1e12
    line = {
        "metric": "MoE-layer fwd+bwd tokens/s through one pipeline stage running the overlapped "
                  "interleaved-1F1B steps (bf16, d=5120, 128E top-6 + 2 shared)",
        "value": Mn * T / (ovl / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ovl, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) tokens and upstream gradients, N(0,0.02) weights)",
        "config": {"workload": f"paired_1f1b_{cfg.name}_x{Mn}", "T_per_microbatch": T,
                   "microbatches": Mn, "d": cfg.d, "E": cfg.E, "k": cfg.k, "S": cfg.S,
                   "I": cfg.I, "schedule": [[f"{k}{m}" for k, m, _ in st] for st in steps],
                   "parallelism": "one pipeline stage (P=1, V=1) on one GPU"},
        "roofline": {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                     "kernel": "whole stage (all GEMM phases of every pass)",
                     "peak_source": f"{peak_src} (bf16_tflops)", "traffic": None,
                     "algorithmic_per_launch": flops},
        "sequential_ms_per_step": seq, "overlapped_ms_per_step": ovl,
        "hidden_fraction": 1.0 - ovl / seq, "clocks": clocks,
        "e2e": None,
        "gpu_launches": Mn * (forward_kernels(T) + BWD_KERNELS) * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1, choices=sorted(CONFIGS))
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--align", type=int, default=16)
    ap.add_argument("--cpu-tokens", type=int, default=32)
    ap.add_argument("--ref-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="time only --config (the default run adds the prefill and fwd+bwd "
                         "workloads to the headline decode line)")
    ap.add_argument("--experts", type=int, default=0, help="shrink E (profiling cases)")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling cases)")
    ap.add_argument("--inter", type=int, default=0, help="override I (profiling cases)")
    ap.add_argument("--ep", type=int, default=0,
                    help="expert parallelism over this many ranks emulated on one GPU")
    ap.add_argument("--dense", action="store_true",
                    help="time the first layer's dense SwiGLU FFN instead of the MoE layer")
    ap.add_argument("--micro", type=int, default=0,
                    help="--ep: also time the step with every rank's batch split into this many "
                         "microbatches on their own streams; --paired: microbatches (default 4)")
    ap.add_argument("--paired", action="store_true",
                    help="one pipeline stage running the overlapped interleaved-1F1B steps "
                         "(training workload, forward and backward of two microbatches together)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.dense:
        return run_dense(args)
    if args.ep:
        return run_ep(args)
    if args.paired:
        if args.micro == 0:
            args.micro = 4
        if args.config == 1:
            args.config = 4
        return run_paired(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
