#!/usr/bin/env python
"""Benchmark of the MGLU forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--tokens T]
    python bench.py --impl reference ...     # the float64 CPU oracle, same workload

A step is one pass of the hot path over one batch: for the decode and prefill
workloads one ``mglu_forward`` call (mask-bit unpacking, the n_m + 1 products
and the fused act-sum epilogue); for the FFN-block workload the up-projection
plus the down-projection.  Mask packing happens once at weight-load time and
is outside the timed region.

The headline workload is the n_m = 8 decode layer (d = 4096, h = 14336, one
token).  With no --workload given, the run then times the other workloads of
the suite the same way and adds them to the same JSON line as sub-records
(``workloads``): the routed n_m = 8 decode step, the n_m = 4 decode layer,
the 4096-token prefill with Swish, with GELU and with the dense gate, and the
FFN block at 1 and 2048 tokens; then the training path's backward on the
prefill layer (``training_backward``).  One JSON line is printed by rank 0.
``gpu_launches`` counts this library's kernel launches per step with the
library's own counter (``mglu_kernel_launches``).

Inputs are seeded synthetic tensors with the workload's shapes.  To keep every
timed launch reading HBM, each step uses the next of R device copies of
(W, packed masks[, W_down]) with R * working set > 4 x L2.  Multi-GPU runs are
independent replicas (each rank its own batch, no collective on the data
path); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import gc
import hashlib
import io
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

METRIC = "MGLU fwd HBM GB/s & tok/s (decode), TFLOP/s (prefill) vs B200 roofline"
DEFAULT_WORKLOAD = "decode_d4096_h14336_nm8"
# the rest of the default run: (workload, tokens, act)
SUITE = [
    ("decode_d4096_h14336_nm8", 1, "swish", 2),  # each token routed to 2 of its 8 masks
    ("decode_d2048_h8192_nm4", 1, "swish"),
    ("prefill_T4096_d2048_h8192_nm4", 4096, "swish"),
    ("prefill_T4096_d2048_h8192_nm4", 4096, "gelu"),
    ("prefill_T4096_d2048_h8192_nm4", 4096, "swish+dense_gate"),  # the dense-gate ablation
    ("ffn_d4096_h14336_nm8", 1, "swish"),
    ("ffn_d4096_h14336_nm8", 2048, "swish"),
]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_POLICY = ("inputs larger than L2: each step reads the next of R rotating device copies of the weights "
             "and packed masks, R x working set > 4 x L2")


# ---------------------------------------------------------------------- setup
def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mglu", "reference"], default="mglu")
    ap.add_argument("--workload", default=None,
                    help=f"time only this workload (default: {DEFAULT_WORKLOAD} plus the suite)")
    ap.add_argument("--tokens", type=int, default=None, help="token count for the sweep workloads")
    ap.add_argument("--act", default="swish", choices=["swish", "gelu", "relu"])
    ap.add_argument("--p", type=float, default=0.5, help="mask density (FFN-block workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparisons", action="store_true",
                    help="skip the torch.matmul baselines (dense SwiGLU, naive MGLU) timed after the run")
    ap.add_argument("--no-suite", action="store_true", help="time the headline workload only")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the training backward on the prefill layer and print its record")
    ap.add_argument("--tstar-sweep", action="store_true",
                    help="also time the FFN block for T in 8..64 with the decode kernel allowed up to 16 tokens "
                         "and with every T on the tensor-core kernel")
    ap.add_argument("--probe-seconds", type=float, default=1.0,
                    help="untimed run of the same step before timing, to settle and sample clocks")
    args = ap.parse_args(argv)
    args.suite = args.workload is None and not args.no_suite
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD
    return args


def workload_shape(name, tokens=None, act="swish", p=0.5, route_k=None):
    from masked_glu_b200 import inputs
    if name not in inputs.WORKLOADS:
        raise SystemExit(f"unknown workload {name}; choose from {list(inputs.WORKLOADS)}")
    w = dict(inputs.WORKLOADS[name])
    if tokens is not None:
        w["T"] = tokens
    w["kind"] = ("ffn" if name.startswith("ffn") else
                 "prefill" if name.startswith("prefill") else
                 "tiny" if name.startswith("tiny") else "decode")
    w["seed"] = inputs.WORKLOAD_SEEDS[name] + (w["T"] if tokens is not None else 0)
    w["name"], w["act"], w["p"] = name, act, p
    w["route_k"] = route_k
    return w


def config_of(w, world):
    """The workload's description, identical in the GPU arm and the
    reference arm."""
    c = {"workload": w["name"], "T": w["T"], "d": w["d"], "h": w["h"], "n_m": w["n_m"], "act": w["act"],
         "p": w["p"] if w["kind"] == "ffn" else 0.5, "l2": L2_POLICY,
         "parallelism": "replicas" if world > 1 else "single"}
    if w.get("route_k") is not None:
        c["route"] = f"top-{w['route_k']} of {w['n_m']} masks per token (hard weights), router in the step"
    return c


def algorithmic(w):
    """Roofline work of one step (and of its dominant kernel, the up-projection)."""
    T, d, h, nm = w["T"], w["d"], w["h"], w["n_m"]
    esz = 4 if w["dtype"] == "f32" else 2
    up_bytes = esz * d * h + nm * d * h // 8 + esz * T * d + esz * T * h
    up_flops = 2 * T * d * h * (nm + 1)
    down_bytes = esz * h * d + esz * T * h + esz * T * d
    down_flops = 2 * T * h * d
    return up_bytes, up_flops, down_bytes, down_flops


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    """Hash of the CUDA sources with comments and blank space removed, so a
    recorded ncu capture stays valid across comment edits but not across any
    change to the code."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "masked_glu_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name)) as f:
                text = f.read()
            text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
            text = re.sub(r"//[^\n]*", " ", text)
            h.update(name.encode() + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload, T):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    capture, if the kernel sources have not changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(f"{workload}:T{T}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------- distributed
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float, device=None) -> float:
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 100 ms while running (read-only queries)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.text = ""
        self.sel = self._selector(device_index)

    @staticmethod
    def _selector(i):
        try:
            import torch
            p = torch.cuda.get_device_properties(i)
            return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            return None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.sel:
            cmd[1:1] = ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.buf = []
        if self.proc:
            self.thread = threading.Thread(target=lambda: self.buf.extend(self.proc.stdout), daemon=True)
            self.thread.start()

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        rows = [r for r in csv.reader(io.StringIO("".join(self.buf))) if len(r) >= 10]
        load = [r for r in rows if _num(r[4]) and _num(r[4]) > 0] or rows
        sm = [_num(r[1]) for r in load if _num(r[1])]
        mx = [_num(r[2]) for r in rows if _num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in load for k in range(4) if r[6 + k].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(load),
                "power_w_max": max((_num(r[3]) or 0) for r in load) if load else None}


def _num(s):
    try:
        return float(s)
    except Exception:
        return None


# ---------------------------------------------------------------------- oracle timing
def time_oracle(w, budget_s=10.0, max_tokens=None, single_s=3.0):
    """Time the float64 oracle on a bounded sample of the workload: whole
    tokens (every output column of a token), as many as fit in ~budget_s on
    all the oracle's OpenMP threads, then a shorter sample (~single_s) on one
    thread."""
    import numpy as np
    import oracle
    from masked_glu_b200 import inputs

    T = w["T"]
    rng = np.random.Generator(np.random.PCG64(w["seed"]))
    d, h, nm = w["d"], w["h"], w["n_m"]
    W = inputs.normal(rng, (h, d), 0.02, w["dtype"]).values
    masks = inputs.bernoulli_masks(rng, nm, h, d, w.get("p", 0.5))
    x = inputs.normal(rng, (1, d), 1.0, w["dtype"]).values
    pk = oracle.pack_masks(masks)
    Wd = inputs.normal(rng, (d, h), 0.02, w["dtype"]).values if w["kind"] == "ffn" else None
    act = {"swish": 0, "gelu": 1, "relu": 2}[w.get("act", "swish")]

    def one_token():
        out, _ = oracle.forward(x, W, pk, nm, act)
        if Wd is not None:
            oracle.down(out, Wd)

    t0 = time.perf_counter()
    one_token()
    t1 = time.perf_counter() - t0
    n = max(1, int(budget_s / max(t1, 1e-6)))
    if max_tokens:
        n = min(n, max_tokens)
    t0 = time.perf_counter()
    for _ in range(n):
        one_token()
    dt = time.perf_counter() - t0
    cores = oracle.max_threads()
    res = {"value": n / dt, "unit": "tok/s", "cores": cores, "kind": "oracle",
           "sample": f"{n} one-token forwards (all {h} output columns each) of {w['name']} "
                     f"(d={d}, n_m={nm}), float64, OpenMP over columns, {dt:.1f} s wall"}
    if single_s > 0:
        oracle.set_threads(1)
        try:
            n1 = max(1, min(int(single_s / max(t1 * cores, 1e-6)), n))
            t0 = time.perf_counter()
            for _ in range(n1):
                one_token()
            res["single_thread_value"] = n1 / (time.perf_counter() - t0)
            res["single_thread_sample"] = f"{n1} one-token forwards, same columns, 1 thread"
        finally:
            oracle.set_threads(cores)
    return res, one_token


def run_reference(args, dist):
    """The float64 oracle as it stands, on the host cores (rank 0 only), on
    the headline workload: each step is one token's forward (every output
    column), a bounded sample of the workload."""
    w = workload_shape(args.workload, args.tokens, args.act, args.p)
    if dist.rank != 0:
        return
    _, one = time_oracle(w, budget_s=0.5, max_tokens=1, single_s=0)
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    tok_s = args.steps / dt
    import oracle
    cores = oracle.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": tok_s, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": f"one token (all {w['h']} columns) of {w['name']} per step; the config's l2 "
                                   f"policy describes the GPU arm"},
        "e2e": {"value": tok_s, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU run
def time_comparisons(T, d, h, nm, act, dev, l2, reps=50, rounds=3):
    """Library baselines on the same box and shapes, for context only (not the
    product path, not counted in gpu_launches): a dense SwiGLU with two bf16
    d x h projections through torch.matmul (cuBLAS), and a naive PyTorch MGLU
    that materialises every masked weight M_i * W in bf16 before multiplying.
    Weights rotate over copies larger than L2; times are per call, the median
    of `rounds` runs of reps x R calls."""
    import torch
    F = torch.nn.functional
    fn_act = F.gelu if act == "gelu" else F.relu if act == "relu" else F.silu
    x = torch.randn(T, d, device=dev).to(torch.bfloat16)

    def timed(fn, R, n):
        for i in range(2 * R):
            fn(i % R)
        torch.cuda.synchronize(dev)
        res = []
        for _ in range(rounds):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(n * R):
                fn(i % R)
            e1.record()
            e1.synchronize()
            res.append(e0.elapsed_time(e1) * 1000.0 / (n * R))
        return statistics.median(res), res

    res = {}
    R = max(2, math.ceil(4 * l2 / (2 * h * d * 2)))
    Wg = [(torch.randn(h, d, device=dev) * 0.02).to(torch.bfloat16) for _ in range(R)]
    Wv = [(torch.randn(h, d, device=dev) * 0.02).to(torch.bfloat16) for _ in range(R)]
    res["dense_swiglu_us"], res["dense_swiglu_rounds_us"] = timed(
        lambda i: fn_act(x @ Wg[i].t()) * (x @ Wv[i].t()), R, reps)
    del Wg, Wv
    R = max(2, math.ceil(4 * l2 / (h * d * 2 * (1 + nm))))
    W = [(torch.randn(h, d, device=dev) * 0.02).to(torch.bfloat16) for _ in range(R)]
    M = [(torch.rand(nm, h, d, device=dev) < 0.5).to(torch.bfloat16) for _ in range(R)]

    def naive(i):
        D = x @ W[i].t()
        out = torch.zeros_like(D)
        for k in range(nm):
            g = x @ (W[i] * M[i][k]).t()
            out = out + fn_act(g) * (D - g)
        return out

    res["naive_torch_mglu_us"], res["naive_torch_mglu_rounds_us"] = timed(naive, R, max(3, reps // 10))
    del W, M
    torch.cuda.empty_cache()
    res["note"] = ("torch.matmul (cuBLAS) baselines on the same shapes: dense SwiGLU = two bf16 d x h "
                   "projections; naive MGLU materialises each M_i * W in bf16; median of "
                   f"{rounds} rounds")
    return res


def measure(args, dist, w, dev, *, sample_clocks):
    """Time one workload: K steps replayed as one CUDA graph (device time,
    max over ranks), per-kernel times from a second replay with event nodes,
    and the end-to-end rate through the host-buffer entry point."""
    import numpy as np
    import torch

    from masked_glu_b200 import inputs, mglu

    T, d, h, nm = w["T"], w["d"], w["h"], w["n_m"]
    kind = w["kind"]
    case = inputs.make_case(T, d, h, nm, seed=w["seed"] + 7919 * dist.rank, p=w["p"], dtype=w["dtype"],
                            with_down=(kind == "ffn"))
    tdt = torch.float32 if w["dtype"] == "f32" else torch.bfloat16

    def up(t):
        if t.dtype == "bf16":
            return torch.from_numpy(t.storage.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(t.storage).to(dev)

    x = up(case.x)
    W0 = up(case.W)
    pk0 = mglu.pack_masks(torch.from_numpy(case.masks).to(dev))
    Wd0 = up(case.W_down) if kind == "ffn" else None
    del case
    gc.collect()
    up_bytes, up_flops, down_bytes, down_flops = algorithmic(w)
    working = up_bytes + (down_bytes if kind == "ffn" else 0)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(1, min(16, math.ceil(4 * l2 / max(1, working - 2 * T * (d + h)))))
    free = torch.cuda.mem_get_info(dev)[0]
    while R > 1 and R * working > 0.5 * free:
        R -= 1
    Ws = [W0] + [W0.clone() for _ in range(R - 1)]
    pks = [pk0] + [pk0.clone() for _ in range(R - 1)]
    Wds = ([Wd0] + [Wd0.clone() for _ in range(R - 1)]) if kind == "ffn" else None
    out = torch.empty((T, h), dtype=tdt, device=dev)
    y = torch.empty((T, d), dtype=tdt, device=dev) if kind == "ffn" else None
    scratch = torch.zeros(mglu.scratch_bytes(max(d, h)), dtype=torch.uint8, device=dev)
    routed = w.get("route_k") is not None
    if routed:
        g = torch.Generator(device="cpu").manual_seed(w["seed"] + 17)
        Wr = (torch.randn(nm, d, generator=g) / math.sqrt(d)).to(tdt).to(dev)
        mw = torch.empty((T, nm), dtype=torch.float32, device=dev)
        msc = torch.empty((T, nm), dtype=torch.float32, device=dev)

    def step(i, ev=None):
        """One step on the current stream; ev = events bracketing its kernels."""
        r = i % R
        if ev is not None:
            ev[0].record()
        if routed:
            # the router and the weighted forward in one call (on the decode
            # kernel the router runs inside it)
            mglu.forward_routed(x, Ws[r], pks[r], nm, Wr, w["route_k"], "hard", w["act"], out=out, weights=mw,
                                scores=msc, scratch=scratch)
        else:
            mglu.forward(x, Ws[r], pks[r], nm, w["act"], out=out, scratch=scratch)
        if ev is not None:
            ev[1].record()
        if kind == "ffn":
            mglu.down_proj(out, Wds[r], out=y, scratch=scratch)
            if ev is not None:
                ev[2].record()

    # warm-up (untimed, eager)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    if mglu.last_device_status() != 0:
        raise SystemExit(f"device status error during warm-up of {w['name']}")
    # this library's kernel launches per step, counted by the library itself
    n_before = mglu.kernel_launches()
    step(0)
    launches_per_step = mglu.kernel_launches() - n_before
    torch.cuda.synchronize(dev)

    # The K timed steps are captured once as a CUDA graph and replayed: the
    # kernels run back to back (each may start its prologue while the
    # previous one drains, as in a decode loop).  A second graph with event
    # nodes around each kernel gives the per-kernel split of a step.
    K = args.steps
    cap = torch.cuda.Stream(dev)

    def capture(with_events):
        g = torch.cuda.CUDAGraph()
        evs = ([[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3 if kind == "ffn" else 2)]
                for _ in range(K)] if with_events else None)
        cap.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.graph(g, stream=cap):
            for i in range(K):
                step(i, evs[i] if evs else None)
        torch.cuda.current_stream(dev).wait_stream(cap)
        return g, evs

    graph, _ = capture(False)
    graph.replay()  # one untimed replay
    torch.cuda.synchronize(dev)

    # an untimed run of the same graph to settle and sample clocks
    sampler = ClockSampler(dist.local) if sample_clocks else None
    if sampler:
        sampler.start()
    t_end = time.perf_counter() + args.probe_seconds
    while time.perf_counter() < t_end:
        graph.replay()
        torch.cuda.synchronize(dev)

    # timed region: exactly K steps (one replay of the captured graph)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record()
    graph.replay()
    t1.record()
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop() if sampler else None
    status = mglu.last_device_status()
    total_ms = dist.max(t0.elapsed_time(t1), dev)
    ms_per_step = total_ms / K
    value = dist.world * T * K / (total_ms / 1000.0)
    del graph

    # per-kernel durations, each kernel bracketed by event nodes (no overlap)
    graph_ev, evs = capture(True)
    graph_ev.replay()
    torch.cuda.synchronize(dev)
    up_iso_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    down_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) if kind == "ffn" else None
    del graph_ev
    # the dominant kernel's average launch duration in the timed region: for a
    # one-kernel step the back-to-back period; for the block its isolated time
    up_ms = ms_per_step if kind != "ffn" else dist.max(up_iso_ms, dev)

    # End to end through the public host-buffer call: one library call per
    # step copies that step's x in from pinned host memory, runs the kernels
    # and copies the result out, in order on its stream.  Consecutive steps
    # alternate over two streams (each with its own pinned buffers and
    # workspace), as a serving loop pipelines requests: one step's copies
    # overlap the other's kernels.
    res = y if kind == "ffn" else out
    stream = torch.cuda.current_stream(dev)
    NS = 2
    e2e_streams = [torch.cuda.Stream(dev) for _ in range(NS)]
    x_hs = [torch.empty((T, d), dtype=tdt, pin_memory=True) for _ in range(NS)]
    for xh in x_hs:
        xh.copy_(x.cpu())
    res_hs = [torch.empty(res.shape, dtype=tdt, pin_memory=True) for _ in range(NS)]
    ws_need = max(256, mglu.host_workspace_bytes(T, d, h, nm, tdt, kind == "ffn"))
    ws_hosts = [torch.zeros(ws_need, dtype=torch.uint8, device=dev) for _ in range(NS)]

    def e2e_step(i):
        r, q = i % R, i % NS
        mglu.forward_host(x_hs[q], Ws[r], pks[r], nm, w["act"], W_down=Wds[r] if kind == "ffn" else None,
                          out_host=res_hs[q], workspace=ws_hosts[q], stream=e2e_streams[q])

    n_host = 50
    if routed:
        K_e2e = 0  # the host-buffer entry point has no routed form
    else:
        K_e2e = K
    for i in range(args.warmup if K_e2e else 0):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    h0 = time.perf_counter()
    for i in range(n_host):
        mglu.forward(x, Ws[i % R], pks[i % R], nm, w["act"], out=out, scratch=scratch)
    host_us = (time.perf_counter() - h0) / n_host * 1e6
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for st in e2e_streams:
        st.wait_event(e0)
    for i in range(K_e2e):
        e2e_step(i)
    for st in e2e_streams:
        done = torch.cuda.Event()
        done.record(st)
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    e2e_ms = dist.max(e0.elapsed_time(e1), dev)
    e2e_value = dist.world * T * K_e2e / (e2e_ms / 1000.0) if K_e2e else None
    status = status or mglu.last_device_status()

    peaks, peak_src = load_peaks()
    decode = T <= 16 and w["dtype"] != "f32"
    if decode or kind == "tiny":
        achieved = up_bytes / (up_ms / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs (copy)"}
    else:
        achieved = up_flops / (up_ms / 1000.0) / 1e12
        pk = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk, "unit": "TFLOP/s",
                "frac": achieved / pk, "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", pk)}
    roof["traffic"] = recorded_traffic(w["name"], T)
    roof["kernel"] = ("mglu up-projection (decode)" if decode else
                      "mglu up-projection (tcgen05)" if w["dtype"] != "f32" else "mglu fp32")
    roof["kernel_us"] = up_ms * 1000.0
    roof["kernel_us_isolated"] = up_iso_ms * 1000.0
    roof["algorithmic_bytes"] = up_bytes
    roof["algorithmic_flops"] = up_flops

    rec = {
        "value": value, "unit": "tok/s", "ms_per_step": ms_per_step, "dtype": w["dtype"],
        "config": config_of(w, dist.world),
        "roofline": roof,
        "e2e": ({"value": e2e_value, "unit": "tok/s", "h2d_bytes_per_step": x_hs[0].numel() * x_hs[0].element_size(),
                 "d2h_bytes_per_step": res_hs[0].numel() * res_hs[0].element_size()} if e2e_value else None),
        "gpu_launches": K * launches_per_step,
        "host_us_per_forward_call": host_us,
        "device_status": status,
        "rotating_copies": R,
        "working_set_mb": R * working / 1e6,
    }
    if clocks is not None:
        rec["clocks"] = clocks
    if kind == "ffn":
        rec["down_kernel_us"] = down_ms * 1000.0
        rec["down_gbs"] = down_bytes / (down_ms / 1000.0) / 1e9
        rec["down_tflops"] = down_flops / (down_ms / 1000.0) / 1e12
    if decode:
        rec["hbm_gbs"] = up_bytes / (up_ms / 1000.0) / 1e9
    else:
        rec["tflops"] = up_flops / (up_ms / 1000.0) / 1e12
    extra = {"l2": l2}
    del Ws, pks, Wds, x, out, y, scratch, ws_hosts
    gc.collect()
    torch.cuda.empty_cache()
    return rec, extra


def measure_backward(args, dist, dev):
    """The training path's backward (straight-through gradients dx, dW and the
    mask-logit gradients) on the prefill layer: K calls timed with CUDA events
    around them on the launching stream, after the warm-up calls."""
    import numpy as np
    import torch

    from masked_glu_b200 import inputs, mglu

    w = workload_shape("prefill_T4096_d2048_h8192_nm4")
    T, d, h, nm = w["T"], w["d"], w["h"], w["n_m"]
    case = inputs.make_case(T, d, h, nm, seed=w["seed"] + 31 + 7919 * dist.rank)

    def up(t):
        return torch.from_numpy(t.storage.view(np.int16)).view(torch.bfloat16).to(dev)

    x, W = up(case.x), up(case.W)
    packed = mglu.pack_masks(torch.from_numpy(case.masks).to(dev))
    del case
    g = torch.Generator(device="cpu").manual_seed(w["seed"] + 37)
    dout = torch.randn((T, h), generator=g).to(torch.bfloat16).to(dev)
    ws = torch.empty(max(256, int(mglu.lib().mglu_backward_workspace_bytes(T, d, h, nm))), dtype=torch.uint8,
                     device=dev)
    for _ in range(args.warmup):
        mglu.backward(x, W, packed, nm, dout, "swish", workspace=ws)
    torch.cuda.synchronize(dev)
    n_before = mglu.kernel_launches()
    mglu.backward(x, W, packed, nm, dout, "swish", workspace=ws)
    launches_per_step = mglu.kernel_launches() - n_before
    torch.cuda.synchronize(dev)
    if mglu.last_device_status() != 0:
        raise SystemExit("device status error during the backward's warm-up")
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dist.local)
    sampler.start()
    dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record()
    for _ in range(K):
        mglu.backward(x, W, packed, nm, dout, "swish", workspace=ws)
    t1.record()
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop()
    ms = dist.max(t0.elapsed_time(t1), dev) / K
    # the recomputed products, dx = G B over K = (n_m + 1) h, and the n_m + 1
    # products E_i = G_i^T x: three contractions of 2 T d h (n_m + 1) each
    flops = 3 * 2 * T * d * h * (nm + 1)
    peaks, peak_src = load_peaks()
    achieved = flops / (ms / 1000.0) / 1e12
    rec = {
        "value": dist.world * T / (ms / 1000.0), "unit": "tok/s", "ms_per_step": ms, "dtype": "bf16",
        "config": {"workload": w["name"], "pass": "backward (dx, dW, mask-logit gradients)", "T": T, "d": d, "h": h,
                   "n_m": nm, "act": "swish"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16_tflops (burst)", "algorithmic_flops": flops,
                     "note": "whole backward: the tensor-core recompute with the gradient epilogue, the masked "
                             "operand, two cuBLAS GEMMs and the combine"},
        "gpu_launches": K * launches_per_step,
        "timing": "K eager calls between CUDA events on the launching stream",
        "clocks": clocks,
        "device_status": mglu.last_device_status(),
    }
    del x, W, packed, dout, ws
    gc.collect()
    torch.cuda.empty_cache()
    return rec


def tstar_sweep(args, dist, dev):
    """Device time of the FFN block (up + down) at T = 8..128 with the decode
    kernel allowed up to 16 tokens and with every T on the tensor-core kernel:
    where the two cross is the dispatch point."""
    import numpy as np
    import torch

    from masked_glu_b200 import inputs, mglu

    w = workload_shape("ffn_d4096_h14336_nm8", 128)
    d, h, nm = w["d"], w["h"], w["n_m"]
    case = inputs.make_case(128, d, h, nm, seed=w["seed"], with_down=True)

    def up(t):
        return torch.from_numpy(t.storage.view(np.int16)).view(torch.bfloat16).to(dev)

    x128, W0, Wd0 = up(case.x), up(case.W), up(case.W_down)
    pk0 = mglu.pack_masks(torch.from_numpy(case.masks).to(dev))
    del case
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(2, math.ceil(4 * l2 / (W0.numel() * 4 + pk0.numel())))
    Ws = [W0] + [W0.clone() for _ in range(R - 1)]
    pks = [pk0] + [pk0.clone() for _ in range(R - 1)]
    Wds = [Wd0] + [Wd0.clone() for _ in range(R - 1)]
    scratch = torch.zeros(mglu.scratch_bytes(max(d, h)), dtype=torch.uint8, device=dev)
    rows = []
    prev = mglu.set_decode_max_tokens(16)
    try:
        for T in (8, 12, 16, 24, 32, 48, 64, 128):
            x = x128[:T].contiguous()
            hid = torch.empty((T, h), dtype=torch.bfloat16, device=dev)
            yy = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
            row = {"T": T}
            for limit in (16, 0):
                if limit == 16 and T > 16:
                    continue
                mglu.set_decode_max_tokens(limit)

                def blk(i):
                    mglu.forward(x, Ws[i % R], pks[i % R], nm, "swish", out=hid, scratch=scratch)
                    mglu.down_proj(hid, Wds[i % R], out=yy, scratch=scratch)

                for i in range(2 * R):
                    blk(i)
                torch.cuda.synchronize(dev)
                n = 8 * R
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for i in range(n):
                    blk(i)
                e1.record()
                e1.synchronize()
                row["decode_us" if limit == 16 else "tensor_core_us"] = dist.max(e0.elapsed_time(e1) * 1000 / n, dev)
            rows.append(row)
    finally:
        mglu.set_decode_max_tokens(prev)
    del Ws, pks, Wds, scratch
    torch.cuda.empty_cache()
    return {"what": "FFN block d=4096 h=14336 n_m=8, up + down per call, weights rotating over copies > 4x L2, "
                    "eager back-to-back calls", "rows": rows}


def run_mglu(args, dist):
    import torch

    from masked_glu_b200 import build as mbuild
    from masked_glu_b200 import mglu

    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    mbuild.build()
    mglu.lib()
    mglu.set_decode_max_tokens(16)

    if args.backward_only:
        rec = measure_backward(args, dist, dev)
        if dist.rank == 0:
            print(json.dumps(dict(rec, metric="MGLU training backward TFLOP/s vs B200 bf16 roofline",
                                  n_gpus=dist.world, steps=args.steps, warmup=args.warmup)), flush=True)
        dist.close()
        return
    w = workload_shape(args.workload, args.tokens, args.act, args.p)
    rec, extra = measure(args, dist, w, dev, sample_clocks=True)
    line = {"metric": METRIC, "value": rec["value"], "unit": "tok/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w["dtype"],
            "data": "synthetic: x ~ N(0,1), W ~ N(0,0.02^2), Bernoulli(p) masks, seeded PCG64"}
    line.update({k: v for k, v in rec.items() if k not in line})
    line["timing"] = ("device-side: one CUDA-graph replay of the K steps back to back (CUDA events around the "
                      "replay); kernel_us_isolated: a second replay with event nodes around each kernel; e2e: one "
                      "mglu_forward_host call per step (pinned host x in, kernels, pinned host result out), "
                      "consecutive steps alternating over two streams")

    if dist.world == 1 and w["dtype"] == "bf16" and not args.no_comparisons:
        line["comparisons"] = time_comparisons(w["T"], w["d"], w["h"], w["n_m"], w["act"], dev, extra["l2"])
        line["comparisons"]["mglu_us"] = rec["roofline"]["kernel_us"] + rec.get("down_kernel_us", 0.0)
        if w["kind"] == "ffn":
            line["comparisons"]["note"] += "; mglu_us includes the down-projection, the baselines do not"

    if args.suite:
        subs = []
        for entry in SUITE:
            name, T, act = entry[:3]
            ws = workload_shape(name, T if name.startswith("ffn") else None, act, 0.5,
                                entry[3] if len(entry) > 3 else None)
            r, _ = measure(args, dist, ws, dev, sample_clocks=True)
            subs.append(r)
        line["workloads"] = subs
        line["training_backward"] = measure_backward(args, dist, dev)
        line["gpu_launches_all_workloads"] = (line["gpu_launches"] + sum(r["gpu_launches"] for r in subs) +
                                              line["training_backward"]["gpu_launches"])
    if args.tstar_sweep:
        line["tstar_sweep"] = tstar_sweep(args, dist, dev)

    # the CPU oracle on a bounded sample: rank 0, one GPU only
    if dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline:
        cb, _ = time_oracle(w)
        line["cpu_baseline"] = cb
    dist.barrier()
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    run_mglu(args, dist)


if __name__ == "__main__":
    main()
