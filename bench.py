#!/usr/bin/env python
"""Benchmark of padding-aware sigmoid attention (forward + backward) on B200.

One step = one forward (sigattn_fwd) and one backward (sigattn_bwd: dQ kernel
+ dK/dV kernel) over one batch of the 16K / head-dim-128 kernel-benchmark
workload without padding (Z=2, H=16, L=16384, D=128, bf16; paperlayer.ai
summary, section 4).  The padded workloads (Z=4, L=16384) are measured the
same way and reported beside it with their padding loss.  Throughput counts
valid-token FLOPs: 4 D H sum n_q n_k forward and 2.5x that backward
(paperlayer.ai summary, appendix A.2).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With --gpus N > 1 and no torchrun environment, the script starts N ranks
itself under torch.distributed.run (127.0.0.1).  Every rank runs its own batch
(weak scaling: the path shards over independent (z, h) problems with no
collective); the time is the max over ranks.  Prints one JSON line on rank 0.

Profiling helpers (no JSON line):
  --only fwd|dq|dkdv|all --shape Z,H,L,D   launches of one kernel on full lengths
  --write-traffic CSV...                    writes profiles/traffic.json from ncu
                                            CSV logs of dram__bytes_read.sum and
                                            dram__bytes_write.sum
"""
from __future__ import annotations

import argparse
import json
import math
import os
import re
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd/bwd TFLOPS (valid tokens) at L=16K d=128, 0%/25% pad; % of B200 BF16 peak"
HEADLINE = 3      # 16K, no padding
PADDED = 4        # 16K, 25% padding
L2_BYTES = 126 * 1024 * 1024
# four lengths evenly spaced over the 25%-padding workload's range [8192, 16384]:
# their mean is 12288 = 75% of L = 16384, so exactly 25% of the tokens are padding
EXACT25_LENGTHS = (8192, 10923, 13653, 16384)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", choices=["fwd", "dq", "dkdv", "all"], default=None,
                    help="launch only this kernel (profiling runs; prints timings, no JSON line)")
    ap.add_argument("--shape", default="2,16,4096,128", help="Z,H,L,D for --only")
    ap.add_argument("--workload", type=int, default=None,
                    help="with --only: run on this workload's shape, lengths and inputs instead")
    ap.add_argument("--sigmoid-mode", choices=["exp", "tanh"], default=None)
    ap.add_argument("--write-traffic", nargs="+", default=None, metavar="CSV",
                    help="write profiles/traffic.json from ncu CSV logs (no GPU needed)")
    ap.add_argument("--no-eager", action="store_true",
                    help="skip the PyTorch-eager context measurement")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(bf16=float(d["bf16_tflops"]), bf16_sustained=float(d["bf16_tflops_sustained"]),
                    hbm=float(d["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(args) -> int:
    """Runs this script as `args.gpus` ranks under torch.distributed.run (one
    node, rendezvous on 127.0.0.1) and returns its exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.run(cmd, timeout=3600).returncode


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        print(f"bench rank {rank} of {world} (local {local}) ready", file=sys.stderr, flush=True)
        if args.impl == "ours":
            import datetime
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- reference arm (the oracle)


def cpu_sample(w, rows: int, seed: int = 0):
    """A bounded sample of one workload for the fp64 oracle: `rows` query rows
    (forward + dQ) and `rows` key rows (dK, dV), spread over (z, h)."""
    from padding_aware_sigmoid_b200 import workloads as W
    inp = W.make_inputs(w)
    g = np.random.default_rng(seed)
    n = W.lengths(w)
    z = g.integers(0, w.Z, size=rows)
    h = g.integers(0, w.H, size=rows)
    r = np.array([g.integers(0, max(int(n[zz]), 1)) for zz in z])
    items = np.stack([z, h, r], axis=1).astype(np.int64)
    # counted FLOPs of the sample: each row carries its n_k (resp. n_q) pairs
    pairs = float(np.sum(n[z]))
    counted = (1.0 + 2.5) * 4.0 * w.D * pairs
    return inp, items, counted


def run_oracle_step(inp, items):
    import oracle
    a = (inp["q"], inp["k"], inp["v"])
    lens = (inp["seqlens_q"], inp["seqlens_k"], inp["alpha"], inp["bias"])
    oracle.fwd_rows(*a, *lens, items)
    oracle.dq_rows(*a, inp["dout"], *lens, items)
    oracle.dkdv_rows(*a, inp["dout"], *lens, items)


def reference_arm(args, world, rank):
    if rank != 0:
        return
    import oracle
    from padding_aware_sigmoid_b200 import workloads as W
    w = W.WORKLOADS[HEADLINE]
    rows = 96
    inp, items, counted = cpu_sample(w, rows)
    for _ in range(max(args.warmup, 0)):
        run_oracle_step(inp, items[:8])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_step(inp, items)
    dt = (time.perf_counter() - t0) / args.steps
    value = counted / dt / 1e12
    cores = oracle.num_threads()
    sample = (f"{rows} query rows (fwd + dQ) and {rows} key rows (dK, dV) per step, drawn from "
              f"the {w.name} workload (Z={w.Z}, H={w.H}, L={w.L}, D={w.D})")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "Z": w.Z, "H": w.H, "L": w.L, "D": w.D,
                   "lengths": "n_q = n_k = 16384", "parallelism": "single host process"},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm


def make_device_inputs(w, device, seed_offset: int, lengths=None):
    """Seeded device inputs of workload `w` (lengths: the workload's own unless given)."""
    import torch
    from padding_aware_sigmoid_b200 import workloads as W
    n = W.lengths(w) if lengths is None else np.asarray(lengths, np.int32)
    g = torch.Generator(device=device).manual_seed(1000 * w.index + seed_offset)
    q, k, v, do = (torch.randn((w.Z, w.L, w.H, w.D), generator=g, device=device,
                               dtype=torch.float32).mul_(w.qkv_scale if i < 3 else 1.0)
                   .to(torch.bfloat16) for i in range(4))
    nd = torch.as_tensor(n, dtype=torch.int32, device=device)
    return dict(q=q, k=k, v=v, dout=do, nq=nd, nk=nd, n=n)


def time_workload(sa, w, inp, steps, warmup, device, sampler=None):
    """Times K steps (fwd + bwd) with CUDA events on the launching stream; also
    the per-call durations of the forward, the dQ and the dK/dV kernels."""
    import torch
    st = torch.cuda.current_stream(device)
    o = torch.empty_like(inp["q"])
    dq, dk, dv = (torch.empty_like(inp["q"]) for _ in range(3))
    args = (inp["q"], inp["k"], inp["v"])

    def step(ev=None):
        if ev is not None:
            ev[0].record(st)
        sa.fwd(*args, inp["nq"], inp["nk"], w.alpha, w.bias, out=o)
        if ev is not None:
            ev[1].record(st)
        sa.bwd_dq(*args, inp["dout"], inp["nq"], inp["nk"], w.alpha, w.bias, dq=dq)
        if ev is not None:
            ev[2].record(st)
        sa.bwd_dkdv(*args, inp["dout"], inp["nq"], inp["nk"], w.alpha, w.bias, dk=dk, dv=dv)
        if ev is not None:
            ev[3].record(st)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(st)
    for i in range(steps):
        step(evs[i])
    end.record(st)
    torch.cuda.synchronize(device)
    total_ms = start.elapsed_time(end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    dq_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    dkdv_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    assert sa.last_device_status(device) == 0
    return total_ms / steps, fwd_ms, dq_ms, dkdv_ms


def graph_kernel_ms(call, device, reps=50, trials=3):
    """Device time of one call with the host out of the way: `reps` calls are
    captured in a CUDA graph, the graph is replayed `trials` times, each replay
    timed with events, and the median per-call time is returned.  For short
    launches (the D = 64 workloads run ~0.1 ms) eager timing includes the host's
    launch cost between the events."""
    import torch
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream(device).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            call()
    st = torch.cuda.current_stream(device)
    g.replay()
    times = []
    for _ in range(trials):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        g.replay()
        e1.record(st)
        torch.cuda.synchronize(device)
        times.append(e0.elapsed_time(e1) / reps)
    del g
    return statistics.median(times)


def e2e_workload(sa, w, steps, warmup, device):
    """Same step through the public API with host buffers: sigattn_fwd_bwd_host
    copies Q, K, V, dO from pinned host memory, runs the forward and the backward,
    and copies O, dQ, dK, dV back, unit by unit (a sample and a group of heads)
    with the copies overlapping the compute; all of it inside the timed region."""
    import torch
    from padding_aware_sigmoid_b200 import workloads as W
    hq, hk, hv, hdo = (torch.empty((w.Z, w.L, w.H, w.D), dtype=torch.bfloat16).pin_memory()
                       for _ in range(4))
    g = torch.Generator().manual_seed(7)
    for t in (hq, hk, hv, hdo):
        t.copy_(torch.randn(t.shape, generator=g).to(torch.bfloat16))
    n = W.lengths(w)
    outs = [torch.empty_like(hq).pin_memory() for _ in range(4)]
    st = torch.cuda.current_stream(device)

    def step():
        sa.fwd_bwd_host(hq, hk, hv, hdo, n, n, w.alpha, w.bias, outs=outs, device=device)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(st)
    for _ in range(steps):
        step()
    e.record(st)
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / steps
    h2d = 4 * hq.numel() * 2 + 2 * 4 * w.Z   # tensors, and the lengths (as kernel arguments)
    d2h = 4 * hq.numel() * 2
    return ms, h2d, d2h


def eager_sigmoid_attention(q, k, v, n, alpha: float, bias: float):
    """Sigmoid attention written with plain PyTorch ops (the pages' PyTorch
    baseline, paper.rainbus.top results table): the full score matrix is
    materialised in bf16, masked by multiplication, then multiplied by V."""
    import torch
    Z, L, H, D = q.shape
    qh, kh, vh = (t.permute(0, 2, 1, 3) for t in (q, k, v))
    s = torch.matmul(qh, kh.transpose(-1, -2)) * alpha + bias
    pos = torch.arange(L, device=q.device)
    keep = (pos[None, :] < n[:, None]).to(q.dtype)            # [Z, L]
    p = torch.sigmoid(s) * keep[:, None, None, :]
    o = torch.matmul(p, vh) * keep[:, None, :, None]
    return o.permute(0, 2, 1, 3)


def eager_context(w, device, heads: int = 4, reps: int = 3):
    """Context only, not the product: forward and backward of the PyTorch-eager
    version on `heads` heads of one sample of workload `w` (its whole score
    matrix fits in HBM), timed with CUDA events, in valid-FLOP TFLOPS."""
    import torch
    g = torch.Generator(device=device).manual_seed(11)
    shape = (1, w.L, heads, w.D)
    q, k, v, do = (torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
                   for _ in range(4))
    for t in (q, k, v):
        t.requires_grad_(True)
    n = torch.full((1,), w.L, dtype=torch.int32, device=device)
    fl = 4.0 * w.D * heads * float(w.L) * w.L
    st = torch.cuda.current_stream(device)
    fwd, bwd = [], []
    for i in range(reps + 1):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(st)
        o = eager_sigmoid_attention(q, k, v, n, w.alpha, w.bias)
        e[1].record(st)
        o.backward(do)
        e[2].record(st)
        torch.cuda.synchronize(device)
        if i > 0:
            fwd.append(e[0].elapsed_time(e[1]))
            bwd.append(e[1].elapsed_time(e[2]))
        del o
        q.grad = k.grad = v.grad = None
    f_ms, b_ms = statistics.median(fwd), statistics.median(bwd)
    del q, k, v, do
    torch.cuda.empty_cache()
    return {"fwd_ms": f_ms, "bwd_ms": b_ms, "fwd_tflops": fl / (f_ms * 1e-3) / 1e12,
            "bwd_tflops": 2.5 * fl / (b_ms * 1e-3) / 1e12,
            "slice": f"Z=1, H={heads}, L={w.L}, D={w.D}, full lengths, bf16 (a slice of the "
                     f"{w.name} workload; every head costs the same)",
            "note": "plain PyTorch ops with autograd on this GPU, timed as context for the "
                    "pages' PyTorch rows; not part of the library"}


def our_arm(args, world, rank, local):
    import torch
    import padding_aware_sigmoid_b200 as sa
    from padding_aware_sigmoid_b200 import workloads as W

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    pk = peaks()
    w3, w4 = W.WORKLOADS[HEADLINE], W.WORKLOADS[PADDED]
    f3 = W.fwd_flops_valid(W.lengths(w3), W.lengths(w3), w3.H, w3.D)
    f4_pad = W.fwd_flops_padded(w4.Z, w4.L, w4.H, w4.D)

    # the D = 64 workloads (2: short ragged sequences, 5: lognormal lengths, large
    # scores), timed the same way with their own valid-FLOP counts, before the
    # D = 128 runs: right after seconds of D = 128 work under the power cap the
    # SM clock is still low, and these ~0.1 ms launches then run up to 28% slower
    # until it recovers
    d64 = {}
    for idx in (2, 5):
        w = W.WORKLOADS[idx]
        inp = make_device_inputs(w, device, rank)
        st_ms, f_ms, q_ms, kv_ms = time_workload(sa, w, inp, max(args.steps // 2, 3),
                                                 args.warmup, device)
        fl = W.fwd_flops_valid(W.lengths(w), W.lengths(w), w.H, w.D)
        a_ = (inp["q"], inp["k"], inp["v"])
        o_, dq_, dk_, dv_ = (torch.empty_like(inp["q"]) for _ in range(4))
        g_f = graph_kernel_ms(lambda: sa.fwd(*a_, inp["nq"], inp["nk"], w.alpha, w.bias, out=o_),
                              device)
        g_q = graph_kernel_ms(lambda: sa.bwd_dq(*a_, inp["dout"], inp["nq"], inp["nk"], w.alpha,
                                                w.bias, dq=dq_), device)
        g_kv = graph_kernel_ms(lambda: sa.bwd_dkdv(*a_, inp["dout"], inp["nq"], inp["nk"],
                                                   w.alpha, w.bias, dk=dk_, dv=dv_), device)
        d64[w.name] = {
            "fwd_tflops": fl / (g_f * 1e-3) / 1e12,
            "bwd_tflops": 2.5 * fl / ((g_q + g_kv) * 1e-3) / 1e12,
            "fwd_ms": g_f, "bwd_dq_ms": g_q, "bwd_dkdv_ms": g_kv,
            "timing": "device time per call: median of 3 replays of a CUDA graph of 50 calls, "
                      "measured before the D = 128 workloads",
            "eager": {"fwd_ms": f_ms, "bwd_dq_ms": q_ms, "bwd_dkdv_ms": kv_ms,
                      "step_ms": st_ms,
                      "note": "calls launched from Python between events: includes host "
                              "launch cost where the kernel is shorter than it"},
            "valid_fraction_of_padded_flops":
                fl / W.fwd_flops_padded(w.Z, w.L, w.H, w.D),
        }
        assert sa.last_device_status(device) == 0
        del o_, dq_, dk_, dv_
        del inp
    torch.cuda.empty_cache()

    inp3 = make_device_inputs(w3, device, rank)
    barrier(world)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize(device)
        step_ms, fwd_ms, dq_ms, dkdv_ms = time_workload(sa, w3, inp3, args.steps, args.warmup,
                                                        device)
    step_ms = max_over_ranks(step_ms, world, device)
    barrier(world)
    del inp3
    # Padding: the 25%-padding workload as drawn (lengths U[8192, 16384] from its
    # seed), the same Z = 4 shape with no padding (so that the loss compares like
    # grids), and lengths evenly spaced over [8192, 16384] whose tokens are
    # exactly 25% padding (mean fill 75%, as the workload intends).
    pad_runs = {}
    for name, lens in (("drawn", W.lengths(w4)), ("nopad_z4", [w4.L] * w4.Z),
                       ("exact25", EXACT25_LENGTHS)):
        inp4 = make_device_inputs(w4, device, rank, lengths=lens)
        st_ms, f_ms, q_ms, kv_ms = time_workload(sa, w4, inp4, max(args.steps // 2, 3),
                                                 args.warmup, device)
        st_ms = max_over_ranks(st_ms, world, device)
        fl = W.fwd_flops_valid(lens, lens, w4.H, w4.D)
        pad_runs[name] = {
            "lengths": [int(x) for x in lens],
            "token_padding_fraction": 1.0 - float(np.sum(lens)) / (w4.Z * w4.L),
            "valid_fraction_of_padded_flops": fl / f4_pad,
            "fwd_ms": f_ms, "bwd_dq_ms": q_ms, "bwd_dkdv_ms": kv_ms, "ms_per_step": st_ms,
            "fwd_tflops": fl / (f_ms * 1e-3) / 1e12,
            "bwd_tflops": 2.5 * fl / ((q_ms + kv_ms) * 1e-3) / 1e12,
            "fwd_tflops_padded_flops": f4_pad / (f_ms * 1e-3) / 1e12,
        }
        del inp4
        torch.cuda.empty_cache()
    ref = pad_runs["nopad_z4"]
    for name in ("drawn", "exact25"):
        r = pad_runs[name]
        r["fwd_padding_loss_pct"] = 100.0 * (1.0 - r["fwd_tflops"] / ref["fwd_tflops"])
        r["bwd_padding_loss_pct"] = 100.0 * (1.0 - r["bwd_tflops"] / ref["bwd_tflops"])

    # each kernel also timed on its own (10 back-to-back launches after the step
    # loop): the GPU's power-limited clock then follows that kernel alone
    import torch as _t
    inp3 = make_device_inputs(w3, device, rank)
    o_, dq_, dk_, dv_ = (_t.empty_like(inp3["q"]) for _ in range(4))
    a3 = (inp3["q"], inp3["k"], inp3["v"])
    alone = {}
    for name, call in (
            ("fwd", lambda: sa.fwd(*a3, inp3["nq"], inp3["nk"], w3.alpha, w3.bias, out=o_)),
            ("bwd_dq", lambda: sa.bwd_dq(*a3, inp3["dout"], inp3["nq"], inp3["nk"], w3.alpha,
                                         w3.bias, dq=dq_)),
            ("bwd_dkdv", lambda: sa.bwd_dkdv(*a3, inp3["dout"], inp3["nq"], inp3["nk"], w3.alpha,
                                             w3.bias, dk=dk_, dv=dv_))):
        for _ in range(3):
            call()
        st_ = _t.cuda.current_stream(device)
        e0, e1 = _t.cuda.Event(enable_timing=True), _t.cuda.Event(enable_timing=True)
        e0.record(st_)
        for _ in range(10):
            call()
        e1.record(st_)
        _t.cuda.synchronize(device)
        alone[name] = e0.elapsed_time(e1) / 10
    del inp3, o_, dq_, dk_, dv_

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_workload(sa, w3, max(args.steps // 4, 3), 2, device)
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        e2e = {"value": world * f3 * 3.5 / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    eager = None
    if rank == 0 and not args.no_eager:
        eager = eager_context(w3, device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        rows = 1024
        inp_cpu, items, counted = cpu_sample(w3, rows, seed=1)
        t0 = time.perf_counter()
        run_oracle_step(inp_cpu, items)
        dt = time.perf_counter() - t0
        cpu = {"value": counted / dt / 1e12, "unit": "TFLOPS", "cores": oracle.num_threads(),
               "kind": "oracle", "seconds": dt,
               "sample": f"{rows} query rows (fwd + dQ) and {rows} key rows (dK, dV) of the "
                         f"{w3.name} workload, fp64, counted with the same FLOP convention"}

    if rank != 0:
        return
    fwd_tf = f3 / (fwd_ms * 1e-3) / 1e12
    bwd_tf = 2.5 * f3 / ((dq_ms + dkdv_ms) * 1e-3) / 1e12
    step_tf = world * 3.5 * f3 / (step_ms * 1e-3) / 1e12
    # dominant kernel: the longest of the three per step
    kernels = {"fwd": (fwd_ms, f3), "bwd_dkdv": (dkdv_ms, 8.0 / 4.0 * f3),
               "bwd_dq": (dq_ms, 6.0 / 4.0 * f3)}
    dom = max(kernels, key=lambda k: kernels[k][0])
    dom_ms, dom_flops = kernels[dom]
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    traffic = _ncu_traffic(dom)
    line = {
        "metric": METRIC,
        "value": step_tf,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w3.name, "Z": w3.Z, "H": w3.H, "L": w3.L, "D": w3.D,
            "lengths": "n_q = n_k = 16384", "global_batch": world * w3.Z, "seq_len": w3.L,
            "parallelism": f"dp{world} over independent (z, h) problems, no collective",
            "l2": "inputs larger than L2: each of Q, K, V, dO is %.0f MB" % (
                w3.Z * w3.L * w3.H * w3.D * 2 / 1e6),
            "sigmoid_mode": "tanh" if sa.get_sigmoid_mode() == sa.SIGMOID_TANH else "exp",
        },
        "fwd_tflops": fwd_tf,
        "bwd_tflops": bwd_tf,
        "fwd_ms": fwd_ms, "bwd_dq_ms": dq_ms, "bwd_dkdv_ms": dkdv_ms,
        "alone": {
            "note": "each kernel launched 10x back to back on its own, outside the step loop",
            "fwd_ms": alone["fwd"], "bwd_dq_ms": alone["bwd_dq"],
            "bwd_dkdv_ms": alone["bwd_dkdv"],
            "fwd_tflops": f3 / (alone["fwd"] * 1e-3) / 1e12,
            "bwd_tflops": 2.5 * f3 / ((alone["bwd_dq"] + alone["bwd_dkdv"]) * 1e-3) / 1e12,
        },
        "fwd_pct_of_peak": 100.0 * fwd_tf / pk["bf16"],
        "bwd_pct_of_peak": 100.0 * bwd_tf / pk["bf16"],
        "pad25": dict(
            pad_runs,
            note="loss = 1 - valid-FLOP TFLOPS of the padded batch / that of the same Z = 4 "
                 "shape without padding; 'drawn' is the workload's seeded draw, 'exact25' has "
                 "exactly 25% padded tokens",
            fwd_padding_loss_pct=pad_runs["exact25"]["fwd_padding_loss_pct"],
            bwd_padding_loss_pct=pad_runs["exact25"]["bwd_padding_loss_pct"]),
        "workloads_d64": d64,
        "roofline": {
            "kernel": dom, "bound": "tensor", "achieved": achieved, "peak": pk["bf16"],
            "unit": "TFLOP/s", "frac": achieved / pk["bf16"], "traffic": traffic,
            "peak_kind": f"{pk['source']} bf16 burst (cuBLAS 8192^3)",
            "frac_of_sustained": achieved / pk["bf16_sustained"],
            "flops_per_launch": dom_flops,
        },
        "clocks": clk.summary(),
        "gpu_launches": 3 * args.steps,   # the timed headline steps: fwd, dQ, dK/dV
        "e2e": e2e,
        "cpu_baseline": cpu,
        "context": {"pytorch_eager": eager},
    }
    print(json.dumps(line), flush=True)


# the device code: every file a kernel is compiled from, including the ring
# depths and thread counts; host code (argument checks, caches, launches) is not
# part of it
DEVICE_SOURCES = ("fwd_sm100.cuh", "fwd_persist_sm100.cuh", "bwd_sm100.cuh", "bwd_persist_sm100.cuh",
                  "sm100.cuh", "sigmoid.cuh")
TRAFFIC_KERNELS = {"fwd": "fwd_tiles_kernel", "bwd_dq": "bwd_dq_kernel",
                   "bwd_dkdv": "bwd_dkdv_kernel"}
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.json")


def _code_tokens(text: str) -> str:
    """C++ source with comments removed and whitespace runs collapsed: what the
    compiler sees (string literals in these headers hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(src: str = "") -> str:
    """sha256 over the device-code headers of the library (names and code, with
    comments and layout ignored, so an edit of comments keeps the captures)."""
    import hashlib
    h = hashlib.sha256()
    src = src or os.path.join(ROOT, "padding_aware_sigmoid_b200", "csrc")
    for name in DEVICE_SOURCES:
        h.update(name.encode())
        with open(os.path.join(src, name), encoding="utf-8") as f:
            h.update(_code_tokens(f.read()).encode())
    return h.hexdigest()


def _ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu capture of the same kernel,
    or None when there is none or the device code changed since it was taken."""
    try:
        with open(TRAFFIC_PATH) as f:
            d = json.load(f)
        if d.get("_meta", {}).get("source_sha256") != kernel_source_hash():
            return None
        return d.get(kernel)
    except Exception:
        return None


_BYTE_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12}


def read_ncu_dram_csv(path: str) -> dict:
    """Per kernel name: list of (read + write) DRAM bytes, one per captured launch,
    from an `ncu --csv --log-file` of dram__bytes_read.sum and dram__bytes_write.sum."""
    import csv
    rows = []
    with open(path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    for r in csv.DictReader(lines):
        rows.append(r)
    per_launch = {}
    for r in rows:
        m = r.get("Metric Name", "")
        if m not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        unit = r.get("Metric Unit", "byte").strip().lower()
        val = float(r["Metric Value"].replace(",", "")) * _BYTE_UNITS[unit]
        key = (r["ID"], r["Kernel Name"])
        per_launch[key] = per_launch.get(key, 0.0) + val
    out = {}
    for (_, name), v in sorted(per_launch.items(), key=lambda kv: int(kv[0][0])):
        out.setdefault(name, []).append(v)
    return out


def write_traffic(paths, command: str = "") -> dict:
    """Writes profiles/traffic.json from ncu CSV logs: the mean bytes per launch of
    each library kernel found, the algorithmic bytes of the workload the captures
    ran on (workload 3 at full size), and the hash of the current device code."""
    from padding_aware_sigmoid_b200 import workloads as W
    w = W.WORKLOADS[HEADLINE]
    tensor = w.Z * w.L * w.H * w.D * 2
    got = {}
    for p in paths:
        for name, vals in read_ncu_dram_csv(p).items():
            for key, kname in TRAFFIC_KERNELS.items():
                if re.search(r"(^|[\s:])%s(<|\(|$)" % kname, name):
                    got.setdefault(key, []).extend(vals)
    d = {k: int(round(sum(v) / len(v))) for k, v in got.items()}
    d["_meta"] = {
        "what": "dram__bytes_read.sum + dram__bytes_write.sum per launch, mean over the "
                "captured launches, workload %s (Z=%d, H=%d, L=%d, D=%d), full size" % (
                    w.name, w.Z, w.H, w.L, w.D),
        "launches": {k: len(v) for k, v in got.items()},
        "algorithmic_bytes": {"fwd": 4 * tensor, "bwd_dq": 5 * tensor, "bwd_dkdv": 6 * tensor},
        "source_sha256": kernel_source_hash(),
        "device_sources": list(DEVICE_SOURCES),
        "command": command,
    }
    with open(TRAFFIC_PATH, "w") as f:
        json.dump(d, f, indent=1)
        f.write("\n")
    return d


def only_kernel(args):
    """Profiling helper: W warm-up and K timed launches of one kernel, either on a
    Z,H,L,D problem with full lengths (bf16, alpha = 1/sqrt(D), b = -ln L) or on
    one workload's shape, lengths and seeded inputs (--workload)."""
    import torch
    import padding_aware_sigmoid_b200 as sa
    from padding_aware_sigmoid_b200 import workloads as W
    dev = torch.device("cuda", 0)
    if args.workload is not None:
        w = W.WORKLOADS[args.workload]
        inp = make_device_inputs(w, dev, 0)
        q, k, v, do, n = inp["q"], inp["k"], inp["v"], inp["dout"], inp["nq"]
        Z, H, L, D = w.Z, w.H, w.L, w.D
        alpha, bias = w.alpha, w.bias
        flops = W.fwd_flops_valid(inp["n"], inp["n"], H, D)
    else:
        Z, H, L, D = (int(x) for x in args.shape.split(","))
        g = torch.Generator(device=dev).manual_seed(0)
        q, k, v, do = (torch.randn((Z, L, H, D), generator=g, device=dev).to(torch.bfloat16)
                       for _ in range(4))
        n = torch.full((Z,), L, dtype=torch.int32, device=dev)
        alpha, bias = 1.0 / math.sqrt(D), -math.log(L)
        flops = 4.0 * D * H * Z * L * L
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    calls = {
        "fwd": lambda: sa.fwd(q, k, v, n, n, alpha, bias, out=o),
        "dq": lambda: sa.bwd_dq(q, k, v, do, n, n, alpha, bias, dq=dq),
        "dkdv": lambda: sa.bwd_dkdv(q, k, v, do, n, n, alpha, bias, dk=dk, dv=dv),
    }
    names = list(calls) if args.only == "all" else [args.only]
    per = {"fwd": flops, "dq": 1.5 * flops, "dkdv": 2.0 * flops}
    for name in names:
        for _ in range(args.warmup):
            calls[name]()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            calls[name]()
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / args.steps
        print(json.dumps({"kernel": name, "shape": [Z, H, L, D], "workload": args.workload,
                          "ms": ms, "tflops_executed_valid_pairs": per[name] / ms / 1e9}),
              flush=True)
    assert sa.last_device_status() == 0


def main():
    args = parse()
    if args.write_traffic is not None:
        print(json.dumps(write_traffic(args.write_traffic, os.environ.get("TRAFFIC_COMMAND", ""))))
        return
    if args.sigmoid_mode is not None:
        import padding_aware_sigmoid_b200 as sa
        sa.set_sigmoid_mode(sa.SIGMOID_TANH if args.sigmoid_mode == "tanh" else sa.SIGMOID_EXP)
    if args.only is not None:
        only_kernel(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args))
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            reference_arm(args, world, rank)
        else:
            our_arm(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
