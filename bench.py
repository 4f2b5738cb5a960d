#!/usr/bin/env python
"""Benchmark: block attention forward + backward on one synthetic jagged batch.

One step = ba_fwd + ba_bwd over a whole batch (every kernel of the path).
Default workload: 256 user histories with lengths uniform in [64, 4096],
8 heads, head_dim 128, block 256, window 2, bf16 (the jagged long-history
case); --config picks another of the five workloads in workloads.py, --swa
the sliding-window variant, --rope the rotary entry points (ba_rope_fwd +
ba_rope_bwd: rotary embedding on q and k with tables covering the longest
example, resident on the device like weights; the forward's rotated q and k
are kept for the backward, as training keeps activations).

Prints ONE JSON line (rank 0). ``value`` is useful TFLOP/s (14 * head_dim
FLOPs per visible query/key pair and head, summed over all ranks) with the
inputs resident in HBM; ``e2e`` is the same metric with pinned-host inputs
copied in and the results copied out inside the timed region.

The same line carries ``other_configs``: the long-context workload (8 x 32768,
block 512, window 4), the jagged workload with component skip, and the jagged
histories with independent 64-token blocks (block 64, window 1), each timed
the same way (N = 1 only), each with its step's HBM bytes against the copy
bandwidth.

Multi-GPU: every rank runs its own batch (seeded per rank) with no
collective on the data path; the step time is the max over ranks. Launched
as ``bench.py --gpus N`` without torchrun, the script starts N ranks itself
(torch.distributed.run, one process per GPU); under torchrun it is one rank.
``--impl reference`` times the CPU oracle on bounded samples instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
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

from block_sparse_attention_kunlun_b200 import flops as F  # noqa: E402
from block_sparse_attention_kunlun_b200.workloads import CONFIGS, make_inputs, rope_tables  # noqa: E402

METRIC = "block-attention fwd+bwd useful TFLOP/s and tokens/s on 1 B200; % of bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    # config 1 is the fp32 forward parity configuration; the benchmark times the bf16 path
    ap.add_argument("--config", type=int, default=3, choices=[c for c in sorted(CONFIGS) if c != 1])
    ap.add_argument("--examples", type=int, default=0,
                    help="keep only the first N examples (small cases for profiling)")
    ap.add_argument("--block", type=int, default=0, help="override the config's block size")
    ap.add_argument("--window", type=int, default=0, help="override the config's window (in blocks)")
    ap.add_argument("--swa", type=int, default=0, metavar="W",
                    help="time sliding-window attention (each query sees its last W tokens; block 1, "
                         "window W) on the config's shapes instead of block attention")
    ap.add_argument("--rope", action="store_true",
                    help="rotary embedding on q and k (ba_rope_fwd / ba_rope_bwd)")
    ap.add_argument("--gdpa", choices=["gelu", "silu"], default=None,
                    help="generalized dot-product attention (ba_gdpa_fwd / ba_gdpa_bwd): the activation "
                         "in place of the softmax, same block rule and shapes")
    ap.add_argument("--mx", action="store_true",
                    help="MXFP8 Q and K in the score product (ba_mx_fwd / ba_mx_bwd), head_dim 128")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="leave out the other_configs workloads (shorter launch lists for profiling)")
    ap.add_argument("--traffic-file", default=os.path.join(ROOT, "profiles", "traffic.json"),
                    help="per-launch DRAM bytes of the dominant kernel from an ncu capture")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n: int, argv, script: str = None, **run_kw) -> subprocess.CompletedProcess:
    """Runs `script argv` as n ranks on this node (one process per GPU) through
    torch.distributed.run on 127.0.0.1 and waits for them. Each rank finds
    RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* in its environment; rank 0 alone
    prints the JSON line. run_kw goes to subprocess.run (e.g. capture_output)."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           script or os.path.abspath(__file__), *argv]
    return subprocess.run(cmd, **run_kw)


def config_workload(args):
    """The config's workload, or its sliding-window variant under --swa; --rope
    adds the rotary embedding (the name says so)."""
    import re
    w = CONFIGS[args.config]
    if args.swa:
        w = w.replace(block=1, window=args.swa,
                      name=re.sub(r"block \d+, window \d+", f"sliding window {args.swa} tokens", w.name))
    elif args.block or args.window:
        b, win = args.block or w.block, args.window or w.window
        w = w.replace(block=b, window=win, name=re.sub(r"block \d+, window \d+", f"block {b}, window {win}", w.name))
    if getattr(args, "rope", False):
        w = w.replace(name=w.name + ", rotary q/k")
    if getattr(args, "mx", False):
        if getattr(args, "rope", False) or getattr(args, "gdpa", None):
            raise SystemExit("--mx takes neither --rope nor --gdpa")
        w = w.replace(name=w.name + ", MXFP8 Q/K")
    if getattr(args, "gdpa", None):
        if w.skip_p > 0:
            raise SystemExit("--gdpa takes no skip flags: pick a workload without component skip")
        w = w.replace(name=w.name + f", GDPA {args.gdpa}")
    return w


def tables_for(lens, head_dim):
    """Rotary tables covering the longest example (float32, CPU)."""
    return rope_tables(max(1, int(max(lens, default=1))), head_dim)


def workload(args, rank=0):
    w = config_workload(args)
    inp = make_inputs(w, seed=w.seed + 7919 * rank)
    if args.examples:
        n = min(args.examples, w.batch)
        lens = inp["lengths"][:n].tolist()
        inp = make_inputs(w.replace(batch=n), seed=w.seed + 7919 * rank, lengths=lens)
    return w, inp


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.rows, self.proc, self.t0, self.t1 = [], None, None, None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        window = [r for t, r in self.rows if self.t0 is None or (self.t0 - 0.15 <= t <= (self.t1 or t) + 0.15)]
        for r in window or [r for _, r in self.rows]:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_baseline(w, inp, pairs_total, budget_frac=0.04, tables=None):
    """Times the CPU oracle (as it stands) on the first examples of the batch
    (its rotary form when tables are given)."""
    import oracle
    offs = inp["seq_offsets"].numpy()
    lens = np.diff(offs)
    skip = inp["skip"].numpy() if inp["skip"] is not None else None
    per_ex = [F.visible_pairs([L], w.block, w.window, None if skip is None else [skip[e]])
              for e, L in enumerate(lens)]
    n, acc = 0, 0
    while n < len(lens) and acc < budget_frac * pairs_total:
        acc += per_ex[n]
        n += 1
    n = max(n, 1)
    s1 = int(offs[n])
    f64 = lambda t: t[:s1].to(torch.float64).numpy()
    sub_offs = offs[: n + 1].astype(np.int32)
    sub_skip = skip[:n] if skip is not None else None
    q, k, v, do = f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["dout"])
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    if tables is None:
        oracle.fwd(sub_offs, q, k, v, w.block, w.window, skip=sub_skip, nthreads=threads)
        oracle.bwd(sub_offs, q, k, v, do, w.block, w.window, skip=sub_skip, nthreads=threads)
    else:
        c, s = (t.to(torch.float64).numpy() for t in tables)
        oracle.rope_fwd(sub_offs, q, k, v, c, s, w.block, w.window, skip=sub_skip, nthreads=threads)
        oracle.rope_bwd(sub_offs, q, k, v, do, c, s, w.block, w.window, skip=sub_skip, nthreads=threads)
    dt = time.perf_counter() - t0
    useful = F.step_flops(acc, w.heads, w.head_dim)["step"]
    return {"value": useful / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "cpu": cpu_model(), "kind": "oracle",
            "sample": f"fwd+bwd of the first {n} of {len(lens)} examples ({s1} tokens, all heads, "
                      f"{acc / max(pairs_total, 1):.1%} of the batch's visible pairs), {dt:.1f} s"}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, one bounded sample per step."""
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    import oracle
    w = config_workload(args)
    inp = make_inputs(w)
    offs = inp["seq_offsets"].numpy()
    lens = np.diff(offs)
    skip = inp["skip"].numpy() if inp["skip"] is not None else np.zeros(len(lens), np.uint8)
    live = [e for e in range(len(lens)) if lens[e] > 0 and not skip[e]]
    order = sorted(live, key=lambda e: lens[e])
    threads = oracle.default_threads()
    # one median-length example per step: bounded CPU work per step
    pick = order[len(order) // 2]
    s0, s1 = int(offs[pick]), int(offs[pick + 1])
    f64 = lambda t: t[s0:s1].to(torch.float64).numpy()
    q, k, v, do = f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["dout"])
    sub = np.array([0, s1 - s0], np.int32)
    pairs = F.visible_pairs([s1 - s0], w.block, w.window)
    useful = F.step_flops(pairs, w.heads, w.head_dim)["step"]

    if args.rope:
        c, s = (t.to(torch.float64).numpy() for t in tables_for(lens, w.head_dim))

    def step():
        if args.gdpa:
            from oracle import gdpa
            gdpa.fwd(sub, q, k, v, w.block, w.window, args.gdpa)
            gdpa.bwd(sub, q, k, v, do, w.block, w.window, args.gdpa)
            return
        if args.mx:
            from oracle import mx
            mx.fwd(sub, q, k, v, w.block, w.window, nthreads=threads)
            mx.bwd(sub, q, k, v, do, w.block, w.window, nthreads=threads)
            return
        if args.rope:
            oracle.rope_fwd(sub, q, k, v, c, s, w.block, w.window, nthreads=threads)
            oracle.rope_bwd(sub, q, k, v, do, c, s, w.block, w.window, nthreads=threads)
            return
        oracle.fwd(sub, q, k, v, w.block, w.window, nthreads=threads)
        oracle.bwd(sub, q, k, v, do, w.block, w.window, nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = useful * args.steps / dt / 1e12
    sample = f"fwd+bwd of one example of length {s1 - s0} (all {w.heads} heads) per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "cpu": cpu_model(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def job_totals(flops, tokens, ms, dist=None, device="cpu"):
    """Whole-job aggregate over ranks: useful FLOPs and tokens are summed, the
    time is the slowest rank's (each rank runs its own batch; nothing else is
    exchanged)."""
    totals = torch.tensor([flops, tokens, ms], dtype=torch.float64, device=device)
    if dist is not None:
        mx = totals[2:].clone()
        dist.all_reduce(totals, op=dist.ReduceOp.SUM)
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        totals[2] = mx[0]
    return tuple(float(x) for x in totals.tolist())


KERNEL_NAMES = {"fwd": "fwd_bf16_sm100_kernel", "bwd_dq": "bwd_dq_sm100_kernel",
                "bwd_dkdv": "bwd_dkdv_sm100_kernel"}


def fused_backward(w, rope=False, gdpa=None):
    """Whether ba_bwd runs this workload's backward as one fused pass (dQ, dK and dV)
    after a per-row statistics pass, which then take the dQ and dK/dV profile slots:
    bf16 block attention without rotation, window 1 and a block dividing 128 (every
    128-row query tile sees only its own key tile)."""
    return (w.dtype == torch.bfloat16 and not rope and not gdpa and w.window == 1
            and w.block <= 128 and 128 % w.block == 0)


class Runner:
    """Device buffers and one training step (ba_fwd + ba_bwd, or the rotary
    entry points) of one workload through the library's public API."""

    def __init__(self, ba, w, inp, dev, rope=False, gdpa=None, mx=False):
        self.ba, self.w, self.inp, self.dev, self.rope, self.gdpa, self.mx = ba, w, inp, dev, rope, gdpa, mx
        self.fused = fused_backward(w, rope, gdpa)
        self.kernel_names = dict(KERNEL_NAMES)
        if self.fused:
            self.kernel_names.update(bwd_dq="bwd_stats_kernel", bwd_dkdv="bwd_dkdv_sm100_kernel (fused dQ)")
        self.lens = inp["lengths"].numpy()
        self.skip_np = inp["skip"].numpy() if inp["skip"] is not None else None
        T, H, D = inp["q"].shape
        self.T, self.H, self.D = T, H, D
        self.pairs = F.visible_pairs(self.lens, w.block, w.window, self.skip_np)
        self.flops = F.step_flops(self.pairs, H, D)
        self.bytes = F.step_bytes(T, H, D)
        self.q, self.k, self.v, self.dout = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
        self.offs = inp["seq_offsets"].to(dev)
        self.skip = inp["skip"].to(dev) if inp["skip"] is not None else None
        self.out, self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(4))
        self.lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        self.prob = ba.make_problem(self.q, self.offs)
        self.stream = torch.cuda.current_stream(dev)
        self.tables = None
        if rope:
            self.tables = tables_for(self.lens, D)
            self.cos_d, self.sin_d = (t.to(dev) for t in self.tables)
            self.q_rot, self.k_rot = torch.empty_like(self.q), torch.empty_like(self.k)
            self.rope_arg = ba.make_rope(self.cos_d, self.sin_d, self.q_rot, self.k_rot)
        size_f = (ba.ba_gdpa_workspace_size if gdpa else ba.ba_mx_fwd_workspace_size if mx
                  else ba.ba_fwd_workspace_size)(self.prob, w.block, w.window)
        size_b = (ba.ba_mx_bwd_workspace_size if mx else ba.ba_bwd_workspace_size)(self.prob, w.block, w.window)
        self.ws_f = ba.workspace_for(size_f, dev)
        self.ws_b = ba.workspace_for(size_b, dev)
        # ba_fwd: work list, (skip), attention; ba_bwd: work list, (skip), staging of the partial query
        # tiles, dQ, dK/dV; the rotary forward adds one rotation pass (the backward reads the kept
        # rotated copies)
        self.launches_per_step = (2 + (self.skip is not None)) + (4 + (self.skip is not None)) + (1 if rope else 0)
        if gdpa:
            self.launches_per_step = 6  # work list + forward; work list + staging + dQ + dK/dV
        if mx:  # two quantisation passes in the forward, two round trips in the backward
            self.launches_per_step += 4

    def step(self):
        ba, w, s = self.ba, self.w, self
        if s.gdpa:
            st = ba.ba_gdpa_fwd(s.prob, s.gdpa, s.q, s.k, s.v, s.offs, w.block, w.window, s.out, s.ws_f,
                                stream=s.stream)
            if st != ba.BA_OK:
                raise ba.BAError(st, "ba_gdpa_fwd")
            st = ba.ba_gdpa_bwd(s.prob, s.gdpa, s.q, s.k, s.v, s.dout, s.offs, w.block, w.window, s.dq, s.dk,
                                s.dv, s.ws_f, stream=s.stream)
            if st != ba.BA_OK:
                raise ba.BAError(st, "ba_gdpa_bwd")
            return
        if s.mx:
            st = ba.ba_mx_fwd(s.prob, s.q, s.k, s.v, s.offs, w.block, w.window, s.skip, s.out, s.lse, s.ws_f,
                              stream=s.stream)
            if st != ba.BA_OK:
                raise ba.BAError(st, "ba_mx_fwd")
            st = ba.ba_mx_bwd(s.prob, s.q, s.k, s.v, s.out, s.lse, s.dout, s.offs, w.block, w.window, s.skip,
                              s.dq, s.dk, s.dv, s.ws_b, stream=s.stream)
            if st != ba.BA_OK:
                raise ba.BAError(st, "ba_mx_bwd")
            return
        if s.rope:
            st = ba.ba_rope_fwd(s.prob, s.rope_arg, s.q, s.k, s.v, s.offs, w.block, w.window, s.skip, s.out,
                                s.lse, s.ws_f, stream=s.stream)
        else:
            st = ba.ba_fwd(s.prob, s.q, s.k, s.v, s.offs, w.block, w.window, s.skip, s.out, s.lse, s.ws_f,
                           stream=s.stream)
        if st != ba.BA_OK:
            raise ba.BAError(st, "ba_fwd")
        if s.rope:
            st = ba.ba_rope_bwd(s.prob, s.rope_arg, s.q, s.k, s.v, s.out, s.lse, s.dout, s.offs, w.block,
                                w.window, s.skip, s.dq, s.dk, s.dv, s.ws_b, stream=s.stream)
        else:
            st = ba.ba_bwd(s.prob, s.q, s.k, s.v, s.out, s.lse, s.dout, s.offs, w.block, w.window, s.skip,
                           s.dq, s.dk, s.dv, s.ws_b, stream=s.stream)
        if st != ba.BA_OK:
            raise ba.BAError(st, "ba_bwd")

    def check_status(self, when):
        if self.ba.ba_device_status(self.ws_f) != self.ba.BA_OK or \
                (not self.gdpa and self.ba.ba_device_status(self.ws_b) != self.ba.BA_OK):
            raise RuntimeError(f"a kernel timed out {when}")

    def timed(self, K, warmup, barrier, clocks=None):
        """W warm-up steps, then K steps between two events on the launching
        stream; per-kernel events through ba_set_profile_events. Returns the
        total ms and the mean ms of each attention kernel."""
        ba = self.ba
        for _ in range(warmup):
            self.step()
        barrier()
        self.check_status("during warm-up")
        ev = lambda: torch.cuda.Event(enable_timing=True)
        per = {n: [(ev(), ev()) for _ in range(K)] for n in KERNEL_NAMES}
        for pairs in per.values():  # torch creates the CUDA event on its first record
            for a, b in pairs:
                a.record(self.stream)
                b.record(self.stream)
        t_start, t_stop = ev(), ev()
        if clocks is not None:
            time.sleep(0.3)
        barrier()
        if clocks is not None:
            clocks.mark("t0")
        t_start.record(self.stream)
        for i in range(K):
            for which, n in enumerate(KERNEL_NAMES):
                ba.ba_set_profile_events(which, *per[n][i])
            self.step()
        t_stop.record(self.stream)
        for which in range(3):
            ba.ba_set_profile_events(which)
        barrier()
        if clocks is not None:
            clocks.mark("t1")
        self.check_status("during the timed steps")
        ms_k = {n: statistics.mean(a.elapsed_time(b) for a, b in per[n]) for n in KERNEL_NAMES}
        return t_start.elapsed_time(t_stop), ms_k

    def kernel_stats(self, ms_k):
        # Per kernel, the FLOPs its own tensor-core work does on visible pairs: forward 4 D (S, PV),
        # dQ pass 6 D (S, dP, dQ), dK/dV pass 8 D (S, dP, dV, dK); per visible pair and head. The
        # fused backward does 10 D (S, dP, dV, dK, dQ); its statistics pass none.
        unit = self.pairs * self.H * self.D
        fl = {"fwd": 4 * unit, "bwd_dq": 6 * unit, "bwd_dkdv": 8 * unit}
        if self.fused:
            fl.update(bwd_dq=0, bwd_dkdv=10 * unit)
        return {n: {"kernel": self.kernel_names[n], "ms": ms_k[n], "tflops": fl[n] / (ms_k[n] / 1e3) / 1e12,
                    "flops_per_launch": fl[n]}
                for n in KERNEL_NAMES}


def other_config_line(ba, cfg, dev, K, warmup, local, hbm_gbs, block=None, window=None):
    """One more workload timed like the main one (its own process memory is
    released afterwards); block/window replace the workload's block rule.
    Its ``hbm`` entry sets the step's algorithmic bytes (each input read once,
    each result written once) against the copy bandwidth: the roof of a mask so
    sparse that a step is bound by HBM, not by the tensor cores."""
    w = CONFIGS[cfg]
    if block is not None:
        w = w.replace(block=block, window=window,
                      name=w.name.replace(f"block {w.block}, window {w.window}", f"block {block}, window {window}"))
    inp = make_inputs(w)
    run = Runner(ba, w, inp, dev)
    clocks = ClockSampler(local)
    ms_total, ms_k = run.timed(K, warmup, lambda: torch.cuda.synchronize(dev), clocks)
    clk = clocks.stop()
    ms = ms_total / K
    d = {"workload": w.name, "ms_per_step": ms, "useful_tflops": run.flops["step"] / (ms / 1e3) / 1e12,
         "tokens_per_s": run.T / (ms / 1e3), "total_tokens": int(run.T),
         "visible_pairs_per_head": run.pairs, "useful_flops_per_step": run.flops["step"],
         "steps": K, "warmup": warmup, "kernels": run.kernel_stats(ms_k), "clocks": clk}
    step_bytes = run.bytes["fwd"] + run.bytes["bwd"]
    d["hbm"] = {"algorithmic_bytes_per_step": step_bytes, "achieved_gbs": step_bytes / (ms / 1e3) / 1e9,
                "peak_gbs": hbm_gbs, "frac": step_bytes / (ms / 1e3) / 1e9 / hbm_gbs,
                "floor_ms": step_bytes / (hbm_gbs * 1e9) * 1e3}
    if run.skip_np is not None:
        d["live_tokens"] = F.live_tokens(run.lens, run.skip_np)
        d["skipped_examples"] = int(run.skip_np.sum())
    del run, inp
    torch.cuda.empty_cache()
    return d


def main(argv=None, runner_cls=None):
    """The benchmark. runner_cls replaces Runner (the GPU step) with a stand-in
    of the same interface; it then runs on the CPU with gloo ranks, which is
    how the multi-rank launch and report are tested without a GPU."""
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU, launched here; each rank re-enters main() below
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:] if argv is None else argv).returncode)

    import block_sparse_attention_kunlun_b200 as ba

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    on_gpu = runner_cls is None
    if on_gpu:
        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
    else:
        dev = torch.device("cpu")
    dist = None
    if world > 1:
        import torch.distributed as dist
        if on_gpu:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))

    w, inp = workload(args, rank)
    run = (runner_cls or Runner)(ba, w, inp, dev, rope=args.rope, gdpa=args.gdpa, mx=args.mx)
    T, H, D = run.T, run.H, run.D
    fl, by = run.flops, run.bytes

    def barrier():
        if on_gpu:
            torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()

    K = args.steps
    clocks = ClockSampler(local) if on_gpu else None
    ms_total, ms_k = run.timed(K, args.warmup, barrier, clocks)
    clk = clocks.stop() if clocks is not None else None

    job_flops, job_tokens, ms_max = job_totals(fl["step"] * K, T * K, ms_total, dist, dev)
    value = job_flops / (ms_max / 1e3) / 1e12

    # end to end through the same API: pinned host in, results out. Steps are pipelined over two
    # buffer sets and three streams (the upload of step i+1 and the download of step i-1 overlap
    # step i's kernels); every step's own copies stay inside the timed region.
    e2e = None
    if not args.no_e2e and on_gpu:
        host_in = [inp[n].pin_memory() for n in ("q", "k", "v", "dout")]
        offs_pin = inp["seq_offsets"].pin_memory()
        skip_pin = inp["skip"].pin_memory() if inp["skip"] is not None else None
        host_out = [torch.empty_like(run.out, device="cpu").pin_memory() for _ in range(4)]
        lse_out = torch.empty((H, T), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in) + offs_pin.numel() * 4 + (
            skip_pin.numel() if skip_pin is not None else 0)
        d2h = sum(t.numel() * t.element_size() for t in host_out) + lse_out.numel() * 4
        Ke = max(3, min(K, 10))
        names = ("q", "k", "v", "dout", "offs", "skip", "out", "dq", "dk", "dv", "lse")
        slots = [{n: getattr(run, n) for n in names}]
        slots.append({n: (torch.empty_like(t) if t is not None else None) for n, t in slots[0].items()})
        s_in, s_out, s_comp = torch.cuda.Stream(dev), torch.cuda.Stream(dev), run.stream
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

        def e2e_step(i):
            j, bufs = i % 2, slots[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[j])  # step i-2 is done reading this set's inputs
                for n, src in zip(("q", "k", "v", "dout"), host_in):
                    bufs[n].copy_(src, non_blocking=True)
                bufs["offs"].copy_(offs_pin, non_blocking=True)
                if skip_pin is not None:
                    bufs["skip"].copy_(skip_pin, non_blocking=True)
                ev_in[j].record(s_in)
            s_comp.wait_event(ev_in[j])
            if i >= 2:
                s_comp.wait_event(ev_out[j])  # step i-2's results have left this set's outputs
            for n in names:
                setattr(run, n, bufs[n])
            run.step()
            ev_comp[j].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                for dst, n in zip(host_out, ("out", "dq", "dk", "dv")):
                    dst.copy_(bufs[n], non_blocking=True)
                lse_out.copy_(bufs["lse"], non_blocking=True)
                ev_out[j].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        ev = lambda: torch.cuda.Event(enable_timing=True)
        a, b = ev(), ev()
        a.record(s_in)
        for i in range(2, 2 + Ke):
            e2e_step(i)
        b.record(s_out)  # after the last step's download, which waited for its kernels
        torch.cuda.synchronize(dev)
        barrier()
        for n in names:
            setattr(run, n, slots[0][n])
        ms_e2e = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(ms_e2e, op=dist.ReduceOp.MAX)
        e2e = {"value": (job_flops / K) * Ke / (float(ms_e2e[0]) / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": float(ms_e2e[0]) / Ke, "steps": Ke,
               "pipelining": "two device buffer sets; upload, kernels and download on three streams"}
        del slots
        torch.cuda.empty_cache()

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks, peaks_src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    timed_s = ms_total / 1e3
    # the burst figure for a region shorter than the seconds the sustained figure takes to settle
    long_region = timed_s >= 5.0
    tensor_peak = sustained if long_region else burst
    kstats = run.kernel_stats(ms_k)
    dom = max(kstats, key=lambda n: kstats[n]["ms"])
    traffic = None
    try:
        with open(args.traffic_file) as f:
            tr = json.load(f)
        key = f"{run.kernel_names[dom]}:config{args.config}" + (f":block{w.block}:window{w.window}"
                                                            if (args.swa or args.block or args.window) else "")
        key += ":rope" if args.rope else ""
        key += f":gdpa-{args.gdpa}" if args.gdpa else ""
        key += ":mx" if args.mx else ""
        if key in tr and tr[key].get("kernel_sha") == kernel_sha(dom):
            traffic = tr[key]["bytes_per_launch"]
    except (OSError, ValueError):
        pass
    achieved = kstats[dom]["tflops"]
    flops_launch = kstats[dom]["flops_per_launch"]
    roofline = {"kernel": run.kernel_names[dom], "bound": "tensor", "achieved": achieved, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved / tensor_peak, "traffic": traffic,
                "peak_source": f"{peaks_src} {'bf16_tflops_sustained' if long_region else 'bf16_tflops (burst)'};"
                               f" timed region {timed_s:.2f} s",
                "algorithmic_flops_per_launch": flops_launch,
                "ms_per_launch": kstats[dom]["ms"], "share_of_step": kstats[dom]["ms"] * K / ms_total}
    if traffic:
        # the roof this kernel can reach at its measured arithmetic intensity
        intensity = flops_launch / traffic
        attainable = min(tensor_peak, intensity * hbm / 1e3)
        roofline.update({"intensity_flop_per_byte": intensity, "hbm_peak_gbs": hbm,
                         "attainable": attainable, "frac_of_attainable": achieved / attainable})
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": int(len(run.lens)), "total_tokens": int(T), "heads": H,
                   "head_dim": D, "block": w.block, "window": w.window, "seed": w.seed,
                   "rotary": bool(args.rope), "attention": f"gdpa-{args.gdpa}" if args.gdpa else "softmax",
                   "score_operands": "MXFP8 (E4M3, E8M0 per 32)" if args.mx else "bf16",
                   "visible_pairs_per_head": run.pairs, "useful_flops_per_step": fl["step"],
                   "l2": f"inputs larger than L2 ({by['fwd'] + by['bwd']:.3g} B touched per step), no flush",
                   "parallelism": f"dp{world} (independent batches, no collective in the step)"},
        "tokens_per_s": job_tokens / (ms_max / 1e3),
        "pct_of_bf16_peak": {"burst": value / burst, "sustained": value / sustained, "source": peaks_src},
        "kernels": kstats,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": run.launches_per_step * K,
        "clocks": clk,
    }
    pairs, lens = run.pairs, run.lens
    if world == 1 and on_gpu and not args.examples and not args.no_other_configs and \
            not (args.swa or args.block or args.window or args.rope or args.gdpa or args.mx):
        del run
        torch.cuda.empty_cache()
        Ko = max(5, min(K, 20))
        line["other_configs"] = {f"config{c}": other_config_line(ba, c, dev, Ko, max(3, args.warmup), local, hbm)
                                 for c in (4, 5) if c != args.config}
        # the pages' independent 64-token blocks on the same jagged histories
        line["other_configs"]["config3_block64_window1"] = other_config_line(
            ba, 3, dev, Ko, max(3, args.warmup), local, hbm, block=64, window=1)
    if not args.no_cpu_baseline and world == 1 and on_gpu and not args.gdpa and not args.mx:
        line["cpu_baseline"] = cpu_baseline(w, inp, pairs, tables=tables_for(lens, D) if args.rope else None)
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def kernel_sha(which: str) -> str:
    """Hash of a kernel's source file and the device headers it includes, to tell
    whether stored counters are current."""
    import hashlib
    src = {"fwd": "ba_fwd_sm100.cu", "bwd_dq": "ba_bwd_dq_sm100.cu", "bwd_dkdv": "ba_bwd_dkdv_sm100.cu"}[which]
    h = hashlib.sha256()
    for name in (src, "ba_common.cuh", "ba_ptx.cuh", "ba_sched.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_kunlun_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
