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

Multi-GPU (torchrun): every rank runs its own batch (seeded per rank) with
no collective on the data path; the step time is the max over ranks.
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


def parse():
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
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic-file", default=os.path.join(ROOT, "profiles", "traffic.json"),
                    help="per-launch DRAM bytes of the dominant kernel from an ncu capture")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


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
    return {"value": useful / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
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
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
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


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import block_sparse_attention_kunlun_b200 as ba

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w, inp = workload(args, rank)
    offs_h = inp["seq_offsets"]
    lens = inp["lengths"].numpy()
    skip_np = inp["skip"].numpy() if inp["skip"] is not None else None
    T, H, D = inp["q"].shape
    pairs = F.visible_pairs(lens, w.block, w.window, skip_np)
    fl = F.step_flops(pairs, H, D)
    by = F.step_bytes(T, H, D)

    # device buffers
    q, k, v, dout = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    offs = offs_h.to(dev)
    skip = inp["skip"].to(dev) if inp["skip"] is not None else None
    out, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((H, T), dtype=torch.float32, device=dev)
    prob = ba.make_problem(q, offs)
    stream = torch.cuda.current_stream(dev)
    if args.rope:
        tables = tables_for(lens, D)
        cos_d, sin_d = (t.to(dev) for t in tables)
        q_rot, k_rot = torch.empty_like(q), torch.empty_like(k)
        rope = ba.make_rope(cos_d, sin_d, q_rot, k_rot)
        ws_f = ba.workspace_for(ba.ba_fwd_workspace_size(prob, w.block, w.window), dev)
        ws_b = ba.workspace_for(ba.ba_bwd_workspace_size(prob, w.block, w.window), dev)
    else:
        tables = None
        ws_f = ba.workspace_for(ba.ba_fwd_workspace_size(prob, w.block, w.window), dev)
        ws_b = ba.workspace_for(ba.ba_bwd_workspace_size(prob, w.block, w.window), dev)

    def step():
        if args.rope:
            st = ba.ba_rope_fwd(prob, rope, q, k, v, offs, w.block, w.window, skip, out, lse, ws_f, stream=stream)
        else:
            st = ba.ba_fwd(prob, q, k, v, offs, w.block, w.window, skip, out, lse, ws_f, stream=stream)
        if st != ba.BA_OK:
            raise ba.BAError(st, "ba_fwd")
        if args.rope:
            st = ba.ba_rope_bwd(prob, rope, q, k, v, out, lse, dout, offs, w.block, w.window, skip, dq, dk, dv,
                                ws_b, stream=stream)
        else:
            st = ba.ba_bwd(prob, q, k, v, out, lse, dout, offs, w.block, w.window, skip, dq, dk, dv, ws_b,
                           stream=stream)
        if st != ba.BA_OK:
            raise ba.BAError(st, "ba_bwd")

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()

    # ba_fwd: work list, (skip), attention; ba_bwd: work list, (skip), dQ, dK/dV;
    # the rotary forward adds one rotation pass (the backward reads the kept rotated copies;
    # fp32 adds a transposed pass after its backward kernels)
    launches_per_step = (2 + (skip is not None)) + (3 + (skip is not None))
    if args.rope:
        launches_per_step += 1 + (w.dtype == torch.float32)

    for _ in range(args.warmup):
        step()
    barrier()
    if ba.ba_device_status(ws_f) != ba.BA_OK or ba.ba_device_status(ws_b) != ba.BA_OK:
        raise RuntimeError("a kernel timed out during warm-up")

    K = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)
    kf = [(ev(), ev()) for _ in range(K)]
    kq = [(ev(), ev()) for _ in range(K)]
    kb = [(ev(), ev()) for _ in range(K)]
    for pair in kf + kq + kb:  # torch creates the CUDA event on its first record
        for e in pair:
            e.record(stream)
    t_start, t_stop = ev(), ev()
    clocks = ClockSampler(local)
    time.sleep(0.3)
    barrier()
    clocks.mark("t0")
    t_start.record(stream)
    for i in range(K):
        ba.ba_set_profile_events(0, *kf[i])
        ba.ba_set_profile_events(1, *kq[i])
        ba.ba_set_profile_events(2, *kb[i])
        step()
    t_stop.record(stream)
    for which in range(3):
        ba.ba_set_profile_events(which)
    barrier()
    clocks.mark("t1")
    clk = clocks.stop()
    ms_total = t_start.elapsed_time(t_stop)
    ms_fwd_k = statistics.mean(a.elapsed_time(b) for a, b in kf)
    ms_dq_k = statistics.mean(a.elapsed_time(b) for a, b in kq)
    ms_dkv_k = statistics.mean(a.elapsed_time(b) for a, b in kb)
    if ba.ba_device_status(ws_f) != ba.BA_OK or ba.ba_device_status(ws_b) != ba.BA_OK:
        raise RuntimeError("a kernel timed out during the timed steps")

    job_flops, job_tokens, ms_max = job_totals(fl["step"] * K, T * K, ms_total, dist, dev)
    value = job_flops / (ms_max / 1e3) / 1e12

    # end to end through the same API: pinned host in, results out
    e2e = None
    if not args.no_e2e:
        host_in = [inp[n].pin_memory() for n in ("q", "k", "v", "dout")]
        offs_pin = offs_h.pin_memory()
        skip_pin = inp["skip"].pin_memory() if inp["skip"] is not None else None
        host_out = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(4)]
        lse_out = torch.empty((H, T), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host_in) + offs_pin.numel() * 4 + (
            skip_pin.numel() if skip_pin is not None else 0)
        d2h = sum(t.numel() * t.element_size() for t in host_out) + lse_out.numel() * 4
        Ke = max(3, min(K, 10))

        def e2e_step():
            for dst, src in zip((q, k, v, dout), host_in):
                dst.copy_(src, non_blocking=True)
            offs.copy_(offs_pin, non_blocking=True)
            if skip_pin is not None:
                skip.copy_(skip_pin, non_blocking=True)
            step()
            for dst, src in zip(host_out, (out, dq, dk, dv)):
                dst.copy_(src, non_blocking=True)
            lse_out.copy_(lse, non_blocking=True)

        e2e_step()
        barrier()
        a, b = ev(), ev()
        a.record(stream)
        for _ in range(Ke):
            e2e_step()
        b.record(stream)
        barrier()
        ms_e2e = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if dist is not None:
            dist.all_reduce(ms_e2e, op=dist.ReduceOp.MAX)
        e2e = {"value": (job_flops / K) * Ke / (float(ms_e2e[0]) / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": float(ms_e2e[0]) / Ke, "steps": Ke}

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    peaks, peaks_src = load_peaks()
    tensor_peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # Per kernel, the FLOPs its own tensor-core work does on visible pairs: forward 4 D (S, PV),
    # dQ pass 6 D (S, dP, dQ), dK/dV pass 8 D (S, dP, dV, dK); per visible pair and head.
    unit = pairs * H * D
    kern = {"fwd": (4 * unit, ms_fwd_k), "bwd_dq": (6 * unit, ms_dq_k), "bwd_dkdv": (8 * unit, ms_dkv_k)}
    kstats = {n: {"ms": ms, "tflops": f / (ms / 1e3) / 1e12, "flops_per_launch": f} for n, (f, ms) in kern.items()}
    dom = max(kstats, key=lambda n: kstats[n]["ms"])
    names = {"fwd": "fwd_bf16_sm100_kernel", "bwd_dq": "bwd_dq_sm100_kernel", "bwd_dkdv": "bwd_dkdv_sm100_kernel"}
    traffic = None
    try:
        with open(args.traffic_file) as f:
            tr = json.load(f)
        key = f"{names[dom]}:config{args.config}" + (f":block{w.block}:window{w.window}"
                                                       if (args.swa or args.block or args.window) else "")
        key += ":rope" if args.rope else ""
        if key in tr and tr[key].get("kernel_sha") == kernel_sha(dom):
            traffic = tr[key]["bytes_per_launch"]
    except (OSError, ValueError):
        pass
    achieved = kstats[dom]["tflops"]
    roofline = {"kernel": names[dom], "bound": "tensor", "achieved": achieved, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved / tensor_peak, "traffic": traffic,
                "peak_source": f"{peaks_src} bf16_tflops_sustained",
                "algorithmic_flops_per_launch": kstats[dom]["flops_per_launch"],
                "ms_per_launch": kstats[dom]["ms"], "share_of_step": kstats[dom]["ms"] * K / ms_total}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": int(len(lens)), "total_tokens": int(T), "heads": H,
                   "head_dim": D, "block": w.block, "window": w.window, "seed": w.seed,
                   "rotary": bool(args.rope),
                   "visible_pairs_per_head": pairs, "useful_flops_per_step": fl["step"],
                   "l2": f"inputs larger than L2 ({by['fwd'] + by['bwd']:.3g} B touched per step), no flush",
                   "parallelism": f"dp{world} (independent batches, no collective in the step)"},
        "tokens_per_s": job_tokens / (ms_max / 1e3),
        "pct_of_bf16_peak": {"sustained": value / tensor_peak, "burst": value / burst_peak,
                             "source": peaks_src},
        "kernels": kstats,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, inp, pairs, tables=tables)
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def kernel_sha(which: str) -> str:
    """Hash of a kernel's source file and the device headers it includes, to tell
    whether stored counters are current."""
    import hashlib
    src = {"fwd": "ba_fwd_sm100.cu", "bwd_dq": "ba_bwd_dq_sm100.cu", "bwd_dkdv": "ba_bwd_dkdv_sm100.cu"}[which]
    h = hashlib.sha256()
    for name in (src, "ba_common.cuh", "ba_ptx.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_kunlun_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
