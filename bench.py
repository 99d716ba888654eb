#!/usr/bin/env python
"""Benchmark of one video-DiT attention layer's hot path on B200.

A step is one pass of the whole path over one batch of synthetic input
already resident in HBM: fused QK-RMSNorm + 3D RoPE (with the block means
fused in), SubBlock block selection, block-sparse attention.  Default
workload: the 5 s 1344x768 layer (B=1, H=40, d=128, latent grid 31x48x84,
N=124992 tokens, 1953 blocks, sparsity 0.75 -> 489 kept blocks per query
block).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  `value` is the effective attention
throughput of the whole step, 4*N*(64*K)*d*B*H flops (kept blocks only)
divided by the step time, summed over ranks (each rank runs its own replica
of the workload: weak scaling, no collective on the data path).
`--impl reference` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-sparse attn ms/layer & eff. TFLOP/s (% bf16 peak); prologue GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.txt")
ATTN_SRC = os.path.join(ROOT, "block_sparse_attention_qk_b200", "csrc", "attention.cu")
SWEEP = (0.5, 0.75, 0.8, 0.9)
EXTRA_CONFIGS = ("10s", "portrait", "dense")  # timed after the main workload, reported per config


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--no-dit", action="store_true", help="skip the AdaLN / SwiGLU measurement")
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="5s", help="5s, 5s_aggr, 10s, portrait, dense, tiny")
    ap.add_argument("--sparsity", type=float, default=None, help="override the workload's sparsity")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling case)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the other configs (10s, portrait, dense)")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for the CPU baseline")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity for a single process)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int, device=None) -> float:
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(flops_per_step: float, steps: int, elapsed_ms: float, world: int, device=None):
    """Whole-job throughput of a timed region: the slowest rank's elapsed time
    (max over ranks) and the FLOPs all ranks processed.  Returns (max_ms,
    TFLOP/s)."""
    max_ms = reduce_max(elapsed_ms, world, device)
    return max_ms, reduce_sum(flops_per_step, world, device) * steps / (max_ms * 1e-3) / 1e12


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS)


def source_hash(path=ATTN_SRC) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload: str, heads: int):
    """DRAM bytes per attention launch from the committed ncu summary, scaled
    to this workload; None if absent or if the kernel source has changed."""
    rec = {}
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                key, sep, val = line.partition(":")
                if sep and not line.startswith("#"):
                    rec[key.strip()] = val.strip()
    except OSError:
        return None
    if "dram_bytes_per_launch" not in rec or "heads" not in rec:
        return None
    if rec.get("source_sha256_16") != source_hash():
        return None
    if rec.get("workload") != workload:
        return None
    per_head = float(rec["dram_bytes_per_launch"]) / float(rec["heads"])
    return per_head * heads


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.remove(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- CPU oracle

def oracle_sample(wl, x_head: dict, K: int, budget_s: float, rng_seed=0) -> dict:
    """Time the fp64 oracle on a bounded sample of one head of the workload
    and extrapolate to the whole layer by unit counts.

    x_head: CPU tensors q, k, v [B, N, 1, d] of one head and w_q, w_k.
    Units: prologue per (token, head) row; pooling + score matrix per head;
    top-K selection per query block; attention per query block."""
    import numpy as np
    import torch

    from oracle import sbattn_oracle as orc

    f = lambda t: t.to(torch.float64).numpy()
    t0 = time.perf_counter()
    qr, kr = orc.qk_norm_rope(f(x_head["q"]), f(x_head["k"]), f(x_head["w_q"]), f(x_head["w_k"]), wl.T, wl.Hh, wl.W,
                              wl.dims, wl.theta, wl.eps)
    t_pro = time.perf_counter() - t0
    qr16, kr16 = orc.round_to_bf16(qr), orc.round_to_bf16(kr)
    t0 = time.perf_counter()
    s = orc.block_scores(orc.block_pool(qr16), orc.block_pool(kr16))[0, 0]
    t_head = time.perf_counter() - t0
    rng = np.random.default_rng(rng_seed)
    vv = f(x_head["v"])
    n_sel = n_att = 0
    t_sel = t_att = 0.0
    deadline = time.perf_counter() + max(1.0, budget_s - t_pro - t_head)
    while time.perf_counter() < deadline or n_att < 2:
        i = int(rng.integers(0, wl.nblk))
        t0 = time.perf_counter()
        kept = orc.select_row(s[i], i, K)
        t_sel += time.perf_counter() - t0
        n_sel += 1
        t0 = time.perf_counter()
        orc.attention_block(qr16, kr16, vv, kept, 0, 0, i)
        t_att += time.perf_counter() - t0
        n_att += 1
    B, H, N, nblk = wl.B, wl.H, wl.N, wl.nblk
    rows_per_head = B * N
    t_full = (t_pro / rows_per_head) * (B * N * H) + t_head * B * H + (t_sel / n_sel + t_att / n_att) * B * H * nblk
    return {"t_full_s": t_full, "t_sample_s": t_pro + t_head + t_sel + t_att,
            "sample": f"1 head of {B}x{H}: prologue of all {N} tokens, pooling + {nblk}x{nblk} scores, "
                      f"selection + attention of {n_att} random query blocks; extrapolated to "
                      f"{B * H * N} rows / {B * H} heads / {B * H * nblk} query blocks"}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def head_slice_cpu(x: dict, h: int) -> dict:
    return {k: (v[:, :, h:h + 1].cpu().contiguous() if v.dim() == 4 else v.cpu()) for k, v in x.items()}


# -------------------------------------------------------------------- arms

def workload_from_args(args):
    from block_sparse_attention_qk_b200.inputs import WORKLOADS

    wl = WORKLOADS[args.workload]
    if args.sparsity is not None:
        wl = wl.with_sparsity(args.sparsity)
    if args.heads is not None:
        from dataclasses import replace

        wl = replace(wl, H=args.heads)
    return wl


def config_of(wl, K, n_gpus):
    return {"workload": f"{wl.name}: B={wl.B} H={wl.H} d={wl.d} grid {wl.T}x{wl.Hh}x{wl.W} "
                        f"N={wl.N} nblk={wl.nblk} sparsity={wl.sparsity} K={K}",
            "B": wl.B, "H": wl.H, "head_dim": wl.d, "grid": [wl.T, wl.Hh, wl.W], "N": wl.N, "nblk": wl.nblk,
            "sparsity": wl.sparsity, "kept_blocks": K, "kept_fraction": K / wl.nblk,
            "parallelism": f"{n_gpus} independent replicas" if n_gpus > 1 else "single GPU",
            "l2_policy": ("inputs (3 x B*N*H*d bf16) larger than the 126 MB L2; no flush"
                          if 3 * wl.B * wl.N * wl.H * wl.d * 2 > 126e6 else
                          "inputs smaller than the 126 MB L2: timed cache-warm (a test size, not a bench line)")}


def measure_dit_ops(sb, x, wl, dev, peaks, iters=5):
    """The fused elementwise steps either side of attention, at this layer's
    size: AdaLN on the hidden states [B, N, H*d] (the Q input reinterpreted)
    and SwiGLU on [B*N, 13824] (the pages give no MLP width; 13824 is read
    for a 5120-wide SwiGLU block).  HBM-bound: GB/s against the measured copy
    bandwidth.  Not part of the timed step."""
    import torch

    C = wl.H * wl.d
    hid = x["q"].view(wl.B, wl.N, C)
    g = torch.Generator(device=dev).manual_seed(11)
    shift = (torch.randn((wl.B, C), generator=g, device=dev) * 0.5).to(torch.bfloat16)
    scale = (torch.randn((wl.B, C), generator=g, device=dev) * 0.3).to(torch.bfloat16)
    a_out = torch.empty_like(hid)
    F = 13824
    rows = wl.B * wl.N
    gate = torch.randn((rows, F), generator=g, device=dev).to(torch.bfloat16)
    up = torch.randn((rows, F), generator=g, device=dev).to(torch.bfloat16)
    s_out = torch.empty_like(gate)

    def timed(fn):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / iters

    a_ms = timed(lambda: sb.adaln_modulate(hid, shift, scale, out=a_out))
    s_ms = timed(lambda: sb.swiglu(gate, up, out=s_out))
    a_bytes = 2.0 * rows * C * 2 + 2.0 * wl.B * C * 2
    s_bytes = 3.0 * rows * F * 2
    res = {}
    for key, ms, nbytes, shape in (("adaln", a_ms, a_bytes, [wl.B, wl.N, C]), ("swiglu", s_ms, s_bytes, [rows, F])):
        gbps = nbytes / (ms * 1e-3) / 1e9
        res[key] = {"ms": round(ms, 4), "gbps": round(gbps, 1), "frac_of_hbm": round(gbps / peaks["hbm_gbs"], 4),
                    "shape": shape, "bytes": nbytes}
    del gate, up, s_out, a_out
    return res


def time_config(sb, name, dev, peaks, warmup=3, steps=3):
    """Device time of one pass of the path on another config (inputs in HBM,
    CUDA events per kernel on the launching stream): attention ms and TFLOP/s
    with its fraction of the measured sustained bf16 rate, prologue ms and
    GB/s with its fraction of the measured HBM copy rate, selection ms."""
    import torch

    from block_sparse_attention_qk_b200.inputs import WORKLOADS, make_inputs

    wl = WORKLOADS[name]
    x = make_inputs(wl, device=dev)
    layer = sb.AttentionLayer(wl.B, wl.T, wl.Hh, wl.W, wl.H, wl.sparsity, device=dev)
    for _ in range(warmup):
        layer.run_device(x["q"], x["k"], x["v"], x["w_q"], x["w_k"])
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        layer.run_device(x["q"], x["k"], x["v"], x["w_q"], x["w_k"], events=evs[i])
    torch.cuda.synchronize(dev)
    layer.check_status()
    pro = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    sel = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    att = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    step = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    K = layer.K
    flops = sb.attention_flops(wl.B, wl.N, wl.H, K)
    tflops = flops / (att * 1e-3) / 1e12
    pro_bytes = 4.0 * wl.B * wl.N * wl.H * wl.d * 2 + 2.0 * wl.B * wl.H * wl.nblk * wl.d * 4
    gbps = pro_bytes / (pro * 1e-3) / 1e9
    res = {"workload": f"{wl.name}: B={wl.B} H={wl.H} grid {wl.T}x{wl.Hh}x{wl.W} N={wl.N} nblk={wl.nblk} "
                       f"sparsity={wl.sparsity} K={K}",
           "ms_per_step": round(step, 3), "attn_ms": round(att, 3), "attn_tflops": round(tflops, 1),
           "attn_frac_of_sustained_bf16": round(tflops / peaks["bf16_tflops_sustained"], 4),
           "attn_flops": flops, "prologue_ms": round(pro, 4), "prologue_gbps": round(gbps, 1),
           "prologue_frac_of_hbm": round(gbps / peaks["hbm_gbs"], 4), "select_ms": round(sel, 4),
           "timing": f"{warmup} warm-up + {steps} timed passes, CUDA events per kernel"}
    del layer, x
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch

    import block_sparse_attention_qk_b200 as sb
    from block_sparse_attention_qk_b200.inputs import make_inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = workload_from_args(args)
    K = sb.keep_count(wl.nblk, wl.sparsity)
    flops = sb.attention_flops(wl.B, wl.N, wl.H, K)
    x = make_inputs(wl, device=dev)
    layer = sb.AttentionLayer(wl.B, wl.T, wl.Hh, wl.W, wl.H, wl.sparsity, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        layer.run_device(x["q"], x["k"], x["v"], x["w_q"], x["w_k"], events=evs)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    layer.check_status()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    layer.check_status()
    total_ms = t_start.elapsed_time(t_end)
    pro_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    sel_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    att_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    max_ms, value = aggregate(flops, args.steps, total_ms, world, dev)
    ms_step = max_ms / args.steps

    # end to end through the public API with host buffers (pinned), copies in
    # the timed region
    e2e = None
    if not args.no_e2e:
        host = {k: v.cpu().pin_memory() for k, v in x.items()}
        out_host = torch.empty(layer.out.shape, dtype=layer.out.dtype, pin_memory=True)
        for _ in range(2):
            layer(host["q"], host["k"], host["v"], host["w_q"], host["w_k"], out_host=out_host)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            layer(host["q"], host["k"], host["v"], host["w_q"], host["w_k"], out_host=out_host)
        layer.drain()  # the end event follows the last step's device-to-host copy
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms, e2e_value = aggregate(flops, args.steps, e0.elapsed_time(e1), world, dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        e2e = {"value": e2e_value, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms / args.steps, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
               "how": "AttentionLayer with pinned host buffers: every step copies its inputs in and its output "
                      "back; two device slots, copies on their own streams overlap the neighbouring steps' "
                      "compute; timed from before the first copy to after the last"}
        del host, out_host

    # sparsity sweep: kept fraction vs attention latency, same tensors
    sweep = []
    if not args.no_sweep and wl.name in ("5s", "5s_aggr"):
        for s in SWEEP:
            lw = sb.AttentionLayer(wl.B, wl.T, wl.Hh, wl.W, wl.H, s, device=dev)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            times = []
            for it in range(4):
                lw.run_device(x["q"], x["k"], x["v"], x["w_q"], x["w_k"], events=e)
                torch.cuda.synchronize(dev)
                if it:
                    times.append(e[2].elapsed_time(e[3]))
            lw.check_status()
            Ks = lw.K
            a_ms = statistics.mean(times)
            sweep.append({"sparsity": s, "kept_blocks": Ks, "kept_fraction": round(Ks / wl.nblk, 4),
                          "attn_ms": round(a_ms, 3),
                          "attn_tflops": round(sb.attention_flops(wl.B, wl.N, wl.H, Ks) / (a_ms * 1e-3) / 1e12, 1)})
            del lw

    peaks = measured_peaks()
    dit = None if args.no_dit else measure_dit_ops(sb, x, wl, dev, peaks)
    attn_tflops = flops / (att_ms * 1e-3) / 1e12
    pro_bytes = 4.0 * wl.B * wl.N * wl.H * wl.d * 2 + 2.0 * wl.B * wl.H * wl.nblk * wl.d * 4
    sel_bytes = 2.0 * wl.B * wl.H * wl.nblk * wl.d * 4 + wl.B * wl.H * wl.nblk * (K + 1) * 4
    traffic = recorded_traffic(wl.name, wl.H)
    roof = {"bound": "tensor", "achieved": round(attn_tflops, 1), "peak": peaks["bf16_tflops_sustained"],
            "unit": "TFLOP/s", "frac": round(attn_tflops / peaks["bf16_tflops_sustained"], 4),
            "traffic": traffic, "kernel": "attention_kernel",
            "peak_kind": f"{peaks['source']} sustained bf16 (kernel runs back to back inside a long step)",
            "frac_of_burst_peak": round(attn_tflops / peaks["bf16_tflops"], 4),
            "frac_of_2250_nominal": round(attn_tflops / 2250.0, 4)}

    line = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(wl, K, world), "roofline": roof,
            "attn_ms_per_layer": round(att_ms, 3), "attn_tflops": round(attn_tflops, 1),
            "prologue_ms": round(pro_ms, 4), "prologue_gbps": round(pro_bytes / (pro_ms * 1e-3) / 1e9, 1),
            "prologue_frac_of_hbm": round(pro_bytes / (pro_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "select_ms": round(sel_ms, 4), "select_gbps": round(sel_bytes / (sel_ms * 1e-3) / 1e9, 1),
            "gpu_launches": layer.launches_per_call * args.steps, "clocks": clk}
    if e2e is not None:
        line["e2e"] = e2e
    if dit is not None:
        line.update(dit)
    if sweep:
        line["sweep"] = sweep

    xh = head_slice_cpu(x, 0) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if not args.no_configs and wl.name == "5s" and args.heads is None and args.sparsity is None:
        del x, layer
        torch.cuda.empty_cache()
        line["configs"] = {name: time_config(sb, name, dev, peaks) for name in EXTRA_CONFIGS}
    if xh is not None:
        r = oracle_sample(wl, xh, K, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(flops / r["t_full_s"] / 1e12, 6), "unit": "TFLOP/s",
                                "cores": blas_threads(), "kind": "oracle", "sample": r["sample"],
                                "extrapolated_layer_s": round(r["t_full_s"], 1)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_reference(args):
    """The fp64 oracle on the host cores: each step is a bounded sample of the
    workload.  `ms_per_step` is the measured time of a step (the sample);
    `value` is the oracle's throughput on the layer, i.e. the layer's FLOPs
    over the layer time extrapolated from the sample's per-unit rates (also
    printed as `extrapolated_layer_ms`)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch

    import block_sparse_attention_qk_b200.inputs as inputs
    from oracle import sbattn_oracle as orc

    wl = workload_from_args(args)
    K = orc.keep_count(wl.nblk, wl.sparsity)
    flops = 4.0 * wl.B * wl.H * wl.N * (64 * K) * wl.d
    one = inputs.Workload(wl.name, B=wl.B, H=1, T=wl.T, Hh=wl.Hh, W=wl.W, sparsity=wl.sparsity, seed=wl.seed)
    xh = inputs.make_inputs(one)  # one head's worth of the same recipe, on the CPU
    budget = max(2.0, min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, xh, K, budget)
    t_full, t_step = [], []
    sample = ""
    for i in range(args.steps):
        t0 = time.perf_counter()
        r = oracle_sample(wl, xh, K, budget, rng_seed=i)
        t_step.append(time.perf_counter() - t0)
        t_full.append(r["t_full_s"])
        sample = r["sample"]
    t = statistics.mean(t_full)
    value = flops / t / 1e12
    line = {"metric": METRIC, "impl": "reference", "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(statistics.mean(t_step) * 1e3, 1),
            "extrapolated_layer_ms": round(t * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, K, world),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample, "extrapolated_layer_s": round(t, 1)},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    del torch
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
