"""Benchmark of the static sparse attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mask I] [--mode block|token_exact]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

One step = one ra_attention_fwd call over every batch element and head of the
workload (mask built once beforehand: it is static).  Default workload: the
HunyuanVideo-shaped radial configuration (f=30 frames, s=3600 tokens per
frame, n=108000, 24 heads, d=128), eq. 4 mask at 128x128 tiles, block mode.

Throughput is effective TFLOP/s on kept-pair FLOPs: 4 * d per computed
(query, key) pair per head (2d for Q K^T, 2d for P V); in block mode the
computed pairs are the valid pairs of the kept tiles.  Under torchrun each rank
runs the same workload on its own GPU (its own batch element of a global batch
of N, weak scaling, no collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "radial sparse-attn fwd ms & effective TFLOP/s (bf16, % of TC peak), 1 B200"
L2_BYTES = 126 * 1024 * 1024
ATTN_SOURCES = ["static_sparse_attention_b200/csrc/ra_attention.cu", "static_sparse_attention_b200/csrc/ra_sm100.cuh",
                "static_sparse_attention_b200/csrc/ra_mask_math.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="hunyuan108k", choices=sorted(synth.CONFIGS))
    ap.add_argument("--mask", type=int, default=0, help="index into the workload's mask list")
    ap.add_argument("--mode", default="block", choices=["block", "token_exact"])
    ap.add_argument("--no-dense-ref", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling cases)")
    return ap.parse_args()


def workload_desc(name, mask, mode, c):
    extra = ""
    if mask["family"] == "window3d":
        extra = f", r_t={mask['r_t']}, r_s={mask['r_s']}"
    if mask["family"] == "swc":
        extra = f", W={mask['window_frames']}"
    if mask.get("sink_tokens"):
        extra += f", {mask['sink_tokens']} global (sink) tokens"
    return (f"{name}: {mask['family']} mask{extra}, {mode} mode, f={c['f']}, s={c['s']} "
            f"({c['grid'][0]}x{c['grid'][1]}), n={c['f'] * c['s']}, B={c['B']}, H={c['H']}, d={c['d']}, "
            f"bf16 Q,K,V iid N(0,1)")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            j = json.load(fh)
        return j.get("bf16_tflops"), j.get("bf16_tflops_sustained"), j.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def sources_sha256():
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, mode, mask_family):
    """DRAM bytes per launch of the forward kernel from the committed ncu summary,
    if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    key = f"{workload}/{mask_family}/{mode}"
    m = re.search(rf"^{re.escape(key)}\s+sources=(\w+)\s+dram_bytes_per_launch=(\d+)", text, flags=re.M)
    if not m or m.group(1) != sources_sha256():
        return None
    return int(m.group(2))


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons during the timed region."""

    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [x for x in sm if x >= 0.5 * max(sm)]
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def physical_gpu(dev: int) -> str:
    """nvidia-smi's index (or UUID) of torch's device `dev`."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if parts:
            return parts[dev] if dev < len(parts) else parts[0]
    return str(dev)


def rank_tensor_ids(rank: int):
    """Input streams (Q, K, V) of one rank: its own batch element of the global batch."""
    return (3 * rank, 3 * rank + 1, 3 * rank + 2)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank measurement over all ranks (timing only, outside the timed region)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def flops_per_call(info, c, mode):
    pairs = info["block_pairs"] if mode == "block" else info["kept_pairs"]
    return 4.0 * c["d"] * pairs * c["B"] * c["H"]


def cpu_oracle_sample(name, mask, mode, c, target_s=15.0, seed_rank=0):
    """Time the oracle (as it stands) on a bounded sample of the workload: query
    rows of head 0 until about target_s seconds of CPU work.  Returns
    (TFLOP/s, threads, sample description)."""
    import oracle
    orc = oracle.default()
    spec = oracle.spec_from(mask, c["f"], c["s"], c["grid"])
    n, d = c["f"] * c["s"], c["d"]
    shape = (1, 1, n, d)
    seed = synth.config_seed(name) + 1000 * seed_rank
    Q, K, V = (synth.normal_bf16(seed, t, shape) for t in range(3))
    omode = oracle.BLOCK if mode == "block" else oracle.TOKEN_EXACT
    rows_all = synth.sample_rows(seed, c["f"], c["s"], count=min(n, 4096))
    rng = np.random.default_rng(seed)
    rng.shuffle(rows_all)
    nrows, done_rows, flop, elapsed = 8, 0, 0.0, 0.0
    while elapsed < target_s and done_rows < len(rows_all):
        rows = rows_all[done_rows:done_rows + nrows]
        t0 = time.perf_counter()
        _, _, nk = orc.attention_rows(Q, K, V, spec, omode, 1 / math.sqrt(d), np.zeros(len(rows), np.int64), rows)
        elapsed += time.perf_counter() - t0
        flop += 4.0 * d * float(nk.sum())
        done_rows += len(rows)
        nrows = min(nrows * 2, 1024)
    desc = (f"{done_rows} query rows of head 0 ({'kept tiles in full' if mode == 'block' else 'token-exact keys'}), "
            f"{int(flop / (4 * d))} computed pairs, {elapsed:.1f} s, including the oracle's brute-force tile "
            f"flags of the rows' query tiles")
    return flop / elapsed / 1e12, orc.threads(), desc


def run_reference(args, c, mask):
    """Reference arm: the oracle as it stands on the host cores, K steps of a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    n_steps = args.steps + args.warmup
    per_step = max(1.0, min(8.0, 120.0 / max(n_steps, 1)))
    vals, threads, descs = [], 1, []
    for i in range(n_steps):
        v, threads, desc = cpu_oracle_sample(args.workload, c["masks"][args.mask], args.mode, c, target_s=per_step)
        if i >= args.warmup:
            vals.append(v)
            descs.append(desc)
    value = float(np.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(args.workload, mask, args.mode, c), "mask": mask["family"],
                   "mode": args.mode},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": descs[-1] if descs else ""},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    c = dict(synth.CONFIGS[args.workload])
    if args.heads:
        c["H"] = args.heads
    mask = c["masks"][args.mask]
    if args.impl == "reference":
        run_reference(args, c, mask)
        return

    import torch
    import torch.distributed as dist

    import static_sparse_attention_b200 as ra

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()

    B, H, d = c["B"], c["H"], c["d"]
    n = c["f"] * c["s"]
    shape = (B, H, n, d)
    seed = synth.config_seed(args.workload)
    # This rank's batch element of the global batch: its own input streams.
    host = [synth.normal_bf16(seed, tid, shape) for tid in rank_tensor_ids(rank)]
    q, k, v = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(f"cuda:{dev}") for h in host)
    o = torch.empty_like(q)
    m = ra.build_mask(mask, c["f"], c["s"], c["grid"])
    info = m.info
    flop = flops_per_call(info, c, args.mode)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()
    bytes_qkvo = 4 * q.numel() * 2

    def step():
        ra.attention_fwd(q, k, v, m, scale=scale, mode=args.mode, out=o, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ra.device_status() == ra.RA_OK

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(dev)) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    status = ra.device_status()
    if status != ra.RA_OK:
        raise SystemExit(f"device status {status} after the timed region")
    total_ms = max_over_ranks(total_ms, world, f"cuda:{dev}")
    ms_per_step = total_ms / args.steps
    value = flop * args.steps * world / (total_ms / 1e3) / 1e12
    avg_launch_s = float(np.mean(launch_ms)) / 1e3
    achieved = flop / avg_launch_s / 1e12

    burst, sustained, hbm, peak_src = measured_peaks()
    timed_alone = total_ms < 1000.0
    peak = burst if timed_alone else sustained
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": recorded_traffic(args.workload, args.mode, mask["family"]),
                "peak_source": f"{peak_src} bf16 {'burst' if timed_alone else 'sustained'} (MEASURED_PEAKS.json)"
                if peak_src == "measured" else "fallback 1.59 PFLOP/s burst / 1.4 sustained",
                "kernel": "attn_fwd_kernel<%d>" % d,
                "flop_per_launch": flop,
                "algorithmic_bytes_per_launch": bytes_qkvo}

    # ---- end to end: host buffers through the C ABI (H2D + kernel + D2H per step)
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).pin_memory() for h in host)
        ho = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
        e2e_steps = max(3, min(args.steps, 10))
        for _ in range(2):
            ra.attention_fwd_host(hq, hk, hv, ho, q, k, v, o, m, scale=scale, mode=args.mode, stream=stream)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            ra.attention_fwd_host(hq, hk, hv, ho, q, k, v, o, m, scale=scale, mode=args.mode, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, f"cuda:{dev}")
        e2e = {"value": flop * e2e_steps * world / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms / e2e_steps, "h2d_bytes_per_step": 3 * q.numel() * 2,
               "d2h_bytes_per_step": o.numel() * 2,
               "path": "ra_attention_fwd_host (pinned host Q,K,V -> device, kernel, device -> pinned host O)"}
        del hq, hk, hv, ho

    # ---- the same kernel with the dense mask on the same inputs (reference point)
    dense_ref = None
    if not args.no_dense_ref and mask["family"] != "dense":
        md = ra.build_mask(dict(family="dense"), c["f"], c["s"])
        dflop = flops_per_call(md.info, c, "block")
        for _ in range(2):
            ra.attention_fwd(q, k, v, md, scale=scale, mode="block", out=o, stream=stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dsteps = max(2, min(args.steps, 5))
        d0.record(stream)
        for _ in range(dsteps):
            ra.attention_fwd(q, k, v, md, scale=scale, mode="block", out=o, stream=stream)
        d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / dsteps
        dense_ref = {"ms": dms, "tflops": dflop / (dms / 1e3) / 1e12, "speedup_of_sparse": dms / ms_per_step}
        md.free()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        val, threads, desc = cpu_oracle_sample(args.workload, mask, args.mode, c)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    tile_total = info["nb"] ** 2
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": workload_desc(args.workload, mask, args.mode, c),
            "mask": mask["family"], "mode": args.mode, "global_batch": B * world, "heads": H, "seq_len": n,
            "head_dim": d, "parallelism": f"{world} independent problems (one per GPU), no collective",
            "l2": f"inputs larger than L2: Q+K+V+O = {bytes_qkvo / 1e9:.2f} GB per GPU vs 126 MB L2",
            "kept_tiles": info["nnz"], "tile_sparsity": 1.0 - info["nnz"] / tile_total,
            "token_sparsity": 1.0 - info["kept_pairs"] / float(n) ** 2,
            "flop_definition": "4*d per computed pair per head; block mode computes every valid pair of kept tiles",
        },
        "pct_of_peak": 100.0 * roofline["frac"],
        "roofline": roofline,
        "clocks": clk.summary(),
        "gpu_launches": args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "dense_same_kernel": dense_ref,
        "pages_context": "HunyuanVideo 509 frames: 88.3% sparsity, 3.71x inference speedup; 117 frames: 1.88x "
                         "(end-to-end, hardware not stated on the pages)",
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
