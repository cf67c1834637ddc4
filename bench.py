"""Benchmark of the static sparse attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mask I] [--mode block|token_exact]
    python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

One step = one ra_attention_fwd call over every batch element and head of the
workload (mask built once beforehand: it is static).  With --pass bwd a step is
one ra_attention_bwd call instead (dQ, dK, dV from the forward's O and lse and a
seeded dO), counted at 10 * d FLOP per computed pair per head (the five
products S, dP, dQ, dK, dV; the kernels recompute S and dP in both passes).

Default workload: the largest radial configuration that the metric is quoted
on, 4x-long (f=128 frames, s=3600 tokens per frame, n=460800, 24 heads, d=128),
eq. 4 mask at 128x128 tiles, block mode; --workload hunyuan108k gives the
HunyuanVideo-shaped one (f=30, n=108000).

Throughput is effective TFLOP/s on kept-pair FLOPs: 4 * d per computed
(query, key) pair per head (2d for Q K^T, 2d for P V); in block mode the
computed pairs are the valid pairs of the kept tiles.  Under torchrun the ranks
split the heads of the one problem (each rank builds the static mask itself and
computes its head range; no collective on the data path; strong scaling), or
with --split batch each rank runs its own batch element (weak scaling); the
only collective is the max over ranks of the device time.  Rank 0 prints one
JSON line.
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
METRIC_BWD = "radial sparse-attn bwd ms & effective TFLOP/s (bf16, % of TC peak), 1 B200"
METRIC_STREAM = "SWC streaming step (KV ring cache) ms per frame & effective TFLOP/s (bf16), 1 B200"
METRIC_POLICY = "dense-first schedule: attention ms per denoising step & effective TFLOP/s (bf16), 1 B200"
L2_BYTES = 126 * 1024 * 1024
ATTN_SOURCES = {
    "fwd": ["static_sparse_attention_b200/csrc/ra_attention.cu", "static_sparse_attention_b200/csrc/ra_sm100.cuh",
            "static_sparse_attention_b200/csrc/ra_mask_math.cuh"],
    "bwd": ["static_sparse_attention_b200/csrc/ra_attention_bwd.cu", "static_sparse_attention_b200/csrc/ra_sm100.cuh",
            "static_sparse_attention_b200/csrc/ra_mask_math.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="long460k", choices=sorted(synth.CONFIGS))
    ap.add_argument("--mask", type=int, default=0, help="index into the workload's mask list")
    ap.add_argument("--mode", default="block", choices=["block", "token_exact"])
    ap.add_argument("--no-dense-ref", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling cases)")
    ap.add_argument("--split", default="heads", choices=["heads", "batch"],
                    help="with N > 1 GPUs: split the heads of the one problem over the ranks (strong scaling, "
                         "default) or give each rank its own batch element (weak scaling)")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd", "stream", "policy"],
                    help="time the forward (default), the backward, the streaming SWC step, or a whole "
                         "dense-first denoising schedule of forward calls")
    ap.add_argument("--policy-steps", type=int, default=50, help="denoising steps of the policy schedule")
    ap.add_argument("--policy-blocks", type=int, default=40, help="attention blocks per denoising step")
    ap.add_argument("--dense-steps", type=int, default=12, help="first steps that run every block dense")
    ap.add_argument("--dense-blocks", type=int, default=2, help="first blocks that run dense at every step")
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


def sources_sha256(kind="fwd"):
    h = hashlib.sha256()
    for rel in ATTN_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def mask_key(mask: dict) -> str:
    """The mask part of a traffic record's key: the family, and the number of
    global (sink) tokens when there are any (they change the tiles walked)."""
    key = mask["family"]
    if mask.get("sink_tokens"):
        key += f"+sink{mask['sink_tokens']}"
    return key


def recorded_traffic(workload, mode, mask_family, kind="fwd"):
    """DRAM bytes per launch (per call, for the backward's kernels together) from
    the committed ncu summary, if it was taken on the current kernel sources
    (else None)."""
    path = os.path.join(ROOT, "profiles", f"attn_{kind}_traffic.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    key = f"{workload}/{mask_family}/{mode}"
    m = re.search(rf"^{re.escape(key)}\s+sources=(\w+)\s+dram_bytes_per_launch=(\d+)", text, flags=re.M)
    if not m or m.group(1) != sources_sha256(kind):
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
    """Input streams (Q, K, V) of one rank under the batch split: its own batch
    element of the global batch."""
    return (3 * rank, 3 * rank + 1, 3 * rank + 2)


def head_range(rank: int, world: int, H: int):
    """Heads [h0, h1) of one problem that rank `rank` of `world` computes under the
    head split: contiguous ranges, sizes differing by at most one, covering
    [0, H) exactly once (heads are independent given the shared static mask)."""
    if not 0 <= rank < world or world > H:
        raise ValueError(f"cannot split {H} heads over {world} ranks (rank {rank})")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def rank_inputs(name: str, c: dict, rank: int, world: int, split: str, extra_ids=()):
    """This rank's Q, K, V (and any extra tensor ids) as bf16 bit patterns.
    split == "heads": heads head_range(rank) of the one problem (the same
    tensors on every rank, sliced); split == "batch": the rank's own batch
    element (its own input streams)."""
    B, H, d = c["B"], c["H"], c["d"]
    n = c["f"] * c["s"]
    seed = synth.config_seed(name)
    if split == "heads":
        h0, h1 = head_range(rank, world, H)
        ids = (0, 1, 2) + tuple(extra_ids)
        return [synth.normal_bf16_heads(seed, tid, (B, H, n, d), h0, h1) for tid in ids]
    ids = rank_tensor_ids(rank) + tuple(t + rank for t in extra_ids)
    return [synth.normal_bf16(seed, tid, (B, H, n, d)) for tid in ids]


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank measurement over all ranks (timing only, outside the timed region)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_two_streams(step, n_steps, main_stream):
    """End-to-end timing with two CUDA streams: step i (which enqueues its own
    host-to-device copies, kernels and device-to-host copy on the stream it is
    given) runs on stream i % 2 with its own staging buffers, so one step's
    copies overlap another step's kernels.  Returns the device time in ms from
    before the first step to after the last."""
    import torch
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main_stream)
    for st in streams:
        st.wait_event(e0)
    for i in range(n_steps):
        step(i, streams[i % 2])
    for st in streams:
        ev = torch.cuda.Event()
        ev.record(st)
        main_stream.wait_event(ev)
    e1.record(main_stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def fwd_kernel_name(info, c, mode):
    """The forward kernel instance the library runs for this mask and mode: rows
    averaging fewer than 4096 computed keys keep P as hi + lo (SPLIT_P)."""
    n = c["f"] * c["s"]
    pairs = info["block_pairs"] if mode == "block" else info["kept_pairs"]
    return f"attn_fwd_kernel<{c['d']}, {'true' if pairs < 4096 * n else 'false'}>"


def flops_per_call(info, c, mode, kind="fwd"):
    pairs = info["block_pairs"] if mode == "block" else info["kept_pairs"]
    return (4.0 if kind == "fwd" else 10.0) * c["d"] * pairs * c["B"] * c["H"]


def cpu_oracle_sample(name, mask, mode, c, target_s=15.0, seed_rank=0, kind="fwd", threads=None):
    """Time the oracle (as it stands) on a bounded sample of the workload: query
    rows of head 0 until about target_s seconds of CPU work.  Forward: the
    attention of each row (4 d FLOP per computed pair).  Backward: the dQ of each
    row, which needs its S, O, dP and dQ (8 d FLOP per computed pair).
    Returns (TFLOP/s, threads, sample description)."""
    import oracle
    orc = oracle.default()
    all_threads = orc.threads()
    if threads:
        orc.set_threads(threads)
    spec = oracle.spec_from(mask, c["f"], c["s"], c["grid"])
    n, d = c["f"] * c["s"], c["d"]
    shape = (1, 1, n, d)
    seed = synth.config_seed(name) + 1000 * seed_rank
    Q, K, V = (synth.normal_bf16(seed, t, shape) for t in range(3))
    dO = synth.normal_bf16(seed, synth.DOUT_TENSOR_ID, shape) if kind == "bwd" else None
    omode = oracle.BLOCK if mode == "block" else oracle.TOKEN_EXACT
    per_pair = 4.0 * d if kind == "fwd" else 8.0 * d
    rows_all = synth.sample_rows(seed, c["f"], c["s"], count=min(n, 4096))
    rng = np.random.default_rng(seed)
    rng.shuffle(rows_all)
    nrows, done_rows, flop, elapsed = 8, 0, 0.0, 0.0
    while elapsed < target_s and done_rows < len(rows_all):
        rows = rows_all[done_rows:done_rows + nrows]
        zeros = np.zeros(len(rows), np.int64)
        t0 = time.perf_counter()
        if kind == "fwd":
            _, _, nk = orc.attention_rows(Q, K, V, spec, omode, 1 / math.sqrt(d), zeros, rows)
        else:
            _, nk = orc.attention_bwd_query_rows(Q, K, V, dO, spec, omode, 1 / math.sqrt(d), zeros, rows,
                                                 return_nkeys=True)
        elapsed += time.perf_counter() - t0
        flop += per_pair * float(nk.sum())
        done_rows += len(rows)
        nrows = min(nrows * 2, 1024)
    used = orc.threads()
    if threads:
        orc.set_threads(all_threads)
    what = "attention" if kind == "fwd" else "dQ (with the S, O, dP it needs)"
    desc = (f"{what} of {done_rows} query rows of head 0 "
            f"({'kept tiles in full' if mode == 'block' else 'token-exact keys'}), "
            f"{int(flop / per_pair)} computed pairs, {elapsed:.1f} s, including the oracle's brute-force tile "
            f"flags of the rows' query tiles")
    return flop / elapsed / 1e12, used, desc


def cpu_oracle_extras(name, mask, mode, c, kind="fwd"):
    """The oracle on one core (a short sample of the same rows) and its mask build
    (brute-force tile counts of 8 query tiles, extrapolated to every tile)."""
    import oracle
    orc = oracle.default()
    v1, _, desc1 = cpu_oracle_sample(name, mask, mode, c, target_s=4.0, kind=kind, threads=1)
    spec = oracle.spec_from(mask, c["f"], c["s"], c["grid"])
    nb = spec.nb
    qbs = np.unique(np.linspace(0, nb - 1, num=min(8, nb)).astype(np.int32))
    t0 = time.perf_counter()
    orc.tile_counts(spec, qbs)
    dt = time.perf_counter() - t0
    return {"value_1core": v1, "sample_1core": desc1,
            "mask_build_s_extrapolated": dt * nb / len(qbs),
            "mask_build_sample": f"brute-force tile counts of {len(qbs)} of {nb} query tiles in {dt:.2f} s "
                                 f"on {orc.threads()} threads, scaled to all {nb}"}


def run_reference(args, c, mask):
    """Reference arm: the oracle as it stands on the host cores, K steps of a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    n_steps = args.steps + args.warmup
    per_step = max(1.0, min(8.0, 120.0 / max(n_steps, 1)))
    vals, threads, descs = [], 1, []
    for i in range(n_steps):
        if args.pass_ == "stream":
            v, threads, desc = cpu_oracle_stream_sample(args.workload, c, c["masks"][args.mask]["window_frames"],
                                                        target_s=per_step)
        else:
            v, threads, desc = cpu_oracle_sample(args.workload, c["masks"][args.mask], args.mode, c,
                                                 target_s=per_step, kind="bwd" if args.pass_ == "bwd" else "fwd")
        if i >= args.warmup:
            vals.append(v)
            descs.append(desc)
    value = float(np.median(vals))
    line = {
        "impl": "reference",
        "metric": {"fwd": METRIC, "bwd": METRIC_BWD, "stream": METRIC_STREAM, "policy": METRIC_POLICY}[args.pass_],
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(args.workload, mask, args.mode, c), "mask": mask["family"],
                   "mode": args.mode},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": descs[-1] if descs else ""},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def init_ranks():
    """(world, rank, device): one process per GPU under torchrun (NCCL), else GPU 0."""
    import torch
    import torch.distributed as dist
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
    return world, rank, torch.cuda.current_device()


def cpu_oracle_stream_sample(name, c, W, target_s=15.0):
    """The oracle on sampled query rows of one frame of the sequence under the
    SWC mask (what one streaming step computes for those rows), head 0."""
    import oracle
    orc = oracle.default()
    s, d = c["s"], c["d"]
    f = min(c["f"], W + 2)
    n = f * s
    spec = oracle.MaskSpec(oracle.SWC, f, s, window_frames=W)
    seed = synth.config_seed(name)
    Q, K, V = (synth.normal_bf16(seed, t, (1, 1, n, d)) for t in range(3))
    rng = np.random.default_rng(seed)
    rows_all = (f - 1) * s + rng.permutation(s)
    nrows, done_rows, flop, elapsed = 4, 0, 0.0, 0.0
    while elapsed < target_s and done_rows < len(rows_all):
        rows = rows_all[done_rows:done_rows + nrows]
        t0 = time.perf_counter()
        _, _, nk = orc.attention_rows(Q, K, V, spec, oracle.TOKEN_EXACT, 1 / math.sqrt(d),
                                      np.zeros(len(rows), np.int64), rows)
        elapsed += time.perf_counter() - t0
        flop += 4.0 * d * float(nk.sum())
        done_rows += len(rows)
        nrows = min(nrows * 2, 512)
    desc = (f"{done_rows} query rows of frame {f - 1} (head 0, SWC W={W}, token-exact over the whole "
            f"{f}-frame sequence), {int(flop / (4 * d))} computed pairs, {elapsed:.1f} s")
    return flop / elapsed / 1e12, orc.threads(), desc


def run_stream(args, c, mask, world, rank, dev):
    """One step = one frame through ra_swc_cache_step in steady state (the ring
    holds W frames): its K, V appended (the oldest evicted) and its s queries
    attending to the W * s cached tokens."""
    import torch
    import torch.distributed as dist

    import static_sparse_attention_b200 as ra

    if mask["family"] != "swc":
        raise SystemExit("--pass stream needs an SWC mask (e.g. --workload wan_radial --mask 1)")
    W = mask["window_frames"]
    B, H, d, s = c["B"], c["H"], c["d"], c["s"]
    nfr = W + 4  # distinct frames cycled through (inputs larger than L2)
    seed = synth.config_seed(args.workload)
    host = [synth.normal_bf16(seed, tid, (B, H, nfr * s, d)) for tid in rank_tensor_ids(rank)]
    full = [torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(f"cuda:{dev}") for h in host]
    frames = [[t[:, :, i * s:(i + 1) * s].contiguous() for t in full] for i in range(nfr)]
    del full
    out = torch.empty((B, H, s, d), dtype=torch.bfloat16, device=f"cuda:{dev}")
    cache = ra.SwcCache(B, H, d, s, W)
    stream = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(d)
    counter = [0]

    def step():
        qf, kf, vf = frames[counter[0] % nfr]
        counter[0] += 1
        cache.step(qf, kf, vf, out=out, scale=scale, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(W + args.warmup):  # fill the ring, then warm up in steady state
        step()
    torch.cuda.synchronize()
    assert ra.device_status() == ra.RA_OK
    flop = 4.0 * d * s * (W * s) * B * H
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(physical_gpu(dev)) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    if ra.device_status() != ra.RA_OK:
        raise SystemExit("device status error after the timed region")
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, f"cuda:{dev}")
    ms_per_step = total_ms / args.steps
    value = flop * args.steps * world / (total_ms / 1e3) / 1e12
    achieved = flop / (float(np.mean([a.elapsed_time(b) for a, b in zip(starts, ends)])) / 1e3) / 1e12
    burst, sustained, _, peak_src = measured_peaks()
    peak = burst if total_ms < 1000.0 else sustained

    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (torch.from_numpy(h[:, :, :s].copy().view(np.int16)).view(torch.bfloat16).pin_memory()
                      for h in host)
        # The cache steps stay in order on `stream`; each frame's host-to-device copy
        # runs ahead on a copy stream and its output's copy-out on a third stream,
        # with two staging sets, so that the copies overlap the neighbouring steps.
        ho = [torch.empty((B, H, s, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        stage = [[torch.empty((B, H, s, d), dtype=torch.bfloat16, device=f"cuda:{dev}") for _ in range(4)]
                 for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()

        def run_e2e(n_steps):
            free = [None, None]  # event: the staging set's previous step is fully done
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            h2d.wait_event(e0)
            d2h.wait_event(e0)
            for i in range(n_steps):
                sq, sk, sv, so = stage[i % 2]
                with torch.cuda.stream(h2d):
                    if free[i % 2] is not None:
                        h2d.wait_event(free[i % 2])
                    sq.copy_(hq, non_blocking=True)
                    sk.copy_(hk, non_blocking=True)
                    sv.copy_(hv, non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(h2d)
                stream.wait_event(ready)
                cache.step(sq, sk, sv, out=so, scale=scale, stream=stream)
                computed = torch.cuda.Event()
                computed.record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(computed)
                    ho[i % 2].copy_(so, non_blocking=True)
                    done = torch.cuda.Event()
                    done.record(d2h)
                free[i % 2] = done
            stream.wait_event(free[(n_steps - 1) % 2])
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1)

        e2e_steps = max(4, min(args.steps, 10))
        run_e2e(2)  # warm-up
        barrier()
        e_ms = max_over_ranks(run_e2e(e2e_steps), world, f"cuda:{dev}")
        barrier()
        e2e = {"value": flop * e2e_steps * world / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms / e2e_steps, "h2d_bytes_per_step": 3 * out.numel() * 2,
               "d2h_bytes_per_step": out.numel() * 2,
               "path": "per frame: pinned host Q,K,V -> device (copy stream), ra_swc_cache_step (in order on one "
                       "stream), device -> pinned host O (third stream); two staging sets"}
    cache.free()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        val, threads, desc = cpu_oracle_stream_sample(args.workload, c, W)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}
    ring_bytes = 2 * B * H * W * s * d * 2
    line = {
        "metric": METRIC_STREAM, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": f"{args.workload} frames streamed through the SWC key/value ring cache: s={s}, W={W}, "
                        f"B={B}, H={H}, d={d}, bf16 Q,K,V iid N(0,1), steady state (ring full)",
            "pass": "stream", "frame_tokens": s, "window_frames": W, "cached_tokens": W * s,
            "l2": f"inputs larger than L2: ring K+V = {ring_bytes / 1e9:.2f} GB per GPU vs 126 MB L2",
            "flop_definition": "4*d per (query, cached key) pair per head: s * W * s pairs per head per frame",
            "parallelism": f"{world} independent streams (one per GPU), no collective",
        },
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic(args.workload, "exact", f"swc{W}-stream", "fwd"),
                     "peak_source": f"{peak_src} bf16 {'burst' if total_ms < 1000.0 else 'sustained'}",
                     "kernel": "attn_fwd_kernel<%d> over the ring (plus two 2D copies of the frame's K, V)" % d,
                     "flop_per_launch": flop},
        "clocks": clk.summary(),
        "gpu_launches": args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_policy(args, c, mask, world, rank, dev):
    """A whole denoising schedule of forward calls: at step t and block l the
    dense mask when t < dense_steps or l < dense_blocks, else the workload's
    sparse mask (the dense warm-up of the first steps and the dense first DiT
    blocks).  One timed step = one denoising step (policy_blocks calls); the
    schedule runs policy_steps of them, so --steps is not used; --warmup (at
    least 3) untimed calls of each mask precede the timed region."""
    import torch
    import torch.distributed as dist

    import static_sparse_attention_b200 as ra

    B, H, d = c["B"], c["H"], c["d"]
    n = c["f"] * c["s"]
    shape = (B, H, n, d)
    seed = synth.config_seed(args.workload)
    host = [synth.normal_bf16(seed, tid, shape) for tid in rank_tensor_ids(rank)]
    q, k, v = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(f"cuda:{dev}") for h in host)
    o = torch.empty_like(q)
    sparse = ra.build_mask(mask, c["f"], c["s"], c["grid"])
    dense = ra.build_mask(dict(family="dense"), c["f"], c["s"])
    policy = ra.DenseFirstPolicy(sparse, dense, dense_steps=args.dense_steps, dense_blocks=args.dense_blocks)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()
    T, L = args.policy_steps, args.policy_blocks
    f_sparse = flops_per_call(sparse.info, c, args.mode)
    f_dense = flops_per_call(dense.info, c, "block")

    def call(m):
        ra.attention_fwd(q, k, v, m, scale=scale, mode=args.mode if m is sparse else "block", out=o, stream=stream)

    # warm-up, and per-call times of each mask for the all-dense and all-sparse reference points
    warmup = max(3, args.warmup)
    per_call = {}
    for name, m in (("sparse", sparse), ("dense", dense)):
        for _ in range(warmup):
            call(m)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            call(m)
        e1.record(stream)
        torch.cuda.synchronize()
        per_call[name] = e0.elapsed_time(e1) / 3
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    flop = 0.0
    n_dense = 0
    with ClockSampler(physical_gpu(dev)) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for t in range(T):
            for l in range(L):
                m = policy.mask(t, l)
                n_dense += m is dense
                flop += f_dense if m is dense else f_sparse
                call(m)
        t1.record(stream)
        torch.cuda.synchronize()
    if ra.device_status() != ra.RA_OK:
        raise SystemExit("device status error after the timed region")
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, f"cuda:{dev}")

    # ---- end to end: two denoising steps of the schedule (the first, dense warm-up
    # step and the last one) through ra_attention_fwd_host, every call copying its
    # Q, K, V in from pinned host memory and its O out; consecutive calls on two
    # streams with their own staging buffers
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).pin_memory() for h in host)
        ho = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        dev_sets = [(q, k, v, o), tuple(torch.empty_like(q) for _ in range(4))]
        e_calls = [policy.mask(t, l) for t in sorted({0, T - 1}) for l in range(L)]
        e_flop = sum(f_dense if m is dense else f_sparse for m in e_calls)

        def e2e_call(i, st):
            m = e_calls[i % len(e_calls)]
            dq_, dk_, dv_, do_ = dev_sets[i % 2]
            ra.attention_fwd_host(hq, hk, hv, ho[i % 2], dq_, dk_, dv_, do_, m, scale=scale,
                                  mode=args.mode if m is sparse else "block", stream=st)

        time_two_streams(e2e_call, 2, stream)  # warm-up
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(time_two_streams(e2e_call, len(e_calls), stream), world, f"cuda:{dev}")
        e2e = {"value": e_flop * world / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms / 2, "h2d_bytes_per_step": 3 * q.numel() * 2 * L,
               "d2h_bytes_per_step": o.numel() * 2 * L,
               "path": "two denoising steps of the schedule (the first and the last), every call through "
                       "ra_attention_fwd_host (pinned host Q,K,V -> device, kernel, device -> pinned host O), "
                       "consecutive calls on two streams with their own staging buffers"}
        del hq, hk, hv, ho, dev_sets
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    calls = T * L
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        # the oracle on bounded samples of both masks, combined with the schedule's
        # mix of calls: the time the schedule's FLOP would take at those rates
        v_s, threads, desc_s = cpu_oracle_sample(args.workload, mask, args.mode, c, target_s=8.0)
        v_d, _, desc_d = cpu_oracle_sample(args.workload, dict(family="dense"), "block", c, target_s=8.0)
        cpu_s = (calls - n_dense) * f_sparse / (v_s * 1e12) + n_dense * f_dense / (v_d * 1e12)
        cpu = {"value": flop / cpu_s / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{mask['family']} mask: {desc_s}; dense mask: {desc_d}; combined by the schedule's "
                         f"{calls - n_dense} {mask['family']} and {n_dense} dense calls"}
    all_dense_ms = calls * per_call["dense"]
    burst, sustained, _, peak_src = measured_peaks()
    achieved = flop / (total_ms / 1e3) / 1e12
    line = {
        "metric": METRIC_POLICY, "value": flop * world / (total_ms / 1e3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": T, "warmup": warmup, "ms_per_step": total_ms / T, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": workload_desc(args.workload, mask, args.mode, c),
            "pass": "policy", "policy": f"dense when step < {args.dense_steps} or block < {args.dense_blocks}, "
                                        f"else {mask['family']}",
            "denoising_steps": T, "blocks_per_step": L, "calls": calls, "dense_calls": n_dense,
            "l2": "inputs larger than L2 (Q+K+V+O per call)",
        },
        "schedule_ms": total_ms, "all_dense_schedule_ms_from_per_call": all_dense_ms,
        "speedup_vs_all_dense": all_dense_ms / total_ms,
        "per_call_ms": per_call,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                     "frac": achieved / sustained, "traffic": None,
                     "peak_source": f"{peak_src} bf16 sustained (a schedule of many calls)",
                     "kernel": "attn_fwd_kernel<%d> (sparse and dense calls)" % d, "flop_per_launch": flop / calls},
        "clocks": clk.summary(),
        "gpu_launches": calls,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "pages_context": "first 2 DiT blocks and first 12 denoising steps dense (Radial Attention, sec. 6)",
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

    world, rank, dev = init_ranks()
    if args.pass_ == "stream":
        run_stream(args, c, mask, world, rank, dev)
        return
    if args.pass_ == "policy":
        run_policy(args, c, mask, world, rank, dev)
        return

    bwd = args.pass_ == "bwd"
    split = args.split if world > 1 else "heads"
    # This rank's share of the work: a head range of the one problem (head
    # split), or its own batch element (batch split).  The mask is built
    # locally on every rank: it is static and shared by all heads.
    h0, h1 = head_range(rank, world, c["H"]) if split == "heads" else (0, c["H"])
    c_rank = dict(c, H=h1 - h0)
    B, H, d = c_rank["B"], c_rank["H"], c_rank["d"]
    n = c["f"] * c["s"]
    shape = (B, H, n, d)
    seed = synth.config_seed(args.workload)
    host = rank_inputs(args.workload, c, rank, world, split, (synth.DOUT_TENSOR_ID,) if bwd else ())
    q, k, v = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(f"cuda:{dev}") for h in host[:3])
    o = torch.empty_like(q)
    m = ra.build_mask(mask, c["f"], c["s"], c["grid"])
    info = m.info
    # the mask is static: built once per shape, outside the timed region; timed here on its own
    t_mb = time.perf_counter()
    ra.build_mask(mask, c["f"], c["s"], c["grid"]).free()  # synchronises
    mask_build_ms = (time.perf_counter() - t_mb) * 1e3
    flop = flops_per_call(info, c_rank, args.mode, args.pass_)
    # FLOP of one step of the whole job: the one problem (head split) or one
    # problem per rank (batch split)
    flop_job = flops_per_call(info, c, args.mode, args.pass_) * (1 if split == "heads" else world)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()
    bytes_qkvo = 4 * q.numel() * 2
    launches_per_step = 1

    if bwd:
        # the backward's inputs: this rank's seeded dO, and O and lse from the forward
        do = torch.from_numpy(host[3].view(np.int16)).view(torch.bfloat16).to(f"cuda:{dev}")
        lse = torch.empty((B, H, n), dtype=torch.float32, device=f"cuda:{dev}")
        ra.attention_fwd(q, k, v, m, scale=scale, mode=args.mode, out=o, lse=lse, stream=stream)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        ws = torch.empty((B, H, n), dtype=torch.float32, device=f"cuda:{dev}")
        bytes_qkvo = 8 * q.numel() * 2 + 2 * lse.numel() * 4  # Q K V O dO in, dQ dK dV out, lse in, D
        launches_per_step = 3  # D = rowsum(dO * O), dQ pass, dK / dV pass

        def step():
            ra.attention_bwd(q, k, v, o, do, lse, m, scale=scale, mode=args.mode, dq=dq, dk=dk, dv=dv,
                             workspace=ws, stream=stream)
    else:
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
    value = flop_job * args.steps / (total_ms / 1e3) / 1e12
    avg_launch_s = float(np.mean(launch_ms)) / 1e3
    achieved = flop / avg_launch_s / 1e12

    burst, sustained, hbm, peak_src = measured_peaks()
    timed_alone = total_ms < 1000.0
    peak = burst if timed_alone else sustained
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": recorded_traffic(args.workload, args.mode, mask_key(mask), args.pass_),
                "peak_source": f"{peak_src} bf16 {'burst' if timed_alone else 'sustained'} (MEASURED_PEAKS.json)"
                if peak_src == "measured" else "fallback 1.59 PFLOP/s burst / 1.4 sustained",
                "kernel": fwd_kernel_name(info, c, args.mode) if not bwd else
                ("ra_attention_bwd call: bwd_dot_kernel<%d> + bwd_dq_kernel<%d> + bwd_dkdv_kernel<%d>" % (d, d, d)),
                "flop_per_launch": flop,
                "flop_executed_per_launch": flops_per_call(info, c_rank, "block", args.pass_),
                "algorithmic_bytes_per_launch": bytes_qkvo,
                "algorithmic_gbs": bytes_qkvo / avg_launch_s / 1e9}
    if roofline["traffic"] is not None:
        # the recorded DRAM bytes are per launch over all heads of the workload as
        # configured; heads are independent, so a launch over fewer scales with them
        base = synth.CONFIGS[args.workload]
        traffic = roofline["traffic"] * (c_rank["B"] * c_rank["H"]) / (base["B"] * base["H"])
        roofline["traffic"] = traffic
        roofline["dram_gbs"] = traffic / avg_launch_s / 1e9
        roofline["dram_frac_of_hbm"] = roofline["dram_gbs"] / hbm

    # ---- end to end: host buffers through the C ABI (H2D + kernel + D2H per step)
    e2e = None
    if not args.no_e2e and bwd:
        # per step: pinned host Q, K, V, O, dO, lse -> device, the backward, dQ, dK, dV -> pinned
        # host; consecutive steps on two streams with their own device buffers
        hosts = [torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).pin_memory() for h in host]
        hosts.append(o.cpu().pin_memory())  # O
        hl = lse.cpu().pin_memory()
        houts = [[torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)] for _ in range(2)]
        sets = [dict(ins=[q, k, v, do, o], lse=lse, outs=[dq, dk, dv], ws=ws)]
        sets.append(dict(ins=[torch.empty_like(q) for _ in range(5)], lse=torch.empty_like(lse),
                         outs=[torch.empty_like(q) for _ in range(3)], ws=torch.empty_like(ws)))

        def e2e_step(i, st):
            b_ = sets[i % 2]
            with torch.cuda.stream(st):
                for hsrc, dst in zip(hosts, b_["ins"]):
                    dst.copy_(hsrc, non_blocking=True)
                b_["lse"].copy_(hl, non_blocking=True)
                qi, ki, vi, doi, oi = b_["ins"]
                ra.attention_bwd(qi, ki, vi, oi, doi, b_["lse"], m, scale=scale, mode=args.mode, dq=b_["outs"][0],
                                 dk=b_["outs"][1], dv=b_["outs"][2], workspace=b_["ws"], stream=st)
                for hdst, src in zip(houts[i % 2], b_["outs"]):
                    hdst.copy_(src, non_blocking=True)

        e2e_steps = max(4, min(args.steps, 10))
        time_two_streams(e2e_step, 2, stream)  # warm-up
        barrier()
        e_ms = max_over_ranks(time_two_streams(e2e_step, e2e_steps, stream), world, f"cuda:{dev}")
        barrier()
        e2e = {"value": flop_job * e2e_steps / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms / e2e_steps, "h2d_bytes_per_step": 5 * q.numel() * 2 + lse.numel() * 4,
               "d2h_bytes_per_step": 3 * q.numel() * 2,
               "path": "per step: pinned host Q,K,V,O,dO,lse -> device, ra_attention_bwd, device -> pinned host "
                       "dQ,dK,dV; consecutive steps on two streams with their own device buffers"}
        del hosts, houts, hl, sets
    if not args.no_e2e and not bwd:
        hq, hk, hv = (torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).pin_memory() for h in host)
        ho = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        dev_sets = [(q, k, v, o), tuple(torch.empty_like(q) for _ in range(4))]  # staging per stream
        e2e_steps = max(4, min(args.steps, 10))

        def e2e_step(i, st):
            dq_, dk_, dv_, do_ = dev_sets[i % 2]
            ra.attention_fwd_host(hq, hk, hv, ho[i % 2], dq_, dk_, dv_, do_, m, scale=scale, mode=args.mode,
                                  stream=st)

        time_two_streams(e2e_step, 2, stream)  # warm-up
        barrier()
        e_ms = max_over_ranks(time_two_streams(e2e_step, e2e_steps, stream), world, f"cuda:{dev}")
        barrier()
        e2e = {"value": flop_job * e2e_steps / (e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms / e2e_steps, "h2d_bytes_per_step": 3 * q.numel() * 2,
               "d2h_bytes_per_step": o.numel() * 2,
               "path": "ra_attention_fwd_host per step (pinned host Q,K,V -> device, kernel, device -> pinned "
                       "host O), consecutive steps on two streams with their own staging buffers"}
        del hq, hk, hv, ho, dev_sets

    # ---- the same kernel with the dense mask on the same inputs (reference point)
    dense_ref = None
    if not args.no_dense_ref and mask["family"] != "dense" and not bwd:
        md = ra.build_mask(dict(family="dense"), c["f"], c["s"])
        dflop = flops_per_call(md.info, c_rank, "block")
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
        val, threads, desc = cpu_oracle_sample(args.workload, mask, args.mode, c, kind=args.pass_)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}
        cpu.update(cpu_oracle_extras(args.workload, mask, args.mode, c, kind=args.pass_))

    # the fraction of what the tensor pipe can do at the clock the run actually
    # had: 148 SMs x 8192 dense bf16 FLOP per clock x the median sampled SM clock
    clk = clk.summary()
    if clk.get("sm_mhz"):
        clock_peak = 148 * 8192 * clk["sm_mhz"] * 1e6 / 1e12
        roofline["clock_peak_tflops"] = clock_peak
        roofline["frac_of_clock_peak"] = achieved / clock_peak
    tile_total = info["nb"] ** 2
    line = {
        "metric": METRIC_BWD if bwd else METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if split == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": workload_desc(args.workload, mask, args.mode, c),
            "mask": mask["family"], "mode": args.mode, "pass": args.pass_,
            "global_batch": c["B"] * (world if split == "batch" else 1), "heads": c["H"], "seq_len": n,
            "head_dim": d,
            "parallelism": (f"heads split over {world} GPUs ({H} or fewer heads each, mask built on every rank), "
                            f"no collective on the data path" if split == "heads" and world > 1 else
                            f"{world} independent problems (one per GPU), no collective" if world > 1 else
                            "one GPU"),
            "l2": f"inputs larger than L2: {'Q+K+V+O' if not bwd else 'Q+K+V+O+dO+dQ+dK+dV'} = "
                  f"{bytes_qkvo / 1e9:.2f} GB per GPU vs 126 MB L2",
            "kept_tiles": info["nnz"], "tile_sparsity": 1.0 - info["nnz"] / tile_total,
            "token_sparsity": 1.0 - info["kept_pairs"] / float(n) ** 2,
            "flop_definition": ("4*d" if not bwd else "10*d (S, dP, dQ, dK, dV)") +
                               " per pair per head; block mode counts (and computes) every valid pair of the kept "
                               "tiles; token-exact mode counts the kept pairs, and roofline.flop_executed_per_launch "
                               "the pairs of the kept tiles the kernel executes",
        },
        "launch_ms": {"median": float(np.median(launch_ms)), "min": float(np.min(launch_ms)),
                      "p90": float(np.percentile(launch_ms, 90)), "launches": len(launch_ms)},
        "mask_build_ms": mask_build_ms,
        "pct_of_peak": 100.0 * roofline["frac"],
        "roofline": roofline,
        "clocks": clk,
        "gpu_launches": args.steps * launches_per_step,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "dense_same_kernel": dense_ref,
        "pages_context": "HunyuanVideo 509 frames: 88.3% sparsity, 3.71x inference speedup; 117 frames: 1.88x "
                         "(end-to-end, hardware not stated on the pages)",
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
