"""Seeded synthetic workloads: shapes, mask parameters and i.i.d. N(0,1) inputs.

This module is shared by the tests, the oracle checks and the benchmark.  It
holds none of the attention method's arithmetic: it names the workloads (their
sizes and mask parameters) and draws their random inputs with a counter-based
generator (SplitMix64 + Box-Muller, see synth.c), rounded to bf16 with
round-to-nearest-even.  The same host buffers feed the oracle and the GPU.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libsynth.so")
_lib = None
_lock = threading.Lock()

BASE_SEED = 20261202
MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15

# ---------------------------------------------------------------------------
# Workloads.  Shapes and mask parameters of the five benchmark configurations
# (token index = frame * s + position, position = h * grid_w + w).
# A mask entry is a dict: family in {"dense", "radial", "window3d", "swc"} plus
# r_t / r_s (window3d) or window_frames (swc), and optionally sink_tokens
# (global tokens; 3600 = the first frame of the 108k workload).
# ---------------------------------------------------------------------------
CONFIGS = {
    "tiny_radial": dict(index=0, f=8, s=64, grid=(8, 8), B=1, H=1, d=64,
                        masks=[dict(family="radial"), dict(family="dense")]),
    "window3d_16": dict(index=1, f=16, s=256, grid=(16, 16), B=2, H=12, d=64,
                        masks=[dict(family="window3d", r_t=1, r_s=1),
                               dict(family="window3d", r_t=2, r_s=4)]),
    "wan_radial": dict(index=2, f=41, s=1560, grid=(30, 52), B=1, H=40, d=128,
                       masks=[dict(family="radial"), dict(family="swc", window_frames=16)]),
    "hunyuan108k": dict(index=3, f=30, s=3600, grid=(45, 80), B=1, H=24, d=128,
                        masks=[dict(family="radial"), dict(family="dense"),
                               dict(family="radial", sink_tokens=3600)]),
    "long460k": dict(index=4, f=128, s=3600, grid=(45, 80), B=1, H=24, d=128,
                     masks=[dict(family="radial")]),
}


def config_seed(name: str) -> int:
    return BASE_SEED + CONFIGS[name]["index"]


def build(force: bool = False) -> str:
    """Compile synth.c into _build/libsynth.so (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_void_p]
            lib.synth_normal.restype = None
            lib.synth_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
            lib.synth_round_bf16.restype = None
            _lib = lib
    return _lib


def normal_bf16(seed: int, tensor_id: int, shape, out: np.ndarray | None = None) -> np.ndarray:
    """i.i.d. N(0,1) rounded to bf16, returned as raw uint16 bit patterns."""
    count = int(np.prod(shape))
    if out is None:
        out = np.empty(count, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == count and out.flags.c_contiguous
    _load().synth_normal(seed, tensor_id, 0, count, None, out.ctypes.data)
    return out.reshape(shape)


def normal_bf16_heads(seed: int, tensor_id: int, shape, h0: int, h1: int) -> np.ndarray:
    """Heads [h0, h1) of normal_bf16(seed, tensor_id, shape) for shape [B, H, n, d],
    drawn directly from the counter-based stream (no other element is drawn)."""
    B, H, n, d = shape
    assert 0 <= h0 <= h1 <= H
    out = np.empty((B, h1 - h0, n, d), dtype=np.uint16)
    per_head = n * d
    for b in range(B):
        dst = out[b].reshape(-1)
        _load().synth_normal(seed, tensor_id, (b * H + h0) * per_head, (h1 - h0) * per_head, None,
                             dst.ctypes.data)
    return out


def normal_f32(seed: int, tensor_id: int, shape) -> np.ndarray:
    """The same stream as normal_bf16 before rounding (fp32)."""
    count = int(np.prod(shape))
    out = np.empty(count, dtype=np.float32)
    _load().synth_normal(seed, tensor_id, 0, count, out.ctypes.data, None)
    return out.reshape(shape)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().synth_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (u.astype(np.uint32) << 16).view(np.float32)


def qkv_bf16(name: str, B: int | None = None, H: int | None = None):
    """Q, K, V of a named workload as bf16 bit patterns, shape [B, H, n, d]."""
    c = CONFIGS[name]
    B = c["B"] if B is None else B
    H = c["H"] if H is None else H
    shape = (B, H, c["f"] * c["s"], c["d"])
    seed = config_seed(name)
    return tuple(normal_bf16(seed, t, shape) for t in range(3))


# Stream id of the output gradient dO (the forward inputs use ids 0, 1, 2 per
# rank, so it stays clear of every rank's Q, K, V).
DOUT_TENSOR_ID = 1 << 20


def dout_bf16(name: str, B: int | None = None, H: int | None = None) -> np.ndarray:
    """Output gradient dO of a named workload, i.i.d. N(0,1) bf16 bits, [B, H, n, d]."""
    c = CONFIGS[name]
    B = c["B"] if B is None else B
    H = c["H"] if H is None else H
    return normal_bf16(config_seed(name), DOUT_TENSOR_ID, (B, H, c["f"] * c["s"], c["d"]))


def _mix(z: int) -> int:
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def sample_rows(seed: int, f: int, s: int, count: int = 256, tile: int = 128) -> np.ndarray:
    """Seeded query rows: the boundary rows (first and last row of the sequence,
    of frame 1 and of the last frame, first row of the last 128-row tile) plus
    SplitMix64 draws until `count` distinct rows.  Sorted, int64."""
    n = f * s
    nb = (n + tile - 1) // tile
    rows = {0, n - 1, min(s, n - 1), min(2 * s - 1, n - 1), (f - 1) * s, (nb - 1) * tile}
    count = min(count, n)
    state = _mix((seed ^ 0xA5A5A5A5) & MASK64)
    t = 0
    while len(rows) < count:
        t += 1
        rows.add(_mix((state + t * GAMMA) & MASK64) % n)
    return np.array(sorted(rows), dtype=np.int64)
