"""Helpers for the GPU parity tests: move synthetic host inputs to the device,
run the library through its binding, and compare with the oracle."""
import math

import numpy as np
import pytest
import torch

import synth

# Tolerances of the parity bar: bf16 GPU output vs the fp64 oracle on the same
# bf16-rounded inputs.
MAX_ABS = 1e-2
REL_L2 = 5e-3


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def ra():
    import static_sparse_attention_b200 as lib
    return lib


def to_device(u16: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> CUDA bf16 tensor of the same shape."""
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def gather_rows(O: np.ndarray, row_bh: np.ndarray, row_q: np.ndarray) -> np.ndarray:
    """O [B, H, n, d] -> rows listed as (b*H + h, q)."""
    B, H, n, d = O.shape
    return O.reshape(B * H, n, d)[row_bh, row_q]


def errors(got: np.ndarray, want: np.ndarray):
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-30))
    return max_abs, rel


def assert_close(got, want, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = errors(got, want)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def all_rows(B, H, n):
    return np.repeat(np.arange(B * H), n), np.tile(np.arange(n), B * H)


def sampled_rows(seed, f, s, B, H, count=256):
    """The same seeded rows (boundary rows included) on every (b, h)."""
    rows = synth.sample_rows(seed, f, s, count)
    return np.repeat(np.arange(B * H), len(rows)), np.tile(rows, B * H)


def scale_for(d):
    return 1.0 / math.sqrt(d)
