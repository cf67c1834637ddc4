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


# ------------------------------------------------------------------ canaries
# Output buffers of the GPU tests sit between two canary bands: a stray store
# just before or after an output (a wrong row bound, a tail tile written past
# n, a wrong head stride) changes a band, which check_canaries() reports.  The
# band is 4096 elements (8 or 16 KB), so the output keeps 16-byte alignment.
CANARY = 4096


class Guarded:
    """A CUDA tensor of `shape` and `dtype` (bf16 or fp32) inside canary bands."""

    def __init__(self, shape, dtype, fill=float("nan")):
        numel = int(np.prod(shape))
        self.buf = torch.empty(numel + 2 * CANARY, dtype=dtype, device="cuda")
        self.t = self.buf[CANARY:CANARY + numel].view(shape)
        self.t.fill_(fill)
        self._bits = torch.int16 if dtype == torch.bfloat16 else torch.int32
        pattern = torch.arange(CANARY, dtype=torch.int64, device="cuda") * 40503 + 12345
        mod = 1 << (16 if dtype == torch.bfloat16 else 32)
        self._pattern = ((pattern % mod) - mod // 2).to(self._bits)
        bits = self.buf.view(self._bits)
        bits[:CANARY] = self._pattern
        bits[-CANARY:] = self._pattern

    def intact(self) -> bool:
        bits = self.buf.view(self._bits)
        return bool(torch.equal(bits[:CANARY], self._pattern) and torch.equal(bits[-CANARY:], self._pattern))


def check_canaries(*guarded, what=""):
    for i, g in enumerate(guarded):
        assert g.intact(), f"{what}: a store landed outside output buffer {i}"
