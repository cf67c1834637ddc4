"""Forward and backward on the random small masks of the CSR test (every family,
f and s drawn at random, ragged tails, global tokens), against the fp64 oracle.

Each case draws its own B, H, d (64 or 128) and mode; the library picks the P
precision as it does for any call.  The forward is compared on every row when
the problem is small and on the seeded rows (boundary rows included) of every
(batch, head) otherwise; the backward on every row of every gradient for the
cases small enough for the oracle's O(n^2 d) pass.  Outputs sit inside canary
bands and start as NaN (tests/_gpu.py)."""
import numpy as np
import pytest

import oracle
import synth
from tests import _gpu
from tests.test_attention_bwd_gpu import _check_full
from tests.test_attention_gpu import _check
from tests.test_mask_gpu import _random_specs

pytestmark = pytest.mark.gpu

SPECS = _random_specs()


def _shape(idx, spec):
    d = (64, 128)[idx % 2]
    B, H = 1 + idx % 2, 1 + (idx // 2) % 3
    return B, H, spec.n, d


@pytest.mark.parametrize("idx", range(len(SPECS)), ids=lambda i: f"{i}_fam{SPECS[i].family}_f{SPECS[i].f}_s{SPECS[i].s}")
def test_forward_random_mask(orc, idx):
    _gpu.need_gpu()
    spec = SPECS[idx]
    B, H, n, d = _shape(idx, spec)
    mode = ("token_exact", "block")[(idx // 3) % 2]
    Q, K, V = (synth.normal_bf16(8000 + idx, t, (B, H, n, d)) for t in range(3))
    rows = None
    if B * H * n > 8192:
        rows = _gpu.sampled_rows(8000 + idx, spec.f, spec.s, B, H, count=256)
    _check(orc, spec, Q, K, V, mode, rows=rows, what=f"random mask {idx} {spec} B={B} H={H} d={d} {mode}")


BWD = [i for i, sp in enumerate(SPECS) if sp.n <= 1500]


@pytest.mark.parametrize("idx", BWD, ids=lambda i: f"{i}_fam{SPECS[i].family}_f{SPECS[i].f}_s{SPECS[i].s}")
def test_backward_random_mask(orc, idx):
    _gpu.need_gpu()
    spec = SPECS[idx]
    B, H, n, d = _shape(idx, spec)
    mode = ("block", "token_exact")[(idx // 3) % 2]
    Qh, Kh, Vh, dOh = (synth.normal_bf16(9000 + idx, t, (B, H, n, d)) for t in (0, 1, 2, synth.DOUT_TENSOR_ID))
    _check_full(orc, spec, Qh, Kh, Vh, dOh, mode, f"random mask {idx} {spec} B={B} H={H} d={d} {mode}")
