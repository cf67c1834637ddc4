"""How far the bf16 output is from the oracle's result rounded to bf16, in bf16
units in the last place (an informative statistic of the output rounding: the
parity bar itself is the max-abs / relative-L2 one of tests/test_attention_gpu.py).

Distances are counted along the ordered bf16 values (adjacent representable
numbers are 1 apart, +0 and -0 coincide).  The asserts are loose floors; the
measured fractions are printed (`pytest -s`)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _gpu
from tests.test_attention_gpu import MODES, _run

def bf16_bits_rn(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, rounded to nearest even (via torch)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def ordered(u: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> integers in the order of the values they encode."""
    u = u.astype(np.int64)
    return np.where(u < 0x8000, u, 0x8000 - u)


def ulp_distance(got_bits: np.ndarray, want: np.ndarray) -> np.ndarray:
    return np.abs(ordered(got_bits) - ordered(bf16_bits_rn(want)))


def test_ulp_distance_helpers():
    one = 0x3F80  # 1.0
    assert ulp_distance(np.array([one], np.uint16), np.array([1.0]))[0] == 0
    assert ulp_distance(np.array([one + 1], np.uint16), np.array([1.0]))[0] == 1
    assert ulp_distance(np.array([0x8000], np.uint16), np.array([0.0]))[0] == 0  # -0 vs +0
    # the smallest positive and negative subnormals are 2 apart, with zero between them
    assert ulp_distance(np.array([0x8001], np.uint16), np.array([2.0 ** -133]))[0] == 2


def _distances(orc, spec, Q, K, V, mode, rows=None):
    o, _, _ = _run(spec, Q, K, V, mode)
    B, H, n, d = Q.shape
    row_bh, row_q = rows if rows is not None else _gpu.all_rows(B, H, n)
    want, _, _ = orc.attention_rows(Q, K, V, spec, MODES[mode], _gpu.scale_for(d), row_bh, row_q)
    got_bits = o.view(torch.int16).cpu().numpy().view(np.uint16).reshape(B * H, n, d)[row_bh, row_q]
    return ulp_distance(got_bits, want).ravel()


def _report(what, dist):
    frac = {k: float(np.mean(dist <= k)) for k in (0, 1, 2, 4)}
    print(f"\n{what}: {dist.size} elements; exact {frac[0]:.3f}, <=1 ulp {frac[1]:.3f}, <=2 {frac[2]:.3f}, "
          f"<=4 {frac[4]:.3f}, max {int(dist.max())}")
    return frac


@pytest.mark.gpu
@pytest.mark.parametrize("pv", [1, 2], ids=["bf16P", "splitP"])
@pytest.mark.parametrize("mode", ["token_exact", "block"])
def test_tiny_all_rows(orc, mode, pv):
    _gpu.need_gpu()
    ra = _gpu.ra()
    ra.check(ra.ra_set_pv_precision(pv), "ra_set_pv_precision")
    try:
        c = synth.CONFIGS["tiny_radial"]
        Q, K, V = synth.qkv_bf16("tiny_radial")
        spec = oracle.spec_from(c["masks"][0], c["f"], c["s"])
        frac = _report(f"tiny radial {mode} {'bf16 P' if pv == 1 else 'split P'}",
                       _distances(orc, spec, Q, K, V, mode))
    finally:
        ra.ra_set_pv_precision(ra.RA_PV_AUTO)
    assert frac[1] >= 0.5 and frac[4] >= 0.9


@pytest.mark.gpu
def test_hunyuan108k_sampled_rows(orc):
    """The 108000-token radial workload (2 of its heads; the library picks bf16 P)
    on the seeded rows of each head."""
    _gpu.need_gpu()
    c = synth.CONFIGS["hunyuan108k"]
    Q, K, V = synth.qkv_bf16("hunyuan108k", H=2)
    spec = oracle.spec_from(c["masks"][0], c["f"], c["s"])
    rows = _gpu.sampled_rows(synth.config_seed("hunyuan108k"), c["f"], c["s"], 1, 2)
    frac = _report("hunyuan108k radial block, 2 heads x 256 rows", _distances(orc, spec, Q, K, V, "block", rows))
    assert frac[1] >= 0.5 and frac[4] >= 0.9
