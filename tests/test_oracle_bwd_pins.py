"""Pins of the oracle's backward (dQ, dK, dV) to torch autograd in fp64 (CPU).

torch's scaled_dot_product_attention with an explicit boolean mask, in fp64, is
differentiated by autograd; the oracle writes the chain rule out by hand.  The
masks come from the independent numpy restatements (literal eq. 4, grid
enumerations), not from the oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import BLOCK, DENSE, RADIAL, SWC, TOKEN_EXACT, WINDOW3D, MaskSpec
from tests import _pins
from tests.test_oracle_pins import _literal_mask


def _autograd(Q, K, V, dO, mask, scale):
    q, k, v = (torch.tensor(np.asarray(t, dtype=np.float64), requires_grad=True) for t in (Q, K, V))
    m = torch.from_numpy(mask)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    out.backward(torch.from_numpy(np.asarray(dO, dtype=np.float64)))
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


SPECS = [MaskSpec(RADIAL, 8, 20), MaskSpec(RADIAL, 5, 50), MaskSpec(WINDOW3D, 3, 30, 5, 6, 1, 2),
         MaskSpec(SWC, 7, 19, window_frames=2), MaskSpec(DENSE, 3, 31), MaskSpec(RADIAL, 6, 23, sink_tokens=10)]


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}_sink{s.sink_tokens}")
@pytest.mark.parametrize("mode", [TOKEN_EXACT, BLOCK])
def test_backward_equals_autograd(orc, spec, mode):
    rng = np.random.default_rng(3)
    B, H, d = 1, 2, 16
    Q, K, V, dO = (rng.standard_normal((B, H, spec.n, d)) for _ in range(4))
    lit = _literal_mask(spec)
    if spec.sink_tokens:
        lit = lit.copy()
        lit[:spec.sink_tokens, :] = True
        lit[:, :spec.sink_tokens] = True
    mask = lit if mode == TOKEN_EXACT else _pins.block_mask_from_tiles(_pins.tile_reduce(lit), spec.n)
    scale = 1 / math.sqrt(d)
    got = orc.attention_bwd(Q, K, V, dO, spec, mode, scale)
    want = _autograd(Q, K, V, dO, mask, scale)
    for g, w, name in zip(got, want, ("dQ", "dK", "dV")):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-10, err_msg=name)


def test_backward_bf16_inputs(orc):
    import synth
    spec = MaskSpec(RADIAL, 8, 16)
    d = 32
    Qb, Kb, Vb, dOb = (synth.normal_bf16(11, t, (1, 1, spec.n, d)) for t in range(4))
    got = orc.attention_bwd(Qb, Kb, Vb, dOb, spec, TOKEN_EXACT, 0.2)
    want = _autograd(*(synth.bf16_bits_to_f32(t) for t in (Qb, Kb, Vb, dOb)), _literal_mask(spec), 0.2)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-10)


ROW_SPECS = SPECS + [MaskSpec(RADIAL, 12, 40), MaskSpec(SWC, 5, 90, window_frames=2, sink_tokens=130)]


@pytest.mark.parametrize("spec", ROW_SPECS, ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}_sink{s.sink_tokens}")
@pytest.mark.parametrize("mode", [TOKEN_EXACT, BLOCK])
def test_sampled_row_gradients_equal_autograd(orc, spec, mode):
    """The one-row-at-a-time dQ and the per-key dK / dV (used at sizes too large for
    the whole backward) against autograd on the same rows."""
    rng = np.random.default_rng(5)
    B, H, d = 1, 2, 16
    Q, K, V, dO = (rng.standard_normal((B, H, spec.n, d)) for _ in range(4))
    lit = _literal_mask(spec)
    if spec.sink_tokens:
        lit = lit.copy()
        lit[:spec.sink_tokens, :] = True
        lit[:, :spec.sink_tokens] = True
    mask = lit if mode == TOKEN_EXACT else _pins.block_mask_from_tiles(_pins.tile_reduce(lit), spec.n)
    scale = 1 / math.sqrt(d)
    dQw, dKw, dVw = _autograd(Q, K, V, dO, mask, scale)
    rows = np.unique(np.r_[0, spec.n - 1, rng.integers(0, spec.n, 20)])
    row_bh = np.repeat(np.arange(B * H), len(rows))
    row_q = np.tile(rows, B * H)
    dQ = orc.attention_bwd_query_rows(Q, K, V, dO, spec, mode, scale, row_bh, row_q)
    np.testing.assert_allclose(dQ, dQw.reshape(B * H, spec.n, d)[row_bh, row_q], rtol=0, atol=1e-10)
    for h in range(H):
        dK, dV = orc.attention_bwd_key_rows(Q[0, h], K[0, h], V[0, h], dO[0, h], spec, mode, scale, rows)
        np.testing.assert_allclose(dK, dKw[0, h, rows], rtol=0, atol=1e-10, err_msg="dK")
        np.testing.assert_allclose(dV, dVw[0, h, rows], rtol=0, atol=1e-10, err_msg="dV")
