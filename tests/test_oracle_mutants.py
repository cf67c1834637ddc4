"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

The copy is edited textually, compiled into a temporary directory and bound
with the same wrapper; the committed oracle is never touched.  (Replacing
w <= s by w < s in the first case of eq. 4 is not listed: at w == s both cases
keep exactly k == l, so that edit does not change the mask.)
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import BLOCK, RADIAL, SWC, TOKEN_EXACT, WINDOW3D, MaskSpec
from tests import _pins

MUTANTS = {
    "drop_second_case_of_eq4": ("if (dist % period == 0 && k == l)", "if (0)"),
    "signed_position_distance": ("if (w <= s && (or_abs(k - l) + 1) * w <= s)", "if (w <= s && ((k - l) + 1) * w <= s)"),
    "strict_band_width": ("if (w <= s && (or_abs(k - l) + 1) * w <= s)", "if (w <= s && (or_abs(k - l) + 1) * w < s)"),
    "floor_instead_of_ceil": ("long long period = (w + s - 1) / s;", "long long period = (w + s) / s;"),
    "log2_of_dist_plus_one": ("or_floor_log2(dist > 1 ? dist : 1)", "or_floor_log2(dist + 1)"),
    "frame_from_modulo": ("return or_radial_kept(q / s, key / s, q % s, key % s, s);",
                          "return or_radial_kept(q / s, key % s, q % s, key / s, s);"),
    "window_strict_w": ("or_abs(wq - wk) <= sp->r_s", "or_abs(wq - wk) < sp->r_s"),
    "window_h_uses_w": ("or_abs(hq - hk) <= sp->r_s", "or_abs(hq - wk) <= sp->r_s"),
    "swc_pseudocode_off_by_one": ("(i - j) <= (long long)sp->window_frames - 1", "(i - j) <= (long long)sp->window_frames"),
    "swc_not_causal": ("return (i - j) >= 0 &&", "return 1 &&"),
    "tile_of_query": ("row[key / OR_TILE] += 1;", "row[q / OR_TILE] += 1;"),
    "full_flag_any": ("(c == OR_TILE * OR_TILE) ? OR_TILE_FULL", "(c > 0) ? OR_TILE_FULL"),
    "dropped_scale": ("x[m] = scale * dot;", "x[m] = dot;"),
    "dropped_normalisation": ("O[r * d + c] = acc[c] / denom;", "O[r * d + c] = acc[c];"),
    "transposed_key_operand": ("or_load(K, dtype, kvbase + key * d + c)", "or_load(K, dtype, kvbase + c * n + key)"),
    "value_of_query_row": ("or_load(V, dtype, kvbase + idx[t] * d + c)", "or_load(V, dtype, kvbase + q * d + c)"),
    "block_tile_of_query": ("[(long long)row_tile_slot[r] * nb + key / OR_TILE]", "[(long long)row_tile_slot[r] * nb + q / OR_TILE]"),
    "lse_without_max": ("lse[r] = mx + log(denom);", "lse[r] = log(denom);"),
    "sink_only_keys": ("if (q < sp->sink_tokens || key < sp->sink_tokens)", "if (key < sp->sink_tokens)"),
    "bwd_dropped_D": ("double dsij = pij * (dpij - Di);", "double dsij = pij * dpij;"),
    "bwd_dK_from_K": ("dK[j * d + c] += scale * dsij * or_load(Q, dtype, i * d + c);",
                      "dK[j * d + c] += scale * dsij * or_load(K, dtype, i * d + c);"),
    "bwd_dV_unweighted": ("dV[j * d + c] += pij * or_load(dO, dtype, i * d + c);",
                          "dV[j * d + c] += or_load(dO, dtype, i * d + c);"),
    "rows_dropped_scale": ("x[m] = dot * scale;", "x[m] = dot;"),
    "rows_transposed_key_operand": ("dot += or_load(Q, dtype, qoff + c) * or_load(K, dtype, koff + c);",
                                    "dot += or_load(Q, dtype, qoff + c) * or_load(K, dtype, kvbase + c * n + key);"),
    "qrows_dropped_D": ("double ds = p * (dp - D);", "double ds = p * dp;"),
    "krows_dV_unweighted": ("dV[r * d + c] += p * or_load(dO, dtype, i * d + c);",
                            "dV[r * d + c] += or_load(dO, dtype, i * d + c);"),
    "krows_lse_of_key": ("double p = exp(scale * dot - lse[i]);", "double p = exp(scale * dot - lse[j]);"),
}


def _build_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / f"lib{name}.so"))
    return oracle.Oracle(oracle.load_library(lib))


def _pins_hold(orc) -> bool:
    """A compact selection of the pins in test_oracle_pins.py; True if all hold."""
    for f, s in [(8, 64), (16, 3), (5, 7), (12, 4)]:
        if not np.array_equal(orc.dense_mask(MaskSpec(RADIAL, f, s)).astype(bool), _pins.radial_mask_literal(f, s)):
            return False
    if not np.array_equal(orc.dense_mask(MaskSpec(WINDOW3D, 3, 30, 5, 6, 1, 2)).astype(bool),
                          _pins.window3d_mask_grid(3, 5, 6, 1, 2)):
        return False
    if not np.array_equal(orc.dense_mask(MaskSpec(SWC, 6, 5, window_frames=2)).astype(bool),
                          _pins.swc_mask_frames(6, 5, 2)):
        return False
    sink_want = _pins.radial_mask_literal(7, 9)
    sink_want[:10, :] = True
    sink_want[:, :10] = True
    if not np.array_equal(orc.dense_mask(MaskSpec(RADIAL, 7, 9, sink_tokens=10)).astype(bool), sink_want):
        return False
    spec = MaskSpec(RADIAL, 11, 100)
    lit = _pins.radial_mask_literal(11, 100)
    counts = _pins.tile_reduce(lit)
    csr = orc.csr(spec)
    rp, ci, cnt, fl = _pins.csr_from_tiles(counts)
    if not (np.array_equal(csr["row_ptr"], rp) and np.array_equal(csr["col_idx"], ci)
            and np.array_equal(csr["count"], cnt) and np.array_equal(csr["flag"], fl)):
        return False
    import torch
    rng = np.random.default_rng(0)
    d = 16
    for spec, lit in [(spec, lit), (MaskSpec(SWC, 9, 130, window_frames=3), _pins.swc_mask_frames(9, 130, 3))]:
        counts = _pins.tile_reduce(lit)
        Q, K, V = (rng.standard_normal((1, 1, spec.n, d)) for _ in range(3))
        rows = np.arange(0, spec.n, 7)
        for mode, mask in [(TOKEN_EXACT, lit), (BLOCK, _pins.block_mask_from_tiles(counts, spec.n))]:
            O, lse, _ = orc.attention_rows(Q, K, V, spec, mode, 0.25, np.zeros_like(rows), rows)
            t = torch.from_numpy
            want = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), attn_mask=t(mask),
                                                                     scale=0.25)[0, 0].numpy()[rows]
            sc = (0.25 * Q[0, 0] @ K[0, 0].T)
            want_lse = torch.logsumexp(t(sc).masked_fill(~t(mask), -math.inf), dim=-1).numpy()[rows]
            if not (np.allclose(O, want, atol=1e-12, rtol=0) and np.allclose(lse, want_lse, atol=1e-12, rtol=0)):
                return False
    # backward against autograd on a small radial case
    bspec = MaskSpec(RADIAL, 6, 10)
    blit = _pins.radial_mask_literal(6, 10)
    Q, K, V, dO = (rng.standard_normal((1, 1, bspec.n, 8)) for _ in range(4))
    got = orc.attention_bwd(Q, K, V, dO, bspec, TOKEN_EXACT, 0.3)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (Q, K, V))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(blit), scale=0.3)
    out.backward(torch.from_numpy(dO))
    grads = (tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())
    for g, w in zip(got, grads):
        if not np.allclose(g, w, atol=1e-10, rtol=0):
            return False
    # the row-at-a-time dQ and key-at-a-time dK, dV on the same case
    rows = np.array([0, 7, 31, bspec.n - 1])
    dq = orc.attention_bwd_query_rows(Q, K, V, dO, bspec, TOKEN_EXACT, 0.3, np.zeros_like(rows), rows)
    dk, dv = orc.attention_bwd_key_rows(Q[0, 0], K[0, 0], V[0, 0], dO[0, 0], bspec, TOKEN_EXACT, 0.3, rows)
    for g, w in zip((dq, dk, dv), grads):
        if not np.allclose(g, w[0, 0, rows], atol=1e-10, rtol=0):
            return False
    return True


def test_unmutated_oracle_passes_compact_pins(orc):
    assert _pins_hold(orc)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    assert not _pins_hold(_build_mutant(tmp_path, name)), f"mutant {name} slipped through the pins"
