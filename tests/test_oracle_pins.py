"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each pin is chosen so that a plausible slip in the oracle (a dropped term of
eq. 4, a wrong comparison, a wrong index, a dropped scale or normalisation, a
transposed operand) fails at least one of them; test_oracle_mutants.py plants
such slips in a copy of the oracle and checks that they are caught.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import BLOCK, DENSE, RADIAL, SWC, TOKEN_EXACT, WINDOW3D, MaskSpec
from tests import _pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- eq. 4 mask

@pytest.mark.parametrize("f", range(1, 17))
def test_radial_mask_equals_literal_eq4(orc, f):
    """Integer eq. 4 in the oracle == eq. 4 transcribed with float log2/floor/ceil."""
    for s in range(1, 33):
        spec = MaskSpec(RADIAL, f, s)
        got = orc.dense_mask(spec).astype(bool)
        want = _pins.radial_mask_literal(f, s)
        assert np.array_equal(got, want), (f, s)


@pytest.mark.parametrize("f,s", [(8, 64), (13, 7), (16, 5), (9, 32), (33, 3)])
def test_radial_mask_symmetries(orc, f, s):
    """eq. 4 depends on |i-j| and |k-l| only: symmetric in (i,j) and in (k,l)."""
    m = orc.dense_mask(MaskSpec(RADIAL, f, s)).reshape(f, s, f, s)  # [i, k, j, l]
    assert np.array_equal(m, m.transpose(2, 1, 0, 3))  # swap i and j
    assert np.array_equal(m, m.transpose(0, 3, 2, 1))  # swap k and l


@pytest.mark.parametrize("f,s", [(8, 64), (1, 5), (2, 1), (17, 3), (30, 36), (41, 20), (64, 16), (100, 9)])
def test_radial_total_matches_closed_form(orc, f, s):
    assert orc.kept_total(MaskSpec(RADIAL, f, s)) == _pins.radial_closed_form_total(f, s)


def test_radial_tiny_config_total(orc):
    # 8 frames x 64 tokens: band counts 64^2 (D=0), 64^2 (D=1), 64*127-63*32 (D=2,3: m=31), ...
    assert orc.kept_total(MaskSpec(RADIAL, 8, 64)) == _pins.radial_closed_form_total(8, 64) == 191872


@pytest.mark.parametrize("s", [1, 2, 3, 4, 7, 8, 16, 64, 100, 128])
def test_radial_zero_count_bound_eq56(orc, s):
    """eq. 5-6: the number of kept entries is at most 4 s^2 f floor(log2 f) for f >= 2.
    At f = 1 the printed bound is 0 while s^2 entries are kept: the bound does not
    cover one frame (reported here, not fixed)."""
    for f in range(2, 40):
        kept = orc.kept_total(MaskSpec(RADIAL, f, s)) if f * s <= 1200 else _pins.radial_closed_form_total(f, s)
        assert kept <= 4 * s * s * f * int(math.floor(math.log2(f))), (f, s)
    one_frame = orc.kept_total(MaskSpec(RADIAL, 1, s))
    assert one_frame == s * s and 4 * s * s * 1 * 0 == 0 < one_frame


def test_radial_bound_large_shapes_closed_form():
    for f, s in [(30, 3600), (41, 1560), (128, 3600)]:
        assert _pins.radial_closed_form_total(f, s) <= 4 * s * s * f * int(math.floor(math.log2(f)))


# Totals of eq. 4 on the three large radial shapes, per head (Radial Attention,
# eq. 4 at the 128 x 128 tiles of sec. 6): kept pairs, kept tiles, FULL tiles,
# fewest and most kept tiles in a query-tile row.
LARGE_RADIAL = {
    (41, 1560): (1322566560, 117526, 48791, 140, 268),      # Wan-shaped
    (30, 3600): (4547300400, 321300, 233963, 212, 464),     # HunyuanVideo-shaped, 108000 tokens
    (128, 3600): (31997441936, 2818574, 1251414, 466, 880),  # 4x long, 460800 tokens
}


@pytest.mark.parametrize("f,s", sorted(LARGE_RADIAL))
def test_radial_large_shape_literal_totals(f, s):
    """The literal totals from the band closed form (kept pairs) and from the
    per-frame-pair interval enumeration (tiles)."""
    kept, nnz, full, rmin, rmax = LARGE_RADIAL[(f, s)]
    assert _pins.radial_closed_form_total(f, s) == kept
    rows, fulls = _pins.radial_tile_stats_intervals(f, s)
    lengths = [len(r) for r in rows]
    assert (sum(lengths), sum(map(len, fulls)), min(lengths), max(lengths)) == (nnz, full, rmin, rmax)


def test_radial_wan_oracle_tiles_equal_literal_totals(orc):
    """The oracle's brute-force tile counts of the whole Wan-shaped mask: the
    literal totals, and the interval enumeration's kept and FULL tiles row by row."""
    f, s = 41, 1560
    kept, nnz, full, rmin, rmax = LARGE_RADIAL[(f, s)]
    counts = orc.tile_counts(MaskSpec(RADIAL, f, s))
    per_row = (counts > 0).sum(axis=1)
    assert (int(counts.sum()), int((counts > 0).sum()), int((counts == 128 * 128).sum())) == (kept, nnz, full)
    assert (int(per_row.min()), int(per_row.max())) == (rmin, rmax)
    rows, fulls = _pins.radial_tile_stats_intervals(f, s)
    for qb in range(counts.shape[0]):
        assert np.array_equal(np.flatnonzero(counts[qb] > 0), rows[qb]), qb
        assert np.array_equal(np.flatnonzero(counts[qb] == 128 * 128), fulls[qb]), qb


def test_radial_long_oracle_tiles_equal_intervals_on_sampled_rows(orc):
    """460800 tokens: the oracle's brute-force tile counts of 16 query tiles
    (first, last, frame boundaries, seeded) equal the interval enumeration whose
    totals are pinned above."""
    f, s = 128, 3600
    nb = f * s // 128
    rng = np.random.default_rng(460800)
    qbs = np.unique(np.r_[0, nb - 1, 28, 29, 1799, 1800, rng.integers(0, nb, 10)]).astype(np.int32)
    counts = orc.tile_counts(MaskSpec(RADIAL, f, s), qbs)
    rows, fulls = _pins.radial_tile_stats_intervals(f, s)
    for r, qb in enumerate(qbs):
        assert np.array_equal(np.flatnonzero(counts[r] > 0), rows[qb]), qb
        assert np.array_equal(np.flatnonzero(counts[r] == 128 * 128), fulls[qb]), qb


# ------------------------------------------------------------ other families

def test_window3d_counts_printed_on_tutorial(orc):
    cases = json.load(open(os.path.join(GOLDEN, "window3d_neighbour_counts.json")))["cases"]
    T = H = W = 7
    centre = 3 * H * W + 3 * W + 3
    for c in cases:
        spec = MaskSpec(WINDOW3D, T, H * W, H, W, c["r_t"], c["r_s"])
        kept = sum(orc.kept(spec, centre, key) for key in range(spec.n))
        assert kept == c["kept_including_self"], c


@pytest.mark.parametrize("T,H,W,r_t,r_s", [(4, 8, 8, 1, 1), (5, 3, 7, 2, 1), (3, 6, 5, 0, 2), (6, 4, 4, 2, 4), (2, 1, 9, 1, 3)])
def test_window3d_matches_grid_enumeration(orc, T, H, W, r_t, r_s):
    spec = MaskSpec(WINDOW3D, T, H * W, H, W, r_t, r_s)
    assert np.array_equal(orc.dense_mask(spec).astype(bool), _pins.window3d_mask_grid(T, H, W, r_t, r_s))


@pytest.mark.parametrize("f,s,W", [(8, 16, 3), (20, 5, 16), (5, 7, 1), (12, 3, 12), (4, 9, 40)])
def test_swc_matches_prose_interval(orc, f, s, W):
    spec = MaskSpec(SWC, f, s, window_frames=W)
    assert np.array_equal(orc.dense_mask(spec).astype(bool), _pins.swc_mask_frames(f, s, W))


def test_swc_pseudocode_variant_is_one_frame_wider(orc):
    """The page's pseudocode keeps q - kv <= W, i.e. W + 1 frames: window_frames = W + 1."""
    f, s, W = 10, 4, 3
    fr = np.repeat(np.arange(f), s)
    pseudo = (fr[:, None] >= fr[None, :]) & ((fr[:, None] - fr[None, :]) <= W)
    assert np.array_equal(orc.dense_mask(MaskSpec(SWC, f, s, window_frames=W + 1)).astype(bool), pseudo)


def test_dense_family_keeps_everything(orc):
    assert orc.dense_mask(MaskSpec(DENSE, 3, 5)).all()


@pytest.mark.parametrize("base,sink", [
    (MaskSpec(RADIAL, 9, 20), 1), (MaskSpec(RADIAL, 12, 7), 20), (MaskSpec(SWC, 8, 11, window_frames=2), 11),
    (MaskSpec(WINDOW3D, 4, 12, 3, 4, 1, 1), 5), (MaskSpec(RADIAL, 5, 9), 45)])
def test_sink_tokens_are_global(orc, base, sink):
    """Global tokens: kept in every row and every column, on top of the family."""
    import dataclasses
    spec = dataclasses.replace(base, sink_tokens=sink)
    want = _literal_mask(base).copy()
    want[:sink, :] = True
    want[:, :sink] = True
    assert np.array_equal(orc.dense_mask(spec).astype(bool), want)


# ------------------------------------------------------------------ tiles/CSR

def _literal_mask(spec: MaskSpec) -> np.ndarray:
    if spec.family == RADIAL:
        return _pins.radial_mask_literal(spec.f, spec.s)
    if spec.family == WINDOW3D:
        return _pins.window3d_mask_grid(spec.f, spec.grid_h, spec.grid_w, spec.r_t, spec.r_s)
    if spec.family == SWC:
        return _pins.swc_mask_frames(spec.f, spec.s, spec.window_frames)
    return np.ones((spec.n, spec.n), dtype=bool)


TILE_SPECS = [
    MaskSpec(RADIAL, 8, 64),            # tiny config: n = 512, every tile kept
    MaskSpec(RADIAL, 11, 100),          # n = 1100: tiles straddle frames, ragged tail of 76
    MaskSpec(RADIAL, 40, 37),           # many frames per tile, sub-sampled diagonals
    MaskSpec(RADIAL, 3, 300),           # n = 900
    MaskSpec(WINDOW3D, 6, 256, 16, 16, 1, 1),
    MaskSpec(WINDOW3D, 5, 99, 9, 11, 2, 4),
    MaskSpec(SWC, 9, 130, window_frames=3),
    MaskSpec(DENSE, 5, 77),
    MaskSpec(RADIAL, 1, 100),           # n < 128: one ragged tile
]


@pytest.mark.parametrize("spec", TILE_SPECS, ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}")
def test_tile_counts_and_csr_match_numpy(orc, spec):
    want_counts = _pins.tile_reduce(_literal_mask(spec))
    got_counts = orc.tile_counts(spec)
    assert np.array_equal(got_counts, want_counts)
    csr = orc.csr(spec)
    rp, ci, cnt, fl = _pins.csr_from_tiles(want_counts)
    assert np.array_equal(csr["row_ptr"], rp)
    assert np.array_equal(csr["col_idx"], ci)
    assert np.array_equal(csr["count"], cnt)
    assert np.array_equal(csr["flag"], fl)


def test_tile_counts_subset_rows(orc):
    spec = MaskSpec(RADIAL, 11, 100)
    full = orc.tile_counts(spec)
    qbs = np.array([8, 0, 3], dtype=np.int32)
    assert np.array_equal(orc.tile_counts(spec, qbs), full[qbs])


# ------------------------------------------------------------------ attention

def _sdpa_rows(Q, K, V, mask_bool, scale):
    """torch scaled_dot_product_attention in fp64 with an explicit boolean mask."""
    q, k, v = (torch.from_numpy(np.asarray(t, dtype=np.float64)) for t in (Q, K, V))
    m = None if mask_bool is None else torch.from_numpy(mask_bool)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale).numpy()


def _all_rows(B, H, n):
    bh = np.repeat(np.arange(B * H), n)
    q = np.tile(np.arange(n), B * H)
    return bh, q


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_attention_dense_equals_sdpa(orc):
    B, H, f, s, d = 2, 3, 5, 40, 32
    Q, K, V = (_rand((B, H, f * s, d), 10 + t) for t in range(3))
    spec = MaskSpec(DENSE, f, s)
    bh, q = _all_rows(B, H, spec.n)
    O, lse, nk = orc.attention_rows(Q, K, V, spec, TOKEN_EXACT, 1 / math.sqrt(d), bh, q)
    want = _sdpa_rows(Q, K, V, None, 1 / math.sqrt(d)).reshape(-1, d)
    np.testing.assert_allclose(O, want, rtol=0, atol=1e-12)
    assert (nk == spec.n).all()
    scores = np.einsum("bhqc,bhkc->bhqk", Q, K) / math.sqrt(d)
    want_lse = torch.logsumexp(torch.from_numpy(scores), dim=-1).numpy().reshape(-1)
    np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("spec", [MaskSpec(RADIAL, 8, 64), MaskSpec(RADIAL, 11, 100), MaskSpec(RADIAL, 40, 9),
                                  MaskSpec(WINDOW3D, 4, 64, 8, 8, 1, 1), MaskSpec(SWC, 9, 30, window_frames=3)],
                         ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}")
@pytest.mark.parametrize("mode", [TOKEN_EXACT, BLOCK])
def test_attention_masked_equals_sdpa(orc, spec, mode):
    """eq. 2 with M from the literal mask (token-exact) or its kept tiles (block)."""
    B, H, d = 1, 2, 64
    Q, K, V = (_rand((B, H, spec.n, d), 20 + t) for t in range(3))
    lit = _literal_mask(spec)
    mask = lit if mode == TOKEN_EXACT else _pins.block_mask_from_tiles(_pins.tile_reduce(lit), spec.n)
    bh, q = _all_rows(B, H, spec.n)
    scale = 1 / math.sqrt(d)
    O, lse, nk = orc.attention_rows(Q, K, V, spec, mode, scale, bh, q)
    want = _sdpa_rows(Q, K, V, mask, scale).reshape(-1, d)
    np.testing.assert_allclose(O, want, rtol=0, atol=1e-12)
    assert np.array_equal(nk, np.tile(mask.sum(axis=1), B * H))


def test_attention_bf16_inputs_widen_exactly(orc):
    """bf16 bit patterns are read as the exact fp32 values they encode."""
    import synth
    spec = MaskSpec(RADIAL, 8, 64)
    d = 64
    Qb, Kb, Vb = (synth.normal_bf16(5, t, (1, 1, spec.n, d)) for t in range(3))
    Qf, Kf, Vf = (synth.bf16_bits_to_f32(t) for t in (Qb, Kb, Vb))
    bh, q = _all_rows(1, 1, spec.n)
    Ob, _, _ = orc.attention_rows(Qb, Kb, Vb, spec, TOKEN_EXACT, 0.125, bh, q)
    want = _sdpa_rows(Qf, Kf, Vf, _literal_mask(spec), 0.125).reshape(-1, d)
    np.testing.assert_allclose(Ob, want, rtol=0, atol=1e-12)


def test_attention_invariants(orc):
    """V = 1 gives O = 1; Q = 0 gives the mean of V over the kept keys."""
    spec = MaskSpec(RADIAL, 11, 100)
    B, H, d = 1, 1, 16
    K = _rand((B, H, spec.n, d), 1)
    V = _rand((B, H, spec.n, d), 2)
    bh, q = _all_rows(B, H, spec.n)
    O, _, _ = orc.attention_rows(_rand((B, H, spec.n, d), 3), K, np.ones_like(V), spec, TOKEN_EXACT, 0.3, bh, q)
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-12)
    O, _, _ = orc.attention_rows(np.zeros_like(K), K, V, spec, TOKEN_EXACT, 0.3, bh, q)
    lit = _literal_mask(spec)
    want = (lit.astype(np.float64) @ V[0, 0]) / lit.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(O, want, rtol=0, atol=1e-12)


def test_attention_one_hot_values_expose_probabilities(orc):
    """With V[key] = e_key (n <= d) the output row is the probability vector."""
    spec = MaskSpec(SWC, 4, 8, window_frames=2)
    n = spec.n
    Q, K = _rand((1, 1, n, n), 7), _rand((1, 1, n, n), 8)
    V = np.eye(n)[None, None]
    bh, q = _all_rows(1, 1, n)
    O, _, _ = orc.attention_rows(Q, K, V, spec, TOKEN_EXACT, 0.5, bh, q)
    lit = _literal_mask(spec)
    assert np.all(O[~lit] == 0.0)
    np.testing.assert_allclose(O.sum(axis=1), 1.0, atol=1e-12)
    want = torch.softmax(torch.from_numpy(0.5 * Q[0, 0] @ K[0, 0].T).masked_fill(~torch.from_numpy(lit), -math.inf),
                         dim=-1).numpy()
    np.testing.assert_allclose(O, want, atol=1e-12)
