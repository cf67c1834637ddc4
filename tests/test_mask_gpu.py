"""GPU block-CSR builder vs the oracle: bit-exact row_ptr, col_idx, count, flag."""
import numpy as np
import pytest

import oracle
import synth
from tests import _gpu, _pins

pytestmark = pytest.mark.gpu


def _gpu_mask(spec: oracle.MaskSpec):
    ra = _gpu.ra()
    fam = {oracle.DENSE: "dense", oracle.RADIAL: "radial", oracle.WINDOW3D: "window3d", oracle.SWC: "swc"}[spec.family]
    return ra.Mask(fam, spec.f, spec.s, spec.grid_h, spec.grid_w, spec.r_t, spec.r_s, spec.window_frames,
                   spec.sink_tokens)


def _assert_csr_equal(got: dict, want: dict):
    for key in ("row_ptr", "col_idx", "count", "flag"):
        assert got[key].dtype == want[key].dtype, key
        assert np.array_equal(got[key], want[key]), key


def _assert_info_matches(m, spec, counts):
    info = m.info
    kept = counts > 0
    nb = spec.nb
    rows_valid = np.minimum(128, spec.n - np.arange(nb) * 128)
    assert info["nnz"] == int(kept.sum())
    assert info["kept_pairs"] == int(counts.sum())
    assert info["block_pairs"] == int((kept * np.outer(rows_valid, rows_valid)).sum())
    assert info["full_tiles"] == int((counts == 128 * 128).sum())
    per_row = kept.sum(axis=1)
    assert info["row_min"] == int(per_row.min()) and info["row_max"] == int(per_row.max())


def _random_specs():
    rng = np.random.default_rng(1234)
    specs = []
    for _ in range(40):
        fam = int(rng.integers(0, 4))
        f = int(rng.integers(1, 40))
        if fam == oracle.WINDOW3D:
            gh, gw = int(rng.integers(1, 20)), int(rng.integers(1, 20))
            specs.append(oracle.MaskSpec(fam, f, gh * gw, gh, gw, int(rng.integers(0, 4)), int(rng.integers(0, 6))))
        elif fam == oracle.SWC:
            specs.append(oracle.MaskSpec(fam, f, int(rng.integers(1, 300)), window_frames=int(rng.integers(1, 20))))
        else:
            specs.append(oracle.MaskSpec(fam, f, int(rng.integers(1, 300))))
    # global (sink) tokens on top of each family, including a sink longer than a tile
    for k, sp in enumerate(list(specs[:12])):
        specs.append(oracle.MaskSpec(sp.family, sp.f, sp.s, sp.grid_h, sp.grid_w, sp.r_t, sp.r_s,
                                     sp.window_frames, sink_tokens=min(sp.n, [1, 37, 128, 300][k % 4])))
    return specs


@pytest.mark.parametrize("spec", _random_specs(), ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}")
def test_random_small_masks_bit_exact(orc, spec):
    _gpu.need_gpu()
    counts = orc.tile_counts(spec)
    m = _gpu_mask(spec)
    _assert_csr_equal(m.to_host(), orc.csr(spec, counts))
    _assert_info_matches(m, spec, counts)


def _config_specs():
    out = []
    for name, c in synth.CONFIGS.items():
        if name == "long460k":
            continue
        for mk in c["masks"]:
            out.append((name, oracle.spec_from(mk, c["f"], c["s"], c["grid"])))
    return out


@pytest.mark.parametrize("name,spec", _config_specs(),
                         ids=lambda x: x if isinstance(x, str) else f"fam{x.family}")
def test_config_masks_bit_exact(orc, name, spec):
    """Every configured mask except the 460k one, whole CSR (brute-force oracle)."""
    _gpu.need_gpu()
    m = _gpu_mask(spec)
    got = m.to_host()
    if spec.family == oracle.DENSE:
        counts = _pins.tile_reduce(np.ones((spec.n, spec.n), dtype=bool)) if spec.n <= 8192 else None
        if counts is None:  # dense at full size: every tile kept, count = valid pairs
            rv = np.minimum(128, spec.n - np.arange(spec.nb) * 128)
            counts = np.outer(rv, rv)
    else:
        counts = orc.tile_counts(spec)
    _assert_csr_equal(got, orc.csr(spec, counts))
    _assert_info_matches(m, spec, counts)


def test_long460k_sampled_rows_and_totals(orc):
    """4x-long radial (n = 460800): 64 seeded query-tile rows bit-exact against the
    oracle, and totals against the closed form of eq. 4."""
    _gpu.need_gpu()
    c = synth.CONFIGS["long460k"]
    spec = oracle.spec_from(c["masks"][0], c["f"], c["s"])
    m = _gpu_mask(spec)
    got = m.to_host()
    assert m.info["kept_pairs"] == _pins.radial_closed_form_total(c["f"], c["s"])
    rows = np.unique(synth.sample_rows(synth.config_seed("long460k"), c["f"], c["s"], 64) // 128).astype(np.int32)
    counts = orc.tile_counts(spec, rows)
    for r, qb in enumerate(rows):
        lo, hi = got["row_ptr"][qb], got["row_ptr"][qb + 1]
        kb = np.nonzero(counts[r])[0]
        assert np.array_equal(got["col_idx"][lo:hi], kb)
        assert np.array_equal(got["count"][lo:hi], counts[r][kb])
        assert np.array_equal(got["flag"][lo:hi], (counts[r][kb] == 128 * 128).astype(np.uint8))
    assert np.all(np.diff(got["row_ptr"]) >= 1)


def test_radial_totals_match_closed_form_on_config_shapes():
    _gpu.need_gpu()
    for name in ("tiny_radial", "wan_radial", "hunyuan108k"):
        c = synth.CONFIGS[name]
        m = _gpu.ra().Mask("radial", c["f"], c["s"])
        assert m.info["kept_pairs"] == _pins.radial_closed_form_total(c["f"], c["s"])
