"""GPU backward (dQ, dK, dV) and the transposed block-CSR vs the oracle.

The forward runs on the GPU first (its O and lse are the backward's inputs, as
in training); the oracle recomputes everything in fp64 from the same bf16 Q, K,
V and dO.

Bar, per gradient tensor (derived from the arithmetic: bf16 outputs carry a
relative rounding error of at most 2^-9, and the bf16 P and dS operands of the
gradient MMAs another 2^-9 per term, which averages out over the summed keys):
    ||g_gpu - g_oracle||_2 / ||g_oracle||_2            <= 5e-3
    max |g_gpu - g_oracle| / max |g_oracle|            <= 1e-2
on every row for the small configurations and on seeded sampled rows at full
size.  Transposed CSR: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _gpu
from tests.test_attention_gpu import EDGE_CASES, MODES
from tests.test_mask_gpu import _gpu_mask, _random_specs

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3
MAX_REL = 1e-2


def assert_grad_close(got, want, what):
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    diff = got - want
    scale = max(float(np.max(np.abs(want))), 1e-30)
    max_rel = float(np.max(np.abs(diff))) / scale
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-30))
    assert max_rel <= MAX_REL and rel <= REL_L2, f"{what}: max_rel={max_rel:.3e} rel_l2={rel:.3e}"
    return max_rel, rel


def _fwd_bwd(spec, Qh, Kh, Vh, dOh, mode):
    ra = _gpu.ra()
    m = _gpu_mask(spec)
    q, k, v, do = (_gpu.to_device(t) for t in (Qh, Kh, Vh, dOh))
    B, H, n, d = q.shape
    lse = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
    scale = _gpu.scale_for(d)
    o = ra.attention_fwd(q, k, v, m, scale=scale, mode=mode, lse=lse)
    dq, dk, dv = ra.attention_bwd(q, k, v, o, do, lse, m, scale=scale, mode=mode)
    assert ra.device_status() == ra.RA_OK
    return dq, dk, dv, m


def _check_full(orc, spec, Qh, Kh, Vh, dOh, mode, what):
    dq, dk, dv, _ = _fwd_bwd(spec, Qh, Kh, Vh, dOh, mode)
    want = orc.attention_bwd(Qh, Kh, Vh, dOh, spec, MODES[mode], _gpu.scale_for(Qh.shape[-1]))
    for g, w, name in zip((dq, dk, dv), want, ("dQ", "dK", "dV")):
        assert_grad_close(_gpu.to_f64(g), w, f"{what} {name}")


# ------------------------------------------------------------ transposed CSR

def _config_specs():
    out = []
    for name, c in synth.CONFIGS.items():
        if name == "long460k":
            continue
        for mk in c["masks"]:
            if mk["family"] != "dense":
                out.append(oracle.spec_from(mk, c["f"], c["s"], c["grid"]))
    return out


@pytest.mark.parametrize("spec", _random_specs() + _config_specs(),
                         ids=lambda s: f"fam{s.family}_f{s.f}_s{s.s}_sink{s.sink_tokens}")
def test_transposed_csr_bit_exact(orc, spec):
    """Column-major block-CSR (key tile -> query tiles) equals the oracle's CSR of
    the transposed tile-count table."""
    _gpu.need_gpu()
    m = _gpu_mask(spec)
    want = orc.csr(spec, np.ascontiguousarray(orc.tile_counts(spec).T))
    got = m.transpose_to_host()
    assert np.array_equal(got["col_ptr"], want["row_ptr"])
    assert np.array_equal(got["row_idx"], want["col_idx"])
    assert np.array_equal(got["tflag"], want["flag"])


# ------------------------------------------------------------ small configs

def test_tiny_radial_backward(orc):
    _gpu.need_gpu()
    c = synth.CONFIGS["tiny_radial"]
    Qh, Kh, Vh = synth.qkv_bf16("tiny_radial")
    dOh = synth.dout_bf16("tiny_radial")
    for mk in c["masks"]:
        spec = oracle.spec_from(mk, c["f"], c["s"], c["grid"])
        for mode in ("token_exact", "block"):
            _check_full(orc, spec, Qh, Kh, Vh, dOh, mode, f"tiny {mk['family']} {mode}")


@pytest.mark.parametrize("mk", synth.CONFIGS["window3d_16"]["masks"], ids=lambda m: f"rt{m['r_t']}_rs{m['r_s']}")
@pytest.mark.parametrize("mode", ["token_exact", "block"])
def test_window3d_backward(orc, mk, mode):
    """3D window at n = 4096 (32 tiles), two heads, every row of every gradient."""
    _gpu.need_gpu()
    c = synth.CONFIGS["window3d_16"]
    Qh, Kh, Vh = synth.qkv_bf16("window3d_16", B=1, H=2)
    dOh = synth.dout_bf16("window3d_16", B=1, H=2)
    spec = oracle.spec_from(mk, c["f"], c["s"], c["grid"])
    _check_full(orc, spec, Qh, Kh, Vh, dOh, mode, f"window3d {mk} {mode}")


@pytest.mark.parametrize("case", EDGE_CASES, ids=lambda c: f"fam{c[0].family}_f{c[0].f}_s{c[0].s}_B{c[1]}H{c[2]}d{c[3]}")
@pytest.mark.parametrize("mode", ["token_exact", "block"])
def test_backward_edge_cases(orc, case, mode):
    """Ragged tails, n < 128, one frame, one token per frame, sinks, d = 64 and 128."""
    _gpu.need_gpu()
    spec, B, H, d = case
    seed = 7000 + spec.f * 131 + spec.s
    Qh, Kh, Vh, dOh = (synth.normal_bf16(seed, t, (B, H, spec.n, d)) for t in (0, 1, 2, synth.DOUT_TENSOR_ID))
    _check_full(orc, spec, Qh, Kh, Vh, dOh, mode, f"edge {spec} {mode}")


def test_backward_deterministic_bits():
    """No atomics: two runs give identical bits."""
    _gpu.need_gpu()
    spec = oracle.MaskSpec(oracle.RADIAL, 11, 100)
    Qh, Kh, Vh, dOh = (synth.normal_bf16(99, t, (1, 2, spec.n, 128)) for t in (0, 1, 2, synth.DOUT_TENSOR_ID))
    a = _fwd_bwd(spec, Qh, Kh, Vh, dOh, "block")[:3]
    b = _fwd_bwd(spec, Qh, Kh, Vh, dOh, "block")[:3]
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


# ------------------------------------------------------------ full size

def _full_inputs(name):
    c = synth.CONFIGS[name]
    Qh, Kh, Vh = synth.qkv_bf16(name)
    return c, Qh, Kh, Vh, synth.dout_bf16(name)


@pytest.mark.parametrize("name,mask_i", [("hunyuan108k", 0), ("wan_radial", 0), ("wan_radial", 1)],
                         ids=lambda x: str(x))
def test_full_size_sampled_query_rows_and_sums(orc, name, mask_i):
    """Full size, all heads, in the benchmark's launch configuration (block mode):
    dQ on 256 // H + 8 seeded rows per head (boundary rows included) against the
    oracle one row at a time, and at
    every head and column the identity that holds at any size
        sum_j dV_j = sum_i dO_i   (rows of P sum to 1).
    Its bound is 8 standard deviations of three roundings: dV to bf16 and the P
    operand to bf16 (2^-9 / sqrt(3) of ||dV|| each), and the fp32 row sums of the
    forward that normalise P (a random walk over the k computed keys of a row,
    2^-23 sqrt(k) per row, times ||dO||)."""
    _gpu.need_gpu()
    c, Qh, Kh, Vh, dOh = _full_inputs(name)
    spec = oracle.spec_from(c["masks"][mask_i], c["f"], c["s"], c["grid"])
    dq, dk, dv, m = _fwd_bwd(spec, Qh, Kh, Vh, dOh, "block")
    B, H, n, d = Qh.shape
    row_bh, row_q = _gpu.sampled_rows(synth.config_seed(name), c["f"], c["s"], B, H, count=256 // H + 8)
    want = orc.attention_bwd_query_rows(Qh, Kh, Vh, dOh, spec, oracle.BLOCK, _gpu.scale_for(d), row_bh, row_q)
    got = _gpu.gather_rows(_gpu.to_f64(dq), row_bh, row_q)
    assert_grad_close(got, want, f"{name} dQ sampled")
    dv_sum = dv.double().sum(dim=2).cpu().numpy()
    dv_norm = np.sqrt((dv.double() ** 2).sum(dim=2).cpu().numpy())
    dO64 = synth.bf16_bits_to_f32(dOh).astype(np.float64)
    dO_sum, dO_norm = dO64.sum(axis=2), np.sqrt((dO64 ** 2).sum(axis=2))
    keys_per_row = m.info["block_pairs"] / n
    eps_b = 2.0 ** -9 / np.sqrt(3.0)
    eps_n = 2.0 ** -23 * np.sqrt(keys_per_row)
    sigma = np.sqrt(2.0 * (eps_b * dv_norm) ** 2 + (eps_n * dO_norm) ** 2)
    err = np.abs(dv_sum - dO_sum)
    assert np.all(err <= 8 * sigma), f"sum_j dV_j != sum_i dO_i: worst {float(np.max(err / sigma)):.1f} sigma"


def _key_rows_check(orc, name, mask_i, H, keys, what):
    c = synth.CONFIGS[name]
    Qh, Kh, Vh = synth.qkv_bf16(name, H=H)
    dOh = synth.dout_bf16(name, H=H)
    spec = oracle.spec_from(c["masks"][mask_i], c["f"], c["s"], c["grid"])
    _, dk, dv, _ = _fwd_bwd(spec, Qh, Kh, Vh, dOh, "block")
    want_k, want_v = orc.attention_bwd_key_rows(Qh[0, 0], Kh[0, 0], Vh[0, 0], dOh[0, 0], spec, oracle.BLOCK,
                                                _gpu.scale_for(c["d"]), keys)
    assert_grad_close(_gpu.to_f64(dk)[0, 0, keys], want_k, f"{what} dK sampled")
    assert_grad_close(_gpu.to_f64(dv)[0, 0, keys], want_v, f"{what} dV sampled")


def test_hunyuan_sampled_key_rows(orc):
    """The 108k radial workload with all 24 heads (the benchmark's launch
    configuration): dK, dV of 16 key rows of head 0 in the first and the last
    (ragged) key tile against the oracle key by key."""
    _gpu.need_gpu()
    n = synth.CONFIGS["hunyuan108k"]["f"] * synth.CONFIGS["hunyuan108k"]["s"]
    keys = np.r_[np.arange(8) * 16 + 5, (n - 1) - np.arange(8) * 9]
    _key_rows_check(orc, "hunyuan108k", 0, None, keys, "hunyuan")


def test_wan_sampled_key_rows(orc):
    """dK, dV of 24 seeded key rows (boundary rows included) of one head of the Wan
    workload (n = 63960) against the oracle key by key."""
    _gpu.need_gpu()
    c = synth.CONFIGS["wan_radial"]
    keys = synth.sample_rows(synth.config_seed("wan_radial") + 1, c["f"], c["s"], 24)
    _key_rows_check(orc, "wan_radial", 0, 1, keys, "wan")
