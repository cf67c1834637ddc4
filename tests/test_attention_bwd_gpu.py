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
    # gradients and the D workspace inside canary bands (no store outside them)
    g = [_gpu.Guarded((B, H, n, d), torch.bfloat16) for _ in range(3)]
    g_ws = _gpu.Guarded((B, H, n), torch.float32)
    dq, dk, dv = ra.attention_bwd(q, k, v, o, do, lse, m, scale=scale, mode=mode, dq=g[0].t, dk=g[1].t,
                                  dv=g[2].t, workspace=g_ws.t)
    assert ra.device_status() == ra.RA_OK
    _gpu.check_canaries(*g, g_ws, what=f"backward {spec} {mode}")
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


# Relative rounding error of one bf16 rounding (8-bit significand, round to
# nearest even): at most 2^-8 in magnitude and uniform over the spacing, so its
# standard deviation is at most 2^-8 / sqrt(3) (attained at the bottom of a binade).
EPS_BF16 = 2.0 ** -8 / np.sqrt(3.0)


@pytest.mark.parametrize("name,mask_i", [("hunyuan108k", 0), ("wan_radial", 0), ("wan_radial", 1)],
                         ids=lambda x: str(x))
def test_full_size_sampled_query_rows_and_sums(orc, name, mask_i):
    """Full size, all heads, in the benchmark's launch configuration (block mode).

    dQ on the same 256 seeded rows in every head (boundary rows included) against
    the oracle one row at a time; and, at every head and column, two identities
    that hold at any size, each within 8 standard deviations of the roundings
    that can break it:

      sum_j dV_j = sum_i dO_i, because the rows of P sum to 1.  Roundings: dV to
        bf16 and the P operand to bf16 (EPS_BF16 ||dV|| each), and the fp32 row
        sums that normalise P (a random walk over the k computed keys of a row,
        2^-23 sqrt(k) per row, times ||dO||).

      sum_j dK_j = 0, because sum_j dS_ij = sum_j P_ij dP_ij - D_i sum_j P_ij and
        sum_j P_ij dP_ij = <dO_i, O_i> = D_i.  The kernel takes D_i from the
        forward's bf16 O, so row i leaves eps_i = <dO_i, O_i - O_fwd_i>, and
        sum_j dK_jc = scale sum_i eps_i Q_ic: a random sum of standard deviation
        scale rms(eps) ||Q_c||, with rms(eps) measured on the sampled rows
        against the oracle's exact O.  Roundings: dK to bf16 and the dS operand
        to bf16 (EPS_BF16 ||dK_c|| each, since dK = scale dS^T Q with unit-variance
        Q gives ||dK_c|| = scale ||dS||_F)."""
    _gpu.need_gpu()
    c, Qh, Kh, Vh, dOh = _full_inputs(name)
    spec = oracle.spec_from(c["masks"][mask_i], c["f"], c["s"], c["grid"])
    ra = _gpu.ra()
    m = _gpu_mask(spec)
    q, k, v, do = (_gpu.to_device(t) for t in (Qh, Kh, Vh, dOh))
    B, H, n, d = q.shape
    scale = _gpu.scale_for(d)
    lse = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
    o = ra.attention_fwd(q, k, v, m, scale=scale, mode="block", lse=lse)
    dq, dk, dv = ra.attention_bwd(q, k, v, o, do, lse, m, scale=scale, mode="block")
    assert ra.device_status() == ra.RA_OK

    row_bh, row_q = _gpu.sampled_rows(synth.config_seed(name), c["f"], c["s"], B, H, count=256)
    want = orc.attention_bwd_query_rows(Qh, Kh, Vh, dOh, spec, oracle.BLOCK, scale, row_bh, row_q)
    got = _gpu.gather_rows(_gpu.to_f64(dq), row_bh, row_q)
    assert_grad_close(got, want, f"{name} dQ sampled")

    keys_per_row = m.info["block_pairs"] / n

    def sum_and_norm(t):  # over the rows of each (b, h), per column, in fp64 on the device
        t64 = t.double()
        out = t64.sum(dim=2).cpu().numpy(), torch.sqrt((t64 ** 2).sum(dim=2)).cpu().numpy()
        del t64
        return out

    # sum_j dV_j = sum_i dO_i
    dv_sum, dv_norm = sum_and_norm(dv)
    dO_sum, dO_norm = sum_and_norm(do)
    eps_n = 2.0 ** -23 * np.sqrt(keys_per_row)
    sigma = np.sqrt(2.0 * (EPS_BF16 * dv_norm) ** 2 + (eps_n * dO_norm) ** 2)
    err = np.abs(dv_sum - dO_sum)
    assert np.all(err <= 8 * sigma), f"sum_j dV_j != sum_i dO_i: worst {float(np.max(err / sigma)):.1f} sigma"

    # sum_j dK_j = 0
    o_exact, _, _ = orc.attention_rows(Qh, Kh, Vh, spec, oracle.BLOCK, scale, row_bh, row_q)
    o_fwd = _gpu.gather_rows(_gpu.to_f64(o), row_bh, row_q)
    dO_rows = synth.bf16_bits_to_f32(dOh.reshape(B * H, n, d)[row_bh, row_q]).astype(np.float64)
    eps = np.sum(dO_rows * (o_exact - o_fwd), axis=1)                      # one per sampled row
    rms_eps = np.sqrt(np.bincount(row_bh, eps ** 2, B * H) / np.bincount(row_bh, None, B * H))
    dk_sum, dk_norm = (x.reshape(B * H, d) for x in sum_and_norm(dk))
    q_norm = sum_and_norm(q)[1].reshape(B * H, d)
    sigma_k = np.sqrt(2.0 * (EPS_BF16 * dk_norm) ** 2 + (scale * rms_eps[:, None] * q_norm) ** 2)
    ratio = np.abs(dk_sum) / sigma_k
    assert np.all(ratio <= 8), f"sum_j dK_j != 0: worst {float(np.max(ratio)):.1f} sigma"


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


@pytest.mark.parametrize("mode", ["block", "token_exact"])
def test_near_first_walk_backward_sampled_rows(orc, mode):
    """A radial mask long enough for the near-first walk of the rows of both the
    block-CSR (dQ pass) and its transpose (dK / dV pass): 64 frames of 1408
    tokens, 704 tiles.  dQ on 256 seeded query rows and dK, dV on the 6 boundary
    key rows (first and last of the sequence, of frame 1 and of the last frame,
    first of the last tile) against the oracle."""
    _gpu.need_gpu()
    spec = oracle.MaskSpec(oracle.RADIAL, 64, 1408)
    B, H, d = 1, 1, 128
    Qh, Kh, Vh, dOh = (synth.normal_bf16(6500, t, (B, H, spec.n, d)) for t in (0, 1, 2, synth.DOUT_TENSOR_ID))
    dq, dk, dv, _ = _fwd_bwd(spec, Qh, Kh, Vh, dOh, mode)
    scale = _gpu.scale_for(d)
    row_bh, row_q = _gpu.sampled_rows(6500, spec.f, spec.s, B, H, count=256)
    want = orc.attention_bwd_query_rows(Qh, Kh, Vh, dOh, spec, MODES[mode], scale, row_bh, row_q)
    assert_grad_close(_gpu.gather_rows(_gpu.to_f64(dq), row_bh, row_q), want, f"walk {mode} dQ sampled")
    keys = synth.sample_rows(6501, spec.f, spec.s, 4)  # the boundary rows
    want_k, want_v = orc.attention_bwd_key_rows(Qh[0, 0], Kh[0, 0], Vh[0, 0], dOh[0, 0], spec, MODES[mode], scale,
                                                keys)
    assert_grad_close(_gpu.to_f64(dk)[0, 0, keys], want_k, f"walk {mode} dK sampled")
    assert_grad_close(_gpu.to_f64(dv)[0, 0, keys], want_v, f"walk {mode} dV sampled")
