"""Streaming SWC attention with the key/value ring cache vs the oracle.

Each streamed frame's output must equal the rows of that frame of the
sliding-window causal attention over the whole sequence (the oracle's SWC mask,
token-exact), to the forward's bar (max-abs <= 1e-2, relative-L2 <= 5e-3,
lse within 2e-3).  The ring must hold exactly the last W frames' K and V."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _gpu

pytestmark = pytest.mark.gpu


def _stream(Qh, Kh, Vh, s, W, frames=None):
    """Feed the frames one by one; returns (outputs [f][B, H, s, d] fp64, lse [f][B, H, s], cache)."""
    ra = _gpu.ra()
    B, H, n, d = Qh.shape
    f = n // s if frames is None else frames
    q, k, v = (_gpu.to_device(t) for t in (Qh, Kh, Vh))
    cache = ra.SwcCache(B, H, d, s, W)
    outs, lses = [], []
    for i in range(f):
        sl = slice(i * s, (i + 1) * s)
        # the step's outputs inside canary bands: no store outside them
        g_o, g_lse = _gpu.Guarded((B, H, s, d), torch.bfloat16), _gpu.Guarded((B, H, s), torch.float32)
        o = cache.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), out=g_o.t,
                       lse=g_lse.t)
        _gpu.check_canaries(g_o, g_lse, what=f"SWC step {i}")
        assert bool(torch.isfinite(o).all()), f"SWC step {i}: an output row was not written"
        outs.append(_gpu.to_f64(o))
        lses.append(g_lse.t.cpu().numpy().astype(np.float64))
    assert ra.device_status() == ra.RA_OK
    return outs, lses, cache


def _check_frames(orc, Qh, Kh, Vh, s, W, outs, lses, frames, rows_per_frame=None, what=""):
    B, H, n, d = Qh.shape
    spec = oracle.MaskSpec(oracle.SWC, n // s, s, window_frames=W)
    for i in frames:
        local = np.arange(s) if rows_per_frame is None else np.unique(
            np.r_[0, s - 1, np.random.default_rng(i).integers(0, s, rows_per_frame)])
        row_bh = np.repeat(np.arange(B * H), len(local))
        row_q = np.tile(i * s + local, B * H)
        want, want_lse, _ = orc.attention_rows(Qh, Kh, Vh, spec, oracle.TOKEN_EXACT, _gpu.scale_for(d), row_bh, row_q)
        got = outs[i].reshape(B * H, s, d)[row_bh, row_q - i * s]
        _gpu.assert_close(got, want, f"{what} frame {i}")
        got_lse = lses[i].reshape(B * H, s)[row_bh, row_q - i * s]
        np.testing.assert_allclose(got_lse, want_lse, rtol=0, atol=2e-3, err_msg=f"{what} frame {i} lse")


@pytest.mark.parametrize("s,W,f,B,H,d", [(130, 3, 9, 1, 2, 128), (64, 4, 11, 2, 1, 64), (100, 1, 4, 1, 1, 128),
                                         (37, 5, 3, 1, 2, 64), (300, 2, 5, 1, 1, 128)],
                         ids=lambda x: str(x))
def test_stream_equals_swc_rows(orc, s, W, f, B, H, d):
    """Every row of every frame: ring not yet full, exactly full, and wrapping;
    frames shorter than a tile and ragged tails; W = 1."""
    _gpu.need_gpu()
    seed = 9100 + s * 7 + W
    Qh, Kh, Vh = (synth.normal_bf16(seed, t, (B, H, f * s, d)) for t in range(3))
    outs, lses, _ = _stream(Qh, Kh, Vh, s, W)
    _check_frames(orc, Qh, Kh, Vh, s, W, outs, lses, range(f), what=f"s={s} W={W}")


def test_ring_holds_the_last_window(orc):
    """After each step the ring holds frames max(0, i-W+1) .. i, frame j in slot j mod W, bit for bit."""
    _gpu.need_gpu()
    s, W, f, B, H, d = 96, 3, 7, 1, 2, 64
    Qh, Kh, Vh = (synth.normal_bf16(4242, t, (B, H, f * s, d)) for t in range(3))
    ra = _gpu.ra()
    q, k, v = (_gpu.to_device(t) for t in (Qh, Kh, Vh))
    cache = ra.SwcCache(B, H, d, s, W)
    for i in range(f):
        sl = slice(i * s, (i + 1) * s)
        cache.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous())
        kr, vr = cache.rings_to_host()
        assert cache.info == dict(frames_seen=i + 1, frames_held=min(i + 1, W))
        for j in range(max(0, i - W + 1), i + 1):
            slot = slice((j % W) * s, (j % W + 1) * s)
            assert np.array_equal(kr[:, :, slot], Kh[:, :, j * s:(j + 1) * s])
            assert np.array_equal(vr[:, :, slot], Vh[:, :, j * s:(j + 1) * s])


def test_reset_restarts_the_stream():
    _gpu.need_gpu()
    s, W, f, B, H, d = 128, 2, 3, 1, 1, 128
    Qh, Kh, Vh = (synth.normal_bf16(77, t, (B, H, f * s, d)) for t in range(3))
    outs, _, cache = _stream(Qh, Kh, Vh, s, W)
    cache.reset()
    assert cache.info == dict(frames_seen=0, frames_held=0)
    q, k, v = (_gpu.to_device(t[:, :, :s]) for t in (Qh, Kh, Vh))
    o = cache.step(q, k, v)
    assert np.array_equal(_gpu.to_f64(o), outs[0])


def test_wan_shaped_stream_sampled_rows(orc):
    """Wan-shaped frames (s = 1560, W = 16, d = 128, 2 heads) over 20 frames: the
    ring fills, wraps and evicts; 64 seeded rows of frames 0, 7, 15, 16 and 19."""
    _gpu.need_gpu()
    s, W, f, B, H, d = 1560, 16, 20, 1, 2, 128
    seed = synth.config_seed("wan_radial") + 50
    Qh, Kh, Vh = (synth.normal_bf16(seed, t, (B, H, f * s, d)) for t in range(3))
    outs, lses, _ = _stream(Qh, Kh, Vh, s, W)
    _check_frames(orc, Qh, Kh, Vh, s, W, outs, lses, [0, 7, 15, 16, 19], rows_per_frame=64, what="wan stream")
