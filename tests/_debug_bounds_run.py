"""Child process of test_debug_bounds_gpu.py: the small parity cases through the
debug library (RA_LIBRARY_VARIANT=debug, every kernel's bounds checks compiled
in).  Exits non-zero, with the reason on stderr, if a check fires or a result
is off; prints "debug bounds ok" otherwise."""
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import static_sparse_attention_b200 as ra  # noqa: E402
import synth  # noqa: E402
from tests import _gpu  # noqa: E402
from tests.test_attention_gpu import EDGE_CASES  # noqa: E402

FAMILY = {oracle.DENSE: "dense", oracle.RADIAL: "radial", oracle.WINDOW3D: "window3d", oracle.SWC: "swc"}


def status(what):
    st = ra.device_status()
    if st != ra.RA_OK:
        site, block = ra.ctypes.c_int(), ra.ctypes.c_int()
        ra.ra_get_device_error_site(ra.ctypes.byref(site), ra.ctypes.byref(block))
        raise SystemExit(f"{what}: device status {st} (site {site.value}, block {block.value})")


def main():
    assert ra.VARIANT == "debug" and ra.LIB_PATH.endswith("libradattn_debug.so"), ra.LIB_PATH
    orc = oracle.default()
    # the checks are compiled in: the self-test's failing check is reported, then cleared
    assert ra.ra_selftest_bounds(None) == ra.RA_ERR_DEVICE_BOUNDS, "bounds self-test not reported"
    status("after the self-test")
    cases = [(oracle.MaskSpec(oracle.RADIAL, 8, 64), 1, 1, 64),
             (oracle.MaskSpec(oracle.WINDOW3D, 16, 256, 16, 16, 1, 1), 2, 2, 64)] + EDGE_CASES
    for spec, B, H, d in cases:
        seed = 5100 + spec.f * 7 + spec.s
        Qh, Kh, Vh, dOh = (synth.normal_bf16(seed, t, (B, H, spec.n, d)) for t in (0, 1, 2, synth.DOUT_TENSOR_ID))
        m = ra.Mask(FAMILY[spec.family], spec.f, spec.s, spec.grid_h, spec.grid_w, spec.r_t, spec.r_s,
                    spec.window_frames, spec.sink_tokens)
        q, k, v, do = (_gpu.to_device(t) for t in (Qh, Kh, Vh, dOh))
        scale = 1.0 / math.sqrt(d)
        for mode, omode in (("token_exact", oracle.TOKEN_EXACT), ("block", oracle.BLOCK)):
            lse = torch.empty((B, H, spec.n), dtype=torch.float32, device="cuda")
            o = ra.attention_fwd(q, k, v, m, scale=scale, mode=mode, lse=lse)
            grads = ra.attention_bwd(q, k, v, o, do, lse, m, scale=scale, mode=mode)
            status(f"{spec} {mode}")
            rows_bh, rows_q = _gpu.all_rows(B, H, spec.n)
            want, _, _ = orc.attention_rows(Qh, Kh, Vh, spec, omode, scale, rows_bh, rows_q)
            _gpu.assert_close(_gpu.gather_rows(_gpu.to_f64(o), rows_bh, rows_q), want, f"debug {spec} {mode}")
            for g in grads:
                assert bool(torch.isfinite(g).all()), f"debug {spec} {mode}: non-finite gradient"
    # a radial mask long enough for the forward's near-first row walk (its row
    # offsets are checked too), on seeded rows
    spec, B, H, d = oracle.MaskSpec(oracle.RADIAL, 64, 1408), 1, 1, 128
    Qh, Kh, Vh = (synth.normal_bf16(5300, t, (B, H, spec.n, d)) for t in range(3))
    q, k, v = (_gpu.to_device(t) for t in (Qh, Kh, Vh))
    m = ra.Mask("radial", spec.f, spec.s)
    lse = torch.empty((B, H, spec.n), dtype=torch.float32, device="cuda")
    o = ra.attention_fwd(q, k, v, m, scale=1.0 / math.sqrt(d), mode="block", lse=lse)
    grads = ra.attention_bwd(q, k, v, o, torch.randn_like(o), lse, m, scale=1.0 / math.sqrt(d), mode="block")
    status(f"{spec} walk")
    for g in grads:
        assert bool(torch.isfinite(g).all()), f"debug {spec} walk: non-finite gradient"
    rows_bh, rows_q = _gpu.sampled_rows(5300, spec.f, spec.s, B, H, 256)
    want, _, _ = orc.attention_rows(Qh, Kh, Vh, spec, oracle.BLOCK, 1.0 / math.sqrt(d), rows_bh, rows_q)
    _gpu.assert_close(_gpu.gather_rows(_gpu.to_f64(o), rows_bh, rows_q), want, f"debug {spec} walk")
    # the streaming SWC step (the forward over the ring with its own tile lists)
    s, W, B, H, d = 130, 3, 1, 2, 128
    Qh, Kh, Vh = (synth.normal_bf16(5200, t, (B, H, 6 * s, d)) for t in range(3))
    q, k, v = (_gpu.to_device(t) for t in (Qh, Kh, Vh))
    cache = ra.SwcCache(B, H, d, s, W)
    for i in range(6):
        sl = slice(i * s, (i + 1) * s)
        cache.step(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous())
    status("SWC stream")
    cache.free()
    print("debug bounds ok")


if __name__ == "__main__":
    main()
