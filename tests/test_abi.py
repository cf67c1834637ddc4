"""The C ABI: the library loads, exports every declared entry point, and rejects
bad arguments with the documented status before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "radattn.h")


@pytest.fixture(scope="module")
def ra():
    import __graft_entry__
    __graft_entry__.build()
    import static_sparse_attention_b200 as ra
    return ra


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\**\s*(ra_[a-z0-9_]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("ra_build_mask", "ra_attention_fwd", "ra_mask_info", "ra_mask_free", "ra_get_device_status",
                 "ra_attention_fwd_host", "ra_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(ra):
    lib = ctypes.CDLL(ra.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version(ra):
    assert ra.ra_status_string(ra.RA_OK) == b"ok"
    assert ra.ra_status_string(ra.RA_ERR_DEVICE_TIMEOUT) == b"device wait timed out"
    assert ra.ra_version() >= 10000


def _build(ra, fam, f, s, params=None):
    out = ctypes.c_void_p()
    p = params or ra.ra_mask_params(0, 0, 0, 0, 0)
    st = ra.ra_build_mask(fam, f, s, ctypes.byref(p), None, ctypes.byref(out))
    return st, out


@pytest.mark.parametrize("fam,f,s,params,status", [
    (7, 4, 4, None, 1),                         # unknown family
    (1, 0, 4, None, 1),                         # f < 1
    (1, 4, 0, None, 1),                         # s < 1
    (2, 4, 12, (3, 5, 1, 1, 0), 1),             # grid_h * grid_w != s
    (2, 4, 12, (3, 4, -1, 1, 0), 1),            # negative radius
    (3, 4, 12, (0, 0, 0, 0, 0), 1),             # window_frames < 1
    (1, 1 << 20, 1 << 12, None, 2),             # n beyond the builder's limit
    (1, 4, 4, (0, 0, 0, 0, 0, -1), 1),          # negative sink_tokens
    (1, 4, 4, (0, 0, 0, 0, 0, 17), 1),          # sink_tokens > n
])
def test_build_mask_rejects_bad_arguments(ra, fam, f, s, params, status):
    p = ra.ra_mask_params(*params) if params else None
    st, out = _build(ra, fam, f, s, p)
    assert st == status
    assert not out.value
    assert ra.ra_last_error()


def test_build_mask_null_out(ra):
    p = ra.ra_mask_params(0, 0, 0, 0, 0)
    assert ra.ra_build_mask(1, 2, 2, ctypes.byref(p), None, None) == ra.RA_ERR_INVALID_ARG


def test_attention_rejects_bad_arguments(ra):
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    args = dict(Q=0x10000, K=0x20000, V=0x30000, O=0x40000, B=1, H=1, d=128, m=fake, scale=0.1, mode=1)

    def call(**kw):
        a = {**args, **kw}
        return ra.ra_attention_fwd(a["Q"], a["K"], a["V"], a["O"], a["B"], a["H"], a["d"], a["m"], a["scale"],
                                   a["mode"], None, None)

    assert call(Q=None) == ra.RA_ERR_INVALID_ARG
    assert call(K=0x20008) == ra.RA_ERR_INVALID_ARG          # not 16-byte aligned
    assert call(m=None) == ra.RA_ERR_INVALID_ARG
    assert call(B=0) == ra.RA_ERR_INVALID_ARG
    assert call(H=70000) == ra.RA_ERR_INVALID_ARG
    assert call(d=96) == ra.RA_ERR_UNSUPPORTED
    assert call(mode=5) == ra.RA_ERR_INVALID_ARG
    assert call(scale=0.0) == ra.RA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_attention_fwd_host(None, None, None, None, None, None, None, None, 1, 1, 64, fake, 0.1, 1,
                                    None) == ra.RA_ERR_INVALID_ARG


def test_backward_rejects_bad_arguments(ra):
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    args = dict(Q=0x10000, K=0x20000, V=0x30000, O=0x40000, dO=0x50000, lse=0x60000, dQ=0x70000, dK=0x80000,
                dV=0x90000, ws=0xA0000, B=1, H=1, d=128, m=fake, scale=0.1, mode=1)

    def call(**kw):
        a = {**args, **kw}
        return ra.ra_attention_bwd(a["Q"], a["K"], a["V"], a["O"], a["dO"], a["lse"], a["dQ"], a["dK"], a["dV"],
                                   a["ws"], a["B"], a["H"], a["d"], a["m"], a["scale"], a["mode"], None)

    assert call(dO=None) == ra.RA_ERR_INVALID_ARG
    assert call(dV=0x90004) == ra.RA_ERR_INVALID_ARG         # not 16-byte aligned
    assert call(lse=None) == ra.RA_ERR_INVALID_ARG
    assert call(ws=None) == ra.RA_ERR_INVALID_ARG
    assert call(m=None) == ra.RA_ERR_INVALID_ARG
    assert call(B=0) == ra.RA_ERR_INVALID_ARG
    assert call(d=256) == ra.RA_ERR_UNSUPPORTED
    assert call(mode=3) == ra.RA_ERR_INVALID_ARG
    assert call(scale=-1.0) == ra.RA_ERR_INVALID_ARG
    # an output aliasing an input or another output (dQ is written before the
    # dK / dV kernel reads Q and dO)
    for out_name in ("dQ", "dK", "dV", "ws"):
        for other in ("Q", "K", "V", "O", "dO", "lse", "dQ", "dK", "dV", "ws"):
            if other != out_name:
                assert call(**{out_name: args[other]}) == ra.RA_ERR_INVALID_ARG, (out_name, other)
                assert b"alias" in ra.ra_last_error()


def test_swc_cache_rejects_bad_arguments(ra):
    h = ctypes.c_void_p()
    assert ra.ra_swc_cache_create(0, 1, 128, 100, 4, ctypes.byref(h)) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_create(1, 1, 96, 100, 4, ctypes.byref(h)) == ra.RA_ERR_UNSUPPORTED
    assert ra.ra_swc_cache_create(1, 1, 128, 0, 4, ctypes.byref(h)) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_create(1, 1, 128, 100, 0, ctypes.byref(h)) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_create(1, 1, 128, 100, 4, None) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_create(1, 1, 64, 1 << 20, 4096, ctypes.byref(h)) == ra.RA_ERR_UNSUPPORTED
    assert ra.ra_swc_cache_step(None, None, None, None, None, 0.1, None, None) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_info(None, None, None) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_reset(None) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_swc_cache_copy_rings_to_host(None, None, None) == ra.RA_ERR_INVALID_ARG
    ra.ra_swc_cache_free(None)


def test_release_library_has_no_bounds_checks(ra):
    """The bounds self-test needs the debug variant; the release build says so
    without touching the GPU."""
    if ra.VARIANT == "release":
        assert ra.ra_selftest_bounds(None) == ra.RA_ERR_UNSUPPORTED
        assert b"RA_DEBUG_BOUNDS" in ra.ra_last_error()
    assert ra.ra_status_string(ra.RA_ERR_DEVICE_BOUNDS) == b"device bounds check failed"


def test_kernel_settings_are_range_checked(ra):
    assert ra.ra_set_pv_precision(7) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_set_pv_precision(-1) == ra.RA_ERR_INVALID_ARG
    for v in (ra.RA_PV_BF16, ra.RA_PV_SPLIT, ra.RA_PV_AUTO):
        assert ra.ra_set_pv_precision(v) == ra.RA_OK


def test_timeout_settings_are_range_checked(ra):
    assert ra.ra_set_wait_timeout_ns(10) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_set_wait_timeout_ns(4_000_000_000) == ra.RA_OK
    assert ra.ra_selftest_wait_timeout(5, None) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_set_pv_precision(7) == ra.RA_ERR_INVALID_ARG
    assert ra.ra_set_pv_precision(ra.RA_PV_AUTO) == ra.RA_OK


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "static_sparse_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "radattn_oracle" not in text, fn
