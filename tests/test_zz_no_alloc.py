"""ra_build_mask_noalloc: the mask builder for callers that cannot allocate.

Engines that own all device memory through their own allocator, processes with
a memory budget fixed at start-up, and loops that cannot take the device-wide
synchronisation of an allocation need a builder that writes into arrays they
already hold and allocates nothing itself.  This entry point keeps its scratch
in a fixed array compiled into the library.  Here it is called through the C
ABI and its block-CSR compared, bit for bit, with the allocating ra_build_mask
over consecutive calls (the shared scratch keeps the previous call's contents),
and its limits are checked.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import _gpu

pytestmark = pytest.mark.gpu

CASES = [
    ("radial", 30, 700, dict()),                                   # n = 21000, ragged tail
    ("window3d", 9, 99, dict(grid_h=9, grid_w=11, r_t=2, r_s=4)),  # n = 891
    ("swc", 41, 1560, dict(window_frames=16)),                     # n = 63960
    ("radial", 32, 4096, dict()),                                  # n = 131072: nb = 1024, the whole scratch
    ("window3d", 31, 4225, dict(grid_h=65, grid_w=65, r_t=1, r_s=3, sink_tokens=300)),  # nb = 1024, ragged tail
    ("radial", 30, 700, dict(sink_tokens=700)),                    # the first frame global
    ("radial", 30, 700, dict()),                                   # the first mask again
]


def _params(ra, kw):
    return ra.ra_mask_params(kw.get("grid_h", 0), kw.get("grid_w", 0), kw.get("r_t", 0), kw.get("r_s", 0),
                             kw.get("window_frames", 0), kw.get("sink_tokens", 0))


def _noalloc(ra, family, f, s, kw, capacity):
    nb = (f * s + 127) // 128
    dev = torch.device("cuda")
    row_ptr = torch.full((nb + 1,), -1, dtype=torch.int32, device=dev)
    col_idx = torch.full((max(capacity, 1),), -1, dtype=torch.int32, device=dev)
    count = torch.full((max(capacity, 1),), -1, dtype=torch.int32, device=dev)
    flag = torch.full((max(capacity, 1),), 255, dtype=torch.uint8, device=dev)
    info = ra.ra_mask_info_t()
    p = _params(ra, kw)
    st = ra.ra_build_mask_noalloc(ra.FAMILIES[family], f, s, ctypes.byref(p), row_ptr.data_ptr(), col_idx.data_ptr(),
                                  count.data_ptr(), flag.data_ptr(), capacity, ctypes.byref(info),
                                  torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    out = dict(row_ptr=row_ptr.cpu().numpy(), col_idx=col_idx.cpu().numpy()[:info.nnz],
               count=count.cpu().numpy()[:info.nnz], flag=flag.cpu().numpy()[:info.nnz])
    return st, out, info


def test_noalloc_matches_the_allocating_builder_on_consecutive_calls():
    _gpu.need_gpu()
    ra = _gpu.ra()
    for family, f, s, kw in CASES:
        ref_mask = ra.Mask(family, f, s, kw.get("grid_h", 0), kw.get("grid_w", 0), kw.get("r_t", 0),
                           kw.get("r_s", 0), kw.get("window_frames", 0), kw.get("sink_tokens", 0))
        ref = ref_mask.to_host()
        st, got, info = _noalloc(ra, family, f, s, kw, capacity=ref["nnz"])
        assert st == ra.RA_OK, ra.ra_last_error()
        for key in ("row_ptr", "col_idx", "count", "flag"):
            assert np.array_equal(got[key], ref[key]), (family, f, s, key)
        got_info = {k: getattr(info, k) for k, _ in ra.ra_mask_info_t._fields_}
        assert got_info == ref_mask.info, (family, f, s)
        assert ra.device_status() == ra.RA_OK


def test_noalloc_limits():
    _gpu.need_gpu()
    ra = _gpu.ra()
    # Beyond the fixed scratch: 1025 query tiles.
    st, _, _ = _noalloc(ra, "radial", 1025, 128, {}, capacity=1)
    assert st == ra.RA_ERR_UNSUPPORTED and b"131072" in ra.ra_last_error()
    # Too small an output: nothing but row_ptr written, nnz reported for sizing.
    st, _, info = _noalloc(ra, "radial", 30, 700, {}, capacity=0)
    assert st == ra.RA_ERR_INVALID_ARG and info.nnz > 0
    st, got, info2 = _noalloc(ra, "radial", 30, 700, {}, capacity=info.nnz)
    assert st == ra.RA_OK and info2.nnz == info.nnz and got["row_ptr"][-1] == info.nnz
