"""Python binding of libradattn.so (the C ABI in include/radattn.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  The C entry points are exposed under their own names
(ra_build_mask, ra_attention_fwd, ...) taking plain integers / pointers, plus a
thin torch-facing layer (Mask, build_mask, attention_fwd, attention_fwd_host)
that passes tensor addresses and the current CUDA stream.

There is no CPU fallback: importing this package fails loudly when the
compiled library is missing (build it with
`python static_sparse_attention_b200/build.py`).
"""
from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# RA_LIBRARY_VARIANT=debug selects the build with device-side bounds checks
# (libradattn_debug.so, `build.py --debug`); the default is the release build.
VARIANT = os.environ.get("RA_LIBRARY_VARIANT", "release")
if VARIANT not in ("release", "debug"):
    raise ImportError(f"RA_LIBRARY_VARIANT must be 'release' or 'debug', not {VARIANT!r}")
LIB_PATH = os.path.join(_PKG, "libradattn_debug.so" if VARIANT == "debug" else "libradattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                      f"`python static_sparse_attention_b200/build.py{' --debug' if VARIANT == 'debug' else ''}`")

_lib = ctypes.CDLL(LIB_PATH)

# ------------------------------------------------------------------ constants
RA_MASK_DENSE, RA_MASK_RADIAL, RA_MASK_WINDOW3D, RA_MASK_SWC = 0, 1, 2, 3
RA_MODE_TOKEN_EXACT, RA_MODE_BLOCK = 0, 1
RA_TILE_PARTIAL, RA_TILE_FULL = 0, 1
(RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_OUT_OF_MEMORY, RA_ERR_DEVICE_TIMEOUT,
 RA_ERR_DEVICE_BOUNDS) = range(7)
RA_TILE = 128
RA_PV_AUTO, RA_PV_BF16, RA_PV_SPLIT = 0, 1, 2
FAMILIES = {"dense": RA_MASK_DENSE, "radial": RA_MASK_RADIAL, "window3d": RA_MASK_WINDOW3D, "swc": RA_MASK_SWC}
MODES = {"token_exact": RA_MODE_TOKEN_EXACT, "block": RA_MODE_BLOCK}


class ra_mask_params(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("r_t", ctypes.c_int), ("r_s", ctypes.c_int),
                ("window_frames", ctypes.c_int), ("sink_tokens", ctypes.c_int)]


class ra_mask_info_t(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int), ("f", ctypes.c_int), ("s", ctypes.c_int), ("nb", ctypes.c_int),
                ("n", ctypes.c_longlong), ("nnz", ctypes.c_longlong), ("full_tiles", ctypes.c_longlong),
                ("kept_pairs", ctypes.c_longlong), ("block_pairs", ctypes.c_longlong),
                ("row_min", ctypes.c_int), ("row_max", ctypes.c_int)]


_vp, _i, _ll, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
_MaskP = ctypes.c_void_p
_SIGS = {
    "ra_build_mask": ([_i, _i, _i, ctypes.POINTER(ra_mask_params), _vp, ctypes.POINTER(_MaskP)], _i),
    "ra_mask_info": ([_MaskP, ctypes.POINTER(ra_mask_info_t)], _i),
    "ra_build_mask_noalloc": ([_i, _i, _i, ctypes.POINTER(ra_mask_params), _vp, _vp, _vp, _vp, _ll,
                               ctypes.POINTER(ra_mask_info_t), _vp], _i),
    "ra_mask_copy_to_host": ([_MaskP, _vp, _vp, _vp, _vp], _i),
    "ra_mask_device_arrays": ([_MaskP, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                               ctypes.POINTER(_vp)], _i),
    "ra_mask_free": ([_MaskP], None),
    "ra_mask_copy_transpose_to_host": ([_MaskP, _vp, _vp, _vp], _i),
    "ra_attention_fwd": ([_vp, _vp, _vp, _vp, _i, _i, _i, _MaskP, _f, _i, _vp, _vp], _i),
    "ra_attention_fwd_host": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _MaskP, _f, _i, _vp], _i),
    "ra_attention_bwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _MaskP, _f, _i, _vp], _i),
    "ra_swc_cache_create": ([_i, _i, _i, _i, _i, ctypes.POINTER(_vp)], _i),
    "ra_swc_cache_step": ([_vp, _vp, _vp, _vp, _vp, _f, _vp, _vp], _i),
    "ra_swc_cache_info": ([_vp, ctypes.POINTER(_ll), ctypes.POINTER(_i)], _i),
    "ra_swc_cache_copy_rings_to_host": ([_vp, _vp, _vp], _i),
    "ra_swc_cache_reset": ([_vp], _i),
    "ra_swc_cache_free": ([_vp], None),
    "ra_get_device_status": ([_vp], _i),
    "ra_get_device_error_site": ([ctypes.POINTER(_i), ctypes.POINTER(_i)], _i),
    "ra_selftest_wait_timeout": ([_ll, _vp], _i),
    "ra_selftest_bounds": ([_vp], _i),
    "ra_set_wait_timeout_ns": ([_ll], _i),
    "ra_set_pv_precision": ([_i], _i),
    "ra_status_string": ([_i], ctypes.c_char_p),
    "ra_last_error": ([], ctypes.c_char_p),
    "ra_version": ([], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res
    globals()[_name] = _fn


class RaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = (ra_last_error() or b"").decode(errors="replace")
        super().__init__(f"{where}: {ra_status_string(status).decode()} ({status}): {detail}")


def check(status: int, where: str) -> None:
    if status != RA_OK:
        raise RaError(status, where)


def _stream_handle(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------- masks
class Mask:
    """A block-CSR mask built on the current CUDA device (owns the C handle)."""

    def __init__(self, family, f: int, s: int, grid_h: int = 0, grid_w: int = 0, r_t: int = 0, r_s: int = 0,
                 window_frames: int = 0, sink_tokens: int = 0, stream=None):
        fam = FAMILIES[family] if isinstance(family, str) else int(family)
        params = ra_mask_params(grid_h, grid_w, r_t, r_s, window_frames, sink_tokens)
        handle = _MaskP()
        check(ra_build_mask(fam, f, s, ctypes.byref(params), _stream_handle(stream), ctypes.byref(handle)),
              "ra_build_mask")
        self._h = handle
        info = ra_mask_info_t()
        check(ra_mask_info(self._h, ctypes.byref(info)), "ra_mask_info")
        self.info = {k: getattr(info, k) for k, _ in ra_mask_info_t._fields_}

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("mask has been freed")
        return self._h

    @property
    def n(self) -> int:
        return self.info["n"]

    def to_host(self) -> dict:
        import numpy as np
        nb, nnz = self.info["nb"], self.info["nnz"]
        row_ptr = np.empty(nb + 1, dtype=np.int32)
        col_idx = np.empty(nnz, dtype=np.int32)
        count = np.empty(nnz, dtype=np.int32)
        flag = np.empty(nnz, dtype=np.uint8)
        check(ra_mask_copy_to_host(self.handle, row_ptr.ctypes.data, col_idx.ctypes.data, count.ctypes.data,
                                   flag.ctypes.data), "ra_mask_copy_to_host")
        return dict(row_ptr=row_ptr, col_idx=col_idx, count=count, flag=flag, nnz=nnz)

    def transpose_to_host(self) -> dict:
        """The transposed block-CSR: col_ptr, row_idx, tflag."""
        import numpy as np
        nb, nnz = self.info["nb"], self.info["nnz"]
        col_ptr = np.empty(nb + 1, dtype=np.int32)
        row_idx = np.empty(nnz, dtype=np.int32)
        tflag = np.empty(nnz, dtype=np.uint8)
        check(ra_mask_copy_transpose_to_host(self.handle, col_ptr.ctypes.data, row_idx.ctypes.data,
                                             tflag.ctypes.data), "ra_mask_copy_transpose_to_host")
        return dict(col_ptr=col_ptr, row_idx=row_idx, tflag=tflag)

    def free(self) -> None:
        if getattr(self, "_h", None) is not None:
            ra_mask_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def build_mask(mask: dict, f: int, s: int, grid=(0, 0), stream=None) -> Mask:
    """Mask from a dict {family, r_t, r_s, window_frames, sink_tokens} (grid used by window3d)."""
    return Mask(mask["family"], f, s, grid[0], grid[1], mask.get("r_t", 0), mask.get("r_s", 0),
                mask.get("window_frames", 0), mask.get("sink_tokens", 0), stream=stream)


# --------------------------------------------------------------- attention
def _check_bf16_cuda(name, t):
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def attention_fwd(q, k, v, mask: Mask, scale: float | None = None, mode="block", out=None, lse=None, stream=None):
    """O = softmax(scale * q k^T + M) v over the mask's kept tiles; q, k, v bf16 [B, H, n, d]."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16_cuda(name, t)
    B, H, n, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or n != mask.n:
        raise ValueError("q, k, v must share shape [B, H, n, d] with n equal to the mask's n")
    if out is None:
        out = torch.empty_like(q)
    _check_bf16_cuda("out", out)
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, n) or not lse.is_contiguous()):
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, n]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    mode = MODES[mode] if isinstance(mode, str) else int(mode)
    check(ra_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, d, mask.handle, scale,
                           mode, None if lse is None else lse.data_ptr(), _stream_handle(stream)),
          "ra_attention_fwd")
    return out


def attention_fwd_host(q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, mask: Mask,
                       scale: float | None = None, mode="block", stream=None):
    """Same call with host inputs / output: enqueues H2D copies, the kernel and the D2H copy."""
    B, H, n, d = q_host.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    mode = MODES[mode] if isinstance(mode, str) else int(mode)
    check(ra_attention_fwd_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), o_host.data_ptr(),
                                q_dev.data_ptr(), k_dev.data_ptr(), v_dev.data_ptr(), o_dev.data_ptr(), B, H, d,
                                mask.handle, scale, mode, _stream_handle(stream)), "ra_attention_fwd_host")
    return o_host


def attention_bwd(q, k, v, out, dout, lse, mask: Mask, scale: float | None = None, mode="block",
                  dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attention_fwd given its output `out`, its fp32 `lse` and the
    output gradient `dout` (all bf16 [B, H, n, d] except lse [B, H, n])."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _check_bf16_cuda(name, t)
    B, H, n, d = q.shape
    if any(t.shape != q.shape for t in (k, v, out, dout)) or n != mask.n:
        raise ValueError("q, k, v, out, dout must share shape [B, H, n, d] with n equal to the mask's n")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, n) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, n]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_bf16_cuda(name, t)
        if t.shape != q.shape:
            raise ValueError(f"{name} must have shape [B, H, n, d]")
    if workspace is None:
        workspace = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    if workspace.dtype != torch.float32 or workspace.numel() < B * H * n or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous fp32 tensor of at least B * H * n elements")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    mode = MODES[mode] if isinstance(mode, str) else int(mode)
    check(ra_attention_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                           lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                           B, H, d, mask.handle, scale, mode, _stream_handle(stream)), "ra_attention_bwd")
    return dq, dk, dv


class SwcCache:
    """Streaming sliding-window causal attention with a key/value ring cache of
    `window_frames` frames of `s` tokens for B x H heads of d channels."""

    def __init__(self, B: int, H: int, d: int, s: int, window_frames: int):
        h = ctypes.c_void_p()
        check(ra_swc_cache_create(B, H, d, s, window_frames, ctypes.byref(h)), "ra_swc_cache_create")
        self._h = h
        self.B, self.H, self.d, self.s, self.W = B, H, d, s, window_frames

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("cache was freed")
        return self._h

    def step(self, q, k, v, out=None, lse=None, scale: float | None = None, stream=None):
        """Feed the next frame (q, k, v bf16 [B, H, s, d]); returns its output."""
        import torch
        for name, t in (("q", q), ("k", k), ("v", v)):
            _check_bf16_cuda(name, t)
            if tuple(t.shape) != (self.B, self.H, self.s, self.d):
                raise ValueError(f"{name} must have shape [B, H, s, d]")
        if out is None:
            out = torch.empty_like(q)
        _check_bf16_cuda("out", out)
        if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (self.B, self.H, self.s)
                                or not lse.is_contiguous()):
            raise ValueError("lse must be a contiguous fp32 tensor [B, H, s]")
        scale = 1.0 / math.sqrt(self.d) if scale is None else float(scale)
        check(ra_swc_cache_step(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), scale,
                                None if lse is None else lse.data_ptr(), _stream_handle(stream)), "ra_swc_cache_step")
        return out

    @property
    def info(self) -> dict:
        seen, held = ctypes.c_longlong(), ctypes.c_int()
        check(ra_swc_cache_info(self.handle, ctypes.byref(seen), ctypes.byref(held)), "ra_swc_cache_info")
        return dict(frames_seen=seen.value, frames_held=held.value)

    def rings_to_host(self):
        """(K ring, V ring) as uint16 bf16 bit patterns [B, H, W * s, d]; frame i in slot i mod W."""
        import numpy as np
        shape = (self.B, self.H, self.W * self.s, self.d)
        k, v = np.empty(shape, dtype=np.uint16), np.empty(shape, dtype=np.uint16)
        check(ra_swc_cache_copy_rings_to_host(self.handle, k.ctypes.data, v.ctypes.data),
              "ra_swc_cache_copy_rings_to_host")
        return k, v

    def reset(self) -> None:
        check(ra_swc_cache_reset(self.handle), "ra_swc_cache_reset")

    def free(self) -> None:
        if getattr(self, "_h", None) is not None:
            ra_swc_cache_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class DenseFirstPolicy:
    """Which mask a denoising step uses in each attention block: dense for the
    first `dense_steps` steps (warm-up) and, at every step, for the first
    `dense_blocks` blocks; the sparse mask elsewhere ("Radial Attention",
    sec. 6: the first 2 DiT blocks and the first 12 denoising steps stay dense)."""

    def __init__(self, sparse: Mask, dense: Mask, dense_steps: int = 12, dense_blocks: int = 2):
        if dense_steps < 0 or dense_blocks < 0:
            raise ValueError("dense_steps and dense_blocks must be >= 0")
        if sparse.n != dense.n:
            raise ValueError("both masks must cover the same tokens")
        self.sparse, self.dense = sparse, dense
        self.dense_steps, self.dense_blocks = dense_steps, dense_blocks

    def is_dense(self, step: int, block: int) -> bool:
        return step < self.dense_steps or block < self.dense_blocks

    def mask(self, step: int, block: int) -> Mask:
        return self.dense if self.is_dense(step, block) else self.sparse

    def dense_calls(self, steps: int, blocks: int) -> int:
        """Dense calls in a schedule of `steps` x `blocks` attention calls."""
        warm = min(self.dense_steps, steps)
        return warm * blocks + (steps - warm) * min(self.dense_blocks, blocks)


def device_status(stream=None) -> int:
    """Synchronise and read (then clear) the device error word; returns the status code."""
    return ra_get_device_status(_stream_handle(stream))
