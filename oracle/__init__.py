"""Plain CPU oracle for static-mask sparse attention (ctypes wrapper of radattn_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in __graft_entry__.py
and bench.py's cpu_baseline / reference arm may import this package.  The
product path (static_sparse_attention_b200) never imports it and has no CPU
fallback.

What it computes (page title, section / equation):
  * "Radial Attention: O(n log n) Sparse Attention with Energy Decay for Long
    Video Generation": eq. 2 (masked softmax attention, M in {0, -inf}),
    eq. 4 (radial mask), eq. 3 (token index j*s + l), sec. 6 (128x128 tiles).
  * "Token Radius Attention" tutorial, sec. 3.2 / 4.2 / 5: cube neighbourhood.
  * "Vera 1.1" temporal module, sec. 2.2: causal sliding window of W frames.

Every function here is pinned by tests/test_oracle_pins.py to something other
than itself: a literal floating-point transcription of eq. 4, counts printed on
the tutorial page, closed forms, symmetry, the eq. 5-6 bound, brute-force numpy
enumeration, and torch's scaled_dot_product_attention in fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "radattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None
_lock = threading.Lock()

TILE = 128
DENSE, RADIAL, WINDOW3D, SWC = 0, 1, 2, 3
TOKEN_EXACT, BLOCK = 0, 1
TILE_PARTIAL, TILE_FULL = 0, 1
_FAMILIES = {"dense": DENSE, "radial": RADIAL, "window3d": WINDOW3D, "swc": SWC}
_IN_DTYPES = {np.dtype(np.uint16): 0, np.dtype(np.float32): 1, np.dtype(np.float64): 2}


class _Spec(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int), ("f", ctypes.c_int), ("s", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("r_t", ctypes.c_int),
                ("r_s", ctypes.c_int), ("window_frames", ctypes.c_int), ("sink_tokens", ctypes.c_int)]


@dataclass(frozen=True)
class MaskSpec:
    family: int
    f: int
    s: int
    grid_h: int = 0
    grid_w: int = 0
    r_t: int = 0
    r_s: int = 0
    window_frames: int = 0
    sink_tokens: int = 0

    @property
    def n(self) -> int:
        return self.f * self.s

    @property
    def nb(self) -> int:
        return (self.n + TILE - 1) // TILE

    def c(self) -> _Spec:
        return _Spec(self.family, self.f, self.s, self.grid_h, self.grid_w, self.r_t, self.r_s,
                     self.window_frames, self.sink_tokens)


def spec_from(mask: dict, f: int, s: int, grid=(0, 0)) -> MaskSpec:
    """MaskSpec from a workload mask entry (see synth.CONFIGS)."""
    fam = _FAMILIES[mask["family"]]
    gh, gw = grid if fam == WINDOW3D else (0, 0)
    return MaskSpec(fam, f, s, gh, gw, mask.get("r_t", 0), mask.get("r_s", 0),
                    mask.get("window_frames", 0), mask.get("sink_tokens", 0))


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle (gcc -O2, OpenMP).  Building the checker is not using it."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def load_library(path: str):
    """Bind the oracle's C entry points from a built shared library."""
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(_Spec)
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int
    lib.oracle_threads.restype = c_int
    lib.oracle_kept.argtypes = [P, i64, i64]
    lib.oracle_kept.restype = c_int
    lib.oracle_dense_mask.argtypes = [P, vp]
    lib.oracle_dense_mask.restype = None
    lib.oracle_kept_total.argtypes = [P]
    lib.oracle_kept_total.restype = i64
    lib.oracle_tile_counts.argtypes = [P, vp, c_int, vp]
    lib.oracle_tile_counts.restype = None
    lib.oracle_csr.argtypes = [vp, i64, vp, vp, vp, vp]
    lib.oracle_csr.restype = i64
    lib.oracle_attention_rows.argtypes = [vp, vp, vp, c_int, i64, c_int, P, c_int, ctypes.c_double, i64,
                                          vp, vp, vp, vp, vp, vp, vp]
    lib.oracle_attention_rows.restype = None
    lib.oracle_attention_bwd.argtypes = [vp, vp, vp, vp, c_int, i64, c_int, P, c_int, ctypes.c_double, vp, vp, vp,
                                         vp]
    lib.oracle_attention_bwd.restype = None
    lib.oracle_set_threads.argtypes = [c_int]
    lib.oracle_set_threads.restype = None
    lib.oracle_attention_bwd_query_rows.argtypes = [vp, vp, vp, vp, c_int, i64, c_int, P, c_int, ctypes.c_double,
                                                    i64, vp, vp, vp, vp, vp, vp]
    lib.oracle_attention_bwd_query_rows.restype = None
    lib.oracle_attention_bwd_key_rows.argtypes = [vp, vp, vp, vp, c_int, i64, c_int, P, c_int, ctypes.c_double,
                                                  vp, i64, vp, vp, vp]
    lib.oracle_attention_bwd_key_rows.restype = None
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB_PATH)
    return _lib


class Oracle:
    """The oracle's operations, bound to one built library (the default, or a
    test's deliberately broken copy)."""

    def __init__(self, lib):
        self.lib = lib

    def threads(self) -> int:
        return self.lib.oracle_threads()

    def set_threads(self, n: int) -> None:
        """Threads of the oracle's parallel loops from now on (timing only; results do not change)."""
        self.lib.oracle_set_threads(int(n))

    def kept(self, spec: MaskSpec, q: int, key: int) -> int:
        sp = spec.c()
        return self.lib.oracle_kept(ctypes.byref(sp), q, key)

    def dense_mask(self, spec: MaskSpec) -> np.ndarray:
        """n x n uint8 token mask (1 = kept), row = query.  Small n only."""
        out = np.empty((spec.n, spec.n), dtype=np.uint8)
        sp = spec.c()
        self.lib.oracle_dense_mask(ctypes.byref(sp), out.ctypes.data)
        return out

    def kept_total(self, spec: MaskSpec) -> int:
        sp = spec.c()
        return int(self.lib.oracle_kept_total(ctypes.byref(sp)))

    def tile_counts(self, spec: MaskSpec, qbs=None) -> np.ndarray:
        """Kept pairs per 128x128 tile for the listed query tiles: [len(qbs), nb] int32."""
        qbs = np.arange(spec.nb, dtype=np.int32) if qbs is None else np.ascontiguousarray(qbs, dtype=np.int32)
        out = np.empty((len(qbs), spec.nb), dtype=np.int32)
        sp = spec.c()
        self.lib.oracle_tile_counts(ctypes.byref(sp), qbs.ctypes.data, len(qbs), out.ctypes.data)
        return out

    def csr(self, spec: MaskSpec, counts: np.ndarray | None = None) -> dict:
        """Block-CSR of kept tiles: row_ptr, col_idx, count, flag (int32/int32/int32/uint8)."""
        if counts is None:
            counts = self.tile_counts(spec)
        counts = np.ascontiguousarray(counts, dtype=np.int32)
        nnz = int(self.lib.oracle_csr(counts.ctypes.data, spec.n, None, None, None, None))
        row_ptr = np.empty(spec.nb + 1, dtype=np.int32)
        col_idx = np.empty(nnz, dtype=np.int32)
        count = np.empty(nnz, dtype=np.int32)
        flag = np.empty(nnz, dtype=np.uint8)
        self.lib.oracle_csr(counts.ctypes.data, spec.n, row_ptr.ctypes.data, col_idx.ctypes.data,
                            count.ctypes.data, flag.ctypes.data)
        return dict(row_ptr=row_ptr, col_idx=col_idx, count=count, flag=flag, nnz=nnz)

    def attention_rows(self, Q, K, V, spec: MaskSpec, mode: int, scale: float, row_bh, row_q):
        """fp64 masked softmax attention for the listed rows.

        Q, K, V: [B, H, n, d] arrays of bf16 bit patterns (uint16), float32 or
        float64.  Returns (O [rows, d] fp64, lse [rows] fp64, nkeys [rows] int64)."""
        Q, K, V = (np.ascontiguousarray(t) for t in (Q, K, V))
        assert Q.dtype == K.dtype == V.dtype and Q.dtype in _IN_DTYPES
        n, d = Q.shape[-2], Q.shape[-1]
        assert n == spec.n
        row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
        row_q = np.ascontiguousarray(row_q, dtype=np.int64)
        nrows = len(row_q)
        if mode == BLOCK:
            qbs, slot = np.unique(row_q // TILE, return_inverse=True)
            tile_flags = (self.tile_counts(spec, qbs) > 0).astype(np.uint8)
            slot = np.ascontiguousarray(slot, dtype=np.int32)
        else:
            tile_flags = np.zeros(1, dtype=np.uint8)
            slot = np.zeros(max(nrows, 1), dtype=np.int32)
        O = np.empty((nrows, d), dtype=np.float64)
        lse = np.empty(nrows, dtype=np.float64)
        nkeys = np.empty(nrows, dtype=np.int64)
        sp = spec.c()
        self.lib.oracle_attention_rows(Q.ctypes.data, K.ctypes.data, V.ctypes.data, _IN_DTYPES[Q.dtype], n, d,
                                       ctypes.byref(sp), mode, float(scale), nrows, row_bh.ctypes.data,
                                       row_q.ctypes.data, tile_flags.ctypes.data, slot.ctypes.data,
                                       O.ctypes.data, lse.ctypes.data, nkeys.ctypes.data)
        return O, lse, nkeys

    def attention_bwd(self, Q, K, V, dO, spec: MaskSpec, mode: int, scale: float):
        """fp64 gradients dQ, dK, dV of the masked attention for every (b, h) slice.

        Q, K, V, dO: [B, H, n, d] arrays (bf16 bit patterns, float32 or float64).
        Returns three float64 arrays of the same shape.  O(B H n^2 d): small n only."""
        Q, K, V, dO = (np.ascontiguousarray(t) for t in (Q, K, V, dO))
        assert Q.dtype == K.dtype == V.dtype == dO.dtype and Q.dtype in _IN_DTYPES
        B, H, n, d = Q.shape
        assert n == spec.n
        flags = (self.tile_counts(spec) > 0).astype(np.uint8) if mode == BLOCK else np.zeros(1, np.uint8)
        out = [np.empty((B, H, n, d), dtype=np.float64) for _ in range(3)]
        sp = spec.c()
        for b in range(B):
            for h in range(H):
                self.lib.oracle_attention_bwd(Q[b, h].ctypes.data, K[b, h].ctypes.data, V[b, h].ctypes.data,
                                              dO[b, h].ctypes.data, _IN_DTYPES[Q.dtype], n, d, ctypes.byref(sp), mode,
                                              float(scale), flags.ctypes.data, out[0][b, h].ctypes.data,
                                              out[1][b, h].ctypes.data, out[2][b, h].ctypes.data)
        return tuple(out)


    def attention_bwd_query_rows(self, Q, K, V, dO, spec: MaskSpec, mode: int, scale: float, row_bh, row_q,
                                 return_nkeys: bool = False):
        """fp64 dQ of the listed query rows (b*H + h, q); [rows, d].  O(keys * d) per row.
        With return_nkeys, also each row's key count."""
        Q, K, V, dO = (np.ascontiguousarray(t) for t in (Q, K, V, dO))
        assert Q.dtype == K.dtype == V.dtype == dO.dtype and Q.dtype in _IN_DTYPES
        n, d = Q.shape[-2], Q.shape[-1]
        assert n == spec.n
        row_bh = np.ascontiguousarray(row_bh, dtype=np.int64)
        row_q = np.ascontiguousarray(row_q, dtype=np.int64)
        nrows = len(row_q)
        if mode == BLOCK:
            qbs, slot = np.unique(row_q // TILE, return_inverse=True)
            tile_flags = (self.tile_counts(spec, qbs) > 0).astype(np.uint8)
            slot = np.ascontiguousarray(slot, dtype=np.int32)
        else:
            tile_flags = np.zeros(1, dtype=np.uint8)
            slot = np.zeros(max(nrows, 1), dtype=np.int32)
        dQ = np.empty((nrows, d), dtype=np.float64)
        nkeys = np.empty(max(nrows, 1), dtype=np.int64)
        sp = spec.c()
        self.lib.oracle_attention_bwd_query_rows(Q.ctypes.data, K.ctypes.data, V.ctypes.data, dO.ctypes.data,
                                                 _IN_DTYPES[Q.dtype], n, d, ctypes.byref(sp), mode, float(scale),
                                                 nrows, row_bh.ctypes.data, row_q.ctypes.data,
                                                 tile_flags.ctypes.data, slot.ctypes.data, dQ.ctypes.data,
                                                 nkeys.ctypes.data)
        return (dQ, nkeys[:nrows]) if return_nkeys else dQ

    def attention_bwd_key_rows(self, Q, K, V, dO, spec: MaskSpec, mode: int, scale: float, keys):
        """fp64 dK, dV of the listed key rows of ONE (b, h) slice: Q, K, V, dO are
        [n, d].  Returns ([len(keys), d], [len(keys), d]).  O(n * keys-per-row * d)."""
        Q, K, V, dO = (np.ascontiguousarray(t) for t in (Q, K, V, dO))
        assert Q.dtype == K.dtype == V.dtype == dO.dtype and Q.dtype in _IN_DTYPES and Q.ndim == 2
        n, d = Q.shape
        assert n == spec.n
        keys = np.ascontiguousarray(keys, dtype=np.int64)
        if mode == BLOCK:
            tile_flags = np.ascontiguousarray((self.tile_counts(spec) > 0).astype(np.uint8))
        else:
            tile_flags = np.zeros(1, dtype=np.uint8)
        dK = np.empty((len(keys), d), dtype=np.float64)
        dV = np.empty((len(keys), d), dtype=np.float64)
        sp = spec.c()
        self.lib.oracle_attention_bwd_key_rows(Q.ctypes.data, K.ctypes.data, V.ctypes.data, dO.ctypes.data,
                                               _IN_DTYPES[Q.dtype], n, d, ctypes.byref(sp), mode, float(scale),
                                               tile_flags.ctypes.data, len(keys), keys.ctypes.data,
                                               dK.ctypes.data, dV.ctypes.data)
        return dK, dV


def default() -> Oracle:
    return Oracle(_load())
