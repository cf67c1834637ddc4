"""The seeded input generator (synth/) against the published definitions it
restates -- SplitMix64's output sequence, the Box-Muller transform, fp32 -> bf16
round-to-nearest-even -- and the properties every workload relies on (counter
access, moments, independent streams).  CPU only."""
import ctypes
import math

import numpy as np
import pytest

import synth

GAMMA = 0x9E3779B97F4A7C15
M64 = (1 << 64) - 1


def _mix(z: int) -> int:
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


@pytest.fixture(scope="module")
def lib():
    lib = synth._load()
    lib.synth_draw.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    lib.synth_draw.restype = ctypes.c_uint64
    lib.synth_stream_start.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    lib.synth_stream_start.restype = ctypes.c_uint64
    return lib


def test_splitmix64_sequence(lib):
    """The first five SplitMix64 outputs from state 1234567, the seed that
    implementations of the generator are commonly checked with; draw t of a stream
    is its (t + 1)-th sequential output."""
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423, 4593380528125082431,
            16408922859458223821]
    assert [lib.synth_draw(1234567, t) for t in range(5)] == want


def test_normals_follow_box_muller(lib):
    """Element e of stream (seed, tensor) is z0 (e even) or z1 (e odd) of the
    Box-Muller pair built from draws 2 (e / 2) and 2 (e / 2) + 1, rounded to fp32."""
    seed, tensor = 20261202, 7
    start = _mix((seed + (tensor + 1) * GAMMA) & M64)
    assert lib.synth_stream_start(seed, tensor) == start
    got = synth.normal_f32(seed, tensor, (96,))
    want = np.empty(96, dtype=np.float32)
    for e in range(96):
        p = e >> 1
        a = _mix((start + (2 * p + 1) * GAMMA) & M64)
        b = _mix((start + (2 * p + 2) * GAMMA) & M64)
        u1 = ((a >> 11) + 1) / 2.0**53   # (0, 1]
        u2 = (b >> 11) / 2.0**53         # [0, 1)
        r = math.sqrt(-2.0 * math.log(u1))
        want[e] = np.float32(r * (math.sin(2 * math.pi * u2) if e & 1 else math.cos(2 * math.pi * u2)))
    # libm may differ from Python's math in the last bit of a double: allow one fp32 ulp
    np.testing.assert_array_max_ulp(got, want, maxulp=1)


def test_bf16_round_to_nearest_even():
    """Ties go to the even bf16 pattern, everything else to the nearest."""
    bits = np.array([0x3F800000, 0x3F808000, 0x3F818000, 0x3F807FFF, 0x3F808001, 0xBF808000, 0xBF818000,
                     0x00000000, 0x80000000, 0x7F7FFFFF, 0x3F7FFFFF], dtype=np.uint32)
    want = np.array([0x3F80, 0x3F80, 0x3F82, 0x3F80, 0x3F81, 0xBF80, 0xBF82,
                     0x0000, 0x8000, 0x7F80, 0x3F80], dtype=np.uint16)
    got = synth.round_bf16(bits.view(np.float32))
    np.testing.assert_array_equal(got, want)
    # the bf16 stream is the rounding of the fp32 stream
    f = synth.normal_f32(3, 1, (4096,))
    np.testing.assert_array_equal(synth.normal_bf16(3, 1, (4096,)), synth.round_bf16(f))
    # widening is exact
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(want[:7]),
                                  np.array([1.0, 1.0, 1.015625, 1.0, 1.0078125, -1.0, -1.015625], np.float32))


def test_counter_access(lib):
    """Any run of elements can be drawn on its own (the oracle and the kernels'
    inputs never need the whole tensor at once)."""
    whole = synth.normal_f32(11, 2, (1000,))
    part = np.empty(300, dtype=np.float32)
    lib.synth_normal(11, 2, 333, 300, part.ctypes.data, None)
    np.testing.assert_array_equal(part, whole[333:633])


def test_moments_and_independent_streams():
    n = 1 << 20
    q = synth.normal_f32(20261205, 0, (n,)).astype(np.float64)
    k = synth.normal_f32(20261205, 1, (n,)).astype(np.float64)
    q2 = synth.normal_f32(20261206, 0, (n,)).astype(np.float64)
    bound = 5.0 / math.sqrt(n)
    for x in (q, k, q2):
        assert abs(x.mean()) < bound
        assert abs(x.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
        assert abs(((x - x.mean()) ** 4).mean() / x.var() ** 2 - 3.0) < 0.05   # normal kurtosis
    for a, b in ((q, k), (q, q2), (k, q2)):
        assert abs(np.corrcoef(a, b)[0, 1]) < bound


@pytest.mark.parametrize("f,s", [(30, 3600), (41, 1560), (128, 3600), (1, 100), (3, 40)])
def test_sampled_rows_hold_the_boundary_rows(f, s):
    """The seeded rows the full-size parity tests check: distinct, sorted, in range,
    the requested count, the same for the same seed, and always including the
    boundary rows (sequence ends, frame 1's first and last row, the last frame's
    first row, the first row of the ragged last tile)."""
    n = f * s
    rows = synth.sample_rows(1234, f, s)
    assert rows.dtype == np.int64 and len(rows) == min(256, n)
    assert np.all(np.diff(rows) > 0) and rows[0] >= 0 and rows[-1] < n
    need = {0, n - 1, (f - 1) * s, ((n + 127) // 128 - 1) * 128}
    if f > 1:
        need |= {s, 2 * s - 1}
    assert need <= set(rows.tolist())
    np.testing.assert_array_equal(rows, synth.sample_rows(1234, f, s))
    assert not np.array_equal(rows, synth.sample_rows(1235, f, s)) or n <= 256


def test_head_slices_equal_the_full_tensor():
    """A rank's heads drawn on their own are the same elements as the slice of the
    whole tensor (B > 1, uneven ranges, empty range)."""
    shape = (2, 5, 37, 16)
    full = synth.normal_bf16(1234, 2, shape)
    for h0, h1 in [(0, 5), (0, 2), (2, 5), (3, 4), (4, 4)]:
        assert np.array_equal(synth.normal_bf16_heads(1234, 2, shape, h0, h1), full[:, h0:h1])
