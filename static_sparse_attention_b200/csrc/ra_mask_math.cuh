// ra_mask_math.cuh -- the static mask families as per-row key intervals.
//
// Token index = frame * s + position ("Radial Attention ..." eq. 3: p_{js+l});
// for the 3D window, position = h * grid_w + w ("Token Radius Attention"
// sec. 3.1, tokens flattened as (t h w)).
//
// For one query row (frame i, position k) the kept keys inside one key frame
// form a single interval for the radial mask, the sliding window and the dense
// mask, and one interval per grid row for the 3D window.  Enumerating those
// intervals over a range of key columns gives both the per-tile kept count
// (mask builder) and the per-row 128-bit keep mask of a partial tile (forward
// kernel), with integer arithmetic only.
#pragma once
#include <cstdint>

namespace ra {

enum : int { FAM_DENSE = 0, FAM_RADIAL = 1, FAM_WINDOW3D = 2, FAM_SWC = 3 };
constexpr int TILE = 128;

struct MaskGeom {
    int family;
    int f, s, n;  // frames, tokens per frame, n = f * s
    int grid_h, grid_w, r_t, r_s;
    int window_frames;
    int sink;  // tokens [0, sink) are global: kept in every row and every column
};

// The family's own runs (no global tokens): calls emit(a, b) for every maximal
// run [a, b] of kept keys of query row (frame qi, position qk) inside the key
// columns [c0, c1] (0 <= c0 <= c1 < n), in ascending order, never overlapping.
template <class Emit>
__device__ __forceinline__ void for_each_family_run(const MaskGeom& g, int qi, int qk, int c0, int c1, Emit&& emit)
{
    const int s = g.s;
    const int j0 = c0 / s, j1 = c1 / s;
    switch (g.family) {
    case FAM_DENSE:
        emit(c0, c1);
        return;
    case FAM_SWC: {
        // "Vera 1.1" sec. 2.2: key frames max(0, i-W+1) .. i, every position.
        const int lo = max(j0, qi - g.window_frames + 1), hi = min(j1, qi);
        if (lo <= hi)
            emit(max(c0, lo * s), min(c1, hi * s + s - 1));
        return;
    }
    case FAM_RADIAL: {
        // eq. 4: with D = |i-j| and w = 2^floor(log2 max(D,1)):
        //   w <= s : keep |k-l| + 1 <= s / w, i.e. |k-l| <= floor(s/w) - 1
        //            (the k == l case is inside that band);
        //   w >  s : keep l == k when D mod ceil(w/s) == 0.
        for (int j = j0; j <= j1; ++j) {
            const int D = qi > j ? qi - j : j - qi;
            const unsigned w = 1u << (31 - __clz(D > 1 ? D : 1));
            int lo, hi;
            if (w <= static_cast<unsigned>(s)) {
                const int r = static_cast<int>(static_cast<unsigned>(s) / w) - 1;
                lo = max(qk - r, 0);
                hi = min(qk + r, s - 1);
            } else {
                const unsigned period = (w + static_cast<unsigned>(s) - 1u) / static_cast<unsigned>(s);
                if (static_cast<unsigned>(D) % period != 0u)
                    continue;
                lo = hi = qk;
            }
            const int a = max(c0, j * s + lo), b = min(c1, j * s + hi);
            if (a <= b)
                emit(a, b);
        }
        return;
    }
    case FAM_WINDOW3D: {
        // "Token Radius Attention" sec. 3.2 / 4.2: |dt| <= r_t, |dh| <= r_s,
        // |dw| <= r_s, neighbours outside the grid are absent.
        const int W = g.grid_w;
        const int qh = qk / W, qw = qk % W;
        const int wlo = max(qw - g.r_s, 0), whi = min(qw + g.r_s, W - 1);
        const int jlo = max(j0, qi - g.r_t), jhi = min(j1, qi + g.r_t);
        for (int j = jlo; j <= jhi; ++j) {
            const int base = j * s;
            int hlo = max(qh - g.r_s, 0), hhi = min(qh + g.r_s, g.grid_h - 1);
            hlo = max(hlo, (max(c0, base) - base) / W);
            hhi = min(hhi, (min(c1, base + s - 1) - base) / W);
            for (int h = hlo; h <= hhi; ++h) {
                const int a = max(c0, base + h * W + wlo), b = min(c1, base + h * W + whi);
                if (a <= b)
                    emit(a, b);
            }
        }
        return;
    }
    default:
        return;
    }
}

// Calls emit(a, b) for every maximal run [a, b] of kept keys of query row
// (frame qi, position qk) inside the key columns [c0, c1] (0 <= c0 <= c1 < n),
// in ascending order, never overlapping.  Global (sink) tokens first: a sink
// query keeps every key; other queries keep the sink keys and then the
// family's keys beyond them.
template <class Emit>
__device__ __forceinline__ void for_each_kept_run(const MaskGeom& g, int qi, int qk, int c0, int c1, Emit&& emit)
{
    if (g.sink > 0) {
        if (qi * g.s + qk < g.sink) {
            emit(c0, c1);
            return;
        }
        if (c0 < g.sink) {
            emit(c0, min(c1, g.sink - 1));
            c0 = g.sink;
            if (c0 > c1)
                return;
        }
    }
    for_each_family_run(g, qi, qk, c0, c1, emit);
}

// Number of kept keys of a query row inside [c0, c1].
__device__ __forceinline__ int kept_in_range(const MaskGeom& g, int qi, int qk, int c0, int c1)
{
    int total = 0;
    for_each_kept_run(g, qi, qk, c0, c1, [&](int a, int b) { total += b - a + 1; });
    return total;
}

// Bits [lo, hi] (0 <= lo <= hi <= 31) set.
__device__ __forceinline__ uint32_t bit_range(int lo, int hi)
{
    const uint32_t upto_hi = (hi >= 31) ? 0xFFFFFFFFu : ((2u << hi) - 1u);
    return upto_hi & ~((1u << lo) - 1u);
}

// 128-bit keep mask of a query row over the tile's columns [c0, c0 + 127]
// (columns >= n are never set).  Bit t of word w <-> column c0 + 32 w + t.
__device__ __forceinline__ void row_keep_mask(const MaskGeom& g, int qi, int qk, int c0, uint32_t& m0, uint32_t& m1,
                                              uint32_t& m2, uint32_t& m3)
{
    m0 = m1 = m2 = m3 = 0u;
    const int c1 = min(c0 + TILE - 1, g.n - 1);
    for_each_kept_run(g, qi, qk, c0, c1, [&](int a, int b) {
        const int lo = a - c0, hi = b - c0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int l = max(lo, 32 * w), h = min(hi, 32 * w + 31);
            if (l <= h) {
                const uint32_t bits = bit_range(l - 32 * w, h - 32 * w);
                if (w == 0) m0 |= bits;
                else if (w == 1) m1 |= bits;
                else if (w == 2) m2 |= bits;
                else m3 |= bits;
            }
        }
    });
}

// The same for a key column: emit(a, b) for every maximal run of queries
// [a, b] inside [c0, c1] that keep key (frame kj, position kk).  The radial
// mask (|i-j|, |k-l|), the 3D window (|dt|, |dh|, |dw|), the dense mask and the
// global tokens are symmetric, so a key's queries are its own row's keys; the
// causal sliding window keeps query frames kj .. kj + W - 1.
template <class Emit>
__device__ __forceinline__ void for_each_kept_query_run(const MaskGeom& g, int kj, int kk, int c0, int c1,
                                                        Emit&& emit)
{
    if (g.family != FAM_SWC) {
        for_each_kept_run(g, kj, kk, c0, c1, emit);
        return;
    }
    if (g.sink > 0) {
        if (kj * g.s + kk < g.sink) {
            emit(c0, c1);
            return;
        }
        if (c0 < g.sink) {
            emit(c0, min(c1, g.sink - 1));
            c0 = g.sink;
            if (c0 > c1)
                return;
        }
    }
    const int s = g.s;
    const int lo = max(c0 / s, kj), hi = min(c1 / s, kj + g.window_frames - 1);
    if (lo <= hi)
        emit(max(c0, lo * s), min(c1, hi * s + s - 1));
}

// 128-bit keep mask of a key column over the query rows [c0, c0 + 127].
__device__ __forceinline__ void col_keep_mask(const MaskGeom& g, int kj, int kk, int c0, uint32_t& m0, uint32_t& m1,
                                              uint32_t& m2, uint32_t& m3)
{
    m0 = m1 = m2 = m3 = 0u;
    const int c1 = min(c0 + TILE - 1, g.n - 1);
    for_each_kept_query_run(g, kj, kk, c0, c1, [&](int a, int b) {
        const int lo = a - c0, hi = b - c0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int l = max(lo, 32 * w), h = min(hi, 32 * w + 31);
            if (l <= h) {
                const uint32_t bits = bit_range(l - 32 * w, h - 32 * w);
                if (w == 0) m0 |= bits;
                else if (w == 1) m1 |= bits;
                else if (w == 2) m2 |= bits;
                else m3 |= bits;
            }
        }
    });
}

}  // namespace ra
