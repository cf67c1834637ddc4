// ra_mask_build.cu -- block-CSR builder for the static masks (integer kernels).
//
// "Radial Attention ..." sec. 6 applies the mask at 128 x 128 tile granularity;
// the pages do not say how a token mask becomes a tile mask.  Reading used
// here: a tile (qb, kb) is kept iff at least one valid (query, key) pair in it
// is kept, its count is the number of kept valid pairs, and it is FULL iff
// count == 128 * 128 (so a tail tile is never FULL).
//
// Kernels:
//   tile_count_kernel  one CTA per query tile, one thread per query row; each
//                      row's kept keys in a key tile come from the interval
//                      form of the family (ra_mask_math.cuh), warp-reduced.
//                      Also per-row kept-tile totals and global statistics.
//   row_scan_kernel    exclusive scan of the per-row kept-tile counts -> row_ptr.
//   compact_kernel     kept tiles of each row in ascending column order.
#include <cuda_runtime.h>

#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <utility>
#include <vector>

#include "ra_internal.h"

namespace ra {
namespace {

// Global statistics written by tile_count_kernel.
struct BuildTotals {
    unsigned long long kept_pairs, block_pairs, full_tiles;
    int row_min, row_max;
};

__global__ void __launch_bounds__(128) tile_count_kernel(MaskGeom g, int nb, int* __restrict__ counts,
                                                         int* __restrict__ row_tiles, BuildTotals* __restrict__ tot)
{
    __shared__ int part[4][TILE];
    __shared__ unsigned long long red[3][4];
    __shared__ int red_tiles[4];
    const int qb = blockIdx.x, t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int q = qb * TILE + t;
    const bool valid = q < g.n;
    const int qi = valid ? q / g.s : 0, qk = valid ? q % g.s : 0;
    const int rows_valid = min(TILE, g.n - qb * TILE);

    unsigned long long kept = 0, block = 0, full = 0;
    int tiles = 0;
    for (int kb0 = 0; kb0 < nb; kb0 += TILE) {
        const int nk = min(TILE, nb - kb0);
        for (int u = 0; u < nk; ++u) {
            const int c0 = (kb0 + u) * TILE, c1 = min(c0 + TILE - 1, g.n - 1);
            int c = valid ? kept_in_range(g, qi, qk, c0, c1) : 0;
            c = __reduce_add_sync(0xFFFFFFFFu, c);
            if (lane == 0)
                part[warp][u] = c;
        }
        __syncthreads();
        if (t < nk) {
            const int kb = kb0 + t;
            const int c = part[0][t] + part[1][t] + part[2][t] + part[3][t];
            counts[static_cast<size_t>(qb) * nb + kb] = c;
            if (c > 0) {
                tiles += 1;
                kept += static_cast<unsigned long long>(c);
                block += static_cast<unsigned long long>(rows_valid) * min(TILE, g.n - kb * TILE);
                full += (c == TILE * TILE) ? 1ull : 0ull;
            }
        }
        __syncthreads();
    }
    // CTA reduction of the per-thread statistics.
    for (int o = 16; o > 0; o >>= 1) {
        kept += __shfl_xor_sync(0xFFFFFFFFu, kept, o);
        block += __shfl_xor_sync(0xFFFFFFFFu, block, o);
        full += __shfl_xor_sync(0xFFFFFFFFu, full, o);
        tiles += __shfl_xor_sync(0xFFFFFFFFu, tiles, o);
    }
    if (lane == 0) {
        red[0][warp] = kept;
        red[1][warp] = block;
        red[2][warp] = full;
        red_tiles[warp] = tiles;
    }
    __syncthreads();
    if (t == 0) {
        unsigned long long k = 0, b = 0, f = 0;
        int n_tiles = 0;
        for (int w = 0; w < 4; ++w) {
            k += red[0][w];
            b += red[1][w];
            f += red[2][w];
            n_tiles += red_tiles[w];
        }
        row_tiles[qb] = n_tiles;
        atomicAdd(&tot->kept_pairs, k);
        atomicAdd(&tot->block_pairs, b);
        atomicAdd(&tot->full_tiles, f);
        atomicMin(&tot->row_min, n_tiles);
        atomicMax(&tot->row_max, n_tiles);
    }
}

// Exclusive scan of row_tiles[0, nb) into row_ptr[0, nb]; one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) row_scan_kernel(const int* __restrict__ row_tiles, int nb,
                                                        int* __restrict__ row_ptr)
{
    __shared__ int warp_sums[32];
    __shared__ int carry_s;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (t == 0)
        carry_s = 0;
    __syncthreads();
    for (int base = 0; base < nb; base += 1024) {
        const int i = base + t;
        const int v = (i < nb) ? row_tiles[i] : 0;
        int x = v;  // inclusive warp scan
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
            if (lane >= o)
                x += y;
        }
        if (lane == 31)
            warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, w, o);
                if (lane >= o)
                    w += y;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        const int incl = x + (warp > 0 ? warp_sums[warp - 1] : 0);
        if (i < nb)
            row_ptr[i] = carry + incl - v;
        __syncthreads();
        if (t == 1023)
            carry_s = carry + incl;
        __syncthreads();
    }
    if (t == 0)
        row_ptr[nb] = carry_s;
}

__global__ void __launch_bounds__(128) compact_kernel(const int* __restrict__ counts, int nb,
                                                      const int* __restrict__ row_ptr, int* __restrict__ col_idx,
                                                      int* __restrict__ count, unsigned char* __restrict__ flag)
{
    __shared__ int warp_tot[4];
    const int qb = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    int out = row_ptr[qb];
    for (int kb0 = 0; kb0 < nb; kb0 += TILE) {
        const int kb = kb0 + t;
        const int c = (kb < nb) ? counts[static_cast<size_t>(qb) * nb + kb] : 0;
        const bool keep = c > 0;
        const unsigned ballot = __ballot_sync(0xFFFFFFFFu, keep);
        const int before = __popc(ballot & ((1u << lane) - 1u));
        if (lane == 0)
            warp_tot[warp] = __popc(ballot);
        __syncthreads();
        int warp_off = 0, chunk = 0;
        for (int w = 0; w < 4; ++w) {
            warp_off += (w < warp) ? warp_tot[w] : 0;
            chunk += warp_tot[w];
        }
        if (keep) {
            const int pos = out + warp_off + before;
            col_idx[pos] = kb;
            count[pos] = c;
            flag[pos] = (c == TILE * TILE) ? RA_TILE_FULL : RA_TILE_PARTIAL;
        }
        out += chunk;
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Scratch of ra_build_mask_noalloc.  Some callers cannot allocate device memory
// on demand (see the header); for them the builder's scratch -- the nb x nb
// tile counts, the per-row kept-tile counts and the statistics -- lives in this
// file-scope array, reserved on every device that loads the library.
constexpr int NOALLOC_MAX_NB = 1024;  // n <= 131072 tokens
constexpr size_t NOALLOC_COUNTS_BYTES = sizeof(int) * static_cast<size_t>(NOALLOC_MAX_NB) * NOALLOC_MAX_NB;
constexpr size_t NOALLOC_ROWS_BYTES = sizeof(int) * NOALLOC_MAX_NB;
constexpr size_t NOALLOC_SCRATCH_BYTES = NOALLOC_COUNTS_BYTES + NOALLOC_ROWS_BYTES + 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

__global__ void init_totals_kernel(BuildTotals* tot)
{
    tot->kept_pairs = 0;
    tot->block_pairs = 0;
    tot->full_tiles = 0;
    tot->row_min = INT_MAX;
    tot->row_max = 0;
}

// Kept query tiles per key tile (a column of the tile-count matrix).
__global__ void __launch_bounds__(128) col_count_kernel(const int* __restrict__ counts, int nb,
                                                        int* __restrict__ col_tiles)
{
    __shared__ int part[4];
    const int kb = blockIdx.x, t = threadIdx.x;
    int c = 0;
    for (int qb = t; qb < nb; qb += TILE)
        c += counts[static_cast<size_t>(qb) * nb + kb] > 0;
    c = __reduce_add_sync(0xFFFFFFFFu, c);
    if ((t & 31) == 0)
        part[t >> 5] = c;
    __syncthreads();
    if (t == 0)
        col_tiles[kb] = part[0] + part[1] + part[2] + part[3];
}

// Kept query tiles of each key tile in ascending order, with the tile's flag.
__global__ void __launch_bounds__(128) col_compact_kernel(const int* __restrict__ counts, int nb,
                                                          const int* __restrict__ col_ptr, int* __restrict__ row_idx,
                                                          unsigned char* __restrict__ tflag)
{
    __shared__ int warp_tot[4];
    const int kb = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    int out = col_ptr[kb];
    for (int qb0 = 0; qb0 < nb; qb0 += TILE) {
        const int qb = qb0 + t;
        const int c = (qb < nb) ? counts[static_cast<size_t>(qb) * nb + kb] : 0;
        const bool keep = c > 0;
        const unsigned ballot = __ballot_sync(0xFFFFFFFFu, keep);
        const int before = __popc(ballot & ((1u << lane) - 1u));
        if (lane == 0)
            warp_tot[warp] = __popc(ballot);
        __syncthreads();
        int warp_off = 0, chunk = 0;
        for (int w = 0; w < 4; ++w) {
            warp_off += (w < warp) ? warp_tot[w] : 0;
            chunk += warp_tot[w];
        }
        if (keep) {
            const int pos = out + warp_off + before;
            row_idx[pos] = qb;
            tflag[pos] = (c == TILE * TILE) ? RA_TILE_FULL : RA_TILE_PARTIAL;
        }
        out += chunk;
        __syncthreads();
    }
}

// Frames from which the forward walks a radial mask's near frames first, and their reach.
constexpr int WALK_MIN_FRAMES = 64;
inline int walk_near_frames(const MaskGeom& g) { return g.f / 4; }
inline bool walked(const MaskGeom& g) { return g.family == FAM_RADIAL && g.f >= WALK_MIN_FRAMES; }

// The order in which the attention kernels' CTAs take their tiles (query tiles
// of the forward and the dQ pass, key tiles of the dK / dV pass, by the mask's
// symmetry in query and key): sorted by in-frame position band, then by frame.  eq. 4 keeps, in every key frame, a band of
// positions centred on the query's own in-frame position, so query tiles of one
// position band over many frames read overlapping key tiles; with the query
// tiles of a head in plain order the resident CTAs instead cover a few whole
// frames, i.e. every position, and at long sequences (a head's K and V well
// beyond the L2 cache) re-read most key tiles from DRAM.  The order is used from
// about 4.5 query tiles per SM (2.25 times the forward's resident CTAs) on, with
// bands of about three query tiles per SM, or four for the masks whose rows the
// forward walks near frames first (walk_kernel below; measured with that walk),
// and at least two bands; smaller masks, and frames shorter than two tiles, keep
// the plain order.  Returns false when the order is the identity.
bool dispatch_order(const MaskGeom& g, int nb, int sm_count, bool walk_rows, std::vector<int>& order)
{
    const long long sms = sm_count > 0 ? sm_count : 148;
    if (g.s < 2 * TILE || (nb + 3 * sms / 2) / (3 * sms) < 2)
        return false;
    const long long per_band = (walk_rows ? 4 : 3) * sms;
    const int bands = static_cast<int>(std::max<long long>(2, (nb + per_band / 2) / per_band));
    order.resize(nb);
    for (int q = 0; q < nb; ++q)
        order[q] = q;
    auto key = [&](int q) {
        const long long first = static_cast<long long>(q) * TILE;
        const long long band = (first % g.s) * bands / g.s;
        return std::make_pair(band, first / g.s);
    };
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return key(a) < key(b); });
    return true;
}

// The walk of each query tile's CSR row by the forward and the dQ pass (and,
// computed over the transposed CSR, of each key tile's row by the dK / dV pass,
// by the mask's symmetry), for long radial masks (used with the dispatch order
// above): first the key tiles of the frames near
// the query tile's own (those whose first row lies in a frame less than `near`
// frames from the frame of the query tile's first row: a contiguous segment
// [a, b) of the ascending row), then the others in ascending order.  The CTAs
// resident together (one position band over consecutive frames) then take
// their near frames, where a row spends most of its tiles, at about the same
// time, and afterwards the far frames, where eq. 4 keeps a few tiles around the
// band's positions, in the same ascending order.  (A mask that keeps whole far
// frames, such as the dense one, would only stagger the CTAs' starting frames.)
// walk[2 q], walk[2 q + 1] = a, b as offsets in the row.
__global__ void __launch_bounds__(128) walk_kernel(MaskGeom g, int nb, int near, const int* __restrict__ row_ptr,
                                                   const int* __restrict__ col_idx, int* __restrict__ walk)
{
    const int q = blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= nb)
        return;
    const long long i = static_cast<long long>(q) * TILE / g.s;  // frame of the tile's first row
    const long long f_lo = i - near + 1, f_hi = i + near - 1;
    // first key tile whose first row lies in frame >= f_lo; last one in frame <= f_hi
    const long long k_lo = f_lo <= 0 ? 0 : (f_lo * g.s + TILE - 1) / TILE;
    const long long k_hi = ((f_hi + 1) * g.s - 1) / TILE;
    const int start = row_ptr[q], end = row_ptr[q + 1];
    int lo = start, hi = end;
    while (lo < hi) {  // lower bound of k_lo
        const int mid = (lo + hi) >> 1;
        if (col_idx[mid] < k_lo)
            lo = mid + 1;
        else
            hi = mid;
    }
    const int a = lo;
    hi = end;
    while (lo < hi) {  // upper bound of k_hi
        const int mid = (lo + hi) >> 1;
        if (col_idx[mid] <= k_hi)
            lo = mid + 1;
        else
            hi = mid;
    }
    walk[2 * q] = a - start;
    walk[2 * q + 1] = lo - start;
}

void free_mask_arrays(ra_mask* m)
{
    cudaFree(m->row_ptr);
    cudaFree(m->col_idx);
    cudaFree(m->count);
    cudaFree(m->flag);
    cudaFree(m->col_ptr);
    cudaFree(m->row_idx);
    cudaFree(m->tflag);
    cudaFree(m->qorder);
    cudaFree(m->walk);
    cudaFree(m->walk_t);
    m->row_ptr = m->col_idx = m->count = m->col_ptr = m->row_idx = m->qorder = m->walk = m->walk_t = nullptr;
    m->flag = m->tflag = nullptr;
}

struct Scratch {
    int* counts = nullptr;
    int* row_tiles = nullptr;
    BuildTotals* tot = nullptr;
    ~Scratch()
    {
        cudaFree(counts);
        cudaFree(row_tiles);
        cudaFree(tot);
    }
};

ra_status validate_geometry(int family, int f, int s, const ra_mask_params* p, MaskGeom* g)
{
    if (family < RA_MASK_DENSE || family > RA_MASK_SWC)
        return fail(RA_ERR_INVALID_ARG, "unknown mask family %d", family);
    if (f < 1 || s < 1)
        return fail(RA_ERR_INVALID_ARG, "f and s must be >= 1 (f=%d, s=%d)", f, s);
    const long long n = static_cast<long long>(f) * s;
    const long long nb = (n + TILE - 1) / TILE;
    if (n > INT_MAX - TILE || nb * nb > INT_MAX)
        return fail(RA_ERR_UNSUPPORTED, "n = %lld tokens is beyond the builder's limit", n);
    std::memset(g, 0, sizeof *g);
    g->family = family;
    g->f = f;
    g->s = s;
    g->n = static_cast<int>(n);
    if (family == RA_MASK_WINDOW3D) {
        if (!p)
            return fail(RA_ERR_INVALID_ARG, "WINDOW3D needs params");
        if (p->grid_h < 1 || p->grid_w < 1 || static_cast<long long>(p->grid_h) * p->grid_w != s)
            return fail(RA_ERR_INVALID_ARG, "WINDOW3D needs grid_h * grid_w == s (%d x %d vs %d)", p->grid_h,
                        p->grid_w, s);
        if (p->r_t < 0 || p->r_s < 0)
            return fail(RA_ERR_INVALID_ARG, "WINDOW3D radii must be >= 0");
        g->grid_h = p->grid_h;
        g->grid_w = p->grid_w;
        g->r_t = p->r_t;
        g->r_s = p->r_s;
    } else if (family == RA_MASK_SWC) {
        if (!p || p->window_frames < 1)
            return fail(RA_ERR_INVALID_ARG, "SWC needs window_frames >= 1");
        g->window_frames = p->window_frames;
    }
    if (p) {
        if (p->sink_tokens < 0 || p->sink_tokens > g->n)
            return fail(RA_ERR_INVALID_ARG, "sink_tokens must be in [0, n] (got %d)", p->sink_tokens);
        g->sink = p->sink_tokens;
    }
    return RA_OK;
}

}  // namespace
}  // namespace ra

using namespace ra;

extern "C" ra_status ra_build_mask(int family, int f, int s, const ra_mask_params* params, ra_stream stream,
                                   ra_mask** out)
{
    if (!out)
        return fail(RA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    MaskGeom g;
    ra_status st = validate_geometry(family, f, s, params, &g);
    if (st != RA_OK)
        return st;
    const int nb = (g.n + TILE - 1) / TILE;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    int device = 0;
    RA_CUDA_TRY(cudaGetDevice(&device));
    ra_mask* m = new ra_mask();
    std::memset(m, 0, sizeof *m);
    m->geom = g;
    m->nb = nb;
    m->device = device;

    Scratch sc;
    auto bail = [&](cudaError_t e, const char* what) {
        free_mask_arrays(m);
        delete m;
        return e == cudaErrorMemoryAllocation ? fail(RA_ERR_OUT_OF_MEMORY, "%s: out of device memory", what)
                                              : cuda_fail(e, what);
    };
    cudaError_t e;
    if ((e = cudaMalloc(&sc.counts, sizeof(int) * static_cast<size_t>(nb) * nb)) != cudaSuccess)
        return bail(e, "tile counts");
    if ((e = cudaMalloc(&sc.row_tiles, sizeof(int) * nb)) != cudaSuccess)
        return bail(e, "row tiles");
    if ((e = cudaMalloc(&sc.tot, sizeof(BuildTotals))) != cudaSuccess)
        return bail(e, "totals");
    if ((e = cudaMalloc(&m->row_ptr, sizeof(int) * (nb + 1))) != cudaSuccess)
        return bail(e, "row_ptr");

    BuildTotals init{0, 0, 0, INT_MAX, 0};
    if ((e = cudaMemcpyAsync(sc.tot, &init, sizeof init, cudaMemcpyHostToDevice, cs)) != cudaSuccess)
        return bail(e, "totals init");
    tile_count_kernel<<<nb, TILE, 0, cs>>>(g, nb, sc.counts, sc.row_tiles, sc.tot);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return bail(e, "tile_count_kernel launch");
    row_scan_kernel<<<1, 1024, 0, cs>>>(sc.row_tiles, nb, m->row_ptr);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return bail(e, "row_scan_kernel launch");
    BuildTotals tot;
    int nnz = 0;
    if ((e = cudaMemcpyAsync(&tot, sc.tot, sizeof tot, cudaMemcpyDeviceToHost, cs)) != cudaSuccess ||
        (e = cudaMemcpyAsync(&nnz, m->row_ptr + nb, sizeof nnz, cudaMemcpyDeviceToHost, cs)) != cudaSuccess ||
        (e = cudaStreamSynchronize(cs)) != cudaSuccess)
        return bail(e, "mask statistics");
    m->nnz = nnz;
    m->kept_pairs = static_cast<long long>(tot.kept_pairs);
    m->block_pairs = static_cast<long long>(tot.block_pairs);
    m->full_tiles = static_cast<long long>(tot.full_tiles);
    m->row_min = tot.row_min;
    m->row_max = tot.row_max;

    if (nnz > 0) {
        if ((e = cudaMalloc(&m->col_idx, sizeof(int) * nnz)) != cudaSuccess)
            return bail(e, "col_idx");
        if ((e = cudaMalloc(&m->count, sizeof(int) * nnz)) != cudaSuccess)
            return bail(e, "count");
        if ((e = cudaMalloc(&m->flag, nnz)) != cudaSuccess)
            return bail(e, "flag");
        compact_kernel<<<nb, TILE, 0, cs>>>(sc.counts, nb, m->row_ptr, m->col_idx, m->count, m->flag);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return bail(e, "compact_kernel launch");
        // transposed block-CSR for the backward pass (same nnz)
        if ((e = cudaMalloc(&m->col_ptr, sizeof(int) * (nb + 1))) != cudaSuccess)
            return bail(e, "col_ptr");
        if ((e = cudaMalloc(&m->row_idx, sizeof(int) * nnz)) != cudaSuccess)
            return bail(e, "row_idx");
        if ((e = cudaMalloc(&m->tflag, nnz)) != cudaSuccess)
            return bail(e, "tflag");
        col_count_kernel<<<nb, TILE, 0, cs>>>(sc.counts, nb, sc.row_tiles);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return bail(e, "col_count_kernel launch");
        row_scan_kernel<<<1, 1024, 0, cs>>>(sc.row_tiles, nb, m->col_ptr);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return bail(e, "column scan launch");
        col_compact_kernel<<<nb, TILE, 0, cs>>>(sc.counts, nb, m->col_ptr, m->row_idx, m->tflag);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return bail(e, "col_compact_kernel launch");
    }
    int sm_count = 0;
    if ((e = cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess)
        return bail(e, "SM count");
    std::vector<int> order;
    if (dispatch_order(g, nb, sm_count, walked(g), order)) {
        if ((e = cudaMalloc(&m->qorder, sizeof(int) * nb)) != cudaSuccess)
            return bail(e, "qorder");
        // synchronous copy from pageable memory: `order` is released on return
        if ((e = cudaMemcpy(m->qorder, order.data(), sizeof(int) * nb, cudaMemcpyHostToDevice)) != cudaSuccess)
            return bail(e, "qorder copy");
        if (nnz > 0 && walked(g)) {
            if ((e = cudaMalloc(&m->walk, sizeof(int) * 2 * static_cast<size_t>(nb))) != cudaSuccess)
                return bail(e, "walk");
            walk_kernel<<<(nb + 127) / 128, 128, 0, cs>>>(g, nb, walk_near_frames(g), m->row_ptr, m->col_idx,
                                                           m->walk);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return bail(e, "walk_kernel launch");
            // the transposed CSR's rows (key tiles, their query tiles): the same
            // walk, by the mask's symmetry in query and key
            if ((e = cudaMalloc(&m->walk_t, sizeof(int) * 2 * static_cast<size_t>(nb))) != cudaSuccess)
                return bail(e, "walk_t");
            walk_kernel<<<(nb + 127) / 128, 128, 0, cs>>>(g, nb, walk_near_frames(g), m->col_ptr, m->row_idx,
                                                           m->walk_t);
            if ((e = cudaGetLastError()) != cudaSuccess)
                return bail(e, "walk_kernel launch (transposed)");
        }
    }
    // The scratch arrays are released by ~Scratch; cudaFree waits for the kernels.
    if ((e = cudaStreamSynchronize(cs)) != cudaSuccess)
        return bail(e, "mask build");
    *out = m;
    return RA_OK;
}

extern "C" ra_status ra_mask_info(const ra_mask* m, ra_mask_info_t* info)
{
    if (!m || !info)
        return fail(RA_ERR_INVALID_ARG, "NULL mask or info");
    info->family = m->geom.family;
    info->f = m->geom.f;
    info->s = m->geom.s;
    info->nb = m->nb;
    info->n = m->geom.n;
    info->nnz = m->nnz;
    info->full_tiles = m->full_tiles;
    info->kept_pairs = m->kept_pairs;
    info->block_pairs = m->block_pairs;
    info->row_min = m->row_min;
    info->row_max = m->row_max;
    return RA_OK;
}

extern "C" ra_status ra_mask_copy_to_host(const ra_mask* m, int* row_ptr, int* col_idx, int* count,
                                          unsigned char* flag)
{
    if (!m)
        return fail(RA_ERR_INVALID_ARG, "NULL mask");
    if (row_ptr)
        RA_CUDA_TRY(cudaMemcpy(row_ptr, m->row_ptr, sizeof(int) * (m->nb + 1), cudaMemcpyDeviceToHost));
    if (m->nnz > 0) {
        if (col_idx)
            RA_CUDA_TRY(cudaMemcpy(col_idx, m->col_idx, sizeof(int) * m->nnz, cudaMemcpyDeviceToHost));
        if (count)
            RA_CUDA_TRY(cudaMemcpy(count, m->count, sizeof(int) * m->nnz, cudaMemcpyDeviceToHost));
        if (flag)
            RA_CUDA_TRY(cudaMemcpy(flag, m->flag, m->nnz, cudaMemcpyDeviceToHost));
    }
    return RA_OK;
}

extern "C" ra_status ra_mask_device_arrays(const ra_mask* m, const int** row_ptr, const int** col_idx,
                                           const int** count, const unsigned char** flag)
{
    if (!m)
        return fail(RA_ERR_INVALID_ARG, "NULL mask");
    if (row_ptr)
        *row_ptr = m->row_ptr;
    if (col_idx)
        *col_idx = m->col_idx;
    if (count)
        *count = m->count;
    if (flag)
        *flag = m->flag;
    return RA_OK;
}

extern "C" void ra_mask_free(ra_mask* m)
{
    if (!m)
        return;
    cudaDeviceSynchronize();
    free_mask_arrays(m);
    delete m;
}

// Device address of g_noalloc_scratch in the current device's context.  Host
// code cannot use the symbol itself as a device address.  The address is looked
// up on every call (a cheap query) rather than cached per device ordinal: a
// cached address would go stale if the device's primary context were reset and
// the module loaded again.
static ra_status noalloc_scratch_address(unsigned char** out)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress(builder scratch)");
    *out = static_cast<unsigned char*>(p);
    return RA_OK;
}

extern "C" ra_status ra_build_mask_noalloc(int family, int f, int s, const ra_mask_params* params, int* row_ptr,
                                           int* col_idx, int* count, unsigned char* flag, long long nnz_capacity,
                                           ra_mask_info_t* info, ra_stream stream)
{
    MaskGeom g;
    ra_status st = validate_geometry(family, f, s, params, &g);
    if (st != RA_OK)
        return st;
    const int nb = (g.n + TILE - 1) / TILE;
    if (nb > NOALLOC_MAX_NB)
        return fail(RA_ERR_UNSUPPORTED,
                    "ra_build_mask_noalloc handles at most %d x 128 = %d tokens (its fixed scratch); n = %d",
                    NOALLOC_MAX_NB, NOALLOC_MAX_NB * TILE, g.n);
    if (!row_ptr || (nnz_capacity > 0 && (!col_idx || !count || !flag)) || nnz_capacity < 0)
        return fail(RA_ERR_INVALID_ARG, "NULL output array or negative capacity");
    unsigned char* scratch = nullptr;
    if ((st = noalloc_scratch_address(&scratch)) != RA_OK)
        return st;
    int* counts = reinterpret_cast<int*>(scratch);
    int* row_tiles = reinterpret_cast<int*>(scratch + NOALLOC_COUNTS_BYTES);
    BuildTotals* tot = reinterpret_cast<BuildTotals*>(scratch + NOALLOC_COUNTS_BYTES + NOALLOC_ROWS_BYTES);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

    // The scratch keeps the previous call's contents: the statistics start from
    // zero here; every count and per-row entry used below is rewritten.
    init_totals_kernel<<<1, 1, 0, cs>>>(tot);
    RA_CUDA_TRY(cudaGetLastError());
    tile_count_kernel<<<nb, TILE, 0, cs>>>(g, nb, counts, row_tiles, tot);
    RA_CUDA_TRY(cudaGetLastError());
    row_scan_kernel<<<1, 1024, 0, cs>>>(row_tiles, nb, row_ptr);
    RA_CUDA_TRY(cudaGetLastError());
    BuildTotals h;
    int nnz = 0;
    RA_CUDA_TRY(cudaMemcpyAsync(&h, tot, sizeof h, cudaMemcpyDeviceToHost, cs));
    RA_CUDA_TRY(cudaMemcpyAsync(&nnz, row_ptr + nb, sizeof nnz, cudaMemcpyDeviceToHost, cs));
    RA_CUDA_TRY(cudaStreamSynchronize(cs));
    if (info) {
        info->family = g.family;
        info->f = g.f;
        info->s = g.s;
        info->nb = nb;
        info->n = g.n;
        info->nnz = nnz;
        info->full_tiles = static_cast<long long>(h.full_tiles);
        info->kept_pairs = static_cast<long long>(h.kept_pairs);
        info->block_pairs = static_cast<long long>(h.block_pairs);
        info->row_min = h.row_min;
        info->row_max = h.row_max;
    }
    if (nnz > nnz_capacity)
        return fail(RA_ERR_INVALID_ARG, "the mask keeps %d tiles but the output arrays hold %lld", nnz, nnz_capacity);
    if (nnz > 0) {
        compact_kernel<<<nb, TILE, 0, cs>>>(counts, nb, row_ptr, col_idx, count, flag);
        RA_CUDA_TRY(cudaGetLastError());
    }
    return RA_OK;
}

extern "C" ra_status ra_mask_copy_transpose_to_host(const ra_mask* m, int* col_ptr, int* row_idx,
                                                    unsigned char* tflag)
{
    if (!m)
        return fail(RA_ERR_INVALID_ARG, "NULL mask");
    if (col_ptr)
        RA_CUDA_TRY(cudaMemcpy(col_ptr, m->col_ptr, sizeof(int) * (m->nb + 1), cudaMemcpyDeviceToHost));
    if (m->nnz > 0) {
        if (row_idx)
            RA_CUDA_TRY(cudaMemcpy(row_idx, m->row_idx, sizeof(int) * m->nnz, cudaMemcpyDeviceToHost));
        if (tflag)
            RA_CUDA_TRY(cudaMemcpy(tflag, m->tflag, m->nnz, cudaMemcpyDeviceToHost));
    }
    return RA_OK;
}
