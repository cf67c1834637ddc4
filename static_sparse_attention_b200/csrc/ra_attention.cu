// ra_attention.cu -- block-sparse attention forward for sm_100a (B200).
//
// Computes, per (batch b, head h, 128-row query tile qb),
//     O = softmax(scale * Q K^T + M) V        ("Radial Attention ..." eq. 2)
// over the kept 128 x 128 tiles of the query tile's block-CSR row
// (sec. 6: 128 x 128 block granularity).  In token-exact mode a PARTIAL tile
// applies the element mask; in block mode every valid pair of a kept tile is
// used.  Keys >= n are masked in both modes; rows >= n are never stored.
//
// One CTA per query tile, two CTAs resident per SM (256 TMEM columns, under
// half the shared memory each).  Keys move in half-tiles of 64: half-tile h of
// the row is half h % 2 of kept tile h / 2.  192 threads in fixed roles:
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); per half-tile
//              reads S from TMEM, masks, keeps the running max / sum, writes P
//              (bf16) back over S, and at the end runs the epilogue O / l.
//   warp 4     producer: TMA loads of Q once, then the K and V half-tiles of
//              the row into two rings (128-byte swizzle).
//   warp 5     MMA: allocates TMEM; runs its loop warp-wide (descriptor
//              arithmetic warp-uniform) and one elected lane issues S_h = Q K_h^T
//              (tcgen05.mma, N = 64) into S buffer h % 2 and O += P_h V_h
//              (A = P from TMEM), in the order S_0, S_1, PV_0, S_2, PV_1, ...:
//              S of the next half-tile is in flight while the softmax works on
//              the current one.
// TMEM columns: S buffers at 0 and 64 (fp32, 64 columns; P overlays each as
// packed bf16), O at 128 (fp32, d columns).
//
// Ordering of the MMAs.  S_{h+2} overwrites the TMEM buffer whose P the P V of
// half-tile h reads.  The PTX ISA orders two asynchronous tcgen05 operations of
// one thread only for the pairs it lists as tcgen05 pipelines ("pipelined
// tcgen05 instructions"): MMA -> MMA only for the same accumulator and shape,
// but MMA -> shift and shift -> MMA for any two of the same cta_group.  So
// before S_{h+2} the MMA lane issues a tcgen05.shift of one 32-byte column
// group of that buffer: P V_h -> shift -> S_{h+2} is a chain of listed pairs,
// the shift only disturbs columns that S_{h+2} then overwrites (its first MMA
// does not accumulate), and no thread waits.  The softmax rescales O only after
// the P V of the previous half-tile has completed.
//
// Work order.  CTA x takes query tile qorder[x] of its head (the mask's
// dispatch order; identity when absent): query tiles sorted by in-frame
// position band, then frame, so that the CTAs resident together share a
// position band across many frames and walk overlapping key tiles of every
// frame (eq. 4's bands are centred on the query's own in-frame position).  On
// long sequences each CTA walks its row's key tiles of the frames near its own
// first (the mask's walk: a contiguous segment of the ascending row), then the
// others in ascending order, so that the resident CTAs stay closer together in
// the far frames.
//
// Online softmax in base 2: x = S * scale * log2(e); p = 2^(x - m) with m a
// running maximum that is only raised (and O, l rescaled) when a half-tile's
// maximum exceeds it by more than 8; p <= 2^8 otherwise, which fp32 and bf16
// hold with the same relative precision as p <= 1, and O / l does not depend on
// m.  After the first half-tile the exponentials are computed against the
// running maximum in the same pass that finds the half-tile's maximum.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>

#include "ra_internal.h"
#include "ra_sm100.cuh"

namespace ra {

// Device error word of the forward kernels: [0] status, [1] site, [2] block.
__device__ int g_err[4];

namespace {

constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 256;
// Keys per half-tile: K, V, S and P move 64 keys at a time.
constexpr int HALF = 64;
// TMEM columns of S / P buffer `buf` (64 fp32 columns) and of O (d fp32 columns).
__host__ __device__ constexpr uint32_t s_col_of(int buf) { return 64u * static_cast<uint32_t>(buf); }
constexpr uint32_t O_COL = 128;
constexpr float RESCALE_THRESHOLD = 8.0f;

// Wait-site codes recorded with a timeout.
enum : int {
    SITE_Q_FULL = 1, SITE_K_EMPTY, SITE_V_EMPTY, SITE_K_FULL, SITE_P_FULL, SITE_V_FULL, SITE_S_FULL,
    SITE_PV_DONE, SITE_O_FINAL, SITE_SELFTEST, SITE_SMEM_ALIGN,
    // bounds checks of the debug build
    SITE_B_QTILE = 40, SITE_B_ROW, SITE_B_KTILE, SITE_B_SELFTEST, SITE_B_WALK
};

template <int D>
struct Layout {
    static constexpr int CHUNKS = D / 64;                          // 128-byte swizzle atoms across d
    static constexpr int Q_CHUNK_BYTES = TILE * 128;                // 128 rows x 128 bytes
    static constexpr int Q_BYTES = CHUNKS * Q_CHUNK_BYTES;          // the 128 x d query tile
    static constexpr int H_CHUNK_BYTES = HALF * 128;                // 64 rows x 128 bytes
    static constexpr int H_BYTES = CHUNKS * H_CHUNK_BYTES;          // a 64 x d half-tile of K or V
    static constexpr int KS = D == 64 ? 4 : 3;                      // K ring stages (half-tiles)
    static constexpr int VS = D == 64 ? 4 : 2;                      // V ring stages (half-tiles)
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + Q_BYTES;
    static constexpr int V_OFF = K_OFF + KS * H_BYTES;
    static constexpr int BAR_OFF = V_OFF + VS * H_BYTES;
    static constexpr int BAR_BYTES = 256;
    // Two CTAs share an SM; the dynamic shared memory is 1024-byte aligned
    // (checked at run time) so no alignment slack is reserved.
    static constexpr int SMEM_BYTES = BAR_OFF + BAR_BYTES;
};

// Barrier slots (8 bytes each) inside the barrier region.
enum : int {
    B_Q_FULL = 0,
    B_K_FULL = 1,    // + stage (up to 4)
    B_K_EMPTY = 5,   // + stage
    B_V_FULL = 9,    // + stage
    B_V_EMPTY = 13,  // + stage
    B_S_FULL = 17,   // + buffer
    B_P_FULL = 19,   // + buffer
    B_PV_DONE = 21,
    B_O_FINAL = 22,
    B_COUNT = 23
};

struct FwdParams {
    MaskGeom g;        // query rows: g.n; the family mask of token-exact partial tiles
    int nb, H, mode;   // nb: query tiles (the grid)
    int nk, nbk;       // key rows and key tiles (n and nb for self-attention)
    const int* row_ptr;
    const int* col_idx;
    const unsigned char* flag;
    const int* qorder; // query tile of CTA x (a permutation of [0, nb)), or null for x itself
    const int* walk;   // [2 nb]: row offsets a, b of each row's near segment, walked first; or null
    int nnz;           // entries of col_idx / flag (bounds checks of the debug build)
    __nv_bfloat16* O;
    float* lse;
    float scale_log2;  // scale * log2(e)
    unsigned long long timeout_ns;
};

// ---- packed fp32 pairs (sm_100 f32x2 instructions: each lane rounds as the
// scalar instruction does) -------------------------------------------------
__device__ __forceinline__ uint64_t f2pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Exponentials, bf16 packing and row sums of one 32-column chunk of S:
// p = 2^(s * c - m) on MUFU ex2.  The row sum is kept in SUM_ACC independent
// accumulators (short dependency chains).  With bf16 P the exponent s * c - m of
// two columns is one fma.rn.f32x2 and the sums are updated a pair at a time
// with add.rn.f32x2 (3-4 % more work per clock than the scalar form); SPLIT
// (which also returns the bf16 residuals) keeps the scalar form.  MAX also
// tracks the raw maximum of the chunk.
constexpr int SUM_ACC = 8;
constexpr int MAX_ACC = 8;
template <bool SPLIT, bool MAX>
__device__ __forceinline__ void exp_chunk(const uint32_t (&r)[32], float c, float negm, float (&acc)[SUM_ACC],
                                          float (&mx)[4], uint32_t (&pk)[16], uint32_t (&pl)[16])
{
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        if (MAX)
            mx[(e >> 1) & 3] = max3(mx[(e >> 1) & 3], __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        float x0, x1;
        if (SPLIT) {  // scalar here: the residuals' registers leave no room for the pairs
            x0 = fmaf(__uint_as_float(r[e]), c, negm);
            x1 = fmaf(__uint_as_float(r[e + 1]), c, negm);
        } else {
            f2unpack(f2fma(f2pack(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), f2pack(c, c),
                           f2pack(negm, negm)),
                     x0, x1);
        }
        const float p0 = fast_exp2(x0);
        const float p1 = fast_exp2(x1);
        if (SPLIT) {
            acc[(e >> 1) % SUM_ACC] += p0 + p1;
        } else {
            const int a = ((e >> 1) % (SUM_ACC / 2)) * 2;  // accumulators a, a + 1 take the pair
            f2unpack(f2add(f2pack(acc[a], acc[a + 1]), f2pack(p0, p1)), acc[a], acc[a + 1]);
        }
        pk[e >> 1] = pack_bf16(p0, p1);
        if (SPLIT) {
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&pk[e >> 1]);
            pl[e >> 1] = pack_bf16(p0 - __low2float(hi), p1 - __high2float(hi));
        }
    }
}

// SPLIT_P: P is kept as hi + lo bf16 pairs (P = hi + lo to ~16 bits) and
// P V runs as two MMAs; used for masks whose rows hold few keys, where the
// rounding of P to bf16 is not averaged out over many keys.
template <int D, bool SPLIT_P>
__global__ void __launch_bounds__(NUM_THREADS, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p)
{
    using L = Layout<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
    const uint32_t bars = sbase + L::BAR_OFF;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR_OFF + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::BAR_OFF + 8 * B_COUNT + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.qorder ? p.qorder[blockIdx.x] : static_cast<int>(blockIdx.x);
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int n = p.g.n;
    WaitCtl wc{abort_flag, g_err, p.timeout_ns};

    if (threadIdx.x == 0) {
        *abort_flag = *reinterpret_cast<volatile int*>(g_err) != 0 ? 1 : 0;
        if (sbase & 1023u)  // the swizzled tiles need 1024-byte alignment: record it, run nothing
            report_timeout(wc, SITE_SMEM_ALIGN);
        // (debug build) the query tile and its CSR row are in range
        if (!*abort_flag && in_bounds(wc, qb >= 0 && qb < p.nb, SITE_B_QTILE))
            in_bounds(wc, 0 <= p.row_ptr[qb] && p.row_ptr[qb] <= p.row_ptr[qb + 1] && p.row_ptr[qb + 1] <= p.nnz,
                      SITE_B_ROW);
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(bar(i), (i == B_P_FULL || i == B_P_FULL + 1) ? 128u : 1u);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort_flag != 0;  // an earlier CTA gave up: do nothing

    const int row_start = skip ? 0 : p.row_ptr[qb];
    const int L_row = skip ? 0 : p.row_ptr[qb + 1] - row_start;
    const int n_half = 2 * L_row;
    // The order of the row's kept tiles: its near segment [wa, wb) first, then
    // the others in ascending order (the identity without a walk).
    int wa = 0, wb = 0;
    if (p.walk && L_row > 0) {
        wa = p.walk[2 * qb];
        wb = p.walk[2 * qb + 1];
        if (!in_bounds(wc, 0 <= wa && wa <= wb && wb <= L_row, SITE_B_WALK))  // (debug build)
            wa = wb = 0;
    }
    auto walk = [wa, wb](int i) {
        const int near = wb - wa;
        return i < near ? wa + i : (i - near < wa ? i - near : i);
    };

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && L_row > 0) {
            tma_prefetch_map(&tmQ);
            tma_prefetch_map(&tmK);
            tma_prefetch_map(&tmV);
            mbar_arrive_expect_tx(bar(B_Q_FULL), L::Q_BYTES);
            for (int c = 0; c < L::CHUNKS; ++c)
                tma_load_3d(sQ + c * L::Q_CHUNK_BYTES, &tmQ, bar(B_Q_FULL), c * 64, qb * TILE, bh);
            int k_issued = 0, v_issued = 0;
            for (int hh = 0; hh < n_half; ++hh) {
                const int kb = p.col_idx[row_start + walk(hh >> 1)];
                if (!in_bounds(wc, kb >= 0 && kb < p.nbk, SITE_B_KTILE))  // (debug build)
                    break;
                const int key0 = kb * TILE + (hh & 1) * HALF;
                const int ks = hh % L::KS, vs = hh % L::VS;
                if (hh >= L::KS && !mbar_wait(bar(B_K_EMPTY + ks), ((hh / L::KS) - 1) & 1, wc, SITE_K_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(B_K_FULL + ks), L::H_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sK + ks * L::H_BYTES + c * L::H_CHUNK_BYTES, &tmK, bar(B_K_FULL + ks), c * 64,
                                key0, bh);
                k_issued = hh + 1;
                if (hh >= L::VS && !mbar_wait(bar(B_V_EMPTY + vs), ((hh / L::VS) - 1) & 1, wc, SITE_V_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(B_V_FULL + vs), L::H_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sV + vs * L::H_BYTES + c * L::H_CHUNK_BYTES, &tmV, bar(B_V_FULL + vs), c * 64,
                                key0, bh);
                v_issued = hh + 1;
            }
            // Let every copy this thread issued land before the CTA can exit.  A
            // load into a stage is issued only after the previous load of that
            // stage was consumed, so only the last load of each stage can be in
            // flight here, and its phase parity identifies it.
            drain_wait(bar(B_Q_FULL), 0, p.timeout_ns);
            for (int j = max(0, k_issued - L::KS); j < k_issued; ++j)
                drain_wait(bar(B_K_FULL + j % L::KS), (j / L::KS) & 1, p.timeout_ns);
            for (int j = max(0, v_issued - L::VS); j < v_issued; ++j)
                drain_wait(bar(B_V_FULL + j % L::VS), (j / L::VS) & 1, p.timeout_ns);
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------------- MMA
        // The whole warp runs the loop, so that the descriptors (built once; each
        // MMA only advances the start address) stay warp-uniform; the elected
        // lane issues the MMAs and commits.  The warp shares its sub-partition
        // with softmax warps.
        if (L_row > 0) {
            const bool leader = elect_one();
            constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, HALF, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(TILE, D, 0, 1);
            const uint64_t q_desc = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t k_desc = smem_desc_sw128(sK, 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(sV, L::H_CHUNK_BYTES, 1024);  // V as MN-major B
            auto wait_all = [&](uint32_t b, uint32_t parity, int site) {
                return __all_sync(0xFFFFFFFFu, mbar_wait(b, parity, wc, site));
            };
            bool ok = wait_all(bar(B_Q_FULL), 0, SITE_Q_FULL);
            tc_fence_after();
            for (int hh = 0; ok && hh <= n_half; ++hh) {
                if (hh < n_half) {
                    // S_hh into buffer hh % 2; its previous occupant's P V
                    // (half-tile hh - 2) was issued in the previous iteration.
                    const int ks = hh % L::KS;
                    if (!(ok = wait_all(bar(B_K_FULL + ks), (hh / L::KS) & 1, SITE_K_FULL)))
                        break;
                    tc_fence_after();
                    // Order S_hh after that P V: MMA -> shift -> MMA (see the header).
                    if (hh >= 2 && leader)
                        tmem_shift_down(tmem + s_col_of(hh & 1));
                    const uint64_t kd = desc_add(k_desc, ks * L::H_BYTES);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = desc_add(q_desc, (kk >> 2) * L::Q_CHUNK_BYTES + (kk & 3) * 32);
                        const uint64_t bd = desc_add(kd, (kk >> 2) * L::H_CHUNK_BYTES + (kk & 3) * 32);
                        mma_ss(leader, tmem + s_col_of(hh & 1), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    if (leader) {
                        mma_commit(bar(B_S_FULL + (hh & 1)));
                        mma_commit(bar(B_K_EMPTY + ks));
                    }
                }
                if (hh >= 1) {
                    const int j = hh - 1, vs = j % L::VS, buf = j & 1;
                    if (!(ok = wait_all(bar(B_P_FULL + buf), (j >> 1) & 1, SITE_P_FULL)) ||
                        !(ok = wait_all(bar(B_V_FULL + vs), (j / L::VS) & 1, SITE_V_FULL)))
                        break;
                    tc_fence_after();
                    const uint64_t vd = desc_add(v_desc, vs * L::H_BYTES);
#pragma unroll
                    for (int kk = 0; kk < HALF / 16; ++kk) {
                        const uint64_t bd = desc_add(vd, kk * 2048);
                        mma_ts(leader, tmem + O_COL, tmem + s_col_of(buf) + kk * 8, bd, idesc_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (SPLIT_P) {
#pragma unroll
                        for (int kk = 0; kk < HALF / 16; ++kk) {
                            const uint64_t bd = desc_add(vd, kk * 2048);
                            mma_ts(leader, tmem + O_COL, tmem + s_col_of(buf) + HALF / 2 + kk * 8, bd, idesc_pv, 1u);
                        }
                    }
                    if (leader) {
                        mma_commit(bar(B_V_EMPTY + vs));
                        mma_commit(bar(B_PV_DONE));
                    }
                }
            }
            if (leader)
                mma_commit(bar(B_O_FINAL));
            // Every MMA issued by the elected lane has completed once O_FINAL fires.
            drain_wait(bar(B_O_FINAL), 0, p.timeout_ns);
        }
    } else {
        // ----------------------------------------------------------------- softmax
        const int t = threadIdx.x;  // == TMEM lane == query row in the tile
        const int row = qb * TILE + t;
        const bool row_valid = row < n;
        const int qi = row_valid ? row / p.g.s : 0, qk = row_valid ? row % p.g.s : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const bool tail = (p.nk % TILE) != 0;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        uint32_t mk[4] = {~0u, ~0u, ~0u, ~0u};
        bool masked = false;
        // CSR entry of the next tile, loaded one tile ahead of its use.
        int next_kb = L_row > 0 ? p.col_idx[row_start + walk(0)] : 0;
        int next_flag = L_row > 0 ? p.flag[row_start + walk(0)] : 0;
        for (int hh = 0; hh < n_half; ++hh) {
            const int i = hh >> 1, half = hh & 1, buf = hh & 1;
            const uint32_t s_col = s_col_of(buf);
            if (half == 0) {
                // Mask of the whole tile: token-exact partial tiles use the
                // family's element mask; the tail key tile masks keys >= nk.
                const int kb = next_kb;
                const bool use_family = p.mode == RA_MODE_TOKEN_EXACT && next_flag != RA_TILE_FULL;
                if (i + 1 < L_row) {
                    next_kb = p.col_idx[row_start + walk(i + 1)];
                    next_flag = p.flag[row_start + walk(i + 1)];
                }
                masked = use_family || (tail && kb == p.nbk - 1);
                if (masked) {
                    if (use_family && row_valid) {
                        row_keep_mask(p.g, qi, qk, kb * TILE, mk[0], mk[1], mk[2], mk[3]);
                    } else {
                        const int valid_cols = min(TILE, p.nk - kb * TILE);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int v = valid_cols - 32 * c;
                            mk[c] = v >= 32 ? 0xFFFFFFFFu : (v <= 0 ? 0u : ((1u << v) - 1u));
                        }
                    }
                }
            }
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_S_FULL + buf), (hh >> 1) & 1, wc, SITE_S_FULL));
            if (!ok)
                break;
            tc_fence_after();
            uint32_t r[2][32];
#pragma unroll
            for (int c = 0; c < 2; ++c)
                tmem_ld32(lane_base + s_col + c * 32, r[c]);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint32_t w = half ? mk[2 + c] : mk[c];
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((w >> e) & 1u))
                            r[c][e] = __float_as_uint(-INFINITY);
                }
            }

            // Exponentials of the half-tile against m_use, P to TMEM; with
            // fused_max the same pass also finds the half-tile's raw maximum.
            auto exp_pass = [&](float m_use, bool fused_max, float& mx_out) -> float {
                float acc[SUM_ACC];
#pragma unroll
                for (int a = 0; a < SUM_ACC; ++a)
                    acc[a] = 0.f;
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16], pl[16];
                    if (fused_max)
                        exp_chunk<SPLIT_P, true>(r[c], p.scale_log2, -m_use, acc, mx, pk, pl);
                    else
                        exp_chunk<SPLIT_P, false>(r[c], p.scale_log2, -m_use, acc, mx, pk, pl);
                    tmem_st16(lane_base + s_col + c * 16, pk);
                    if (SPLIT_P)
                        tmem_st16(lane_base + s_col + HALF / 2 + c * 16, pl);
                }
#pragma unroll
                for (int w = SUM_ACC / 2; w >= 1; w /= 2)
#pragma unroll
                    for (int a = 0; a < w; ++a)
                        acc[a] += acc[a + w];
                mx_out = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                return acc[0];
            };
            // Raise the running max (warp-uniformly) when the half-tile's maximum
            // m_tile exceeds it by more than 8: rescale O and l, once the P V of
            // the previous half-tile has completed (the ones before it have: S_hh
            // was issued after them).
            bool raise_ok = true;
            auto raise_max = [&](float m_tile) {
                const float m_new = fmaxf(m_run, m_tile);
                const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
                if (hh > 0) {
                    raise_ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_PV_DONE), (hh - 1) & 1, wc, SITE_PV_DONE));
                    if (!raise_ok)
                        return;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + O_COL + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(lane_base + O_COL + c * 32, o);
                    }
                }
                l_run *= alpha;
                m_run = m_new;
            };
            float sum, mx_raw;
            if (__any_sync(0xFFFFFFFFu, m_run == -INFINITY)) {
                // No reference maximum yet in this warp: the max first, then the pass.
                float mc[MAX_ACC];
#pragma unroll
                for (int a = 0; a < MAX_ACC; ++a)
                    mc[a] = -INFINITY;
#pragma unroll
                for (int idx = 0; idx < HALF; ++idx)
                    mc[idx % MAX_ACC] = fmaxf(mc[idx % MAX_ACC], __uint_as_float(r[idx / 32][idx % 32]));
#pragma unroll
                for (int w = MAX_ACC / 2; w >= 1; w /= 2)
#pragma unroll
                    for (int a = 0; a < w; ++a)
                        mc[a] = fmaxf(mc[a], mc[a + w]);
                const float m_tile = mc[0] * p.scale_log2;  // scale > 0
                if (__any_sync(0xFFFFFFFFu, m_tile > m_run + RESCALE_THRESHOLD))
                    raise_max(m_tile);
                sum = exp_pass(m_run == -INFINITY ? 0.f : m_run, false, mx_raw);
            } else {
                // One pass against the running maximum, which the half-tile's own
                // maximum rarely exceeds by more than 8; when it does, the pass is
                // redone after raising the maximum (its P and sum are discarded).
                sum = exp_pass(m_run, true, mx_raw);
                const float m_tile = mx_raw * p.scale_log2;
                if (__any_sync(0xFFFFFFFFu, m_tile > m_run + RESCALE_THRESHOLD)) {
                    raise_max(m_tile);
                    sum = exp_pass(m_run, false, mx_raw);
                }
            }
            if (!(ok = raise_ok))
                break;
            l_run += sum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL + buf));
        }

        // ------------------------------------------------------------ epilogue
        if (L_row > 0 && ok)
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_O_FINAL), 0, wc, SITE_O_FINAL));
        tc_fence_after();
        if (ok && !*abort_flag) {
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16* orow = p.O + (static_cast<size_t>(bh) * n + row) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (L_row > 0) {
                    tmem_ld32(lane_base + O_COL + c * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        o[e] = 0u;
                }
                uint4 v[4];
                uint32_t* w = reinterpret_cast<uint32_t*>(v);
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                    w[e >> 1] = pack_bf16(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = v[u];
                }
            }
            if (p.lse && row_valid)
                p.lse[static_cast<size_t>(bh) * n + row] =
                    l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) {
        __syncwarp();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Bounded-wait self-test: one thread waits on a barrier nothing arrives at.
__global__ void wait_selftest_kernel(unsigned long long timeout_ns)
{
    __shared__ __align__(8) uint64_t barrier_word;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_addr(&barrier_word), 1);
        fence_barrier_init();
        WaitCtl wc{&abort_flag, g_err, timeout_ns};
        mbar_wait(smem_addr(&barrier_word), 0, wc, SITE_SELFTEST);
    }
}

#ifdef RA_DEBUG_BOUNDS
// Bounds-check self-test: one thread fails a check on an index it never uses.
__global__ void bounds_selftest_kernel()
{
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        WaitCtl wc{&abort_flag, g_err, 0};
        in_bounds(wc, false, SITE_B_SELFTEST);
    }
}
#endif

template <int D, bool SPLIT_P>
ra_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p, int B,
                     cudaStream_t cs)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(attn_fwd_kernel<D, SPLIT_P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Layout<D>::SMEM_BYTES);
        if (attr_err == cudaSuccess)  // two CTAs per SM need the whole carveout as shared memory
            attr_err = cudaFuncSetAttribute(attn_fwd_kernel<D, SPLIT_P>,
                                            cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err, "cudaFuncSetAttribute(attn_fwd_kernel)");
    dim3 grid(p.nb, p.H, B);
    attn_fwd_kernel<D, SPLIT_P><<<grid, NUM_THREADS, Layout<D>::SMEM_BYTES, cs>>>(mq, mk, mv, p);
    return cuda_fail(cudaGetLastError(), "attn_fwd_kernel launch");
}

// Rows averaging fewer computed keys than this use the split-P kernel.
constexpr long long SPLIT_P_MAX_KEYS_PER_ROW = 4096;
std::atomic<int> g_pv_policy{RA_PV_AUTO};


ra_status check_fwd_args(const void* Q, const void* K, const void* V, const void* O, int B, int H, int d,
                         const ra_mask* m, float scale, int mode)
{
    if (!Q || !K || !V || !O)
        return fail(RA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return fail(RA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    if (!m)
        return fail(RA_ERR_INVALID_ARG, "NULL mask");
    if (B < 1 || H < 1 || B > 65535 || H > 65535)
        return fail(RA_ERR_INVALID_ARG, "B and H must be in [1, 65535] (B=%d, H=%d)", B, H);
    if (d != 64 && d != 128)
        return fail(RA_ERR_UNSUPPORTED, "head dim %d is not supported (64 or 128)", d);
    if (mode != RA_MODE_TOKEN_EXACT && mode != RA_MODE_BLOCK)
        return fail(RA_ERR_INVALID_ARG, "unknown mode %d", mode);
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(RA_ERR_INVALID_ARG, "scale must be finite and > 0");
    const long long elems = static_cast<long long>(B) * H * m->geom.n;
    if (elems > (1LL << 40))
        return fail(RA_ERR_UNSUPPORTED, "tensor too large");
    if (O == Q || O == K || O == V)
        return fail(RA_ERR_INVALID_ARG, "O may not alias Q, K or V");
    int dev = 0;
    RA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev != m->device)
        return fail(RA_ERR_INVALID_ARG, "mask was built on device %d, current device is %d", m->device, dev);
    return RA_OK;
}

}  // namespace
}  // namespace ra

using namespace ra;

extern "C" ra_status ra_attention_fwd(const void* Q, const void* K, const void* V, void* O, int B, int H, int d,
                                      const ra_mask* m, float scale, int mode, float* lse, ra_stream stream)
{
    ra_status st = check_fwd_args(Q, K, V, O, B, H, d, m, scale, mode);
    if (st != RA_OK)
        return st;
    if (m->nnz == 0)
        return fail(RA_ERR_INVALID_ARG, "mask has no kept tile");
    CUtensorMap mq, mk, mv;
    const int BH = B * H, n = m->geom.n;
    if ((st = make_map(&mq, Q, BH, n, d, TILE)) != RA_OK || (st = make_map(&mk, K, BH, n, d, HALF)) != RA_OK ||
        (st = make_map(&mv, V, BH, n, d, HALF)) != RA_OK)
        return st;
    FwdParams p;
    std::memset(&p, 0, sizeof p);
    p.g = m->geom;
    p.nb = m->nb;
    p.nk = n;
    p.nbk = m->nb;
    p.H = H;
    p.mode = mode;
    p.row_ptr = m->row_ptr;
    p.col_idx = m->col_idx;
    p.flag = m->flag;
    p.qorder = m->qorder;
    p.walk = m->walk;
    p.nnz = static_cast<int>(m->nnz);
    p.O = static_cast<__nv_bfloat16*>(O);
    p.lse = lse;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = wait_timeout_ns();
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const long long pairs = mode == RA_MODE_BLOCK ? m->block_pairs : m->kept_pairs;
    const int policy = g_pv_policy.load(std::memory_order_relaxed);
    const bool split = policy == RA_PV_SPLIT ||
                       (policy == RA_PV_AUTO && pairs < SPLIT_P_MAX_KEYS_PER_ROW * static_cast<long long>(n));
    if (d == 64)
        return split ? launch_fwd<64, true>(mq, mk, mv, p, B, cs) : launch_fwd<64, false>(mq, mk, mv, p, B, cs);
    return split ? launch_fwd<128, true>(mq, mk, mv, p, B, cs) : launch_fwd<128, false>(mq, mk, mv, p, B, cs);
}

namespace ra {
ra_status attention_fwd_rect(const void* Q, const void* K, const void* V, void* O, int B, int H, int d, int nq,
                             int nk, int k_head_rows, const int* row_ptr, const int* col_idx,
                             const unsigned char* flag, int nbq, int nnz, float scale, float* lse, cudaStream_t cs)
{
    ra_status st;
    CUtensorMap mq, mk, mv;
    const int BH = B * H;
    if ((st = make_map(&mq, Q, BH, nq, d, TILE)) != RA_OK ||
        (st = make_map_rows(&mk, K, BH, nk, k_head_rows, d, HALF)) != RA_OK ||
        (st = make_map_rows(&mv, V, BH, nk, k_head_rows, d, HALF)) != RA_OK)
        return st;
    FwdParams p;
    std::memset(&p, 0, sizeof p);
    p.g.family = FAM_DENSE;
    p.g.f = 1;
    p.g.s = nq;
    p.g.n = nq;
    p.nb = nbq;
    p.nk = nk;
    p.nbk = (nk + TILE - 1) / TILE;
    p.H = H;
    p.mode = RA_MODE_BLOCK;
    p.row_ptr = row_ptr;
    p.col_idx = col_idx;
    p.flag = flag;
    p.nnz = nnz;
    p.O = static_cast<__nv_bfloat16*>(O);
    p.lse = lse;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = wait_timeout_ns();
    const int policy = g_pv_policy.load(std::memory_order_relaxed);
    const bool split = policy == RA_PV_SPLIT || (policy == RA_PV_AUTO && nk < SPLIT_P_MAX_KEYS_PER_ROW);
    if (d == 64)
        return split ? launch_fwd<64, true>(mq, mk, mv, p, B, cs) : launch_fwd<64, false>(mq, mk, mv, p, B, cs);
    return split ? launch_fwd<128, true>(mq, mk, mv, p, B, cs) : launch_fwd<128, false>(mq, mk, mv, p, B, cs);
}
}  // namespace ra

extern "C" ra_status ra_attention_fwd_host(const void* Q_host, const void* K_host, const void* V_host, void* O_host,
                                           void* Q_dev, void* K_dev, void* V_dev, void* O_dev, int B, int H, int d,
                                           const ra_mask* m, float scale, int mode, ra_stream stream)
{
    if (!Q_host || !K_host || !V_host || !O_host)
        return fail(RA_ERR_INVALID_ARG, "NULL host pointer");
    ra_status st = check_fwd_args(Q_dev, K_dev, V_dev, O_dev, B, H, d, m, scale, mode);
    if (st != RA_OK)
        return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(B) * H * m->geom.n * d * 2;
    RA_CUDA_TRY(cudaMemcpyAsync(Q_dev, Q_host, bytes, cudaMemcpyHostToDevice, cs));
    RA_CUDA_TRY(cudaMemcpyAsync(K_dev, K_host, bytes, cudaMemcpyHostToDevice, cs));
    RA_CUDA_TRY(cudaMemcpyAsync(V_dev, V_host, bytes, cudaMemcpyHostToDevice, cs));
    if ((st = ra_attention_fwd(Q_dev, K_dev, V_dev, O_dev, B, H, d, m, scale, mode, nullptr, stream)) != RA_OK)
        return st;
    RA_CUDA_TRY(cudaMemcpyAsync(O_host, O_dev, bytes, cudaMemcpyDeviceToHost, cs));
    return RA_OK;
}

namespace ra {
ra_status device_error_word(int** out)
{
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_err);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    *out = static_cast<int*>(p);
    return RA_OK;
}
}  // namespace ra

extern "C" ra_status ra_get_device_status(ra_stream stream)
{
    RA_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    int word[4];
    RA_CUDA_TRY(cudaMemcpyFromSymbol(word, g_err, sizeof word));
    if (word[0] == 0)
        return RA_OK;
    const int zero[4] = {0, 0, 0, 0};
    RA_CUDA_TRY(cudaMemcpyToSymbol(g_err, zero, sizeof zero));
    return fail(static_cast<ra_status>(word[0]), "device wait gave up (site %d, block %d)", word[1], word[2]);
}

extern "C" ra_status ra_get_device_error_site(int* site, int* block)
{
    int word[4];
    RA_CUDA_TRY(cudaMemcpyFromSymbol(word, g_err, sizeof word));
    if (site)
        *site = word[1];
    if (block)
        *block = word[2];
    return RA_OK;
}

extern "C" ra_status ra_selftest_wait_timeout(long long timeout_ns, ra_stream stream)
{
    if (timeout_ns < 1000000LL || timeout_ns > 10000000000LL)
        return fail(RA_ERR_INVALID_ARG, "timeout_ns must be in [1e6, 1e10]");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    ra_status st = ra_get_device_status(stream);  // start from a clean word
    if (st != RA_OK && st != RA_ERR_DEVICE_TIMEOUT)
        return st;
    wait_selftest_kernel<<<1, 32, 0, cs>>>(static_cast<unsigned long long>(timeout_ns));
    RA_CUDA_TRY(cudaGetLastError());
    return ra_get_device_status(stream);
}

extern "C" ra_status ra_selftest_bounds(ra_stream stream)
{
#ifdef RA_DEBUG_BOUNDS
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    ra_status st = ra_get_device_status(stream);  // start from a clean word
    if (st != RA_OK && st != RA_ERR_DEVICE_TIMEOUT && st != RA_ERR_DEVICE_BOUNDS)
        return st;
    bounds_selftest_kernel<<<1, 32, 0, cs>>>();
    RA_CUDA_TRY(cudaGetLastError());
    return ra_get_device_status(stream);
#else
    (void)stream;
    return fail(RA_ERR_UNSUPPORTED, "bounds checks are compiled only into the debug library (-DRA_DEBUG_BOUNDS)");
#endif
}

extern "C" ra_status ra_set_pv_precision(int policy)
{
    if (policy != RA_PV_AUTO && policy != RA_PV_BF16 && policy != RA_PV_SPLIT)
        return fail(RA_ERR_INVALID_ARG, "unknown P precision policy %d", policy);
    g_pv_policy.store(policy, std::memory_order_relaxed);
    return RA_OK;
}
