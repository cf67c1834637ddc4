// ra_attention.cu -- block-sparse attention forward for sm_100a (B200).
//
// Computes, per (batch b, head h, 128-row query tile qb),
//     O = softmax(scale * Q K^T + M) V        ("Radial Attention ..." eq. 2)
// over the kept 128 x 128 tiles of the query tile's block-CSR row
// (sec. 6: 128 x 128 block granularity).  In token-exact mode a PARTIAL tile
// applies the element mask; in block mode every valid pair of a kept tile is
// used.  Keys >= n are masked in both modes; rows >= n are never stored.
//
// One CTA per query tile, 6 warps with fixed roles:
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); reads S from
//              TMEM, masks, keeps a running max / sum, writes P (bf16) back to
//              TMEM over S, rescales O in TMEM when the max grows by > 2^8,
//              and runs the epilogue O / l -> bf16.
//   warp 4     producer: one thread issues TMA loads of Q once and of the K / V
//              tiles of the row into two-stage rings (128-byte swizzle).
//   warp 5     MMA: allocates 512 TMEM columns; one thread issues
//              S_j = Q K_j^T (tcgen05.mma, A and B from shared memory) into one of
//              three S buffers, and O += P_j V_j (A = P from TMEM, B = V from
//              shared memory); completion is signalled by tcgen05.commit.
// TMEM columns: S buffers at 0, 128, 256 (fp32, 128 columns each; P overlays
// the first 64 columns as packed bf16 pairs), O at 384 (fp32, d columns).
//
// Online softmax in base 2: x = S * scale * log2(e); p = 2^(x - m) with m a
// running maximum that is only raised (and O, l rescaled) when a tile's maximum
// exceeds it by more than 8; p <= 2^8 otherwise, which fp32 and bf16 hold
// exactly as well as p <= 1, and O / l is independent of the reference m.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>

#include "ra_internal.h"
#include "ra_sm100.cuh"

namespace ra {

// Device error word of the forward kernels: [0] status, [1] site, [2] block.
__device__ int g_err[4];

namespace {

constexpr int NUM_THREADS = 192;
constexpr int KV_STAGES = 2;
constexpr int S_BUFS = 3;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 384;
constexpr float RESCALE_THRESHOLD = 8.0f;

// Wait-site codes recorded with a timeout.
enum : int {
    SITE_Q_FULL = 1, SITE_K_EMPTY, SITE_V_EMPTY, SITE_S_FREE, SITE_K_FULL, SITE_P_FULL, SITE_V_FULL,
    SITE_S_FULL, SITE_PV_DONE, SITE_O_FINAL, SITE_DRAIN, SITE_SELFTEST
};

template <int D>
struct Layout {
    static constexpr int CHUNKS = D / 64;                  // 128-byte swizzle atoms across d
    static constexpr int CHUNK_BYTES = TILE * 128;          // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES; // one 128 x d bf16 tile
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + TILE_BYTES;
    static constexpr int V_OFF = K_OFF + KV_STAGES * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + KV_STAGES * TILE_BYTES;
    static constexpr int BAR_BYTES = 256;
    // + alignment slack; at least 120 KB so that one CTA (and its 512 TMEM
    // columns) owns the SM.
    static constexpr int SMEM_NEEDED = BAR_OFF + BAR_BYTES + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEEDED > 120 * 1024 ? SMEM_NEEDED : 120 * 1024;
};

// Barrier slots (8 bytes each) inside the barrier region.
enum : int {
    B_Q_FULL = 0,
    B_K_FULL = 1,       // + stage
    B_K_EMPTY = 3,      // + stage
    B_V_FULL = 5,       // + stage
    B_V_EMPTY = 7,      // + stage
    B_S_FULL = 9,       // + buffer
    B_P_FULL = 12,      // + buffer
    B_S_FREE = 15,      // + buffer
    B_PV_DONE = 18,
    B_O_FINAL = 19,
    B_COUNT = 20
};

struct FwdParams {
    MaskGeom g;
    int nb, H, mode;
    const int* row_ptr;
    const int* col_idx;
    const unsigned char* flag;
    __nv_bfloat16* O;
    float* lse;
    float scale_log2;  // scale * log2(e)
    unsigned long long timeout_ns;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Wait without the CTA abort flag: used only to drain in-flight copies and
// MMAs before the CTA releases its memory.
__device__ bool drain_wait(uint32_t bar, uint32_t parity, unsigned long long timeout_ns)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > timeout_ns)
            return false;
    }
    return true;
}

// SPLIT_P: P is kept as hi + lo bf16 pairs (P = hi + lo to ~16 bits) and
// P V runs as two MMAs; used for masks whose rows hold few keys, where the
// rounding of P to bf16 is not averaged out over many keys.
template <int D, bool SPLIT_P>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p)
{
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles.
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_addr);
    const uint32_t sQ = sbase + L::Q_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
    const uint32_t bars = sbase + L::BAR_OFF;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR_OFF + 8 * B_COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::BAR_OFF + 8 * B_COUNT + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int n = p.g.n;
    WaitCtl wc{abort_flag, g_err, p.timeout_ns};

    if (threadIdx.x == 0) {
        *abort_flag = *reinterpret_cast<volatile int*>(g_err) != 0 ? 1 : 0;
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(bar(i), (i >= B_P_FULL && i < B_P_FULL + S_BUFS) ? 128u : 1u);
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

    const int row_start = p.row_ptr[qb];
    const int L_row = skip ? 0 : p.row_ptr[qb + 1] - row_start;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && L_row > 0) {
            tma_prefetch_map(&tmQ);
            tma_prefetch_map(&tmK);
            tma_prefetch_map(&tmV);
            mbar_arrive_expect_tx(bar(B_Q_FULL), L::TILE_BYTES);
            for (int c = 0; c < L::CHUNKS; ++c)
                tma_load_3d(sQ + c * L::CHUNK_BYTES, &tmQ, bar(B_Q_FULL), c * 64, qb * TILE, bh);
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < L_row; ++j) {
                const int st = j & 1;
                const int kb = p.col_idx[row_start + j];
                if (j >= KV_STAGES && !mbar_wait(bar(B_K_EMPTY + st), ((j >> 1) - 1) & 1, wc, SITE_K_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(B_K_FULL + st), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sK + st * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmK, bar(B_K_FULL + st), c * 64,
                                kb * TILE, bh);
                k_issued = j + 1;
                if (j >= KV_STAGES && !mbar_wait(bar(B_V_EMPTY + st), ((j >> 1) - 1) & 1, wc, SITE_V_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(B_V_FULL + st), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sV + st * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmV, bar(B_V_FULL + st), c * 64,
                                kb * TILE, bh);
                v_issued = j + 1;
            }
            // Let every copy this thread issued land before the CTA can exit.  A
            // load into a stage is issued only after the previous load of that
            // stage was consumed, so only the last load of each stage can be in
            // flight here, and its phase parity identifies it.
            drain_wait(bar(B_Q_FULL), 0, p.timeout_ns);
            for (int j = max(0, k_issued - KV_STAGES); j < k_issued; ++j)
                drain_wait(bar(B_K_FULL + (j & 1)), (j >> 1) & 1, p.timeout_ns);
            for (int j = max(0, v_issued - KV_STAGES); j < v_issued; ++j)
                drain_wait(bar(B_V_FULL + (j & 1)), (j >> 1) & 1, p.timeout_ns);
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0 && L_row > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, TILE, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(TILE, D, 0, 1);
            bool ok = mbar_wait(bar(B_Q_FULL), 0, wc, SITE_Q_FULL);
            tc_fence_after();
            for (int j = 0; ok && j <= L_row; ++j) {
                if (j < L_row) {
                    const int sb = j % S_BUFS, st = j & 1;
                    if (j >= S_BUFS && !(ok = mbar_wait(bar(B_S_FREE + sb), ((j / S_BUFS) - 1) & 1, wc, SITE_S_FREE)))
                        break;
                    if (!(ok = mbar_wait(bar(B_K_FULL + st), (j >> 1) & 1, wc, SITE_K_FULL)))
                        break;
                    tc_fence_after();
                    const uint32_t kbase = sK + st * L::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32;
                        mma_ss(tmem + sb * TILE, smem_desc_sw128(sQ + off, 16, 1024),
                               smem_desc_sw128(kbase + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_S_FULL + sb));
                    mma_commit(bar(B_K_EMPTY + st));
                }
                if (j >= 1) {
                    const int i = j - 1, sb = i % S_BUFS, st = i & 1;
                    if (!(ok = mbar_wait(bar(B_P_FULL + sb), (i / S_BUFS) & 1, wc, SITE_P_FULL)))
                        break;
                    if (!(ok = mbar_wait(bar(B_V_FULL + st), (i >> 1) & 1, wc, SITE_V_FULL)))
                        break;
                    tc_fence_after();
                    const uint32_t vbase = sV + st * L::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < TILE / 16; ++kk)
                        mma_ts(tmem + O_COL, tmem + sb * TILE + kk * 8,
                               smem_desc_sw128(vbase + kk * 2048, L::CHUNK_BYTES, 1024), idesc_pv,
                               (i > 0 || kk > 0) ? 1u : 0u);
                    if (SPLIT_P) {
#pragma unroll
                        for (int kk = 0; kk < TILE / 16; ++kk)
                            mma_ts(tmem + O_COL, tmem + sb * TILE + 64 + kk * 8,
                                   smem_desc_sw128(vbase + kk * 2048, L::CHUNK_BYTES, 1024), idesc_pv, 1u);
                    }
                    mma_commit(bar(B_V_EMPTY + st));
                    mma_commit(bar(B_S_FREE + sb));
                    mma_commit(bar(B_PV_DONE));
                }
            }
            mma_commit(bar(B_O_FINAL));
            // Every MMA issued by this thread has completed once O_FINAL fires.
            drain_wait(bar(B_O_FINAL), 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int t = threadIdx.x;  // == TMEM lane == query row in the tile
        const int row = qb * TILE + t;
        const bool row_valid = row < n;
        const int qi = row_valid ? row / p.g.s : 0, qk = row_valid ? row % p.g.s : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const bool tail = (n % TILE) != 0;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int i = 0; i < L_row; ++i) {
            const int sb = i % S_BUFS;
            const int kb = p.col_idx[row_start + i];
            const bool partial = p.flag[row_start + i] != RA_TILE_FULL;
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_S_FULL + sb), (i / S_BUFS) & 1, wc, SITE_S_FULL));
            if (!ok)
                break;
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(lane_base + sb * TILE + c * 32, r[c]);
            tmem_wait_ld();

            // Mask: token-exact partial tiles use the family's element mask;
            // the tail key tile masks keys >= n in both modes.
            const bool use_family = p.mode == RA_MODE_TOKEN_EXACT && partial;
            if (use_family || (tail && kb == p.nb - 1)) {
                uint32_t mk[4];
                if (use_family && row_valid) {
                    row_keep_mask(p.g, qi, qk, kb * TILE, mk[0], mk[1], mk[2], mk[3]);
                } else {
                    const int valid_cols = min(TILE, n - kb * TILE);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int v = valid_cols - 32 * c;
                        mk[c] = v >= 32 ? 0xFFFFFFFFu : (v <= 0 ? 0u : ((1u << v) - 1u));
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((mk[c] >> e) & 1u))
                            r[c][e] = __float_as_uint(-INFINITY);
            }

            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    mx = fmaxf(mx, __uint_as_float(r[c][e]));
            const float m_tile = mx * p.scale_log2;  // scale > 0

            // Raise the running max (warp-uniformly) only when it grows by > 2^8.
            const bool grow = m_tile > m_run + RESCALE_THRESHOLD;
            if (__any_sync(0xFFFFFFFFu, grow)) {
                const float m_new = fmaxf(m_run, m_tile);
                const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
                if (i > 0) {
                    // O holds P_0..P_{i-1} V: wait for the last PV before rescaling it.
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(B_PV_DONE), (i - 1) & 1, wc, SITE_PV_DONE));
                    if (!ok)
                        break;
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
            }
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[16], pl[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float p0 = fast_exp2(fmaf(__uint_as_float(r[c][e]), p.scale_log2, -m_use));
                    const float p1 = fast_exp2(fmaf(__uint_as_float(r[c][e + 1]), p.scale_log2, -m_use));
                    sum += p0 + p1;
                    pk[e >> 1] = pack_bf16(p0, p1);
                    if (SPLIT_P) {
                        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&pk[e >> 1]);
                        pl[e >> 1] = pack_bf16(p0 - __low2float(hi), p1 - __high2float(hi));
                    }
                }
                tmem_st16(lane_base + sb * TILE + c * 16, pk);
                if (SPLIT_P)
                    tmem_st16(lane_base + sb * TILE + 64 + c * 16, pl);
            }
            l_run += sum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL + sb));
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

// ------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// [B*H, n, d] bf16, boxes of 128 rows x 64 columns, 128-byte swizzle; rows
// beyond n read as zero.
ra_status make_map(CUtensorMap* map, const void* base, int BH, int n, int d)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(n) * d * 2};
    cuuint32_t box[3] = {64, TILE, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return RA_OK;
}

template <int D, bool SPLIT_P>
ra_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p, int B,
                     cudaStream_t cs)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(attn_fwd_kernel<D, SPLIT_P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Layout<D>::SMEM_BYTES);
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

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

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
    if ((st = make_map(&mq, Q, BH, n, d)) != RA_OK || (st = make_map(&mk, K, BH, n, d)) != RA_OK ||
        (st = make_map(&mv, V, BH, n, d)) != RA_OK)
        return st;
    FwdParams p;
    std::memset(&p, 0, sizeof p);
    p.g = m->geom;
    p.nb = m->nb;
    p.H = H;
    p.mode = mode;
    p.row_ptr = m->row_ptr;
    p.col_idx = m->col_idx;
    p.flag = m->flag;
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

extern "C" ra_status ra_set_pv_precision(int policy)
{
    if (policy != RA_PV_AUTO && policy != RA_PV_BF16 && policy != RA_PV_SPLIT)
        return fail(RA_ERR_INVALID_ARG, "unknown P precision policy %d", policy);
    g_pv_policy.store(policy, std::memory_order_relaxed);
    return RA_OK;
}
