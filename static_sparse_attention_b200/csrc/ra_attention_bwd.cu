// ra_attention_bwd.cu -- backward of the block-sparse attention for sm_100a.
//
// Gradients of O = softmax(scale * Q K^T + M) V ("Radial Attention ..." eq. 2)
// over the kept 128 x 128 tiles (sec. 6), given dO and the forward's
// log-sum-exp L:
//   P = exp(scale * S - L),  D_i = <dO_i, O_i>,  dP = dO V^T,  dS = P (dP - D)
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO.
// Deterministic: no atomics, each output tile is owned by one CTA.
//
//   bwd_dot_kernel     D = rowsum(dO * O) (fp32), one warp per row.
//   bwd_dq_kernel      one CTA per query tile, walking its block-CSR row:
//       S = Q K^T and dP = dO V^T (tcgen05.mma into TMEM), dS (registers,
//       bf16 back into TMEM), dQ += dS K (A = dS from TMEM).
//   bwd_dkdv_kernel    one CTA per key tile, walking the transposed CSR:
//       S^T = K Q^T and dP^T = V dO^T, P^T (bf16 into shared memory) and
//       dS^T (bf16 into TMEM), dK += dS^T Q and dV += P^T dO.
// Both recompute P from L instead of storing it, and take the walked side one
// 128-row tile per step, so that every product is an M = 128, N >= 128
// tcgen05.mma (N = 64 runs at about two thirds of the rate).  Each has 320
// threads: two gradient warpgroups that split the step's 128 columns (a thread
// owns one resident row; TMEM lane = row), a TMA producer warp and an MMA warp.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "ra_internal.h"
#include "ra_sm100.cuh"

namespace ra {
namespace {

constexpr uint32_t BWD_TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;

enum : int { BSITE_RES = 21, BSITE_X_EMPTY, BSITE_Y_EMPTY, BSITE_X_FULL, BSITE_Y_FULL, BSITE_S_FULL, BSITE_DS_FULL,
             BSITE_ACC, BSITE_FINAL,
             // bounds checks of the debug build
             BSITE_B_ROW = 50, BSITE_B_TILE, BSITE_B_WALK };

// The order in which a CTA takes the entries of its CSR row: the row's near
// segment [a, b) first, then the others in ascending order (the identity
// without a walk array).
struct RowWalk {
    int a = 0, b = 0;
    __device__ int operator()(int i) const
    {
        const int near = b - a;
        return i < near ? a + i : (i - near < a ? i - near : i);
    }
};

__device__ __forceinline__ RowWalk row_walk(const int* walk, int tile, int len, const WaitCtl& wc)
{
    RowWalk w;
    if (walk && len > 0) {
        w.a = walk[2 * tile];
        w.b = walk[2 * tile + 1];
        if (!in_bounds(wc, 0 <= w.a && w.a <= w.b && w.b <= len, BSITE_B_WALK))  // (debug build)
            w.a = w.b = 0;
    }
    return w;
}

struct BwdParams {
    MaskGeom g;
    int nb, H, mode;
    const int* ptr;            // row_ptr (dQ pass) or col_ptr (dK/dV pass)
    const int* idx;            // col_idx or row_idx
    const unsigned char* flag; // flag or tflag
    const int* order;          // tile of CTA x (the mask's dispatch order), or null for x itself
    const int* walk;           // [2 nb]: offsets a, b of each row's near segment, walked first; or null
    int nnz;                   // entries of idx / flag (bounds checks of the debug build)
    const float* lse;          // [B*H, n] natural log
    const float* Dv;           // [B*H, n] rowsum(dO * O)
    __nv_bfloat16* out0;       // dQ, or dK
    __nv_bfloat16* out1;       // unused, or dV
    float scale, scale_log2;
    int* err;
    unsigned long long timeout_ns;
};

// Barrier over one gradient warpgroup (named barrier `id`, 128 threads).
__device__ __forceinline__ void sync_wg(uint32_t id) { asm volatile("barrier.sync %0, 128;" ::"r"(id) : "memory"); }

// The same barrier, also ANDing a predicate across the warpgroup, so that its
// four warps take the same abort decision.
__device__ __forceinline__ bool sync_and_wg(uint32_t id, bool pred)
{
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(pred)), "r"(id)
        : "memory");
    return out != 0;
}

// Packed fp32 pairs (sm_100 f32x2 instructions): one instruction for two
// lanes' worth of IEEE fma / add / mul, each rounded to nearest as the scalar
// forms are, so the gradients keep the same bits as with scalar arithmetic.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t f2pack_u(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
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
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Gradient of one pair of walked columns: p = 2^(s c + nl), ds = p (dp + nd),
// where nl = -L log2 e and nd = -D of the pair's rows.  A masked-out element
// arrives as s = -inf (c > 0), so its p is exactly 0.
__device__ __forceinline__ void grad_pair(uint32_t s0, uint32_t s1, uint32_t dp0, uint32_t dp1, uint64_t c2,
                                          uint64_t nl2, uint64_t nd2, float& p0, float& p1, float& ds0, float& ds1)
{
    float x0, x1;
    f2unpack(f2fma(f2pack_u(s0, s1), c2, nl2), x0, x1);
    p0 = fast_exp2(x0);
    p1 = fast_exp2(x1);
    f2unpack(f2mul(f2pack(p0, p1), f2add(f2pack_u(dp0, dp1), nd2)), ds0, ds1);
}

// The same with explicit keep bits: p = 0 where a bit is clear.  The dK / dV
// walk uses it on every tile (its keep bits are all set outside token-exact
// partial tiles); the -inf pass of mask_chunk costs that kernel a register
// spill.
__device__ __forceinline__ void grad_pair_keep(uint32_t s0, uint32_t s1, uint32_t dp0, uint32_t dp1, uint64_t c2,
                                               uint64_t nl2, uint64_t nd2, bool k0, bool k1, float& p0, float& p1,
                                               float& ds0, float& ds1)
{
    float x0, x1;
    f2unpack(f2fma(f2pack_u(s0, s1), c2, nl2), x0, x1);
    p0 = k0 ? fast_exp2(x0) : 0.f;
    p1 = k1 ? fast_exp2(x1) : 0.f;
    f2unpack(f2mul(f2pack(p0, p1), f2add(f2pack_u(dp0, dp1), nd2)), ds0, ds1);
}

// Sets the elements of a 32-column chunk of S whose bit in `keep` is clear to -inf.
__device__ __forceinline__ void mask_chunk(uint32_t (&s)[32], uint32_t keep)
{
#pragma unroll
    for (int e = 0; e < 32; ++e)
        if (!((keep >> e) & 1u))
            s[e] = __float_as_uint(-INFINITY);
}

// ---------------------------------------------------------------------------
// dQ kernel with 128-key steps.  A tcgen05.mma of M = 128 runs at the full
// rate only for N >= 128 (N = 64 reaches about two thirds), so S = Q K^T and
// dP = dO V^T are computed for a whole 128-key tile per step.  TMEM: S in two
// buffers (columns 0 and 128), dP in one (256; the gradient warps load it into
// registers first and release it at once), dQ at 384.  The MMA warp issues
// dP_j, then S_j, then the gradient MMA of step j - 1.  S_j overwrites the dS
// that the gradient MMA of step j - 2 reads; a tcgen05.shift on that buffer
// between the two orders them (MMA -> shift -> MMA are pipelined pairs of the
// PTX ISA, executed in issue order), with no wait.
// 320 threads: two gradient warpgroups (columns 64 wg .. 64 wg + 63 of each
// step), warp 8 issues the TMA loads, warp 9 the MMAs.
constexpr int DQ_THREADS = 320, DQ_GRAD_THREADS = 256, DQ_PRODUCER_WARP = 8, DQ_MMA_WARP = 9;
constexpr uint32_t DQ_COL_DP = 256, DQ_COL_ACC = 384;
__host__ __device__ constexpr uint32_t dq_s_col(int b) { return 128u * static_cast<uint32_t>(b); }

template <int D>
struct DqLayout {
    static constexpr int CHUNKS = D / 64;
    static constexpr int CHUNK_BYTES = TILE * 128;          // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES; // a 128 x d tile
    static constexpr int KS = D == 64 ? 3 : 2;               // K tile ring
    static constexpr int VS = D == 64 ? 3 : 2;               // V tile ring
    static constexpr int Q_OFF = 0, DO_OFF = TILE_BYTES;
    static constexpr int K_OFF = 2 * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + KS * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + VS * TILE_BYTES;
    static constexpr int SMEM_NEEDED = BAR_OFF + 256 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEEDED > 120 * 1024 ? SMEM_NEEDED : 120 * 1024;
};

template <int KS, int VS>
struct DqBars {
    static constexpr int RES_FULL = 0;
    static constexpr int K_FULL = 1;
    static constexpr int K_EMPTY = K_FULL + KS;
    static constexpr int V_FULL = K_EMPTY + KS;
    static constexpr int V_EMPTY = V_FULL + VS;
    static constexpr int S_FULL = V_EMPTY + VS;  // + buffer: S_j and dP_j complete
    static constexpr int DP_FREE = S_FULL + 2;   // the gradient warps have loaded dP
    static constexpr int DS_FULL = DP_FREE + 1;  // + buffer: dS of the step written
    static constexpr int FINAL = DS_FULL + 2;
    static constexpr int COUNT = FINAL + 1;
};

template <int D>
__global__ void __launch_bounds__(DQ_THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const BwdParams p)
{
    using L = DqLayout<D>;
    using BB = DqBars<L::KS, L::VS>;
    static_assert(BB::COUNT * 8 + 8 <= 256, "barrier area");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_addr);
    const uint32_t sQ = sbase + L::Q_OFF, sDO = sbase + L::DO_OFF, sK = sbase + L::K_OFF, sV = sbase + L::V_OFF;
    const uint32_t bars = sbase + L::BAR_OFF;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR_OFF + 8 * BB::COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::BAR_OFF + 8 * BB::COUNT + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.order ? p.order[blockIdx.x] : static_cast<int>(blockIdx.x);
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int n = p.g.n;
    WaitCtl wc{abort_flag, p.err, p.timeout_ns};

    if (threadIdx.x == 0) {
        *abort_flag = *reinterpret_cast<volatile int*>(p.err) != 0 ? 1 : 0;
        for (int i = 0; i < BB::COUNT; ++i) {
            const bool grad = i == BB::DP_FREE || i == BB::DS_FULL || i == BB::DS_FULL + 1;
            mbar_init(bar(i), grad ? static_cast<uint32_t>(DQ_GRAD_THREADS) : 1u);
        }
        fence_barrier_init();
        fence_proxy_async_smem();
        // (debug build) this CTA's tile and its CSR row are in range
        if (!*abort_flag && in_bounds(wc, qb >= 0 && qb < p.nb, BSITE_B_TILE))
            in_bounds(wc, 0 <= p.ptr[qb] && p.ptr[qb] <= p.ptr[qb + 1] && p.ptr[qb + 1] <= p.nnz, BSITE_B_ROW);
    }
    if (warp == DQ_MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), BWD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort_flag != 0;
    const int start = skip ? 0 : p.ptr[qb];
    const int len = skip ? 0 : p.ptr[qb + 1] - start;
    const RowWalk walk = row_walk(p.walk, qb, len, wc);

    if (warp == DQ_PRODUCER_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && len > 0) {
            mbar_arrive_expect_tx(bar(BB::RES_FULL), 2 * L::TILE_BYTES);
            for (int c = 0; c < L::CHUNKS; ++c) {
                tma_load_3d(sQ + c * L::CHUNK_BYTES, &tmQ, bar(BB::RES_FULL), c * 64, qb * TILE, bh);
                tma_load_3d(sDO + c * L::CHUNK_BYTES, &tmDO, bar(BB::RES_FULL), c * 64, qb * TILE, bh);
            }
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < len; ++j) {
                const int tile = p.idx[start + walk(j)];
                if (!in_bounds(wc, tile >= 0 && tile < p.nb, BSITE_B_TILE))  // (debug build)
                    break;
                const int row0 = tile * TILE;
                const int ks = j % L::KS, vs = j % L::VS;
                if (j >= L::VS && !mbar_wait(bar(BB::V_EMPTY + vs), ((j / L::VS) - 1) & 1, wc, BSITE_Y_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(BB::V_FULL + vs), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sV + vs * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmV, bar(BB::V_FULL + vs), c * 64, row0,
                                bh);
                v_issued = j + 1;
                if (j >= L::KS && !mbar_wait(bar(BB::K_EMPTY + ks), ((j / L::KS) - 1) & 1, wc, BSITE_X_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(BB::K_FULL + ks), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sK + ks * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmK, bar(BB::K_FULL + ks), c * 64, row0,
                                bh);
                k_issued = j + 1;
            }
            drain_wait(bar(BB::RES_FULL), 0, p.timeout_ns);
            for (int j = max(0, k_issued - L::KS); j < k_issued; ++j)
                drain_wait(bar(BB::K_FULL + j % L::KS), (j / L::KS) & 1, p.timeout_ns);
            for (int j = max(0, v_issued - L::VS); j < v_issued; ++j)
                drain_wait(bar(BB::V_FULL + j % L::VS), (j / L::VS) & 1, p.timeout_ns);
        }
    } else if (warp == DQ_MMA_WARP) {
        // ----------------------------------------------------------------- MMA
        if (len > 0) {
            const bool leader = elect_one();
            constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, TILE, 0, 0);  // A, B K-major, N = 128
            constexpr uint32_t idesc_acc = idesc_bf16_f32(TILE, D, 0, 1);   // A from TMEM, B MN-major
            // The whole warp runs the loop, so that the descriptors (built once;
            // each MMA only advances the start address) stay warp-uniform; the
            // elected lane issues the MMAs and commits.  The warp shares its
            // sub-partition with gradient warps.
            const uint64_t dQd = smem_desc_sw128(sQ, 16, 1024), dOd = smem_desc_sw128(sDO, 16, 1024);
            const uint64_t dKd = smem_desc_sw128(sK, 16, 1024), dVd = smem_desc_sw128(sV, 16, 1024);
            const uint64_t dKmn = smem_desc_sw128(sK, L::CHUNK_BYTES, 1024);  // K tiles as MN-major B
            // D[col] = A(resident 128 x d) * B(128-row tile)^T over d.
            auto mma_s = [&](uint32_t col, uint64_t a, uint64_t b2) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32;
                    const uint64_t ad = desc_add(a, off), bd = desc_add(b2, off);
                    mma_ss(leader, tmem + col, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // dQ += dS_j K_j: dS packed by the warpgroups, keys 16 kk .. 16 kk + 15
            // at columns 64 (kk / 4) + 8 (kk % 4) of the step's S buffer.
            auto issue_acc = [&](int j) {
                const int bf = j & 1, ks = j % L::KS;  // dS_j in S buffer bf
                const uint64_t kdesc = desc_add(dKmn, ks * L::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < TILE / 16; ++kk) {
                    const uint64_t bd = desc_add(kdesc, kk * 2048);
                    mma_ts(leader, tmem + DQ_COL_ACC, tmem + dq_s_col(bf) + (kk >> 2) * 64 + (kk & 3) * 8, bd,
                           idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
                }
                if (leader)
                    mma_commit(bar(BB::K_EMPTY + ks));
            };
            auto wait_all = [&](uint32_t b, uint32_t parity, int site) {
                return __all_sync(0xFFFFFFFFu, mbar_wait(b, parity, wc, site));
            };
            bool ok = wait_all(bar(BB::RES_FULL), 0, BSITE_RES);
            tc_fence_after();
            int acc_issued = 0;
            for (int j = 0; ok && j < len; ++j) {
                const int bf = j & 1, ks = j % L::KS, vs = j % L::VS;
                // dP_j into the single dP buffer, once the gradient warps have loaded dP_{j-1}
                if (!(ok = wait_all(bar(BB::V_FULL + vs), (j / L::VS) & 1, BSITE_Y_FULL)))
                    break;
                if (j >= 1 && !(ok = wait_all(bar(BB::DP_FREE), (j - 1) & 1, BSITE_DS_FULL)))
                    break;
                tc_fence_after();
                mma_s(DQ_COL_DP, dOd, desc_add(dVd, vs * L::TILE_BYTES));
                if (leader)
                    mma_commit(bar(BB::V_EMPTY + vs));
                // S_j into buffer bf, after the gradient MMA of step j - 2 that
                // reads dS from it: MMAs into different accumulators are not
                // ordered, MMA -> shift -> MMA is
                if (!(ok = wait_all(bar(BB::K_FULL + ks), (j / L::KS) & 1, BSITE_X_FULL)))
                    break;
                tc_fence_after();
                if (j >= 2 && leader)
                    tmem_shift_down(tmem + dq_s_col(bf));
                mma_s(dq_s_col(bf), dQd, desc_add(dKd, ks * L::TILE_BYTES));
                if (leader)
                    mma_commit(bar(BB::S_FULL + bf));
                if (j >= 1) {
                    if (!(ok = wait_all(bar(BB::DS_FULL + (bf ^ 1)), ((j - 1) >> 1) & 1, BSITE_DS_FULL)))
                        break;
                    tc_fence_after();
                    issue_acc(j - 1);
                    acc_issued = j;
                }
            }
            if (ok && acc_issued == len - 1) {
                if (wait_all(bar(BB::DS_FULL + ((len - 1) & 1)), ((len - 1) >> 1) & 1, BSITE_DS_FULL)) {
                    tc_fence_after();
                    issue_acc(len - 1);
                }
            }
            if (leader)
                mma_commit(bar(BB::FINAL));
            drain_wait(bar(BB::FINAL), 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------ gradient warps
        const int wg = warp >> 2;            // warpgroup: columns 64 wg .. 64 wg + 63 of each step
        const int t = threadIdx.x & 127;     // == TMEM lane: query row of the tile
        const int row = qb * TILE + t;
        const bool row_valid = row < n;
        const int rf = row_valid ? row / p.g.s : 0, rp = row_valid ? row % p.g.s : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t my_col = 64u * static_cast<uint32_t>(wg);
        const bool tail = (n % TILE) != 0;
        const float row_l2 = row_valid ? p.lse[static_cast<size_t>(bh) * n + row] * LOG2E : 0.f;
        const float row_d = row_valid ? p.Dv[static_cast<size_t>(bh) * n + row] : 0.f;
        // a row with no kept key (lse = -inf) has P = 0 everywhere
        const float nl = row_l2 > -INFINITY ? -row_l2 : -INFINITY;
        const uint64_t c2 = f2pack(p.scale_log2, p.scale_log2), nl2 = f2pack(nl, nl), nd2 = f2pack(-row_d, -row_d);
        bool ok = true;
        // CSR entry of the next step, loaded one step ahead of its use
        int next_kb = len > 0 ? p.idx[start + walk(0)] : 0;
        int next_flag = len > 0 ? p.flag[start + walk(0)] : 0;
        for (int j = 0; j < len; ++j) {
            const int bf = j & 1;
            const int kb = next_kb;
            const bool use_family = p.mode == RA_MODE_TOKEN_EXACT && next_flag != RA_TILE_FULL;
            if (j + 1 < len) {
                next_kb = p.idx[start + walk(j + 1)];
                next_flag = p.flag[start + walk(j + 1)];
            }
            const bool masked = use_family || (tail && kb == p.nb - 1);
            uint32_t mk[4] = {~0u, ~0u, ~0u, ~0u};
            if (masked) {
                if (use_family && row_valid) {
                    row_keep_mask(p.g, rf, rp, kb * TILE, mk[0], mk[1], mk[2], mk[3]);
                } else {
                    const int valid_cols = min(TILE, n - kb * TILE);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int v = valid_cols - 32 * c;
                        mk[c] = v >= 32 ? 0xFFFFFFFFu : (v <= 0 ? 0u : ((1u << v) - 1u));
                    }
                }
            }
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(BB::S_FULL + bf), (j >> 1) & 1, wc, BSITE_S_FULL));
            if (!ok)
                break;
            tc_fence_after();
            // dP (and the first S chunk) first, then release the dP buffer for the
            // next step's MMA; the second S chunk loads while the first is processed
            uint32_t dv[2][32], sv[2][32];
            tmem_ld32(lane_base + DQ_COL_DP + my_col, dv[0]);
            tmem_ld32(lane_base + DQ_COL_DP + my_col + 32, dv[1]);
            tmem_ld32(lane_base + dq_s_col(bf) + my_col, sv[0]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(BB::DP_FREE));
            tmem_ld32(lane_base + dq_s_col(bf) + my_col + 32, sv[1]);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (c == 1)
                    tmem_wait_ld();
                if (masked)  // warp-uniform
                    mask_chunk(sv[c], wg ? (c ? mk[3] : mk[2]) : (c ? mk[1] : mk[0]));
                uint32_t dk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p0, p1, ds0, ds1;
                    grad_pair(sv[c][e], sv[c][e + 1], dv[c][e], dv[c][e + 1], c2, nl2, nd2, p0, p1, ds0, ds1);
                    dk[e >> 1] = pack_bf16(ds0, ds1);
                }
                // Packed into columns this warpgroup has already read.
                tmem_st16(lane_base + dq_s_col(bf) + my_col + c * 16, dk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(BB::DS_FULL + bf));
        }
        // ------------------------------------------------------------ epilogue
        if (len > 0 && ok)
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(BB::FINAL), 0, wc, BSITE_FINAL));
        tc_fence_after();
        // tcgen05.ld is warp-collective: every lane loads, only rows < n store;
        // warpgroup wg stores dQ columns [wg d/2, (wg + 1) d/2)
        if (__all_sync(0xFFFFFFFFu, ok && !*abort_flag)) {
            __nv_bfloat16* dst_row = p.out0 + (static_cast<size_t>(bh) * n + row) * D;
            constexpr int C_PER_WG = D / 64;
#pragma unroll
            for (int cc = 0; cc < C_PER_WG; ++cc) {
                const int c = wg * C_PER_WG + cc;
                uint32_t o[32];
                if (len > 0) {
                    tmem_ld32(lane_base + DQ_COL_ACC + c * 32, o);
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
                    w[e >> 1] = pack_bf16(__uint_as_float(o[e]) * p.scale, __uint_as_float(o[e + 1]) * p.scale);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = v[u];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == DQ_MMA_WARP) {
        __syncwarp();
        tmem_dealloc(tmem, BWD_TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// dK / dV kernel with 128-query steps (N = 128 products).  One CTA per key
// tile walks the transposed block-CSR.  TMEM (512 columns) holds S^T (0),
// dP^T (128; dS^T is packed back over its first half), dK (256) and dV (384),
// so P^T, the A operand of dV += P^T dO, goes to shared memory in the
// 128-byte-swizzled K-major layout.  Per step j the MMA warp issues S^T_{j+1}
// as soon as the gradient warps have loaded S^T_j and dP^T_j into registers;
// the half of dK_j that reads the first 32-column chunk of each warpgroup's
// dS^T as soon as those chunks are written (while the gradient warps work on
// their second chunks), the other half when the step's dS^T is complete; then
// dP^T_{j+1} over the dS^T columns, ordered after dK_j by a tcgen05.shift
// (MMA -> shift -> MMA are pipelined pairs of the PTX ISA, executed in issue
// order), with no wait; then dV_j.  320 threads: two gradient warpgroups
// (query columns 64 wg .. 64 wg + 63 of each step), warp 8 issues the TMA
// loads, warp 9 the MMAs.
constexpr int KV_THREADS = 320, KV_GRAD_THREADS = 256, KV_PRODUCER_WARP = 8, KV_MMA_WARP = 9;
constexpr uint32_t KV_COL_S = 0, KV_COL_DP = 128, KV_COL_DK = 256, KV_COL_DV = 384;

template <int D>
struct KvLayout {
    static constexpr int CHUNKS = D / 64;
    static constexpr int CHUNK_BYTES = TILE * 128;           // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;  // a 128 x d tile
    static constexpr int PT_BYTES = 2 * CHUNK_BYTES;         // P^T: 128 keys x 128 queries bf16
    static constexpr int QS = D == 64 ? 3 : 2;                // Q tile ring
    static constexpr int OS = D == 64 ? 3 : 2;                // dO tile ring
    static constexpr int K_OFF = 0, V_OFF = TILE_BYTES;
    static constexpr int Q_OFF = 2 * TILE_BYTES;
    static constexpr int DO_OFF = Q_OFF + QS * TILE_BYTES;
    static constexpr int PT_OFF = DO_OFF + OS * TILE_BYTES;
    static constexpr int STAT_OFF = PT_OFF + PT_BYTES;        // [L2, D][128] floats
    static constexpr int BAR_OFF = STAT_OFF + 2 * TILE * 4;
    static constexpr int SMEM_NEEDED = BAR_OFF + 256 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEEDED > 120 * 1024 ? SMEM_NEEDED : 120 * 1024;
    static_assert(SMEM_NEEDED <= 232448, "shared memory");
};

template <int QS, int OS>
struct KvBars {
    static constexpr int RES_FULL = 0;
    static constexpr int Q_FULL = 1;
    static constexpr int Q_EMPTY = Q_FULL + QS;
    static constexpr int O_FULL = Q_EMPTY + QS;
    static constexpr int O_EMPTY = O_FULL + OS;
    static constexpr int S_FULL = O_EMPTY + OS;  // S^T_j and dP^T_j complete (and every earlier MMA)
    static constexpr int S_FREE = S_FULL + 1;    // the gradient warps have loaded S^T_j and dP^T_j
    static constexpr int DS_FULL = S_FREE + 1;   // P^T_j (shared memory) and dS^T_j (TMEM) written
    static constexpr int DS_HALF = DS_FULL + 1;  // the first 32-column chunk of each warpgroup's dS^T_j written
    static constexpr int DV_DONE = DS_HALF + 1;  // dV += P^T_j dO_j complete (P^T may be overwritten)
    static constexpr int FINAL = DV_DONE + 1;
    static constexpr int COUNT = FINAL + 1;
};

template <int D>
__global__ void __launch_bounds__(KV_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p)
{
    using L = KvLayout<D>;
    using BB = KvBars<L::QS, L::OS>;
    static_assert(BB::COUNT * 8 + 8 <= 256, "barrier area");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw_addr);
    const uint32_t sK = sbase + L::K_OFF, sV = sbase + L::V_OFF, sQ = sbase + L::Q_OFF, sO = sbase + L::DO_OFF;
    const uint32_t sPT = sbase + L::PT_OFF;
    const uint32_t bars = sbase + L::BAR_OFF;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR_OFF + 8 * BB::COUNT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::BAR_OFF + 8 * BB::COUNT + 4);
    float* st_l2 = reinterpret_cast<float*>(smem + L::STAT_OFF);
    float* st_d = st_l2 + TILE;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb = p.order ? p.order[blockIdx.x] : static_cast<int>(blockIdx.x);
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int n = p.g.n;
    WaitCtl wc{abort_flag, p.err, p.timeout_ns};

    if (threadIdx.x == 0) {
        *abort_flag = *reinterpret_cast<volatile int*>(p.err) != 0 ? 1 : 0;
        for (int i = 0; i < BB::COUNT; ++i) {
            const bool grad = i == BB::S_FREE || i == BB::DS_FULL || i == BB::DS_HALF;
            mbar_init(bar(i), grad ? static_cast<uint32_t>(KV_GRAD_THREADS) : 1u);
        }
        fence_barrier_init();
        fence_proxy_async_smem();
        // (debug build) this CTA's tile and its CSR row are in range
        if (!*abort_flag && in_bounds(wc, kb >= 0 && kb < p.nb, BSITE_B_TILE))
            in_bounds(wc, 0 <= p.ptr[kb] && p.ptr[kb] <= p.ptr[kb + 1] && p.ptr[kb + 1] <= p.nnz, BSITE_B_ROW);
    }
    if (warp == KV_MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), BWD_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip = *abort_flag != 0;
    const int start = skip ? 0 : p.ptr[kb];
    const int len = skip ? 0 : p.ptr[kb + 1] - start;
    const RowWalk walk = row_walk(p.walk, kb, len, wc);

    if (warp == KV_PRODUCER_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && len > 0) {
            mbar_arrive_expect_tx(bar(BB::RES_FULL), 2 * L::TILE_BYTES);
            for (int c = 0; c < L::CHUNKS; ++c) {
                tma_load_3d(sK + c * L::CHUNK_BYTES, &tmK, bar(BB::RES_FULL), c * 64, kb * TILE, bh);
                tma_load_3d(sV + c * L::CHUNK_BYTES, &tmV, bar(BB::RES_FULL), c * 64, kb * TILE, bh);
            }
            int q_issued = 0, o_issued = 0;
            for (int j = 0; j < len; ++j) {
                const int tile = p.idx[start + walk(j)];
                if (!in_bounds(wc, tile >= 0 && tile < p.nb, BSITE_B_TILE))  // (debug build)
                    break;
                const int row0 = tile * TILE;
                const int qs = j % L::QS, os = j % L::OS;
                if (j >= L::QS && !mbar_wait(bar(BB::Q_EMPTY + qs), ((j / L::QS) - 1) & 1, wc, BSITE_X_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(BB::Q_FULL + qs), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sQ + qs * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmQ, bar(BB::Q_FULL + qs), c * 64, row0,
                                bh);
                q_issued = j + 1;
                if (j >= L::OS && !mbar_wait(bar(BB::O_EMPTY + os), ((j / L::OS) - 1) & 1, wc, BSITE_Y_EMPTY))
                    break;
                mbar_arrive_expect_tx(bar(BB::O_FULL + os), L::TILE_BYTES);
                for (int c = 0; c < L::CHUNKS; ++c)
                    tma_load_3d(sO + os * L::TILE_BYTES + c * L::CHUNK_BYTES, &tmDO, bar(BB::O_FULL + os), c * 64,
                                row0, bh);
                o_issued = j + 1;
            }
            drain_wait(bar(BB::RES_FULL), 0, p.timeout_ns);
            for (int j = max(0, q_issued - L::QS); j < q_issued; ++j)
                drain_wait(bar(BB::Q_FULL + j % L::QS), (j / L::QS) & 1, p.timeout_ns);
            for (int j = max(0, o_issued - L::OS); j < o_issued; ++j)
                drain_wait(bar(BB::O_FULL + j % L::OS), (j / L::OS) & 1, p.timeout_ns);
        }
    } else if (warp == KV_MMA_WARP) {
        // ----------------------------------------------------------------- MMA
        if (len > 0) {
            const bool leader = elect_one();
            constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, TILE, 0, 0);  // A, B K-major, N = 128
            constexpr uint32_t idesc_acc = idesc_bf16_f32(TILE, D, 0, 1);   // A K-major, B MN-major
            // The whole warp runs the loop, so that the descriptors (built once;
            // each MMA only advances the start address) stay warp-uniform; the
            // elected lane issues the MMAs and commits.  The warp shares its
            // sub-partition with gradient warps.
            const uint64_t dKd = smem_desc_sw128(sK, 16, 1024), dVd = smem_desc_sw128(sV, 16, 1024);
            const uint64_t dQd = smem_desc_sw128(sQ, 16, 1024), dOd = smem_desc_sw128(sO, 16, 1024);
            const uint64_t dPTd = smem_desc_sw128(sPT, 16, 1024);
            const uint64_t dQmn = smem_desc_sw128(sQ, L::CHUNK_BYTES, 1024);  // Q tiles as MN-major B
            const uint64_t dOmn = smem_desc_sw128(sO, L::CHUNK_BYTES, 1024);  // dO tiles as MN-major B
            // D[col] = A(resident 128 x d) * B(128-row tile)^T over d.
            auto mma_s = [&](uint32_t col, uint64_t a, uint64_t b2) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32;
                    const uint64_t ad = desc_add(a, off), bd = desc_add(b2, off);
                    mma_ss(leader, tmem + col, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // dK += dS^T_j Q_j: dS^T packed by the warpgroups, queries 16 kk .. 16 kk + 15
            // at columns 64 (kk / 4) + 8 (kk % 4) of the dP^T buffer.  Half h of
            // the products: kk = 4 wg + 2 h + {0, 1}, the h-th 32-column chunk of
            // each warpgroup; the Q tile is released after the second half.
            auto issue_dk = [&](int j, int half) {
                const int qs = j % L::QS;
                const uint64_t qdesc = desc_add(dQmn, qs * L::TILE_BYTES);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int kk = 4 * (u >> 1) + 2 * half + (u & 1);
                    const uint64_t bd = desc_add(qdesc, kk * 2048);
                    mma_ts(leader, tmem + KV_COL_DK, tmem + KV_COL_DP + (kk >> 2) * 64 + (kk & 3) * 8, bd,
                           idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
                }
                if (leader && half == 1)
                    mma_commit(bar(BB::Q_EMPTY + qs));
            };
            // dV += P^T_j dO_j: P^T from shared memory (K-major over the queries).
            auto issue_dv = [&](int j) {
                const int os = j % L::OS;
                const uint64_t odesc = desc_add(dOmn, os * L::TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < TILE / 16; ++kk) {
                    const uint64_t ad = desc_add(dPTd, (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32);
                    const uint64_t bd = desc_add(odesc, kk * 2048);
                    mma_ss(leader, tmem + KV_COL_DV, ad, bd, idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
                }
                if (leader) {
                    mma_commit(bar(BB::DV_DONE));
                    mma_commit(bar(BB::O_EMPTY + os));
                }
            };
            auto wait_all = [&](uint32_t b, uint32_t parity, int site) {
                return __all_sync(0xFFFFFFFFu, mbar_wait(b, parity, wc, site));
            };
            bool ok = wait_all(bar(BB::RES_FULL), 0, BSITE_RES) && wait_all(bar(BB::Q_FULL), 0, BSITE_X_FULL);
            if (ok) {
                tc_fence_after();
                mma_s(KV_COL_S, dKd, dQd);
                ok = wait_all(bar(BB::O_FULL), 0, BSITE_Y_FULL);
            }
            if (ok) {
                tc_fence_after();
                mma_s(KV_COL_DP, dVd, dOd);
                if (leader)
                    mma_commit(bar(BB::S_FULL));
            }
            for (int j = 0; ok && j < len; ++j) {
                const int jn = j + 1;
                if (jn < len) {
                    // S^T_{j+1} over S^T_j, which the gradient warps have loaded
                    if (!(ok = wait_all(bar(BB::Q_FULL + jn % L::QS), (jn / L::QS) & 1, BSITE_X_FULL)) ||
                        !(ok = wait_all(bar(BB::S_FREE), j & 1, BSITE_S_FULL)))
                        break;
                    tc_fence_after();
                    mma_s(KV_COL_S, dKd, desc_add(dQd, (jn % L::QS) * L::TILE_BYTES));
                }
                if (!(ok = wait_all(bar(BB::DS_HALF), j & 1, BSITE_DS_FULL)))
                    break;
                tc_fence_after();
                issue_dk(j, 0);
                if (!(ok = wait_all(bar(BB::DS_FULL), j & 1, BSITE_DS_FULL)))
                    break;
                tc_fence_after();
                issue_dk(j, 1);
                if (jn < len) {
                    // dP^T_{j+1} over the dS^T_j that dK_j reads, ordered after
                    // dK_j by MMA -> shift -> MMA (MMAs into different
                    // accumulators are not ordered), and ahead of dV_j, so that
                    // the next step's gradient warps start sooner
                    if (!(ok = wait_all(bar(BB::O_FULL + jn % L::OS), (jn / L::OS) & 1, BSITE_Y_FULL)))
                        break;
                    tc_fence_after();
                    if (leader)
                        tmem_shift_down(tmem + KV_COL_DP);
                    mma_s(KV_COL_DP, dVd, desc_add(dOd, (jn % L::OS) * L::TILE_BYTES));
                    if (leader)
                        mma_commit(bar(BB::S_FULL));
                }
                issue_dv(j);
            }
            if (leader)
                mma_commit(bar(BB::FINAL));
            drain_wait(bar(BB::FINAL), 0, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------ gradient warps
        const int wg = warp >> 2;            // warpgroup: query columns 64 wg .. 64 wg + 63 of each step
        const int t = threadIdx.x & 127;     // == TMEM lane: key row of the tile
        const int row = kb * TILE + t;
        const bool row_valid = row < n;
        const int rf = row_valid ? row / p.g.s : 0, rp = row_valid ? row % p.g.s : 0;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const uint32_t my_col = 64u * static_cast<uint32_t>(wg);
        const uint32_t wg_bar = 1u + static_cast<uint32_t>(wg);
        // this thread's row of P^T (K-major, 128-byte swizzle): chunk wg holds its 64 queries
        uint8_t* pt_row = smem + L::PT_OFF + wg * L::CHUNK_BYTES + t * 128;
        bool ok = true;
        // Statistic of one query column of the step's (this warpgroup's 64),
        // negated: threads 0-63 -L log2 e (-inf beyond n, so P is exactly 0
        // there), threads 64-127 -D.  Loaded one step ahead of its use, with the
        // CSR entry.
        auto column_stat = [&](int qblock) -> float {
            if (!in_bounds(wc, qblock >= 0 && qblock < p.nb, BSITE_B_TILE))  // (debug build)
                return -INFINITY;
            const int q = qblock * TILE + static_cast<int>(my_col) + (t & 63);
            if (q >= n)
                return t < 64 ? -INFINITY : -0.f;
            if (t >= 64)
                return -p.Dv[static_cast<size_t>(bh) * n + q];
            // a query row with no kept key (lse = -inf) has P = 0 everywhere
            const float l = p.lse[static_cast<size_t>(bh) * n + q];
            return l > -INFINITY ? -(l * LOG2E) : -INFINITY;
        };
        const uint64_t c2 = f2pack(p.scale_log2, p.scale_log2);
        int next_qb = len > 0 ? p.idx[start + walk(0)] : 0;
        int next_flag = len > 0 ? p.flag[start + walk(0)] : 0;
        float next_stat = len > 0 ? column_stat(next_qb) : 0.f;
        for (int j = 0; j < len; ++j) {
            const int qb = next_qb;
            const bool masked = p.mode == RA_MODE_TOKEN_EXACT && next_flag != RA_TILE_FULL;
            const float stat = next_stat;
            if (j + 1 < len) {
                next_qb = p.idx[start + walk(j + 1)];
                next_flag = p.flag[start + walk(j + 1)];
                next_stat = column_stat(next_qb);
            }
            // keep bits of this warpgroup's two 32-column chunks
            uint32_t mk[2] = {~0u, ~0u};
            if (masked && row_valid) {
                uint32_t m4[4];
                col_keep_mask(p.g, rf, rp, qb * TILE, m4[0], m4[1], m4[2], m4[3]);
                mk[0] = wg ? m4[2] : m4[0];
                mk[1] = wg ? m4[3] : m4[1];
            }
            sync_wg(wg_bar);  // the previous step's readers of the statistics are done
            (t < 64 ? st_l2 : st_d)[my_col + (t & 63)] = stat;
            ok = ok && mbar_wait(bar(BB::S_FULL), j & 1, wc, BSITE_S_FULL);
            // one decision per warpgroup; also publishes its staged statistics
            ok = sync_and_wg(wg_bar, ok);
            if (!ok)
                break;
            tc_fence_after();
            // S^T first, then release it for S^T_{j+1}; dP^T stays until dK_j has
            // read the dS^T packed over it
            uint32_t sv[2][32], dv[2][32];
            tmem_ld32(lane_base + KV_COL_S + my_col, sv[0]);
            tmem_ld32(lane_base + KV_COL_S + my_col + 32, sv[1]);
            tmem_ld32(lane_base + KV_COL_DP + my_col, dv[0]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(BB::S_FREE));
            tmem_ld32(lane_base + KV_COL_DP + my_col + 32, dv[1]);  // lands while chunk 0 is processed
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (c == 1)
                    tmem_wait_ld();
                const float4* l2v = reinterpret_cast<const float4*>(st_l2 + my_col + c * 32);
                const float4* dsv = reinterpret_cast<const float4*>(st_d + my_col + c * 32);
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e4 = 0; e4 < 32; e4 += 4) {
                    const float4 l4 = l2v[e4 >> 2], d4 = dsv[e4 >> 2];  // same address in every lane
                    float pe[4], ds[4];
                    grad_pair_keep(sv[c][e4], sv[c][e4 + 1], dv[c][e4], dv[c][e4 + 1], c2, f2pack(l4.x, l4.y),
                                   f2pack(d4.x, d4.y), (mk[c] >> e4) & 1u, (mk[c] >> (e4 + 1)) & 1u, pe[0], pe[1],
                                   ds[0], ds[1]);
                    grad_pair_keep(sv[c][e4 + 2], sv[c][e4 + 3], dv[c][e4 + 2], dv[c][e4 + 3], c2,
                                   f2pack(l4.z, l4.w), f2pack(d4.z, d4.w), (mk[c] >> (e4 + 2)) & 1u,
                                   (mk[c] >> (e4 + 3)) & 1u, pe[2], pe[3], ds[2], ds[3]);
                    pk[e4 >> 1] = pack_bf16(pe[0], pe[1]);
                    pk[(e4 >> 1) + 1] = pack_bf16(pe[2], pe[3]);
                    dk[e4 >> 1] = pack_bf16(ds[0], ds[1]);
                    dk[(e4 >> 1) + 1] = pack_bf16(ds[2], ds[3]);
                }
                // dV_{j-1} reads P^T_{j-1}: wait for it before the first overwrite.
                // A failed wait is acted on at the next step's warpgroup barrier,
                // so that the four warps leave the loop together.
                if (c == 0 && j > 0)
                    ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(BB::DV_DONE), (j - 1) & 1, wc, BSITE_ACC)) && ok;
                // P^T: 16-byte units 4 c .. 4 c + 3 of the row, at unit ^ (row % 8)
#pragma unroll
                for (int uu = 0; uu < 4; ++uu) {
                    const int unit = 4 * c + uu;
                    *reinterpret_cast<uint4*>(pt_row + ((unit ^ (t & 7)) * 16)) =
                        make_uint4(pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
                }
                // dS^T packed over dP^T columns this warpgroup has already loaded
                tmem_st16(lane_base + KV_COL_DP + my_col + c * 16, dk);
                if (c == 0) {
                    // the first chunk's dS^T: its half of dK_j can start
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(BB::DS_HALF));
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();  // P^T is read by the tensor cores
            tc_fence_before();
            mbar_arrive(bar(BB::DS_FULL));
        }
        // ------------------------------------------------------------ epilogue
        // warpgroup 0 stores dK (times the softmax scale), warpgroup 1 dV
        if (len > 0 && ok)
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar(BB::FINAL), 0, wc, BSITE_FINAL));
        tc_fence_after();
        if (__all_sync(0xFFFFFFFFu, ok && !*abort_flag)) {
            __nv_bfloat16* dst_row = (wg ? p.out1 : p.out0) + (static_cast<size_t>(bh) * n + row) * D;
            const float mul = wg ? 1.f : p.scale;
            const uint32_t col0 = wg ? KV_COL_DV : KV_COL_DK;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (len > 0) {
                    tmem_ld32(lane_base + col0 + c * 32, o);
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
                    w[e >> 1] = pack_bf16(__uint_as_float(o[e]) * mul, __uint_as_float(o[e + 1]) * mul);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = v[u];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == KV_MMA_WARP) {
        __syncwarp();
        tmem_dealloc(tmem, BWD_TMEM_COLS);
    }
}

// D[r] = <dO[r], O[r]> over d, one warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_dot_kernel(const __nv_bfloat16* __restrict__ O,
                                                      const __nv_bfloat16* __restrict__ dO, float* __restrict__ Dv,
                                                      long long rows)
{
    const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long r = warp_id; r < rows; r += nwarps) {
        float acc = 0.f;
#pragma unroll
        for (int k = lane * 2; k < D; k += 64) {
            const __nv_bfloat162 o = *reinterpret_cast<const __nv_bfloat162*>(O + r * D + k);
            const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(dO + r * D + k);
            acc = fmaf(__low2float(o), __low2float(g), acc);
            acc = fmaf(__high2float(o), __high2float(g), acc);
        }
        for (int off = 16; off > 0; off >>= 1)
            acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
        if (lane == 0)
            Dv[r] = acc;
    }
}

template <int D>
ra_status launch_dkdv(const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& q, const CUtensorMap& dO,
                      const BwdParams& p, int B, cudaStream_t cs)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        KvLayout<D>::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err, "cudaFuncSetAttribute(bwd_dkdv_kernel)");
    dim3 grid(p.nb, p.H, B);
    bwd_dkdv_kernel<D><<<grid, KV_THREADS, KvLayout<D>::SMEM_BYTES, cs>>>(k, v, q, dO, p);
    return cuda_fail(cudaGetLastError(), "bwd_dkdv_kernel launch");
}

template <int D>
ra_status launch_dq(const CUtensorMap& q, const CUtensorMap& dO, const CUtensorMap& k, const CUtensorMap& v,
                    const BwdParams& p, int B, cudaStream_t cs)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        DqLayout<D>::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return cuda_fail(attr_err, "cudaFuncSetAttribute(bwd_dq_kernel)");
    dim3 grid(p.nb, p.H, B);
    bwd_dq_kernel<D><<<grid, DQ_THREADS, DqLayout<D>::SMEM_BYTES, cs>>>(q, dO, k, v, p);
    return cuda_fail(cudaGetLastError(), "bwd_dq_kernel launch");
}

template <int D>
ra_status run_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* lse,
                  void* dQ, void* dK, void* dV, float* Dws, int B, int H, const ra_mask* m, float scale, int mode,
                  cudaStream_t cs)
{
    const int BH = B * H, n = m->geom.n;
    const long long rows = static_cast<long long>(BH) * n;
    const int dot_blocks = static_cast<int>(std::min<long long>((rows + 7) / 8, 148LL * 16));
    bwd_dot_kernel<D><<<dot_blocks, 256, 0, cs>>>(static_cast<const __nv_bfloat16*>(O),
                                                  static_cast<const __nv_bfloat16*>(dO), Dws, rows);
    ra_status st = cuda_fail(cudaGetLastError(), "bwd_dot_kernel launch");
    if (st != RA_OK)
        return st;
    CUtensorMap rq, rk, rv, rdo;  // 128-row boxes
    if ((st = make_map(&rq, Q, BH, n, D, TILE)) != RA_OK || (st = make_map(&rdo, dO, BH, n, D, TILE)) != RA_OK ||
        (st = make_map(&rk, K, BH, n, D, TILE)) != RA_OK || (st = make_map(&rv, V, BH, n, D, TILE)) != RA_OK)
        return st;
    BwdParams p;
    std::memset(&p, 0, sizeof p);
    p.g = m->geom;
    p.nb = m->nb;
    p.H = H;
    p.mode = mode;
    p.nnz = static_cast<int>(m->nnz);
    // Query tiles (dQ pass) and key tiles (dK / dV pass) in the mask's dispatch
    // order: by in-frame position band, then frame, so that the CTAs resident
    // together walk overlapping tiles (eq. 4 is symmetric in query and key).
    p.order = m->qorder;
    p.lse = lse;
    p.Dv = Dws;
    p.scale = scale;
    p.scale_log2 = scale * LOG2E;
    p.timeout_ns = wait_timeout_ns();
    if ((st = device_error_word(&p.err)) != RA_OK)
        return st;
    // dQ: query tiles over the block-CSR rows; resident Q, dO; rings of whole K, V tiles
    p.ptr = m->row_ptr;
    p.idx = m->col_idx;
    p.flag = m->flag;
    p.walk = m->walk;
    p.out0 = static_cast<__nv_bfloat16*>(dQ);
    p.out1 = nullptr;
    if ((st = launch_dq<D>(rq, rdo, rk, rv, p, B, cs)) != RA_OK)
        return st;
    // dK, dV: key tiles over the transposed block-CSR; resident K, V; rings of whole Q, dO tiles
    p.ptr = m->col_ptr;
    p.idx = m->row_idx;
    p.flag = m->tflag;
    p.walk = m->walk_t;
    p.out0 = static_cast<__nv_bfloat16*>(dK);
    p.out1 = static_cast<__nv_bfloat16*>(dV);
    return launch_dkdv<D>(rk, rv, rq, rdo, p, B, cs);
}

}  // namespace
}  // namespace ra

using namespace ra;

extern "C" ra_status ra_attention_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                      const float* lse, void* dQ, void* dK, void* dV, float* D_workspace, int B,
                                      int H, int d, const ra_mask* m, float scale, int mode, ra_stream stream)
{
    const void* ptrs[8] = {Q, K, V, O, dO, dQ, dK, dV};
    for (int i = 0; i < 8; ++i) {
        if (!ptrs[i])
            return fail(RA_ERR_INVALID_ARG, "NULL tensor pointer");
        if (!aligned16(ptrs[i]))
            return fail(RA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    }
    if (!lse || !D_workspace)
        return fail(RA_ERR_INVALID_ARG, "NULL lse or workspace");
    {
        const void* all[10] = {Q, K, V, O, dO, lse, dQ, dK, dV, D_workspace};
        for (int i = 6; i < 10; ++i)
            for (int j = 0; j < 10; ++j)
                if (j != i && all[i] == all[j])
                    return fail(RA_ERR_INVALID_ARG, "outputs (dQ, dK, dV, D_workspace) may not alias another buffer");
    }
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
    if (m->nnz == 0 || !m->col_ptr)
        return fail(RA_ERR_INVALID_ARG, "mask has no kept tile");
    // dQ is written before the dK / dV kernel reads Q and dO, and D before it is
    // read with lse: an output overlapping any other buffer would corrupt the
    // result silently, so every output range must be disjoint from the rest.
    const size_t tbytes = static_cast<size_t>(B) * H * m->geom.n * d * 2;
    const size_t sbytes = static_cast<size_t>(B) * H * m->geom.n * sizeof(float);
    const void* bufs[10] = {Q, K, V, O, dO, lse, dQ, dK, dV, D_workspace};
    const size_t sizes[10] = {tbytes, tbytes, tbytes, tbytes, tbytes, sbytes, tbytes, tbytes, tbytes, sbytes};
    auto overlap = [&](int i, int j) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(bufs[i]), b = reinterpret_cast<uintptr_t>(bufs[j]);
        return a < b + sizes[j] && b < a + sizes[i];
    };
    for (int i = 6; i < 10; ++i)
        for (int j = 0; j < 10; ++j)
            if (j != i && overlap(i, j))
                return fail(RA_ERR_INVALID_ARG, "outputs (dQ, dK, dV, D_workspace) may not overlap any other buffer");
    int dev = 0;
    RA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev != m->device)
        return fail(RA_ERR_INVALID_ARG, "mask was built on device %d, current device is %d", m->device, dev);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    return d == 64 ? run_bwd<64>(Q, K, V, O, dO, lse, dQ, dK, dV, D_workspace, B, H, m, scale, mode, cs)
                   : run_bwd<128>(Q, K, V, O, dO, lse, dQ, dK, dV, D_workspace, B, H, m, scale, mode, cs);
}
