/*
 * radattn_oracle.c -- plain CPU oracle for static-mask sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference arm of bench.py use it.  It shares no code, header,
 * table or constant generator with the CUDA library; it restates the method
 * from its published definition, slowly and in the most direct order.
 *
 * Sources followed (page title, then section / equation):
 *   [RA]  "Radial Attention: O(n log n) Sparse Attention with Energy Decay for
 *         Long Video Generation" (summary page):
 *           eq. 1  dense attention softmax(QK^T/sqrt(d))V
 *           eq. 2  sparse attention softmax((QK^T + M)/sqrt(d))V, M in {-inf,0}
 *           eq. 3  token index j*s + l (frame j, in-frame position l)
 *           eq. 4  the 4D radial mask M~[i,j,k,l]
 *           eq. 5-6 zero-count bound (checked by the tests, not here)
 *           sec. 6 "128x128 block-level sparsity granularity"
 *   [TR]  "Token Radius Attention" tutorial with code, sec. 3.1 (tokens are
 *         (t h w) flattened), sec. 3.2 / 4.2 / 5 (cube neighbourhood of
 *         temporal radius r_t and spatial radius r_s)
 *   [VR]  "Vera 1.1" temporal module, sec. 2.1-2.2 (causal AND sliding window:
 *         query frame i sees key frames [max(0, i-W+1), i])
 *
 * Readings taken where the pages are silent or ambiguous:
 *   - floor(log2(x)) is evaluated exactly as (bit length of x) - 1.
 *   - |k-l| is the distance of in-frame flattened positions (eq. 3, eq. 4).
 *   - the condition |k-l|+1 <= s / 2^b is a real-number comparison, tested
 *     exactly as (|k-l|+1) * 2^b <= s.
 *   - a 128x128 tile is kept iff at least one valid (query, key) pair in it is
 *     kept; FULL iff all 128*128 pairs are valid and kept; otherwise PARTIAL.
 *   - the 3D window excludes out-of-grid neighbours (no zero padding) and uses
 *     softmax over the neighbour set, as the tutorial's own note asks.
 *   - the sliding window keeps key frames with 0 <= i - j <= W - 1 (the prose
 *     interval; the printed pseudocode has an off-by-one and a typo).
 *   - a query row with no kept key outputs 0 with log-sum-exp -inf.
 *
 * All floating point is fp64; bf16 inputs are widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* mask families and modes: same numeric values as the library's public enums,
 * restated here so the two sides share no header. */
#define OR_DENSE 0
#define OR_RADIAL 1
#define OR_WINDOW3D 2
#define OR_SWC 3

#define OR_TOKEN_EXACT 0
#define OR_BLOCK 1

#define OR_TILE_PARTIAL 0
#define OR_TILE_FULL 1

#define OR_TILE 128 /* [RA] sec. 6: 128x128 block granularity */

#define OR_IN_BF16 0
#define OR_IN_F32 1
#define OR_IN_F64 2

typedef struct {
    int family;
    int f;             /* frames */
    int s;             /* tokens per frame */
    int grid_h;        /* 3D window: s == grid_h * grid_w */
    int grid_w;
    int r_t;           /* 3D window: temporal radius */
    int r_s;           /* 3D window: spatial radius */
    int window_frames; /* sliding window: W */
    int sink_tokens;   /* global tokens: the first sink_tokens tokens */
} or_spec;

/* Threads the parallel loops below use. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the oracle's OpenMP loops use from now on (n >= 1). */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

static long long or_abs(long long x) { return x < 0 ? -x : x; }

/* floor(log2(x)) for x >= 1: position of the highest set bit. */
static int or_floor_log2(long long x)
{
    int b = -1;
    while (x > 0) {
        x >>= 1;
        b++;
    }
    return b;
}

/* [RA] eq. 4 for query (frame i, position k) and key (frame j, position l). */
static int or_radial_kept(long long i, long long j, long long k, long long l, long long s)
{
    long long dist = or_abs(i - j);
    long long w = 1LL << or_floor_log2(dist > 1 ? dist : 1); /* 2^floor(log2(max(|i-j|,1))) */
    /* first case: w <= s and |k-l| + 1 <= s / w */
    if (w <= s && (or_abs(k - l) + 1) * w <= s)
        return 1;
    /* second case: |i-j| mod ceil(w / s) == 0 and k == l */
    long long period = (w + s - 1) / s;
    if (dist % period == 0 && k == l)
        return 1;
    return 0;
}

/* [TR] sec. 3.2 / 4.2: the (2 r_t + 1) x (2 r_s + 1)^2 cube around the query. */
static int or_window3d_kept(const or_spec* sp, long long q, long long key)
{
    long long s = sp->s, gw = sp->grid_w;
    long long tq = q / s, pq = q % s, tk = key / s, pk = key % s;
    long long hq = pq / gw, wq = pq % gw, hk = pk / gw, wk = pk % gw;
    return or_abs(tq - tk) <= sp->r_t && or_abs(hq - hk) <= sp->r_s && or_abs(wq - wk) <= sp->r_s;
}

/* [VR] sec. 2.2: causal and at most W frames back, own frame included. */
static int or_swc_kept(const or_spec* sp, long long q, long long key)
{
    long long i = q / sp->s, j = key / sp->s;
    return (i - j) >= 0 && (i - j) <= (long long)sp->window_frames - 1;
}

/* M[q, key] == 0 ?  (token index = frame * s + position, [RA] eq. 3)
 * Global (sink) tokens -- the "sink" of the [RA] sec. 4 bound, the global
 * tokens of [TR] sec. 6.1 -- are kept in every row and every column. */
int oracle_kept(const or_spec* sp, long long q, long long key)
{
    long long s = sp->s;
    if (q < sp->sink_tokens || key < sp->sink_tokens)
        return 1;
    switch (sp->family) {
    case OR_DENSE:
        return 1;
    case OR_RADIAL:
        return or_radial_kept(q / s, key / s, q % s, key % s, s);
    case OR_WINDOW3D:
        return or_window3d_kept(sp, q, key);
    case OR_SWC:
        return or_swc_kept(sp, q, key);
    }
    return 0;
}

/* Whole token mask (n x n bytes, row = query).  Small n only. */
void oracle_dense_mask(const or_spec* sp, unsigned char* out)
{
    long long n = (long long)sp->f * sp->s;
    for (long long q = 0; q < n; q++)
        for (long long key = 0; key < n; key++)
            out[q * n + key] = (unsigned char)oracle_kept(sp, q, key);
}

/* Number of kept pairs in the whole mask, by enumeration. */
long long oracle_kept_total(const or_spec* sp)
{
    long long n = (long long)sp->f * sp->s, total = 0;
#pragma omp parallel for reduction(+ : total) schedule(dynamic, 16)
    for (long long q = 0; q < n; q++)
        for (long long key = 0; key < n; key++)
            total += oracle_kept(sp, q, key);
    return total;
}

/* Kept-pair count of every tile (qb, kb) for the listed query tiles, by
 * enumeration of every pair: out[r * nb + kb] for qbs[r]. */
void oracle_tile_counts(const or_spec* sp, const int* qbs, int nq, int* out)
{
    long long n = (long long)sp->f * sp->s;
    long long nb = (n + OR_TILE - 1) / OR_TILE;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nq; r++) {
        int* row = out + (long long)r * nb;
        for (long long kb = 0; kb < nb; kb++)
            row[kb] = 0;
        for (long long q = (long long)qbs[r] * OR_TILE; q < (long long)(qbs[r] + 1) * OR_TILE && q < n; q++)
            for (long long key = 0; key < n; key++)
                if (oracle_kept(sp, q, key))
                    row[key / OR_TILE] += 1;
    }
}

/* Block-CSR from a full nb x nb count matrix: kept tiles of each row in
 * ascending column order.  Returns nnz.  Pass null arrays to only count. */
long long oracle_csr(const int* counts, long long n, int* row_ptr, int* col_idx, int* count,
                     unsigned char* flag)
{
    long long nb = (n + OR_TILE - 1) / OR_TILE, nnz = 0;
    for (long long qb = 0; qb < nb; qb++) {
        if (row_ptr)
            row_ptr[qb] = (int)nnz;
        for (long long kb = 0; kb < nb; kb++) {
            int c = counts[qb * nb + kb];
            if (c > 0) {
                if (col_idx) {
                    col_idx[nnz] = (int)kb;
                    count[nnz] = c;
                    flag[nnz] = (c == OR_TILE * OR_TILE) ? OR_TILE_FULL : OR_TILE_PARTIAL;
                }
                nnz++;
            }
        }
    }
    if (row_ptr)
        row_ptr[nb] = (int)nnz;
    return nnz;
}

static double or_load(const void* base, int dtype, long long idx)
{
    if (dtype == OR_IN_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16; /* bf16 is the top half of f32 */
        float v;
        memcpy(&v, &bits, sizeof v);
        return (double)v;
    }
    if (dtype == OR_IN_F32)
        return (double)((const float*)base)[idx];
    return ((const double*)base)[idx];
}

/*
 * Attention for a list of query rows ([RA] eq. 2 with M in {0,-inf}):
 *   keys  = { key : M[q,key] == 0 }                    (token-exact mode)
 *         = { key < n : tile (q/128, key/128) kept }  (block mode: kept tiles in full)
 *   x     = scale * <Q[q], K[key]>,  p = exp(x - max x) / sum exp(x - max x)
 *   O[q]  = sum p * V[key],  lse = log sum exp(x)
 * Q, K, V are [B, H, n, d] row-major; row r is (row_bh[r] = b*H + h, row_q[r]).
 * In block mode tile_flags[t * nb + kb] != 0 says tile (row_tile[r], kb) is
 * kept, where t = row_tile_slot[r] indexes the caller's list of query tiles.
 */
void oracle_attention_rows(const void* Q, const void* K, const void* V, int dtype, long long n, int d,
                           const or_spec* sp, int mode, double scale, long long nrows,
                           const long long* row_bh, const long long* row_q,
                           const unsigned char* tile_flags, const int* row_tile_slot, double* O,
                           double* lse, long long* nkeys)
{
    long long nb = (n + OR_TILE - 1) / OR_TILE;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)n);
        long long* idx = (long long*)malloc(sizeof(long long) * (size_t)n);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < nrows; r++) {
            long long q = row_q[r];
            long long qoff = (row_bh[r] * n + q) * d;
            long long kvbase = row_bh[r] * n * d;
            long long m = 0;
            for (long long key = 0; key < n; key++) {
                int use;
                if (mode == OR_TOKEN_EXACT)
                    use = oracle_kept(sp, q, key);
                else
                    use = tile_flags[(long long)row_tile_slot[r] * nb + key / OR_TILE] != 0;
                if (!use)
                    continue;
                double dot = 0.0;
                for (int c = 0; c < d; c++)
                    dot += or_load(Q, dtype, qoff + c) * or_load(K, dtype, kvbase + key * d + c);
                x[m] = scale * dot;
                idx[m] = key;
                m++;
            }
            nkeys[r] = m;
            if (m == 0) {
                for (int c = 0; c < d; c++)
                    O[r * d + c] = 0.0;
                lse[r] = -INFINITY;
                continue;
            }
            double mx = x[0];
            for (long long t = 1; t < m; t++)
                if (x[t] > mx)
                    mx = x[t];
            double denom = 0.0;
            for (int c = 0; c < d; c++)
                acc[c] = 0.0;
            for (long long t = 0; t < m; t++) {
                double w = exp(x[t] - mx);
                denom += w;
                for (int c = 0; c < d; c++)
                    acc[c] += w * or_load(V, dtype, kvbase + idx[t] * d + c);
            }
            for (int c = 0; c < d; c++)
                O[r * d + c] = acc[c] / denom;
            lse[r] = mx + log(denom);
        }
        free(x);
        free(idx);
        free(acc);
    }
}

/*
 * Gradients of the masked softmax attention ([RA] eq. 2) for one (batch, head)
 * slice, by the chain rule written out in its plainest order:
 *   x_ij  = scale <Q_i, K_j>,  P_ij = exp(x_ij - lse_i) over the row's keys
 *   O_i   = sum_j P_ij V_j,    D_i  = <dO_i, O_i>
 *   dP_ij = <dO_i, V_j>,       dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij K_j
 *   dK_j  = scale sum_i dS_ij Q_i
 *   dV_j  = sum_i P_ij dO_i
 * Keys of row i as in oracle_attention_rows (token-exact: kept pairs; block:
 * every valid key of a kept tile, from tile_flags[qb * nb + kb]).
 * Q, K, V, dO: [n, d] (dtype as in oracle_attention_rows); dQ, dK, dV: [n, d]
 * fp64, overwritten.  O(n^2 d): small n only.
 */
void oracle_attention_bwd(const void* Q, const void* K, const void* V, const void* dO, int dtype, long long n,
                          int d, const or_spec* sp, int mode, double scale, const unsigned char* tile_flags,
                          double* dQ, double* dK, double* dV)
{
    long long nb = (n + OR_TILE - 1) / OR_TILE;
    double* x = (double*)malloc(sizeof(double) * (size_t)n);
    unsigned char* use = (unsigned char*)malloc((size_t)n);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    for (long long t = 0; t < n * d; t++)
        dQ[t] = dK[t] = dV[t] = 0.0;
    for (long long i = 0; i < n; i++) {
        double mx = -INFINITY;
        for (long long j = 0; j < n; j++) {
            if (mode == OR_TOKEN_EXACT)
                use[j] = (unsigned char)oracle_kept(sp, i, j);
            else
                use[j] = tile_flags[(i / OR_TILE) * nb + j / OR_TILE] != 0;
            if (!use[j])
                continue;
            double dot = 0.0;
            for (int c = 0; c < d; c++)
                dot += or_load(Q, dtype, i * d + c) * or_load(K, dtype, j * d + c);
            x[j] = scale * dot;
            if (x[j] > mx)
                mx = x[j];
        }
        if (mx == -INFINITY)
            continue; /* a row with no key: no gradient */
        double denom = 0.0;
        for (long long j = 0; j < n; j++)
            if (use[j])
                denom += exp(x[j] - mx);
        double lse = mx + log(denom);
        /* O_i and D_i */
        for (int c = 0; c < d; c++)
            o[c] = 0.0;
        for (long long j = 0; j < n; j++)
            if (use[j]) {
                double pij = exp(x[j] - lse);
                for (int c = 0; c < d; c++)
                    o[c] += pij * or_load(V, dtype, j * d + c);
            }
        double Di = 0.0;
        for (int c = 0; c < d; c++)
            Di += or_load(dO, dtype, i * d + c) * o[c];
        for (long long j = 0; j < n; j++) {
            if (!use[j])
                continue;
            double pij = exp(x[j] - lse);
            double dpij = 0.0;
            for (int c = 0; c < d; c++)
                dpij += or_load(dO, dtype, i * d + c) * or_load(V, dtype, j * d + c);
            double dsij = pij * (dpij - Di);
            for (int c = 0; c < d; c++) {
                dQ[i * d + c] += scale * dsij * or_load(K, dtype, j * d + c);
                dK[j * d + c] += scale * dsij * or_load(Q, dtype, i * d + c);
                dV[j * d + c] += pij * or_load(dO, dtype, i * d + c);
            }
        }
    }
    free(x);
    free(use);
    free(o);
}

/* Keys of query q (token-exact: M[q, key] == 0; block: every key of a kept
 * tile, flags[key / 128] != 0 with flags the query tile's row of tile flags),
 * their scores x = scale <Q_q, K_key> and the row's log-sum-exp.  Returns the
 * number of keys; idx / x receive them. */
static long long or_row_scores(const void* Q, const void* K, int dtype, long long n, int d, const or_spec* sp,
                               int mode, double scale, long long q, const unsigned char* flags,
                               long long qoff, long long kvbase, long long* idx, double* x, double* lse)
{
    long long m = 0;
    for (long long key = 0; key < n; key++) {
        int use = mode == OR_TOKEN_EXACT ? oracle_kept(sp, q, key) : flags[key / OR_TILE] != 0;
        if (!use)
            continue;
        long long koff = kvbase + key * d;
        double dot = 0.0;
        for (int c = 0; c < d; c++)
            dot += or_load(Q, dtype, qoff + c) * or_load(K, dtype, koff + c);
        x[m] = dot * scale;
        idx[m] = key;
        m++;
    }
    if (m == 0) {
        *lse = -INFINITY;
        return 0;
    }
    double mx = x[0];
    for (long long t = 1; t < m; t++)
        if (x[t] > mx)
            mx = x[t];
    double denom = 0.0;
    for (long long t = 0; t < m; t++)
        denom += exp(x[t] - mx);
    *lse = mx + log(denom);
    return m;
}

/*
 * dQ of listed query rows, from the same definitions as oracle_attention_bwd
 * (dQ_i = scale sum_j P_ij (<dO_i, V_j> - D_i) K_j, D_i = <dO_i, O_i>), one row
 * at a time in O(keys * d): for sampled rows of workloads too large for the
 * whole backward.  Rows and tile flags as in oracle_attention_rows; dQ is
 * [nrows, d] fp64; nkeys (may be NULL) receives each row's key count.
 */
void oracle_attention_bwd_query_rows(const void* Q, const void* K, const void* V, const void* dO, int dtype,
                                     long long n, int d, const or_spec* sp, int mode, double scale, long long nrows,
                                     const long long* row_bh, const long long* row_q,
                                     const unsigned char* tile_flags, const int* row_tile_slot, double* dQ,
                                     long long* nkeys)
{
    long long nb = (n + OR_TILE - 1) / OR_TILE;
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)n);
        long long* idx = (long long*)malloc(sizeof(long long) * (size_t)n);
        double* o = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < nrows; r++) {
            long long q = row_q[r];
            long long qoff = (row_bh[r] * n + q) * d;
            long long kvbase = row_bh[r] * n * d;
            const unsigned char* flags = mode == OR_TOKEN_EXACT ? NULL : tile_flags + (long long)row_tile_slot[r] * nb;
            double lse;
            long long m = or_row_scores(Q, K, dtype, n, d, sp, mode, scale, q, flags, qoff, kvbase, idx, x, &lse);
            if (nkeys)
                nkeys[r] = m;
            for (int c = 0; c < d; c++)
                dQ[r * d + c] = 0.0;
            if (m == 0)
                continue;
            for (int c = 0; c < d; c++)
                o[c] = 0.0;
            for (long long t = 0; t < m; t++) {
                long long koff = kvbase + idx[t] * d;
                double p = exp(x[t] - lse);
                for (int c = 0; c < d; c++)
                    o[c] += p * or_load(V, dtype, koff + c);
            }
            double D = 0.0;
            for (int c = 0; c < d; c++)
                D += or_load(dO, dtype, qoff + c) * o[c];
            for (long long t = 0; t < m; t++) {
                long long koff = kvbase + idx[t] * d;
                double p = exp(x[t] - lse), dp = 0.0;
                for (int c = 0; c < d; c++)
                    dp += or_load(dO, dtype, qoff + c) * or_load(V, dtype, koff + c);
                double ds = p * (dp - D);
                for (int c = 0; c < d; c++)
                    dQ[r * d + c] += scale * ds * or_load(K, dtype, koff + c);
            }
        }
        free(x);
        free(idx);
        free(o);
    }
}

/*
 * dK and dV of listed key rows of one (batch, head) slice (Q, K, V, dO: [n, d]):
 * first lse_i and D_i of every query row that keeps at least one listed key,
 * then for each listed key j
 *   dK_j = scale sum_i P_ij (<dO_i, V_j> - D_i) Q_i,   dV_j = sum_i P_ij dO_i
 * over the queries i whose row keeps j.  O(n * keys * d) for the statistics,
 * O(n * d) per listed key.  tile_flags: the whole nb x nb table (block mode).
 * dK, dV: [nkeys, d] fp64.
 */
void oracle_attention_bwd_key_rows(const void* Q, const void* K, const void* V, const void* dO, int dtype,
                                   long long n, int d, const or_spec* sp, int mode, double scale,
                                   const unsigned char* tile_flags, long long nkeys, const long long* key_idx,
                                   double* dK, double* dV)
{
    long long nb = (n + OR_TILE - 1) / OR_TILE;
    double* lse = (double*)malloc(sizeof(double) * (size_t)n);
    double* Dv = (double*)malloc(sizeof(double) * (size_t)n);
#pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)n);
        long long* idx = (long long*)malloc(sizeof(long long) * (size_t)n);
        double* o = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
        for (long long i = 0; i < n; i++) {
            int needed = 0;
            for (long long r = 0; r < nkeys && !needed; r++)
                needed = mode == OR_TOKEN_EXACT ? oracle_kept(sp, i, key_idx[r])
                                                : tile_flags[(i / OR_TILE) * nb + key_idx[r] / OR_TILE] != 0;
            if (!needed)
                continue; /* row i keeps none of the listed keys: its statistics are not used */
            const unsigned char* flags = mode == OR_TOKEN_EXACT ? NULL : tile_flags + (i / OR_TILE) * nb;
            long long m = or_row_scores(Q, K, dtype, n, d, sp, mode, scale, i, flags, i * d, 0, idx, x, &lse[i]);
            for (int c = 0; c < d; c++)
                o[c] = 0.0;
            for (long long t = 0; t < m; t++) {
                double p = exp(x[t] - lse[i]);
                for (int c = 0; c < d; c++)
                    o[c] += p * or_load(V, dtype, idx[t] * d + c);
            }
            double D = 0.0;
            for (int c = 0; c < d; c++)
                D += or_load(dO, dtype, i * d + c) * o[c];
            Dv[i] = D;
        }
        free(x);
        free(idx);
        free(o);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (long long r = 0; r < nkeys; r++) {
        long long j = key_idx[r];
        for (int c = 0; c < d; c++)
            dK[r * d + c] = dV[r * d + c] = 0.0;
        for (long long i = 0; i < n; i++) {
            int use = mode == OR_TOKEN_EXACT ? oracle_kept(sp, i, j)
                                             : tile_flags[(i / OR_TILE) * nb + j / OR_TILE] != 0;
            if (!use)
                continue;
            double dot = 0.0, dp = 0.0;
            for (int c = 0; c < d; c++) {
                dot += or_load(Q, dtype, i * d + c) * or_load(K, dtype, j * d + c);
                dp += or_load(dO, dtype, i * d + c) * or_load(V, dtype, j * d + c);
            }
            double p = exp(scale * dot - lse[i]);
            double ds = p * (dp - Dv[i]);
            for (int c = 0; c < d; c++) {
                dK[r * d + c] += scale * ds * or_load(Q, dtype, i * d + c);
                dV[r * d + c] += p * or_load(dO, dtype, i * d + c);
            }
        }
    }
    free(lse);
    free(Dv);
}
