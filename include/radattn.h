/*
 * radattn.h -- C ABI of the B200 (sm_100a) static sparse attention library.
 *
 * The library computes, on one GPU, the sparse attention of
 * "Radial Attention: O(n log n) Sparse Attention with Energy Decay for Long
 * Video Generation", eq. 2:
 *
 *     O = softmax((Q K^T + M) / sqrt(d)) V,     M in {0, -inf}^{n x n},
 *
 * over a frame-major token sequence (token index = frame * s + position,
 * eq. 3), for a static mask M from one of four families:
 *
 *   RA_MASK_RADIAL    eq. 4 of the same page (spatio-temporal energy decay);
 *   RA_MASK_WINDOW3D  the cube neighbourhood of the "Token Radius Attention"
 *                     tutorial, sec. 3.2 / 4.2 (temporal radius r_t, spatial
 *                     radius r_s, position = h * grid_w + w);
 *   RA_MASK_SWC       the causal sliding window of the "Vera 1.1" temporal
 *                     module, sec. 2.2 (query frame i sees frames i-W+1 .. i);
 *   RA_MASK_DENSE     M = 0 (eq. 1, the dense reference point).
 *
 * The mask is applied at the 128 x 128 tile granularity of the Radial
 * Attention page, sec. 6: ra_build_mask lists the kept tiles of each 128-row
 * query tile as a block-CSR with per-tile kept counts and FULL / PARTIAL flags.
 * ra_attention_fwd then runs either token-exact (partial tiles apply the
 * element mask) or block-granular (every valid pair of a kept tile is used).
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device addresses on the current device; host
 *     pointers are ordinary (ideally pinned) host memory.  The caller owns every
 *     buffer it passes; the library owns a ra_mask until ra_mask_free.
 *   - Tensors are contiguous, row-major [B, H, n, d] bf16 (raw 16-bit), 16-byte
 *     aligned.  d is 64 or 128.
 *   - Errors are returned as ra_status, never thrown; ra_last_error() gives a
 *     one-line detail for the calling thread.  Work is enqueued on `stream`
 *     (NULL = the legacy default stream) and is asynchronous unless stated.
 *   - A kernel that gives up a bounded internal wait records
 *     RA_ERR_DEVICE_TIMEOUT in a per-device error word; ra_get_device_status
 *     reads (and clears) it.  Kernels never trap.  The word is sticky: while it
 *     is set, every later forward, backward or SWC-step kernel on that device
 *     does no work and leaves its outputs unwritten, although its entry point
 *     returned RA_OK when it was enqueued.  Check ra_get_device_status before
 *     trusting outputs produced after a possible timeout; it clears the word.
 *   - Results are deterministic: the same inputs give the same bits.
 */
#ifndef RADATTN_H
#define RADATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ra_stream; /* a cudaStream_t */

typedef enum {
    RA_MASK_DENSE = 0,
    RA_MASK_RADIAL = 1,
    RA_MASK_WINDOW3D = 2,
    RA_MASK_SWC = 3
} ra_family;

typedef enum {
    RA_MODE_TOKEN_EXACT = 0, /* partial tiles apply the element mask M */
    RA_MODE_BLOCK = 1        /* every valid pair of a kept tile is computed */
} ra_mode;

typedef enum { RA_TILE_PARTIAL = 0, RA_TILE_FULL = 1 } ra_tile_flag;

typedef enum {
    RA_OK = 0,
    RA_ERR_INVALID_ARG = 1,
    RA_ERR_UNSUPPORTED = 2,
    RA_ERR_CUDA = 3,
    RA_ERR_OUT_OF_MEMORY = 4,
    RA_ERR_DEVICE_TIMEOUT = 5,
    RA_ERR_DEVICE_BOUNDS = 6 /* debug build only: a kernel's bounds check failed */
} ra_status;

#define RA_TILE 128 /* tile edge, "Radial Attention" sec. 6 */

/* Family parameters; fields a family does not use are ignored. */
typedef struct {
    int grid_h, grid_w; /* WINDOW3D: s == grid_h * grid_w */
    int r_t, r_s;       /* WINDOW3D: temporal and spatial radius, >= 0 */
    int window_frames;  /* SWC: W >= 1 */
    int sink_tokens;    /* every family: the first sink_tokens tokens are global --
                           visible to every query and seeing every key ("centre band
                           + sink" of the Radial Attention bound, sec. 4; global
                           tokens of the tutorial, sec. 6.1).  0 (default) = none. */
} ra_mask_params;

typedef struct ra_mask ra_mask; /* opaque; owns its device arrays */

/* Summary of a built mask. */
typedef struct {
    int family, f, s;
    int nb;                  /* ceil(n / 128) */
    long long n;             /* f * s */
    long long nnz;           /* kept tiles */
    long long full_tiles;    /* tiles flagged RA_TILE_FULL */
    long long kept_pairs;    /* (query, key) pairs with M == 0 */
    long long block_pairs;   /* valid pairs inside kept tiles (what block mode computes) */
    int row_min, row_max;    /* fewest / most kept tiles in a query-tile row */
} ra_mask_info_t;

/*
 * ra_build_mask -- evaluate a mask family on the GPU and build its block-CSR.
 *   family, f, s, params : the mask (eq. 4 / the window cube / the sliding
 *                          window / dense) over n = f * s tokens.
 *   out                  : receives a new mask; free it with ra_mask_free.
 * Arrays (device, owned by the mask): row_ptr int32[nb + 1]; col_idx int32[nnz]
 * (ascending within a row); count int32[nnz] (kept pairs of the tile);
 * flag uint8[nnz] (RA_TILE_FULL iff count == 128 * 128).  A tile is kept iff it
 * holds at least one kept valid pair.  The mask also holds the transposed
 * block-CSR (for each key tile its query tiles: col_ptr, row_idx, tflag), which
 * ra_attention_bwd walks for dK and dV.
 * Synchronises `stream` once (to size the arrays).  Limits: f, s >= 1,
 * n <= 2^31 - 1 and nb * nb <= 2^31 - 1.  INVALID_ARG on bad parameters,
 * OUT_OF_MEMORY / CUDA on device failures (nothing is leaked).
 */
ra_status ra_build_mask(int family, int f, int s, const ra_mask_params* params, ra_stream stream,
                        ra_mask** out);

/*
 * ra_build_mask_noalloc -- ra_build_mask for callers that cannot allocate.
 * (No counterpart in the paper: this is a deployment variant of the builder.)
 *
 * Some callers must not have a library allocate device memory behind their
 * back: engines whose own allocator owns the whole device, processes that
 * reserve a fixed memory budget at start-up, and loops that cannot afford the
 * device-wide synchronisation an allocation may imply.  This entry point builds
 * the same block-CSR as ra_build_mask into arrays the caller supplies and calls
 * no allocating routine.  Its scratch (the tile counts and row statistics) is a
 * fixed array of 4 MiB + 4.25 KiB compiled into the library, which every device
 * that loads the library holds until the process exits.
 *   row_ptr               : device int32[nb + 1], written.
 *   col_idx, count, flag  : device int32 / int32 / uint8 arrays of nnz_capacity
 *                           entries, written with the kept tiles.
 *   info                  : optional host struct, filled even when the capacity
 *                           is too small (so the caller can size the arrays).
 * Limit: n <= 131072 tokens (nb <= 1024); larger masks get RA_ERR_UNSUPPORTED.
 * RA_ERR_INVALID_ARG if nnz exceeds nnz_capacity (nothing but row_ptr written).
 * Every call synchronises `stream` (to read nnz), so no call may be made while
 * `stream` is being captured into a CUDA graph.  Each call looks up the
 * scratch's device address in the current context (the first call on a device
 * may load the library's module there).  All calls share the one scratch
 * array, so calls that can overlap on the GPU (different streams, no ordering)
 * race; calls ordered on one stream are safe.
 */
ra_status ra_build_mask_noalloc(int family, int f, int s, const ra_mask_params* params, int* row_ptr, int* col_idx,
                                int* count, unsigned char* flag, long long nnz_capacity, ra_mask_info_t* info,
                                ra_stream stream);

/* Fill *info.  Host only, no synchronisation. */
ra_status ra_mask_info(const ra_mask* m, ra_mask_info_t* info);

/* Copy the block-CSR to caller-allocated host arrays (sizes from ra_mask_info).
 * Any pointer may be NULL to skip that array.  Synchronous. */
ra_status ra_mask_copy_to_host(const ra_mask* m, int* row_ptr, int* col_idx, int* count, unsigned char* flag);

/* Device addresses of the block-CSR arrays (read-only, valid until ra_mask_free). */
ra_status ra_mask_device_arrays(const ra_mask* m, const int** row_ptr, const int** col_idx, const int** count,
                                const unsigned char** flag);

/* Copy the transposed block-CSR (per key tile, the query tiles that keep it, in
 * ascending order, with the tile's FULL / PARTIAL flag) to caller-allocated host
 * arrays: col_ptr int32[nb + 1], row_idx int32[nnz], tflag uint8[nnz].  The
 * backward pass walks it.  Any pointer may be NULL.  Synchronous. */
ra_status ra_mask_copy_transpose_to_host(const ra_mask* m, int* col_ptr, int* row_idx, unsigned char* tflag);

/* Release a mask (NULL is ignored).  Synchronises the device first. */
void ra_mask_free(ra_mask* m);

/*
 * ra_attention_fwd -- O = softmax(scale * Q K^T + M) V on the kept tiles.
 *   Q, K, V : device, bf16 [B, H, n, d], contiguous, 16-byte aligned.
 *   O       : device, bf16 [B, H, n, d], written (may not alias Q, K or V).
 *   d       : 64 or 128 (else RA_ERR_UNSUPPORTED).
 *   m       : a mask built for n = f * s tokens (shared by every batch and head).
 *   scale   : softmax scale, normally 1 / sqrt(d) (eq. 1-2).
 *   mode    : RA_MODE_TOKEN_EXACT or RA_MODE_BLOCK.
 *   lse     : NULL, or device fp32 [B, H, n] receiving the natural-log
 *             log-sum-exp of each row's kept scores.
 * A row with no kept key (none exists in the four families) gets O = 0 and
 * lse = -inf.  Asynchronous on `stream`; no allocation.
 */
ra_status ra_attention_fwd(const void* Q, const void* K, const void* V, void* O, int B, int H, int d,
                           const ra_mask* m, float scale, int mode, float* lse, ra_stream stream);

/*
 * ra_attention_fwd_host -- the same call with inputs and output in host memory.
 *   Q_host, K_host, V_host : host bf16 [B, H, n, d] (pinned for asynchronous copies).
 *   O_host                 : host bf16 [B, H, n, d], written.
 *   Q_dev .. O_dev         : caller-owned device staging buffers of the same size.
 * Enqueues three host-to-device copies, the forward kernel and one
 * device-to-host copy on `stream`, then returns; synchronise `stream` before
 * reading O_host.
 */
ra_status ra_attention_fwd_host(const void* Q_host, const void* K_host, const void* V_host, void* O_host,
                                void* Q_dev, void* K_dev, void* V_dev, void* O_dev, int B, int H, int d,
                                const ra_mask* m, float scale, int mode, ra_stream stream);

/*
 * ra_attention_bwd -- gradients of ra_attention_fwd ("Radial Attention ..."
 * eq. 2 with the 128 x 128 tile mask of sec. 6).  The page trains its LoRA
 * adapters through the sparse attention (sec. 6: block-sparse FlashAttention-2
 * for training; sec. 7: training speedups) without writing the backward out;
 * these are the standard softmax-attention gradients restricted to the kept pairs.  With
 * P = exp(scale * Q K^T + M - lse), D_i = <dO_i, O_i>, dS = P * (dO V^T - D):
 *   dQ = scale * dS K,   dK = scale * dS^T Q,   dV = P^T dO.
 *   Q, K, V, O, dO : device, bf16 [B, H, n, d], contiguous, 16-byte aligned;
 *                    O is the forward's output for the same Q, K, V, m, mode.
 *   lse            : device fp32 [B, H, n], the forward's log-sum-exp.
 *   dQ, dK, dV     : device, bf16 [B, H, n, d], written.
 *   D_workspace    : device fp32 [B, H, n], caller-owned scratch (receives D).
 *                    None of dQ, dK, dV, D_workspace may overlap any other
 *                    buffer of the call (RA_ERR_INVALID_ARG).
 *   d, m, scale, mode : as for ra_attention_fwd (same values as the forward).
 * dQ walks the block-CSR rows, dK and dV the transposed block-CSR; no atomics,
 * so the result is deterministic.  Asynchronous on `stream`; no allocation.
 */
ra_status ra_attention_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                           const float* lse, void* dQ, void* dK, void* dV, float* D_workspace, int B, int H, int d,
                           const ra_mask* m, float scale, int mode, ra_stream stream);

/*
 * Streaming sliding-window causal attention with a key/value ring cache
 * (the Vera 1.1 temporal module, sec. 3.1: during inference the K and V of the
 * frames inside the window are cached; as the window moves on, the oldest
 * frame's K and V are evicted and the new frame's added, so memory stays fixed).
 *
 * ra_swc_cache_create -- a cache for B x H heads of d (64 or 128) channels,
 *   s tokens per frame and a window of W = window_frames frames.  Allocates two
 *   device rings of B * H * W * s * d bf16 (K and V) plus a few KB of tile lists;
 *   synchronous.  The cache is bound to the current device.
 * ra_swc_cache_step -- feed the next frame (index i = frames fed so far):
 *   Q_frame, K_frame, V_frame : device bf16 [B, H, s, d], contiguous, 16-byte aligned.
 *   O_frame                   : device bf16 [B, H, s, d], written.
 *   lse                       : NULL or device fp32 [B, H, s] (natural log).
 *   The frame's K and V replace frame i - W's in the ring; then O_frame is the
 *   attention of the frame's queries over every token of frames max(0, i-W+1) .. i,
 *   the rows of frame i of the SWC mask (RA_MASK_SWC, same W) over the whole
 *   sequence.  Asynchronous on `stream`; steps must be ordered (one stream).
 * ra_swc_cache_info  -- frames fed so far and frames held (min(fed, W)).  Host only.
 * ra_swc_cache_copy_rings_to_host -- copy the K and V rings, each
 *   [B, H, W * s, d] bf16 with frame i in slot i mod W, to host arrays (either
 *   may be NULL).  Synchronises the device.
 * ra_swc_cache_reset -- forget every frame (the next step is frame 0).  Host only.
 * ra_swc_cache_free  -- synchronise the device and release the cache (NULL ignored).
 */
typedef struct ra_swc_cache ra_swc_cache;
ra_status ra_swc_cache_create(int B, int H, int d, int s, int window_frames, ra_swc_cache** out);
ra_status ra_swc_cache_step(ra_swc_cache* c, const void* Q_frame, const void* K_frame, const void* V_frame,
                            void* O_frame, float scale, float* lse, ra_stream stream);
ra_status ra_swc_cache_info(const ra_swc_cache* c, long long* frames_seen, int* frames_held);
ra_status ra_swc_cache_copy_rings_to_host(const ra_swc_cache* c, void* K_host, void* V_host);
ra_status ra_swc_cache_reset(ra_swc_cache* c);
void ra_swc_cache_free(ra_swc_cache* c);

/* Synchronise `stream`, then read and clear the current device's error word.
 * RA_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since the last call. */
ra_status ra_get_device_status(ra_stream stream);

/* Site code and block index recorded with the last device error (0 if none). */
ra_status ra_get_device_error_site(int* site, int* block);

/* Bounded-wait self-test: launches one CTA whose mbarrier wait nothing ever
 * completes, with the given limit (1e6 .. 1e10 ns).  Returns the device status
 * it observed, RA_ERR_DEVICE_TIMEOUT when the bound works; the error word is
 * cleared afterwards.  Synchronous. */
ra_status ra_selftest_wait_timeout(long long timeout_ns, ra_stream stream);

/* Bounds-check self-test.  The library built with -DRA_DEBUG_BOUNDS
 * (libradattn_debug.so: every global index and TMA coordinate a kernel derives
 * from its inputs is checked before use, and a failure records
 * RA_ERR_DEVICE_BOUNDS with its site in the error word and skips the access,
 * without trapping) launches one CTA whose check fails on an index it never
 * uses, and returns the device status it observed: RA_ERR_DEVICE_BOUNDS when
 * the checks are compiled in; the error word is cleared afterwards.  The
 * release library returns RA_ERR_UNSUPPORTED.  Synchronous. */
ra_status ra_selftest_bounds(ra_stream stream);

/* Limit of every bounded wait in the library's kernels (default 4e9 ns). */
ra_status ra_set_wait_timeout_ns(long long timeout_ns);

/* Precision of P in the P V product (process-wide setting).
 *   RA_PV_AUTO   (default) bf16 P, except for masks whose rows average fewer
 *                than 4096 computed keys: there P is held as a hi + lo pair of
 *                bf16 numbers and P V runs as two MMAs, because over few keys the
 *                rounding of each weight to bf16 is not averaged out.
 *   RA_PV_BF16   always bf16 P (one MMA).
 *   RA_PV_SPLIT  always hi + lo P (two MMAs).
 * INVALID_ARG for any other value. */
typedef enum { RA_PV_AUTO = 0, RA_PV_BF16 = 1, RA_PV_SPLIT = 2 } ra_pv_precision;
ra_status ra_set_pv_precision(int policy);

const char* ra_status_string(ra_status s);

/* One-line description of the calling thread's last error ("" if none). */
const char* ra_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int ra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RADATTN_H */
