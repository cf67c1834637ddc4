// ra_internal.h -- state and helpers shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "radattn.h"
#include "ra_mask_math.cuh"

// A built mask: geometry plus the device block-CSR (owned).
struct ra_mask {
    ra::MaskGeom geom;
    int nb;
    int device;
    long long nnz, full_tiles, kept_pairs, block_pairs;
    int row_min, row_max;
    int* row_ptr;          // [nb + 1]
    int* col_idx;          // [nnz]
    int* count;            // [nnz]
    unsigned char* flag;   // [nnz]
    // Transposed block-CSR (per key tile, the query tiles that keep it), for the
    // backward pass: col_ptr [nb + 1], row_idx [nnz] ascending, tflag [nnz].
    int* col_ptr;
    int* row_idx;
    unsigned char* tflag;
    // Dispatch order of the attention kernels' tiles: CTA x of the forward and
    // of the dQ pass runs query tile qorder[x], CTA x of the dK / dV pass key
    // tile qorder[x]; null when it is the identity.
    int* qorder;
    // [2 nb]: the walk of each CSR row (near frames first) by the forward and
    // the dQ pass: row offsets a, b of the near segment; null when rows are
    // walked in order.  walk_t: the same for the transposed CSR (dK / dV pass).
    int* walk;
    int* walk_t;
};

namespace ra {

// Record a one-line detail for ra_last_error() and return `s`.
ra_status fail(ra_status s, const char* fmt, ...);

// Map a CUDA error to a status (RA_OK when e == cudaSuccess).
ra_status cuda_fail(cudaError_t e, const char* what);

// Limit of every bounded device wait, in ns.
unsigned long long wait_timeout_ns();

// TMA map of a [B*H, n, d] bf16 tensor as a 3D tensor (d, n, B*H), boxes of
// box_rows rows x 64 columns with 128-byte swizzle; rows beyond n read as zero.
ra_status make_map(CUtensorMap* map, const void* base, int BH, int n, int d, int box_rows);

// The same for the first `rows` rows of each head of a [B*H, head_rows, d]
// tensor (rows <= head_rows): rows beyond `rows` read as zero.
ra_status make_map_rows(CUtensorMap* map, const void* base, int BH, int rows, int head_rows, int d, int box_rows);

// Forward attention of nq query rows per head over the first nk key rows of
// each head of K and V ([B*H, k_head_rows, d]), walking a caller-supplied
// block-CSR over nbq query tiles whose key tiles are all treated as FULL
// (keys >= nk are masked).  Block mode, no family mask: for masks that keep
// every listed key, such as the window held by the SWC key/value cache.
ra_status attention_fwd_rect(const void* Q, const void* K, const void* V, void* O, int B, int H, int d, int nq,
                             int nk, int k_head_rows, const int* row_ptr, const int* col_idx,
                             const unsigned char* flag, int nbq, int nnz, float scale, float* lse,
                             cudaStream_t stream);

// Device address of the forward / backward kernels' error word on the current device.
ra_status device_error_word(int** out);

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace ra

#define RA_CUDA_TRY(expr)                                 \
    do {                                                  \
        cudaError_t ra_e_ = (expr);                       \
        if (ra_e_ != cudaSuccess)                         \
            return ra::cuda_fail(ra_e_, #expr);           \
    } while (0)
