// ra_internal.h -- state and helpers shared by the library's translation units.
#pragma once
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
};

namespace ra {

// Record a one-line detail for ra_last_error() and return `s`.
ra_status fail(ra_status s, const char* fmt, ...);

// Map a CUDA error to a status (RA_OK when e == cudaSuccess).
ra_status cuda_fail(cudaError_t e, const char* what);

// Limit of every bounded device wait, in ns.
unsigned long long wait_timeout_ns();

}  // namespace ra

#define RA_CUDA_TRY(expr)                                 \
    do {                                                  \
        cudaError_t ra_e_ = (expr);                       \
        if (ra_e_ != cudaSuccess)                         \
            return ra::cuda_fail(ra_e_, #expr);           \
    } while (0)
