// ra_api.cu -- status strings, per-thread error details, library settings and
// TMA tensor maps.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "ra_internal.h"

namespace ra {
namespace {
thread_local char g_last_error[256] = "";
std::atomic<unsigned long long> g_timeout_ns{4000000000ull};
}  // namespace

ra_status fail(ra_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

ra_status cuda_fail(cudaError_t e, const char* what)
{
    if (e == cudaSuccess)
        return RA_OK;
    cudaGetLastError();  // clear a sticky-free launch error so later calls start clean
    return fail(e == cudaErrorMemoryAllocation ? RA_ERR_OUT_OF_MEMORY : RA_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
}

unsigned long long wait_timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }

namespace {
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

}  // namespace

// [B*H, head_rows, d] bf16 as a 3D tensor (d, rows, B*H): boxes of box_rows
// rows x 64 columns, 128-byte swizzle; rows beyond `rows` read as zero.
ra_status make_map_rows(CUtensorMap* map, const void* base, int BH, int rows, int head_rows, int d, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    if (rows < 1 || rows > head_rows)
        return fail(RA_ERR_INVALID_ARG, "tensor map rows %d outside [1, %d]", rows, head_rows);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(head_rows) * d * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(RA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return RA_OK;
}

ra_status make_map(CUtensorMap* map, const void* base, int BH, int n, int d, int box_rows)
{
    return make_map_rows(map, base, BH, n, n, d, box_rows);
}

}  // namespace ra

extern "C" const char* ra_status_string(ra_status s)
{
    switch (s) {
    case RA_OK:
        return "ok";
    case RA_ERR_INVALID_ARG:
        return "invalid argument";
    case RA_ERR_UNSUPPORTED:
        return "unsupported";
    case RA_ERR_CUDA:
        return "CUDA error";
    case RA_ERR_OUT_OF_MEMORY:
        return "out of device memory";
    case RA_ERR_DEVICE_TIMEOUT:
        return "device wait timed out";
    case RA_ERR_DEVICE_BOUNDS:
        return "device bounds check failed";
    }
    return "unknown status";
}

extern "C" const char* ra_last_error(void) { return ra::g_last_error; }

extern "C" ra_status ra_set_wait_timeout_ns(long long timeout_ns)
{
    if (timeout_ns < 1000000LL || timeout_ns > 60000000000LL)
        return ra::fail(RA_ERR_INVALID_ARG, "timeout_ns must be in [1e6, 6e10]");
    ra::g_timeout_ns.store(static_cast<unsigned long long>(timeout_ns), std::memory_order_relaxed);
    return RA_OK;
}

extern "C" int ra_version(void) { return 1 * 10000 + 0 * 100 + 0; }
