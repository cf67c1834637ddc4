// ra_api.cu -- status strings, per-thread error details and library settings.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>

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
