// Host-side status plumbing: last-error text per thread, CUDA error mapping.
#include <cstdarg>
#include <cstdio>

#include "common.cuh"

namespace i4 {

static thread_local char g_last_error[512] = "";

int fail(int status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

int cuda_check(cudaError_t err, const char *what) {
    if (err == cudaSuccess) return I4_OK;
    return fail(I4_ECUDA, "%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
}

int launch_check(const char *what) { return cuda_check(cudaGetLastError(), what); }

}  // namespace i4

extern "C" const char *i4_last_error(void) { return i4::g_last_error; }

extern "C" const char *i4_version(void) { return "i4rt 0.1 (sm_100a)"; }
