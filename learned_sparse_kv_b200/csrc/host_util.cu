// host_util.cu -- error reporting and device queries shared by the ABI entry points.
#include <stdarg.h>
#include <string.h>

#include <atomic>

#include "common.cuh"

namespace lsa {

static thread_local char g_last_error[512] = "";

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
}

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

int check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return LSA_OK;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

static std::atomic<int> g_test_stall{0};

int take_test_stall(int which) { return (g_test_stall.fetch_and(~which) & which) ? 1 : 0; }

// Host copy failure switch: -1 off; otherwise the number of copies that still succeed
// before one reports failure (the switch then turns itself off).
static std::atomic<int> g_fail_copy{-1};

bool take_copy_failure() {
    int n = g_fail_copy.load();
    while (n >= 0) {
        if (g_fail_copy.compare_exchange_weak(n, n - 1)) return n == 0;
    }
    return false;
}

}  // namespace lsa

extern "C" const char *lsa_last_error(void) { return lsa::g_last_error; }

extern "C" int lsa_test_stall_next_wait(int which) {
    if (which != LSA_TEST_STALL_ATTENTION && which != LSA_TEST_STALL_INDEXER)
        return lsa::fail(LSA_ERR_INVALID_ARG, "lsa_test_stall_next_wait: unknown kernel %d", which);
    lsa::g_test_stall.fetch_or(which);
    return LSA_OK;
}

extern "C" int lsa_test_fail_copy(int after) {
    if (after < -1) return lsa::fail(LSA_ERR_INVALID_ARG, "lsa_test_fail_copy: after must be >= -1 (got %d)", after);
    lsa::g_fail_copy.store(after);
    return LSA_OK;
}

extern "C" const char *lsa_version(void) { return "lsa-b200 0.1 (sm_100a)"; }
