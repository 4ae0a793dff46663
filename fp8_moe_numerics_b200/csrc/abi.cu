// abi.cu -- status handling and size helpers of the mxmoe C ABI.
#include "mx_common.cuh"

#include <atomic>

namespace {
thread_local int g_last_cuda_error = 0;
constexpr int kMaxDevices = 64;
// 0 unknown, 1 sm_100, -1 other; read and written by every host thread that
// calls an entry point (relaxed: each thread that finds 0 computes the same
// value and stores it)
std::atomic<int> g_device_ok[kMaxDevices] = {};
}  // namespace

int mx_set_cuda_error(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return MX_ECUDA;
}

namespace {
std::atomic<unsigned long long> g_kernel_launches{0};
}  // namespace

void mx_count_launch(void) { g_kernel_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" unsigned long long mx_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

int mx_launch_status(void) {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MX_OK : mx_set_cuda_error(e);
}

int mx_check_device(void) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return mx_set_cuda_error(e);
    if (dev >= 0 && dev < kMaxDevices) {
        const int known = g_device_ok[dev].load(std::memory_order_relaxed);
        if (known) return known > 0 ? MX_OK : MX_EUNSUPPORTED;
    }
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
        return mx_set_cuda_error(e);
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < kMaxDevices) g_device_ok[dev].store(ok ? 1 : -1, std::memory_order_relaxed);
    return ok ? MX_OK : MX_EUNSUPPORTED;
}

extern "C" int mx_version(void) { return 1; }

extern "C" int mx_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" size_t mx_sf_bytes(int64_t rows, int64_t cols, int block, int sf_layout) {
    if (rows < 0 || cols <= 0 || (block != 16 && block != 32) || cols % block) return 0;
    const int64_t S = cols / block;
    if (sf_layout == MX_SF_ROWMAJOR) return (size_t)(rows * S);
    if (sf_layout == MX_SF_MMA) {
        if (rows % 128 || S % 4) return 0;
        return (size_t)(rows * S);                  // atoms tile the array exactly
    }
    return 0;
}

extern "C" size_t mx_route_workspace_bytes(int64_t T, int64_t E) {
    if (T < 0 || E <= 0) return 0;
    const int64_t chunks = T / 256 + (T % 256 != 0);
    if (chunks > (INT64_MAX / (int64_t)sizeof(int32_t) - E) / E) return SIZE_MAX;   // would overflow int64
    return (size_t)((chunks * E + E) * sizeof(int32_t));
}

MX_BOUNDS_READER(mx_bounds_word_abi)

extern "C" int mx_debug_bounds_build(void) {
#ifdef MX_DEBUG_BOUNDS
    return 1;
#else
    return 0;
#endif
}

extern "C" unsigned long long mx_debug_bounds_violations(int clear) {
    const bool c = clear != 0;
    return (unsigned long long)mx_bounds_word_abi(c) + mx_bounds_word_quant(c) + mx_bounds_word_glue(c) +
           mx_bounds_word_gemm(c) + mx_bounds_word_s2f6(c) + mx_bounds_word_nvfp4_bwd(c);
}
