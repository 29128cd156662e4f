// dlm_api.cu -- status strings, version, the device check and the
// device-status read-back of the C ABI.
#include <atomic>
#include <mutex>

#include "dlm_device.cuh"
#include "dlm_host.h"

#include <cstdio>

namespace dlm {

static thread_local char g_last_error[256] = "";

void record_cuda_error(cudaError_t e, const char* where) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorString(e),
                  cudaGetErrorName(e));
}

// Test hook (dlm_test_skip_device_check): when set, check_device passes
// without asking the runtime, so that on a host without a usable device each
// call goes on to its own CUDA calls and their error paths run.
static std::atomic<int> g_skip_device_check{0};

dlm_status_t check_device() {
    if (g_skip_device_check.load(std::memory_order_relaxed)) return DLM_OK;
    // compute capability 10.0 (B200) only; cached per device ordinal
    static std::mutex mu;
    static int known[64];   // 0 = unknown, 1 = ok, 2 = unsupported
    int dev = 0;
    cudaError_t e0 = cudaGetDevice(&dev);
    if (e0 != cudaSuccess) { cudaGetLastError(); return cuda_status(e0, "cudaGetDevice"); }
    if (dev < 0 || dev >= 64) return DLM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> g(mu);
    if (known[dev] == 0) {
        int major = 0, minor = 0;
        cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_status(e, "cudaDeviceGetAttribute (compute capability)");
        }
        known[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    return known[dev] == 1 ? DLM_OK : DLM_ERR_UNSUPPORTED;
}

// One thread waits on an mbarrier phase that nothing completes; the bounded
// wait gives up after `limit_ns`, records DLM_DEV_WAIT_TIMEOUT and the kernel
// returns normally.
__global__ void k_selftest_wait(uint64_t limit_ns, uint32_t* status) {
    __shared__ uint64_t bar;
    const uint32_t a = smem_addr(&bar);
    mbar_init(a, 1);                      // expects one arrival that never comes
    fence_mbar_init_cluster();
    mbar_wait_limit(a, 0, limit_ns, status);
}

}  // namespace dlm

extern "C" dlm_status_t dlm_selftest_bounded_wait(uint64_t limit_ns, uint32_t* dev_status,
                                                  dlm_stream_t stream) {
    if (!dev_status || limit_ns == 0 || limit_ns > 10000000000ull) return DLM_ERR_INVALID_ARGUMENT;
    dlm_status_t st = dlm::check_device();
    if (st != DLM_OK) return st;
    dlm::k_selftest_wait<<<1, 1, 0, (cudaStream_t)stream>>>(limit_ns, dev_status);
    return dlm::last_launch_status("k_selftest_wait launch");
}

extern "C" const char* dlm_status_string(dlm_status_t status) {
    switch (status) {
        case DLM_OK: return "DLM_OK";
        case DLM_ERR_INVALID_ARGUMENT: return "DLM_ERR_INVALID_ARGUMENT";
        case DLM_ERR_UNSUPPORTED: return "DLM_ERR_UNSUPPORTED";
        case DLM_ERR_WORKSPACE_TOO_SMALL: return "DLM_ERR_WORKSPACE_TOO_SMALL";
        case DLM_ERR_CUDA: return "DLM_ERR_CUDA";
        default: return "DLM_ERR_UNKNOWN";
    }
}

extern "C" int dlm_version(void) { return 200; }   // 0.2.0: + dlm_loss_fwd_bwd_ex

extern "C" const char* dlm_last_cuda_error(void) { return dlm::g_last_error; }

extern "C" dlm_status_t dlm_test_skip_device_check(int32_t enabled) {
    if (enabled != 0 && enabled != 1) return DLM_ERR_INVALID_ARGUMENT;
    dlm::g_skip_device_check.store(enabled, std::memory_order_relaxed);
    return DLM_OK;
}

extern "C" dlm_status_t dlm_get_device_status(const void* workspace, uint32_t* host_status,
                                              dlm_stream_t stream) {
    if (!workspace || !host_status) return DLM_ERR_INVALID_ARGUMENT;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(host_status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) cudaGetLastError();
    return dlm::cuda_status(e, "dlm_get_device_status");
}
