// runtime.cu -- per-device facts cached once per process: the SM count and
// which kernels already have their shared-memory limit raised.  These are the
// library's only mutable host state; both are guarded for concurrent callers.
#include <atomic>
#include <mutex>

#include "quik_internal.h"

namespace quik {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
// (kernel, device) pairs already configured; a fixed table, so that launches
// never allocate host memory either.
constexpr int kMaxKernels = 64;
std::mutex g_attr_mu;
const void *g_attr_kernel[kMaxKernels];
unsigned long long g_attr_devmask[kMaxKernels];
int g_attr_n = 0;
}  // namespace

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            return 148;
        g_sm_count[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

bool attribute_set_once(const void *kernel, int dyn_smem_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    int slot = -1;
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr_kernel[i] == kernel) slot = i;
    if (slot >= 0 && (g_attr_devmask[slot] >> dev) & 1ull) return true;
    if (slot < 0) {
        if (g_attr_n == kMaxKernels) return false;
        slot = g_attr_n++;
        g_attr_kernel[slot] = kernel;
        g_attr_devmask[slot] = 0;
    }
    // raise to the largest size any launch of this kernel uses
    int max_optin = 0;
    if (cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
        return false;
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return false;
    const int want = static_cast<int>(max_optin - fa.sharedSizeBytes);
    if (dyn_smem_bytes > want) return false;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, want) !=
        cudaSuccess)
        return false;
    g_attr_devmask[slot] |= 1ull << dev;
    return true;
}

}  // namespace quik
