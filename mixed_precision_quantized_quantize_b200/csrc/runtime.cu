// runtime.cu -- per-device facts cached once per process: the SM count and
// which kernels already have their shared-memory limit raised.  These are the
// library's only mutable host state; both are guarded for concurrent callers.
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "quik_internal.h"

namespace quik {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::mutex g_attr_mu;
std::set<std::pair<const void *, int>> g_attr_done;  // (kernel, device)
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
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (g_attr_done.count({kernel, dev})) return true;
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
    g_attr_done.insert({kernel, dev});
    return true;
}

}  // namespace quik
