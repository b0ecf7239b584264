// runtime.cu -- per-device facts cached once per process: the SM count,
// which kernels already have their shared-memory limit raised, and the last
// value of each device error counter that a check has seen.  These are the
// library's only mutable host state; all are safe for concurrent callers.
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
// last value of each device counter reported by a check, per device
std::atomic<unsigned> g_seen[kCounters][kMaxDevices];
}  // namespace

unsigned counter_increase(int counter, unsigned value) {
    int dev = 0;
    if (counter < 0 || counter >= kCounters || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
        dev >= kMaxDevices)
        return 0;
    // unsigned difference: correct across a wrap of the 32-bit counter
    return value - g_seen[counter][dev].exchange(value, std::memory_order_acq_rel);
}

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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point, so that
// the library needs no link-time libcuda.
static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
              uint64_t rows, uint64_t stride, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {stride};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace quik
