// noalloc.cu -- quik_linear for callers that cannot allocate device memory.
//
// quik_linear needs a workspace for the quantised activations.  Most callers
// allocate it once and pass it in.  Some cannot: a host framework that owns
// every device allocation through its own fixed memory plan and gives a
// plugin no workspace, or a latency-critical path where cudaMalloc (which may
// synchronise the whole device) is not allowed.  quik_linear_noalloc serves
// them from a workspace that lives in this library's own device data segment,
// a fixed-size array that every GPU loading the library holds until the
// process exits.  Nothing is allocated on any call.
#include <atomic>
#include <mutex>

#include "quik_internal.h"

namespace {

constexpr size_t kScratchBytes = QUIK_NOALLOC_SCRATCH_BYTES;  // from include/quik.h
constexpr int kMaxDevices = 64;

// The workspace itself.  Its host-side name is only a handle for the runtime:
// kernels must be given the device address that cudaGetSymbolAddress returns.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

std::atomic<void *> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the workspace on the current device, looked up once per
// device (with that device current) and cached.
void *scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
            return nullptr;
        p = addr;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" {

quik_status quik_linear_noalloc(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                                const void *Wq, const float *w_scale, const void *Wo,
                                const float *wo_scale, const void *bias_f16, void *Y_f16,
                                quik_stream_t stream) {
    const size_t need = quik_workspace_size(shape);
    if (need == 0) return QUIK_ERR_INVALID_ARG;  // invalid shape
    if (need > kScratchBytes) return QUIK_ERR_UNSUPPORTED;
    void *ws = scratch_address();
    if (ws == nullptr) return QUIK_ERR_CUDA;
    // The quantise kernel rewrites every byte of the workspace that the GEMM
    // reads, so nothing has to be cleared between calls.
    return quik_linear(shape, X_f16, perm, Wq, w_scale, Wo, wo_scale, bias_f16, Y_f16, ws,
                       kScratchBytes, stream);
}

}  // extern "C"
