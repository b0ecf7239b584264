// quik_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/quik.h"

// Optional self-checks (build with -DQUIK_CHECKS): bounds and alignment of
// every computed index are verified before use; the first violation is
// recorded as (tag << 32 | source line) in a per-file device word and the
// access is skipped.  Off in normal builds (the macro folds to `true`).
#ifdef QUIK_CHECKS
#define QUIK_CHECK_DECL __device__ unsigned long long g_check_word;
#define QUIK_CHECK(cond, tag)                                                                  \
    ((cond) ? true                                                                             \
            : (atomicCAS(&g_check_word, 0ull,                                                  \
                         (static_cast<unsigned long long>(tag) << 32) | __LINE__),             \
               false))
#else
#define QUIK_CHECK_DECL
#define QUIK_CHECK(cond, tag) true
#endif

namespace quik {

constexpr int kMaxK = 32768;       // largest K the quantiser stages in shared memory
constexpr int kMaxKNorm = 24576;   // with the RMS norm folded in (a second K-wide table)
constexpr int kGroup = 128;        // the one supported group width
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s bound on every in-kernel wait
constexpr int kDecodeTokens = 32;  // up to this many tokens the product is decode-shaped

// Reorder + quantise + pack `rows` rows of a [rows, K] fp16 matrix.
struct QuantizeArgs {
    const uint16_t *X;
    const int32_t *perm;
    int rows, K, k_o, group;
    bool out_int8;
    bool bits8;  // INT8 codes (divisor and clamp 127, one byte each) instead of packed INT4
    // INT4 codes written wide, as the signed bytes 16 c [rows, K_i] in the
    // persistent GEMM's operand order (per 32 positions: the 16 even ones,
    // then the 16 odd ones); per-row scales only
    bool wide = false;
    uint8_t *Q;
    float *scale;
    void *O;
    float *o_scale;
    // RMS norm folded in (NULL: none): the rows are normalised with weight
    // gamma [K] (source channel order) and eps before they are quantised
    const uint16_t *gamma = nullptr;
    float eps = 0.0f;
};
cudaError_t launch_quantize_rows(const QuantizeArgs &a, cudaStream_t stream);

// 2:4-sparse INT4 rows of a [rows, K] fp16 matrix: reorder, keep the two
// largest magnitudes of every aligned group of four INT4 positions, quantise
// (per-row scale), write kept codes [rows, K_i / 4] and position pairs
// [rows, K_i / 8]; the outlier block as launch_quantize_rows.
struct Prune24Args {
    const uint16_t *W;
    const int32_t *perm;
    int rows, K, k_o;
    bool out_int8;
    uint8_t *Qs;
    uint8_t *meta;
    float *scale;
    void *O;
    float *o_scale;
};
cudaError_t launch_prune24_rows(const Prune24Args &a, cudaStream_t stream);
// The dense packed INT4 rows [rows, K_i / 2] of 2:4 rows (K_i % 128 == 0).
cudaError_t launch_expand24(const uint8_t *Qs, const uint8_t *meta, int rows, int Ki, uint8_t *Q,
                            cudaStream_t stream);
// The device error counters only ever grow: kernels add to them and nothing
// resets them, so a kernel that compares the counter with the value it saw at
// its start learns of every error recorded since.  A check reports the
// increase since the previous check of the same counter on the current device.
enum { kCounterGemmWaits = 0, kCounterQuantWaits = 1, kCounterBadPerm = 2, kCounterPGemmWaits = 3, kCounters = 4 };
unsigned counter_increase(int counter, unsigned value);
// Expired waits in the quantise kernels since the last check (returned), and
// perm entries outside [0, K) met since the last check (in *bad_perm when
// given); synchronous.
unsigned int take_quantize_errors(unsigned int *bad_perm);

// INT4 x INT4 (+ outlier) product with the dequantising epilogue, or the raw
// integer sums when acc_dbg is set.
struct GemmArgs {
    int M, N, K, k_o, group;
    bool out_int8;
    bool a8;  // Xq holds INT8 codes [M, K_i] (W4A8) instead of packed INT4
    bool w8;  // Wq holds INT8 codes [N, K_i] (W8A8; with a8)
    bool x_wide = false;  // Xq holds the bytes 16 c [M, K_i] in operand order (quantiser's wide output)
    const void *Xq;
    const float *sx;
    const void *Xo;
    const float *sxo;
    const void *Wq;       // packed codes, or the kept codes [N, K_i / 4] of 2:4 weights
    const uint8_t *Wmeta = nullptr;  // 2:4 weights: position pairs [N, K_i / 8]
    bool sparse24 = false;           // W is 2:4-sparse (Wq + Wmeta)
    const float *sw;
    const void *Wo;
    const float *swo;
    const uint16_t *bias;
    uint16_t *Y;
    bool debug;          // write the integer sums instead of Y
    bool after_quantize; // the previous kernel on the stream is this library's quantiser of Xq
                         // (the GEMM may then start early: programmatic dependent launch)
    int32_t *acc_dbg;    // [M,N] or [G,M,N] integer sums of the INT4 part (debug only)
    int32_t *acc_o_dbg;  // INT8 outliers' integer sums (debug only)
};

// Number of SMs of the current device (cached per device).
int sm_count();
// Raise `kernel`'s dynamic shared-memory limit on the current device to the
// device maximum (once per kernel and device); false if dyn_smem_bytes
// cannot fit or a CUDA call fails.
bool attribute_set_once(const void *kernel, int dyn_smem_bytes);
quik_status launch_gemm(const GemmArgs &a, cudaStream_t stream);
// The persistent CTA-pair kernel (per-channel scales, INT4 activations and
// weights, FP16 or no outliers, more than kDecodeTokens tokens, K_i > 0).
bool persistent_gemm_takes(const GemmArgs &a);
quik_status launch_gemm_persistent(const GemmArgs &a, cudaStream_t stream);
// Expired waits in the persistent kernel since the last check.
unsigned int persistent_gemm_errors();
// quik_test_stall's switches (test entry)
cudaError_t set_quantize_stall(int on);
cudaError_t set_persistent_gemm_stall(int on);
// 2-D row-major TMA map: `inner` elements per row (contiguous), `rows` rows,
// `stride` bytes between rows; box of box_inner x box_rows; elements outside
// the tensor read as zero.
bool make_map(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
              uint64_t rows, uint64_t stride, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle sw);

quik_status sync_check(cudaStream_t stream);
quik_status launch_timeout_selftest(uint32_t limit_us, cudaStream_t stream);

}  // namespace quik
