// quantize.cu -- reorder + dynamic symmetric INT4 quantisation + nibble packing
// of the rows of an fp16 matrix, with the outlier block copied (FP16) or
// quantised to INT8.  Serves activations (one row per token; "Atom: Low-bit
// Quantization for Efficient and Accurate LLM Serving", summary: dynamic
// per-input scales, reordering fused into one pass, idea I2) and the offline
// weight pack (one row per output channel; QUIK sample names pack_to_i4 /
// two_compl).
//
// One CTA owns one row at a time (grid-stride over rows, 256 threads):
//   1. the CTA stages perm (as uint16) once; the rows arrive in a ring of up
//      to three shared-memory buffers, each filled by one TMA bulk copy issued
//      as soon as the buffer is free, so several rows per CTA are in flight;
//   2. each thread gathers 8 reordered positions per 32-bit output word
//      (up to MAXW words, kept in registers), takes their absmax;
//   3. per-row scale: block reduction; per-group scale (128 positions =
//      16 words = 16 adjacent lanes): 4-step xor shuffle;
//   4. codes are packed 8 per word and stored coalesced (a warp writes 128
//      contiguous bytes);
//   5. outlier positions Ki..K-1 are gathered and copied, or quantised with
//      their own absmax/127 scale.
// The kernel is bound by HBM bandwidth (2 bytes read per element, 0.5 byte
// written per INT4 element).
#include <algorithm>
#include <atomic>

#include <cuda_fp16.h>

#include "quik_internal.h"
#include "sm100.cuh"

namespace quik {

QUIK_CHECK_DECL

// Count of bounded waits that ran out in this file's kernels (read and
// cleared by quik_sync_check through take_quantize_errors).
__device__ unsigned int g_quant_error;

namespace {

constexpr int kQThreads = 256;

struct QParams {
    const uint16_t *X;
    const int32_t *perm;
    int rows, K, k_o;
    int nring;  // row buffers per CTA (1..3)
    uint8_t *Q;
    float *scale;
    void *O;
    float *o_scale;
};

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// Rounding by the addition of 1.5 * 2^23: for |t| < 2^22 the fp32 sum
// t + 1.5*2^23 is rounded (to nearest, ties to even) to an integer, so its bit
// pattern is 0x4B400000 + rint(t) and (sum - 1.5*2^23) == rint(t) exactly.
constexpr float kRound = 12582912.0f;
constexpr uint32_t kRoundBits = 0x4B400000u;
// Packing 8 codes q_k into nibbles: word = 0x88888888 + sum_k q_k * 16^k
// holds the offset digits q_k + 8 in [1, 15] without carries; xor 0x88888888
// turns them into 4-bit two's complement.  With the rounding bit patterns
// b_k = 0x4B400000 + q_k the constant term is folded in advance (mod 2^32).
constexpr uint32_t kPackBias = 0x88888888u - kRoundBits * 0x11111111u;

// Exact code of one value (the rare near-tie path): rint of the correctly
// rounded fp32 quotient, clamped, 0 when s == 0.
__device__ __forceinline__ int exact_code(float v, float s, int qmax) {
    if (s == 0.0f) return 0;
    const int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-qmax, min(qmax, q));
}

// Eight codes of one 32-bit output word from four half2 values.
//   Fast path: t = v * fl(1/s).  With u = 2^-24, |t - fl(v/s)| <= 3u|v/s|(1+u)
//   <= 1.3e-6 for |v/s| <= 7 (|v| <= max|v|, so |v/s| <= 7(1+u)^2), hence
//   unless t lies within 2e-6 of a half-integer (the only points where rint
//   changes value) fl(v/s) rounds to the same integer.  |t - rint(t)| is
//   computed exactly (Sterbenz), and a word with any near-tie is redone with
//   IEEE divisions.  No clamp is needed: |rint(t)| <= 7.
__device__ __forceinline__ uint32_t pack_codes8(const uint32_t (&h)[4], float s, float rs) {
    uint32_t word = kPackBias;
    float dmax = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[k]));
        // explicit roundings: the product must not be contracted into the add
        const float t0 = __fmul_rn(f.x, rs), t1 = __fmul_rn(f.y, rs);
        const float m0 = __fadd_rn(t0, kRound), m1 = __fadd_rn(t1, kRound);
        dmax = fmaxf(dmax, fmaxf(fabsf(__fsub_rn(t0, __fsub_rn(m0, kRound))),
                                 fabsf(__fsub_rn(t1, __fsub_rn(m1, kRound)))));
        word += __float_as_uint(m0) << (8 * k);
        word += __float_as_uint(m1) << (8 * k + 4);
    }
    if (dmax > 0.5f - 2e-6f) {  // near a tie somewhere in this word: exact divisions
        word = 0x88888888u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int q0 = exact_code(h2f(static_cast<uint16_t>(h[k] & 0xffffu)), s, 7);
            const int q1 = exact_code(h2f(static_cast<uint16_t>(h[k] >> 16)), s, 7);
            word += static_cast<uint32_t>(q0) << (8 * k);
            word += static_cast<uint32_t>(q1) << (8 * k + 4);
        }
    }
    return word ^ 0x88888888u;
}

// INT8 outlier code (same fast path; |v/s| <= 127 widens the tie margin).
__device__ __forceinline__ int code8(float v, float s, float rs) {
    const float t = __fmul_rn(v, rs);
    const float m = __fadd_rn(t, kRound);
    if (fabsf(__fsub_rn(t, __fsub_rn(m, kRound))) > 0.5f - 4e-5f) return exact_code(v, s, 127);
    return static_cast<int>(__float_as_uint(m) - kRoundBits);
}

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

__device__ __forceinline__ float half2_absmax(uint32_t m2) {
    const __half2 a = __habs2(*reinterpret_cast<const __half2 *>(&m2));
    return fmaxf(__low2float(a), __high2float(a));
}

template <bool GROUPED, bool OUT_INT8, int MAXW>
__global__ void __launch_bounds__(kQThreads) quantize_rows_kernel(QParams p) {
    extern __shared__ __align__(16) uint8_t qsmem[];
    __shared__ float red_a[kQThreads / 32];
    __shared__ float red_b[kQThreads / 32];
    __shared__ uint64_t row_full[3];
    __shared__ int give_up;
    const int K = p.K, Ki = K - p.k_o;
    const int Kp = (K + 7) & ~7;
    uint16_t *perm_s = reinterpret_cast<uint16_t *>(qsmem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwords = Ki / 8;
    const int G = GROUPED ? Ki / kGroup : 1;
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2;

    auto ring = [&](int j) { return perm_s + Kp * (1 + j % p.nring); };
    auto issue = [&](int j) {  // thread 0: bulk-copy this CTA's j-th row into its buffer
        const int row = blockIdx.x + j * gridDim.x;
        if (row < p.rows) {
            ptx::mbar_arrive_expect_tx(&row_full[j % p.nring], row_bytes);
            ptx::bulk_load(ring(j), p.X + static_cast<size_t>(row) * K, row_bytes, &row_full[j % p.nring]);
        }
    };
    // Stage perm as uint16: one bulk copy of the int32 vector into the (still
    // unused) row buffers, then an in-shared-memory narrowing.  A strided loop
    // of global loads here would cost one memory latency per iteration.
    __shared__ uint64_t perm_full;
    int32_t *perm32 = reinterpret_cast<int32_t *>(perm_s + Kp);  // needs 4K <= 2 Kp nring bytes
    if (tid == 0) {
        for (int s = 0; s < p.nring; ++s) ptx::mbar_init(&row_full[s], 1);
        ptx::mbar_init(&perm_full, 1);
        give_up = 0;
        ptx::fence_barrier_init();
        ptx::mbar_arrive_expect_tx(&perm_full, static_cast<uint32_t>(K) * 4);
        ptx::bulk_load(perm32, p.perm, static_cast<uint32_t>(K) * 4, &perm_full);
        if (!ptx::mbar_wait_bounded(&perm_full, 0, kWaitLimitNs)) {
            give_up = 1;
            atomicAdd(&g_quant_error, 1u);
        }
    }
    __syncthreads();
    for (int i = tid; i < K / 4; i += kQThreads) {  // K % 4 == 0
        const int4 v = reinterpret_cast<const int4 *>(perm32)[i];
        reinterpret_cast<uint2 *>(perm_s)[i] =
            make_uint2(static_cast<uint32_t>(v.x) | (static_cast<uint32_t>(v.y) << 16),
                       static_cast<uint32_t>(v.z) | (static_cast<uint32_t>(v.w) << 16));
    }
    __syncthreads();  // perm_s ready; the row buffers may now be overwritten
    if (give_up) return;
    if (tid == 0)
        for (int j = 0; j < p.nring; ++j) issue(j);

    for (int j = 0;; ++j) {
        const int row = blockIdx.x + j * gridDim.x;
        if (row >= p.rows) break;
        // (1) wait for this row's buffer (bounded; on expiry the row is skipped)
        if (tid == 0 && !ptx::mbar_wait_bounded(&row_full[j % p.nring], (j / p.nring) & 1, kWaitLimitNs)) {
            give_up = 1;
            atomicAdd(&g_quant_error, 1u);
        }
        __syncthreads();
        if (give_up) break;
        const uint16_t *row_s = ring(j);

        // (2) gather 8 reordered values per word (as 4 half2), absmax per word
        uint32_t v[MAXW][4];
        float wmax[MAXW];
#pragma unroll
        for (int i = 0; i < MAXW; ++i) {
            const int w = tid + i * kQThreads;
            wmax[i] = 0.0f;
            if (w < nwords && QUIK_CHECK(8 * w + 8 <= Kp, 2)) {
                const uint4 ix = *reinterpret_cast<const uint4 *>(perm_s + 8 * w);
                const uint32_t idx[4] = {ix.x, ix.y, ix.z, ix.w};
                __half2 m2 = __float2half2_rn(0.0f);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (!QUIK_CHECK((idx[k] & 0xffffu) < (uint32_t)K && (idx[k] >> 16) < (uint32_t)K, 1)) {
                        v[i][k] = 0;
                        continue;
                    }
                    const uint32_t a = row_s[idx[k] & 0xffffu], b = row_s[idx[k] >> 16];
                    v[i][k] = a | (b << 16);
                    m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __half2 *>(&v[i][k])));
                }
                wmax[i] = half2_absmax(*reinterpret_cast<const uint32_t *>(&m2));
            }
        }

        // (3) scales
        float s[MAXW];
        if (GROUPED) {
#pragma unroll
            for (int i = 0; i < MAXW; ++i) {
                float m = wmax[i];
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                s[i] = __fdiv_rn(m, 7.0f);
                const int w = tid + i * kQThreads;
                if (w < nwords && (lane & 15) == 0 && QUIK_CHECK(w / 16 < G, 3))
                    p.scale[static_cast<size_t>(row) * G + w / 16] = s[i];
            }
        } else {
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < MAXW; ++i) m = fmaxf(m, wmax[i]);
            m = warp_max(m);
            if (lane == 0) red_a[warp] = m;
            __syncthreads();
            m = red_a[0];
#pragma unroll
            for (int k = 1; k < kQThreads / 32; ++k) m = fmaxf(m, red_a[k]);
            const float sr = __fdiv_rn(m, 7.0f);
#pragma unroll
            for (int i = 0; i < MAXW; ++i) s[i] = sr;
            if (tid == 0) p.scale[row] = sr;
        }

        // (4) codes, 8 per word, code 2i in the low nibble of byte i
        uint32_t *qrow = reinterpret_cast<uint32_t *>(p.Q + static_cast<size_t>(row) * (Ki / 2));
#pragma unroll
        for (int i = 0; i < MAXW; ++i) {
            const int w = tid + i * kQThreads;
            if (w < nwords && QUIK_CHECK(4 * w + 4 <= Ki / 2, 4)) {
                const float rs = s[i] != 0.0f ? __frcp_rn(s[i]) : 0.0f;
                qrow[w] = pack_codes8(v[i], s[i], rs);
            }
        }

        // (5) the outlier block
        if (p.k_o > 0) {
            if (!OUT_INT8) {
                uint16_t *o = static_cast<uint16_t *>(p.O) + static_cast<size_t>(row) * p.k_o;
                for (int i = tid; i < p.k_o; i += kQThreads)
                    if (QUIK_CHECK(perm_s[Ki + i] < K, 5)) o[i] = row_s[perm_s[Ki + i]];
            } else {
                float m = 0.0f;
                for (int i = tid; i < p.k_o; i += kQThreads)
                    m = fmaxf(m, fabsf(h2f(row_s[perm_s[Ki + i]])));
                m = warp_max(m);
                if (lane == 0) red_b[warp] = m;
                __syncthreads();
                m = red_b[0];
#pragma unroll
                for (int k = 1; k < kQThreads / 32; ++k) m = fmaxf(m, red_b[k]);
                const float so = __fdiv_rn(m, 127.0f);
                const float rso = so != 0.0f ? __frcp_rn(so) : 0.0f;
                if (tid == 0) p.o_scale[row] = so;
                int8_t *o = static_cast<int8_t *>(p.O) + static_cast<size_t>(row) * p.k_o;
                for (int i = tid; i < p.k_o; i += kQThreads)
                    o[i] = static_cast<int8_t>(code8(h2f(row_s[perm_s[Ki + i]]), so, rso));
            }
        } else if (OUT_INT8 && p.o_scale != nullptr && tid == 0) {
            p.o_scale[row] = 0.0f;
        }
        __syncthreads();  // buffer and reduction slots are free again
        if (tid == 0) issue(j + p.nring);
    }
    // never leave the CTA with a bulk copy still writing its shared memory
    if (tid == 0)
        for (int s = 0; s < p.nring; ++s) {
            // the last row issued into slot s, if any
            int last = -1;
            for (int j = s; blockIdx.x + j * gridDim.x < p.rows; j += p.nring) last = j;
            if (last >= 0) ptx::mbar_wait_bounded(&row_full[s], (last / p.nring) & 1, kWaitLimitNs);
        }
}

template <bool GROUPED, bool OUT_INT8, int MAXW>
cudaError_t launch_q(QParams p, cudaStream_t stream) {
    auto kern = quantize_rows_kernel<GROUPED, OUT_INT8, MAXW>;
    const int Kp = (p.K + 7) & ~7;
    const size_t row_bytes = static_cast<size_t>(Kp) * sizeof(uint16_t);
    // perm (uint16) plus up to three row buffers within ~200 KB of shared memory
    p.nring = static_cast<int>(std::min<size_t>(3, (200u << 10) / row_bytes - 1));
    if (p.nring < 2) return cudaErrorInvalidConfiguration;  // the ring also stages perm (int32)
    const size_t smem = row_bytes * (1 + p.nring);
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), static_cast<int>(smem)))
        return cudaErrorInvalidConfiguration;
    // grid: every CTA that fits at once, rows grid-strided; the occupancy of
    // the last shared-memory size seen is cached (one query per new K)
    static std::atomic<long long> occ_cache{-1};  // (smem << 8) | CTAs per SM
    long long c = occ_cache.load(std::memory_order_relaxed);
    int per_sm = 0;
    if (c >= 0 && (c >> 8) == static_cast<long long>(smem)) {
        per_sm = static_cast<int>(c & 0xff);
    } else {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kQThreads, smem);
        if (e != cudaSuccess) return e;
        occ_cache.store((static_cast<long long>(smem) << 8) | (per_sm & 0xff), std::memory_order_relaxed);
    }
    const int grid = std::max(1, std::min(p.rows, sm_count() * std::max(per_sm, 1)));
    kern<<<grid, kQThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

template <bool GROUPED, bool OUT_INT8>
cudaError_t launch_q_w(const QParams &p, cudaStream_t stream) {
    const int words_per_thread = ((p.K - p.k_o) / 8 + kQThreads - 1) / kQThreads;
    if (words_per_thread <= 2) return launch_q<GROUPED, OUT_INT8, 2>(p, stream);
    if (words_per_thread <= 4) return launch_q<GROUPED, OUT_INT8, 4>(p, stream);
    if (words_per_thread <= 8) return launch_q<GROUPED, OUT_INT8, 8>(p, stream);
    return launch_q<GROUPED, OUT_INT8, 16>(p, stream);
}

}  // namespace

cudaError_t launch_quantize_rows(const QuantizeArgs &a, cudaStream_t stream) {
    QParams p{a.X, a.perm, a.rows, a.K, a.k_o, 1, a.Q, a.scale, a.O, a.o_scale};
    if (a.group > 0)
        return a.out_int8 ? launch_q_w<true, true>(p, stream) : launch_q_w<true, false>(p, stream);
    return a.out_int8 ? launch_q_w<false, true>(p, stream) : launch_q_w<false, false>(p, stream);
}

unsigned int take_quantize_errors() {
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_quant_error, sizeof(word)) != cudaSuccess) return 0;
    if (word != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(zero));
    }
    return word;
}

}  // namespace quik

#ifdef QUIK_CHECKS
extern "C" __attribute__((visibility("default"))) unsigned long long qchk_quantize_word() {
    unsigned long long v = 0;
    cudaMemcpyFromSymbol(&v, quik::g_check_word, sizeof(v));
    return v;
}
#endif
