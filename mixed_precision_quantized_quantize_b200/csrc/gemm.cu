// gemm.cu -- the hybrid W4A4 + outlier product on sm_100a tensor cores.
//
// Computes, for a BM x BN tile of Y (QUIK abstract; "Atom: Low-bit
// Quantization for Efficient and Accurate LLM Serving", summary and ideas
// I1 / I3):
//   A[m,n]  = sum_{j < K_i} qx[m,j] qw[n,j]        exact, INT32 (tensor cores)
//   O[m,n]  = sum_{i < k_o} Xo[m,i] Wo[n,i]         fp16 -> fp32, or int8 -> int32
//   Y[m,n]  = A sx[m] sw[n] + O (x sxo[m] swo[n] for INT8) + bias[n]  -> fp16
// or, with groups of 128 (Atom summary, fine-grained groups), one INT32 sum
// A_g per group, each dequantised with sx[m,g] sw[n,g] and added in fp32.
//
// Blackwell has no INT4 MMA.  Each 4-bit code c is widened to the signed
// byte 16*c, which needs no sign extension: for a packed word w the odd
// codes are w & 0xF0F0F0F0 and the even codes (w << 4) & 0xF0F0F0F0.  The
// tcgen05 kind::i8 MMA then accumulates 256 * A exactly in INT32 (|A| <=
// 49*K_i, so 256*|A| < 2^31 for K_i < 171196) and the epilogue shifts right
// by 8.  Both operands place the even codes of a 16-byte packed chunk in the
// first 16 unpacked bytes and the odd codes in the next 16, the same
// K-permutation on both sides, so every dot product is unchanged.
//
// Two kernels:
//   * per-channel scales: a CTA pair per 256 x 256 tile (cta_group::2),
//     activations in tensor memory, B through shared memory (described
//     above w4a4_gemm_pair_kernel);
//   * per-group scales: one CTA per 128 x 128 tile, both operands in shared
//     memory.  Warp 0 is the TMA producer of a packed staging ring, warp 1
//     allocates TMEM and issues tcgen05.mma, NT warps unpack into the
//     128-byte swizzled K-major operand ring (then copy the outlier tiles),
//     NE warps drain each group's INT32 sum while the next group accumulates
//     in the other TMEM buffer.
// Every mbarrier wait is bounded (2 s); on expiry the CTA counts the error in
// g_error_word, stops issuing work, waits for its in-flight copies and MMAs,
// frees TMEM and exits; other CTAs see the count change and give up too.
#include <algorithm>
#include <cstring>

#include <cuda_fp16.h>

#include "quik_internal.h"
#include "sm100.cuh"

namespace quik {

__device__ unsigned int g_error_word;
QUIK_CHECK_DECL

// Optional pipeline timeline (build with -DQUIK_TRACE): SM clock stamps of
// each role's per-k-block events for the first two CTAs of a launch.
#ifdef QUIK_TRACE
constexpr int kTraceCtas = 2, kTraceEvents = 12, kTraceKb = 96;
__device__ unsigned long long g_trace[kTraceCtas][kTraceEvents][kTraceKb];
#define QUIK_TRACE_AT(ev, kb)                                                                   \
    do {                                                                                        \
        const int _c = blockIdx.x + blockIdx.y * gridDim.x;                                     \
        if (_c < kTraceCtas && (kb) >= 0 && (kb) < kTraceKb) g_trace[_c][ev][kb] = clock64();   \
    } while (0)
#else
#define QUIK_TRACE_AT(ev, kb) \
    do {                      \
    } while (0)
#endif
// events: 0 producer issued packed k-block (TMEM-A kernel: last B warp arrived),
// 1 unpack start (after waits), 2 unpack done (TMEM-A kernel: last A warp), 3 MMA issued k-block, 4 epilogue saw accumulator,
// 5 epilogue done, 6 CTA start, 7 CTA end

namespace {

using namespace ptx;

constexpr int BM = 128;       // tile rows (tokens); one TMEM lane per row
constexpr int KB = 128;       // INT4 codes per k-block = one scale group
constexpr int PK_ROW = 64;    // packed bytes per row per k-block
constexpr int OP_ROW = 128;   // unpacked bytes per row per k-block (one swizzle row)

template <int BN_, bool GROUPED_, bool OUT_INT8_, bool DEBUG_, int NT_, int NE_, int SP_, int SU_,
          int MINB_>
struct Cfg {
    static constexpr int BN = BN_;
    static constexpr bool GROUPED = GROUPED_;
    static constexpr bool OUT_INT8 = OUT_INT8_;
    static constexpr bool DEBUG = DEBUG_;
    static constexpr int NT = NT_;  // unpack warps
    static constexpr int NE = NE_;  // epilogue warps (multiple of 4)
    static constexpr int MINB = MINB_;
    static constexpr int THREADS = (2 + NT + NE) * 32;
    static constexpr int SP = SP_;  // packed staging stages
    static constexpr int SU = SU_;  // operand stages
    static constexpr int PK_STAGE = (BM + BN) * PK_ROW;
    static constexpr int OP_STAGE = (BM + BN) * OP_ROW;
    static constexpr int OP_OFF = 0;
    static constexpr int PK_OFF = SU * OP_STAGE;
    static constexpr int SMEM = PK_OFF + SP * PK_STAGE + 1024;  // + alignment slack
    // TMEM columns: non-grouped: INT32 sum [0,BN) + outlier sum [BN,2BN);
    // grouped: NACC group buffers [b BN, (b+1) BN) taken in turn, so the MMA
    // can run NACC - 1 groups ahead of the drain.
    static constexpr int NACC = GROUPED ? 512 / BN : 2;
    static constexpr int TMEM_COLS = NACC * BN;
    static constexpr int CHUNKS = (BM + BN) * (PK_ROW / 16);     // 16-byte packed chunks
    static constexpr int CHUNKS_PER_THREAD = CHUNKS / (NT * 32);
    static constexpr int EPI_COLS = BN / (NE / 4);                // columns per epilogue warp
    static_assert(CHUNKS % (NT * 32) == 0, "unpack work must split evenly");
    static_assert(NE % 4 == 0, "epilogue warps cover the four TMEM lane quadrants");
    static_assert(TMEM_COLS * MINB <= 512, "TMEM of all resident CTAs");
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation is a power of two");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <bool OUT_INT8, bool DEBUG>
using CfgGroup = Cfg<128, true, OUT_INT8, DEBUG, 4, 8, 4, 4, 1>;

struct GemmParams {
    int M, N, Ki, k_o, nkb_i, nkb_o, G;
    int tma_y;  // pair kernel: Y leaves through shared memory and TMA stores
    const float *sx, *sw, *sxo, *swo;
    const uint16_t *bias;
    uint16_t *Y;
    int32_t *acc_dbg, *acc_o_dbg;
};

struct AbortState {
    volatile int *flag;  // this CTA has given up (shared memory)
    unsigned err0;       // the device error count when this CTA started
};

__device__ __forceinline__ void set_abort(const AbortState &ab) {
    *ab.flag = 1;
    atomicAdd(&g_error_word, 1u);
}

// Bounded wait.  Gives up at once when another role of this CTA has given up
// or when any CTA has recorded an error since this CTA started.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const AbortState &ab) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*ab.flag) return false;
        if ((it & 255u) == 255u && *reinterpret_cast<volatile unsigned *>(&g_error_word) != ab.err0) {
            *ab.flag = 1;
            return false;
        }
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            set_abort(ab);
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Exact int32 -> fp32 for |v| < 2^22: place v in the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float small_int_to_float(int32_t v) {
    return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// The integer sum A from the tensor-core accumulator.  INT4 codes enter the
// MMA as 16 c, so the accumulator holds 256 A (W4A4: |A| <= 49 K_i < 2^22,
// exact by the magic-number add), 16 A (W4A8) or A (W8A8).  With INT8
// activations |A| can pass 2^22: a rounding conversion, exact below 2^24.
template <bool A8, bool W8>
__device__ __forceinline__ int32_t acc_int(uint32_t raw) {
    return static_cast<int32_t>(raw) >> (W8 ? 0 : A8 ? 4 : 8);
}
template <bool A8, bool W8>
__device__ __forceinline__ float acc_float(uint32_t raw) {
    return A8 ? __int2float_rn(acc_int<A8, W8>(raw)) : small_int_to_float(acc_int<A8, W8>(raw));
}

// W4A8: 32 INT8 codes (two 16-byte chunks, codes in order) in the order the
// INT4 unpack gives the weights' codes: even positions of the 32, then odd.
__device__ __forceinline__ void order_i8_chunk(const uint4 a, const uint4 b, uint32_t *w) {
    const uint32_t x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(w[i]) : "r"(x[2 * i]), "r"(x[2 * i + 1]));
        asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(w[4 + i]) : "r"(x[2 * i]), "r"(x[2 * i + 1]));
    }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, C::MINB)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_xq,
                     const __grid_constant__ CUtensorMap tm_wq,
                     const __grid_constant__ CUtensorMap tm_xo,
                     const __grid_constant__ CUtensorMap tm_wo, const GemmParams p) {
    constexpr int BN = C::BN, SP = C::SP, SU = C::SU, NT = C::NT, NE = C::NE;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t pk_full[SP], pk_empty[SP], op_full[SU], op_empty[SU];
    __shared__ uint64_t acc_full[C::NACC], acc_empty[C::NACC], mma_done;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;
    __shared__ __align__(16) float epi_sw[NE][C::EPI_COLS];

    // 1024-byte aligned base (the swizzle pattern repeats every 1024 bytes)
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // token tiles vary fastest: the CTAs that share a W tile run in the same
    // wave, so each W tile leaves DRAM about once (L2 serves the others)
    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SP; ++s) {
            mbar_init(&pk_full[s], 1);
            mbar_init(&pk_empty[s], NT);
        }
        for (int s = 0; s < SU; ++s) {
            mbar_init(&op_full[s], NT);
            mbar_init(&op_empty[s], 1);
        }
        for (int b = 0; b < C::NACC; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], NE);
        }
        mbar_init(&mma_done, 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_error_word);
        fence_barrier_init();
    }
    if (threadIdx.x == 0) QUIK_TRACE_AT(6, 0);
    if (warp == 1) tmem_alloc(&tmem_base_s, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const AbortState abort_flag{&abort_s, err0_s};
    (void)QUIK_CHECK((smem_base & 1023u) == 0 && smem_base + C::SMEM - 1024 <= 232448u, 12);
    (void)QUIK_CHECK((tmem & 0xFFFFu) + C::TMEM_COLS <= 512u && (tmem >> 16) == 0, 13);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (p.nkb_i > 0) {
                tma_prefetch_desc(&tm_xq);
                tma_prefetch_desc(&tm_wq);
            }
            int last_pk[SP];
            for (int s = 0; s < SP; ++s) last_pk[s] = -1;
            bool ok = true;
            for (int kb = 0; kb < p.nkb_i && ok; ++kb) {
                const int s = kb % SP;
                if (!(ok = wait_bar(&pk_empty[s], ((kb / SP) & 1) ^ 1, abort_flag))) break;
                uint8_t *dst = smem + C::PK_OFF + s * C::PK_STAGE;
                mbar_arrive_expect_tx(&pk_full[s], C::PK_STAGE);
                tma_load_2d(dst, &tm_xq, kb * PK_ROW, m0, &pk_full[s]);
                tma_load_2d(dst + BM * PK_ROW, &tm_wq, kb * PK_ROW, n0, &pk_full[s]);
                last_pk[s] = kb;
                QUIK_TRACE_AT(0, kb);
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            for (int s = 0; s < SP; ++s)
                if (last_pk[s] >= 0) mbar_wait_bounded(&pk_full[s], (last_pk[s] / SP) & 1, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_i8 = idesc_s8_s32(BM, BN);
            const uint32_t id_f16 = idesc_f16_f32(BM, BN);
            bool ok = true;
            for (int kb = 0; kb < p.nkb_i && ok; ++kb) {
                const int s = kb % SU;
                uint32_t d = tmem;
                if (C::GROUPED) {
                    const int b = kb % C::NACC;
                    if (!(ok = wait_bar(&acc_empty[b], ((kb / C::NACC) & 1) ^ 1, abort_flag))) break;
                    d = tmem + b * BN;
                }
                if (!(ok = wait_bar(&op_full[s], (kb / SU) & 1, abort_flag))) break;
                tc_fence_after();
                QUIK_TRACE_AT(3, kb);
                const uint32_t a_addr = smem_base + C::OP_OFF + s * C::OP_STAGE;
                const uint32_t b_addr = a_addr + BM * OP_ROW;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t acc = C::GROUPED ? (k > 0) : (kb > 0 || k > 0);
                    mma_i8(d, sw128_kmajor_desc(a_addr + 32 * k), sw128_kmajor_desc(b_addr + 32 * k),
                           id_i8, acc);
                }
                mma_commit(&op_empty[s]);
                if (C::GROUPED) mma_commit(&acc_full[kb % C::NACC]);
            }
            if (p.nkb_o > 0 && ok) {
                uint32_t d = tmem + BN;
                int b = 0;
                if (C::GROUPED) {
                    b = p.nkb_i % C::NACC;
                    ok = wait_bar(&acc_empty[b], ((p.nkb_i / C::NACC) & 1) ^ 1, abort_flag);
                    d = tmem + b * BN;
                }
                for (int ko = 0; ko < p.nkb_o && ok; ++ko) {
                    const int kb = p.nkb_i + ko, s = kb % SU;
                    if (!(ok = wait_bar(&op_full[s], (kb / SU) & 1, abort_flag))) break;
                    tc_fence_after();
                    const uint32_t a_addr = smem_base + C::OP_OFF + s * C::OP_STAGE;
                    const uint32_t b_addr = a_addr + BM * OP_ROW;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t acc = (ko > 0 || k > 0);
                        const uint64_t ad = sw128_kmajor_desc(a_addr + 32 * k);
                        const uint64_t bd = sw128_kmajor_desc(b_addr + 32 * k);
                        if (C::OUT_INT8)
                            mma_i8(d, ad, bd, id_i8, acc);
                        else
                            mma_f16(d, ad, bd, id_f16, acc);
                    }
                    mma_commit(&op_empty[s]);
                }
                if (C::GROUPED && ok) mma_commit(&acc_full[b]);
            }
            if (!C::GROUPED) mma_commit(&acc_full[0]);
            // all MMAs issued by this thread have finished before TMEM is freed
            mma_commit(&mma_done);
            mbar_wait_bounded(&mma_done, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp < 2 + NT) {
        // ------------------------------------------------------------ unpack INT4 -> INT8
        // These warps fill every operand stage in k-block order (unpacked INT4
        // k-blocks, then the outlier k-blocks by TMA), so each of their waits
        // is for the current or the previous phase of its barrier, the
        // condition under which a parity wait is exact.
        const int t = threadIdx.x - 64;
        int last_op[SU];
        for (int s = 0; s < SU; ++s) last_op[s] = -1;
        if (t == 0 && p.nkb_o > 0) {
            tma_prefetch_desc(&tm_xo);
            tma_prefetch_desc(&tm_wo);
        }
        for (int kb = 0; kb < p.nkb_i + p.nkb_o; ++kb) {
            const int sp = kb % SP, su = kb % SU;
            if (kb >= p.nkb_i) {
                // outlier k-block: 64 fp16 (or 128 int8) channels = 128 bytes per row
                const bool ok = wait_bar(&op_empty[su], ((kb / SU) & 1) ^ 1, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) break;
                if (lane == 0) {
                    if (t == 0) {
                        const int ko = kb - p.nkb_i;
                        const int x = C::OUT_INT8 ? ko * 128 : ko * 64;
                        uint8_t *dst = smem + C::OP_OFF + su * C::OP_STAGE;
                        mbar_arrive_expect_tx(&op_full[su], C::OP_STAGE);
                        tma_load_2d(dst, &tm_xo, x, m0, &op_full[su]);
                        tma_load_2d(dst + BM * OP_ROW, &tm_wo, x, n0, &op_full[su]);
                        last_op[su] = kb;
                    } else {
                        mbar_arrive(&op_full[su]);
                    }
                }
                __syncwarp();
                continue;
            }
            bool ok = wait_bar(&pk_full[sp], (kb / SP) & 1, abort_flag) &&
                      wait_bar(&op_empty[su], ((kb / SU) & 1) ^ 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (t == 0) QUIK_TRACE_AT(1, kb);
            const uint8_t *pk = smem + C::PK_OFF + sp * C::PK_STAGE;
            uint8_t *op = smem + C::OP_OFF + su * C::OP_STAGE;
#pragma unroll
            for (int i = 0; i < C::CHUNKS_PER_THREAD; ++i) {
                // A rows [0, BM) then B rows [BM, BM+BN): one matrix of BM+BN rows
                const int c = t + i * NT * 32;
                const int r = c >> 2, ch = c & 3;
                if (!QUIK_CHECK(r < BM + C::BN && t >= 0 && t < NT * 32, 10)) continue;
                const uint4 v = *reinterpret_cast<const uint4 *>(pk + r * PK_ROW + ch * 16);
                uint4 lo, hi;
                lo.x = (v.x << 4) & 0xF0F0F0F0u;  hi.x = v.x & 0xF0F0F0F0u;
                lo.y = (v.y << 4) & 0xF0F0F0F0u;  hi.y = v.y & 0xF0F0F0F0u;
                lo.z = (v.z << 4) & 0xF0F0F0F0u;  hi.z = v.z & 0xF0F0F0F0u;
                lo.w = (v.w << 4) & 0xF0F0F0F0u;  hi.w = v.w & 0xF0F0F0F0u;
                uint8_t *row = op + r * OP_ROW;
                *reinterpret_cast<uint4 *>(row + (((2 * ch) ^ (r & 7)) << 4)) = lo;
                *reinterpret_cast<uint4 *>(row + (((2 * ch + 1) ^ (r & 7)) << 4)) = hi;
            }
            fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&pk_empty[sp]);
                mbar_arrive(&op_full[su]);
            }
            if (t == 0) QUIK_TRACE_AT(2, kb);
        }
        // never leave the CTA with a bulk copy still writing its shared memory
        if (t == 0)
            for (int s = 0; s < SU; ++s)
                if (last_op[s] >= 0) mbar_wait_bounded(&op_full[s], (last_op[s] / SU) & 1, kWaitLimitNs);
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - (2 + NT);
        const int q = warp & 3;  // TMEM lanes [32q, 32q+32) are this warp's
        const int col0 = (ew >> 2) * C::EPI_COLS;
        const int row = m0 + q * 32 + lane;
        const bool row_ok = row < p.M;
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        float *ssw = epi_sw[ew];

        if (!C::GROUPED) {
            // this warp's per-column weight scales, loaded before the accumulator is ready
            for (int c = lane; c < C::EPI_COLS; c += 32) {
                const int n = n0 + col0 + c;
                ssw[c] = (n < p.N && p.Ki > 0) ? p.sw[n] : 0.0f;
            }
            __syncwarp();
            bool ok = wait_bar(&acc_full[0], 0, abort_flag);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                if (ew == 0 && lane == 0) QUIK_TRACE_AT(4, 0);
                const float sxr = (row_ok && p.Ki > 0 && QUIK_CHECK(row < p.M, 15)) ? p.sx[row] : 0.0f;
                const float sxo = (row_ok && C::OUT_INT8 && p.nkb_o > 0) ? p.sxo[row] : 0.0f;
                for (int cc = 0; cc < C::EPI_COLS; cc += 32) {
                    const int nb = n0 + col0 + cc;
                    uint32_t a[32], o[32];
                    if (p.Ki > 0) tmem_ld_32x32b_x32(t_lane + col0 + cc, a);
                    if (p.nkb_o > 0) tmem_ld_32x32b_x32(t_lane + BN + col0 + cc, o);
                    tmem_ld_wait();
                    if (C::DEBUG) {
                        if (row_ok) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int n = nb + j;
                                if (n < p.N) {
                                    if (p.Ki > 0)
                                        p.acc_dbg[(size_t)row * p.N + n] = static_cast<int32_t>(a[j]) >> 8;
                                    if (C::OUT_INT8 && p.nkb_o > 0 && p.acc_o_dbg)
                                        p.acc_o_dbg[(size_t)row * p.N + n] = static_cast<int32_t>(o[j]);
                                }
                            }
                        }
                        continue;
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float y[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int jj = j + h, n = nb + jj;
                            float v = 0.0f;
                            if (p.Ki > 0)
                                v = small_int_to_float(static_cast<int32_t>(a[jj]) >> 8) * sxr * ssw[cc + jj];
                            if (p.nkb_o > 0) {
                                if (C::OUT_INT8) {
                                    const float swo = n < p.N ? __ldg(p.swo + n) : 0.0f;
                                    v += static_cast<float>(static_cast<int32_t>(o[jj])) * sxo * swo;
                                } else {
                                    v += __uint_as_float(o[jj]);
                                }
                            }
                            if (p.bias != nullptr && n < p.N)
                                v += __half2float(__ushort_as_half(__ldg(p.bias + n)));
                            y[h] = v;
                        }
                        packed[j / 2] = pack_half2(y[0], y[1]);
                    }
                    if (row_ok) {
                        uint16_t *yrow = p.Y + (size_t)row * p.N;
                        if (nb + 32 <= p.N && (p.N & 7) == 0) {
                            uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                            for (int v4 = 0; v4 < 4; ++v4)
                                dst[v4] = make_uint4(packed[4 * v4], packed[4 * v4 + 1],
                                                     packed[4 * v4 + 2], packed[4 * v4 + 3]);
                        } else {
                            for (int j = 0; j < 32; ++j)
                                if (nb + j < p.N)
                                    yrow[nb + j] = static_cast<uint16_t>(packed[j / 2] >> (16 * (j & 1)));
                        }
                    }
                    __syncwarp();
                }
                tc_fence_before();
                if (ew == 0 && lane == 0) QUIK_TRACE_AT(5, 0);
            }
        } else {
            // grouped: running fp32 sums of this warp's EPI_COLS columns, in registers
            float ysum[C::EPI_COLS];
#pragma unroll
            for (int j = 0; j < C::EPI_COLS; ++j) ysum[j] = 0.0f;
            bool ok = true;
            for (int g = 0; g < p.nkb_i && ok; ++g) {
                const int b = g % C::NACC;
                // stage this group's weight scales for the warp's columns
#pragma unroll
                for (int cc = 0; cc < C::EPI_COLS; cc += 32) {
                    const int n = n0 + col0 + cc + lane;
                    ssw[cc + lane] = (n < p.N && QUIK_CHECK(g < p.G && cc + lane < C::EPI_COLS, 16))
                                         ? p.sw[(size_t)n * p.G + g] : 0.0f;
                }
                // fold the 16 x 16 operand scaling (2^-8) into the row factor
                const float sxg = (row_ok && QUIK_CHECK(g < p.G, 15))
                                      ? p.sx[(size_t)row * p.G + g] * (1.0f / 256.0f) : 0.0f;
                __syncwarp();
                ok = wait_bar(&acc_full[b], (g / C::NACC) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < C::EPI_COLS; cc += 32) {
                    uint32_t a[32];
                    (void)QUIK_CHECK(b * BN + col0 + cc + 32 <= C::TMEM_COLS, 14);
                    tmem_ld_32x32b_x32(t_lane + b * BN + col0 + cc, a);
                    tmem_ld_wait();
                    if (C::DEBUG) {
                        if (row_ok)
                            for (int j = 0; j < 32; ++j) {
                                const int n = n0 + col0 + cc + j;
                                if (n < p.N)
                                    p.acc_dbg[((size_t)g * p.M + row) * p.N + n] =
                                        static_cast<int32_t>(a[j]) >> 8;
                            }
                        continue;
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float f = small_int_to_float(static_cast<int32_t>(a[j])) * ssw[cc + j];
                        ysum[cc + j] = fmaf(f, sxg, ysum[cc + j]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            if (ok && p.nkb_o > 0) {
                const int b = p.nkb_i % C::NACC;
                ok = wait_bar(&acc_full[b], (p.nkb_i / C::NACC) & 1, abort_flag);
                if (__all_sync(0xffffffffu, ok)) {
                    tc_fence_after();
                    const float sxo = (row_ok && C::OUT_INT8) ? p.sxo[row] : 0.0f;
#pragma unroll
                    for (int cc = 0; cc < C::EPI_COLS; cc += 32) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(t_lane + b * BN + col0 + cc, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int n = n0 + col0 + cc + j;
                            if (C::DEBUG) {
                                if (C::OUT_INT8 && row_ok && n < p.N && p.acc_o_dbg)
                                    p.acc_o_dbg[(size_t)row * p.N + n] = static_cast<int32_t>(o[j]);
                            } else if (C::OUT_INT8) {
                                const float swo = n < p.N ? __ldg(p.swo + n) : 0.0f;
                                ysum[cc + j] += static_cast<float>(static_cast<int32_t>(o[j])) * sxo * swo;
                            } else {
                                ysum[cc + j] += __uint_as_float(o[j]);
                            }
                        }
                    }
                    tc_fence_before();
                } else {
                    ok = false;
                }
            }
            if (ok && !C::DEBUG && row_ok) {
                uint16_t *yrow = p.Y + (size_t)row * p.N;
#pragma unroll
                for (int cc = 0; cc < C::EPI_COLS; cc += 32) {
                    const int nb = n0 + col0 + cc;
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float y0 = ysum[cc + j], y1 = ysum[cc + j + 1];
                        if (p.bias != nullptr) {
                            if (nb + j < p.N) y0 += __half2float(__ushort_as_half(__ldg(p.bias + nb + j)));
                            if (nb + j + 1 < p.N) y1 += __half2float(__ushort_as_half(__ldg(p.bias + nb + j + 1)));
                        }
                        packed[j / 2] = pack_half2(y0, y1);
                    }
                    if (nb + 32 <= p.N && (p.N & 7) == 0) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(packed[4 * v4], packed[4 * v4 + 1], packed[4 * v4 + 2],
                                                 packed[4 * v4 + 3]);
                    } else {
                        for (int j = 0; j < 32; ++j)
                            if (nb + j < p.N)
                                yrow[nb + j] = static_cast<uint16_t>(packed[j / 2] >> (16 * (j & 1)));
                    }
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) QUIK_TRACE_AT(7, 0);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

__device__ __forceinline__ void unpack16(const uint4 v, uint4 &lo, uint4 &hi) {
    lo.x = (v.x << 4) & 0xF0F0F0F0u;  hi.x = v.x & 0xF0F0F0F0u;
    lo.y = (v.y << 4) & 0xF0F0F0F0u;  hi.y = v.y & 0xF0F0F0F0u;
    lo.z = (v.z << 4) & 0xF0F0F0F0u;  hi.z = v.z & 0xF0F0F0F0u;
    lo.w = (v.w << 4) & 0xF0F0F0F0u;  hi.w = v.w & 0xF0F0F0F0u;
}

// ============================================================================
// Per-channel-scale kernel on a CTA pair (cta_group::2), activations in
// tensor memory.
//
// Two CTAs of a cluster share one 256 x 256 output tile.  Each holds 128 rows
// of A and of the output, and half of B (128 of the 256 columns) in its
// shared memory; the leader issues tcgen05.mma.cta_group::2 with M = 256,
// which reads both halves.  The A rows never touch shared memory: A threads
// load their row's packed codes from global memory (several k-blocks ahead),
// unpack in registers and write tensor memory with tcgen05.st; the MMA reads
// A from TMEM.  Only B goes through shared memory: per k-block and SM, TMA
// staging 8 KB, read back 8 KB, unpacked 16 KB, MMA read 16 KB.  (With one
// CTA per 128 x 256 tile that is 96 KB per k-block, which bounds the kernel
// by shared-memory bandwidth.)  The B unpack warps keep no global loads in
// flight, so the proxy fence that publishes their stores to the MMA only
// waits for their own shared-memory stores.
//
// Peer warps signal the leader's "operand full" barriers with remote mbarrier
// arrivals on cluster addresses (the instruction's default semantics, as in
// CUTLASS's two-SM pipelines; an explicit release at cluster scope measured
// 1.6x slower end to end); MMA completion reaches both CTAs through a
// multicast commit.
//
//   warp 0        TMEM allocator (both CTAs); the leader's lane 0 issues the MMAs
//   warp 1        TMA producer of the packed staging ring, in unit order:
//                 one unit per INT4 k-block (this CTA's 128 rows of the B
//                 tile), two per outlier k-block (Wo rows, then Xo rows)
//   warps 2-5     A: one thread per tile row (= its TMEM lane): load, unpack,
//                 tcgen05.st 32 columns per k-block; then the epilogue
//   warps 6-13    B: staging -> 128-byte swizzled K-major operand stage
//                 (unpacked INT4 k-blocks; copied outlier tiles)
// TMEM (each CTA): INT32 sums in columns [0,256); A stages [256, 256+32 S)
// while the INT4 k-blocks run; after them (and a drain of the MMA pipe) the
// outlier sums in [256, 512), with both outlier operands in shared memory.
namespace pair {
constexpr int BN = 256;                   // pair tile columns (each CTA holds BN/2 of B)
constexpr int BNH = BN / 2;
constexpr int S = 4;                      // operand stages
constexpr int SP = 4;                     // packed staging stages
constexpr int NA = 4, NB = 8;  // A warps, B warps (per CTA)
constexpr int THREADS = (2 + NA + NB) * 32;
constexpr int B_BYTES = BNH * OP_ROW;     // this CTA's unpacked half of B / outlier W rows
constexpr int XO_BYTES = BM * OP_ROW;     // outlier X tile (this CTA's 128 rows)
constexpr int STAGE = B_BYTES + XO_BYTES;
constexpr int UNIT = BM * OP_ROW;         // staging unit: 16 KB
constexpr int PK_OFF = S * STAGE;
constexpr int SMEM = PK_OFF + SP * UNIT + 1024;
constexpr int ACC_COL = 0, A_COL = 256, O_COL = 256, TMEM_COLS = 512;
constexpr int PF = 4;                     // k-blocks of A loads in flight per thread
static_assert(NA == 4 && NB == 8, "the epilogue splits each lane quadrant's 8 column chunks 3 / 3 / 2");
static_assert(STAGE % 1024 == 0 && B_BYTES % 1024 == 0, "128-byte-swizzled staging blocks");
static_assert(XO_BYTES == 128 * 128 && S * 64 >= BN, "the output tile stages in the stages' outlier-X areas");
static_assert(A_COL + 32 * S <= TMEM_COLS, "A stages fit in tensor memory");
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace pair

template <bool OUT_INT8, bool DEBUG, bool A8, bool W8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::THREADS, 1)
    w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_wq,
                          const __grid_constant__ CUtensorMap tm_wo,
                          const __grid_constant__ CUtensorMap tm_xo,
                          const __grid_constant__ CUtensorMap tm_y,
                          const uint8_t *__restrict__ Xq, const GemmParams p) {
    using namespace pair;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t op_full[S], op_empty[S], pk_full[SP], pk_empty[SP];
    __shared__ uint64_t acc_full, drain, mma_done;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;
    __shared__ __align__(16) float col_sw[BN], col_swo[BN], col_bias[BN];

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();     // 0 = leader
    const int m0 = blockIdx.y * 2 * BM + rank * BM;  // this CTA's A / output rows
    const int n0 = (blockIdx.x >> 1) * BN;           // the pair's output columns
    const int nb0 = n0 + rank * BNH;                 // this CTA's rows of W (half of B)
    const int nkb = p.nkb_i + p.nkb_o;
    const int nunits = p.nkb_i + 2 * p.nkb_o;        // staging units
    const int rb = A8 ? p.Ki : p.Ki / 2;             // bytes of an Xq row

    if (threadIdx.x == 0) {
        QUIK_TRACE_AT(6, 0);
        for (int st = 0; st < S; ++st) {
            mbar_init(&op_full[st], 2 * (NA + NB));  // used in the leader only
            mbar_init(&op_empty[st], 1);
        }
        for (int st = 0; st < SP; ++st) {
            mbar_init(&pk_full[st], 1);
            mbar_init(&pk_empty[st], NB);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&drain, 1);
        mbar_init(&mma_done, 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_error_word);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barrier initialisation and TMEM allocation visible to both CTAs
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const AbortState ab{&abort_s, err0_s};
    // the leader's "operand full" barriers, as cluster addresses
    auto leader_full = [&](int st) { return mapa_shared(smem_u32(&op_full[st]), 0); };

    if (warp == 0) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0) {
            const uint32_t id_i8 = idesc_s8_s32(2 * BM, BN);
            const uint32_t id_f16 = idesc_f16_f32(2 * BM, BN);
            bool ok = true;
            for (int kb = 0; kb < p.nkb_i && ok; ++kb) {
                const int st = kb % S;
                if (!(ok = wait_bar(&op_full[st], (kb / S) & 1, ab))) break;
                tc_fence_after();
                QUIK_TRACE_AT(3, kb);
                const uint32_t b_addr = smem_base + st * STAGE;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma2_i8_ts(tmem + ACC_COL, tmem + A_COL + 32 * st + 8 * k,
                               sw128_kmajor_desc(b_addr + 32 * k), id_i8, (kb > 0 || k > 0));
                mma2_commit_both(&op_empty[st]);
            }
            if (ok && p.nkb_o > 0) {
                if (p.nkb_i > 0) {
                    // the outlier sums overwrite the A-stage columns: every INT4
                    // MMA finishes reading them first
                    mma2_commit_local(&drain);
                    ok = wait_bar(&drain, 0, ab);
                }
                for (int kb = p.nkb_i; kb < nkb && ok; ++kb) {
                    const int st = kb % S, ko = kb - p.nkb_i;
                    if (!(ok = wait_bar(&op_full[st], (kb / S) & 1, ab))) break;
                    tc_fence_after();
                    const uint32_t b_addr = smem_base + st * STAGE;
                    const uint32_t a_addr = b_addr + B_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = sw128_kmajor_desc(a_addr + 32 * k);
                        const uint64_t bd = sw128_kmajor_desc(b_addr + 32 * k);
                        if (OUT_INT8)
                            mma2_i8(tmem + O_COL, ad, bd, id_i8, (ko > 0 || k > 0));
                        else
                            mma2_f16(tmem + O_COL, ad, bd, id_f16, (ko > 0 || k > 0));
                    }
                    mma2_commit_both(&op_empty[st]);
                }
            }
            mma2_commit_both(&acc_full);
            mma2_commit_local(&mma_done);
            mbar_wait_bounded(&mma_done, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMA producer (each CTA)
        if (lane == 0) {
            if (p.nkb_i > 0) tma_prefetch_desc(&tm_wq);
            if (p.nkb_o > 0) {
                tma_prefetch_desc(&tm_wo);
                tma_prefetch_desc(&tm_xo);
            }
            int last[SP];
            for (int st = 0; st < SP; ++st) last[st] = -1;
            for (int u = 0; u < nunits; ++u) {
                const int st = u % SP;
                if (!wait_bar(&pk_empty[st], ((u / SP) & 1) ^ 1, ab)) break;
                uint8_t *dst = smem + PK_OFF + st * UNIT;
                QUIK_TRACE_AT(11, u);
                if (u < p.nkb_i) {  // this CTA's 128 rows of the B tile (packed, or INT8 codes)
                    constexpr int WB = W8 ? OP_ROW : PK_ROW;
                    mbar_arrive_expect_tx(&pk_full[st], BNH * WB);
                    tma_load_2d(dst, &tm_wq, u * WB, nb0, &pk_full[st]);
                } else {
                    const int v = u - p.nkb_i, ko = v / 2;
                    if (v == 0) grid_dependency_wait();  // Xo comes from the previous kernel
                    mbar_arrive_expect_tx(&pk_full[st], UNIT);
                    if (v % 2 == 0)  // this CTA's 128 rows of Wo, 128 bytes each
                        tma_load_2d(dst, &tm_wo, ko * OP_ROW, nb0, &pk_full[st]);
                    else             // this CTA's 128 rows of Xo
                        tma_load_2d(dst, &tm_xo, ko * OP_ROW, m0, &pk_full[st]);
                }
                last[st] = u;
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            for (int st = 0; st < SP; ++st)
                if (last[st] >= 0) mbar_wait_bounded(&pk_full[st], (last[st] / SP) & 1, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // A warps (TMEM operand) and B warps (shared-memory operand) feed the
        // MMA, then all 12 run the epilogue
        bool ok = true;
        if (warp < 2 + NA) {
            // ------------------------------------------------------------ A rows -> TMEM (each CTA)
            const int q = warp & 3;
            const int r = q * 32 + lane;  // tile row = TMEM lane
            const int grow = m0 + r;
            const bool row_ok = grow < p.M;
            const uint8_t *xrow = Xq + (size_t)grow * rb;
            const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
            // a k-block of a row: 4 chunks of 16 packed bytes, or 8 of INT8 codes
            constexpr int CH = A8 ? 8 : 4, KB_BYTES = A8 ? OP_ROW : PK_ROW, PFA = A8 ? PF / 2 : PF;
            uint4 buf[PFA][CH];
            grid_dependency_wait();  // Xq (and later sx) come from the previous kernel
            auto load = [&](int kb, uint4(&d)[CH]) {
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int off = kb * KB_BYTES + c * 16;
                    d[c] = (row_ok && off < rb) ? ldg_nc_v4(xrow + off) : make_uint4(0, 0, 0, 0);
                }
            };
#pragma unroll
            for (int j = 0; j < PFA; ++j)
                if (j < p.nkb_i) load(j, buf[j]);
            for (int kb0 = 0; kb0 < p.nkb_i && ok; kb0 += PFA) {
#pragma unroll
                for (int j = 0; j < PFA; ++j) {
                    const int kb = kb0 + j;
                    if (kb >= p.nkb_i || !ok) break;
                    const int st = kb % S;
                    ok = wait_bar(&op_empty[st], ((kb / S) & 1) ^ 1, ab);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    uint32_t w[32];
                    if constexpr (A8 && W8) {  // both sides in code order
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            w[4 * c + 0] = buf[j][c].x; w[4 * c + 1] = buf[j][c].y;
                            w[4 * c + 2] = buf[j][c].z; w[4 * c + 3] = buf[j][c].w;
                        }
                    } else if constexpr (A8) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) order_i8_chunk(buf[j][2 * c], buf[j][2 * c + 1], w + 8 * c);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint4 lo, hi;
                            unpack16(buf[j][c], lo, hi);
                            w[8 * c + 0] = lo.x; w[8 * c + 1] = lo.y; w[8 * c + 2] = lo.z; w[8 * c + 3] = lo.w;
                            w[8 * c + 4] = hi.x; w[8 * c + 5] = hi.y; w[8 * c + 6] = hi.z; w[8 * c + 7] = hi.w;
                        }
                    }
                    tmem_st_32x32b_x32(t_lane + A_COL + 32 * st, w);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(leader_full(st));
    #ifdef QUIK_TRACE
                    if (lane == 0 && blockIdx.x + blockIdx.y * gridDim.x < kTraceCtas && kb < kTraceKb)
                        atomicMax(&g_trace[blockIdx.x + blockIdx.y * gridDim.x][2][kb], clock64());
    #endif
                    if (kb + PFA < p.nkb_i) load(kb + PFA, buf[j]);
                }
            }
            // outlier k-blocks: both operands arrive through shared memory
            for (int kb = p.nkb_i; kb < nkb && ok; ++kb) {
                const int st = kb % S;
                ok = wait_bar(&op_empty[st], ((kb / S) & 1) ^ 1, ab);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                if (lane == 0) mbar_arrive_remote(leader_full(st));
            }

        } else {
            // ------------------------------------------------------------ B half: staging -> operand stage
            const int tb = threadIdx.x - 32 * (2 + NA);  // 0 .. 32*NB-1
            int u = 0;
            for (int kb = 0; kb < nkb && ok; ++kb) {
                const int st = kb % S;
                ok = wait_bar(&op_empty[st], ((kb / S) & 1) ^ 1, ab);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                uint8_t *bst = smem + st * STAGE;
                if (tb == 0) QUIK_TRACE_AT(1, kb);
                const int nparts = kb < p.nkb_i ? 1 : 2;
                for (int part = 0; part < nparts && ok; ++part, ++u) {
                    const int ps = u % SP;
                    ok = wait_bar(&pk_full[ps], (u / SP) & 1, ab);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    if (tb == 0 && part == 0) QUIK_TRACE_AT(8, kb);
                    const uint8_t *pk = smem + PK_OFF + ps * UNIT;
                    if (kb < p.nkb_i && !W8) {
                        // 128 rows x 4 chunks: unpack each 16-byte chunk into two
                        const int ch = tb & 3;
#pragma unroll
                        for (int i = 0; i < 128 / (8 * NB); ++i) {
                            const int row = tb / 4 + 8 * NB * i;
                            const uint4 v = *reinterpret_cast<const uint4 *>(pk + row * PK_ROW + ch * 16);
                            uint4 lo, hi;
                            unpack16(v, lo, hi);
                            uint8_t *rp = bst + row * OP_ROW;
                            *reinterpret_cast<uint4 *>(rp + (((2 * ch) ^ (row & 7)) << 4)) = lo;
                            *reinterpret_cast<uint4 *>(rp + (((2 * ch + 1) ^ (row & 7)) << 4)) = hi;
                        }
                    } else {
                        // INT8 weight rows and Wo rows (part 0) into the B area, Xo rows
                        // (part 1) into the A area: 128 rows x 8 chunks each
                        const int c = tb & 7;
                        uint8_t *dst = part == 0 ? bst : bst + B_BYTES;
#pragma unroll
                        for (int i = 0; i < 32 / NB; ++i) {
                            const int row = tb / 8 + 4 * NB * i;
                            const uint4 v = *reinterpret_cast<const uint4 *>(pk + row * OP_ROW + c * 16);
                            *reinterpret_cast<uint4 *>(dst + row * OP_ROW + ((c ^ (row & 7)) << 4)) = v;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pk_empty[ps]);
                }
                if (!ok) break;
                if (tb == 0) QUIK_TRACE_AT(9, kb);
                fence_proxy_async_smem();  // generic-proxy stores -> visible to the pair's MMA
                if (tb == 0) QUIK_TRACE_AT(10, kb);
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(leader_full(st));
    #ifdef QUIK_TRACE
                if (lane == 0 && blockIdx.x + blockIdx.y * gridDim.x < kTraceCtas && kb < kTraceKb)
                    atomicMax(&g_trace[blockIdx.x + blockIdx.y * gridDim.x][0][kb], clock64());
    #endif
            }
        }

        // ------------------------------------------------------------ epilogue (each CTA)
        // The 12 A and B warps: each on its TMEM lane quadrant (warp % 4) and a
        // third of the 256 columns (32-column chunks 0-2 / 3-5 / 6-7).  With
        // tma_y the fp16 tile is staged, 128-byte swizzled, in the four stages'
        // outlier-X areas (64 columns each; every MMA has finished reading them)
        // and leaves by TMA stores; else each thread stores its row directly.
        grid_dependency_wait();           // sx and sxo come from the previous kernel
        const int ep = threadIdx.x - 64;  // 0 .. 32 * (NA + NB) - 1
        for (int c = ep; c < BN; c += 32 * (NA + NB)) {
            const int n = n0 + c;
            const bool in = n < p.N;
            col_sw[c] = (in && p.Ki > 0) ? p.sw[n] : 0.0f;
            col_swo[c] = (in && OUT_INT8 && p.nkb_o > 0) ? p.swo[n] : 0.0f;
            col_bias[c] = (in && p.bias != nullptr) ? __half2float(__ushort_as_half(p.bias[n])) : 0.0f;
        }
        named_barrier_sync(1, 32 * (NA + NB));
        ok = ok && wait_bar(&acc_full, 0, ab);
        if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            if (warp == 3 && lane == 0) QUIK_TRACE_AT(4, 0);
            const int q = warp & 3;
            const int wq = warp < 2 + NA ? 0 : warp < 6 + NA ? 1 : 2;  // A, first or second B warp
            const int ch_lo = wq == 0 ? 0 : wq == 1 ? 3 : 6, ch_hi = wq == 0 ? 3 : wq == 1 ? 6 : 8;
            const int r = q * 32 + lane;  // tile row = TMEM lane
            const int grow = m0 + r;
            const bool row_ok = grow < p.M;
            const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
            const float sxr = (row_ok && p.Ki > 0) ? p.sx[grow] : 0.0f;
            const float sxo = (row_ok && OUT_INT8 && p.nkb_o > 0) ? p.sxo[grow] : 0.0f;
            uint16_t *yrow = p.Y + (size_t)grow * p.N;
            for (int ch = ch_lo; ch < ch_hi; ++ch) {
                const int cc = ch * 32, nb = n0 + cc;
                uint32_t a[32], o[32];
                if (p.Ki > 0) tmem_ld_32x32b_x32(t_lane + ACC_COL + cc, a);
                if (p.nkb_o > 0) tmem_ld_32x32b_x32(t_lane + O_COL + cc, o);
                tmem_ld_wait();
                if (DEBUG) {
                    if (row_ok) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int n = nb + jj;
                            if (n < p.N) {
                                if (p.Ki > 0)
                                    p.acc_dbg[(size_t)grow * p.N + n] = acc_int<A8, W8>(a[jj]);
                                if (OUT_INT8 && p.nkb_o > 0 && p.acc_o_dbg)
                                    p.acc_o_dbg[(size_t)grow * p.N + n] = static_cast<int32_t>(o[jj]);
                            }
                        }
                    }
                    continue;
                }
                uint32_t packed[16];
#pragma unroll
                for (int jj = 0; jj < 32; jj += 2) {
                    float y[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = cc + jj + h;
                        float v = acc_float<A8, W8>(a[jj + h]) * sxr * col_sw[c];
                        if (p.Ki == 0) v = 0.0f;
                        if (p.nkb_o > 0) {
                            if (OUT_INT8)
                                v += static_cast<float>(static_cast<int32_t>(o[jj + h])) * sxo * col_swo[c];
                            else
                                v += __uint_as_float(o[jj + h]);
                        }
                        y[h] = v + col_bias[c];
                    }
                    packed[jj / 2] = pack_half2(y[0], y[1]);
                }
                if (p.tma_y) {
                    // 64-column block ch/2 lives in stage (ch/2)'s outlier-X area
                    uint8_t *blk = smem + (ch >> 1) * STAGE + B_BYTES + r * 128;
                    const int c16 = (ch & 1) * 4;
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        *reinterpret_cast<uint4 *>(blk + (((c16 + v4) ^ (r & 7)) << 4)) =
                            make_uint4(packed[4 * v4], packed[4 * v4 + 1], packed[4 * v4 + 2], packed[4 * v4 + 3]);
                } else if (row_ok) {
                    if (nb + 32 <= p.N && (p.N & 7) == 0) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + nb);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(packed[4 * v4], packed[4 * v4 + 1],
                                                 packed[4 * v4 + 2], packed[4 * v4 + 3]);
                    } else {
                        for (int jj = 0; jj < 32; ++jj)
                            if (nb + jj < p.N)
                                yrow[nb + jj] = static_cast<uint16_t>(packed[jj / 2] >> (16 * (jj & 1)));
                    }
                }
            }
            tc_fence_before();
            if (p.tma_y) fence_proxy_async_smem();  // staged tile -> visible to the TMA stores
            if (warp == 3 && lane == 0) QUIK_TRACE_AT(5, 0);
        }
        named_barrier_sync(1, 32 * (NA + NB));  // tile staged
        if (threadIdx.x == 32 * (2 + NA) && p.tma_y && ok && m0 < p.M) {
            for (int b = 0; b < BN / 64; ++b)
                if (n0 + 64 * b < p.N) tma_store_2d(&tm_y, smem + b * STAGE + B_BYTES, n0 + 64 * b, m0);
            bulk_commit_group();
            bulk_wait_group0();  // the stores complete before the CTA leaves
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs or remote arrivals may touch it
    if (threadIdx.x == 0) QUIK_TRACE_AT(7, 0);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// ============================================================================
// Decode-shaped product: M <= 32 tokens, per-channel scales, k_o <= 256.
//
// With a few tokens the layer is bound by reading W (N x K_i / 2 bytes), and a
// 128-row token tile would leave most MMA rows empty.  Here the operands swap:
// the MMA computes D[n, m] = sum_k W'[n,k] X'[m,k] with W as its 128-row A
// operand and the tokens as its N (16 or 32), so no MMA row is idle.  One CTA
// owns 128 rows of W:
//   warp 0       TMEM allocator; lane 0 issues the MMAs: first the outlier
//                block (kind::f16, or kind::i8 for INT8 outliers; both
//                operands by TMA in the 128-byte-swizzled layout), then the
//                INT4 k-blocks (kind::i8, A from tensor memory)
//   warp 1       TMA producer: the outlier tiles once; then per k-block one
//                unit of the packed W tile (128 rows x 64 bytes, 64-byte
//                swizzle) and the packed token rows (32 x 64 bytes), in a
//                10-deep ring
//   warps 2-17   W, four groups of four warps taking k-blocks in turn (group
//                g owns operand stage g, so four k-blocks are in flight; one
//                group alone spends ~750 dependent cycles per k-block): row r
//                = TMEM lane r reads its 64 packed bytes (the swizzle keeps
//                the reads conflict-free), unpacks them and writes tensor
//                memory; the group also unpacks the k-block's token rows into
//                the 128-byte-swizzled X stage.  They keep no global loads in
//                flight, so the proxy fence that publishes the X stage waits
//                only for their own shared-memory stores.  Group 0 runs the
//                epilogue, which writes Y[m, n] for fixed m across the lanes
//                (coalesced).
namespace gemv {
constexpr int BW = 128;                      // W rows per CTA = TMEM lanes
constexpr int MT = kDecodeTokens;            // most tokens (the MMA's N: 16 or 32)
#ifndef QUIK_GEMV_S
#define QUIK_GEMV_S 8
#endif
#ifndef QUIK_GEMV_NI
#define QUIK_GEMV_NI 2
#endif
constexpr int S = QUIK_GEMV_S;               // operand stages (A in TMEM, X in shared memory)
#ifndef QUIK_GEMV_SPW
#define QUIK_GEMV_SPW 10
#endif
constexpr int SPW = QUIK_GEMV_SPW;           // staging units
constexpr int WUNIT = BW * PK_ROW;           // 8 KB of packed W
constexpr int XUNIT = MT * PK_ROW;           // 2 KB of packed token rows (MP rows are loaded)
constexpr int XSTAGE = MT * OP_ROW;          // 4 KB
constexpr int OKB = 2;                       // outlier k-blocks of 128-byte rows:
constexpr int KO_MAX_F16 = 64 * OKB;         //   k_o <= 128 fp16 channels
constexpr int KO_MAX_I8 = 128 * OKB;         //   or 256 int8 channels
constexpr int WO_TILE = BW * OP_ROW;         // 16 KB: 128 rows x 128 bytes
constexpr int XO_TILE = MT * OP_ROW;         // 4 KB
constexpr int NG = 4;                        // W warp groups (4 warps each)
constexpr int NW = 4 * NG;                   // W warps
constexpr int NI = QUIK_GEMV_NI;             // MMA issuers, each with its own accumulator
constexpr int THREADS = (1 + NW + NI) * 32;
constexpr int XU_OFF = SPW * WUNIT;          // W staging first, then the token-row staging
constexpr int X_OFF = XU_OFF + SPW * XUNIT;
constexpr int WO_OFF = X_OFF + S * XSTAGE;
constexpr int XO_OFF = WO_OFF + OKB * WO_TILE;
constexpr int SMEM = XO_OFF + OKB * XO_TILE + 1024;  // + alignment
constexpr int ACC_COL = 0, O_COL = 32 * NI, A_COL = O_COL + 32;  // one accumulator per issuer
constexpr int TMEM_COLS = A_COL + 32 * S <= 256 ? 256 : 512;
static_assert(A_COL + 32 * S <= TMEM_COLS, "A stages fit in tensor memory");
static_assert(S % NG == 0, "group g owns operand stages g, g + NG, ...");
static_assert(S % NI == 0, "each stage belongs to one issuer");
static_assert(X_OFF % 1024 == 0 && WO_OFF % 1024 == 0 && XO_OFF % 1024 == 0, "128-byte-swizzled tiles");
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace gemv

template <bool OUT_INT8, bool DEBUG>
__global__ void __launch_bounds__(gemv::THREADS, 1)
    w4a4_gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_wo, const __grid_constant__ CUtensorMap tm_xo,
                     const GemmParams p) {
    using namespace gemv;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t w_full[SPW], w_empty[SPW], op_full[S], op_empty[S], o_full, acc_full, mma_done[NI];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BW;
    const int MP = p.M <= 16 ? 16 : 32;  // the MMA's N
    const int nkb = p.nkb_i;
    // outlier k-blocks of 128 bytes: 64 fp16 or 128 int8 channels each
    const int oke = OUT_INT8 ? 128 : 64;
    const int nko = (p.k_o + oke - 1) / oke;

    const int early = nkb < SPW ? nkb : SPW;  // W units loaded before the CTA barrier
    if (threadIdx.x == 0) QUIK_TRACE_AT(6, 0);
    if (warp == 1 && lane == 0) {
        // The producer's barriers, and the first ring of W tiles at once: W
        // is not the previous kernel's output, and the first tiles' DRAM
        // latency then overlaps the rest of the set-up.  Their token rows
        // (and the tokens' outlier tile) follow after the grid dependency.
        for (int i = 0; i < SPW; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 4);  // the four warps of the k-block's group
        }
        mbar_init(&o_full, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        if (nkb > 0) {
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_x);
        }
        for (int u = 0; u < early; ++u) {
            mbar_arrive_expect_tx(&w_full[u], WUNIT + MP * PK_ROW);
            tma_load_2d(smem + u * WUNIT, &tm_w, u * PK_ROW, n0, &w_full[u]);
            QUIK_TRACE_AT(11, u);
        }
        if (nko > 0) {
            tma_prefetch_desc(&tm_wo);
            tma_prefetch_desc(&tm_xo);
            mbar_arrive_expect_tx(&o_full, nko * (WO_TILE + MP * OP_ROW));
            for (int kb = 0; kb < nko; ++kb)
                tma_load_2d(smem + WO_OFF + kb * WO_TILE, &tm_wo, kb * oke, n0, &o_full);
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&op_full[i], 4);
            mbar_init(&op_empty[i], 1);
        }
        mbar_init(&acc_full, NI);
        for (int i = 0; i < NI; ++i) mbar_init(&mma_done[i], 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_error_word);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const AbortState ab{&abort_s, err0_s};

    const int issuer = warp == 0 ? 0 : warp >= 2 + NW ? warp - 1 - NW : -1;
    if (issuer >= 0) {
        // ------------------------------------------------------------ MMA issuers
        // Issuer i takes k-blocks i, i + NI, ... into its own accumulator
        // (TMEM columns 32 i ..), so NI MMA streams are in flight; issuer 0
        // also does the outlier block.  The epilogue adds the accumulators.
        if (lane == 0) {
            bool ok = true;
            if (issuer == 0 && nko > 0) {  // the outlier block: both operands in shared memory
                ok = wait_bar(&o_full, 0, ab);
                QUIK_TRACE_AT(2, 0);
                if (ok) {
                    tc_fence_after();
                    const uint32_t id_o = OUT_INT8 ? idesc_s8_s32(BW, MP) : idesc_f16_f32(BW, MP);
                    for (int kb = 0; kb < nko; ++kb) {
                        const uint32_t wo = smem_base + WO_OFF + kb * WO_TILE;
                        const uint32_t xo = smem_base + XO_OFF + kb * XO_TILE;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ad = sw128_kmajor_desc(wo + 32 * k);
                            const uint64_t bd = sw128_kmajor_desc(xo + 32 * k);
                            if (OUT_INT8)
                                mma_i8(tmem + O_COL, ad, bd, id_o, (kb > 0 || k > 0));
                            else
                                mma_f16(tmem + O_COL, ad, bd, id_o, (kb > 0 || k > 0));
                        }
                    }
                }
            }
            const uint32_t idesc = idesc_s8_s32(BW, MP);
            const uint32_t acc = tmem + ACC_COL + 32 * issuer;
            for (int kb = issuer; kb < nkb && ok; kb += NI) {
                const int st = kb % S;
                if (!(ok = wait_bar(&op_full[st], (kb / S) & 1, ab))) break;
                QUIK_TRACE_AT(3, kb);
                tc_fence_after();
                const uint32_t xb = smem_base + X_OFF + st * XSTAGE;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_i8_ts(acc, tmem + A_COL + 32 * st + 8 * k, sw128_kmajor_desc(xb + 32 * k), idesc,
                              (kb > issuer || k > 0));
                mma_commit(&op_empty[st]);
            }
            if (ok) mma_commit(&acc_full);
            mma_commit(&mma_done[issuer]);
            mbar_wait_bounded(&mma_done[issuer], 0, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            grid_dependency_wait();  // Xq and Xo come from the previous kernel
            for (int kb = 0; kb < nko; ++kb)
                tma_load_2d(smem + XO_OFF + kb * XO_TILE, &tm_xo, kb * oke, 0, &o_full);
            for (int u = 0; u < early; ++u)
                tma_load_2d(smem + XU_OFF + u * XUNIT, &tm_x, u * PK_ROW, 0, &w_full[u]);
            int filled = early;  // units issued
            for (int u = early; u < nkb; ++u, ++filled) {
                const int st = u % SPW;
                if (!wait_bar(&w_empty[st], ((u / SPW) & 1) ^ 1, ab)) break;
                mbar_arrive_expect_tx(&w_full[st], WUNIT + MP * PK_ROW);
                tma_load_2d(smem + st * WUNIT, &tm_w, u * PK_ROW, n0, &w_full[st]);
                tma_load_2d(smem + XU_OFF + st * XUNIT, &tm_x, u * PK_ROW, 0, &w_full[st]);
                QUIK_TRACE_AT(11, u);
            }
            // never leave the CTA with a bulk copy still writing its shared
            // memory: slot i last held unit i + SPW * ((filled - 1 - i) / SPW)
            for (int i = 0; i < early; ++i)
                mbar_wait_bounded(&w_full[i], ((filled - 1 - i) / SPW) & 1, kWaitLimitNs);
            if (nko > 0) mbar_wait_bounded(&o_full, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ W rows -> TMEM, token rows -> X stage
        const int q = warp & 3;           // TMEM lane quadrant
        const int r = q * 32 + lane;      // W row in the tile = TMEM lane
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        const int grp = (warp - 2) >> 2;  // this warp's group: k-blocks grp, grp + NG, ...
        // this lane's share of the token rows: MP rows x 4 16-byte chunks over
        // the group's 4 warps (one chunk per lane; lanes >= MP idle for MP = 16)
        const int xw = (warp - 2) & 3;
        const int x_row = xw * (MP / 4) + (lane >> 2), x_ch = lane & 3;
        const bool x_on = lane < MP;
        // epilogue operands of group 0, loaded now so that the epilogue waits
        // on no global load: the row's weight scales and bias (not the
        // previous kernel's output) before the grid dependency, the token
        // scales (lane m holds token m's) after it
        const int n = n0 + r;
        const bool n_ok = n < p.N;
        float swn = 0.0f, swon = 0.0f, bn = 0.0f, sxm = 0.0f, sxom = 0.0f;
        if (grp == 0 && !DEBUG) {
            if (n_ok && p.Ki > 0) swn = p.sw[n];
            if (n_ok && OUT_INT8 && nko > 0) swon = p.swo[n];
            if (n_ok && p.bias != nullptr) bn = __half2float(__ushort_as_half(p.bias[n]));
        }
        grid_dependency_wait();  // sx (and sxo) come from the previous kernel
        if (grp == 0 && !DEBUG && lane < p.M) {
            if (p.Ki > 0) sxm = p.sx[lane];
            if (OUT_INT8 && nko > 0) sxom = p.sxo[lane];
        }
        bool ok = true;
        for (int kb = grp; kb < nkb && ok; kb += NG) {
            const int st = kb % S, ps = kb % SPW;
            ok = wait_bar(&op_empty[st], ((kb / S) & 1) ^ 1, ab);
            if (xw == 0 && lane == 0) QUIK_TRACE_AT(1, kb);
            ok = ok && wait_bar(&w_full[ps], (kb / SPW) & 1, ab);
            if (xw == 0 && lane == 0) QUIK_TRACE_AT(8, kb);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            // the packed bytes into registers, then the staging slot goes
            // back to the producer before the unpack: token row x_row, chunk
            // x_ch; W row r, 4 chunks of 16 bytes (64-byte swizzle)
            uint4 xv = make_uint4(0, 0, 0, 0), wv[4];
            if (x_on)
                xv = *reinterpret_cast<const uint4 *>(smem + XU_OFF + ps * XUNIT + x_row * PK_ROW + x_ch * 16);
            const uint8_t *wr = smem + ps * WUNIT + r * PK_ROW;
#pragma unroll
            for (int c = 0; c < 4; ++c) wv[c] = *reinterpret_cast<const uint4 *>(wr + ((c ^ ((r >> 1) & 3)) << 4));
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_empty[ps]);
            if (x_on) {  // two 16-byte unpacked chunks into the 128-byte-swizzled X stage
                uint4 lo, hi;
                unpack16(xv, lo, hi);
                uint8_t *xr = smem + X_OFF + st * XSTAGE + x_row * OP_ROW;
                *reinterpret_cast<uint4 *>(xr + (((2 * x_ch) ^ (x_row & 7)) << 4)) = lo;
                *reinterpret_cast<uint4 *>(xr + (((2 * x_ch + 1) ^ (x_row & 7)) << 4)) = hi;
            }
            uint32_t w[32];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 lo, hi;
                unpack16(wv[c], lo, hi);
                w[8 * c + 0] = lo.x; w[8 * c + 1] = lo.y; w[8 * c + 2] = lo.z; w[8 * c + 3] = lo.w;
                w[8 * c + 4] = hi.x; w[8 * c + 5] = hi.y; w[8 * c + 6] = hi.z; w[8 * c + 7] = hi.w;
            }
            if (xw == 0 && lane == 0) QUIK_TRACE_AT(9, kb);
            tmem_st_32x32b_x32(t_lane + A_COL + 32 * st, w);
            tmem_st_wait();
            fence_proxy_async_smem();  // the X stage's stores -> visible to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&op_full[st]);
                if (xw == 0) QUIK_TRACE_AT(0, kb);
            }
        }
        // ------------------------------------------------------------ epilogue (group 0)
        if (grp == 0) {
            ok = ok && wait_bar(&acc_full, 0, ab);
            if (xw == 0 && lane == 0) QUIK_TRACE_AT(4, 0);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                // two halves of 16 tokens (the second only when M > 16)
                for (int h = 0; h < 32 && h < p.M; h += 16) {
                    uint32_t a[16], o[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) a[j] = o[j] = 0;
                    if (nkb > 0) tmem_ld_32x32b_x16(t_lane + ACC_COL + h, a);
                    if (nko > 0) tmem_ld_32x32b_x16(t_lane + O_COL + h, o);
                    tmem_ld_wait();
                    // the other issuers' accumulators (those that took a k-block);
                    // all are multiples of 256, so the sum is exact
                    for (int i = 1; i < NI && i < nkb; ++i) {
                        uint32_t t[16];
                        tmem_ld_32x32b_x16(t_lane + ACC_COL + 32 * i + h, t);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) a[j] += t[j];
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = h + j;
                        const float sx_m = __shfl_sync(0xffffffffu, sxm, m);
                        const float sxo_m = __shfl_sync(0xffffffffu, sxom, m);
                        if (m >= p.M || !n_ok) continue;
                        const size_t at = (size_t)m * p.N + n;
                        if (DEBUG) {
                            if (p.Ki > 0) p.acc_dbg[at] = static_cast<int32_t>(a[j]) >> 8;
                            if (OUT_INT8 && nko > 0 && p.acc_o_dbg) p.acc_o_dbg[at] = static_cast<int32_t>(o[j]);
                            continue;
                        }
                        float y = p.Ki > 0 ? small_int_to_float(static_cast<int32_t>(a[j]) >> 8) * sx_m * swn : 0.0f;
                        if (nko > 0)
                            y += OUT_INT8 ? static_cast<float>(static_cast<int32_t>(o[j])) * sxo_m * swon
                                          : __uint_as_float(o[j]);
                        p.Y[at] = __half_as_ushort(__float2half_rn(y + bn));
                    }
                }
                if (xw == 0 && lane == 0) QUIK_TRACE_AT(5, 0);
                tc_fence_before();
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    if (threadIdx.x == 0) QUIK_TRACE_AT(7, 0);
}

// ============================================================================
// 2:4-sparse INT4 weights ("QUIK" abstract: quantisation plus 2:4 sparsity) on
// the sparse tensor-core MMA, for up to 32 tokens per CTA.
//
// W is the MMA's A operand, 128 rows per CTA, stored compressed: the two kept
// INT4 codes of every aligned group of four positions (one byte per group) and
// the group's position pair (one nibble i0 | i1 << 2).  Per k-block of 256
// positions the group warps widen the kept codes to INT8 (x16, in order) into
// a 128-byte-swizzled shared-memory stage (128 rows x 128 bytes) and store the
// pairs in tensor memory (lane = W row; one sparse MMA reads 64 bits, two
// columns at a 4-column-aligned address, group g in bits 4g .. 4g+3).  The
// tokens are the N operand (16 or 32 rows, widened to INT8 x16 in order, two
// 128-byte-wide tiles per k-block); a second grid dimension covers more tokens.
// Four sparse MMAs (K = 64 each) per k-block; the accumulator holds 256 A.
// The outlier block and the epilogue are those of the decode kernel above.
// ============================================================================
namespace sp24 {
constexpr int BW = 128;                      // W rows per CTA = TMEM lanes
constexpr int MT = 32;                       // tokens per CTA (the MMA's N: 16 or 32)
constexpr int KBL = 256;                     // positions per k-block
constexpr int WROW = 64;                     // packed kept codes per row per k-block (bytes)
constexpr int MROW = 32;                     // position pairs per row per k-block (bytes)
constexpr int XROW = 128;                    // packed token codes per row per k-block (bytes)
constexpr int S = 4;                         // operand stages
constexpr int SPW = 4;                       // staging units
constexpr int WUNIT = BW * WROW;             // 8 KB
constexpr int MUNIT = BW * MROW;             // 4 KB
constexpr int XUNIT = MT * XROW;             // 4 KB
constexpr int UNIT = WUNIT + MUNIT + XUNIT;  // 16 KB
constexpr int ASTAGE = BW * 128;             // widened kept codes: 128 rows x 128 bytes
constexpr int XTILE = MT * 128;              // one 128-byte-wide half of the widened token rows
constexpr int STAGE = ASTAGE + 2 * XTILE;    // 24 KB
constexpr int OKB = 2;                       // outlier k-blocks of 128-byte rows
constexpr int KO_MAX_F16 = 64 * OKB, KO_MAX_I8 = 128 * OKB;
constexpr int WO_TILE = BW * 128, XO_TILE = MT * 128;
constexpr int NG = 4, NW = 4 * NG, NI = 2;   // unpack groups (4 warps each), MMA issuers
constexpr int THREADS = (1 + NW + NI) * 32;
constexpr int OP_OFF = SPW * UNIT;
constexpr int WO_OFF = OP_OFF + S * STAGE;
constexpr int XO_OFF = WO_OFF + OKB * WO_TILE;
constexpr int SMEM = XO_OFF + OKB * XO_TILE + 1024;  // + alignment
constexpr int ACC_COL = 0, O_COL = 32 * NI, META_COL = O_COL + 32;
constexpr int META_STAGE = 16;               // four MMAs x 4 columns (2 used)
constexpr int TMEM_COLS = 256;
static_assert(META_COL % 4 == 0 && META_COL + S * META_STAGE <= TMEM_COLS, "metadata in tensor memory");
static_assert(S % NG == 0 && S % NI == 0, "group g owns stages g, g + NG, ...; one issuer per stage");
static_assert(WUNIT % 1024 == 0 && (WUNIT + MUNIT) % 1024 == 0 && UNIT % 1024 == 0, "swizzled staging");
static_assert(OP_OFF % 1024 == 0 && STAGE % 1024 == 0 && ASTAGE % 1024 == 0 && XTILE % 1024 == 0,
              "128-byte-swizzled operand tiles");
static_assert(WO_OFF % 1024 == 0 && XO_OFF % 1024 == 0, "128-byte-swizzled outlier tiles");
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace sp24

// 32 packed INT4 codes (16 bytes, code 2i in the low nibble of byte i) ->
// 32 INT8 values 16 c in order (two 16-byte chunks).
__device__ __forceinline__ void widen16_ordered(const uint4 v, uint4 &a, uint4 &b) {
    const uint32_t x[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (x[i] << 4) & 0xF0F0F0F0u;  // codes 0, 2, 4, 6 of the word
        const uint32_t hi = x[i] & 0xF0F0F0F0u;         // codes 1, 3, 5, 7
        asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(o[2 * i]) : "r"(lo), "r"(hi));
        asm("prmt.b32 %0, %1, %2, 0x7362;" : "=r"(o[2 * i + 1]) : "r"(lo), "r"(hi));
    }
    a = make_uint4(o[0], o[1], o[2], o[3]);
    b = make_uint4(o[4], o[5], o[6], o[7]);
}

template <bool OUT_INT8, bool DEBUG>
__global__ void __launch_bounds__(sp24::THREADS, 1)
    w4a4_gemv24_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_m,
                       const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wo,
                       const __grid_constant__ CUtensorMap tm_xo, const GemmParams p) {
    using namespace sp24;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t w_full[SPW], w_empty[SPW], op_full[S], op_empty[S], o_full, acc_full, mma_done[NI];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BW;
    const int m0 = blockIdx.y * MT;
    const int MP = p.M <= 16 ? 16 : 32;  // the MMA's N (token rows past M read as 0)
    const int nkb = p.nkb_i;
    const int oke = OUT_INT8 ? 128 : 64;
    const int nko = (p.k_o + oke - 1) / oke;
    const uint32_t unit_bytes = WUNIT + MUNIT + MP * XROW;

    const int early = nkb < SPW ? nkb : SPW;  // W units loaded before the CTA barrier
    if (warp == 1 && lane == 0) {
        // the producer's barriers and the first W units (kept codes and pairs:
        // not the previous kernel's output); their token rows follow after
        // the grid dependency
        for (int i = 0; i < SPW; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 4);  // the four warps of the k-block's group
        }
        mbar_init(&o_full, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        if (nkb > 0) {
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_m);
            tma_prefetch_desc(&tm_x);
        }
        for (int u = 0; u < early; ++u) {
            mbar_arrive_expect_tx(&w_full[u], unit_bytes);
            tma_load_2d(smem + u * UNIT, &tm_w, u * WROW, n0, &w_full[u]);
            tma_load_2d(smem + u * UNIT + WUNIT, &tm_m, u * MROW, n0, &w_full[u]);
        }
        if (nko > 0) {
            tma_prefetch_desc(&tm_wo);
            tma_prefetch_desc(&tm_xo);
            mbar_arrive_expect_tx(&o_full, nko * (WO_TILE + MP * 128));
            for (int kb = 0; kb < nko; ++kb)
                tma_load_2d(smem + WO_OFF + kb * WO_TILE, &tm_wo, kb * oke, n0, &o_full);
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&op_full[i], 4);
            mbar_init(&op_empty[i], 1);
        }
        mbar_init(&acc_full, NI);
        for (int i = 0; i < NI; ++i) mbar_init(&mma_done[i], 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_error_word);
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const AbortState ab{&abort_s, err0_s};

    const int issuer = warp == 0 ? 0 : warp >= 2 + NW ? warp - 1 - NW : -1;
    if (issuer >= 0) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            bool ok = true;
            if (issuer == 0 && nko > 0) {  // the dense outlier block
                ok = wait_bar(&o_full, 0, ab);
                if (ok) {
                    tc_fence_after();
                    const uint32_t id_o = OUT_INT8 ? idesc_s8_s32(BW, MP) : idesc_f16_f32(BW, MP);
                    for (int kb = 0; kb < nko; ++kb) {
                        const uint32_t wo = smem_base + WO_OFF + kb * WO_TILE;
                        const uint32_t xo = smem_base + XO_OFF + kb * XO_TILE;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ad = sw128_kmajor_desc(wo + 32 * k);
                            const uint64_t bd = sw128_kmajor_desc(xo + 32 * k);
                            if (OUT_INT8)
                                mma_i8(tmem + O_COL, ad, bd, id_o, (kb > 0 || k > 0));
                            else
                                mma_f16(tmem + O_COL, ad, bd, id_o, (kb > 0 || k > 0));
                        }
                    }
                }
            }
            const uint32_t idesc = idesc_s8_s32_sparse(BW, MP);
            const uint32_t acc = tmem + ACC_COL + 32 * issuer;
            for (int kb = issuer; kb < nkb && ok; kb += NI) {
                const int st = kb % S;
                if (!(ok = wait_bar(&op_full[st], (kb / S) & 1, ab))) break;
                tc_fence_after();
                const uint32_t a0 = smem_base + OP_OFF + st * STAGE;
                const uint32_t x0 = a0 + ASTAGE;
#pragma unroll
                for (int j = 0; j < 4; ++j)  // kept codes 32 bytes apart, tokens 64
                    mma_sp_i8(acc, sw128_kmajor_desc(a0 + 32 * j),
                              sw128_kmajor_desc(x0 + (j >> 1) * XTILE + 64 * (j & 1)),
                              tmem + META_COL + META_STAGE * st + 4 * j, idesc, (kb > issuer || j > 0));
                mma_commit(&op_empty[st]);
            }
            if (ok) mma_commit(&acc_full);
            mma_commit(&mma_done[issuer]);
            mbar_wait_bounded(&mma_done[issuer], 0, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            grid_dependency_wait();  // Xq and Xo come from the previous kernel
            for (int kb = 0; kb < nko; ++kb)
                tma_load_2d(smem + XO_OFF + kb * XO_TILE, &tm_xo, kb * oke, m0, &o_full);
            for (int u = 0; u < early; ++u)
                tma_load_2d(smem + u * UNIT + WUNIT + MUNIT, &tm_x, u * XROW, m0, &w_full[u]);
            int filled = early;
            for (int u = early; u < nkb; ++u, ++filled) {
                const int st = u % SPW;
                if (!wait_bar(&w_empty[st], ((u / SPW) & 1) ^ 1, ab)) break;
                mbar_arrive_expect_tx(&w_full[st], unit_bytes);
                tma_load_2d(smem + st * UNIT, &tm_w, u * WROW, n0, &w_full[st]);
                tma_load_2d(smem + st * UNIT + WUNIT, &tm_m, u * MROW, n0, &w_full[st]);
                tma_load_2d(smem + st * UNIT + WUNIT + MUNIT, &tm_x, u * XROW, m0, &w_full[st]);
            }
            // never leave the CTA with a bulk copy still writing its shared memory
            for (int i = 0; i < early; ++i)
                mbar_wait_bounded(&w_full[i], ((filled - 1 - i) / SPW) & 1, kWaitLimitNs);
            if (nko > 0) mbar_wait_bounded(&o_full, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ kept codes -> A stage,
        // position pairs -> tensor memory, token rows -> X tiles
        const int q = warp & 3;           // TMEM lane quadrant
        const int r = q * 32 + lane;      // W row in the tile = TMEM lane
        const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
        const int grp = (warp - 2) >> 2;  // this warp's group: k-blocks grp, grp + NG, ...
        const int xt = ((warp - 2) & 3) * 32 + lane;  // 0 .. 127 within the group
        const int n = n0 + r;
        const bool n_ok = n < p.N;
        float swn = 0.0f, swon = 0.0f, bn = 0.0f, sxm = 0.0f, sxom = 0.0f;
        if (grp == 0 && !DEBUG) {
            if (n_ok && p.Ki > 0) swn = p.sw[n];
            if (n_ok && OUT_INT8 && nko > 0) swon = p.swo[n];
            if (n_ok && p.bias != nullptr) bn = __half2float(__ushort_as_half(p.bias[n]));
        }
        grid_dependency_wait();  // sx (and sxo) come from the previous kernel
        if (grp == 0 && !DEBUG && m0 + lane < p.M) {
            if (p.Ki > 0) sxm = p.sx[m0 + lane];
            if (OUT_INT8 && nko > 0) sxom = p.sxo[m0 + lane];
        }
        bool ok = true;
        for (int kb = grp; kb < nkb && ok; kb += NG) {
            const int st = kb % S, ps = kb % SPW;
            ok = wait_bar(&op_empty[st], ((kb / S) & 1) ^ 1, ab);
            ok = ok && wait_bar(&w_full[ps], (kb / SPW) & 1, ab);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const uint8_t *unit = smem + ps * UNIT;
            // the packed bytes into registers; the staging slot then goes back
            // to the producer: W row r (4 chunks, 64-byte swizzle), its 32
            // bytes of pairs, and two of the MP x 8 token chunks (128-byte swizzle)
            uint4 wv[4], mv[2], xv[2];
            const uint8_t *wr = unit + r * WROW;
#pragma unroll
            for (int c = 0; c < 4; ++c) wv[c] = *reinterpret_cast<const uint4 *>(wr + ((c ^ ((r >> 1) & 3)) << 4));
            mv[0] = *reinterpret_cast<const uint4 *>(unit + WUNIT + r * MROW);
            mv[1] = *reinterpret_cast<const uint4 *>(unit + WUNIT + r * MROW + 16);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int task = xt + 128 * i, xr = task >> 3, xc = task & 7;
                xv[i] = make_uint4(0, 0, 0, 0);
                if (xr < MP)
                    xv[i] = *reinterpret_cast<const uint4 *>(unit + WUNIT + MUNIT + xr * XROW + ((xc ^ (xr & 7)) << 4));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_empty[ps]);
            // kept codes: 64 packed bytes -> 128 widened bytes of row r
            uint8_t *ar = smem + OP_OFF + st * STAGE + r * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 a, b;
                widen16_ordered(wv[c], a, b);
                *reinterpret_cast<uint4 *>(ar + (((2 * c) ^ (r & 7)) << 4)) = a;
                *reinterpret_cast<uint4 *>(ar + (((2 * c + 1) ^ (r & 7)) << 4)) = b;
            }
            // token chunk (xr, xc): widened bytes 32 xc .. 32 xc + 31 -> tile xc / 4
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int task = xt + 128 * i, xr = task >> 3, xc = task & 7;
                if (xr >= MP) continue;
                uint4 a, b;
                widen16_ordered(xv[i], a, b);
                uint8_t *xrow = smem + OP_OFF + st * STAGE + ASTAGE + (xc >> 2) * XTILE + xr * 128;
                *reinterpret_cast<uint4 *>(xrow + (((2 * (xc & 3)) ^ (xr & 7)) << 4)) = a;
                *reinterpret_cast<uint4 *>(xrow + (((2 * (xc & 3) + 1) ^ (xr & 7)) << 4)) = b;
            }
            // position pairs: 64 bits per MMA at a 4-column-aligned address.
            // Groups past K_i (read as 0 in a ragged last k-block) get the
            // valid pair (0, 1); their kept codes and tokens are 0.
            uint32_t mw[8] = {mv[0].x, mv[0].y, mv[0].z, mv[0].w, mv[1].x, mv[1].y, mv[1].z, mv[1].w};
            const int valid_words = (p.Ki - kb * KBL) / 32;  // 8 groups per word
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i >= valid_words) mw[i] = 0x44444444u;
            const uint32_t mt[16] = {mw[0], mw[1], 0u, 0u, mw[2], mw[3], 0u, 0u,
                                     mw[4], mw[5], 0u, 0u, mw[6], mw[7], 0u, 0u};
            tmem_st_32x32b_x16(t_lane + META_COL + META_STAGE * st, mt);
            tmem_st_wait();
            fence_proxy_async_smem();  // the stage's stores -> visible to the MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&op_full[st]);
        }
        // ------------------------------------------------------------ epilogue (group 0)
        if (grp == 0) {
            ok = ok && wait_bar(&acc_full, 0, ab);
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after();
                for (int h = 0; h < 32 && m0 + h < p.M; h += 16) {
                    uint32_t a[16], o[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) a[j] = o[j] = 0;
                    if (nkb > 0) tmem_ld_32x32b_x16(t_lane + ACC_COL + h, a);
                    if (nko > 0) tmem_ld_32x32b_x16(t_lane + O_COL + h, o);
                    tmem_ld_wait();
                    for (int i = 1; i < NI && i < nkb; ++i) {
                        uint32_t t[16];
                        tmem_ld_32x32b_x16(t_lane + ACC_COL + 32 * i + h, t);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) a[j] += t[j];
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + h + j;
                        const float sx_m = __shfl_sync(0xffffffffu, sxm, h + j);
                        const float sxo_m = __shfl_sync(0xffffffffu, sxom, h + j);
                        if (m >= p.M || !n_ok) continue;
                        const size_t at = (size_t)m * p.N + n;
                        if (DEBUG) {
                            if (p.Ki > 0) p.acc_dbg[at] = static_cast<int32_t>(a[j]) >> 8;
                            if (OUT_INT8 && nko > 0 && p.acc_o_dbg) p.acc_o_dbg[at] = static_cast<int32_t>(o[j]);
                            continue;
                        }
                        float y = p.Ki > 0 ? small_int_to_float(static_cast<int32_t>(a[j]) >> 8) * sx_m * swn : 0.0f;
                        if (nko > 0)
                            y += OUT_INT8 ? static_cast<float>(static_cast<int32_t>(o[j])) * sxo_m * swon
                                          : __uint_as_float(o[j]);
                        p.Y[at] = __half_as_ushort(__float2half_rn(y + bn));
                    }
                }
                tc_fence_before();
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ----------------------------------------------------------------- host side
template <class C>
quik_status run(const GemmArgs &a, cudaStream_t stream) {
    static_assert(sizeof(C) > 0, "");
    const int Ki = a.K - a.k_o;
    CUtensorMap mxq, mwq, mxo, mwo;
    std::memset(&mxq, 0, sizeof(mxq));
    std::memset(&mwq, 0, sizeof(mwq));
    std::memset(&mxo, 0, sizeof(mxo));
    std::memset(&mwo, 0, sizeof(mwo));
    if (Ki > 0) {
        if (!make_map(&mxq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, Ki / 2, a.M, Ki / 2, PK_ROW, BM,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !make_map(&mwq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, Ki / 2, a.N, Ki / 2, PK_ROW,
                      C::BN, CU_TENSOR_MAP_SWIZZLE_NONE))
            return QUIK_ERR_CUDA;
    }
    const bool outliers = a.k_o > 0 && a.Xo != nullptr;  // debug entry may skip them
    if (outliers) {
        const bool i8 = C::OUT_INT8;
        const CUtensorMapDataType dt =
            i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        const uint64_t es = i8 ? 1 : 2;
        const uint32_t bi = i8 ? 128 : 64;
        if (!make_map(&mxo, dt, a.Xo, a.k_o, a.M, a.k_o * es, bi, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&mwo, dt, a.Wo, a.k_o, a.N, a.k_o * es, bi, C::BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    GemmParams p{};
    p.M = a.M;
    p.N = a.N;
    p.Ki = Ki;
    p.k_o = a.k_o;
    p.nkb_i = (Ki + KB - 1) / KB;
    p.nkb_o = !outliers ? 0 : (C::OUT_INT8 ? (a.k_o + 127) / 128 : (a.k_o + 63) / 64);
    p.G = a.group > 0 ? Ki / a.group : 1;
    p.sx = a.sx;
    p.sw = a.sw;
    p.sxo = a.sxo;
    p.swo = a.swo;
    p.bias = a.bias;
    p.Y = a.Y;
    p.acc_dbg = a.acc_dbg;
    p.acc_o_dbg = a.acc_o_dbg;

    auto kern = w4a4_gemm_kernel<C>;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), C::SMEM)) return QUIK_ERR_CUDA;
    const dim3 grid((a.M + BM - 1) / BM, (a.N + C::BN - 1) / C::BN);
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(mxq, mwq, mxo, mwo, p);
    return cudaGetLastError() == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

template <bool OUT_INT8, bool DEBUG, bool A8, bool W8>
quik_status run_pair(const GemmArgs &a, cudaStream_t stream) {
    const int Ki = a.K - a.k_o;
    const bool outliers = a.k_o > 0 && a.Xo != nullptr;  // debug entry may skip them
    const uint64_t ob = static_cast<uint64_t>(a.k_o) * (OUT_INT8 ? 1 : 2);  // outlier bytes per row
    CUtensorMap mwq, mwo, mxo;
    std::memset(&mwq, 0, sizeof(mwq));
    std::memset(&mwo, 0, sizeof(mwo));
    std::memset(&mxo, 0, sizeof(mxo));
    // B k-blocks: 128 rows x 64 packed bytes, or x 128 INT8 codes
    const uint64_t wrow = W8 ? Ki : Ki / 2;
    if (Ki > 0 && !make_map(&mwq, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, wrow, a.N, wrow,
                            W8 ? OP_ROW : PK_ROW, pair::BNH, CU_TENSOR_MAP_SWIZZLE_NONE))
        return QUIK_ERR_CUDA;
    // outlier blocks as plain bytes, 128 rows x 128 bytes per unit
    if (outliers &&
        (!make_map(&mwo, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wo, ob, a.N, ob, OP_ROW, pair::BNH,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
         !make_map(&mxo, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xo, ob, a.M, ob, OP_ROW, BM,
                   CU_TENSOR_MAP_SWIZZLE_NONE)))
        return QUIK_ERR_CUDA;
    GemmParams p{};
    p.M = a.M;
    p.N = a.N;
    p.Ki = Ki;
    p.k_o = a.k_o;
    p.nkb_i = (Ki + KB - 1) / KB;
    p.nkb_o = !outliers ? 0 : (OUT_INT8 ? (a.k_o + 127) / 128 : (a.k_o + 63) / 64);
    p.G = 1;
    p.sx = a.sx;
    p.sw = a.sw;
    p.sxo = a.sxo;
    p.swo = a.swo;
    p.bias = a.bias;
    p.Y = a.Y;
    p.acc_dbg = a.acc_dbg;
    p.acc_o_dbg = a.acc_o_dbg;
    // Y by TMA stores of 128-row x 64-column blocks (128-byte swizzle) when its
    // rows are 16-byte multiples; else per-thread stores
    CUtensorMap my;
    std::memset(&my, 0, sizeof(my));
    p.tma_y = !DEBUG && (a.N % 8 == 0) &&
              make_map(&my, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.Y, a.N, a.M, static_cast<uint64_t>(a.N) * 2,
                       64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
    auto kern = w4a4_gemm_pair_kernel<OUT_INT8, DEBUG, A8, W8>;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), pair::SMEM)) return QUIK_ERR_CUDA;
    const dim3 grid(2 * ((a.N + pair::BN - 1) / pair::BN), (a.M + 2 * BM - 1) / (2 * BM));
    if (!a.after_quantize) {
        kern<<<grid, pair::THREADS, pair::SMEM, stream>>>(mwq, mwo, mxo, my,
                                                          static_cast<const uint8_t *>(a.Xq), p);
        return cudaGetLastError() == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
    }
    // programmatic dependent launch: the CTAs may start while the quantiser
    // finishes; every read of its outputs waits on the grid dependency first
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(pair::THREADS);
    cfg.dynamicSmemBytes = pair::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint8_t *xq = static_cast<const uint8_t *>(a.Xq);
    return cudaLaunchKernelEx(&cfg, kern, mwq, mwo, mxo, my, xq, p) == cudaSuccess ? QUIK_OK
                                                                                  : QUIK_ERR_CUDA;
}

// Decode-shaped launches: one CTA per 128 rows of W.
template <bool OUT_INT8, bool DEBUG>
quik_status run_gemv(const GemmArgs &a, cudaStream_t stream) {
    const int Ki = a.K - a.k_o;
    const bool outliers = a.k_o > 0 && a.Xo != nullptr;  // the debug entry may skip them
    CUtensorMap mw, mx, mwo, mxo;
    std::memset(&mw, 0, sizeof(mw));
    std::memset(&mx, 0, sizeof(mx));
    std::memset(&mwo, 0, sizeof(mwo));
    std::memset(&mxo, 0, sizeof(mxo));
    if (Ki > 0) {
        // packed W rows: 64 bytes (one k-block) x 128 rows per box, 64-byte swizzle;
        // packed token rows: 64 bytes x 16 or 32 rows per box, the MMA's N (rows
        // past M read as 0)
        const uint32_t mp = a.M <= 16 ? 16 : 32;
        if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, Ki / 2, a.N, Ki / 2, PK_ROW, gemv::BW,
                      CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, Ki / 2, a.M, Ki / 2, PK_ROW, mp,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return QUIK_ERR_CUDA;
    }
    if (outliers) {
        // outlier blocks: 128-byte rows (64 fp16 or 128 int8 channels), the
        // swizzled K-major layout the MMA reads
        const CUtensorMapDataType dt = OUT_INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        const uint32_t oke = OUT_INT8 ? 128 : 64;
        const uint64_t pitch = static_cast<uint64_t>(a.k_o) * (OUT_INT8 ? 1 : 2);
        if (!make_map(&mwo, dt, a.Wo, a.k_o, a.N, pitch, oke, gemv::BW, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&mxo, dt, a.Xo, a.k_o, a.M, pitch, oke, a.M <= 16 ? 16 : 32, CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    GemmParams p{};
    p.M = a.M;
    p.N = a.N;
    p.Ki = Ki;
    p.k_o = outliers ? a.k_o : 0;
    p.nkb_i = (Ki + KB - 1) / KB;
    p.nkb_o = 0;
    p.G = 1;
    p.sx = a.sx;
    p.sw = a.sw;
    p.sxo = a.sxo;
    p.swo = a.swo;
    p.bias = a.bias;
    p.Y = a.Y;
    p.acc_dbg = a.acc_dbg;
    p.acc_o_dbg = a.acc_o_dbg;
    auto kern = w4a4_gemv_kernel<OUT_INT8, DEBUG>;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), gemv::SMEM)) return QUIK_ERR_CUDA;
    const dim3 grid((a.N + gemv::BW - 1) / gemv::BW);
    if (!a.after_quantize) {
        kern<<<grid, gemv::THREADS, gemv::SMEM, stream>>>(mw, mx, mwo, mxo, p);
        return cudaGetLastError() == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(gemv::THREADS);
    cfg.dynamicSmemBytes = gemv::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, mx, mwo, mxo, p) == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

// 2:4-sparse weights: kept codes [N, K_i / 4] and position pairs
// [N, K_i / 8]; tiles of 128 W rows x 32 tokens (16 when M <= 16).
template <bool OUT_INT8, bool DEBUG>
quik_status run_gemv24(const GemmArgs &a, cudaStream_t stream) {
    const int Ki = a.K - a.k_o;
    const bool outliers = a.k_o > 0 && a.Xo != nullptr;  // the debug entry may skip them
    const uint32_t mp = a.M <= 16 ? 16 : 32;
    CUtensorMap mw, mm, mx, mwo, mxo;
    std::memset(&mw, 0, sizeof(mw));
    std::memset(&mm, 0, sizeof(mm));
    std::memset(&mx, 0, sizeof(mx));
    std::memset(&mwo, 0, sizeof(mwo));
    std::memset(&mxo, 0, sizeof(mxo));
    if (Ki > 0) {
        // kept codes: 64 bytes (256 positions) x 128 rows per box, 64-byte
        // swizzle; pairs: 32 bytes x 128 rows; token rows: 128 bytes x 16 or
        // 32 rows, 128-byte swizzle (rows past M read as 0)
        if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, Ki / 4, a.N, Ki / 4, sp24::WROW, sp24::BW,
                      CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map(&mm, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wmeta, Ki / 8, a.N, Ki / 8, sp24::MROW, sp24::BW,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
            !make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, Ki / 2, a.M, Ki / 2, sp24::XROW, mp,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    if (outliers) {
        const CUtensorMapDataType dt = OUT_INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
        const uint32_t oke = OUT_INT8 ? 128 : 64;
        const uint64_t pitch = static_cast<uint64_t>(a.k_o) * (OUT_INT8 ? 1 : 2);
        if (!make_map(&mwo, dt, a.Wo, a.k_o, a.N, pitch, oke, sp24::BW, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&mxo, dt, a.Xo, a.k_o, a.M, pitch, oke, mp, CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    GemmParams p{};
    p.M = a.M;
    p.N = a.N;
    p.Ki = Ki;
    p.k_o = outliers ? a.k_o : 0;
    p.nkb_i = (Ki + sp24::KBL - 1) / sp24::KBL;
    p.nkb_o = 0;
    p.G = 1;
    p.sx = a.sx;
    p.sw = a.sw;
    p.sxo = a.sxo;
    p.swo = a.swo;
    p.bias = a.bias;
    p.Y = a.Y;
    p.acc_dbg = a.acc_dbg;
    p.acc_o_dbg = a.acc_o_dbg;
    auto kern = w4a4_gemv24_kernel<OUT_INT8, DEBUG>;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), sp24::SMEM)) return QUIK_ERR_CUDA;
    const dim3 grid((a.N + sp24::BW - 1) / sp24::BW, (a.M + sp24::MT - 1) / sp24::MT);
    if (!a.after_quantize) {
        kern<<<grid, sp24::THREADS, sp24::SMEM, stream>>>(mw, mm, mx, mwo, mxo, p);
        return cudaGetLastError() == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(sp24::THREADS);
    cfg.dynamicSmemBytes = sp24::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mw, mm, mx, mwo, mxo, p) == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

// Per-channel scales: the CTA-pair kernel (faster than a single-CTA kernel
// with 128-row tiles at every M measured, 16 to 4096); per-group scales: the
// shared-memory-operand kernel.
template <bool DEBUG>
quik_status dispatch(const GemmArgs &a, cudaStream_t stream) {
    if (a.sparse24) {  // 2:4-sparse INT4 weights: per-channel scales, INT4 activations
        if (a.group != 0 || a.a8 || a.w8 || (a.K - a.k_o) % 128 != 0 ||
            a.k_o > (a.out_int8 ? sp24::KO_MAX_I8 : sp24::KO_MAX_F16))
            return QUIK_ERR_UNSUPPORTED;
        return a.out_int8 ? run_gemv24<true, DEBUG>(a, stream) : run_gemv24<false, DEBUG>(a, stream);
    }
    if (a.a8) {  // INT8 activations (W4A8, W8A8): per-token scales, the pair kernel
        if (a.group != 0) return QUIK_ERR_UNSUPPORTED;
        if (a.w8)
            return a.out_int8 ? run_pair<true, DEBUG, true, true>(a, stream)
                              : run_pair<false, DEBUG, true, true>(a, stream);
        return a.out_int8 ? run_pair<true, DEBUG, true, false>(a, stream)
                          : run_pair<false, DEBUG, true, false>(a, stream);
    }
    if (a.w8) return QUIK_ERR_UNSUPPORTED;
    if (a.group == 0 && a.M <= gemv::MT && a.k_o <= (a.out_int8 ? gemv::KO_MAX_I8 : gemv::KO_MAX_F16))
        return a.out_int8 ? run_gemv<true, DEBUG>(a, stream) : run_gemv<false, DEBUG>(a, stream);
    if (persistent_gemm_takes(a)) return launch_gemm_persistent(a, stream);
    if (a.group == 0)
        return a.out_int8 ? run_pair<true, DEBUG, false, false>(a, stream)
                          : run_pair<false, DEBUG, false, false>(a, stream);
    return a.out_int8 ? run<CfgGroup<true, DEBUG>>(a, stream) : run<CfgGroup<false, DEBUG>>(a, stream);
}

// A CTA waiting on a barrier that nothing completes: exercises the bounded
// wait and the error word without a fault.
__global__ void timeout_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns)) atomicAdd(&g_error_word, 1u);
    __syncthreads();
}

}  // namespace

quik_status launch_gemm(const GemmArgs &a, cudaStream_t stream) {
    return a.debug ? dispatch<true>(a, stream) : dispatch<false>(a, stream);
}

quik_status launch_timeout_selftest(uint32_t limit_us, cudaStream_t stream) {
    timeout_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull);
    return cudaGetLastError() == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

#ifdef QUIK_TRACE
extern "C" __attribute__((visibility("default"))) int qtrace_read(unsigned long long *dst) {
    return cudaMemcpyFromSymbol(dst, g_trace, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
extern "C" __attribute__((visibility("default"))) int qtrace_clear() {
    static unsigned long long zero[sizeof(g_trace) / sizeof(unsigned long long)];
    return cudaMemcpyToSymbol(g_trace, zero, sizeof(g_trace)) == cudaSuccess ? 0 : -1;
}
#endif

#ifdef QUIK_CHECKS
extern "C" __attribute__((visibility("default"))) unsigned long long qchk_gemm_word() {
    unsigned long long v = 0;
    cudaMemcpyFromSymbol(&v, g_check_word, sizeof(v));
    return v;
}
#endif

quik_status sync_check(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return QUIK_ERR_CUDA;
    unsigned int word = 0, bad_perm = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return QUIK_ERR_CUDA;
    // the counters are never reset on the device: a kernel running on another
    // stream keeps its start-time snapshot valid, and no increase is lost
    const unsigned int waits = counter_increase(kCounterGemmWaits, word) + persistent_gemm_errors();
    const unsigned int qwaits = take_quantize_errors(&bad_perm);
    if (waits != 0 || qwaits != 0) return QUIK_ERR_TIMEOUT;
    if (bad_perm != 0) return QUIK_ERR_INVALID_ARG;
    return QUIK_OK;
}

}  // namespace quik
