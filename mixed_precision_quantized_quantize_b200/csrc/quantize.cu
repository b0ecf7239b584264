// quantize.cu -- reorder + dynamic symmetric INT4 quantisation + nibble packing
// of the rows of an fp16 matrix, with the outlier block copied (FP16) or
// quantised to INT8.  Serves activations (one row per token; "Atom: Low-bit
// Quantization for Efficient and Accurate LLM Serving", summary: dynamic
// per-input scales, reordering fused into one pass, idea I2) and the offline
// weight pack (one row per output channel; QUIK sample names pack_to_i4 /
// two_compl).
//
// Work split.  A team of TT = 32 * ceil(words / (32 W)) threads (a word = 8
// codes; W words per thread) owns one row at a time; a CTA holds up to four
// teams, which share one table of perm and otherwise run independently (their
// own named barrier, their own ring of 2-4 row slots); CTAs are persistent and
// rows are strided over all teams of the grid.  Per CTA:
//   0. thread 0 starts one bulk copy of perm (int32) and those of every
//      team's first rows (one per slot); all threads then turn perm in place into the
//      table of byte offsets into a row (uint32; for K > 16384 uint16 element
//      indices, built from 16-byte global loads).  An entry outside [0, K)
//      becomes 0 and is reported (never used as an address).
// Per row, in one team:
//   1. the team leader waits for the row; a named barrier (OR-reducing a
//      timeout flag) hands it to the team and frees the slot of the previous
//      row, which the leader refills with the row a ring ahead;
//   2. each thread gathers 8 reordered positions per word (as 4 half2), W
//      words in registers, and takes their absmax;
//   3. per-row scale: warp shuffles and a second team barrier; per-group
//      scale (128 positions = 16 words = 16 adjacent lanes): 4-step xor
//      shuffle.  s = fl(m / 7) is computed exactly in integer arithmetic
//      (m is an fp16 value: at most 11 significant bits);
//   4. codes are packed 8 per word (paired fp32 arithmetic) and stored
//      coalesced (a warp writes 128 contiguous bytes);
//   5. outlier positions Ki..K-1 are gathered and copied, or quantised with
//      their own scale fl(absmax / 127).
// The kernel is meant to be bound by HBM bandwidth (2 bytes read per
// element, 0.5 byte written per INT4 code).
#include <algorithm>
#include <atomic>

#include <cuda_fp16.h>

#include "quik_internal.h"
#include "sm100.cuh"

namespace quik {

QUIK_CHECK_DECL

// Count of bounded waits that ran out in this file's kernels, and of perm
// entries outside [0, K).  Both only grow; quik_sync_check reports their
// increase since its previous call (take_quantize_errors).
__device__ unsigned int g_quant_error;
__device__ unsigned int g_quant_bad_perm;
// Test entry (quik_test_stall): nonzero makes each team leader's first row
// wait on a barrier that nothing completes, so the bounded wait runs out and
// the kernel takes its error path.
__device__ int g_quant_stall;

namespace {

using ptx::f2;
using ptx::grid_launch_dependents;
using ptx::f2_fma;
using ptx::f2_split;
using ptx::f2_sub;

constexpr int kQMaxThreads = 512;  // 16 warps: up to 2048 words (W = 4) or 4096 (W = 8)
constexpr int kQMaxTeams = 4;
constexpr int kQMaxRing = 4;

struct QParams {
    const uint16_t *X;
    const int32_t *perm;
    int rows, K, k_o;
    int team_threads;  // TT, a multiple of 32
    int teams;         // teams per CTA (1 .. 4)
    int ring;          // row slots per team (2 .. 4)
    uint8_t *Q;
    float *scale;
    void *O;
    float *o_scale;
    int bits8;  // per-token rows only: INT8 codes (one byte each, divisor 127)
    int wide;   // per-token rows only: INT4 codes as the bytes 16 c in the persistent GEMM's operand order
    const uint16_t *gamma;  // RMS-norm weight [K] in source channel order (NORM kernels only)
    float eps;              // RMS-norm epsilon (NORM kernels only)
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

// fl(m / D) for an odd divisor 2^(L-1) < D < 2^L and m >= 0 zero or a
// normal fp32 (an fp16 value widened, or with the fused norm a product of two
// fp16 values, at least 2^-48).  With m = S 2^(E-150), S the 24-bit significand, the
// quotient's 24-bit significand is the integer nearest to S 2^sh / D for the
// shift sh in {L-1, L} that puts it in [2^23, 2^24]; the rounding is exact
// integer arithmetic and never meets a tie (2 * remainder is even, D odd).
template <uint32_t D, int L>
__device__ __forceinline__ float div_exact(float m) {
    static_assert((D & 1u) && D > (1u << (L - 1)) && D < (1u << L), "odd D in (2^(L-1), 2^L)");
    const uint32_t b = __float_as_uint(m);
    if (b == 0u) return 0.0f;
    const uint32_t E = b >> 23;
    const uint32_t S = (b & 0x7FFFFFu) | 0x800000u;
    const int sh = (static_cast<uint64_t>(S) << L) < (static_cast<uint64_t>(D) << 24) ? L : L - 1;
    const uint32_t num = S << sh;  // < 2^31
    uint32_t q = num / D;
    const uint32_t rem = num - q * D;
    q += (2u * rem > D) ? 1u : 0u;
    uint32_t e = E - static_cast<uint32_t>(sh);
    if (q == (1u << 24)) {  // rounded up to the next binade
        q = 1u << 23;
        e += 1u;
    }
    return __uint_as_float((e << 23) | (q & 0x7FFFFFu));
}

// Hardware reciprocal (relative error at most 2^-23 for normal s; 0 for s == 0).
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return s != 0.0f ? r : 0.0f;
}

// The half2 (lo of a, lo of b) from two 16-bit loads.
__device__ __forceinline__ uint32_t pair16(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// Per lane, the operand of larger magnitude (its sign is not used): an
// absmax that needs no separate |.|.
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Exact code of one value (the rare near-tie path): rint of the correctly
// rounded fp32 quotient, clamped, 0 when s == 0.
__device__ __forceinline__ int exact_code(float v, float s, int qmax) {
    if (s == 0.0f) return 0;
    const int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-qmax, min(qmax, q));
}

// The eight values of one word, as fp32: four half2 (widened exactly) or
// four fp32 pairs (the products h * gamma of the fused norm).
__device__ __forceinline__ uint64_t pair_f32(const uint32_t (&h)[4], int k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[k]));
    return f2(f.x, f.y);
}
__device__ __forceinline__ uint64_t pair_f32(const uint64_t (&z)[4], int k) { return z[k]; }
__device__ __forceinline__ float value_f32(const uint32_t (&h)[4], int k, int hi) {
    return h2f(static_cast<uint16_t>(hi ? h[k] >> 16 : h[k] & 0xffffu));
}
__device__ __forceinline__ float value_f32(const uint64_t (&z)[4], int k, int hi) {
    float a, b;
    f2_split(z[k], a, b);
    return hi ? b : a;
}

// Eight codes of one 32-bit output word from four half2 values (or four
// fp32 pairs).
//   Fast path: r = rint(v * rs) of the exact product (one fused
//   multiply-add with 1.5 * 2^23), rs the hardware reciprocal of s (relative
//   error <= 2u, u = 2^-24).  |v rs - fl(v/s)| <= |v/s| 3u <= 1.3e-6 for
//   |v/s| <= 7(1+u) (|v| <= max|v|), so unless v rs lies within 2e-6 of a
//   half-integer (the only points where rint changes value) fl(v/s) rounds
//   to r as well.  The residual v rs - r comes from a second fused
//   multiply-add (relative error u), and a word with any near-tie is redone
//   with IEEE divisions.  No clamp is needed: |r| <= 7.
template <typename V>
__device__ __forceinline__ uint32_t pack_codes8(const V &h, float s, float rs) {
    uint32_t word = kPackBias;
    float dmax = 0.0f;
    const uint64_t rs2 = f2(rs, rs), kr2 = f2(kRound, kRound);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t v2 = pair_f32(h, k);
        const uint64_t m = f2_fma(v2, rs2, kr2);           // 1.5*2^23 + rint(v rs)
        const uint64_t r = f2_sub(m, kr2);                 // rint(v rs), exact
        float r0, r1;
        f2_split(r, r0, r1);
        const uint64_t d = f2_fma(v2, rs2, f2(-r0, -r1));  // v rs - rint(v rs)
        float m0, m1, d0, d1;
        f2_split(m, m0, m1);
        f2_split(d, d0, d1);
        dmax = max3(dmax, fabsf(d0), fabsf(d1));
        word += __float_as_uint(m0) << (8 * k);
        word += __float_as_uint(m1) << (8 * k + 4);
    }
    if (dmax > 0.5f - 2e-6f) {  // near a tie somewhere in this word: exact divisions
        word = 0x88888888u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int q0 = exact_code(value_f32(h, k, 0), s, 7);
            const int q1 = exact_code(value_f32(h, k, 1), s, 7);
            word += static_cast<uint32_t>(q0) << (8 * k);
            word += static_cast<uint32_t>(q1) << (8 * k + 4);
        }
    }
    return word ^ 0x88888888u;
}

// Eight INT8 codes, one byte each in position order, from four half2 values
// (W4A8 activations; or four fp32 pairs): the fast path below for every
// value, and IEEE divisions for a word with any near-tie.
template <typename V>
__device__ __forceinline__ uint2 pack_codes8_i8(const V &h, float s, float rs) {
    uint32_t q[8];
    float dmax = 0.0f;
    const uint64_t rs2 = f2(rs, rs), kr2 = f2(kRound, kRound);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t v2 = pair_f32(h, k);
        const uint64_t m = f2_fma(v2, rs2, kr2);           // 1.5*2^23 + rint(v rs)
        const uint64_t r = f2_sub(m, kr2);
        float r0, r1;
        f2_split(r, r0, r1);
        const uint64_t d = f2_fma(v2, rs2, f2(-r0, -r1));  // v rs - rint(v rs)
        float m0, m1, d0, d1;
        f2_split(m, m0, m1);
        f2_split(d, d0, d1);
        dmax = max3(dmax, fabsf(d0), fabsf(d1));
        q[2 * k] = __float_as_uint(m0) - kRoundBits;        // the code, two's complement
        q[2 * k + 1] = __float_as_uint(m1) - kRoundBits;
    }
    if (dmax > 0.5f - 4e-5f) {  // near a tie somewhere in this word: exact divisions
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            q[2 * k] = static_cast<uint32_t>(exact_code(value_f32(h, k, 0), s, 127));
            q[2 * k + 1] = static_cast<uint32_t>(exact_code(value_f32(h, k, 1), s, 127));
        }
    }
    // low byte of each code, in order
    auto bytes4 = [](uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
        uint32_t ab, cd, r;
        asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(ab) : "r"(a), "r"(b));
        asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(cd) : "r"(c), "r"(d));
        asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(ab), "r"(cd));
        return r;
    };
    return make_uint2(bytes4(q[0], q[1], q[2], q[3]), bytes4(q[4], q[5], q[6], q[7]));
}

// INT8 outlier code (same fast path; |v/s| <= 127(1+u) gives an error bound
// of 2.3e-5 inside the 4e-5 tie margin).
__device__ __forceinline__ int code8(float v, float s, float rs) {
    const float m = __fmaf_rn(v, rs, kRound);
    const float r = __fsub_rn(m, kRound);
    if (fabsf(__fmaf_rn(v, rs, -r)) > 0.5f - 4e-5f) return exact_code(v, s, 127);
    return static_cast<int>(__float_as_uint(m) - kRoundBits);
}

// z = h * gamma for the eight values of one word (h: four half2 of the row,
// gamma: the word's eight reordered norm weights).  A product of two fp16
// values has at most 22 significant bits and lies within fp32's normal
// range, so every z is exact.
__device__ __forceinline__ void norm_products(const uint32_t (&h)[4], uint4 g, uint64_t (&z)[4]) {
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 gf = __half22float2(*reinterpret_cast<const __half2 *>(&gw[k]));
        z[k] = ptx::f2_mul(pair_f32(h, k), f2(gf.x, gf.y));
    }
}

// The norm's sum of squares, exact.  Every finite fp16 value is an integer
// multiple of 2^-24, so its square is an integer multiple of 2^-48 below
// 2^80, and at most 2^15 of them (K <= 24576) sum below 2^95: a 96-bit
// integer (lo, hi) in units of 2^-48 holds the sum exactly, whatever the
// order of the additions.  (Non-finite inputs give an unspecified sum.)
struct SumSq {
    uint64_t lo;
    uint32_t hi;
};

__device__ __forceinline__ void sumsq_add(SumSq &s, uint64_t lo, uint32_t hi) {
    s.lo += lo;
    s.hi += hi + (s.lo < lo ? 1u : 0u);
}

// h^2 of the fp16 bit pattern h16 (low 16 bits): h = m 2^(max(e,1) - 25)
// with m = f (e = 0) or 1024 + f, so h^2 = m^2 2^(sh - 48), sh = 2e - 2 (0
// for e = 0) <= 58.
__device__ __forceinline__ void sumsq_add_half(SumSq &s, uint32_t h16) {
    const uint32_t e = (h16 >> 10) & 31u, f = h16 & 1023u;
    const uint64_t m = e ? (f | 1024u) : f;
    const uint32_t sh = e ? 2u * e - 2u : 0u;
    const uint64_t m2 = m * m;  // < 2^22
    sumsq_add(s, m2 << sh, sh > 42u ? static_cast<uint32_t>(m2 >> (64u - sh)) : 0u);
}

__device__ __forceinline__ SumSq sumsq_warp(SumSq s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t lo = __shfl_xor_sync(0xffffffffu, s.lo, o);
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, s.hi, o);
        sumsq_add(s, lo, hi);
    }
    return s;
}

// The exact sum rounded once to fp64 (to nearest, ties to even).  Above 64
// bits the value is shifted right by n bits into 64, the bits shifted out
// folded into bit 0 (a sticky bit: the rounding position of a 64-bit
// significand is bit 11, so only a remainder's zero-or-not reaches it),
// converted by the correctly rounded 64-bit conversion, and scaled back by
// 2^n; both scalings by powers of two are exact.
__device__ __forceinline__ double sumsq_to_double(SumSq s) {
    if (s.hi == 0) return __dmul_rn(__ull2double_rn(s.lo), 0x1p-48);
    const int n = 32 - __clz(s.hi);  // 1 .. 31
    const uint64_t v = (static_cast<uint64_t>(s.hi) << (64 - n)) | (s.lo >> n) |
                       ((s.lo & ((1ull << n) - 1)) != 0 ? 1ull : 0ull);
    const double two_n48 = __longlong_as_double(static_cast<long long>(1023 + n - 48) << 52);
    return __dmul_rn(__ull2double_rn(v), two_n48);
}

// The RMS norm's row factor 1 / sqrt(ss / K + eps) in fp64, each step IEEE
// rounded, from ss = the exact sum of squares rounded once to fp64: the
// factor, and so the fp32 scales and fp16 outliers that carry it, do not
// depend on the order in which the row's values were summed.
__device__ __forceinline__ double rms_factor(double ss, int K, float eps) {
    return __drcp_rn(__dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(K)),
                                          static_cast<double>(eps))));
}
// fl32(s * r) and fl16(z * r): one fp64 product, rounded once.
__device__ __forceinline__ float times_r(float s, double r) {
    return __double2float_rn(__dmul_rn(static_cast<double>(s), r));
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

// Named barrier over one team (ids 1..4; id 0 is __syncthreads), returning
// the OR of `pred` over the team's threads.
__device__ __forceinline__ bool team_sync_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void team_sync(int id, int nthreads) {
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// P32: the perm table holds byte offsets (uint32); else element indices (uint16).
// NORM: the rows are first RMS-normalised with weight p.gamma and p.eps (the
// norm in front of a projection, with this quantiser folded into it: Atom,
// idea I2).  The row factor r = 1/sqrt(mean(h^2) + eps) changes no code, so
// codes and base scales are those of z = h * gamma (exact in fp32) and r
// multiplies the stored scales and the FP16 outliers.  A second shared table
// holds gamma in reordered order; the sum of squares is gathered alongside.
template <bool GROUPED, bool OUT_INT8, int W, bool P32, bool NORM>
__global__ void __launch_bounds__(kQMaxThreads) __maxnreg__(W > 4 ? 128 : (GROUPED && NORM) ? 96 : (GROUPED || NORM) ? 64 : 56)
    quantize_rows_kernel(QParams p) {
    extern __shared__ __align__(16) uint8_t qsmem[];
    __shared__ float red[kQMaxTeams][2][kQMaxThreads / 32];  // warp maxima, two slots per team
    __shared__ SumSq red_ss[kQMaxTeams][2][kQMaxThreads / 32];  // warp sums of squares (NORM)
    __shared__ uint64_t row_full[kQMaxTeams][kQMaxRing];
    __shared__ uint64_t stall_bar;  // never completed (quik_test_stall)
    const int K = p.K, Ki = K - p.k_o;  // K % 16 == 0
    const int TT = p.team_threads;
    const int team = threadIdx.x / TT, tl = threadIdx.x - team * TT;  // team-local thread
    const int lane = threadIdx.x & 31, twarp = tl >> 5;
    const int bar_id = 1 + team;
    const int nwords = Ki / 8;
    const int G = GROUPED ? Ki / kGroup : 1;
    const uint32_t row_bytes = static_cast<uint32_t>(K) * 2;
    const uint32_t perm_bytes = P32 ? row_bytes * 2 : row_bytes;
    // the reordered norm weights (fp16 [K]) follow the perm table
    const uint32_t tab_bytes = perm_bytes + (NORM ? row_bytes : 0u);
    const uint16_t *gtab = reinterpret_cast<const uint16_t *>(qsmem + perm_bytes);
    const int stride = gridDim.x * p.teams;  // rows between a team's consecutive rows
    const int first = blockIdx.x * p.teams + team;
    const int NR = p.ring;
    auto slot_off = [&](int t, int j) { return tab_bytes + (t * NR + j % NR) * row_bytes; };
    auto issue = [&](int t, int j) {  // bulk-copy team t's j-th row into its slot j % NR
        const int row = blockIdx.x * p.teams + t + j * stride;
        if (row < p.rows) {
            ptx::mbar_arrive_expect_tx(&row_full[t][j % NR], row_bytes);
            ptx::bulk_load(qsmem + slot_off(t, j), p.X + static_cast<size_t>(row) * K, row_bytes,
                           &row_full[t][j % NR]);
        }
    };
    __shared__ uint64_t perm_full;
    // a GEMM launched after this kernel with a programmatic dependency may be
    // scheduled now (it waits for this grid before it reads Xq and the scales)
    grid_launch_dependents();
    if (threadIdx.x == 0) {
        for (int t = 0; t < p.teams; ++t)
            for (int r = 0; r < NR; ++r) ptx::mbar_init(&row_full[t][r], 1);
        ptx::mbar_init(&perm_full, 1);
        ptx::mbar_init(&stall_bar, 1);
        ptx::fence_barrier_init();
        if (P32) {  // the int32 perm lands in the table area and is converted in place
            ptx::mbar_arrive_expect_tx(&perm_full, perm_bytes);
            ptx::bulk_load(qsmem, p.perm, perm_bytes, &perm_full);
        }
        for (int t = 0; t < p.teams; ++t)
            for (int r = 0; r < NR; ++r) issue(t, r);
    }
    // (0) the perm table, while the first rows are in flight
    bool perm_lost = false;  // the perm copy did not arrive in time
    {
        const unsigned uk = static_cast<unsigned>(K);
        bool bad = false;
        if (P32) {
            __syncthreads();  // perm_full initialised
            perm_lost = !ptx::mbar_wait_bounded_sleep(&perm_full, 0, kWaitLimitNs);
        }
        for (int i = threadIdx.x; i < K / 4; i += blockDim.x) {
            uint4 v;
            if (P32) {
                v = reinterpret_cast<const uint4 *>(qsmem)[i];
            } else {
                const int4 g = __ldg(reinterpret_cast<const int4 *>(p.perm) + i);
                v = make_uint4(static_cast<uint32_t>(g.x), static_cast<uint32_t>(g.y),
                               static_cast<uint32_t>(g.z), static_cast<uint32_t>(g.w));
            }
            uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                bad |= e[c] >= uk;
                e[c] = e[c] < uk ? e[c] : 0u;
            }
            if (P32)
                reinterpret_cast<uint4 *>(qsmem)[i] = make_uint4(2 * e[0], 2 * e[1], 2 * e[2], 2 * e[3]);
            else
                reinterpret_cast<uint2 *>(qsmem)[i] = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
            if (NORM) {
                uint32_t g[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) g[c] = __ldg(p.gamma + e[c]);
                reinterpret_cast<uint2 *>(qsmem + perm_bytes)[i] = make_uint2(g[0] | (g[1] << 16), g[2] | (g[3] << 16));
            }
        }
        if (bad && blockIdx.x == 0) atomicAdd(&g_quant_bad_perm, 1u);
    }
    // perm table and row barriers visible to all; if the perm copy was lost no
    // row is processed (a late copy could still overwrite the table)
    perm_lost = __syncthreads_or(perm_lost);
    if (perm_lost && threadIdx.x == 0) {
        atomicAdd(&g_quant_error, 1u);
        ptx::mbar_wait_bounded(&perm_full, 0, kWaitLimitNs);
    }
    if (team >= p.teams) return;

    int issued = 0;  // leader: this team's rows 0 .. issued-1 have been requested
    while (issued < NR && first + issued * stride < p.rows) ++issued;
    for (int j = 0; !perm_lost; ++j) {
        const int row = first + j * stride;
        if (row >= p.rows) break;
        // (1) the leader waits for this row (bounded); the barrier hands it to
        // the team and ends every thread's use of the previous slot
        bool ok = true;
        if (tl == 0)
            ok = (j == 0 && *reinterpret_cast<volatile int *>(&g_quant_stall) != 0)
                     ? ptx::mbar_wait_bounded_sleep(&stall_bar, 0, kWaitLimitNs)
                     : ptx::mbar_wait_bounded_sleep(&row_full[team][j % NR], (j / NR) & 1, kWaitLimitNs);
        if (team_sync_or(bar_id, TT, !ok)) {
            if (tl == 0) atomicAdd(&g_quant_error, 1u);
            break;
        }
        if (tl == 0 && j > 0) {  // the slot of row j-1 takes row j-1+NR
            issue(team, j - 1 + NR);
            if (first + (j - 1 + NR) * stride < p.rows) issued = j + NR;
        }
        const uint8_t *row_s = qsmem + slot_off(team, j);
        auto at = [&](uint32_t off) -> uint32_t { return *reinterpret_cast<const uint16_t *>(row_s + off); };
        auto element = [&](uint32_t k) -> uint32_t {  // byte offset of reordered position k
            if (P32) return reinterpret_cast<const uint32_t *>(qsmem)[k];
            return 2u * reinterpret_cast<const uint16_t *>(qsmem)[k];
        };

        // (2) gather 8 reordered values per word (as 4 half2), absmax per word
        // (of h * gamma with the norm, whose sum of squares of h is gathered too)
        uint32_t v[W][4];
        float wmax[W];
        SumSq ss = {0ull, 0u};  // exact sum of h^2 (NORM)
#pragma unroll
        for (int i = 0; i < W; ++i) {
            const int w = tl + i * TT;
            wmax[i] = 0.0f;
            if (w < nwords) {
                uint32_t off[8];
                if (P32) {
                    const uint4 a = reinterpret_cast<const uint4 *>(qsmem)[2 * w];
                    const uint4 b = reinterpret_cast<const uint4 *>(qsmem)[2 * w + 1];
                    off[0] = a.x; off[1] = a.y; off[2] = a.z; off[3] = a.w;
                    off[4] = b.x; off[5] = b.y; off[6] = b.z; off[7] = b.w;
                } else {
                    const uint4 a = reinterpret_cast<const uint4 *>(qsmem)[w];
                    const uint32_t x[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        off[2 * c] = 2u * (x[c] & 0xffffu);
                        off[2 * c + 1] = 2u * (x[c] >> 16);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) v[i][k] = pair16(at(off[2 * k]), at(off[2 * k + 1]));
                if (NORM) {
                    uint64_t z[4];
                    norm_products(v[i], reinterpret_cast<const uint4 *>(gtab)[w], z);
                    float a = 0.0f;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        sumsq_add_half(ss, v[i][k] & 0xffffu);
                        sumsq_add_half(ss, v[i][k] >> 16);
                        float z0, z1;
                        f2_split(z[k], z0, z1);
                        a = max3(a, fabsf(z0), fabsf(z1));
                    }
                    wmax[i] = a;
                } else {
                    wmax[i] = half2_absmax(absmax2(absmax2(v[i][0], v[i][1]), absmax2(v[i][2], v[i][3])));
                }
            }
        }
        // the norm's row factor: the sum of squares runs over every channel,
        // the outlier block included
        double rn = 1.0;
        if (NORM) {
            for (int i = tl; i < p.k_o; i += TT) sumsq_add_half(ss, at(element(Ki + i)));
            ss = sumsq_warp(ss);
            if (GROUPED) {  // the per-token path below shares the max's barrier
                if (lane == 0) red_ss[team][j & 1][twarp] = ss;
                team_sync(bar_id, TT);
                ss = SumSq{0ull, 0u};
                for (int k = 0; k < (TT >> 5); ++k) sumsq_add(ss, red_ss[team][j & 1][k].lo, red_ss[team][j & 1][k].hi);
                rn = rms_factor(sumsq_to_double(ss), K, p.eps);
            }
        }

        // (3) scales
        float s[W], r[W];
        if (GROUPED) {
#pragma unroll
            for (int i = 0; i < W; ++i) {
                float m = wmax[i];
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                s[i] = div_exact<7, 3>(m);
                r[i] = rcp_approx(s[i]);
                const int w = tl + i * TT;
                if (w < nwords && (lane & 15) == 0 && QUIK_CHECK(w / 16 < G, 3))
                    p.scale[static_cast<size_t>(row) * G + w / 16] = NORM ? times_r(s[i], rn) : s[i];
            }
        } else {
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < W; ++i) m = fmaxf(m, wmax[i]);
            m = warp_max(m);
            if (lane == 0) {
                red[team][j & 1][twarp] = m;
                if (NORM) red_ss[team][j & 1][twarp] = ss;
            }
            team_sync(bar_id, TT);
            m = 0.0f;
            for (int k = 0; k < (TT >> 5); ++k) m = fmaxf(m, red[team][j & 1][k]);
            if (NORM) {
                ss = SumSq{0ull, 0u};
                for (int k = 0; k < (TT >> 5); ++k) sumsq_add(ss, red_ss[team][j & 1][k].lo, red_ss[team][j & 1][k].hi);
                rn = rms_factor(sumsq_to_double(ss), K, p.eps);
            }
            const float sr = p.bits8 ? div_exact<127, 7>(m) : div_exact<7, 3>(m), rr = rcp_approx(sr);
#pragma unroll
            for (int i = 0; i < W; ++i) {
                s[i] = sr;
                r[i] = rr;
            }
            if (tl == 0) p.scale[row] = NORM ? times_r(sr, rn) : sr;
        }

        // (4) codes, 8 per word, code 2i in the low nibble of byte i (or one
        // byte per code for INT8 activations)
        if (!GROUPED && p.bits8) {
            uint2 *qrow8 = reinterpret_cast<uint2 *>(p.Q + static_cast<size_t>(row) * Ki);
#pragma unroll
            for (int i = 0; i < W; ++i) {
                const int w = tl + i * TT;
                if (w < nwords && QUIK_CHECK(8 * w + 8 <= Ki, 4)) {
                    if (NORM) {
                        uint64_t z[4];
                        norm_products(v[i], reinterpret_cast<const uint4 *>(gtab)[w], z);
                        qrow8[w] = pack_codes8_i8(z, s[i], r[i]);
                    } else {
                        qrow8[w] = pack_codes8_i8(v[i], s[i], r[i]);
                    }
                }
            }
        } else if (!GROUPED && p.wide) {
            // one signed byte 16 c per code; per 32 positions, the 16 even ones
            // then the 16 odd ones (the order in which the GEMM widens packed
            // weights, so both operands share one K order)
            uint8_t *qrow = p.Q + static_cast<size_t>(row) * Ki;
#pragma unroll
            for (int i = 0; i < W; ++i) {
                const int w = tl + i * TT;
                if (w < nwords && QUIK_CHECK(8 * w + 8 <= Ki, 4)) {
                    uint32_t word;
                    if (NORM) {
                        uint64_t z[4];
                        norm_products(v[i], reinterpret_cast<const uint4 *>(gtab)[w], z);
                        word = pack_codes8(z, s[i], r[i]);
                    } else {
                        word = pack_codes8(v[i], s[i], r[i]);
                    }
                    uint32_t *g = reinterpret_cast<uint32_t *>(qrow + 32 * (w >> 2)) + (w & 3);
                    g[0] = (word << 4) & 0xF0F0F0F0u;  // codes 8w, 8w+2, 8w+4, 8w+6
                    g[4] = word & 0xF0F0F0F0u;         // codes 8w+1, 8w+3, 8w+5, 8w+7
                }
            }
        } else {
            uint32_t *qrow = reinterpret_cast<uint32_t *>(p.Q + static_cast<size_t>(row) * (Ki / 2));
#pragma unroll
            for (int i = 0; i < W; ++i) {
                const int w = tl + i * TT;
                if (w < nwords && QUIK_CHECK(4 * w + 4 <= Ki / 2, 4)) {
                    if (NORM) {
                        uint64_t z[4];
                        norm_products(v[i], reinterpret_cast<const uint4 *>(gtab)[w], z);
                        qrow[w] = pack_codes8(z, s[i], r[i]);
                    } else {
                        qrow[w] = pack_codes8(v[i], s[i], r[i]);
                    }
                }
            }
        }

        // (5) the outlier block
        if (p.k_o > 0) {
            if (!OUT_INT8) {
                uint16_t *o = static_cast<uint16_t *>(p.O) + static_cast<size_t>(row) * p.k_o;
                for (int i = tl; i < p.k_o; i += TT) {
                    if (NORM) {  // fl16(h * gamma * r), the product in fp64
                        const float z = __fmul_rn(h2f(static_cast<uint16_t>(at(element(Ki + i)))),
                                                  h2f(gtab[Ki + i]));
                        o[i] = __half_as_ushort(__double2half(__dmul_rn(static_cast<double>(z), rn)));
                    } else {
                        o[i] = static_cast<uint16_t>(at(element(Ki + i)));
                    }
                }
            } else {
                // the outlier values (times gamma with the norm: exact)
                auto ov = [&](int i) -> float {
                    const float h = h2f(static_cast<uint16_t>(at(element(Ki + i))));
                    return NORM ? __fmul_rn(h, h2f(gtab[Ki + i])) : h;
                };
                float m = 0.0f;
                for (int i = tl; i < p.k_o; i += TT) m = fmaxf(m, fabsf(ov(i)));
                m = warp_max(m);
                // the other reduction slot: this row's slot is read above and
                // is not written again before the next row's opening barrier
                if (lane == 0) red[team][(j & 1) ^ 1][twarp] = m;
                team_sync(bar_id, TT);
                m = 0.0f;
                for (int k = 0; k < (TT >> 5); ++k) m = fmaxf(m, red[team][(j & 1) ^ 1][k]);
                const float so = div_exact<127, 7>(m), rso = rcp_approx(so);
                if (tl == 0) p.o_scale[row] = NORM ? times_r(so, rn) : so;
                int8_t *o = static_cast<int8_t *>(p.O) + static_cast<size_t>(row) * p.k_o;
                for (int i = tl; i < p.k_o; i += TT) o[i] = static_cast<int8_t>(code8(ov(i), so, rso));
            }
        } else if (OUT_INT8 && p.o_scale != nullptr && tl == 0) {
            p.o_scale[row] = 0.0f;
        }
    }
    // never leave the CTA with a bulk copy still writing its shared memory:
    // wait for the last row requested into each of the team's slots
    if (tl == 0)
        for (int j = issued > NR ? issued - NR : 0; j < issued; ++j)
            ptx::mbar_wait_bounded(&row_full[team][j % NR], (j / NR) & 1, kWaitLimitNs);
}

struct QShape {
    int W, TT, teams, ring;
    bool p32;
    size_t smem;
};

// Registers per thread of one kernel instance (queried once), and the
// static shared memory it holds beyond the 1 KB that ctas_per_sm assumes.
template <bool GROUPED, bool OUT_INT8, int W, bool P32, bool NORM>
int q_regs(size_t *extra_static = nullptr) {
    static std::atomic<int> regs{0};
    static std::atomic<int> extra{0};
    int r = regs.load(std::memory_order_relaxed);
    if (r == 0) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, quantize_rows_kernel<GROUPED, OUT_INT8, W, P32, NORM>) != cudaSuccess)
            return 0;
        extra.store(fa.sharedSizeBytes > 1024 ? static_cast<int>(fa.sharedSizeBytes - 1024) : 0,
                    std::memory_order_relaxed);
        r = fa.numRegs;
        regs.store(r, std::memory_order_relaxed);
    }
    if (extra_static != nullptr) *extra_static = static_cast<size_t>(extra.load(std::memory_order_relaxed));
    return r;
}

// CTAs of `threads` threads, `regs` registers each and `smem` bytes of
// dynamic shared memory that fit on one SM (sm_100: 64 K registers allocated
// per warp in units of 256, 2048 threads, 228 KB of shared memory with 1 KB
// reserved per CTA).
int ctas_per_sm(int threads, int regs, size_t smem) {
    if (regs <= 0) return 0;
    const int warps = (threads + 31) / 32;
    const int regs_per_warp = ((regs * 32 + 255) / 256) * 256;
    const int by_regs = 65536 / (regs_per_warp * warps);
    const int by_threads = 2048 / (warps * 32);
    const int by_smem = static_cast<int>((228u << 10) / (smem + 1024 + 1024));  // + static shared memory
    return std::max(0, std::min(std::min(by_regs, by_threads), std::min(by_smem, 32)));
}

// W (words per thread): with few rows per SM (at most two), the fewest that
// fit one row in 16 warps, for the shortest row latency; otherwise the fewest
// that keep a team at 4 warps, up to 16 warps at W = 4 (K_i <= 16384), then
// W = 8 (K_i <= 32768).  Then teams per CTA (at most 4 and 512 threads), row
// slots per team (2 .. 4) and the perm table's width (uint32 byte offsets, or
// uint16 indices with an extraction per element) are chosen for the most
// teams per SM; ties go to the uint32 table, then to more slots.  With the
// fused norm a second table (the reordered norm weights, one row's size)
// shares the shared memory.
template <bool GROUPED, bool OUT_INT8, bool NORM>
QShape q_shape(int rows, int K, int k_o) {
    const int nwords = (K - k_o) / 8;
    int W;
    if (rows <= 2 * sm_count())
        W = nwords <= 512 ? 1 : nwords <= 1024 ? 2 : nwords <= 2048 ? 4 : 8;
    else
        W = nwords <= 128 ? 1 : nwords <= 256 ? 2 : nwords <= 2048 ? 4 : 8;
    const int TT = std::max(32, 32 * ((nwords + 32 * W - 1) / (32 * W)));
    const size_t row = static_cast<size_t>(K) * 2;
    QShape best{W, TT, 0, 0, true, 0};
    int best_score = -1;
    for (int p32 = 1; p32 >= 0; --p32) {
        int regs = 0;
        size_t xs = 0;  // static shared memory past 1 KB
        switch (W) {
            case 1: regs = p32 ? q_regs<GROUPED, OUT_INT8, 1, true, NORM>(&xs) : q_regs<GROUPED, OUT_INT8, 1, false, NORM>(&xs); break;
            case 2: regs = p32 ? q_regs<GROUPED, OUT_INT8, 2, true, NORM>(&xs) : q_regs<GROUPED, OUT_INT8, 2, false, NORM>(&xs); break;
            case 4: regs = p32 ? q_regs<GROUPED, OUT_INT8, 4, true, NORM>(&xs) : q_regs<GROUPED, OUT_INT8, 4, false, NORM>(&xs); break;
            default: regs = p32 ? q_regs<GROUPED, OUT_INT8, 8, true, NORM>(&xs) : q_regs<GROUPED, OUT_INT8, 8, false, NORM>(&xs); break;
        }
        const size_t table = (p32 ? 2 * row : row) + (NORM ? row : 0);
        for (int teams = std::min(kQMaxTeams, kQMaxThreads / TT); teams >= 1; --teams)
            for (int ring = kQMaxRing; ring >= 2; --ring) {
                const size_t smem = table + static_cast<size_t>(teams) * ring * row;
                if (smem + xs > (227u << 10) - 1024) continue;
                const int per_sm = ctas_per_sm(TT * teams, regs, smem + xs);
                if (per_sm == 0) continue;
                // teams per SM first; then the wider table; then deeper rings
                const int score = (per_sm * teams) * 16 + p32 * 8 + ring;
                if (score > best_score) {
                    best_score = score;
                    best = QShape{W, TT, teams, ring, p32 != 0, smem};
                }
            }
    }
    return best;
}

template <bool GROUPED, bool OUT_INT8, int W, bool P32, bool NORM>
cudaError_t launch_q(QParams p, const QShape &qs, cudaStream_t stream) {
    auto kern = quantize_rows_kernel<GROUPED, OUT_INT8, W, P32, NORM>;
    p.team_threads = qs.TT;
    p.teams = qs.teams;
    p.ring = qs.ring;
    const int threads = qs.TT * qs.teams;
    if (qs.teams < 1 || qs.ring < 2 || qs.ring > kQMaxRing || threads > kQMaxThreads ||
        qs.smem > (227u << 10))
        return cudaErrorInvalidConfiguration;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), static_cast<int>(qs.smem)))
        return cudaErrorInvalidConfiguration;
    size_t xs = 0;
    const int per_sm = ctas_per_sm(threads, q_regs<GROUPED, OUT_INT8, W, P32, NORM>(&xs), qs.smem + xs);
    // grid: every CTA that fits at once (persistent), or fewer when the rows run out
    const int need = (p.rows + qs.teams - 1) / qs.teams;
    const int grid = std::max(1, std::min(need, sm_count() * std::max(per_sm, 1)));
    kern<<<grid, threads, qs.smem, stream>>>(p);
    return cudaGetLastError();
}

template <bool GROUPED, bool OUT_INT8, bool NORM>
cudaError_t launch_q_w(const QParams &p, cudaStream_t stream) {
    const QShape qs = q_shape<GROUPED, OUT_INT8, NORM>(p.rows, p.K, p.k_o);
    switch (qs.W * 2 + (qs.p32 ? 1 : 0)) {
        case 3: return launch_q<GROUPED, OUT_INT8, 1, true, NORM>(p, qs, stream);
        case 2: return launch_q<GROUPED, OUT_INT8, 1, false, NORM>(p, qs, stream);
        case 5: return launch_q<GROUPED, OUT_INT8, 2, true, NORM>(p, qs, stream);
        case 4: return launch_q<GROUPED, OUT_INT8, 2, false, NORM>(p, qs, stream);
        case 9: return launch_q<GROUPED, OUT_INT8, 4, true, NORM>(p, qs, stream);
        case 8: return launch_q<GROUPED, OUT_INT8, 4, false, NORM>(p, qs, stream);
        case 17: return launch_q<GROUPED, OUT_INT8, 8, true, NORM>(p, qs, stream);
        default: return launch_q<GROUPED, OUT_INT8, 8, false, NORM>(p, qs, stream);
    }
}

template <bool NORM>
cudaError_t launch_q_n(const QParams &p, int group, bool out_int8, cudaStream_t stream) {
    if (group > 0)
        return out_int8 ? launch_q_w<true, true, NORM>(p, stream) : launch_q_w<true, false, NORM>(p, stream);
    return out_int8 ? launch_q_w<false, true, NORM>(p, stream) : launch_q_w<false, false, NORM>(p, stream);
}

// ----------------------------------------------------------------- 2:4-sparse weight rows
// The offline pack of 2:4-sparse INT4 weights ("QUIK" abstract: quantisation
// plus 2:4 sparsity).  One CTA of 256 threads per row, plain code: the
// reordered row is gathered into shared memory (fp16), the row's absmax over
// the INT4 positions gives s = fl(m / 7); every aligned group of four keeps
// its two largest magnitudes (lower position on ties) with codes
// clamp(rint(v / s), -7, 7) from IEEE divisions; the outlier block is copied
// (FP16) or quantised with fl(max / 127) (INT8).
constexpr int kP24Threads = 256;

__device__ __forceinline__ float block_max(float m, float *red) {
    m = warp_max(m);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = m;
    __syncthreads();
    m = 0.0f;
    for (int i = 0; i < kP24Threads / 32; ++i) m = fmaxf(m, red[i]);
    __syncthreads();  // red is reused
    return m;
}

__global__ void __launch_bounds__(kP24Threads) prune24_rows_kernel(Prune24Args a) {
    extern __shared__ uint16_t row_s[];  // the reordered row, K fp16 values
    __shared__ float red[kP24Threads / 32];
    const int K = a.K, Ki = K - a.k_o, row = blockIdx.x;
    const uint16_t *x = a.W + static_cast<size_t>(row) * K;
    bool bad = false;
    for (int j = threadIdx.x; j < K; j += kP24Threads) {
        const int c = a.perm[j];
        bad |= c < 0 || c >= K;
        row_s[j] = (c >= 0 && c < K) ? x[c] : static_cast<uint16_t>(0);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0 && row == 0) atomicAdd(&g_quant_bad_perm, 1u);
    float m = 0.0f;
    for (int j = threadIdx.x; j < Ki; j += kP24Threads) m = fmaxf(m, fabsf(h2f(row_s[j])));
    const float s = __fdiv_rn(block_max(m, red), 7.0f);
    if (threadIdx.x == 0 && a.scale != nullptr) a.scale[row] = s;  // may be NULL when K_i == 0
    // two groups (one metadata byte) per step
    for (int u = threadIdx.x; u < Ki / 8; u += kP24Threads) {
        uint32_t nibs = 0;
        for (int h = 0; h < 2; ++h) {
            const int t = 2 * u + h;
            float g[4];
            for (int i = 0; i < 4; ++i) g[i] = h2f(row_s[4 * t + i]);
            int ka = 0;
            for (int i = 1; i < 4; ++i)
                if (fabsf(g[i]) > fabsf(g[ka])) ka = i;
            int kb = -1;
            for (int i = 0; i < 4; ++i)
                if (i != ka && (kb < 0 || fabsf(g[i]) > fabsf(g[kb]))) kb = i;
            const int i0 = min(ka, kb), i1 = max(ka, kb);
            const int q0 = exact_code(g[i0], s, 7), q1 = exact_code(g[i1], s, 7);
            a.Qs[static_cast<size_t>(row) * (Ki / 4) + t] =
                static_cast<uint8_t>((q0 & 0xF) | ((q1 & 0xF) << 4));
            nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * h);
        }
        a.meta[static_cast<size_t>(row) * (Ki / 8) + u] = static_cast<uint8_t>(nibs);
    }
    if (a.k_o > 0) {
        if (!a.out_int8) {
            uint16_t *o = static_cast<uint16_t *>(a.O) + static_cast<size_t>(row) * a.k_o;
            for (int i = threadIdx.x; i < a.k_o; i += kP24Threads) o[i] = row_s[Ki + i];
        } else {
            float om = 0.0f;
            for (int i = threadIdx.x; i < a.k_o; i += kP24Threads) om = fmaxf(om, fabsf(h2f(row_s[Ki + i])));
            const float so = __fdiv_rn(block_max(om, red), 127.0f);
            if (threadIdx.x == 0) a.o_scale[row] = so;
            int8_t *o = static_cast<int8_t *>(a.O) + static_cast<size_t>(row) * a.k_o;
            for (int i = threadIdx.x; i < a.k_o; i += kP24Threads)
                o[i] = static_cast<int8_t>(exact_code(h2f(row_s[Ki + i]), so, 127));
        }
    } else if (a.out_int8 && a.o_scale != nullptr && threadIdx.x == 0) {
        a.o_scale[row] = 0.0f;
    }
}

// The dense packed INT4 rows [rows, K_i / 2] that 2:4 rows stand for: the
// two kept codes of every group at their positions, zero elsewhere.  One
// thread per four metadata bytes: eight groups, 32 positions, 16 bytes of the
// dense row (every row pitch is a multiple of 16 bytes for K_i % 128 == 0).
__global__ void expand24_kernel(const uint8_t *__restrict__ Qs, const uint8_t *__restrict__ meta,
                                long long total, int Ki, uint4 *__restrict__ Q) {
    const int per_row = Ki / 32;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long row = i / per_row;
        const int u = static_cast<int>(i - row * per_row);
        const uint32_t m4 = *reinterpret_cast<const uint32_t *>(meta + row * (Ki / 8) + 4 * u);
        const uint2 q8 = *reinterpret_cast<const uint2 *>(Qs + row * (Ki / 4) + 8 * u);
        uint32_t out[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {  // metadata byte w: groups 2w and 2w + 1
            const uint32_t m = (m4 >> (8 * w)) & 0xFFu;
            const uint32_t qw = w < 2 ? q8.x : q8.y;  // their kept-code bytes
            uint32_t word = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t nib = (m >> (4 * h)) & 0xFu;
                const uint32_t codes = (qw >> (8 * (2 * (w & 1) + h))) & 0xFFu;
                const int p0 = 4 * h + static_cast<int>(nib & 3u), p1 = 4 * h + static_cast<int>(nib >> 2);
                word |= (codes & 0xFu) << (4 * p0);
                word |= (codes >> 4) << (4 * p1);
            }
            out[w] = word;
        }
        Q[row * (Ki / 32) + u] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

}  // namespace

cudaError_t launch_quantize_rows(const QuantizeArgs &a, cudaStream_t stream) {
    QParams p{a.X, a.perm, a.rows, a.K, a.k_o, 0, 0, 0, a.Q, a.scale, a.O, a.o_scale, a.bits8 ? 1 : 0,
              a.wide ? 1 : 0, a.gamma, a.eps};
    // INT8 codes and the wide INT4 form: per-row scales only
    if ((a.bits8 || a.wide) && a.group > 0) return cudaErrorInvalidValue;
    if (a.bits8 && a.wide) return cudaErrorInvalidValue;
    if (a.gamma != nullptr) return launch_q_n<true>(p, a.group, a.out_int8, stream);
    return launch_q_n<false>(p, a.group, a.out_int8, stream);
}

cudaError_t launch_prune24_rows(const Prune24Args &a, cudaStream_t stream) {
    if ((a.K - a.k_o) % 8 != 0) return cudaErrorInvalidValue;
    const int smem = a.K * 2;
    if (!attribute_set_once(reinterpret_cast<const void *>(prune24_rows_kernel), smem))
        return cudaErrorInvalidConfiguration;
    prune24_rows_kernel<<<a.rows, kP24Threads, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_expand24(const uint8_t *Qs, const uint8_t *meta, int rows, int Ki, uint8_t *Q,
                            cudaStream_t stream) {
    if (Ki % 128 != 0) return cudaErrorInvalidValue;
    const long long total = static_cast<long long>(rows) * (Ki / 32);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const long long want = (total + threads - 1) / threads;
    const int grid = static_cast<int>(want < 8LL * sm_count() ? want : 8LL * sm_count());
    expand24_kernel<<<grid, threads, 0, stream>>>(Qs, meta, total, Ki, reinterpret_cast<uint4 *>(Q));
    return cudaGetLastError();
}

cudaError_t set_quantize_stall(int on) {
    return cudaMemcpyToSymbol(g_quant_stall, &on, sizeof(on));
}

unsigned int take_quantize_errors(unsigned int *bad_perm) {
    unsigned int word = 0, bad = 0;
    if (cudaMemcpyFromSymbol(&word, g_quant_error, sizeof(word)) != cudaSuccess) return 0;
    if (cudaMemcpyFromSymbol(&bad, g_quant_bad_perm, sizeof(bad)) != cudaSuccess) return 0;
    if (bad_perm != nullptr) *bad_perm = counter_increase(kCounterBadPerm, bad);
    return counter_increase(kCounterQuantWaits, word);
}

}  // namespace quik

#ifdef QUIK_CHECKS
extern "C" __attribute__((visibility("default"))) unsigned long long qchk_quantize_word() {
    unsigned long long v = 0;
    cudaMemcpyFromSymbol(&v, quik::g_check_word, sizeof(v));
    return v;
}
#endif
