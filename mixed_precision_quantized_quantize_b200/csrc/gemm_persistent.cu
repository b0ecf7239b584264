// gemm_persistent.cu -- the per-channel-scale W4A4 product with FP16
// outliers as a persistent, warp-specialised kernel on CTA pairs.
//
// Computes Y[m,n] = A[m,n] sx[m] sw[n] + O[m,n] + bias[n] (QUIK abstract;
// "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
// summary and idea I1), A the exact INT4 x INT4 sum, O the FP16 outlier
// product in fp32.
//
// Orientation.  The MMA's 256-row operand is W (each CTA of a pair holds 128
// output channels), its N is 256 tokens (128 per CTA), so D[n, m] sits in
// tensor memory with one output channel per lane.  W needs unpacking (INT4 ->
// the signed byte 16 c); the activations arrive by TMA straight into the
// 128-byte-swizzled operand layout, either as bytes 16 c written by
// quik_linear's quantiser (no unpack in this kernel) or, for quik_gemm's packed
// Xq, through the same unpack as W.  Both operands sit in shared memory; the
// tensor core's operand reads barely compete with the unpack warps' loads and
// stores (measured: SS MMAs plus ~120 B/clk of LDS/STS traffic slow each
// other by under 10 %), while tensor memory is left entirely to two
// accumulators of 256 columns, so a tile's epilogue overlaps the next tile's
// main loop.
//
// FP16 outliers use the same accumulator: once a tile's INT4 k-blocks are
// done, the epilogue rescales the integer sums in place to fp32
// y = A sx sw + bias (tcgen05.ld / tcgen05.st), and the outlier MMAs
// (kind::f16) accumulate onto y.  Those MMAs are issued a few k-blocks into
// the next tile, by which time the rescale is done, so the tensor pipe does
// not wait for it.
//
// Warps (each CTA):
//   0      TMEM allocation (both CTAs); the leader's lane 0 issues the MMAs
//   1      TMA producer of the operand stages: activation tiles (16 c bytes),
//          outlier tiles (Wo, Xo fp16, 128-byte swizzled)
//   2      TMA producer of the packed staging ring (W, and packed X for
//          quik_gemm)
//   3-6    unpack packed tiles into the operand stages
//   7-14   epilogue: two warps per TMEM lane quadrant, one per column half
// The leader's "operand full" barrier counts the unpack warps of both CTAs;
// each unpack warp arrives once it has written its part and seen its CTA's
// TMA tiles land.  MMA completion reaches both CTAs by multicast commits.
// Tiles are 256 output channels x 256 tokens, token tiles fastest, taken
// round-robin by the pairs.  Every wait is bounded (2 s); on expiry the CTA
// counts it in g_pgemm_error, stops, drains its copies and MMAs and exits.
#include <algorithm>
#include <cstring>

#include <cuda_fp16.h>

#include "quik_internal.h"
#include "sm100.cuh"

namespace quik {

// Expired waits in this file's kernel.  It only grows; quik_sync_check
// reports its increase.
__device__ unsigned int g_pgemm_error;
// Test entry (quik_test_stall): nonzero makes the MMA issuer wait first on a
// barrier that nothing completes, so its bounded wait runs out and every role
// of every CTA takes the abort path.
__device__ int g_pgemm_stall;

// Optional pipeline timeline (build with -DQUIK_TRACE): SM clock stamps of
// each role's events per work unit, for the first pair of a launch.
#ifdef QUIK_TRACE
constexpr int kPtEvents = 16, kPtUnits = 128;  // 10-15: six unpack warps' arrivals
__device__ unsigned long long g_ptrace[2][kPtEvents][kPtUnits];
#define PTRACE(ev, i)                                                                          \
    do {                                                                                       \
        if (blockIdx.x < 2 && (i) >= 0 && (i) < kPtUnits) g_ptrace[blockIdx.x][ev][i] = clock64(); \
    } while (0)
#else
#define PTRACE(ev, i) \
    do {              \
    } while (0)
#endif
// events: 0 operand producer issued unit u, 1 staging producer issued INT4
// unit q, 2 unpack passed op_empty, 3 unpack passed pk_full, 4 unpack wrote
// its part, 5 unpack arrived on op_full, 6 MMA issued unit u, 7 epilogue
// (4 j + 0: int_done seen, + 1 rescaled, + 2 acc_full seen, + 3 stored),
// 8 start (0: clock64, 1: globaltimer)

namespace {

using namespace ptx;

namespace pk {
constexpr int BW = 128;            // output channels per CTA (the pair's MMA has M = 256)
constexpr int BT = 256;            // tokens per pair tile: the MMA's N
constexpr int BTH = BT / 2;        // tokens per CTA (its half of the B operand)
constexpr int KB = 128;            // codes per k-block
constexpr int ROW = 128;           // operand bytes per row and k-block (one swizzle row)
constexpr int PKROW = 64;          // packed bytes per row and k-block
constexpr int OKB = 64;            // fp16 outlier channels per outlier unit (128 bytes)
constexpr int A_BYTES = BW * ROW;  // 16 KB
constexpr int B_BYTES = BTH * ROW; // 16 KB
constexpr int STAGE = A_BYTES + B_BYTES;
// Warp w runs on scheduler w % 4.  The three single-thread roles, whose
// polling would slow a compute warp sharing their scheduler (measured: an
// unpack warp next to a polling role ran 1.5 K cycles late per k-block),
// share scheduler 0: warp 0 issues the MMAs, warp 4 produces the operand
// stages, warp 8 the packed staging ring.  The unpack warps are the nine
// others below 12 (schedulers 1-3), in three groups of three (warps 4g+1 ..
// 4g+3) that take the work units in turn, so each group's per-unit waits and
// hand-offs overlap the other groups' unpacking.  Warps 12-15 are the
// epilogue, one per TMEM lane quadrant (warp % 4 is the quadrant a warp may
// access).
constexpr int NG = 3, GW = 3;      // unpack groups, warps per group
constexpr int GT = 32 * GW;        // threads per unpack group
constexpr int NE = 4;              // epilogue warps
constexpr int W_MMA = 0, W_XPROD = 4, W_PPROD = 8, W_EPI = 12;
constexpr int THREADS = 16 * 32;
constexpr int OUT_DELAY = 6;       // INT4 units of tile j before tile j-1's outlier units
constexpr int TMEM_COLS = 512;     // two accumulators of 256 columns
__host__ __device__ constexpr bool is_unpack_warp(int w) { return w < W_EPI && (w & 3) != 0; }
__host__ __device__ constexpr int unpack_group(int w) { return w >> 2; }
__host__ __device__ constexpr int unpack_lane0(int w) { return 32 * ((w & 3) - 1); }  // first thread in the group
static_assert(unpack_group(11) == NG - 1 && W_EPI + NE == 16, "warp layout");
}  // namespace pk

template <bool X4>
struct PkCfg {
    static constexpr int S = X4 ? 4 : 5;   // operand stages (32 KB each)
    static constexpr int SP = X4 ? 5 : 6;  // packed staging units
    static constexpr int UNIT = (X4 ? 2 : 1) * pk::BW * pk::PKROW;  // W (+ X) packed k-block
    static constexpr int PK_OFF = S * pk::STAGE;
    static constexpr int EPI_OFF = PK_OFF + SP * UNIT;  // per epilogue warp: 32 x 32 fp16 output tile
    static constexpr int EPI_TILE = 32 * 32 * 2;
    static constexpr int SMEM = EPI_OFF + pk::NE * EPI_TILE + 1024;  // + alignment slack
    static_assert(SMEM + 4096 <= 232448, "shared memory budget (dynamic + static)");
};

struct PParams {
    int M, N, Ki;
    int nkb_i;   // INT4 k-blocks (>= 1)
    int nkb_o;   // fp16 outlier units of 64 channels (0: none)
    int n_tt;    // token tiles
    int ntiles;  // tiles of the whole product
    int tma_y;   // Y leaves by TMA stores of 32 x 32 tiles (N % 8 == 0); else by plain stores
    const float *sx, *sw;
    const uint16_t *bias;
    uint16_t *Y;
    int32_t *acc_dbg;  // DEBUG: the integer sums [M, N]
};

struct Abort {
    volatile int *flag;  // this CTA has given up (shared memory)
    unsigned err0;       // g_pgemm_error when this CTA started
};

// Bounded wait.  Gives up at once when another role of this CTA has given up
// or when any CTA has recorded an expired wait since this CTA started (those
// checks run every 16th poll).
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, const Abort &ab) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) != 0) continue;
        if (*ab.flag) return false;
        if (*reinterpret_cast<volatile unsigned *>(&g_pgemm_error) != ab.err0) {
            *ab.flag = 1;
            return false;
        }
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *ab.flag = 1;
            atomicAdd(&g_pgemm_error, 1u);
            return false;
        }
    }
}

// The TMA producers' wait: between polls the thread sleeps, so that the MMA
// issuer, which shares their scheduler, keeps its issue slots (a producer's
// latency is hidden by the stages it runs ahead of the MMA).
__device__ __forceinline__ bool wait_bar_lazy(uint64_t *bar, uint32_t parity, const Abort &ab) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) != 0) continue;
        if (*ab.flag) return false;
        if (*reinterpret_cast<volatile unsigned *>(&g_pgemm_error) != ab.err0) {
            *ab.flag = 1;
            return false;
        }
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *ab.flag = 1;
            atomicAdd(&g_pgemm_error, 1u);
            return false;
        }
    }
}

// The epilogue's waits span a tile's main loop: lane 0 polls lazily and the
// rest of the warp waits at the warp barrier, so the warp leaves the issue
// slots of its scheduler (shared with the MMA issuer or an unpack group) free.
__device__ __forceinline__ bool warp_wait_lazy(uint64_t *bar, uint32_t parity, const Abort &ab, int lane) {
    int ok = 1;
    if (lane == 0) ok = wait_bar_lazy(bar, parity, ab) ? 1 : 0;
    __syncwarp();
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// A warp's wait: every lane polls and the warp agrees on the outcome
// (measured faster than one polling lane with the others parked at a warp
// barrier).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const Abort &ab) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, ab));
}

// Exact int32 -> fp32 for |v| < 2^22: place v in the mantissa of 1.5 * 2^23.
__device__ __forceinline__ float int_to_float_exact(int32_t v) {
    return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// y = A sx[m] sw + bias for one 32-column chunk, A = acc >> 8 (the INT4 codes
// enter the MMA as 16 c): pairs of columns in paired fp32 arithmetic, the
// scaling and the bias in one fused multiply-add per pair.
__device__ __forceinline__ void dequant32(uint32_t (&a)[32], const float *sx, float sw, float bias) {
    const uint64_t sw2 = f2(sw, sw), b2 = f2(bias, bias);
#pragma unroll
    for (int jj = 0; jj < 32; jj += 2) {
        const float2 s = *reinterpret_cast<const float2 *>(sx + jj);
        const uint64_t v = f2_mul(f2(int_to_float_exact(static_cast<int32_t>(a[jj]) >> 8),
                                     int_to_float_exact(static_cast<int32_t>(a[jj + 1]) >> 8)),
                                  f2(s.x, s.y));
        float y0, y1;
        f2_split(f2_fma(v, sw2, b2), y0, y1);
        a[jj] = __float_as_uint(y0);
        a[jj + 1] = __float_as_uint(y1);
    }
}

// 32 packed codes (16 bytes) -> the signed bytes 16 c: even positions in the
// first 16 bytes, odd positions in the next 16 (the same order on both
// operands, so every dot product is unchanged).
__device__ __forceinline__ void widen16(const uint4 v, uint4 &lo, uint4 &hi) {
    lo.x = (v.x << 4) & 0xF0F0F0F0u;  hi.x = v.x & 0xF0F0F0F0u;
    lo.y = (v.y << 4) & 0xF0F0F0F0u;  hi.y = v.y & 0xF0F0F0F0u;
    lo.z = (v.z << 4) & 0xF0F0F0F0u;  hi.z = v.z & 0xF0F0F0F0u;
    lo.w = (v.w << 4) & 0xF0F0F0F0u;  hi.w = v.w & 0xF0F0F0F0u;
}

// One packed k-block of 128 rows (64 bytes each) into the 128-byte-swizzled
// K-major operand layout (chunk c of row r at chunk c ^ (r % 8)): 512
// 16-byte chunks over one unpack group's threads.  Consecutive threads take
// consecutive chunks, so a warp's loads cover 512 contiguous bytes and each
// group of eight stores hits eight distinct chunk columns: no bank conflicts.
__device__ __forceinline__ void unpack_rows(const uint8_t *pk, uint8_t *dst, int tg) {
#pragma unroll
    for (int i = 0; i < (512 + pk::GT - 1) / pk::GT; ++i) {
        const int c = tg + pk::GT * i;
        if (c >= 512) break;
        const int row = c >> 2, ch = c & 3;
        const uint4 v = *reinterpret_cast<const uint4 *>(pk + row * pk::PKROW + ch * 16);
        uint4 lo, hi;
        widen16(v, lo, hi);
        uint8_t *rp = dst + row * pk::ROW;
        *reinterpret_cast<uint4 *>(rp + (((2 * ch) ^ (row & 7)) << 4)) = lo;
        *reinterpret_cast<uint4 *>(rp + (((2 * ch + 1) ^ (row & 7)) << 4)) = hi;
    }
}

// The order in which every role meets a pair's work units: tile j's INT4
// k-blocks, with tile j-1's outlier units after the first OUT_DELAY of them
// (by then the epilogue has rescaled tile j-1's accumulator), and the last
// tile's outlier units at the end.  f(j, outlier, k) returns false to stop.
template <class F>
__device__ __forceinline__ void for_each_unit(int ntp, int nkb_i, int nkb_o, F &&f) {
    for (int j = 0; j < ntp; ++j) {
        for (int k = 0; k < nkb_i; ++k) {
            if (j > 0 && k == pk::OUT_DELAY)
                for (int o = 0; o < nkb_o; ++o)
                    if (!f(j - 1, true, o)) return;
            if (!f(j, false, k)) return;
        }
        if (j > 0 && nkb_i <= pk::OUT_DELAY)
            for (int o = 0; o < nkb_o; ++o)
                if (!f(j - 1, true, o)) return;
    }
    if (ntp > 0)
        for (int o = 0; o < nkb_o; ++o)
            if (!f(ntp - 1, true, o)) return;
}

// The MMA issuer's position in the operand ring.
struct Ring {
    int st;       // stage of the next unit
    uint32_t ph;  // its op_full phase parity
    int u;        // units issued (trace only)
};

// One work unit on the pair MMA: wait for its stage, four MMAs (K = 32 bytes
// each) into `acc`, release the stage.  F16: the FP16 outlier kind onto the
// accumulator; else kind::i8, `acc_in` 0 for a tile's first k-block.
template <bool F16, int S_ISSUE>
__device__ __forceinline__ bool issue_unit(Ring &r, uint64_t *op_full, uint64_t *op_empty, uint64_t d0,
                                           uint32_t acc, uint32_t idesc, uint32_t acc_in, const Abort &ab) {
    if (!wait_bar(&op_full[r.st], r.ph, ab)) return false;
    tc_fence_after();
    PTRACE(6, r.u);
    const uint64_t da = d0 + static_cast<uint64_t>((r.st * pk::STAGE) >> 4), db = da + (pk::A_BYTES >> 4);
    if (F16) {
        mma2_f16(acc, da, db, idesc, 1u);
        mma2_f16(acc, da + 2, db + 2, idesc, 1u);
        mma2_f16(acc, da + 4, db + 4, idesc, 1u);
        mma2_f16(acc, da + 6, db + 6, idesc, 1u);
    } else {
        mma2_i8(acc, da, db, idesc, acc_in);
        mma2_i8(acc, da + 2, db + 2, idesc, 1u);
        mma2_i8(acc, da + 4, db + 4, idesc, 1u);
        mma2_i8(acc, da + 6, db + 6, idesc, 1u);
    }
    mma2_commit_both(&op_empty[r.st]);
    PTRACE(9, r.u);
    ++r.u;
    if (++r.st == S_ISSUE) {
        r.st = 0;
        r.ph ^= 1u;
    }
    return true;
}

// X4: the activations are packed INT4 [M, K_i / 2] (quik_gemm), unpacked
// like W; else they are the bytes 16 c [M, K_i] in operand order (written by
// quik_linear's quantiser) and go straight from TMA to the MMA.
// DEBUG: write the integer sums instead of Y (no outliers, no scales).
template <bool X4, bool DEBUG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pk::THREADS, 1)
    w4a4_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tm_w,
                                const __grid_constant__ CUtensorMap tm_x,
                                const __grid_constant__ CUtensorMap tm_wo,
                                const __grid_constant__ CUtensorMap tm_xo,
                                const __grid_constant__ CUtensorMap tm_y, const PParams p) {
    using namespace pk;
    using C = PkCfg<X4>;
    constexpr int S = C::S, SP = C::SP;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t op_full[S], op_empty[S], x_full[S], pk_full[SP], pk_empty[SP];
    __shared__ uint64_t acc_empty[2], rescaled[2], int_done[2], acc_full[2], mma_done, rescaled_last;
    __shared__ uint64_t stall_bar;  // never completed (quik_test_stall)
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;
    __shared__ __align__(16) float sx_s[2][BT];

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int ntp = pair < p.ntiles ? (p.ntiles - pair + npairs - 1) / npairs : 0;
#ifdef QUIK_TRACE
    if (threadIdx.x == 0 && blockIdx.x < 2) {
        g_ptrace[blockIdx.x][8][0] = clock64();
        g_ptrace[blockIdx.x][8][1] = global_timer_ns();
    }
#endif

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&op_full[i], 2 * GW);  // the unit's unpack group in both CTAs (leader only)
            mbar_init(&op_empty[i], 1);
            mbar_init(&x_full[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_empty[b], 2 * NE);  // leader only
            mbar_init(&rescaled[b], 2 * NE);   // leader only
            mbar_init(&int_done[b], 1);
            mbar_init(&acc_full[b], 1);
        }
        mbar_init(&mma_done, 1);
        mbar_init(&rescaled_last, 2 * 16);  // every warp of both CTAs (leader only)
        mbar_init(&stall_bar, 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_pgemm_error);
        fence_barrier_init();
    }
    // this CTA's rows of W and tokens of the B operand for the pair's j-th tile
    auto w_row0 = [&](int j) { return ((pair + j * npairs) / p.n_tt) * 256 + static_cast<int>(rank) * BW; };
    auto t_row0 = [&](int j) { return ((pair + j * npairs) % p.n_tt) * BT + static_cast<int>(rank) * BTH; };
    // The staging producer sets up its own ring and requests the first packed
    // W k-blocks at once: W is not the previous kernel's output, and their
    // latency then overlaps the rest of the set-up (with packed X the units
    // also hold X, which must wait for the grid dependency).
    const int early = X4 ? 0 : min(SP, ntp * p.nkb_i);
    if (warp == W_PPROD && lane == 0) {
        for (int i = 0; i < SP; ++i) {
            mbar_init(&pk_full[i], 1);
            mbar_init(&pk_empty[i], GW);
        }
        fence_barrier_init();
        if (early > 0) tma_prefetch_desc(&tm_w);
        for (int q = 0; q < early; ++q) {
            mbar_arrive_expect_tx(&pk_full[q], C::UNIT);
            tma_load_2d(smem + C::PK_OFF + q * C::UNIT, &tm_w, PKROW * (q % p.nkb_i), w_row0(q / p.nkb_i),
                        &pk_full[q]);
        }
    }
    if (warp == W_MMA) tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers and TMEM allocation visible to both CTAs
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const Abort ab{&abort_s, err0_s};

    // A warp's view of tile j in the epilogue: TMEM lane quadrant warp % 4
    // (the lanes this warp may access), its output channel, scales and bias.
    struct TileLane {
        uint32_t acc;
        int gn, tok0;
        bool n_ok;
        float swn, bn;
        const float *sxr;
    };
    auto tile_lane = [&](int j) {
        TileLane t;
        const int qd = warp & 3;
        t.acc = tmem + (static_cast<uint32_t>(qd * 32) << 16) + 256u * (j & 1);
        t.gn = w_row0(j) + qd * 32 + lane;
        t.n_ok = t.gn < p.N;
        t.tok0 = ((pair + j * npairs) % p.n_tt) * BT;
        t.swn = (!DEBUG && t.n_ok) ? p.sw[t.gn] : 0.0f;
        t.bn = (!DEBUG && t.n_ok && p.bias != nullptr) ? __half2float(__ushort_as_half(p.bias[t.gn])) : 0.0f;
        t.sxr = &sx_s[j & 1][0];
        return t;
    };
    // y = A sx sw + bias in place, 32-column chunks c0, c0 + cstep, ...
    auto rescale_chunks = [&](const TileLane &t, uint32_t acc, int c0, int cstep) {
#pragma unroll 1
        for (int c = c0; c < BT / 32; c += cstep) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(acc + 32 * c, a);
            tmem_ld_wait();
            dequant32(a, t.sxr + 32 * c, t.swn, t.bn);
            tmem_st_32x32b_x32(acc + 32 * c, a);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
    };
    // fp16 Y for chunks c0, c0 + cstep, ... (the integer sums with DEBUG),
    // through the warp's 32 x 32 staging tile and TMA stores when tma_y
    auto final_chunks = [&](int j, const TileLane &t, uint32_t acc, uint16_t *ystage, int c0, int cstep) {
#pragma unroll 1
        for (int c = c0; c < BT / 32; c += cstep) {
            uint32_t a[32];
            tmem_ld_32x32b_x32(acc + 32 * c, a);
            tmem_ld_wait();
            if (!DEBUG && p.nkb_o == 0) dequant32(a, t.sxr + 32 * c, t.swn, t.bn);  // else rescaled already
            const int m0 = t.tok0 + 32 * c;
            if (DEBUG) {
                if (t.n_ok) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (m0 + jj < p.M)
                            p.acc_dbg[static_cast<size_t>(m0 + jj) * p.N + t.gn] = static_cast<int32_t>(a[jj]) >> 8;
                }
                continue;
            }
            if (p.tma_y) {
                // transpose through the staging tile ([token][channel], a warp's
                // stores of one token are 64 contiguous bytes), then one TMA
                // store; the tile's previous store must have read it first
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj)
                    ystage[jj * 32 + lane] = __half_as_ushort(__float2half_rn(__uint_as_float(a[jj])));
                fence_proxy_async_smem();  // generic stores -> visible to the TMA store
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tm_y, ystage, w_row0(j) + 32 * (warp & 3), m0);  // clipped at N and M
                    bulk_commit_group();
                }
            } else {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj)
                    if (t.n_ok && m0 + jj < p.M)
                        p.Y[static_cast<size_t>(m0 + jj) * p.N + t.gn] =
                            __half_as_ushort(__float2half_rn(__uint_as_float(a[jj])));
            }
        }
    };
    // the issuer's state, kept for the last tile's outlier units (issued from
    // the all-warps pass below)
    const uint32_t id_f16 = idesc_f16_f32(2 * BW, BT);
    const uint64_t d0 = sw128_kmajor_desc(smem_base);  // + (byte offset >> 4) per stage and k-step
    Ring ring{0, 0u, 0};
    bool issue_ok = true;
    if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // Straight-line issue code: the tensor core queues about one MMA ahead
        // of its issuer, so every cycle between two MMAs beyond one MMA's
        // execution is lost.  Measured on the pair MMA, a runtime branch
        // choosing the MMA kind around each MMA costs ~190 cycles per k-block
        // and a generic per-unit dispatch ~330; plain loops with one branch per
        // k-block run at 98 % of the MMA rate.  The loops follow the unit order
        // of for_each_unit.
        if (rank == 0 && lane == 0) {
            const uint32_t id_i8 = idesc_s8_s32(2 * BW, BT);
            bool ok = *reinterpret_cast<volatile int *>(&g_pgemm_stall) == 0 || wait_bar(&stall_bar, 0, ab);
            for (int j = 0; j < ntp && ok; ++j) {
                const int b = j & 1;
                const uint32_t acc = tmem + 256u * b;
                if (j >= 2 && !(ok = wait_bar(&acc_empty[b], ((j >> 1) - 1) & 1, ab))) break;
                // INT4 k-blocks 0 .. k1-1, tile j-1's outlier units, the rest
                const int k1 = j > 0 ? min(OUT_DELAY, p.nkb_i) : p.nkb_i;
                for (int k = 0; k < k1 && ok; ++k)
                    ok = issue_unit<false, S>(ring, op_full, op_empty, d0, acc, id_i8, k > 0 ? 1u : 0u, ab);
                if (ok && j > 0 && p.nkb_o > 0) {
                    const int bo = (j - 1) & 1;
                    ok = wait_bar(&rescaled[bo], ((j - 1) >> 1) & 1, ab);
                    for (int o = 0; o < p.nkb_o && ok; ++o)
                        ok = issue_unit<true, S>(ring, op_full, op_empty, d0, tmem + 256u * bo, id_f16, 1u, ab);
                    if (ok) mma2_commit_both(&acc_full[bo]);
                }
                for (int k = k1; k < p.nkb_i && ok; ++k)
                    ok = issue_unit<false, S>(ring, op_full, op_empty, d0, acc, id_i8, 1u, ab);
                if (ok) mma2_commit_both(p.nkb_o > 0 ? &int_done[b] : &acc_full[b]);
            }
            issue_ok = ok;
        }
        __syncwarp();
    } else if (warp == W_XPROD) {
        // ------------------------------------------------------------ operand-stage TMA producer
        if (lane == 0) {
            if (!X4) tma_prefetch_desc(&tm_x);
            if (p.nkb_o > 0) {
                tma_prefetch_desc(&tm_wo);
                tma_prefetch_desc(&tm_xo);
            }
            int u = 0;
            bool dep = false;
            for_each_unit(ntp, p.nkb_i, p.nkb_o, [&](int j, bool outl, int k) -> bool {
                const int st = u % S;
                if (!wait_bar_lazy(&op_empty[st], ((u / S) & 1) ^ 1, ab)) return false;
                uint8_t *a_st = smem + st * STAGE;
                if ((outl || !X4) && !dep) {
                    grid_dependency_wait();  // activations come from the previous kernel
                    dep = true;
                }
                if (outl) {
                    mbar_arrive_expect_tx(&x_full[st], A_BYTES + B_BYTES);
                    tma_load_2d(a_st, &tm_wo, OKB * k, w_row0(j), &x_full[st]);
                    tma_load_2d(a_st + A_BYTES, &tm_xo, OKB * k, t_row0(j), &x_full[st]);
                } else if (!X4) {
                    mbar_arrive_expect_tx(&x_full[st], B_BYTES);
                    tma_load_2d(a_st + A_BYTES, &tm_x, KB * k, t_row0(j), &x_full[st]);
                } else {
                    mbar_arrive(&x_full[st]);  // one phase per unit on every stage
                }
                PTRACE(0, u);
                ++u;
                return true;
            });
            // never leave the CTA with a bulk copy still writing its shared memory:
            // wait for each stage's latest phase (the last of the u units issued
            // on it), whatever completed it; an older phase's parity could alias
            for (int v = u - 1; v >= 0 && v >= u - S; --v) mbar_wait_bounded(&x_full[v % S], (v / S) & 1, kWaitLimitNs);
        }
        __syncwarp();
    } else if (warp == W_PPROD) {
        // ------------------------------------------------------------ packed staging TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            if (X4) tma_prefetch_desc(&tm_x);
            int q = 0;
            bool dep = false;
            for_each_unit(ntp, p.nkb_i, p.nkb_o, [&](int j, bool outl, int k) -> bool {
                if (outl) return true;
                const int ps = q % SP;
                if (q < early) {  // requested before the set-up barrier
                    PTRACE(1, q);
                    ++q;
                    return true;
                }
                if (!wait_bar_lazy(&pk_empty[ps], ((q / SP) & 1) ^ 1, ab)) return false;
                uint8_t *dst = smem + C::PK_OFF + ps * C::UNIT;
                mbar_arrive_expect_tx(&pk_full[ps], C::UNIT);
                tma_load_2d(dst, &tm_w, PKROW * k, w_row0(j), &pk_full[ps]);  // W: not the previous kernel's
                if (X4) {
                    if (!dep) {
                        grid_dependency_wait();
                        dep = true;
                    }
                    tma_load_2d(dst + BW * PKROW, &tm_x, PKROW * k, t_row0(j), &pk_full[ps]);
                }
                PTRACE(1, q);
                ++q;
                return true;
            });
            for (int v = q - 1; v >= 0 && v >= q - SP; --v) mbar_wait_bounded(&pk_full[v % SP], (v / SP) & 1, kWaitLimitNs);
        }
        __syncwarp();
    } else if (is_unpack_warp(warp)) {
        // ------------------------------------------------------------ unpack groups
        const int g = unpack_group(warp);
        const int tb = unpack_lane0(warp) + lane;  // thread in the group: 0 .. GT - 1
        int u = 0, q = 0;
        for_each_unit(ntp, p.nkb_i, p.nkb_o, [&](int j, bool outl, int k) -> bool {
            if (u % NG != g) {  // another group's unit
                ++u;
                if (!outl) ++q;
                return true;
            }
            const int st = u % S;
            if (!warp_wait(&op_empty[st], ((u / S) & 1) ^ 1, ab)) return false;
            if (tb == 0) PTRACE(2, u);
            if (!outl) {
                const int ps = q % SP;
                if (!warp_wait(&pk_full[ps], (q / SP) & 1, ab)) return false;
                if (tb == 0) PTRACE(3, u);
                const uint8_t *src = smem + C::PK_OFF + ps * C::UNIT;
                uint8_t *a_st = smem + st * STAGE;
                unpack_rows(src, a_st, tb);
                if (X4) unpack_rows(src + BW * PKROW, a_st + A_BYTES, tb);
                __syncwarp();
                if (lane == 0) mbar_arrive(&pk_empty[ps]);
                fence_proxy_async_smem();  // generic-proxy stores -> visible to the pair's MMA
                if (tb == 0) PTRACE(4, u);
                ++q;
            }
            if ((outl || !X4) && !warp_wait(&x_full[st], (u / S) & 1, ab)) return false;
            __syncwarp();
            if (tb == 0) PTRACE(5, u);
            if (lane == 0) {
                if (rank == 0)
                    mbar_arrive(&op_full[st]);
                else
                    mbar_arrive_remote(mapa_shared(smem_u32(&op_full[st]), 0));
            }
            if (lane == 0) PTRACE(10 + (warp & 3) - 1, u);
            ++u;
            return true;
        });
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - W_EPI;  // 0 .. 3
        const int et = threadIdx.x - 32 * W_EPI;  // 0 .. 127
        uint16_t *ystage = reinterpret_cast<uint16_t *>(smem + C::EPI_OFF + e * C::EPI_TILE);
        if (!DEBUG) grid_dependency_wait();  // sx comes from the previous kernel
        // After a failed wait a warp skips the work of the remaining tiles but
        // still meets every named barrier, so no other warp is left waiting.
        bool ok = true;
        for (int j = 0; j < ntp; ++j) {
            const int b = j & 1, uj = j >> 1;
            const int tok0 = ((pair + j * npairs) % p.n_tt) * BT;
            if (!DEBUG) {
                for (int c = et; c < BT; c += 32 * NE) {
                    const int m = tok0 + c;
                    sx_s[b][c] = m < p.M ? p.sx[m] : 0.0f;
                }
            }
            if (j == ntp - 1) break;  // the last tile: every warp of the CTA, below
            named_barrier_sync(1, 32 * NE);  // sx_s[b] filled (and tile j-2 done with it)
            if (!ok) continue;
            const TileLane t = tile_lane(j);
            const uint32_t acc = t.acc;
            if (p.nkb_o > 0) {
                if (!(ok = warp_wait_lazy(&int_done[b], uj & 1, ab, lane))) continue;
                tc_fence_after();
                if (et == 0) PTRACE(7, 4 * j);
                // y = A sx sw + bias in place; the outlier MMAs accumulate onto it
                rescale_chunks(t, acc, 0, 1);
                if (et == 0) PTRACE(7, 4 * j + 1);
                if (lane == 0) {
                    if (rank == 0)
                        mbar_arrive(&rescaled[b]);
                    else
                        mbar_arrive_remote(mapa_shared(smem_u32(&rescaled[b]), 0));
                }
            }
            if (!(ok = warp_wait_lazy(&acc_full[b], uj & 1, ab, lane))) continue;
            tc_fence_after();
            if (et == 0) PTRACE(7, 4 * j + 2);
            final_chunks(j, t, acc, ystage, 0, 1);
            tc_fence_before();
            __syncwarp();
            if (et == 0) PTRACE(7, 4 * j + 3);
            if (lane == 0) {
                if (rank == 0)
                    mbar_arrive(&acc_empty[b]);
                else
                    mbar_arrive_remote(mapa_shared(smem_u32(&acc_empty[b]), 0));
            }
        }
        if (lane == 0 && p.tma_y) bulk_wait_group_read0();  // tile ntp-2's stores have read their tiles
    }

    // ------------------------------------------------------------ the last tile, every warp
    // Its two epilogue passes are the exposed tail of the kernel: all 16 warps
    // of each CTA share them (warp w: TMEM lane quadrant w % 4, column chunks
    // w / 4 and w / 4 + 4), and the last tile's outlier units are issued in
    // between.  Each warp stages its 32 x 32 output tiles in the operand
    // ring, which every MMA has finished reading by then.
    named_barrier_sync(2, THREADS);  // every role done with its loop; the last tile's sx_s filled
    if (ntp > 0) {
        const int j = ntp - 1, b = j & 1, uj = j >> 1;
        bool ok = abort_s == 0;
        const TileLane t = tile_lane(j);
        const uint32_t acc = t.acc;
        const int c0 = warp >> 2;
        if (p.nkb_o > 0) {
            if (ok && (ok = warp_wait_lazy(&int_done[b], uj & 1, ab, lane))) {
                tc_fence_after();
                rescale_chunks(t, acc, c0, 4);
            }
            if (lane == 0) {  // also after a failed wait: the issuer's wait below then ends at once
                if (rank == 0)
                    mbar_arrive(&rescaled_last);
                else
                    mbar_arrive_remote(mapa_shared(smem_u32(&rescaled_last), 0));
            }
            if (warp == W_MMA && rank == 0 && lane == 0 && issue_ok) {
                bool iok = wait_bar(&rescaled_last, 0, ab);
                for (int o = 0; o < p.nkb_o && iok; ++o)
                    iok = issue_unit<true, S>(ring, op_full, op_empty, d0, tmem + 256u * b, id_f16, 1u, ab);
                if (iok) mma2_commit_both(&acc_full[b]);
            }
            __syncwarp();
        }
        if (ok && (ok = warp_wait_lazy(&acc_full[b], uj & 1, ab, lane))) {
            tc_fence_after();
            final_chunks(j, t, acc, reinterpret_cast<uint16_t *>(smem + warp * C::EPI_TILE), c0, 4);
            // the stores have read their staging tiles before the CTA leaves (the
            // global writes complete with the grid)
            if (lane == 0 && p.tma_y) bulk_wait_group_read0();
        }
        if (warp == W_MMA && rank == 0 && lane == 0) {
            // TMEM and the stages stay allocated until every issued MMA is done
            mma2_commit_local(&mma_done);
            mbar_wait_bounded(&mma_done, 0, kWaitLimitNs);
        }
        __syncwarp();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs or remote arrivals may touch it
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- two token halves per weight unit
// The same pipeline with tiles of 256 weight rows x 512 tokens: every widened
// weight unit feeds the MMAs of two 256-token halves, each into its own
// 256-column accumulator (all of tensor memory), so the weight unpack and its
// shared-memory traffic are paid once per 512 tokens.  X4: the activations
// come packed through the staging ring with the weights and are widened too
// (half the bytes each SM must pull in by TMA per MMA, whose rate the loads
// otherwise bound); else they come widened straight into the operand stage.  With both accumulators in one tile there is no next tile for the
// epilogue to hide under: after each tile's k-blocks every warp of both CTAs
// takes a share of its passes (rescale, the outlier MMAs, the output), as in
// the last tile of the kernel above.  The operand ring is idle meanwhile and
// holds the output staging tiles.
namespace pk2 {
constexpr int NT = 2;                                  // 256-token halves per tile
constexpr int BT = NT * pk::BT;                        // 512 tokens per tile
constexpr int STAGE = pk::A_BYTES + NT * pk::B_BYTES;  // 48 KB
constexpr int EPI_TILE = 32 * 32 * 2;                  // a warp's 32 x 32 fp16 output tile
constexpr int SP = 3;                                  // packed staging units
static_assert(STAGE % 1024 == 0, "128-byte-swizzled operand tiles");
}  // namespace pk2

template <bool X4>
struct Pk2Cfg {
    static constexpr int S = X4 ? 3 : 4;  // operand stages (48 KB each)
    // packed k-block: W, and with X4 the two token halves
    static constexpr int UNIT = pk::BW * pk::PKROW + (X4 ? pk2::NT * pk::BTH * pk::PKROW : 0);
    static constexpr int PK_OFF = S * pk2::STAGE;
    static constexpr int SMEM = PK_OFF + pk2::SP * UNIT + 1024;  // + alignment slack
    static_assert(SMEM + 4096 <= 232448, "shared memory budget (dynamic + static)");
    static_assert(16 * pk2::EPI_TILE <= S * pk2::STAGE, "the output staging tiles fit in the operand ring");
};

// One work unit on the pair MMA for both token halves: wait for its stage,
// four MMAs per half (K = 32 bytes each) into that half's accumulator,
// release the stage.
template <bool F16, int S_ISSUE>
__device__ __forceinline__ bool issue_unit2(Ring &r, uint64_t *op_full, uint64_t *op_empty, uint64_t d0,
                                            uint32_t tmem, uint32_t idesc, uint32_t acc_in, const Abort &ab) {
    if (!wait_bar(&op_full[r.st], r.ph, ab)) return false;
    tc_fence_after();
    const uint64_t da = d0 + static_cast<uint64_t>((r.st * pk2::STAGE) >> 4);
    const uint64_t db0 = da + (pk::A_BYTES >> 4), db1 = db0 + (pk::B_BYTES >> 4);
    if (F16) {
        mma2_f16(tmem, da, db0, idesc, 1u);
        mma2_f16(tmem, da + 2, db0 + 2, idesc, 1u);
        mma2_f16(tmem, da + 4, db0 + 4, idesc, 1u);
        mma2_f16(tmem, da + 6, db0 + 6, idesc, 1u);
        mma2_f16(tmem + 256u, da, db1, idesc, 1u);
        mma2_f16(tmem + 256u, da + 2, db1 + 2, idesc, 1u);
        mma2_f16(tmem + 256u, da + 4, db1 + 4, idesc, 1u);
        mma2_f16(tmem + 256u, da + 6, db1 + 6, idesc, 1u);
    } else {
        mma2_i8(tmem, da, db0, idesc, acc_in);
        mma2_i8(tmem, da + 2, db0 + 2, idesc, 1u);
        mma2_i8(tmem, da + 4, db0 + 4, idesc, 1u);
        mma2_i8(tmem, da + 6, db0 + 6, idesc, 1u);
        mma2_i8(tmem + 256u, da, db1, idesc, acc_in);
        mma2_i8(tmem + 256u, da + 2, db1 + 2, idesc, 1u);
        mma2_i8(tmem + 256u, da + 4, db1 + 4, idesc, 1u);
        mma2_i8(tmem + 256u, da + 6, db1 + 6, idesc, 1u);
    }
    mma2_commit_both(&op_empty[r.st]);
    ++r.u;
    if (++r.st == S_ISSUE) {
        r.st = 0;
        r.ph ^= 1u;
    }
    return true;
}

// DEBUG: write the integer sums instead of Y (no outliers, no scales).
template <bool X4, bool DEBUG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pk::THREADS, 1)
    w4a4_gemm_persistent2_kernel(const __grid_constant__ CUtensorMap tm_w,
                                 const __grid_constant__ CUtensorMap tm_x,
                                 const __grid_constant__ CUtensorMap tm_wo,
                                 const __grid_constant__ CUtensorMap tm_xo,
                                 const __grid_constant__ CUtensorMap tm_y, const PParams p) {
    using namespace pk;
    using C2 = Pk2Cfg<X4>;
    constexpr int S = C2::S, SP = pk2::SP;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t op_full[S], op_empty[S], x_full[S], pk_full[SP], pk_empty[SP];
    __shared__ uint64_t int_done, acc_full, rescaled, epi_done, mma_done;
    __shared__ uint64_t stall_bar;  // never completed (quik_test_stall)
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ unsigned err0_s;
    __shared__ __align__(16) float sx_s[pk2::BT];

    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    const uint32_t smem_base = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int ntp = pair < p.ntiles ? (p.ntiles - pair + npairs - 1) / npairs : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&op_full[i], 2 * GW);  // the unit's unpack group in both CTAs (leader only)
            mbar_init(&op_empty[i], 1);
            mbar_init(&x_full[i], 1);
        }
        mbar_init(&int_done, 1);
        mbar_init(&acc_full, 1);
        mbar_init(&rescaled, 2 * 16);  // every warp of both CTAs (leader only)
        mbar_init(&epi_done, 2 * 16);  // every warp of both CTAs (leader only)
        mbar_init(&mma_done, 1);
        mbar_init(&stall_bar, 1);
        abort_s = 0;
        err0_s = *reinterpret_cast<volatile unsigned *>(&g_pgemm_error);
        fence_barrier_init();
    }
    // this CTA's rows of W and tokens of token half h for the pair's j-th tile
    auto w_row0 = [&](int j) { return ((pair + j * npairs) / p.n_tt) * 256 + static_cast<int>(rank) * BW; };
    auto tok0 = [&](int j) { return ((pair + j * npairs) % p.n_tt) * pk2::BT; };
    auto t_row0 = [&](int j, int h) { return tok0(j) + h * pk::BT + static_cast<int>(rank) * BTH; };
    // W units requested before the set-up barrier (W is not the previous
    // kernel's output; with X4 the units also hold X, which must wait)
    const int early = X4 ? 0 : min(SP, ntp * p.nkb_i);
    if (warp == W_PPROD && lane == 0) {
        for (int i = 0; i < SP; ++i) {
            mbar_init(&pk_full[i], 1);
            mbar_init(&pk_empty[i], GW);
        }
        fence_barrier_init();
        if (early > 0) tma_prefetch_desc(&tm_w);
        for (int q = 0; q < early; ++q) {
            mbar_arrive_expect_tx(&pk_full[q], C2::UNIT);
            tma_load_2d(smem + C2::PK_OFF + q * C2::UNIT, &tm_w, PKROW * (q % p.nkb_i), w_row0(q / p.nkb_i),
                        &pk_full[q]);
        }
    }
    if (warp == W_MMA) tmem_alloc_pair(&tmem_base_s, TMEM_COLS);
    tc_fence_before();
    cluster_sync();  // barriers and TMEM allocation visible to both CTAs
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const Abort ab{&abort_s, err0_s};
    const uint32_t id_i8 = idesc_s8_s32(2 * BW, pk::BT);
    const uint32_t id_f16 = idesc_f16_f32(2 * BW, pk::BT);
    const uint64_t d0 = sw128_kmajor_desc(smem_base);
    Ring ring{0, 0u, 0};
    bool issue_ok = rank != 0 || warp != W_MMA || lane != 0 ||
                    *reinterpret_cast<volatile int *>(&g_pgemm_stall) == 0 || wait_bar(&stall_bar, 0, ab);
    int u_x = 0, q_p = 0;     // the producers' unit counters (all tiles)
    int u_g = 0, q_g = 0;     // the unpack warps' unit and staging counters (all tiles)
    bool ok = true;           // this warp's waits have all succeeded
    const int qd = warp & 3;  // TMEM lane quadrant this warp may access
    if (warp == W_XPROD && lane == 0) {
        tma_prefetch_desc(&tm_x);
        if (p.nkb_o > 0) {
            tma_prefetch_desc(&tm_wo);
            tma_prefetch_desc(&tm_xo);
        }
    }
    if (warp == W_PPROD && lane == 0) tma_prefetch_desc(&tm_w);

    for (int j = 0; j < ntp; ++j) {
        // ------------------------------------------------------------ tile j's k-blocks
        if (warp == W_MMA) {
            if (rank == 0 && lane == 0 && issue_ok) {
                // both CTAs have read tile j-1's accumulators
                if (j > 0) issue_ok = wait_bar(&epi_done, (j - 1) & 1, ab);
                for (int k = 0; k < p.nkb_i && issue_ok; ++k)
                    issue_ok = issue_unit2<false, S>(ring, op_full, op_empty, d0, tmem, id_i8, k > 0 ? 1u : 0u, ab);
                if (issue_ok) mma2_commit_both(p.nkb_o > 0 ? &int_done : &acc_full);
            }
            __syncwarp();
        } else if (warp == W_XPROD) {
            if (lane == 0) {
                if (j == 0) grid_dependency_wait();  // the activations come from the previous kernel
                for (int v = 0; v < p.nkb_i + p.nkb_o && ok; ++v, ++u_x) {
                    const int st = u_x % S;
                    if (!(ok = wait_bar_lazy(&op_empty[st], ((u_x / S) & 1) ^ 1, ab))) break;
                    uint8_t *a_st = smem + st * pk2::STAGE;
                    if (v < p.nkb_i && X4) {
                        mbar_arrive(&x_full[st]);  // one phase per unit on every stage
                    } else if (v < p.nkb_i) {
                        mbar_arrive_expect_tx(&x_full[st], pk2::NT * B_BYTES);
                        for (int h = 0; h < pk2::NT; ++h)
                            tma_load_2d(a_st + A_BYTES + h * B_BYTES, &tm_x, KB * v, t_row0(j, h), &x_full[st]);
                    } else {
                        const int o = v - p.nkb_i;
                        mbar_arrive_expect_tx(&x_full[st], A_BYTES + pk2::NT * B_BYTES);
                        tma_load_2d(a_st, &tm_wo, OKB * o, w_row0(j), &x_full[st]);
                        for (int h = 0; h < pk2::NT; ++h)
                            tma_load_2d(a_st + A_BYTES + h * B_BYTES, &tm_xo, OKB * o, t_row0(j, h), &x_full[st]);
                    }
                }
            }
            __syncwarp();
        } else if (warp == W_PPROD) {
            if (lane == 0) {
                if (X4 && j == 0) grid_dependency_wait();  // packed X comes from the previous kernel
                for (int k = 0; k < p.nkb_i && ok; ++k, ++q_p) {
                    if (q_p < early) continue;  // requested before the set-up barrier
                    const int ps = q_p % SP;
                    if (!(ok = wait_bar_lazy(&pk_empty[ps], ((q_p / SP) & 1) ^ 1, ab))) break;
                    uint8_t *dst = smem + C2::PK_OFF + ps * C2::UNIT;
                    mbar_arrive_expect_tx(&pk_full[ps], C2::UNIT);
                    tma_load_2d(dst, &tm_w, PKROW * k, w_row0(j), &pk_full[ps]);
                    if (X4)
                        for (int h = 0; h < pk2::NT; ++h)
                            tma_load_2d(dst + BW * PKROW + h * BTH * PKROW, &tm_x, PKROW * k, t_row0(j, h), &pk_full[ps]);
                }
            }
            __syncwarp();
        } else if (is_unpack_warp(warp)) {
            const int g = unpack_group(warp);
            const int tb = unpack_lane0(warp) + lane;  // thread in the group: 0 .. GT - 1
            for (int v = 0; v < p.nkb_i + p.nkb_o && ok; ++v, ++u_g) {
                const bool outl = v >= p.nkb_i;
                if (u_g % NG != g) {  // another group's unit
                    if (!outl) ++q_g;
                    continue;
                }
                const int st = u_g % S;
                if (!(ok = warp_wait(&op_empty[st], ((u_g / S) & 1) ^ 1, ab))) break;
                if (!outl) {
                    const int ps = q_g % SP;
                    if (!(ok = warp_wait(&pk_full[ps], (q_g / SP) & 1, ab))) break;
                    const uint8_t *src = smem + C2::PK_OFF + ps * C2::UNIT;
                    uint8_t *a_st = smem + st * pk2::STAGE;
                    unpack_rows(src, a_st, tb);
                    if (X4)
                        for (int h = 0; h < pk2::NT; ++h)
                            unpack_rows(src + BW * PKROW + h * BTH * PKROW, a_st + A_BYTES + h * B_BYTES, tb);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pk_empty[ps]);
                    fence_proxy_async_smem();  // generic-proxy stores -> visible to the pair's MMA
                    ++q_g;
                }
                if (!(ok = warp_wait(&x_full[st], (u_g / S) & 1, ab))) break;
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0)
                        mbar_arrive(&op_full[st]);
                    else
                        mbar_arrive_remote(mapa_shared(smem_u32(&op_full[st]), 0));
                }
            }
            // keep the counters in step after an early stop (the remaining
            // tiles' work is skipped, but the loops' counts stay consistent)
        }

        // ------------------------------------------------------------ tile j's epilogue, every warp
        named_barrier_sync(2, THREADS);  // tile j-1's passes and every role's part of tile j are done
        if (!DEBUG) {
            grid_dependency_wait();  // sx comes from the previous kernel
            const int m = tok0(j) + threadIdx.x;
            sx_s[threadIdx.x] = m < p.M ? p.sx[m] : 0.0f;
        }
        named_barrier_sync(2, THREADS);  // sx_s filled
        bool eok = abort_s == 0;
        const int gn = w_row0(j) + qd * 32 + lane;  // this lane's output channel (TMEM lane)
        const bool n_ok = gn < p.N;
        const float swn = (!DEBUG && n_ok) ? p.sw[gn] : 0.0f;
        const float bn = (!DEBUG && n_ok && p.bias != nullptr) ? __half2float(__ushort_as_half(p.bias[gn])) : 0.0f;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const int c0 = warp >> 2;  // chunks c0, c0 + 4, c0 + 8, c0 + 12 of the 16 (two halves x 8)
        if (p.nkb_o > 0) {
            if (eok && (eok = warp_wait_lazy(&int_done, j & 1, ab, lane))) {
                tc_fence_after();
#pragma unroll 1
                for (int c = c0; c < 16; c += 4) {
                    const int col = 256 * (c >> 3) + 32 * (c & 7);
                    uint32_t a[32];
                    tmem_ld_32x32b_x32(t_lane + col, a);
                    tmem_ld_wait();
                    dequant32(a, sx_s + col, swn, bn);
                    tmem_st_32x32b_x32(t_lane + col, a);
                }
                tmem_st_wait();
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) {  // also after a failed wait: the issuer's wait below then ends at once
                if (rank == 0)
                    mbar_arrive(&rescaled);
                else
                    mbar_arrive_remote(mapa_shared(smem_u32(&rescaled), 0));
            }
            if (warp == W_MMA && rank == 0 && lane == 0 && issue_ok) {
                issue_ok = wait_bar(&rescaled, j & 1, ab);
                for (int o = 0; o < p.nkb_o && issue_ok; ++o)
                    issue_ok = issue_unit2<true, S>(ring, op_full, op_empty, d0, tmem, id_f16, 1u, ab);
                if (issue_ok) mma2_commit_both(&acc_full);
            }
            __syncwarp();
        }
        if (eok && (eok = warp_wait_lazy(&acc_full, j & 1, ab, lane))) {
            tc_fence_after();
            uint16_t *ystage = reinterpret_cast<uint16_t *>(smem + warp * pk2::EPI_TILE);
#pragma unroll 1
            for (int c = c0; c < 16; c += 4) {
                const int col = 256 * (c >> 3) + 32 * (c & 7);
                uint32_t a[32];
                tmem_ld_32x32b_x32(t_lane + col, a);
                tmem_ld_wait();
                if (!DEBUG && p.nkb_o == 0) dequant32(a, sx_s + col, swn, bn);  // else rescaled already
                const int m0 = tok0(j) + col;
                if (DEBUG) {
                    if (n_ok) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (m0 + jj < p.M)
                                p.acc_dbg[static_cast<size_t>(m0 + jj) * p.N + gn] = static_cast<int32_t>(a[jj]) >> 8;
                    }
                    continue;
                }
                if (p.tma_y) {
                    // transpose through the warp's staging tile, then one TMA store
                    if (lane == 0) bulk_wait_group_read0();
                    __syncwarp();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        ystage[jj * 32 + lane] = __half_as_ushort(__float2half_rn(__uint_as_float(a[jj])));
                    fence_proxy_async_smem();  // generic stores -> visible to the TMA store
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_y, ystage, w_row0(j) + 32 * qd, m0);  // clipped at N and M
                        bulk_commit_group();
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (n_ok && m0 + jj < p.M)
                            p.Y[static_cast<size_t>(m0 + jj) * p.N + gn] =
                                __half_as_ushort(__float2half_rn(__uint_as_float(a[jj])));
                }
            }
            // the staging tiles are read before the ring takes the next tile's operands
            if (lane == 0 && p.tma_y) bulk_wait_group_read0();
            tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) {  // this warp is done with the accumulators
            if (rank == 0)
                mbar_arrive(&epi_done);
            else
                mbar_arrive_remote(mapa_shared(smem_u32(&epi_done), 0));
        }
        named_barrier_sync(2, THREADS);  // the ring may take tile j+1's operands
    }

    // ---------------------------------------------------------------- teardown
    if (warp == W_XPROD && lane == 0)  // no bulk copy may still write the ring
        for (int v = u_x - 1; v >= 0 && v >= u_x - S; --v) mbar_wait_bounded(&x_full[v % S], (v / S) & 1, kWaitLimitNs);
    if (warp == W_PPROD && lane == 0) {
        const int issued = max(q_p, early);
        for (int v = issued - 1; v >= 0 && v >= issued - SP; --v)
            mbar_wait_bounded(&pk_full[v % SP], (v / SP) & 1, kWaitLimitNs);
    }
    if (warp == W_MMA && rank == 0 && lane == 0) {
        // TMEM and the stages stay allocated until every issued MMA is done
        mma2_commit_local(&mma_done);
        mbar_wait_bounded(&mma_done, 0, kWaitLimitNs);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs or remote arrivals may touch it
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

template <bool X4, bool DEBUG>
quik_status run_persistent(const GemmArgs &a, cudaStream_t stream) {
    using C = PkCfg<X4>;
    const int Ki = a.K - a.k_o;
    const bool outliers = !DEBUG && a.k_o > 0 && a.Xo != nullptr;
    CUtensorMap mw, mx, mwo, mxo;
    std::memset(&mw, 0, sizeof(mw));
    std::memset(&mx, 0, sizeof(mx));
    std::memset(&mwo, 0, sizeof(mwo));
    std::memset(&mxo, 0, sizeof(mxo));
    // packed W: 64 bytes x 128 rows per k-block
    if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, Ki / 2, a.N, Ki / 2, pk::PKROW, pk::BW,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return QUIK_ERR_CUDA;
    if (X4) {  // packed X, unpacked like W
        if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, Ki / 2, a.M, Ki / 2, pk::PKROW, pk::BTH,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
            return QUIK_ERR_CUDA;
    } else {  // the bytes 16 c: 128 bytes x 128 rows, straight into the swizzled operand layout
        if (!make_map(&mx, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq, Ki, a.M, Ki, pk::ROW, pk::BTH,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    if (outliers) {
        const uint64_t pitch = static_cast<uint64_t>(a.k_o) * 2;
        if (!make_map(&mwo, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.Wo, a.k_o, a.N, pitch, pk::OKB, pk::BW,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&mxo, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.Xo, a.k_o, a.M, pitch, pk::OKB, pk::BTH,
                      CU_TENSOR_MAP_SWIZZLE_128B))
            return QUIK_ERR_CUDA;
    }
    // Y: 32 x 32 fp16 boxes when its rows are 16-byte multiples
    CUtensorMap my;
    std::memset(&my, 0, sizeof(my));
    const bool tma_y = !DEBUG && a.N % 8 == 0 &&
                       make_map(&my, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.Y, a.N, a.M,
                                static_cast<uint64_t>(a.N) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
    PParams p{};
    p.M = a.M;
    p.N = a.N;
    p.Ki = Ki;
    p.tma_y = tma_y ? 1 : 0;
    p.nkb_i = (Ki + pk::KB - 1) / pk::KB;
    p.nkb_o = outliers ? (a.k_o + pk::OKB - 1) / pk::OKB : 0;
    const int n_wt = (a.N + 2 * pk::BW - 1) / (2 * pk::BW);
    p.sx = a.sx;
    p.sw = a.sw;
    p.bias = a.bias;
    p.Y = a.Y;
    p.acc_dbg = a.acc_dbg;
    const int np_max = std::max(1, sm_count() / 2);
    // 512-token tiles (widened activations, at most S outlier units) when
    // they fit in one wave where 256-token tiles need two or more: measured,
    // the main loop runs at the same rate per k-block and token either way,
    // but a 512-token tile's epilogue does not overlap a next tile, so the
    // larger tiles pay only where they remove a wave (the attention
    // projection at 2048 tokens: GEMM 42.8 -> 37.9 us; at 2048 x 11008, three
    // waves against five, they were slower: 92.1 against 83.2 us)
    const int tiles1 = ((a.M + pk::BT - 1) / pk::BT) * n_wt, tiles2 = ((a.M + pk2::BT - 1) / pk2::BT) * n_wt;
    const bool two = !DEBUG && p.nkb_o <= Pk2Cfg<X4>::S && tiles2 <= np_max && tiles1 > np_max;
    p.n_tt = two ? (a.M + pk2::BT - 1) / pk2::BT : (a.M + pk::BT - 1) / pk::BT;
    p.ntiles = p.n_tt * n_wt;
    auto kern = two ? w4a4_gemm_persistent2_kernel<X4, false> : w4a4_gemm_persistent_kernel<X4, DEBUG>;
    const int smem_bytes = two ? Pk2Cfg<X4>::SMEM : C::SMEM;
    if (!attribute_set_once(reinterpret_cast<const void *>(kern), smem_bytes)) return QUIK_ERR_CUDA;
    const int npairs = std::max(1, std::min(p.ntiles, np_max));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * npairs);
    cfg.blockDim = dim3(pk::THREADS);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    // programmatic dependent launch after this library's quantiser: the CTAs
    // start while it finishes; every read of its outputs waits first
    cfg.numAttrs = a.after_quantize ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mw, mx, mwo, mxo, my, p) == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

}  // namespace

bool persistent_gemm_takes(const GemmArgs &a) {
    return a.group == 0 && !a.a8 && !a.w8 && !a.sparse24 && a.K - a.k_o > 0 &&
           (a.k_o == 0 || !a.out_int8) && a.M > kDecodeTokens;
}

quik_status launch_gemm_persistent(const GemmArgs &a, cudaStream_t stream) {
    if (a.x_wide) return a.debug ? run_persistent<false, true>(a, stream) : run_persistent<false, false>(a, stream);
    return a.debug ? run_persistent<true, true>(a, stream) : run_persistent<true, false>(a, stream);
}

#ifdef QUIK_TRACE
extern "C" __attribute__((visibility("default"))) int ptrace_read(unsigned long long *dst) {
    return cudaMemcpyFromSymbol(dst, g_ptrace, sizeof(g_ptrace)) == cudaSuccess ? 0 : -1;
}
#endif

cudaError_t set_persistent_gemm_stall(int on) {
    return cudaMemcpyToSymbol(g_pgemm_stall, &on, sizeof(on));
}

unsigned int persistent_gemm_errors() {
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_pgemm_error, sizeof(word)) != cudaSuccess) return 0;
    return counter_increase(kCounterPGemmWaits, word);
}

}  // namespace quik
