/*
 * quik.h -- C ABI of the B200 (sm_100a) hybrid W4A4 + outlier linear layer.
 *
 * The layer (QUIK abstract; Atom summary, key points and ideas I1-I3):
 *   X  fp16 [M, K] activations, W fp16 [N, K] weights, perm int32 [K].
 *   Reordered channel j is source channel perm[j]; the last k_o reordered
 *   channels are the outliers, kept in FP16 (QUIK) or INT8 (Atom, idea I3),
 *   the other K_i = K - k_o are quantised to symmetric INT4 (Atom key point
 *   "symmetric quantization") with a dynamic scale per token (activations)
 *   or per output channel (weights), or per group of 128 reordered channels
 *   (Atom summary, "fine-grained group quantization").
 *   Y fp16 [M, N] = sum_g A_g * sx[m,g] * sw[n,g] + O[m,n] + bias[n],
 *   A_g = exact integer sum of INT4 code products over group g,
 *   O = outlier-block product (FP16 inputs, fp32 sum; or INT8 -> INT32 times
 *   the two INT8 scales).
 *
 * Quantiser (readings where the pages are silent):
 *   s = max|v| / 7 in fp32 over the INT4 positions of the row (or group);
 *   q = clamp(rint(v / s), -7, 7), IEEE fp32 division, round half to even;
 *   a zero row/group has s = 0 and codes 0.  INT8 outliers use 127.
 *
 * Byte layout of packed INT4 (Xq, Wq): row-major [rows, K_i / 2]; byte i of a
 * row holds code 2i in bits 0-3 and code 2i+1 in bits 4-7, two's complement.
 * Scales: fp32, [rows] or [rows, G] (G = K_i / 128) row-major.
 *
 * 8-bit activations (W4A8; QQQ abstract: 4-bit weights with 8-bit
 * activations, per-channel GEMM), selected by quik_shape.act_bits == 8: the
 * activations' non-outlier positions use the INT8 rule of the outlier block,
 * s = max|v| / 127 per token and q = clamp(rint(v / s), -127, 127); Xq is then
 * int8 [M, K_i] row-major, one byte per code in reordered order.  Weights stay
 * packed INT4.  Per-token scales only (group_size 0).
 *
 * 8-bit weights (W8A8, the INT8 baseline the same pages compare with),
 * selected by quik_shape.weight_bits == 8 together with act_bits == 8: the
 * weights take the same INT8 rule per output channel and Wq is int8 [N, K_i].

 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE memory owned by the caller; no call
 *     allocates device memory and none keeps a pointer after returning.  The
 *     one device buffer the library owns is quik_linear_noalloc's static
 *     workspace (below), part of the library's device module.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream) and is asynchronous: nothing synchronises.
 *   - Every function returns a quik_status; nothing throws across the ABI.
 *   - Arguments are validated before any launch: non-NULL pointers that are
 *     16-byte aligned, M, N >= 1, 0 <= k_o <= K, K_i % 32 == 0, k_o % 16 == 0,
 *     K <= 32768, group_size 0 or 128 (then K_i % 128 == 0), act_bits and
 *     weight_bits 0, 4 or 8.  Any violation returns QUIK_ERR_INVALID_ARG with
 *     nothing enqueued; act_bits 8 with group_size 128, and weight_bits 8
 *     without act_bits 8, return QUIK_ERR_UNSUPPORTED.  Pointers that are
 *     unused for the shape (outlier buffers when k_o == 0, INT8 scales in FP16
 *     mode, bias) may be NULL.
 *   - perm must be a permutation of 0..K-1.  Entries outside [0, K) are
 *     never used as addresses: they read channel 0, are counted, and
 *     quik_sync_check reports QUIK_ERR_INVALID_ARG.  Repeated entries are not
 *     detected.
 *   - A launch failure returns QUIK_ERR_CUDA.  Every wait inside the GEMM
 *     kernel is bounded; if one runs out the kernel records it in a device
 *     error word and exits cleanly, and quik_sync_check reports
 *     QUIK_ERR_TIMEOUT.
 *   - Thread safety: entry points may be called concurrently from several
 *     host threads (no mutable host state besides one-time initialisation).
 */
#ifndef QUIK_H_
#define QUIK_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QUIK_API __attribute__((visibility("default")))
#else
#define QUIK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QUIK_OK = 0,
    QUIK_ERR_INVALID_ARG = 1,
    QUIK_ERR_UNSUPPORTED = 2,
    QUIK_ERR_CUDA = 3,
    QUIK_ERR_TIMEOUT = 4
} quik_status;

typedef enum {
    QUIK_OUTLIER_FP16 = 0, /* QUIK: outlier block stays FP16 */
    QUIK_OUTLIER_INT8 = 1  /* Atom idea I3: outlier block in INT8, fp32 scale per row */
} quik_outlier_t;

typedef struct {
    int32_t M;          /* tokens (rows of X and Y) */
    int32_t N;          /* output channels (rows of W, columns of Y) */
    int32_t K;          /* input channels */
    int32_t k_o;        /* outlier channels (last k_o of the reordering) */
    int32_t group_size; /* 0: per-token / per-channel scales; 128: per group */
    int32_t outlier;    /* a quik_outlier_t */
    int32_t act_bits;   /* activation codes: 0 or 4 -> INT4 (W4A4); 8 -> INT8 (W4A8) */
    int32_t weight_bits; /* weight codes: 0 or 4 -> INT4; 8 -> INT8 (W8A8, needs act_bits 8) */
} quik_shape;

/* Opaque cudaStream_t. */
typedef void *quik_stream_t;

/*
 * quik_workspace_size -- bytes of device workspace quik_linear needs for the
 * quantised activations (packed codes, scales, outlier block), each part
 * 256-byte aligned.  Returns 0 for an invalid shape.
 */
QUIK_API size_t quik_workspace_size(const quik_shape *shape);

/*
 * quik_quantize_reorder -- step "dynamic quantisation + reordering" of the
 * activations (Atom summary and idea I2; QUIK abstract).  One kernel reads X
 * once, gathers the columns through perm, computes the per-token (or
 * per-group) INT4 scales, packs the codes and copies (FP16) or quantises
 * (INT8) the outlier block.
 *   X_f16    [M, K] fp16, row-major
 *   perm     [K] int32
 *   Xq       out [M, K_i/2] packed INT4 (act_bits 8: int8 [M, K_i])
 *   x_scale  out fp32 [M] or [M, G]
 *   Xo       out [M, k_o] fp16 or int8 (may be NULL when k_o == 0)
 *   xo_scale out fp32 [M], INT8 outliers only (NULL otherwise)
 */
QUIK_API quik_status quik_quantize_reorder(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                                  void *Xq, float *x_scale, void *Xo, float *xo_scale,
                                  quik_stream_t stream);

/*
 * quik_pack_weights -- offline weight preparation (QUIK sample names
 * pack_to_i4 / two_compl; Atom idea I1): the same reorder + symmetric
 * quantiser applied to the rows of W (one scale per output channel, or per
 * channel and group), round-to-nearest codes.  INT4 (Wq [N, K_i/2]), or INT8
 * (Wq int8 [N, K_i]) when weight_bits == 8.
 *   W_f16 [N, K] fp16; Wq out [N, K_i/2]; w_scale out [N] or [N, G];
 *   Wo out [N, k_o] fp16 or int8; wo_scale out [N] (INT8 outliers only).
 */
QUIK_API quik_status quik_pack_weights(const quik_shape *shape, const void *W_f16, const int32_t *perm,
                              void *Wq, float *w_scale, void *Wo, float *wo_scale,
                              quik_stream_t stream);

/*
 * quik_gemm -- INT4 x INT4 product with exact INT32 accumulation (tensor
 * cores, Atom key points), the outlier sub-product, and the dequantising
 * epilogue Y = A*sx*sw (+ per group) + O + bias, rounded to fp16.
 *   Xq [M, K_i/2] (act_bits 8: int8 [M, K_i]), x_scale, Xo [M, k_o], xo_scale :
 *                                                   quantised activations
 *   Wq [N, K_i/2], w_scale, Wo [N, k_o], wo_scale : packed weights
 *   bias_f16 [N] or NULL;  Y_f16 out [M, N] fp16 row-major
 */
QUIK_API quik_status quik_gemm(const quik_shape *shape,
                      const void *Xq, const float *x_scale, const void *Xo, const float *xo_scale,
                      const void *Wq, const float *w_scale, const void *Wo, const float *wo_scale,
                      const void *bias_f16, void *Y_f16, quik_stream_t stream);

/*
 * quik_linear -- the whole layer on fp16 activations: quik_quantize_reorder
 * into `workspace` followed by quik_gemm, both on `stream`.
 *   workspace : device buffer of at least quik_workspace_size(shape) bytes
 *               (caller-owned; reused freely between calls on one stream).
 */
QUIK_API quik_status quik_linear(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                        const void *Wq, const float *w_scale, const void *Wo,
                        const float *wo_scale, const void *bias_f16, void *Y_f16,
                        void *workspace, size_t workspace_bytes, quik_stream_t stream);

/*
 * quik_linear_timed -- quik_linear with the CUDA event `between` (a
 * cudaEvent_t passed as void *, created by the caller) recorded on `stream`
 * after the quantiser's launch and before the GEMM's.  A measurement aid of
 * this library (no counterpart in the papers): with the event between them
 * the GEMM waits for the quantiser to finish instead of starting during its
 * tail, so events recorded before the call, `between`, and after the call
 * time the layer's two kernels one by one.  Y is bit-identical to
 * quik_linear's.  `between` NULL: QUIK_ERR_INVALID_ARG; a failed record:
 * QUIK_ERR_CUDA; otherwise as quik_linear.
 */
QUIK_API quik_status quik_linear_timed(const quik_shape *shape, const void *X_f16,
                                       const int32_t *perm, const void *Wq, const float *w_scale,
                                       const void *Wo, const float *wo_scale, const void *bias_f16,
                                       void *Y_f16, void *workspace, size_t workspace_bytes,
                                       void *between, quik_stream_t stream);

/*
 * quik_rmsnorm_quantize_reorder -- the RMS norm that precedes a projection,
 * with the projection's dynamic quantisation and reordering folded into it
 * (Atom summary and idea I2: quantisation and reordering are fused into
 * operators that already run).  For each row h of X:
 *     r = 1 / sqrt(mean_k(h[k]^2) + eps)         (all K channels)
 *     y[k] = h[k] * r * gamma[k]
 * and y is quantised as by quik_quantize_reorder, with one reading: r > 0 is
 * common to the whole row and changes no code, so the codes and the fp32
 * base scales are those of z = h * gamma (exact in fp32), and r multiplies
 * what is stored:
 *     x_scale  = fl32(fl32(max|z| / 7) * r)      (per token, or per group)
 *     xo_scale = fl32(fl32(max|z_o| / 127) * r)  (INT8 outliers)
 *     Xo       = fl16(fl32(z * r))               (FP16 outliers)
 * The normalised fp16 row is never written.  The sum of squares is taken in
 * fp32 and r with IEEE-rounded steps, so scales and FP16 outliers carry the
 * rounding of that sum; codes do not depend on it.
 *   X_f16     [M, K] fp16 (the hidden state before the norm), row-major
 *   gamma_f16 [K] fp16, the norm's weight in SOURCE channel order
 *   eps       finite and > 0 (else QUIK_ERR_INVALID_ARG)
 *   perm, Xq, x_scale, Xo, xo_scale : as quik_quantize_reorder
 * K up to 24576 (the kernel stages perm and the reordered gamma side by side
 * in shared memory); a larger K returns QUIK_ERR_UNSUPPORTED.  Other errors,
 * validation and stream semantics as quik_quantize_reorder.
 */
QUIK_API quik_status quik_rmsnorm_quantize_reorder(const quik_shape *shape, const void *X_f16,
                                                   const void *gamma_f16, float eps,
                                                   const int32_t *perm, void *Xq, float *x_scale,
                                                   void *Xo, float *xo_scale, quik_stream_t stream);

/*
 * quik_rmsnorm_linear -- quik_linear behind an RMS norm:
 * quik_rmsnorm_quantize_reorder into `workspace` (quik_workspace_size(shape)
 * bytes, caller-owned) followed by quik_gemm, on `stream`.  Arguments as
 * quik_linear plus gamma_f16 [K] and eps of quik_rmsnorm_quantize_reorder.
 */
QUIK_API quik_status quik_rmsnorm_linear(const quik_shape *shape, const void *X_f16,
                                         const void *gamma_f16, float eps, const int32_t *perm,
                                         const void *Wq, const float *w_scale, const void *Wo,
                                         const float *wo_scale, const void *bias_f16, void *Y_f16,
                                         void *workspace, size_t workspace_bytes,
                                         quik_stream_t stream);

/*
 * 2:4-sparse INT4 weights (QUIK abstract: quantisation combined with 2:4
 * sparsity).  Within the INT4 part of each reordered weight row, every
 * aligned group of four positions 4t .. 4t+3 keeps its two values of largest
 * magnitude (on equal magnitudes, the lower position) and the other two are
 * zero; the row's scale and the kept values' codes follow the dense rule
 * (s = max|w| / 7 per output channel); the outlier block stays dense.  The
 * product runs on the sparse tensor-core MMA (W as the 2:4 operand).
 * Storage:
 *   Wq24  u8 [N, K_i / 4]: byte t = the group's lower kept code (bits 0-3)
 *         and higher kept code (bits 4-7), two's complement nibbles;
 *   Wmeta u8 [N, K_i / 8]: group t's positions i0 | i1 << 2 (i0 < i1) in
 *         bits 4 (t % 2) .. 4 (t % 2) + 3 of byte t / 2.
 * Shapes: group_size 0, INT4 activations and weights (act_bits, weight_bits
 * 0 or 4), K_i % 128 == 0, k_o <= 128 (FP16) or 256 (INT8); anything else
 * returns QUIK_ERR_UNSUPPORTED.  Activations are dense (quik_quantize_reorder).
 */

/*
 * quik_pack_weights_24 -- offline: prune W [N, K] fp16 to 2:4 as above,
 * quantise and store the kept codes, position pairs, per-channel scales
 * w_scale [N] and the outlier block Wo / wo_scale (as quik_pack_weights).
 */
QUIK_API quik_status quik_pack_weights_24(const quik_shape *shape, const void *W_f16,
                                          const int32_t *perm, void *Wq24, void *Wmeta,
                                          float *w_scale, void *Wo, float *wo_scale,
                                          quik_stream_t stream);

/*
 * quik_gemm_24 -- quik_gemm with 2:4-sparse weights (Wq24, Wmeta): exact
 * integer sums over the kept positions, the outlier product and the same
 * dequantising epilogue.  Tiles of 128 output channels x 32 tokens.
 */
QUIK_API quik_status quik_gemm_24(const quik_shape *shape, const void *Xq, const float *x_scale,
                                  const void *Xo, const float *xo_scale, const void *Wq24,
                                  const void *Wmeta, const float *w_scale, const void *Wo,
                                  const float *wo_scale, const void *bias_f16, void *Y_f16,
                                  quik_stream_t stream);

/*
 * quik_expand_weights_24 -- the dense packed INT4 weights Wq [N, K_i / 2]
 * (the layout of quik_pack_weights) that 2:4 weights stand for: the kept
 * codes at their positions, zero elsewhere.  quik_gemm on them gives the
 * same integer sums as quik_gemm_24 on (Wq24, Wmeta).  Needs only
 * K_i % 128 == 0 (else QUIK_ERR_UNSUPPORTED); shape->M is not used.
 */
QUIK_API quik_status quik_expand_weights_24(const quik_shape *shape, const void *Wq24,
                                            const void *Wmeta, void *Wq, quik_stream_t stream);

/*
 * quik_workspace_size_24 -- bytes of workspace quik_linear_24 needs:
 * quik_workspace_size(shape), plus room for the expanded weights when
 * M > 32.  Returns 0 for a shape the 2:4 path does not take.
 */
QUIK_API size_t quik_workspace_size_24(const quik_shape *shape);

/*
 * quik_linear_24 -- quik_quantize_reorder into `workspace`
 * (quik_workspace_size_24(shape) bytes) followed by the product.  Up to 32
 * tokens the product is quik_gemm_24 (the sparse MMA: 3 bits per weight
 * position cross HBM instead of 4).  With more tokens the weights are
 * expanded into the workspace (quik_expand_weights_24) and quik_gemm's dense
 * kernel runs: the sparse MMA's dense operand would take all of an SM's
 * shared-memory bandwidth at prefill tile widths.  The integer sums are the
 * same either way.
 */
QUIK_API quik_status quik_linear_24(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                                    const void *Wq24, const void *Wmeta, const float *w_scale,
                                    const void *Wo, const float *wo_scale, const void *bias_f16,
                                    void *Y_f16, void *workspace, size_t workspace_bytes,
                                    quik_stream_t stream);

/*
 * quik_gemm_24_i32_debug -- test entry: the sparse product's integer sums
 * acc [M, N] int32 (and the INT8 outlier sums, as quik_gemm_i32_debug).
 */
QUIK_API quik_status quik_gemm_24_i32_debug(const quik_shape *shape, const void *Xq,
                                            const void *Wq24, const void *Wmeta, const void *Xo,
                                            const void *Wo, int32_t *acc, int32_t *acc_outlier,
                                            quik_stream_t stream);

/*
 * quik_linear_noalloc -- quik_linear for callers that cannot allocate device
 * memory.  (No counterpart in the papers; an addition of this library.)
 *
 * Some callers have no way to provide quik_linear's workspace: a host
 * framework that owns every device allocation through a fixed memory plan and
 * hands its plugins no workspace, or a latency-critical path that must not
 * call cudaMalloc, which may synchronise the whole device.  This entry point
 * takes the same arguments as quik_linear minus the workspace and uses a
 * workspace of QUIK_NOALLOC_SCRATCH_BYTES that the library keeps in its own
 * device data segment: every GPU that loads the library holds it until the
 * process exits.  Calls allocate and free nothing (but see the first call,
 * below).
 *   - Shapes whose quik_workspace_size exceeds QUIK_NOALLOC_SCRATCH_BYTES
 *     return QUIK_ERR_UNSUPPORTED (use quik_linear with your own workspace).
 *   - All calls on a device share that one workspace: two calls whose work
 *     overlaps on the GPU (different streams, no ordering between them) race
 *     and may corrupt each other's results.  Order them on one stream.
 *   - The workspace keeps the last call's contents; each call rewrites every
 *     byte it reads, so no clearing is needed.
 *   - The first call on each device looks up the workspace's device address
 *     (with that device current) and caches it; make that first call before
 *     any stream capture.  Under CUDA's default lazy module loading, that
 *     first call is also when the runtime loads the library's device module
 *     on the device and commits the workspace's memory, which can allocate
 *     and synchronise.  A caller that may not allocate at all should make
 *     one warm-up call (or run with CUDA_MODULE_LOADING=EAGER, which commits
 *     the workspace when the library's module loads) before entering the
 *     region where allocation is forbidden; later calls allocate nothing.
 *   - The cached address belongs to the device's current context: after
 *     cudaDeviceReset on a device, do not call this entry point on that
 *     device again in the same process.
 * Errors and argument rules are those of quik_linear.
 */
#define QUIK_NOALLOC_SCRATCH_BYTES (64u << 20)
QUIK_API quik_status quik_linear_noalloc(const quik_shape *shape, const void *X_f16,
                                         const int32_t *perm, const void *Wq,
                                         const float *w_scale, const void *Wo,
                                         const float *wo_scale, const void *bias_f16,
                                         void *Y_f16, quik_stream_t stream);

/*
 * quik_gemm_i32_debug -- test entry: the exact integer sums of the INT4 part
 * as computed by the tensor-core main loop, acc [M, N] int32 (or [G, M, N]
 * with groups), and for INT8 outliers the outlier block's integer sums
 * acc_outlier [M, N] (NULL otherwise).
 */
QUIK_API quik_status quik_gemm_i32_debug(const quik_shape *shape, const void *Xq, const void *Wq,
                                const void *Xo, const void *Wo, int32_t *acc,
                                int32_t *acc_outlier, quik_stream_t stream);

/*
 * quik_sync_check -- synchronise `stream`, then report the device error
 * counters of the current device: QUIK_ERR_TIMEOUT if a bounded wait ran out
 * in any kernel since the previous check, else QUIK_ERR_INVALID_ARG if a
 * quantiser met a perm entry outside [0, K) since then, QUIK_ERR_CUDA on a
 * CUDA error, else QUIK_OK.  The counters are never reset on the device (a
 * kernel running on another stream meanwhile is not disturbed); each check
 * reports what was added since the previous one, whichever stream it came
 * from.
 */
QUIK_API quik_status quik_sync_check(quik_stream_t stream);

/*
 * quik_selftest_timeout -- test entry for the failure detector: launches one
 * CTA that waits on a barrier nothing will complete, with a wait limit of
 * `limit_us` microseconds (1 .. 1000000).  The wait runs out, the kernel
 * records QUIK_ERR_TIMEOUT and returns; quik_sync_check then reports it.
 */
QUIK_API quik_status quik_selftest_timeout(uint32_t limit_us, quik_stream_t stream);

/*
 * quik_test_stall -- test entry: makes a production kernel take its timeout
 * path without a fault.  site 1: each team leader of the quantiser
 * (quik_quantize_reorder and the layer calls' quantiser) first waits on a
 * barrier that nothing completes; site 2: the persistent GEMM's MMA issuer
 * (more than 32 tokens, per-channel scales, FP16 or no outliers) does.  The
 * wait runs out after the kernels' limit (2 s), the kernel records the error
 * and exits through its abort path (its other waits give up at once), and
 * quik_sync_check reports QUIK_ERR_TIMEOUT; that call's outputs are
 * unspecified.  site 0 restores normal operation.  The switch is global to
 * the library and the device that is current; it is copied synchronously.
 * Returns QUIK_ERR_INVALID_ARG for another site, QUIK_ERR_CUDA if the copy
 * fails.
 */
QUIK_API quik_status quik_test_stall(int site);

/* Static string for a status code. */
QUIK_API const char *quik_status_string(quik_status status);

#ifdef __cplusplus
}
#endif

#endif /* QUIK_H_ */
