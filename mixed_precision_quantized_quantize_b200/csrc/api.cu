// api.cu -- the extern "C" entry points declared in include/quik.h:
// argument validation, workspace layout and kernel dispatch.  No device
// memory is allocated here; every buffer belongs to the caller.
#include <cmath>
#include <cstdint>

#include "quik_internal.h"

namespace {

using quik::kGroup;
using quik::kMaxK;
using quik::kMaxKNorm;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }
inline bool ok_opt(const void *p) { return p == nullptr || aligned16(p); }
inline size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

quik_status check_shape(const quik_shape *s) {
    if (s == nullptr) return QUIK_ERR_INVALID_ARG;
    if (s->M < 1 || s->N < 1 || s->K < 1 || s->K > kMaxK) return QUIK_ERR_INVALID_ARG;
    if (s->k_o < 0 || s->k_o > s->K) return QUIK_ERR_INVALID_ARG;
    const int Ki = s->K - s->k_o;
    if (Ki % 32 != 0 || s->k_o % 16 != 0) return QUIK_ERR_INVALID_ARG;
    if (s->group_size < 0) return QUIK_ERR_INVALID_ARG;
    if (s->group_size != 0 && s->group_size != kGroup) return QUIK_ERR_UNSUPPORTED;
    if (s->group_size == kGroup && Ki % kGroup != 0) return QUIK_ERR_INVALID_ARG;
    if (s->outlier != QUIK_OUTLIER_FP16 && s->outlier != QUIK_OUTLIER_INT8)
        return QUIK_ERR_INVALID_ARG;
    if (s->act_bits != 0 && s->act_bits != 4 && s->act_bits != 8) return QUIK_ERR_INVALID_ARG;
    if (s->weight_bits != 0 && s->weight_bits != 4 && s->weight_bits != 8) return QUIK_ERR_INVALID_ARG;
    if (s->act_bits == 8 && s->group_size != 0) return QUIK_ERR_UNSUPPORTED;
    if (s->weight_bits == 8 && s->act_bits != 8) return QUIK_ERR_UNSUPPORTED;
    return QUIK_OK;
}

inline int groups_of(const quik_shape *s) {
    const int Ki = s->K - s->k_o;
    return s->group_size > 0 ? Ki / s->group_size : 1;
}
inline bool needs_scale(const quik_shape *s) { return groups_of(s) > 0; }
inline bool int8_out(const quik_shape *s) { return s->outlier == QUIK_OUTLIER_INT8; }
inline bool act8(const quik_shape *s) { return s->act_bits == 8; }
inline bool wt8(const quik_shape *s) { return s->weight_bits == 8; }
// quik_linear's quantiser writes the wide INT4 form (the bytes 16 c, read by
// the persistent GEMM without unpacking) exactly when that kernel takes the
// product: per-channel scales, INT4 activations and weights, FP16 or no
// outliers, K_i > 0 and more than kDecodeTokens tokens.
inline bool wide_acts(const quik_shape *s) {
    return s->group_size == 0 && !act8(s) && !wt8(s) && s->K - s->k_o > 0 &&
           (s->k_o == 0 || !int8_out(s)) && s->M > quik::kDecodeTokens;
}

// Rows of one operand: packed codes, scales, outlier block (+ INT8 scales).
quik_status check_quant_ptrs(const quik_shape *s, const void *Q, const float *scale,
                             const void *O, const float *o_scale) {
    const int Ki = s->K - s->k_o;
    if (Ki > 0 && !ok_ptr(Q)) return QUIK_ERR_INVALID_ARG;
    if (needs_scale(s) && !ok_ptr(scale)) return QUIK_ERR_INVALID_ARG;
    if (s->k_o > 0 && !ok_ptr(O)) return QUIK_ERR_INVALID_ARG;
    if (int8_out(s) && s->k_o > 0 && !ok_ptr(o_scale)) return QUIK_ERR_INVALID_ARG;
    if (!ok_opt(Q) || !ok_opt(scale) || !ok_opt(O) || !ok_opt(o_scale)) return QUIK_ERR_INVALID_ARG;
    return QUIK_OK;
}

// bits8: INT8 codes (activations with act_bits 8, weights with weight_bits 8).
// gamma (optional): the rows are RMS-normalised with this weight and eps first.
quik_status quantize(const quik_shape *s, int rows, bool bits8, const void *X, const int32_t *perm,
                     void *Q, float *scale, void *O, float *o_scale, cudaStream_t stream,
                     const void *gamma = nullptr, float eps = 0.0f, bool wide = false) {
    quik::QuantizeArgs a;
    a.X = static_cast<const uint16_t *>(X);
    a.perm = perm;
    a.rows = rows;
    a.K = s->K;
    a.k_o = s->k_o;
    a.group = s->group_size;
    a.out_int8 = int8_out(s);
    a.bits8 = bits8;
    a.wide = wide;
    a.Q = static_cast<uint8_t *>(Q);
    a.scale = scale;
    a.O = O;
    a.o_scale = o_scale;
    a.gamma = static_cast<const uint16_t *>(gamma);
    a.eps = eps;
    return quik::launch_quantize_rows(a, stream) == cudaSuccess ? QUIK_OK : QUIK_ERR_CUDA;
}

// The RMS norm's weight and epsilon: gamma [K] fp16, eps finite and > 0.
inline bool ok_norm(const void *gamma, float eps) {
    return ok_ptr(gamma) && std::isfinite(eps) && eps > 0.0f;
}

// 2:4-sparse weights: INT4 codes with per-channel scales, K_i % 128 == 0 (the
// rows of position pairs are whole 16-byte units), and an outlier block of at
// most 128 FP16 or 256 INT8 channels.
quik_status check_shape24(const quik_shape *s) {
    quik_status st = check_shape(s);
    if (st != QUIK_OK) return st;
    if (s->group_size != 0 || act8(s) || wt8(s) || (s->K - s->k_o) % 128 != 0 ||
        s->k_o > (int8_out(s) ? 256 : 128))
        return QUIK_ERR_UNSUPPORTED;
    return QUIK_OK;
}

// Kept codes [rows, K_i / 4], position pairs [rows, K_i / 8], per-row scales.
quik_status check_ptrs24(const quik_shape *s, const void *Qs, const void *meta, const float *scale,
                         const void *O, const float *o_scale) {
    const int Ki = s->K - s->k_o;
    if (Ki > 0 && (!ok_ptr(Qs) || !ok_ptr(meta) || !ok_ptr(scale))) return QUIK_ERR_INVALID_ARG;
    if (s->k_o > 0 && !ok_ptr(O)) return QUIK_ERR_INVALID_ARG;
    if (int8_out(s) && s->k_o > 0 && !ok_ptr(o_scale)) return QUIK_ERR_INVALID_ARG;
    if (!ok_opt(Qs) || !ok_opt(meta) || !ok_opt(scale) || !ok_opt(O) || !ok_opt(o_scale))
        return QUIK_ERR_INVALID_ARG;
    return QUIK_OK;
}

// 2:4 layers of more tokens than one sparse tile run the dense kernel on the
// weights expanded into the workspace (the sparse MMA's B operand would take
// all of an SM's shared-memory bandwidth at prefill tile widths).
constexpr int kSparseTokens = 32;

struct Workspace {
    size_t xq, sx, xo, sxo, total;
};

Workspace layout(const quik_shape *s) {
    const size_t M = static_cast<size_t>(s->M);
    const size_t Ki = static_cast<size_t>(s->K - s->k_o);
    const size_t G = static_cast<size_t>(groups_of(s));
    Workspace w;
    w.xq = 0;
    w.sx = w.xq + round256(act8(s) || wide_acts(s) ? M * Ki : M * Ki / 2);
    w.xo = w.sx + round256(M * G * sizeof(float));
    w.sxo = w.xo + round256(M * s->k_o * (int8_out(s) ? 1 : 2));
    w.total = w.sxo + round256(int8_out(s) ? M * sizeof(float) : 0);
    return w;
}

}  // namespace

extern "C" {

size_t quik_workspace_size(const quik_shape *shape) {
    if (check_shape(shape) != QUIK_OK) return 0;
    return layout(shape).total;
}

quik_status quik_quantize_reorder(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                                  void *Xq, float *x_scale, void *Xo, float *xo_scale,
                                  quik_stream_t stream) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(X_f16) || !ok_ptr(perm)) return QUIK_ERR_INVALID_ARG;
    if ((st = check_quant_ptrs(shape, Xq, x_scale, Xo, xo_scale)) != QUIK_OK) return st;
    return quantize(shape, shape->M, act8(shape), X_f16, perm, Xq, x_scale, Xo, xo_scale,
                    static_cast<cudaStream_t>(stream));
}

quik_status quik_rmsnorm_quantize_reorder(const quik_shape *shape, const void *X_f16,
                                          const void *gamma_f16, float eps, const int32_t *perm,
                                          void *Xq, float *x_scale, void *Xo, float *xo_scale,
                                          quik_stream_t stream) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(X_f16) || !ok_ptr(perm) || !ok_norm(gamma_f16, eps)) return QUIK_ERR_INVALID_ARG;
    if ((st = check_quant_ptrs(shape, Xq, x_scale, Xo, xo_scale)) != QUIK_OK) return st;
    if (shape->K > kMaxKNorm) return QUIK_ERR_UNSUPPORTED;
    return quantize(shape, shape->M, act8(shape), X_f16, perm, Xq, x_scale, Xo, xo_scale,
                    static_cast<cudaStream_t>(stream), gamma_f16, eps);
}

quik_status quik_pack_weights(const quik_shape *shape, const void *W_f16, const int32_t *perm,
                              void *Wq, float *w_scale, void *Wo, float *wo_scale,
                              quik_stream_t stream) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(W_f16) || !ok_ptr(perm)) return QUIK_ERR_INVALID_ARG;
    if ((st = check_quant_ptrs(shape, Wq, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    return quantize(shape, shape->N, wt8(shape), W_f16, perm, Wq, w_scale, Wo, wo_scale,
                    static_cast<cudaStream_t>(stream));
}

static quik_status gemm_impl(const quik_shape *shape, const void *Xq, const float *x_scale,
                             const void *Xo, const float *xo_scale, const void *Wq,
                             const float *w_scale, const void *Wo, const float *wo_scale,
                             const void *bias, void *Y, bool debug, int32_t *acc,
                             int32_t *acc_o, cudaStream_t stream, bool after_quantize = false,
                             bool x_wide = false) {
    quik::GemmArgs a;
    a.M = shape->M;
    a.N = shape->N;
    a.K = shape->K;
    a.k_o = shape->k_o;
    a.group = shape->group_size;
    a.out_int8 = int8_out(shape);
    a.a8 = act8(shape);
    a.w8 = wt8(shape);
    a.x_wide = x_wide;
    a.Xq = Xq;
    a.sx = x_scale;
    a.Xo = Xo;
    a.sxo = xo_scale;
    a.Wq = Wq;
    a.sw = w_scale;
    a.Wo = Wo;
    a.swo = wo_scale;
    a.bias = static_cast<const uint16_t *>(bias);
    a.Y = static_cast<uint16_t *>(Y);
    a.debug = debug;
    a.after_quantize = after_quantize;
    a.acc_dbg = acc;
    a.acc_o_dbg = acc_o;
    return quik::launch_gemm(a, stream);
}

quik_status quik_gemm(const quik_shape *shape, const void *Xq, const float *x_scale,
                      const void *Xo, const float *xo_scale, const void *Wq,
                      const float *w_scale, const void *Wo, const float *wo_scale,
                      const void *bias_f16, void *Y_f16, quik_stream_t stream) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    if ((st = check_quant_ptrs(shape, Xq, x_scale, Xo, xo_scale)) != QUIK_OK) return st;
    if ((st = check_quant_ptrs(shape, Wq, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    if (!ok_ptr(Y_f16) || !ok_opt(bias_f16)) return QUIK_ERR_INVALID_ARG;
    return gemm_impl(shape, Xq, x_scale, Xo, xo_scale, Wq, w_scale, Wo, wo_scale, bias_f16, Y_f16,
                     false, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

static quik_status linear_impl(const quik_shape *shape, const void *X_f16, const void *gamma,
                               float eps, const int32_t *perm, const void *Wq,
                               const float *w_scale, const void *Wo, const float *wo_scale,
                               const void *bias_f16, void *Y_f16, void *workspace,
                               size_t workspace_bytes, quik_stream_t stream,
                               cudaEvent_t between = nullptr) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(X_f16) || !ok_ptr(perm) || !ok_ptr(Y_f16) || !ok_opt(bias_f16))
        return QUIK_ERR_INVALID_ARG;
    if (gamma != nullptr && !ok_norm(gamma, eps)) return QUIK_ERR_INVALID_ARG;
    if (gamma != nullptr && shape->K > kMaxKNorm) return QUIK_ERR_UNSUPPORTED;
    if ((st = check_quant_ptrs(shape, Wq, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    const Workspace w = layout(shape);
    if (!ok_ptr(workspace) || workspace_bytes < w.total) return QUIK_ERR_INVALID_ARG;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *Xq = ws + w.xq;
    float *sx = reinterpret_cast<float *>(ws + w.sx);
    void *Xo = ws + w.xo;
    float *sxo = int8_out(shape) ? reinterpret_cast<float *>(ws + w.sxo) : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool wide = wide_acts(shape);
    if ((st = quantize(shape, shape->M, act8(shape), X_f16, perm, Xq, sx, Xo, sxo, s, gamma, eps,
                       wide)) != QUIK_OK)
        return st;
    // the GEMM follows this quantiser on the same stream: its set-up and weight
    // loads may overlap the quantiser's tail (not with an event between them)
    if (between != nullptr && cudaEventRecord(between, s) != cudaSuccess) return QUIK_ERR_CUDA;
    return gemm_impl(shape, Xq, sx, Xo, sxo, Wq, w_scale, Wo, wo_scale, bias_f16, Y_f16, false,
                     nullptr, nullptr, s, between == nullptr, wide);
}

quik_status quik_linear(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                        const void *Wq, const float *w_scale, const void *Wo,
                        const float *wo_scale, const void *bias_f16, void *Y_f16,
                        void *workspace, size_t workspace_bytes, quik_stream_t stream) {
    return linear_impl(shape, X_f16, nullptr, 0.0f, perm, Wq, w_scale, Wo, wo_scale, bias_f16,
                       Y_f16, workspace, workspace_bytes, stream);
}

quik_status quik_linear_timed(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                              const void *Wq, const float *w_scale, const void *Wo,
                              const float *wo_scale, const void *bias_f16, void *Y_f16,
                              void *workspace, size_t workspace_bytes, void *between,
                              quik_stream_t stream) {
    if (between == nullptr) return QUIK_ERR_INVALID_ARG;
    return linear_impl(shape, X_f16, nullptr, 0.0f, perm, Wq, w_scale, Wo, wo_scale, bias_f16,
                       Y_f16, workspace, workspace_bytes, stream, static_cast<cudaEvent_t>(between));
}

quik_status quik_rmsnorm_linear(const quik_shape *shape, const void *X_f16, const void *gamma_f16,
                                float eps, const int32_t *perm, const void *Wq,
                                const float *w_scale, const void *Wo, const float *wo_scale,
                                const void *bias_f16, void *Y_f16, void *workspace,
                                size_t workspace_bytes, quik_stream_t stream) {
    if (gamma_f16 == nullptr) return QUIK_ERR_INVALID_ARG;
    return linear_impl(shape, X_f16, gamma_f16, eps, perm, Wq, w_scale, Wo, wo_scale, bias_f16,
                       Y_f16, workspace, workspace_bytes, stream);
}

quik_status quik_pack_weights_24(const quik_shape *shape, const void *W_f16, const int32_t *perm,
                                 void *Wq24, void *Wmeta, float *w_scale, void *Wo,
                                 float *wo_scale, quik_stream_t stream) {
    quik_status st = check_shape24(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(W_f16) || !ok_ptr(perm)) return QUIK_ERR_INVALID_ARG;
    if ((st = check_ptrs24(shape, Wq24, Wmeta, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    quik::Prune24Args a;
    a.W = static_cast<const uint16_t *>(W_f16);
    a.perm = perm;
    a.rows = shape->N;
    a.K = shape->K;
    a.k_o = shape->k_o;
    a.out_int8 = int8_out(shape);
    a.Qs = static_cast<uint8_t *>(Wq24);
    a.meta = static_cast<uint8_t *>(Wmeta);
    a.scale = w_scale;
    a.O = Wo;
    a.o_scale = wo_scale;
    return quik::launch_prune24_rows(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? QUIK_OK
                                                                                        : QUIK_ERR_CUDA;
}

static quik_status gemm24_impl(const quik_shape *shape, const void *Xq, const float *x_scale,
                               const void *Xo, const float *xo_scale, const void *Wq24,
                               const void *Wmeta, const float *w_scale, const void *Wo,
                               const float *wo_scale, const void *bias, void *Y, bool debug,
                               int32_t *acc, int32_t *acc_o, cudaStream_t stream,
                               bool after_quantize = false) {
    quik::GemmArgs a;
    a.M = shape->M;
    a.N = shape->N;
    a.K = shape->K;
    a.k_o = shape->k_o;
    a.group = 0;
    a.out_int8 = int8_out(shape);
    a.a8 = false;
    a.w8 = false;
    a.Xq = Xq;
    a.sx = x_scale;
    a.Xo = Xo;
    a.sxo = xo_scale;
    a.Wq = Wq24;
    a.Wmeta = static_cast<const uint8_t *>(Wmeta);
    a.sparse24 = true;
    a.sw = w_scale;
    a.Wo = Wo;
    a.swo = wo_scale;
    a.bias = static_cast<const uint16_t *>(bias);
    a.Y = static_cast<uint16_t *>(Y);
    a.debug = debug;
    a.after_quantize = after_quantize;
    a.acc_dbg = acc;
    a.acc_o_dbg = acc_o;
    return quik::launch_gemm(a, stream);
}

quik_status quik_gemm_24(const quik_shape *shape, const void *Xq, const float *x_scale,
                         const void *Xo, const float *xo_scale, const void *Wq24,
                         const void *Wmeta, const float *w_scale, const void *Wo,
                         const float *wo_scale, const void *bias_f16, void *Y_f16,
                         quik_stream_t stream) {
    quik_status st = check_shape24(shape);
    if (st != QUIK_OK) return st;
    if ((st = check_quant_ptrs(shape, Xq, x_scale, Xo, xo_scale)) != QUIK_OK) return st;
    if ((st = check_ptrs24(shape, Wq24, Wmeta, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    if (!ok_ptr(Y_f16) || !ok_opt(bias_f16)) return QUIK_ERR_INVALID_ARG;
    return gemm24_impl(shape, Xq, x_scale, Xo, xo_scale, Wq24, Wmeta, w_scale, Wo, wo_scale,
                       bias_f16, Y_f16, false, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

size_t quik_workspace_size_24(const quik_shape *shape) {
    if (check_shape24(shape) != QUIK_OK) return 0;
    size_t total = layout(shape).total;
    if (shape->M > kSparseTokens)
        total += round256(static_cast<size_t>(shape->N) * static_cast<size_t>(shape->K - shape->k_o) / 2);
    return total;
}

quik_status quik_expand_weights_24(const quik_shape *shape, const void *Wq24, const void *Wmeta,
                                   void *Wq, quik_stream_t stream) {
    // a change of format only: the 2:4 storage rule (K_i % 128 == 0) is all it needs
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    const int Ki = shape->K - shape->k_o;
    if (Ki % 128 != 0) return QUIK_ERR_UNSUPPORTED;
    if (Ki == 0) return QUIK_OK;
    if (!ok_ptr(Wq24) || !ok_ptr(Wmeta) || !ok_ptr(Wq)) return QUIK_ERR_INVALID_ARG;
    return quik::launch_expand24(static_cast<const uint8_t *>(Wq24), static_cast<const uint8_t *>(Wmeta),
                                 shape->N, Ki, static_cast<uint8_t *>(Wq),
                                 static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QUIK_OK
               : QUIK_ERR_CUDA;
}

quik_status quik_linear_24(const quik_shape *shape, const void *X_f16, const int32_t *perm,
                           const void *Wq24, const void *Wmeta, const float *w_scale,
                           const void *Wo, const float *wo_scale, const void *bias_f16,
                           void *Y_f16, void *workspace, size_t workspace_bytes,
                           quik_stream_t stream) {
    quik_status st = check_shape24(shape);
    if (st != QUIK_OK) return st;
    if (!ok_ptr(X_f16) || !ok_ptr(perm) || !ok_ptr(Y_f16) || !ok_opt(bias_f16))
        return QUIK_ERR_INVALID_ARG;
    if ((st = check_ptrs24(shape, Wq24, Wmeta, w_scale, Wo, wo_scale)) != QUIK_OK) return st;
    const Workspace w = layout(shape);
    if (!ok_ptr(workspace) || workspace_bytes < quik_workspace_size_24(shape)) return QUIK_ERR_INVALID_ARG;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *Xq = ws + w.xq;
    float *sx = reinterpret_cast<float *>(ws + w.sx);
    void *Xo = ws + w.xo;
    float *sxo = int8_out(shape) ? reinterpret_cast<float *>(ws + w.sxo) : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (shape->M > kSparseTokens) {
        // prefill: expand the weights, quantise, then the dense kernel (the
        // GEMM directly follows the quantiser, as quik_linear's does)
        void *Wd = ws + w.total;
        const bool wide = wide_acts(shape);
        if ((st = quik_expand_weights_24(shape, Wq24, Wmeta, Wd, stream)) != QUIK_OK) return st;
        if ((st = quantize(shape, shape->M, false, X_f16, perm, Xq, sx, Xo, sxo, s, nullptr, 0.0f,
                           wide)) != QUIK_OK)
            return st;
        return gemm_impl(shape, Xq, sx, Xo, sxo, Wd, w_scale, Wo, wo_scale, bias_f16, Y_f16, false,
                         nullptr, nullptr, s, true, wide);
    }
    if ((st = quantize(shape, shape->M, false, X_f16, perm, Xq, sx, Xo, sxo, s)) != QUIK_OK) return st;
    return gemm24_impl(shape, Xq, sx, Xo, sxo, Wq24, Wmeta, w_scale, Wo, wo_scale, bias_f16, Y_f16,
                       false, nullptr, nullptr, s, true);
}

quik_status quik_gemm_24_i32_debug(const quik_shape *shape, const void *Xq, const void *Wq24,
                                   const void *Wmeta, const void *Xo, const void *Wo, int32_t *acc,
                                   int32_t *acc_outlier, quik_stream_t stream) {
    quik_status st = check_shape24(shape);
    if (st != QUIK_OK) return st;
    const int Ki = shape->K - shape->k_o;
    if (Ki > 0 && (!ok_ptr(Xq) || !ok_ptr(Wq24) || !ok_ptr(Wmeta) || !ok_ptr(acc)))
        return QUIK_ERR_INVALID_ARG;
    const bool want_o = int8_out(shape) && shape->k_o > 0;
    if (want_o && (!ok_ptr(Xo) || !ok_ptr(Wo) || !ok_ptr(acc_outlier))) return QUIK_ERR_INVALID_ARG;
    return gemm24_impl(shape, Xq, nullptr, want_o ? Xo : nullptr, nullptr, Wq24, Wmeta, nullptr,
                       want_o ? Wo : nullptr, nullptr, nullptr, nullptr, true, acc,
                       want_o ? acc_outlier : nullptr, static_cast<cudaStream_t>(stream));
}

quik_status quik_gemm_i32_debug(const quik_shape *shape, const void *Xq, const void *Wq,
                                const void *Xo, const void *Wo, int32_t *acc,
                                int32_t *acc_outlier, quik_stream_t stream) {
    quik_status st = check_shape(shape);
    if (st != QUIK_OK) return st;
    const int Ki = shape->K - shape->k_o;
    if (Ki > 0 && (!ok_ptr(Xq) || !ok_ptr(Wq) || !ok_ptr(acc))) return QUIK_ERR_INVALID_ARG;
    const bool want_o = int8_out(shape) && shape->k_o > 0;
    if (want_o && (!ok_ptr(Xo) || !ok_ptr(Wo) || !ok_ptr(acc_outlier))) return QUIK_ERR_INVALID_ARG;
    // the epilogue is skipped: scales and outputs are not read or written
    return gemm_impl(shape, Xq, nullptr, want_o ? Xo : nullptr, nullptr, Wq, nullptr,
                     want_o ? Wo : nullptr, nullptr, nullptr, nullptr, true, acc,
                     want_o ? acc_outlier : nullptr, static_cast<cudaStream_t>(stream));
}

quik_status quik_sync_check(quik_stream_t stream) {
    return quik::sync_check(static_cast<cudaStream_t>(stream));
}

quik_status quik_selftest_timeout(uint32_t limit_us, quik_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return QUIK_ERR_INVALID_ARG;
    return quik::launch_timeout_selftest(limit_us, static_cast<cudaStream_t>(stream));
}

quik_status quik_test_stall(int site) {
    if (site < 0 || site > 2) return QUIK_ERR_INVALID_ARG;
    if (quik::set_quantize_stall(site == 1) != cudaSuccess) return QUIK_ERR_CUDA;
    if (quik::set_persistent_gemm_stall(site == 2) != cudaSuccess) return QUIK_ERR_CUDA;
    return QUIK_OK;
}

const char *quik_status_string(quik_status status) {
    switch (status) {
        case QUIK_OK: return "QUIK_OK";
        case QUIK_ERR_INVALID_ARG: return "QUIK_ERR_INVALID_ARG";
        case QUIK_ERR_UNSUPPORTED: return "QUIK_ERR_UNSUPPORTED";
        case QUIK_ERR_CUDA: return "QUIK_ERR_CUDA";
        case QUIK_ERR_TIMEOUT: return "QUIK_ERR_TIMEOUT";
    }
    return "QUIK_ERR_UNKNOWN";
}

}  // extern "C"
