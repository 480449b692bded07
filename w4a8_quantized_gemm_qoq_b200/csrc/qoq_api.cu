// C-ABI entry points of libqoq.so (declared in include/qoq.h): argument
// validation, size queries and dispatch to the kernels. Nothing here
// allocates, frees or synchronises; every launch goes to the caller's stream.
#include <cmath>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qoq_internal.h"

using namespace qoq;

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

qoq_status check_nk(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return QOQ_ERR_INVALID_ARG;
    if (N % kTileN != 0 || K % kTileK != 0 || K > kMaxK || N > (int64_t)INT32_MAX / 2) return QOQ_ERR_UNSUPPORTED;
    return QOQ_OK;
}

qoq_status check_group(int group) {
    return (group == kGroup || group == 0) ? QOQ_OK : QOQ_ERR_INVALID_ARG;
}

qoq_status gemm_common(const int8_t *X8, const void *s_x, const int32_t *rowsum, const void *blob, int64_t M,
                       int64_t N, int64_t K, int group, void *out, bool fp16_out, void *ws, size_t *ws_bytes,
                       void *stream, bool saturating = false) {
    if (ws_bytes == nullptr) return QOQ_ERR_INVALID_ARG;
    if (M < 0 || M > INT32_MAX) return QOQ_ERR_INVALID_ARG;
    qoq_status st = check_nk(N, K);
    if (st != QOQ_OK) return st;
    if ((st = check_group(group)) != QOQ_OK) return st;
    if (M * N > (int64_t)1 << 40) return QOQ_ERR_UNSUPPORTED;
    const size_t need = workspace_bytes_for(M, N, K);
    if (ws == nullptr) {
        *ws_bytes = need;
        return QOQ_OK;
    }
    if (*ws_bytes < need) return QOQ_ERR_WORKSPACE;
    if (M == 0) return QOQ_OK;
    if (X8 == nullptr || blob == nullptr || out == nullptr) return QOQ_ERR_INVALID_ARG;
    if (fp16_out && s_x == nullptr) return QOQ_ERR_INVALID_ARG;
    if (group == 0 && rowsum == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned(X8, 16) || !aligned(blob, 16) || !aligned(out, 16) || !aligned(ws, 16)) return QOQ_ERR_ALIGNMENT;
    if ((s_x && !aligned(s_x, 2)) || (rowsum && !aligned(rowsum, 4))) return QOQ_ERR_ALIGNMENT;
    GemmArgs a;
    a.X8 = X8;
    a.s_x = s_x;
    a.rowsum = rowsum;
    a.blob = blob;
    a.M = M;
    a.N = N;
    a.K = K;
    a.group = group;
    a.out = out;
    a.fp16_out = fp16_out;
    a.ws = ws;
    a.saturating = saturating;
    a.ws_capacity = *ws_bytes;
    return launch_gemm(a, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

qoq_status qoq_quantize_act_per_token(const void *X_fp16, int64_t M, int64_t K, int8_t *X8, void *s_x_fp16,
                                      int32_t *rowsum, void *stream) {
    if (M < 0 || M > INT32_MAX || K <= 0) return QOQ_ERR_INVALID_ARG;
    if (K % kTileK != 0 || K > kMaxK) return QOQ_ERR_UNSUPPORTED;
    if (M == 0) return QOQ_OK;
    if (X_fp16 == nullptr || X8 == nullptr || s_x_fp16 == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned(X_fp16, 16) || !aligned(X8, 16) || !aligned(s_x_fp16, 2) || (rowsum && !aligned(rowsum, 4)))
        return QOQ_ERR_ALIGNMENT;
    return launch_act_quant(X_fp16, M, K, X8, s_x_fp16, rowsum, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_rmsnorm_quant(const void *X_fp16, const void *gamma_fp16, int64_t M, int64_t K, float eps,
                             int8_t *X8, void *s_x_fp16, int32_t *rowsum, void *stream) {
    if (M < 0 || M > INT32_MAX || K <= 0) return QOQ_ERR_INVALID_ARG;
    if (!(eps > 0.0f) || !(eps < INFINITY)) return QOQ_ERR_INVALID_ARG;
    if (K % 8 != 0 || K > kMaxProducerWidth) return QOQ_ERR_UNSUPPORTED;
    if (M == 0) return QOQ_OK;
    if (X_fp16 == nullptr || gamma_fp16 == nullptr || X8 == nullptr || s_x_fp16 == nullptr)
        return QOQ_ERR_INVALID_ARG;
    if (!aligned(X_fp16, 16) || !aligned(gamma_fp16, 16) || !aligned(X8, 16) || !aligned(s_x_fp16, 2) ||
        (rowsum && !aligned(rowsum, 4)))
        return QOQ_ERR_ALIGNMENT;
    return launch_rmsnorm_quant(X_fp16, gamma_fp16, M, K, eps, X8, s_x_fp16, rowsum,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_silu_mul_quant(const void *GU_fp16, int64_t M, int64_t I, int8_t *X8, void *s_x_fp16,
                              int32_t *rowsum, void *stream) {
    if (M < 0 || M > INT32_MAX || I <= 0) return QOQ_ERR_INVALID_ARG;
    if (I % 8 != 0 || I > kMaxProducerWidth) return QOQ_ERR_UNSUPPORTED;
    if (M == 0) return QOQ_OK;
    if (GU_fp16 == nullptr || X8 == nullptr || s_x_fp16 == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned(GU_fp16, 16) || !aligned(X8, 16) || !aligned(s_x_fp16, 2) || (rowsum && !aligned(rowsum, 4)))
        return QOQ_ERR_ALIGNMENT;
    return launch_silu_mul_quant(GU_fp16, M, I, X8, s_x_fp16, rowsum, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_quantize_weights(const void *W_fp16, int64_t N, int64_t K, int group_size, void *blob,
                                size_t *blob_bytes, void *stream) {
    if (blob_bytes == nullptr) return QOQ_ERR_INVALID_ARG;
    qoq_status st = check_nk(N, K);
    if (st != QOQ_OK) return st;
    if ((st = check_group(group_size)) != QOQ_OK) return st;
    const BlobLayout L = blob_layout(N, K, group_size);
    if (blob == nullptr) {
        *blob_bytes = (size_t)L.total;
        return QOQ_OK;
    }
    if (*blob_bytes < (size_t)L.total) return QOQ_ERR_WORKSPACE;
    if (W_fp16 == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned(W_fp16, 16) || !aligned(blob, 16)) return QOQ_ERR_ALIGNMENT;
    return launch_weight_quant(W_fp16, N, K, group_size, blob, L, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_w4a8_gemm(const int8_t *X8, const int32_t *rowsum, const void *blob, int64_t M, int64_t N,
                         int64_t K, int group_size, int32_t *acc, void *workspace, size_t *workspace_bytes,
                         void *stream) {
    return gemm_common(X8, nullptr, rowsum, blob, M, N, K, group_size, acc, false, workspace, workspace_bytes,
                       stream);
}

qoq_status qoq_gemm_fp16_out(const int8_t *X8, const void *s_x_fp16, const int32_t *rowsum, const void *blob,
                             int64_t M, int64_t N, int64_t K, int group_size, void *Y_fp16, void *workspace,
                             size_t *workspace_bytes, void *stream) {
    return gemm_common(X8, s_x_fp16, rowsum, blob, M, N, K, group_size, Y_fp16, true, workspace,
                       workspace_bytes, stream);
}

qoq_status qoq_gemm_fp16_out_saturating(const int8_t *X8, const void *s_x_fp16, const void *blob, int64_t M,
                                        int64_t N, int64_t K, int group_size, void *Y_fp16, void *workspace,
                                        size_t *workspace_bytes, void *stream) {
    // Built for group_size 128 and two token tiles: M <= 16, and M > 512 on
    // CTA pairs (N / 128 even).
    if (group_size != kGroup) return QOQ_ERR_UNSUPPORTED;
    if (M > 16 && (M <= 512 || token_tile_for(M, N, K) != 256 || (N / kTileN) % 2 != 0)) return QOQ_ERR_UNSUPPORTED;
    return gemm_common(X8, s_x_fp16, nullptr, blob, M, N, K, group_size, Y_fp16, true, workspace, workspace_bytes,
                       stream, true);
}

qoq_status qoq_w4a8_linear(const void *X_fp16, const void *blob, int64_t M, int64_t N, int64_t K, int group_size,
                           void *Y_fp16, void *workspace, size_t *workspace_bytes, void *stream) {
    if (workspace_bytes == nullptr) return QOQ_ERR_INVALID_ARG;
    if (M < 0 || M > INT32_MAX) return QOQ_ERR_INVALID_ARG;
    qoq_status st = check_nk(N, K);
    if (st != QOQ_OK) return st;
    if ((st = check_group(group_size)) != QOQ_OK) return st;
    if (M * N > (int64_t)1 << 40 || M * K > (int64_t)1 << 40) return QOQ_ERR_UNSUPPORTED;
    const size_t need = linear_workspace_bytes(M, N, K);
    if (workspace == nullptr) {
        *workspace_bytes = need;
        return QOQ_OK;
    }
    if (*workspace_bytes < need) return QOQ_ERR_WORKSPACE;
    if (M == 0) return QOQ_OK;
    if (X_fp16 == nullptr || blob == nullptr || Y_fp16 == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned(X_fp16, 16) || !aligned(blob, 16) || !aligned(Y_fp16, 16) || !aligned(workspace, 256))
        return QOQ_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const FusedLayout F = fused_layout(M, K, workspace_bytes_for(M, N, K));
    GemmArgs a;
    a.blob = blob;
    a.M = M;
    a.N = N;
    a.K = K;
    a.group = group_size;
    a.out = Y_fp16;
    a.fp16_out = true;
    a.ws = workspace;
    a.ws_capacity = *workspace_bytes;
    const int tok = token_tile_for(M, N, K);
    if (tok <= kDecodeMaxTok && linear_fused(M, N, K)) {
        // One launch: the decode kernel quantises the rows itself.
        a.X = X_fp16;
        a.X8 = nullptr;
        a.s_x = nullptr;
        a.rowsum = nullptr;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return QOQ_ERR_CUDA;
        return launch_decode_gemm(a, s, tok, sms < kMaxGrid ? sms : kMaxGrid);
    }
    // Otherwise the per-token quantiser, then the GEMM, both into and out of
    // the workspace.
    int8_t *X8 = reinterpret_cast<int8_t *>(ws + F.off_x8);
    void *s_x = ws + F.off_sx;
    int32_t *rowsum = reinterpret_cast<int32_t *>(ws + F.off_rowsum);
    if (launch_act_quant(X_fp16, M, K, X8, s_x, rowsum, s) != cudaSuccess) return QOQ_ERR_CUDA;
    a.X8 = X8;
    a.s_x = s_x;
    a.rowsum = rowsum;
    return launch_gemm(a, s);
}

qoq_status qoq_kv4_cache_write(const void *src_fp16, int64_t B, int64_t Hkv, int64_t max_tokens, int64_t t0,
                               int64_t n_tokens, int64_t D, uint8_t *codes, void *scales_fp16, void *zeros_fp16,
                               void *stream) {
    if (B < 0 || Hkv <= 0 || max_tokens <= 0 || t0 < 0 || n_tokens < 0) return QOQ_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return QOQ_ERR_UNSUPPORTED;
    if (t0 + n_tokens > max_tokens || max_tokens > INT32_MAX) return QOQ_ERR_INVALID_ARG;
    if (B * Hkv * max_tokens > ((int64_t)1 << 40)) return QOQ_ERR_UNSUPPORTED;
    if (B == 0 || n_tokens == 0) return QOQ_OK;
    if (src_fp16 == nullptr || codes == nullptr || scales_fp16 == nullptr || zeros_fp16 == nullptr)
        return QOQ_ERR_INVALID_ARG;
    if (!aligned(src_fp16, 16) || !aligned(codes, 16) || !aligned(scales_fp16, 2) || !aligned(zeros_fp16, 2))
        return QOQ_ERR_ALIGNMENT;
    return launch_kv4_cache_write(src_fp16, B, Hkv, max_tokens, t0, n_tokens, D, codes, scales_fp16, zeros_fp16,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_kv4_decode_attention(const void *q_fp16, const uint8_t *k_codes, const void *k_scales,
                                    const void *k_zeros, const uint8_t *v_codes, const void *v_scales,
                                    const void *v_zeros, const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv,
                                    int64_t max_tokens, int64_t D, void *out_fp16, void *workspace,
                                    size_t *workspace_bytes, void *stream) {
    if (workspace_bytes == nullptr) return QOQ_ERR_INVALID_ARG;
    if (B < 0 || Hq <= 0 || Hkv <= 0 || max_tokens <= 0) return QOQ_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || Hq / Hkv > 8 || (D != 64 && D != 128)) return QOQ_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535 || max_tokens > INT32_MAX / 2) return QOQ_ERR_UNSUPPORTED;
    const size_t need = kv4_workspace_bytes(B, Hkv, max_tokens, D);
    if (workspace == nullptr) {
        *workspace_bytes = need;
        return QOQ_OK;
    }
    if (*workspace_bytes < need) return QOQ_ERR_WORKSPACE;
    if (B == 0) return QOQ_OK;
    if (q_fp16 == nullptr || k_codes == nullptr || k_scales == nullptr || k_zeros == nullptr || v_codes == nullptr ||
        v_scales == nullptr || v_zeros == nullptr || out_fp16 == nullptr)
        return QOQ_ERR_INVALID_ARG;
    if (!aligned(q_fp16, 16) || !aligned(k_codes, 16) || !aligned(v_codes, 16) || !aligned(out_fp16, 16) ||
        !aligned(workspace, 256) || !aligned(k_scales, 2) || !aligned(k_zeros, 2) || !aligned(v_scales, 2) ||
        !aligned(v_zeros, 2) || (seq_lens && !aligned(seq_lens, 4)))
        return QOQ_ERR_ALIGNMENT;
    return launch_kv4_attention(q_fp16, k_codes, k_scales, k_zeros, v_codes, v_scales, v_zeros, seq_lens, B, Hq, Hkv,
                                max_tokens, D, out_fp16, workspace, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

qoq_status qoq_plan(int64_t M, int64_t N, int64_t K, int32_t *token_tile, int32_t *linear_launches) {
    if (M < 0 || M > INT32_MAX) return QOQ_ERR_INVALID_ARG;
    qoq_status st = check_nk(N, K);
    if (st != QOQ_OK) return st;
    const int tok = token_tile_for(M, N, K);
    if (token_tile) *token_tile = tok;
    if (linear_launches) *linear_launches = (tok <= kDecodeMaxTok && linear_fused(M, N, K)) ? 1 : 2;
    return QOQ_OK;
}

const char *qoq_status_string(qoq_status status) {
    switch (status) {
        case QOQ_OK: return "QOQ_OK";
        case QOQ_ERR_INVALID_ARG: return "QOQ_ERR_INVALID_ARG";
        case QOQ_ERR_UNSUPPORTED: return "QOQ_ERR_UNSUPPORTED";
        case QOQ_ERR_ALIGNMENT: return "QOQ_ERR_ALIGNMENT";
        case QOQ_ERR_WORKSPACE: return "QOQ_ERR_WORKSPACE";
        case QOQ_ERR_BAD_BLOB: return "QOQ_ERR_BAD_BLOB";
        case QOQ_ERR_CUDA: return "QOQ_ERR_CUDA";
        case QOQ_ERR_TIMEOUT: return "QOQ_ERR_TIMEOUT";
    }
    return "QOQ_ERR_UNKNOWN";
}

}  // extern "C"
