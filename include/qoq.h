/*
 * qoq.h -- C ABI of libqoq.so, the QoQ W4A8 GEMM for NVIDIA B200 (sm_100a).
 *
 * What it computes (QServe: W4A8KV4 Quantization and System Co-design for
 * Efficient LLM Serving, arXiv 2405.04532; paperlayer.ai summary sections 4-6,
 * study.space summary):
 *
 *   Y = diag(s_x) . (X8 . Wint^T) . diag(s_w)
 *
 * X8 are FP16 activations quantised per token to INT8 with FP16 scale s_x.
 * Wint are 4-bit weights brought back to INT8 inside the GEMM: progressive
 * group quantisation first quantises W per output channel to INT8 with an FP16
 * scale s_w, kept in the protective range [-119, 119], then quantises each
 * group of 128 INT8 values along K to UINT4 codes q with an integer scale s and
 * zero z, so Wint = (q - z) * s = q*s - z*s always fits INT8 with no
 * saturation. The product runs on INT8 tensor cores with exact INT32
 * accumulation; a fused epilogue applies s_x and s_w in FP32 and stores FP16.
 * A per-channel variant (group_size 0) has no INT8 level: UINT4 codes per
 * output channel with an FP16 scale and zero, the zero-point correction
 * z * sum_k X8 applied in the epilogue.
 *
 * Conventions for every call
 *   - All buffers are DEVICE memory owned by the caller. The library never
 *     allocates, frees or synchronises; all work is enqueued on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).
 *   - Arguments are validated before anything is launched; a failed check
 *     returns its status and enqueues nothing.
 *   - Shapes: N and K are positive multiples of 128, K <= 65536; M >= 0
 *     (M == 0 is a no-op). Matrices are row-major and dense.
 *   - Pointers to matrices, the blob and the workspace must be 16-byte
 *     aligned; scale and rowsum vectors need their natural alignment.
 *   - Inputs must be finite.
 *   - QOQ_ERR_CUDA is returned when a launch fails; errors found on the device
 *     (a blob whose header does not match the arguments, a pipeline wait that
 *     ran out) are written to the workspace status word (below).
 */
#ifndef QOQ_H
#define QOQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Leading workspace bytes that hold control words (status + arrival counters). */
#define QOQ_WORKSPACE_CONTROL_BYTES 1280

typedef enum {
    QOQ_OK = 0,
    QOQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad group size   */
    QOQ_ERR_UNSUPPORTED = 2,   /* N or K not a multiple of 128, K too large      */
    QOQ_ERR_ALIGNMENT = 3,     /* pointer misaligned                             */
    QOQ_ERR_WORKSPACE = 4,     /* blob or workspace capacity too small           */
    QOQ_ERR_BAD_BLOB = 5,      /* blob header does not match N, K, group_size    */
    QOQ_ERR_CUDA = 6,          /* a CUDA runtime call or launch failed           */
    QOQ_ERR_TIMEOUT = 7        /* a device pipeline wait ran out (status word)   */
} qoq_status;

/*
 * Per-token INT8 quantisation of activations.
 * (paperlayer.ai summary, section 6 "Evaluation": per-token INT8 activations;
 *  section 5: QServe fuses this into the preceding layer.)
 *
 *   s_x[m]    = FP16(max_k |X[m,k]| / 127)           (FP32 divide, one rounding)
 *   X8[m,k]   = clamp(RNE(X[m,k] / s_x[m]), -127, 127), 0 when s_x[m] == 0
 *   rowsum[m] = sum_k X8[m,k]
 *
 * X_fp16  [M][K] FP16, read.        X8     [M][K] int8, written.
 * s_x     [M] FP16, written.        rowsum [M] int32, written; may be NULL.
 */
qoq_status qoq_quantize_act_per_token(const void *X_fp16, int64_t M, int64_t K,
                                      int8_t *X8, void *s_x_fp16, int32_t *rowsum,
                                      void *stream);

/*
 * Fused activation producers: the layer in front of a GEMM writes the GEMM's
 * per-token INT8 activations directly, with no FP16 tensor in between.
 * (paperlayer.ai summary, section 5 "QServe Serving System", "Runtime and
 *  precision mapping": activation quantisation is fused into the preceding
 *  normalisation or activation layer.)
 *
 * Both compute an FP32 row h per token and quantise it like
 * qoq_quantize_act_per_token: s_x = FP16(max_k |h_k| / 127),
 * X8 = clamp(RNE(h / FP32(s_x)), -127, 127) (0 where s_x == 0),
 * rowsum = sum_k X8. Every floating-point step is one correctly rounded
 * binary32 operation, so the results are reproducible bit for bit:
 *
 * qoq_rmsnorm_quant (RMSNorm):
 *   ss = sum_k x_k^2 computed exactly, then rounded once to FP32;
 *   r = sqrt(ss / K + eps);  h_k = (x_k / r) * gamma_k.
 *   X_fp16 [M][K] FP16, read.   gamma_fp16 [K] FP16, read.   eps > 0, finite.
 *
 * qoq_silu_mul_quant (SiLU-gated product of a merged gate/up projection):
 *   h_k = (g_k / (1 + e^-g_k)) * u_k, with g = GU[m][0..I), u = GU[m][I..2I)
 *   and e^x in FP32 by Cody-Waite argument reduction (x = n ln2 + r), the
 *   degree-7 Taylor polynomial of e^r (Horner) and an exact scaling by 2^n
 *   (0 below x = -87.33654, +inf above x = 88.72284).
 *   GU_fp16 [M][2I] FP16, read.
 *
 * Outputs: X8 [M][K or I] int8, s_x [M] FP16, rowsum [M] int32 (may be NULL).
 * K (or I) must be a positive multiple of 8, at most 32768 (otherwise
 * QOQ_ERR_UNSUPPORTED); X, gamma, GU and X8 16-byte aligned. M == 0 is a no-op.
 */
qoq_status qoq_rmsnorm_quant(const void *X_fp16, const void *gamma_fp16, int64_t M,
                             int64_t K, float eps, int8_t *X8, void *s_x_fp16,
                             int32_t *rowsum, void *stream);

qoq_status qoq_silu_mul_quant(const void *GU_fp16, int64_t M, int64_t I, int8_t *X8,
                              void *s_x_fp16, int32_t *rowsum, void *stream);

/*
 * Offline weight quantisation and packing into the compute-order blob.
 * (paperlayer.ai summary, section 4 "Progressive Group Quantization" and
 *  section 5 "compute-aware weight reordering"; study.space summary.)
 *
 * group_size 128: level 1  s_w[n] = FP16(max_k |W[n,k]| / 119),
 *                          Q8 = clamp(RNE(W / s_w), -119, 119);
 *                 level 2  per group of 128 along K with vmin/vmax of Q8:
 *                          s = max(1, RNE((vmax - vmin) / 15)),
 *                          z = RNE(-vmin / s), q = clamp(RNE(Q8 / s) + z, 0, 15).
 * group_size 0:   per channel, range [min(0, min W), max(0, max W)]:
 *                          s = FP16(range / 15), z = RNE(-min / s) (stored FP16),
 *                          q = clamp(RNE(W / s) + z, 0, 15).
 *
 * Blob layout (little-endian): a 256-byte header (magic 'QOQW', version 1,
 * N, K, group, block bytes, section offsets, total bytes); code blocks, one per
 * (128-row n-tile, 128-column k-tile), n-tile major; each block holds the codes
 * as [chunk c = 0..3][row r = 0..127][16 bytes], where word j of a chunk covers
 * columns k0 = 32c + 8j .. k0 + 7 and its byte b is q[k0+b] | q[k0+b+4] << 4,
 * followed in group mode by [row][u8 s, s8 z*s]; then FP16 s_w (or s) [N] and,
 * per-channel, FP16 z [N], each section 256-byte aligned.
 *
 * W_fp16 [N][K] FP16, read. blob: device buffer of *blob_bytes bytes, written.
 * Size query: blob == NULL stores the required size in *blob_bytes and returns
 * QOQ_OK without launching. A capacity below it returns QOQ_ERR_WORKSPACE.
 */
qoq_status qoq_quantize_weights(const void *W_fp16, int64_t N, int64_t K, int group_size,
                                void *blob, size_t *blob_bytes, void *stream);

/*
 * W4A8 GEMM, exact INT32 result (the main loop without the FP scaling).
 * (paperlayer.ai summary, section 4: weights dequantised to INT8 in the main
 *  loop, four codes per register op; section 5: subtraction after
 *  multiplication, zero-point correction in the epilogue.)
 *
 * group_size 128: acc[m,n] = sum_k X8[m,k] * Wint[n,k]
 * group_size 0:   acc[m,n] = sum_k X8[m,k] * q[n,k] - z[n] * rowsum[m]
 *
 * X8 [M][K] int8; rowsum [M] int32 (required when group_size == 0, else may be
 * NULL); blob from qoq_quantize_weights with the same N, K, group_size;
 * acc [M][N] int32, written.
 *
 * Workspace: device memory of *workspace_bytes bytes, ZERO-FILLED by the caller
 * before its first use. Its first QOQ_WORKSPACE_CONTROL_BYTES bytes are
 * control words that every call which completes leaves zero again (an int32
 * status word at offset 0, then per-tile arrival counters); the rest is scratch for the
 * stream-K partial sums. So one workspace serves any number of calls on one
 * stream; calls that may overlap on the device need separate workspaces. The
 * status word is 0, or a qoq_status code (QOQ_ERR_BAD_BLOB, QOQ_ERR_TIMEOUT)
 * written by the device. With QOQ_ERR_TIMEOUT the next three int32 words say
 * where a bounded wait (1 s) gave up: the wait site (1 producer waiting for a
 * free stage, 2 MMA waiting for a drained accumulator, 3 MMA waiting for a
 * stage's operands, 4 dequantiser waiting for a stage's copies, 5 epilogue
 * waiting for an accumulator, 6 a flag wait (only the watchdog self-test
 * uses it), 7 last arriver of a split tile waiting for the owner's partial
 * sums, which the owner stores after it has arrived, 8 waiting
 * for every token row of the fused quantisation, 9 waiting for a free A/X
 * stage), the
 * CTA index, and the unit, segment or contributor index. After such an error,
 * zero-fill the control bytes again. Size query: workspace == NULL stores the required size for
 * (M, N, K, group_size) in *workspace_bytes and returns QOQ_OK.
 *
 * Concurrency: a tile split between CTAs is finished by whichever of them
 * arrives last, and no CTA waits for one that may not have started, so calls
 * with separate workspaces may run at the same time on different streams.
 */
qoq_status qoq_w4a8_gemm(const int8_t *X8, const int32_t *rowsum, const void *blob,
                         int64_t M, int64_t N, int64_t K, int group_size,
                         int32_t *acc, void *workspace, size_t *workspace_bytes,
                         void *stream);

/*
 * W4A8 GEMM with the fused FP16 epilogue: the timed hot path.
 * (paperlayer.ai summary, section 5: INT8 tensor cores, FP16 outputs,
 *  per-channel scaling fused into the GEMM epilogue.)
 *
 * Y[m,n] = FP16( FP32(acc[m,n]) * (FP32(s_x[m]) * FP32(s_w[n])) )
 * with acc as in qoq_w4a8_gemm and s_w the blob's per-channel FP16 scale
 * (group_size 0: the per-channel scale s).
 *
 * s_x [M] FP16; Y [M][N] FP16, written. Other arguments, the workspace and
 * its status word as for qoq_w4a8_gemm.
 */
qoq_status qoq_gemm_fp16_out(const int8_t *X8, const void *s_x_fp16, const int32_t *rowsum,
                             const void *blob, int64_t M, int64_t N, int64_t K, int group_size,
                             void *Y_fp16, void *workspace, size_t *workspace_bytes,
                             void *stream);

/*
 * The whole linear layer in one call: per-token quantisation of FP16
 * activations, then the W4A8 GEMM with the fused FP16 epilogue.
 * (paperlayer.ai summary, section 5 "QServe Serving System", "Runtime and
 *  precision mapping": activation quantisation is fused into the kernel that
 *  produces the GEMM's input, so the FP16 activations are read once.)
 *
 *   X8, s_x, rowsum = qoq_quantize_act_per_token(X)   (same arithmetic)
 *   Y = qoq_gemm_fp16_out(X8, s_x, rowsum, blob)       (same arithmetic)
 *
 * By default the call launches the quantiser and then the GEMM (two
 * launches; the GEMM's weight copies start while the quantiser runs). For
 * token tiles of at most 64 tokens (decode batches) a one-launch form is
 * built as well: the GEMM's CTAs quantise the token rows first (rows are
 * claimed from a counter in the workspace, so no CTA waits for one that has
 * not started) and stream their first weight tiles meanwhile. It measured
 * slower on B200 (its claim/publish/poll chain costs more than the second
 * launch), so it runs only when the environment variable QOQ_FORCE_CONFIG
 * holds fuse=1; qoq_plan reports which form a problem gets. Either way the
 * codes, scales and row sums are written into the workspace, after the
 * GEMM's scratch.
 *
 * X_fp16 [M][K] FP16, read; Y_fp16 [M][N] FP16, written; blob as for
 * qoq_gemm_fp16_out. The workspace must be 256-byte aligned, zero-filled by
 * the caller before its first use, and of the size the query
 * (workspace == NULL) reports for this (M, N, K, group_size); its control
 * words and status word behave as for qoq_w4a8_gemm (the claim counters
 * are control words too, left zero by every call that completes).
 */
qoq_status qoq_w4a8_linear(const void *X_fp16, const void *blob, int64_t M, int64_t N, int64_t K,
                           int group_size, void *Y_fp16, void *workspace, size_t *workspace_bytes,
                           void *stream);

/*
 * Ablation of the protective range: qoq_gemm_fp16_out with a weight decode
 * that saturates every dequantised byte to [-128, 127], as a kernel must when
 * dequantised weights can leave the INT8 range. (paperlayer.ai summary,
 * section 4 "Progressive Group Quantization": the range is shrunk to
 * [-119, 119] so that the intermediate weights never overflow INT8, because
 * saturation would otherwise cost up to 67% of the GEMM's throughput.)
 *
 * With blobs from qoq_quantize_weights (protective range) the saturation
 * never acts, so the result is bit-identical to qoq_gemm_fp16_out; the call
 * exists to measure what the saturating decode costs on this GPU. Arguments,
 * workspace and status word as for qoq_gemm_fp16_out. Built for
 * group_size 128 and two token tiles: M <= 16 (decode) and M > 512 on CTA
 * pairs (N / 128 even); other sizes return QOQ_ERR_UNSUPPORTED without a
 * launch.
 */
qoq_status qoq_gemm_fp16_out_saturating(const int8_t *X8, const void *s_x_fp16, const void *blob, int64_t M,
                                        int64_t N, int64_t K, int group_size, void *Y_fp16, void *workspace,
                                        size_t *workspace_bytes, void *stream);

/*
 * W4A8 GEMM with the fused FP16 epilogue, for callers that cannot allocate
 * device memory (a pre-planned memory arena, a thread that must not touch the
 * device allocator while other work owns it, a runtime that forbids cudaMalloc
 * after start-up). The QServe pages have no counterpart: it exists only so the
 * workspace of qoq_gemm_fp16_out need not be allocated by the caller.
 *
 * Same computation and arguments as qoq_gemm_fp16_out, except that the
 * stream-K scratch lives in one fixed 8 MiB device array inside the library,
 * which every GPU that loads the library keeps until the process exits. That
 * bounds the problem: the call needs 1280 + C * T * 512 bytes (one INT32
 * partial-sum tile of T x 128 per CTA), where T is the token tile the library
 * picks for (M, N, K) and C the CTAs of the launch (min(SM count, token
 * tiles * N/128 * K/128); twice the CTA pairs for 256-token tiles). On a
 * 148-SM B200 every problem whose token tile is at most 64 fits (4.9 MB at
 * most): all M <= 64, and M up to 256 where few weight tiles make the library
 * keep 64-token tiles (e.g. N = K = 4096). Larger problems return
 * QOQ_ERR_WORKSPACE and launch nothing.
 *
 * status: optional device int32; when non-NULL the call copies the device
 * status word of this call (0, QOQ_ERR_BAD_BLOB or QOQ_ERR_TIMEOUT) into it
 * on the same stream.
 *
 * The library neither allocates nor frees anything in this call: it clears the
 * array's control words (cudaMemsetAsync), launches the GEMM and, if asked,
 * copies the status word. The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current, so make the
 * first call on a device before any stream capture. All calls share the one
 * array, which keeps the last call's contents: calls that may overlap on the
 * device (different streams, or different host threads) race on it and must
 * be serialised by the caller.
 */
qoq_status qoq_gemm_fp16_out_static_ws(const int8_t *X8, const void *s_x_fp16, const int32_t *rowsum,
                                       const void *blob, int64_t M, int64_t N, int64_t K, int group_size,
                                       void *Y_fp16, int32_t *status, void *stream);

/*
 * Self-test of the device-side bounded waits (failure detection without a
 * fault; the paper has no counterpart). One small kernel waits, each for at
 * most limit_ns nanoseconds (1 .. 2e9), on an mbarrier phase that never
 * completes and on a global flag that nothing sets; each wait must give up,
 * record its failure and return. The kernel then exits normally and the
 * context stays usable.
 *
 * status: device int32[32], 16-byte aligned, owned by the caller; zeroed by
 * the call (on `stream`). After the stream completes: status[0..3] =
 * {QOQ_ERR_TIMEOUT, wait site 4, block 0, detail 1} for the mbarrier wait and
 * status[8..11] = {QOQ_ERR_TIMEOUT, wait site 6, block 0, detail 2} for the
 * flag wait (sites as in the GEMM workspace status words).
 * Returns QOQ_ERR_INVALID_ARG / QOQ_ERR_ALIGNMENT before any launch,
 * QOQ_ERR_CUDA if the launch fails.
 */
qoq_status qoq_watchdog_selftest(int32_t *status, int64_t limit_ns, void *stream);

/*
 * KV4 cache: per-head, dynamic, asymmetric 4-bit keys and values.
 * (paperlayer.ai summary, section 5 "QServe Serving System", "KV4 attention":
 *  per-head dynamic KV4 scales and zero points, attention arithmetic on CUDA
 *  cores; section 6 "Evaluation", "Experimental setup": per-head asymmetric
 *  INT4 KV caches.)
 *
 * Every vector of D values (one sequence, one KV head, one token) gets its own
 * FP16 scale s and zero z, computed when the token is written (nothing is
 * calibrated), with the per-channel weight quantiser's arithmetic:
 *   lo = min(0, min x), hi = max(0, max x), s = FP16((hi - lo) / 15),
 *   z = RNE(-lo / s) (an integer 0..15, stored exactly in FP16),
 *   q = clamp(RNE(x / s) + z, 0, 15); s == 0 gives q = z = 0.
 * Each FP32 step is one correctly rounded operation.
 *
 * Cache layout (caller-owned device memory, max_tokens slots per sequence):
 *   codes  uint8 [B][Hkv][max_tokens][D/2], byte j = q[2j] | q[2j+1] << 4
 *   scales FP16  [B][Hkv][max_tokens]
 *   zeros  FP16  [B][Hkv][max_tokens]
 *
 * qoq_kv4_cache_write quantises src FP16 [B][Hkv][n_tokens][D] (row-major,
 * 16-byte aligned) into slots t0 .. t0 + n_tokens - 1 of every (sequence, KV
 * head): the whole cache at once (t0 = 0) or the decode step's new token
 * (n_tokens = 1). D must be 64 or 128, t0 + n_tokens <= max_tokens, codes
 * 16-byte aligned, scales and zeros 2-byte aligned (else QOQ_ERR_UNSUPPORTED /
 * QOQ_ERR_INVALID_ARG / QOQ_ERR_ALIGNMENT before any launch). n_tokens == 0
 * or B == 0 is a no-op.
 */
qoq_status qoq_kv4_cache_write(const void *src_fp16, int64_t B, int64_t Hkv, int64_t max_tokens, int64_t t0,
                               int64_t n_tokens, int64_t D, uint8_t *codes, void *scales_fp16,
                               void *zeros_fp16, void *stream);

/*
 * KV4 decode attention: one query token per sequence against its KV4 cache,
 * grouped-query (query head hq reads KV head hq / (Hq / Hkv)).
 * (paperlayer.ai summary, section 5, "KV4 attention"; section 6, "Ablation
 *  and breakdown": the attention kernel at batch 64 x 1024 tokens.)
 *
 *   k_t, v_t = (q_t - z_t) * s_t            (dequantised key / value, t < T_b)
 *   score_t = (q . k_t) / sqrt(D);  p = softmax_t(score);  out = sum_t p_t v_t
 *
 * The products run on tensor cores with FP16 inputs and FP32 accumulation:
 * the 4-bit codes enter them exactly (as FP16 values c * 2^-24 and c * 2^-20),
 * the zero points are subtracted in FP32 (z * sum(q) from each score,
 * z * (P s) from each output), the softmax weights times the value scale are
 * rounded to FP16 for the second product, and the output is rounded once to
 * FP16. The order of the sums is the kernel's (64-token tiles per warp,
 * spans of 256 * t tokens per CTA, combined with the usual running-maximum
 * rescaling), so results are compared with the exact mathematics under a
 * tolerance (|o - o*| <= 2^-10 max|v| + 2^-24 per head), not bit for bit.
 *
 * q_fp16 [B][Hq][D] FP16; the K and V caches as written by
 * qoq_kv4_cache_write (same B, Hkv, max_tokens, D); seq_lens int32 [B] with
 * 1 <= T_b <= max_tokens, or NULL for T_b = max_tokens; out_fp16 [B][Hq][D]
 * FP16, written. Hq must be a multiple of Hkv with Hq / Hkv <= 8, D 64 or 128.
 *
 * Workspace: device memory of *workspace_bytes bytes (size query with
 * workspace == NULL; 256-byte aligned), zero-filled by the caller before its
 * first use. Bytes [0, 256) are the status words: int32 [0] stays 0, or
 * becomes QOQ_ERR_TIMEOUT with [1] = 10 (a warp's wait for its K/V code copy
 * ran out after 1 s), [2] = the CTA's x index, [3] = 2 * tile + (0 for K,
 * 1 for V); the caller clears it. Then 4 * B * Hkv bytes of per-(sequence,
 * head) counters that every call which completes leaves zero; the rest is
 * scratch for the CTAs' partial results. Calls that may overlap on the
 * device need separate workspaces. A seq_lens entry outside [1, max_tokens]
 * is clamped into it.
 */
qoq_status qoq_kv4_decode_attention(const void *q_fp16, const uint8_t *k_codes, const void *k_scales,
                                    const void *k_zeros, const uint8_t *v_codes, const void *v_scales,
                                    const void *v_zeros, const int32_t *seq_lens, int64_t B, int64_t Hq,
                                    int64_t Hkv, int64_t max_tokens, int64_t D, void *out_fp16, void *workspace,
                                    size_t *workspace_bytes, void *stream);

/*
 * Launch plan of a problem (no device work; the library has no counterpart
 * in the QServe pages): the token tile (MMA N: 16, 32, 64, 128 or 256) the
 * GEMM calls use for (M, N, K), and how many kernels qoq_w4a8_linear
 * launches for it (2, or 1 when the one-launch form is selected by
 * QOQ_FORCE_CONFIG=fuse=1 and the token tile is at most 64). Either
 * output pointer may be NULL. Returns QOQ_ERR_INVALID_ARG / _UNSUPPORTED for
 * shapes the GEMM calls reject.
 */
qoq_status qoq_plan(int64_t M, int64_t N, int64_t K, int32_t *token_tile, int32_t *linear_launches);

/* Name of a status code (static string, never NULL). */
const char *qoq_status_string(qoq_status status);

#ifdef __cplusplus
}
#endif

#endif /* QOQ_H */
