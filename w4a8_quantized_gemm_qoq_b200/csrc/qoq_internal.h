// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qoq.h"

namespace qoq {

constexpr int kTileN = 128;        // weight rows per tile (TMEM lanes)
constexpr int kTileK = 128;        // K per tile = one quantisation group
constexpr int kGroup = 128;
constexpr int kMaxK = 65536;
constexpr int kMaxGrid = 256;      // upper bound of the persistent grid (>= SM count)
constexpr int kTileGroup = 8;      // token tiles per group of the GEMM's tile order

// Programmatic dependent launch (griddepcontrol) between the activation
// quantiser and the GEMM: each kernel releases its successor right after its
// own set-up, and touches what a predecessor may write only after
// griddepcontrol.wait; the GEMM issues its first weight copies before that
// wait. Kernels of other libraries in the stream are unaffected: a launch
// without the attribute, or after a kernel that never releases early, waits
// for full completion as usual.
constexpr bool kProgrammaticLaunch = true;
constexpr uint32_t kMagic = 0x57514F51u;   // 'Q','O','Q','W'
constexpr uint32_t kVersion = 1u;
constexpr int kHeaderBytes = 256;

// Byte layout of a packed weight blob.
struct BlobLayout {
    int64_t NT, KT;
    int64_t block;      // bytes per (n-tile, k-tile) block
    int64_t off_codes, off_scale, off_zero, total;
};

inline int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

inline BlobLayout blob_layout(int64_t N, int64_t K, int group) {
    BlobLayout L;
    L.NT = N / kTileN;
    L.KT = K / kTileK;
    L.block = 8192 + (group ? 256 : 0);
    L.off_codes = kHeaderBytes;
    L.off_scale = L.off_codes + L.NT * L.KT * L.block;
    if (group) {
        L.off_zero = 0;
        L.total = L.off_scale + align256(2 * N);
    } else {
        L.off_zero = L.off_scale + align256(2 * N);
        L.total = L.off_zero + align256(2 * N);
    }
    return L;
}

// Overrides of the launch heuristics from the QOQ_FORCE_CONFIG environment
// variable (config.cu); 0 = not forced.
struct ForcedConfig {
    int tok = 0;   // token tile
    int cps = 0;   // CTAs per SM of the decode kernel
    int fuse = 0;  // qoq_w4a8_linear at token tiles <= 64: 1 = separate quantiser, 2 = fused launch
    int kvt = 0;   // KV4 attention: 64-token tiles per warp
    int aqt = 0;   // activation quantiser: threads per CTA (one row per CTA)
    int aq2 = 0;   // activation quantiser: 1 = the two-pass form, 2 = the register form
    int lateck = 0;   // GEMM kernels: contributors' arrivals delayed by this many us (tests)
    int prs = 0;   // RMSNorm producer, warp rows: 1 = row kept in registers, 2 = formed twice, 3 = staged in smem
    int pst = 0;   // SiLU-gated producer, rows above 8192: 1 = narrower CTA shape, 2 = wider
};

// Whether qoq_w4a8_linear quantises the activations inside the decode GEMM's
// launch for a problem whose token tile is at most 64.
bool linear_fused(int64_t M, int64_t N, int64_t K);
const ForcedConfig &forced_config();

// Token-tile width (MMA N) for an M x N x K problem. Small M uses the
// smallest tile that holds all tokens. Beyond that the choice trades weight
// re-reads and dequantisation (once per token tile) against enough work units
// for every SM and the stream-K partial-sum traffic; the thresholds below come
// from B200 measurements on Llama-3-8B and Qwen1.5-72B linear shapes. Long K
// prefers the widest tile, whose tensor work per k-tile hides the dequant.
inline int token_tile_for(int64_t M, int64_t N, int64_t K) {
    const int64_t NT = N / kTileN, KT = K / kTileK;
    auto blocks = [&](int64_t tok) { return ((M + tok - 1) / tok) * NT * KT; };
    if (forced_config().tok) return forced_config().tok;
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return blocks(64) >= 2500 ? 64 : 32;
    if (M <= 128) return blocks(128) >= 6000 ? 128 : 64;
    if (M <= 256) return blocks(128) >= 10000 ? 128 : 64;
    if (M <= 512) return KT >= 128 ? 256 : 128;
    return 256;
}

// Workspace: [0, 256) status word + reserved; then int32 arrival counters
// [kMaxGrid], one per split tile (together QOQ_WORKSPACE_CONTROL_BYTES, left
// zero by every call); then int32 partial tiles (scratch, `slots` per CTA).
static_assert(256 + 4 * kMaxGrid == QOQ_WORKSPACE_CONTROL_BYTES, "workspace control layout");

// Workspace bytes a launch of `grid_ctas` CTAs with token tile `tok` uses:
// the control words, then `slots` INT32 partial tiles per CTA. The general kernel
// (token tiles of 128 and 256) uses them as scratch; the decode kernel (token
// tiles up to 64) as the sum buffers of its split tiles, which must be zero
// when a launch starts and which every launch that completes leaves zero.
constexpr int kDecodeMaxTok = 64;
// slots: partial-sum tiles per CTA (the decode kernel 1; the general kernel 2,
// one for the tile it contributes to and one for the tile it owns, which a
// CTA can hold at the same time when it is not the last to arrive at either).
inline size_t scratch_bytes_for_grid(int tok, int64_t grid_ctas, int slots) {
    return QOQ_WORKSPACE_CONTROL_BYTES + sizeof(int32_t) * (size_t)slots * grid_ctas * tok * kTileN;
}

// CTAs per SM of the decode kernel for a problem: one (the whole SM, deepest
// weight ring) or two (half an SM, so that consecutive launches overlap).
int decode_ctas_per_sm(int64_t M, int64_t N, int64_t K);

// Workspace size the size query reports: enough for any grid (kMaxGrid CTAs).
inline size_t workspace_bytes_for(int64_t M, int64_t N, int64_t K) {
    return scratch_bytes_for_grid(token_tile_for(M, N, K), kMaxGrid, 2);
}

// qoq_w4a8_linear keeps the quantised activations in the workspace, after
// the GEMM's scratch: codes [M][K], FP16 scales [M], row sums [M].
struct FusedLayout {
    size_t off_x8, off_sx, off_rowsum, total;
};
inline FusedLayout fused_layout(int64_t M, int64_t K, size_t base) {
    FusedLayout F;
    F.off_x8 = (size_t)align256((int64_t)base);
    F.off_sx = (size_t)align256((int64_t)(F.off_x8 + (size_t)M * K));
    F.off_rowsum = (size_t)align256((int64_t)(F.off_sx + 2 * (size_t)M));
    F.total = F.off_rowsum + 4 * (size_t)M;
    return F;
}
inline size_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    return fused_layout(M, K, workspace_bytes_for(M, N, K)).total;
}

// Kernel launchers (return cudaSuccess or the launch error).
cudaError_t launch_act_quant(const void *X, int64_t M, int64_t K, int8_t *X8, void *s_x, int32_t *rowsum,
                             cudaStream_t stream);
cudaError_t launch_weight_quant(const void *W, int64_t N, int64_t K, int group, void *blob,
                                const BlobLayout &L, cudaStream_t stream);
cudaError_t launch_rmsnorm_quant(const void *X, const void *gamma, int64_t M, int64_t K, float eps, int8_t *X8,
                                 void *s_x, int32_t *rowsum, cudaStream_t stream);
cudaError_t launch_silu_mul_quant(const void *GU, int64_t M, int64_t I, int8_t *X8, void *s_x, int32_t *rowsum,
                                  cudaStream_t stream);

// KV4 cache and decode attention (kv4_attention.cu).
cudaError_t launch_kv4_cache_write(const void *src, int64_t B, int64_t Hkv, int64_t Tmax, int64_t t0, int64_t nt,
                                   int64_t D, uint8_t *codes, void *scales, void *zeros, cudaStream_t stream);
size_t kv4_workspace_bytes(int64_t B, int64_t Hkv, int64_t Tmax, int64_t D);
cudaError_t launch_kv4_attention(const void *q, const uint8_t *kc, const void *ks, const void *kz, const uint8_t *vc,
                                 const void *vs, const void *vz, const int32_t *seq_lens, int64_t B, int64_t Hq,
                                 int64_t Hkv, int64_t Tmax, int64_t D, void *out, void *ws, cudaStream_t stream);

// Row width limit of the fused producers (the row lives in registers: at most
// 8 chunks of 8 elements per thread of a 512-thread row, or 4 of a 1024-thread row).
constexpr int kMaxProducerWidth = 32768;

struct GemmArgs {
    const void *X = nullptr;   // FP16 activations: quantised in the same launch (decode kernel), else null
    const int8_t *X8;
    const void *s_x;
    const int32_t *rowsum;
    const void *blob;
    int64_t M, N, K;
    int group;
    void *out;          // int32 [M][N] or fp16 [M][N]
    bool fp16_out;
    void *ws;
    // Ablation only (qoq_gemm_fp16_out_saturating): decode the weights with
    // per-byte saturation to [-128, 127], as a kernel without the protective
    // range would have to.
    bool saturating = false;
    // Bytes of `ws` the caller provides; a launch whose grid would need more
    // returns QOQ_ERR_WORKSPACE without launching.
    size_t ws_capacity = 0;
};
qoq_status launch_gemm(const GemmArgs &a, cudaStream_t stream);

// Workspace bytes the launch for this problem on the current device will
// actually use (its grid, not the kMaxGrid bound): the same grid rule as
// launch_gemm. Returns 0 if the device cannot be queried.
size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K, int group, bool saturating = false);

// The decode-regime kernel (token tiles 16, 32, 64; gemm_decode.cu). With
// a.X set it quantises the activations itself (into the workspace).
qoq_status launch_decode_gemm(const GemmArgs &a, cudaStream_t stream, int tok, int units_max);

}  // namespace qoq
