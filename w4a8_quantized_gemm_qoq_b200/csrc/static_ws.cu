// qoq_gemm_fp16_out_static_ws: the W4A8 GEMM with fused FP16 epilogue for
// callers that cannot allocate device memory -- for example code running
// inside a pre-planned memory arena, a host thread that must not call into
// the allocator while a CUDA graph or another library owns the device heap,
// or an embedding runtime that forbids cudaMalloc after start-up. Instead of
// a caller-supplied workspace, the stream-K scratch (status word, arrival
// counters and partial tiles) lives in one file-scope device array of a fixed
// size that every GPU which loads the library keeps until the process exits.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>

#include "qoq_internal.h"

namespace {

// 8 MiB: the control words plus one INT32 partial tile per CTA for token
// tiles of up to 64 tokens: 1280 + 148 * 64 * 512 bytes (4.85 MB) on a 148-SM
// B200.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch, looked up once per device with that
// device current. In host code the symbol itself is only a stand-in, never a
// device pointer.
std::mutex g_mu;
void *g_scratch_ptr[64];

qoq_status static_scratch_address(int dev, void **out) {
    if (dev < 0 || dev >= 64) return QOQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return QOQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return QOQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" qoq_status qoq_gemm_fp16_out_static_ws(const int8_t *X8, const void *s_x_fp16, const int32_t *rowsum,
                                                  const void *blob, int64_t M, int64_t N, int64_t K,
                                                  int group_size, void *Y_fp16, int32_t *status, void *stream) {
    using namespace qoq;
    if (M < 0 || M > INT32_MAX || N <= 0 || K <= 0) return QOQ_ERR_INVALID_ARG;
    if (N % kTileN != 0 || K % kTileK != 0 || K > kMaxK || N > (int64_t)INT32_MAX / 2) return QOQ_ERR_UNSUPPORTED;
    if (group_size != kGroup && group_size != 0) return QOQ_ERR_INVALID_ARG;
    if (M == 0) return QOQ_OK;
    if (X8 == nullptr || s_x_fp16 == nullptr || blob == nullptr || Y_fp16 == nullptr) return QOQ_ERR_INVALID_ARG;
    if (group_size == 0 && rowsum == nullptr) return QOQ_ERR_INVALID_ARG;
    if (!aligned16(X8) || !aligned16(blob) || !aligned16(Y_fp16)) return QOQ_ERR_ALIGNMENT;
    if ((reinterpret_cast<uintptr_t>(s_x_fp16) & 1u) || (reinterpret_cast<uintptr_t>(rowsum) & 3u) ||
        (reinterpret_cast<uintptr_t>(status) & 3u))
        return QOQ_ERR_ALIGNMENT;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
    // Scratch this call needs: the control words plus one partial tile per
    // CTA of the grid the launch will use (the launcher's own rule, which
    // checks the same bound again before it launches).
    const size_t need = gemm_scratch_bytes(M, N, K, group_size);
    if (need == 0) return QOQ_ERR_CUDA;
    if (need > kStaticScratchBytes) return QOQ_ERR_WORKSPACE;

    void *scratch = nullptr;
    qoq_status st = static_scratch_address(dev, &scratch);
    if (st != QOQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps whatever the previous call left (after an error, not
    // necessarily zeros); the control words and the partial-sum buffers this
    // call uses must start at zero.
    if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return QOQ_ERR_CUDA;

    GemmArgs a;
    a.X8 = X8;
    a.s_x = s_x_fp16;
    a.rowsum = rowsum;
    a.blob = blob;
    a.M = M;
    a.N = N;
    a.K = K;
    a.group = group_size;
    a.out = Y_fp16;
    a.fp16_out = true;
    a.ws = scratch;
    a.ws_capacity = kStaticScratchBytes;
    st = launch_gemm(a, s);
    if (st != QOQ_OK) return st;
    if (status != nullptr &&
        cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return QOQ_ERR_CUDA;
    return QOQ_OK;
}
