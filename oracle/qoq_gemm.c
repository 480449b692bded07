/*
 * CPU reference integer GEMM for the QoQ W4A8 path -- TEST INFRASTRUCTURE.
 * Only the tests, the smoke check and the benchmark's CPU-baseline arm call it.
 *
 * QServe keeps every W4A8 GEMM on INT8 tensor cores with exact integer
 * accumulation (QServe: W4A8KV4 Quantization and System Co-design for
 * Efficient LLM Serving -- paperlayer.ai summary, section 8 "Conclusion";
 * study.space summary).  The exact result is therefore the definition
 *     acc[m][n] = sum_k X8[m][k] * Wint[n][k]
 * written out as a plain triple loop in 64-bit integers: no blocking, no
 * reordering, no vectorisation hints.
 *
 * X8:   int8 [M][K] row-major.  Wint: int8 [N][K] row-major (the dequantised
 * weights).  acc: int64 [M][N] row-major, written by this call.
 * Returns the largest |acc| seen so the caller can assert it fits int32.
 *
 * The output elements are independent exact integer sums, so they are shared
 * out over the host's cores (OpenMP, when built with it); each sum is still
 * the same plain loop over k, and the result does not depend on the split.
 */
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the GEMM below uses (1 without OpenMP). */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

int64_t oracle_gemm_s8s8_i64(const int8_t *X8, const int8_t *Wint, int64_t *acc,
                             int64_t M, int64_t N, int64_t K)
{
    int64_t amax = 0;
#ifdef _OPENMP
#pragma omp parallel for collapse(2) reduction(max : amax) schedule(static)
#endif
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k)
                sum += (int64_t)X8[m * K + k] * (int64_t)Wint[n * K + k];
            acc[m * N + n] = sum;
            int64_t a = sum < 0 ? -sum : sum;
            if (a > amax) amax = a;
        }
    }
    return amax;
}
