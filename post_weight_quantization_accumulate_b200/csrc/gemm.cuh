// gemm.cuh -- fp32 matrix products used inside the factorisation and the
// lazy-batch update.
#pragma once
#include "common.cuh"

namespace gptq {

enum GemmFlags : int {
    kGemmLowerA = 1,  // A is lower triangular: only k <= m contributes
    kGemmLowerB = 2,  // B is lower triangular: only k >= n contributes
    kGemmLowerC = 4,  // only the lower triangle (col <= row) of C is written
};

// C = alpha * A * B + beta * C (row-major; beta == 0 ignores C's contents).
// trans_b: B is stored as [N, K] (ldb) instead of [K, N].
// batch > 1: blockIdx.z selects A + z*sA, B + z*sB, C + z*sC.
int launch_sgemm(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                 int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                 int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream);

}  // namespace gptq
