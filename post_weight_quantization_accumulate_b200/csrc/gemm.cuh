// gemm.cuh -- fp32 matrix products used inside the factorisation and the
// lazy-batch update.
#pragma once
#include "common.cuh"

namespace gptq {

enum GemmFlags : int {
    kGemmLowerA = 1,  // A is lower triangular: only k <= m contributes
    kGemmLowerB = 2,  // B is lower triangular: only k >= n contributes
    kGemmLowerC = 4,  // only the lower triangle (col <= row) of C is needed: tiles above
                      // the diagonal are skipped, entries above it inside diagonal
                      // tiles may be updated too
};

// C = alpha * A * B + beta * C (row-major; beta == 0 ignores C's contents).
// trans_b: B is stored as [N, K] (ldb) instead of [K, N].
// batch > 1: matrix z of the batch is A + z*sA, B + z*sB, C + z*sC.
// Runs on the tensor cores (3xTF32, gemm_tc.cu) whenever A and B are 16-byte
// aligned with leading dimensions and batch strides that are multiples of 4
// floats (the TMA rules), else on the SIMT kernel (gemm_simt.cu).
// max_ctas > 0 caps the number of CTAs (and so of SMs) the product occupies,
// which leaves SMs free for latency-critical work on another stream.
// max_ctas < 0: one CTA per output tile (tensor-core path) instead of at most
// one per SM looping over tiles, so the product's CTAs retire tile by tile
// and work of higher-priority streams gets SMs as they free up.
// A_lo, B_lo (optional, same layout and strides as A and B): the operands'
// low parts x - trunc_tf32(x), prepared by the caller; with both given the
// tensor-core path skips its conversion pass and uses 128 x 256 tiles.
// pdl: launch the tensor-core product as a programmatic dependent launch (its
// prologue overlaps the previous kernel on the stream; see launch_k).
// stamp (optional, device, two words preset to ~0 and 0): the tensor-core
// product records its span there, atomicMin of the time its first CTA passes
// the dependency wait and atomicMax of the time its last CTA ends
// (globaltimer, ns).  The SIMT path records nothing.
int launch_sgemm(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                 int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                 int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream,
                 int max_ctas = 0, const float* A_lo = nullptr, const float* B_lo = nullptr,
                 bool pdl = false, unsigned long long* stamp = nullptr);

int launch_sgemm_simt(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                      int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                      int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream);
int launch_gemm_tc(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                   int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                   int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream,
                   int max_ctas = 0, const float* A_lo = nullptr, const float* B_lo = nullptr,
                   bool pdl = false, unsigned long long* stamp = nullptr);
bool gemm_tc_supported(const float* A, int64_t lda, int64_t sA, const float* B, int64_t ldb,
                       int64_t sB, int batch);

}  // namespace gptq
