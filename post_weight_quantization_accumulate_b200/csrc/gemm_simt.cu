// gemm_simt.cu -- fp32 SIMT matrix product with triangular-structure flags.
// 128 x 128 output tile per CTA, K slices of 16 double-buffered through
// shared memory, 8 x 8 outputs per thread.
#include "gemm.cuh"

namespace gptq {
namespace {

constexpr int BM = 128, BN = 128, BK = 16, PAD = 4;

template <bool TRANS_B>
__global__ void __launch_bounds__(256)
    sgemm_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, int64_t lda,
                 int64_t sA, const float* __restrict__ B, int64_t ldb, int64_t sB, float beta,
                 float* __restrict__ C, int64_t ldc, int64_t sC, int flags)
{
    __shared__ __align__(16) float As[2][BK][BM + PAD];
    __shared__ __align__(16) float Bs[2][BK][BN + PAD];
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    if ((flags & kGemmLowerC) && n0 > m0 + BM - 1) return;
    A += blockIdx.z * sA;
    B += blockIdx.z * sB;
    C += blockIdx.z * sC;
    int kbeg = 0, kend = K;
    if (flags & kGemmLowerB) kbeg = (n0 / BK) * BK;
    if (flags & kGemmLowerA) kend = min(K, m0 + BM);
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;

    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

    float ra[8], rb[8];
    // A tile: thread -> row tid/2, k (tid%2)*8 .. +7
    const int a_row = tid >> 1, a_k = (tid & 1) * 8;
    // B tile (K x N): k = tid/16, n = (tid%16)*8 .. +7 ; (N x K stored): n = tid/2, k = (tid%2)*8
    auto load = [&](int k0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = m0 + a_row, k = k0 + a_k + i;
            ra[i] = (r < M && k < kend) ? A[static_cast<int64_t>(r) * lda + k] : 0.f;
        }
        if (!TRANS_B) {
            const int k = k0 + (tid >> 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int n = n0 + (tid & 15) * 8 + i;
                rb[i] = (k < kend && n < N) ? B[static_cast<int64_t>(k) * ldb + n] : 0.f;
            }
        } else {
            const int n = n0 + (tid >> 1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int k = k0 + (tid & 1) * 8 + i;
                rb[i] = (k < kend && n < N) ? B[static_cast<int64_t>(n) * ldb + k] : 0.f;
            }
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 8; ++i) As[buf][a_k + i][a_row] = ra[i];
        if (!TRANS_B) {
#pragma unroll
            for (int i = 0; i < 8; ++i) Bs[buf][tid >> 4][(tid & 15) * 8 + i] = rb[i];
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) Bs[buf][(tid & 1) * 8 + i][tid >> 1] = rb[i];
        }
    };

    if (kbeg < kend) {
        load(kbeg);
        store(0);
        __syncthreads();
        int buf = 0;
        for (int k0 = kbeg; k0 < kend; k0 += BK) {
            const bool more = k0 + BK < kend;
            if (more) load(k0 + BK);
#pragma unroll
            for (int k = 0; k < BK; ++k) {
                const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
                const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4 + 64]);
                const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
                const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4 + 64]);
                const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
            if (more) store(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = m0 + ty * 4 + (i & 3) + (i >> 2) * 64;
        if (r >= M) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = n0 + tx * 4 + (j & 3) + (j >> 2) * 64;
            if (c >= N) continue;
            if ((flags & kGemmLowerC) && c > r) continue;
            float* p = C + static_cast<int64_t>(r) * ldc + c;
            const float v = alpha * acc[i][j];
            *p = (beta == 0.f) ? v : fmaf(beta, *p, v);
        }
    }
}

}  // namespace

int launch_sgemm(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                 int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                 int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream, int max_ctas,
                 const float* A_lo, const float* B_lo, bool pdl, unsigned long long* stamp)
{
    if (gemm_tc_supported(A, lda, sA, B, ldb, sB, batch)) {
        // the low parts are used only when they obey the same TMA rules
        const bool lo_ok = A_lo && B_lo && gemm_tc_supported(A_lo, lda, sA, B_lo, ldb, sB, batch);
        return launch_gemm_tc(trans_b, M, N, K, alpha, A, lda, sA, B, ldb, sB, beta, C, ldc, sC,
                              batch, flags, stream, max_ctas, lo_ok ? A_lo : nullptr,
                              lo_ok ? B_lo : nullptr, pdl, stamp);
    }
    // the SIMT kernel is launched plainly (it waits for the previous kernel)
    return launch_sgemm_simt(trans_b, M, N, K, alpha, A, lda, sA, B, ldb, sB, beta, C, ldc, sC,
                             batch, flags, stream);
}

int launch_sgemm_simt(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                      int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                      int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream)
{
    if (M <= 0 || N <= 0 || batch <= 0) return GPTQ_OK;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, batch);
    if (trans_b)
        sgemm_kernel<true><<<grid, 256, 0, stream>>>(M, N, K, alpha, A, lda, sA, B, ldb, sB, beta,
                                                     C, ldc, sC, flags);
    else
        sgemm_kernel<false><<<grid, 256, 0, stream>>>(M, N, K, alpha, A, lda, sA, B, ldb, sB,
                                                      beta, C, ldc, sC, flags);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

}  // namespace gptq
