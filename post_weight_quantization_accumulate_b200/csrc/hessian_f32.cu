// hessian_f32.cu -- H += 2 X^T X for float32 activations on the bf16 tensor-core
// Hessian (GPTQ overview, "Złożoność obliczeniowa": H = 2 X X^T).
//
// Each value splits into two bf16 parts, x = hi + lo + r with hi = bf16(x),
// lo = bf16(x - hi) and |r| <= 2^-18 |x| (x - hi is exact in fp32).  With the
// parts side by side, Z = [hi | lo] (n x 2d), the bf16 kernel computes
//   2 Z^T Z = [[A11, A12], [A12^T, A22]],  A11 = 2 hi^T hi, A12 = 2 hi^T lo, ...
// from exact bf16 products with fp32 sums, and
//   2 X^T X = A11 + (A12 + A12^T) + A22 + O(2^-17) relative per product.
// The cross blocks are added to each other first, so the folded H stays
// bitwise symmetric.  The token stream is processed in chunks through a
// caller-owned workspace: [2d x 2d] fp32 block Hessian, then Z of one chunk.
#include "common.cuh"

#include <cuda_bf16.h>

namespace gptq {

int launch_hessian_upper(float* H, const uint16_t* X, int64_t n_rows, int64_t d, cudaStream_t s);
int launch_mirror(float* H, int64_t d, cudaStream_t s);

namespace {

// Z[t][k] = bf16(x), Z[t][d + k] = bf16(x - bf16(x)) for rows [0, rows), four
// columns per thread.
__global__ void split_bf16_pair_kernel(const float* __restrict__ X, uint16_t* __restrict__ Z,
                                       int64_t rows, int64_t d)
{
    const int64_t q = d / 4;
    const int64_t total = rows * q;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = i / q, k = 4 * (i % q);
        const float4 v = *reinterpret_cast<const float4*>(X + t * d + k);
        const float x[4] = {v.x, v.y, v.z, v.w};
        uint16_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat16 h = __float2bfloat16_rn(x[e]);
            const __nv_bfloat16 l = __float2bfloat16_rn(x[e] - __bfloat162float(h));
            hi[e] = __bfloat16_as_ushort(h);
            lo[e] = __bfloat16_as_ushort(l);
        }
        uint16_t* zr = Z + t * 2 * d;
        *reinterpret_cast<uint2*>(zr + k) =
            make_uint2(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16));
        *reinterpret_cast<uint2*>(zr + d + k) =
            make_uint2(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16));
    }
}

// H[i][j] += (A11[i][j] + (A12[i][j] + A12[j][i])) + A22[i][j] from the full
// symmetric block Hessian H2 [2d][2d].
__global__ void fold_blocks_kernel(float* __restrict__ H, const float* __restrict__ H2, int64_t d)
{
    const int64_t total = d * d;
    const int64_t ld = 2 * d;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / d, j = e % d;
        const float a11 = H2[i * ld + j];
        const float a12 = H2[i * ld + d + j];
        const float a21 = H2[j * ld + d + i];
        const float a22 = H2[(d + i) * ld + d + j];
        H[e] += (a11 + (a12 + a21)) + a22;
    }
}

}  // namespace

size_t hessian_f32_workspace_bytes(int64_t d, int64_t chunk)
{
    const size_t h2 = static_cast<size_t>(2 * d) * static_cast<size_t>(2 * d) * sizeof(float);
    const size_t z = static_cast<size_t>(chunk) * static_cast<size_t>(2 * d) * sizeof(uint16_t);
    return ((h2 + 255) / 256) * 256 + z;
}

int run_hessian_f32(float* H, const float* X, int64_t n, int64_t d, int64_t chunk, void* ws,
                    cudaStream_t s)
{
    const size_t h2_bytes = static_cast<size_t>(2 * d) * static_cast<size_t>(2 * d) * sizeof(float);
    float* H2 = static_cast<float*>(ws);
    uint16_t* Z = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + ((h2_bytes + 255) / 256) * 256);
    GPTQ_CUDA_CHECK(cudaMemsetAsync(H2, 0, h2_bytes, s));
    const int grid_cap = sm_count() * 8;
    for (int64_t t = 0; t < n; t += chunk) {
        const int64_t rows = n - t < chunk ? n - t : chunk;
        const int64_t items = rows * (d / 4);
        const int blocks = static_cast<int>(std::min<int64_t>((items + 255) / 256, grid_cap));
        split_bf16_pair_kernel<<<blocks, 256, 0, s>>>(X + t * d, Z, rows, d);
        GPTQ_LAUNCH_CHECK();
        int rc = launch_hessian_upper(H2, Z, rows, 2 * d, s);
        if (rc) return rc;
    }
    int rc = launch_mirror(H2, 2 * d, s);
    if (rc) return rc;
    const int blocks = static_cast<int>(std::min<int64_t>((d * d + 255) / 256, grid_cap));
    fold_blocks_kernel<<<blocks, 256, 0, s>>>(H, H2, d);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

}  // namespace gptq
