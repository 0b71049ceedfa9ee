// quantize.cu -- the GPTQ column loop with per-group asymmetric quantization,
// OBS error compensation and lazy-batch updates, then unpermute + int4 pack.
//
// GPTQ overview page, "Jak działa": weights are quantized column by column in
// a fixed order; after each column the not-yet-quantized weights are
// corrected (OBS rule, inverse Hessian); block updates; 4- or 3-bit weights
// with a scale per group.  "Hiperparametry": bits, weights per scale.
// AutoGPTQ page, "Mixed Precision Scheme": int4 weights, dequantized on the
// fly at inference (the packed layout written here).
//
// Per column c of a row (processing order), with U = Cholesky factor of the
// inverse Hessian:
//   q = clamp(rint(w_c / s) + z, 0, maxq);  w^ = s (q - z);  e = (w_c - w^) / U[c][c]
//   w[c+1 : block end] -= e U[c][c+1 : block end]         (fused kernel, registers)
//   W[:, block end:]    -= E_blk U[blk, block end:]        (once per block, GEMM)
// Rows are independent once U is known, so a CTA owns 32 rows; each row is
// split over 4 threads of one warp that hold 32 columns each in registers.
// The column value is broadcast with one shuffle, every thread computes the
// same (q, e), and updates its own 32 columns from the U row in shared memory.
#include "common.cuh"
#include "gemm.cuh"

namespace gptq {

namespace {

constexpr int QB = 128;           // largest block width
constexpr int QTPR = 4;           // threads per row
constexpr int QCPT = 32;          // columns per thread
constexpr int QROWS = 32;         // rows per CTA
constexpr int QTHREADS = QROWS * QTPR;
constexpr int US_LD = QTPR * (QCPT + 4);   // padded so the 4 column parts hit distinct banks
constexpr size_t kBlockSmem = (static_cast<size_t>(QB) * US_LD + QB) * sizeof(float);

struct QArgs {
    float* Wp;            // [d_out][d_in] working weights, processing order
    const float* U;       // [d_in][d_in]
    int d_out, d_in, j0, bw, block, bits, gs, n_groups;
    float* scales;        // [d_out][n_groups]
    float* zeros;
    uint8_t* codes_p;     // [d_out][d_in], processing order
    float* E;             // [d_out][QB]
    float* err_sq;        // [d_out] or null
};

__device__ __forceinline__ void grid_from_range(float mn, float mx, float maxq, float& s, float& z)
{
    if (mn == mx) {
        mn = -1.f;
        mx = 1.f;
    }
    s = __fdiv_rn(mx - mn, maxq);
    z = rintf(__fdiv_rn(-mn, s));
}

__global__ void __launch_bounds__(QTHREADS) gptq_block_kernel(QArgs a)
{
    extern __shared__ __align__(16) float qsm[];
    float* Us = qsm;
    float* udiag = qsm + QB * US_LD;
    const int tid = threadIdx.x;
    const int j0 = a.j0, bw = a.bw, d_in = a.d_in;

    for (int idx = tid; idx < QB * QB; idx += QTHREADS) {
        const int c = idx / QB, k = idx % QB;
        float v = 0.f;
        if (c < bw && k < bw && k > c) v = a.U[static_cast<int64_t>(j0 + c) * d_in + j0 + k];
        Us[c * US_LD + (k >> 5) * (QCPT + 4) + (k & 31)] = v;
    }
    for (int c = tid; c < QB; c += QTHREADS)
        udiag[c] = (c < bw) ? a.U[static_cast<int64_t>(j0 + c) * (d_in + 1)] : 1.f;
    __syncthreads();

    const int lrow = tid / QTPR, part = tid % QTPR;
    const int r = blockIdx.x * QROWS + lrow;
    const bool valid = r < a.d_out;
    const int lane = tid & 31;
    const int lane_base = lane & ~(QTPR - 1);
    const float maxq = static_cast<float>((1 << a.bits) - 1);
    const int64_t rowoff = static_cast<int64_t>(r) * d_in;

    float w[QCPT];
    {
        const int c0 = part * QCPT;
#pragma unroll
        for (int m = 0; m < QCPT; m += 4) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid && c0 + m < bw) v = *reinterpret_cast<const float4*>(a.Wp + rowoff + j0 + c0 + m);
            w[m] = v.x;
            w[m + 1] = v.y;
            w[m + 2] = v.z;
            w[m + 3] = v.w;
        }
    }

    // grid of the group in effect at the block start
    float s = 1.f, z = 0.f;
    if (a.gs < 0) {
        if (valid) {
            s = a.scales[r];
            z = a.zeros[r];
        }
    } else if (a.gs > a.block) {
        const int g = j0 / a.gs;
        if (j0 % a.gs == 0) {
            float mn = 0.f, mx = 0.f;
            for (int k = part; k < a.gs; k += QTPR) {
                const float v = valid ? a.Wp[rowoff + j0 + k] : 0.f;
                mn = fminf(mn, v);
                mx = fmaxf(mx, v);
            }
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            grid_from_range(mn, mx, maxq, s, z);
            if (valid && part == 0) {
                a.scales[static_cast<int64_t>(r) * a.n_groups + g] = s;
                a.zeros[static_cast<int64_t>(r) * a.n_groups + g] = z;
            }
        } else if (valid) {
            s = a.scales[static_cast<int64_t>(r) * a.n_groups + g];
            z = a.zeros[static_cast<int64_t>(r) * a.n_groups + g];
        }
    }
    const bool inblock_groups = a.gs > 0 && a.gs <= a.block;

    uint32_t cq[QCPT / 4];
#pragma unroll
    for (int i = 0; i < QCPT / 4; ++i) cq[i] = 0u;
    float ereg[QCPT];
#pragma unroll
    for (int i = 0; i < QCPT; ++i) ereg[i] = 0.f;
    float errsum = 0.f;

    for (int po = 0; po < QTPR; ++po) {
#pragma unroll
        for (int m = 0; m < QCPT; ++m) {
            const int c = po * QCPT + m;
            if (c >= bw) break;
            if (inblock_groups && (c % a.gs) == 0) {
                float mn = 0.f, mx = 0.f;
#pragma unroll
                for (int mm = 0; mm < QCPT; ++mm) {
                    const int col = part * QCPT + mm;
                    const bool in = col >= c && col < c + a.gs && col < bw;
                    const float v = in ? w[mm] : 0.f;
                    mn = fminf(mn, v);
                    mx = fmaxf(mx, v);
                }
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                grid_from_range(mn, mx, maxq, s, z);
                if (valid && part == 0) {
                    const int g = (j0 + c) / a.gs;
                    a.scales[static_cast<int64_t>(r) * a.n_groups + g] = s;
                    a.zeros[static_cast<int64_t>(r) * a.n_groups + g] = z;
                }
            }
            const float wc = __shfl_sync(0xffffffffu, w[m], lane_base | po);
            float q = rintf(__fdiv_rn(wc, s)) + z;
            q = fminf(fmaxf(q, 0.f), maxq);
            const float what = s * (q - z);
            const float e = __fdiv_rn(wc - what, udiag[c]);
            if (part == po) {
                w[m] = what;
                ereg[m] = e;
                cq[m >> 2] |= static_cast<uint32_t>(q) << (8 * (m & 3));
                errsum = fmaf(e, e, errsum);
            }
            const float* urow = Us + c * US_LD + part * (QCPT + 4);
#pragma unroll
            for (int mm = 0; mm < QCPT; mm += 4) {
                const float4 u4 = *reinterpret_cast<const float4*>(urow + mm);
                w[mm] = fmaf(-e, u4.x, w[mm]);
                w[mm + 1] = fmaf(-e, u4.y, w[mm + 1]);
                w[mm + 2] = fmaf(-e, u4.z, w[mm + 2]);
                w[mm + 3] = fmaf(-e, u4.w, w[mm + 3]);
            }
        }
    }

    errsum += __shfl_xor_sync(0xffffffffu, errsum, 1);
    errsum += __shfl_xor_sync(0xffffffffu, errsum, 2);
    if (!valid) return;
    const int c0 = part * QCPT;
#pragma unroll
    for (int m = 0; m < QCPT; m += 4) {
        if (c0 + m < bw) {
            *reinterpret_cast<float4*>(a.Wp + rowoff + j0 + c0 + m) =
                make_float4(w[m], w[m + 1], w[m + 2], w[m + 3]);
            *reinterpret_cast<float4*>(a.E + static_cast<int64_t>(r) * QB + c0 + m) =
                make_float4(ereg[m], ereg[m + 1], ereg[m + 2], ereg[m + 3]);
            *reinterpret_cast<uint32_t*>(a.codes_p + rowoff + j0 + c0 + m) = cq[m >> 2];
        }
    }
    if (a.err_sq && part == 0) a.err_sq[r] += errsum;
}

// One (scale, zero) per row from the whole original row (group_size = -1).
__global__ void row_grid_kernel(const float* __restrict__ W, int d_out, int d_in, int bits,
                                float* __restrict__ scales, float* __restrict__ zeros)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= d_out) return;
    const float* row = W + static_cast<int64_t>(warp) * d_in;
    float mn = 0.f, mx = 0.f;
    for (int k = lane; k < d_in; k += 32) {
        mn = fminf(mn, row[k]);
        mx = fmaxf(mx, row[k]);
    }
    for (int o = 16; o; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
        float s, z;
        grid_from_range(mn, mx, static_cast<float>((1 << bits) - 1), s, z);
        scales[warp] = s;
        zeros[warp] = z;
    }
}

// inv[perm[k]] = k, with a range check of perm.
__global__ void invert_perm_kernel(const int32_t* __restrict__ perm, int d, int32_t* __restrict__ inv,
                                   int* status)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= d) return;
    const int p = perm[k];
    if (p < 0 || p >= d) {
        record_status(status, GPTQ_ERR_INVALID_ARG);
        return;
    }
    inv[p] = k;
}

// Wp[r][k] = W[r][perm[k]]
__global__ void gather_cols_kernel(const float* __restrict__ W, int d_out, int d_in,
                                   const int32_t* __restrict__ perm, float* __restrict__ Wp)
{
    const int64_t n = static_cast<int64_t>(d_out) * d_in;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = idx / d_in;
        const int k = static_cast<int>(idx - r * d_in);
        int p = perm[k];
        p = (p < 0 || p >= d_in) ? 0 : p;
        Wp[idx] = W[r * d_in + p];
    }
}

// Original-order outputs: codes, packed nibbles, and (with a permutation) W^.
// One thread per pair of original columns (2i, 2i+1).
__global__ void finish_kernel(const uint8_t* __restrict__ codes_p, const float* __restrict__ Wp,
                              const int32_t* __restrict__ inv, int d_out, int d_in,
                              float* __restrict__ W, uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ packed)
{
    const int half = d_in / 2;
    const int64_t n = static_cast<int64_t>(d_out) * half;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = idx / half;
        const int i = static_cast<int>(idx - r * half);
        const int c0 = 2 * i, c1 = 2 * i + 1;
        int k0 = inv ? inv[c0] : c0;
        int k1 = inv ? inv[c1] : c1;
        k0 = (k0 < 0 || k0 >= d_in) ? 0 : k0;   // a malformed permutation stays in bounds
        k1 = (k1 < 0 || k1 >= d_in) ? 0 : k1;
        const int64_t ro = r * d_in;
        const uint8_t q0 = codes_p[ro + k0], q1 = codes_p[ro + k1];
        if (codes) {
            codes[ro + c0] = q0;
            codes[ro + c1] = q1;
        }
        if (packed) packed[r * half + i] = static_cast<uint8_t>((q0 & 15) | ((q1 & 15) << 4));
        if (inv) {
            W[ro + c0] = Wp[ro + k0];
            W[ro + c1] = Wp[ro + k1];
        }
    }
}

__global__ void g_idx_kernel(const int32_t* __restrict__ perm, int d, int gs, int32_t* __restrict__ g_idx)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= d) return;
    int p = perm ? perm[k] : k;
    if (p < 0 || p >= d) return;
    g_idx[p] = gs > 0 ? k / gs : 0;
}

__global__ void zero_f32_kernel(float* p, int64_t n)
{
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = 0.f;
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ src, float* __restrict__ dst, int64_t n)
{
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        dst[i] = __uint_as_float(static_cast<uint32_t>(src[i]) << 16);
}

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t quantize_workspace_bytes(int64_t d_out, int64_t d_in)
{
    const size_t n = static_cast<size_t>(d_out) * static_cast<size_t>(d_in);
    return 256 + up256(n * sizeof(float)) + up256(n) +
           up256(static_cast<size_t>(d_out) * QB * sizeof(float)) +
           up256(static_cast<size_t>(d_in) * sizeof(int32_t));
}

int run_quantize(float* W, const float* U, const int32_t* perm, int64_t d_out64, int64_t d_in64,
                 int bits, int gs, int block, uint8_t* codes, float* scales, float* zeros,
                 uint8_t* packed, int32_t* g_idx, float* err_sq, void* workspace,
                 cudaStream_t stream)
{
    const int d_out = static_cast<int>(d_out64), d_in = static_cast<int>(d_in64);
    const size_t n = static_cast<size_t>(d_out) * d_in;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* Wp = reinterpret_cast<float*>(ws + 256);
    uint8_t* codes_p = ws + 256 + up256(n * sizeof(float));
    float* E = reinterpret_cast<float*>(ws + 256 + up256(n * sizeof(float)) + up256(n));
    int32_t* inv = reinterpret_cast<int32_t*>(ws + 256 + up256(n * sizeof(float)) + up256(n) +
                                              up256(static_cast<size_t>(d_out) * QB * sizeof(float)));
    const int nsm = sm_count();
    int* status = device_status_ptr();
    const int n_groups = gs > 0 ? d_in / gs : 1;

    static bool attr_set[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmem)));
        attr_set[dev] = true;
    }

    float* work = W;
    if (perm) {
        invert_perm_kernel<<<(d_in + 255) / 256, 256, 0, stream>>>(perm, d_in, inv, status);
        GPTQ_LAUNCH_CHECK();
        gather_cols_kernel<<<nsm * 8, 256, 0, stream>>>(W, d_out, d_in, perm, Wp);
        GPTQ_LAUNCH_CHECK();
        work = Wp;
    }
    if (err_sq) {
        zero_f32_kernel<<<(d_out + 255) / 256, 256, 0, stream>>>(err_sq, d_out);
        GPTQ_LAUNCH_CHECK();
    }
    if (gs < 0) {
        row_grid_kernel<<<(d_out * 32 + 255) / 256, 256, 0, stream>>>(work, d_out, d_in, bits,
                                                                       scales, zeros);
        GPTQ_LAUNCH_CHECK();
    }
    const int grid = (d_out + QROWS - 1) / QROWS;
    for (int j0 = 0; j0 < d_in; j0 += block) {
        const int bw = (d_in - j0 < block) ? d_in - j0 : block;
        QArgs a{work, U, d_out, d_in, j0, bw, block, bits, gs, n_groups, scales, zeros,
                codes_p, E, err_sq};
        gptq_block_kernel<<<grid, QTHREADS, kBlockSmem, stream>>>(a);
        GPTQ_LAUNCH_CHECK();
        const int rest = d_in - j0 - bw;
        if (rest > 0) {
            int rc = launch_sgemm(false, d_out, rest, bw, -1.f, E, QB, 0,
                                  U + static_cast<int64_t>(j0) * d_in + j0 + bw, d_in, 0, 1.f,
                                  work + j0 + bw, d_in, 0, 1, 0, stream);
            if (rc) return rc;
        }
    }
    if (codes || packed || perm) {
        finish_kernel<<<nsm * 8, 256, 0, stream>>>(codes_p, Wp, perm ? inv : nullptr, d_out, d_in,
                                                   W, codes, packed);
        GPTQ_LAUNCH_CHECK();
    }
    if (g_idx) {
        g_idx_kernel<<<(d_in + 255) / 256, 256, 0, stream>>>(perm, d_in, gs, g_idx);
        GPTQ_LAUNCH_CHECK();
    }
    return GPTQ_OK;
}

int run_bf16_to_f32(float* dst, const uint16_t* src, int64_t n, cudaStream_t stream)
{
    if (n <= 0) return GPTQ_OK;
    int blocks = static_cast<int>((n + 255) / 256);
    if (blocks > sm_count() * 16) blocks = sm_count() * 16;
    bf16_to_f32_kernel<<<blocks, 256, 0, stream>>>(src, dst, n);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

}  // namespace gptq
