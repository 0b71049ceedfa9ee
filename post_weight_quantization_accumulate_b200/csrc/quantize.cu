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
constexpr int kOuterMax = 1024;   // widest outer window of the two-level lazy batch
constexpr int QTPR = 8;           // threads per row
constexpr int QCPT = QB / QTPR;   // registers per thread (column 8m + p belongs to part p)
constexpr int QSUB = 16;          // columns per unrolled sub-block
constexpr int QRPS = QSUB / QTPR; // registers a sub-block occupies per thread
constexpr int QROWS = 16;         // rows per CTA
constexpr int QTHREADS = QROWS * QTPR;
constexpr int UT_PART = QCPT + 4; // padded part stride (80 bytes): the 8 parts of a U row
                                  // read by one 8-lane phase hit distinct banks
constexpr int UT_LD = QTPR * UT_PART;
constexpr int ES_LD = QB + 4;
constexpr size_t kBlockSmem =
    (static_cast<size_t>(QB) * UT_LD + QB + static_cast<size_t>(QROWS) * ES_LD) * sizeof(float) +
    static_cast<size_t>(QROWS) * ES_LD;

struct QArgs {
    float* Wp;            // [d_out][d_in] working weights, processing order
    const float* U;       // [d_in][d_in]
    int d_out, d_in, j0, bw, block, bits, gs, n_groups;
    float* scales;        // [d_out][n_groups]
    float* zeros;
    uint8_t* codes_p;     // [d_out][d_in], processing order
    float* E;             // [d_out][kOuterMax] errors of the current outer window
    int e_off;            // column of this block inside the outer window
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

// rint(w / s) with w / s correctly rounded, from the product w * rs (rs the
// correctly rounded 1 / s).  The product is within 2^-23 relative of w / s,
// so the two round to the same integer unless w / s lies that close to a
// half-integer; only then is the division carried out.
__device__ __forceinline__ float rint_div(float w, float s, float rs)
{
    const float t = w * rs;
    const float fr = t - floorf(t);
    if (fabsf(fr - 0.5f) <= 4.8e-7f * fmaxf(fabsf(t), 1.f)) return rintf(__fdiv_rn(w, s));
    return rintf(t);
}

// Register slot of in-block column k (owned by part k % QTPR) while sub-block
// S is processed: the QCPT-slot window rotates by QRPS slots per sub-block,
// so the current sub-block always sits in slots 0..QRPS-1.
__device__ __forceinline__ int slot_of(int k, int S) { return (k / QTPR - QRPS * S) & (QCPT - 1); }

// Scale and zero of the group starting at in-block column c, from the row's
// current values: each part reduces its registers whose column lies in
// [c, c + gs) and below bw, then the QTPR parts combine.
__device__ __forceinline__ void group_grid(const float (&w)[QCPT], int S, int part, int c, int gs,
                                           int bw, float maxq, float& s, float& z)
{
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int mm = 0; mm < QCPT; ++mm) {
        const int col = QTPR * ((mm + QRPS * S) & (QCPT - 1)) + part;
        const bool in = col >= c && col < c + gs && col < bw;
        const float v = in ? w[mm] : 0.f;
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int o = 1; o < QTPR; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    grid_from_range(mn, mx, maxq, s, z);
}

// One lazy-batch block [j0, j0 + bw) of the column loop for QROWS rows.
// Part p of a row holds columns 8m + p of the block in 16 registers.  Per
// column c every part knows the row's current value through `nxt` (a copy of
// column c+1 fetched one step early with a shuffle), computes the same q and
// e, and corrects its own registers with U row c from shared memory.  The U
// rows are stored in the register order of their sub-block, in which columns
// already quantized have coefficient 0.  Only 16 steps are unrolled; the
// window rotates after each sub-block, which keeps the code small enough for
// the instruction cache.  Nothing is stored inside a step: the step's U row
// is read first, errors and codes stay in registers until the sub-block ends.
// kGroupsInStep: a group may start inside a 16-column sub-block (group sizes
// that are not multiples of 16); otherwise groups start at sub-block starts.
template <bool kGroupsInStep>
__global__ void __launch_bounds__(QTHREADS) gptq_block_kernel(QArgs a)
{
    extern __shared__ __align__(16) float qsm[];
    float* Ut = qsm;                         // [c][p][slot]
    float* rdiag = qsm + QB * UT_LD;         // 1 / U[c][c]
    float* Es = rdiag + QB;                  // [row][c] errors e
    uint8_t* Cs = reinterpret_cast<uint8_t*>(Es + QROWS * ES_LD);  // [row][c] codes
    const int tid = threadIdx.x;
    const int j0 = a.j0, bw = a.bw, d_in = a.d_in;

    // U block: 128 rows x 32 float4 loads, 8 in flight per thread
#pragma unroll 1
    for (int base = 0; base < QB * (QB / 4); base += QTHREADS * 8) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = base + i * QTHREADS + tid;
            const int c = idx / (QB / 4), k = (idx % (QB / 4)) * 4;
            v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c < bw && k < bw)
                v[i] = *reinterpret_cast<const float4*>(a.U + static_cast<int64_t>(j0 + c) * d_in + j0 + k);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = base + i * QTHREADS + tid;
            const int c = idx / (QB / 4), k = (idx % (QB / 4)) * 4;
            const int S = c / QSUB;
            const float e4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int kk = k + t;
                Ut[c * UT_LD + (kk % QTPR) * UT_PART + slot_of(kk, S)] = (kk > c && kk < bw) ? e4[t] : 0.f;
            }
            if (k <= c && c < k + 4 && c < bw) {
                const int t = c - k;
                const float dv = t == 0 ? v[i].x : t == 1 ? v[i].y : t == 2 ? v[i].z : v[i].w;
                rdiag[c] = 1.f / dv;
            }
        }
    }
    __syncthreads();

    const int lrow = tid / QTPR, part = tid % QTPR;
    const int r = blockIdx.x * QROWS + lrow;
    const bool valid = r < a.d_out;
    const int lane = tid & 31;
    const int lane_base = lane & ~(QTPR - 1);
    const float maxq = static_cast<float>((1 << a.bits) - 1);
    const int64_t rowoff = static_cast<int64_t>(r) * d_in;

    float w[QCPT];
#pragma unroll
    for (int m = 0; m < QCPT; ++m)
        w[m] = (valid && QTPR * m + part < bw) ? a.Wp[rowoff + j0 + QTPR * m + part] : 0.f;

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
#pragma unroll
            for (int o = 1; o < QTPR; o <<= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
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
    float rs = 1.f / s;
    const int gs_in = (a.gs > 0 && a.gs <= a.block) ? a.gs : 0;
    int next_group = gs_in ? 0 : 1 << 30;

    float errsum = 0.f;
    float nxt = __shfl_sync(0xffffffffu, w[0], lane_base | 0);   // column 0
    const int nsub = (bw + QSUB - 1) / QSUB;

#pragma unroll 1
    for (int S = 0; S < nsub; ++S) {
        const float* ub = Ut + S * QSUB * UT_LD;
        const float* rd = rdiag + S * QSUB;
        if (!kGroupsInStep && S * QSUB == next_group) {
            group_grid(w, S, part, S * QSUB, gs_in, bw, maxq, s, z);
            rs = 1.f / s;
            if (valid && part == 0) {
                const int g = (j0 + S * QSUB) / gs_in;
                a.scales[static_cast<int64_t>(r) * a.n_groups + g] = s;
                a.zeros[static_cast<int64_t>(r) * a.n_groups + g] = z;
            }
            next_group += gs_in;
        }
        float e_own[QRPS], q_own[QRPS];
#pragma unroll
        for (int i = 0; i < QRPS; ++i) e_own[i] = q_own[i] = 0.f;
#pragma unroll
        for (int cl = 0; cl < QSUB; ++cl) {
            const int c = S * QSUB + cl;
            if (c < bw) {
                const int m = cl / QTPR, po = cl % QTPR;
                const int mn1 = (cl + 1) / QTPR, pn1 = (cl + 1) % QTPR;
                const float* urow = ub + cl * UT_LD;
                // operands of this step that do not depend on its error
                float u[QCPT];
#pragma unroll
                for (int mm = (m & ~3); mm < QCPT; mm += 4) {
                    const float4 u4 = *reinterpret_cast<const float4*>(urow + part * UT_PART + mm);
                    u[mm] = u4.x;
                    u[mm + 1] = u4.y;
                    u[mm + 2] = u4.z;
                    u[mm + 3] = u4.w;
                }
                const float unext = urow[pn1 * UT_PART + mn1];
                const float rdc = rd[cl];
                // column c+1 after the corrections of steps < c (its owner's register)
                const float pre = __shfl_sync(0xffffffffu, w[mn1], lane_base | pn1);
                if (kGroupsInStep && c == next_group) {
                    group_grid(w, S, part, c, gs_in, bw, maxq, s, z);
                    rs = 1.f / s;
                    if (valid && part == 0) {
                        const int g = (j0 + c) / gs_in;
                        a.scales[static_cast<int64_t>(r) * a.n_groups + g] = s;
                        a.zeros[static_cast<int64_t>(r) * a.n_groups + g] = z;
                    }
                    next_group += gs_in;
                }
                const float wc = nxt;
                float q = rint_div(wc, s, rs) + z;
                q = fminf(fmaxf(q, 0.f), maxq);
                const float what = s * (q - z);
                const float e = (wc - what) * rdc;
                nxt = fmaf(-e, unext, pre);
                if (part == po) {
                    w[m] = what;
                    e_own[m] = e;
                    q_own[m] = q;
                    errsum = fmaf(e, e, errsum);
                }
#pragma unroll
                for (int mm = m; mm < QCPT; ++mm) w[mm] = fmaf(-e, u[mm], w[mm]);
            }
        }
        // sub-block S is final in slots 0..QRPS-1: store, then rotate the window
#pragma unroll
        for (int i = 0; i < QRPS; ++i) {
            const int col = S * QSUB + QTPR * i + part;
            if (col < bw) {
                if (valid) a.Wp[rowoff + j0 + col] = w[i];
                Es[lrow * ES_LD + col] = e_own[i];
                Cs[lrow * ES_LD + col] = static_cast<uint8_t>(q_own[i]);
            }
        }
        float t[QRPS];
#pragma unroll
        for (int i = 0; i < QRPS; ++i) t[i] = w[i];
#pragma unroll
        for (int i = 0; i < QCPT - QRPS; ++i) w[i] = w[i + QRPS];
#pragma unroll
        for (int i = 0; i < QRPS; ++i) w[QCPT - QRPS + i] = t[i];
    }

#pragma unroll
    for (int o = 1; o < QTPR; o <<= 1) errsum += __shfl_xor_sync(0xffffffffu, errsum, o);
    __syncthreads();
    // errors and codes of the CTA's rows, row-contiguous
    for (int idx = tid; idx < QROWS * QB; idx += QTHREADS) {
        const int rl = idx / QB, c = idx % QB;
        const int rr = blockIdx.x * QROWS + rl;
        if (rr < a.d_out && c < bw) {
            a.E[static_cast<int64_t>(rr) * kOuterMax + a.e_off + c] = Es[rl * ES_LD + c];
            a.codes_p[static_cast<int64_t>(rr) * d_in + j0 + c] = Cs[rl * ES_LD + c];
        }
    }
    if (valid && a.err_sq && part == 0) a.err_sq[r] += errsum;
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
           up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float)) +
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
                                              up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float)));
    const int nsm = sm_count();
    int* status = device_status_ptr();
    const int n_groups = gs > 0 ? d_in / gs : 1;

    static bool attr_set[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmem)));
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmem)));
        attr_set[dev] = true;
    }
    // groups start only at 16-column sub-block starts when group_size is a
    // multiple of 16 that fits the block (or there are no in-block groups)
    const bool groups_in_step = gs > 0 && gs <= block && (gs % QSUB) != 0;

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
    // Two-level lazy batch: a block's errors correct the rest of its outer
    // window right away (K = block), and the columns beyond the window once
    // per window (K = window width).  A group wider than a block must lie in
    // one window; groups wider than kOuterMax use one level.
    int outer;
    if (gs > kOuterMax)
        outer = block;
    else if (gs > block)
        outer = (kOuterMax / gs) * gs;
    else
        outer = (kOuterMax / block) * block;
    const int grid = (d_out + QROWS - 1) / QROWS;
    for (int J0 = 0; J0 < d_in; J0 += outer) {
        const int J1 = (d_in - J0 < outer) ? d_in : J0 + outer;
        for (int j0 = J0; j0 < J1; j0 += block) {
            const int bw = (J1 - j0 < block) ? J1 - j0 : block;
            QArgs a{work, U, d_out, d_in, j0, bw, block, bits, gs, n_groups, scales, zeros,
                    codes_p, E, j0 - J0, err_sq};
            if (groups_in_step)
                gptq_block_kernel<true><<<grid, QTHREADS, kBlockSmem, stream>>>(a);
            else
                gptq_block_kernel<false><<<grid, QTHREADS, kBlockSmem, stream>>>(a);
            GPTQ_LAUNCH_CHECK();
            const int rest_in = J1 - j0 - bw;
            if (rest_in > 0) {
                int rc = launch_sgemm(false, d_out, rest_in, bw, -1.f, E + (j0 - J0), kOuterMax, 0,
                                      U + static_cast<int64_t>(j0) * d_in + j0 + bw, d_in, 0, 1.f,
                                      work + j0 + bw, d_in, 0, 1, 0, stream);
                if (rc) return rc;
            }
        }
        const int rest = d_in - J1;
        if (rest > 0) {
            int rc = launch_sgemm(false, d_out, rest, J1 - J0, -1.f, E, kOuterMax, 0,
                                  U + static_cast<int64_t>(J0) * d_in + J1, d_in, 0, 1.f,
                                  work + J1, d_in, 0, 1, 0, stream);
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
