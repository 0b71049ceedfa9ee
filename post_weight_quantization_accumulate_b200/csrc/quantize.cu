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
// Rows are independent once U is known.  Each row is split over 4 adjacent
// lanes of a warp; lane part p holds the row's in-block columns 32p..32p+31 in
// registers.  Every lane of the row computes the same (q, e) for the current
// column and corrects its own 32 registers with U row c from shared memory.
// The block's U rows are laid out once per call by u_layout_kernel and arrive
// in shared memory by bulk copies, one per 16-column sub-block.
#include "common.cuh"
#include "gemm.cuh"

namespace gptq {

namespace {

constexpr int QB = 128;           // largest block width
constexpr int kOuterMax = 1024;   // widest outer window of the two-level lazy batch
constexpr int QTPR = 4;           // lanes per row
constexpr int QCPT = QB / QTPR;   // registers per lane: part p holds columns 32p .. 32p+31
constexpr int QSUB = 16;          // columns per unrolled sub-block (one bulk copy each)
constexpr int QNSUB = QB / QSUB;
constexpr int QROWS = 32;         // rows per CTA
constexpr int QTHREADS = QROWS * QTPR;
// U rows of a sub-block: [16 rows][4 parts][40] (32 coefficients + 8 pad, so the
// four parts of a row fall in distinct bank groups), then 16 pairs
// (1 / U[c][c], U[c][c+1]).
constexpr int UT_PART = QCPT + 8;
constexpr int UT_LD = QTPR * UT_PART;
constexpr int UCH_FLOATS = QSUB * UT_LD + 2 * QSUB;
constexpr int UCH_BYTES = UCH_FLOATS * 4;          // 10368, a multiple of 16
constexpr size_t kBlockSmem = static_cast<size_t>(QNSUB) * UCH_BYTES + 128;
static_assert(UCH_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");

struct QArgs {
    float* Wp;            // [d_out][d_in] working weights, processing order
    const float* Ul;      // U blocks in sub-block layout (u_layout_kernel)
    int d_out, d_in, j0, bw, block, bits, gs, n_groups;
    float* scales;        // [d_out][n_groups]
    float* zeros;
    uint8_t* codes_p;     // [d_out][d_in], processing order
    float* E;             // [d_out][kOuterMax] errors of the current outer window
    int e_off;            // column of this block inside the outer window
    float* err_sq;        // [d_out] or null
    int* status;
};

// Sub-block layout of U's diagonal blocks: chunk (b, S) covers rows
// j0 + 16S .. j0 + 16S + 15 of block b (j0 = b * block, width bw).  Entry
// [cl][p][k] is U[j0+c][j0+32p+k] for in-block column 32p+k > c (zero on and
// below the diagonal and beyond bw); pair cl is (1 / U[c][c], U[c][c+1]),
// zero past bw.  One CTA per chunk.
__global__ void u_layout_kernel(const float* __restrict__ U, int d_in, int block, int nch_blk,
                                float* __restrict__ Ul)
{
    const int b = blockIdx.x / nch_blk, S = blockIdx.x % nch_blk;
    const int j0 = b * block;
    const int bw = min(block, d_in - j0);
    float* out = Ul + static_cast<int64_t>(blockIdx.x) * UCH_FLOATS;
    for (int idx = threadIdx.x; idx < UCH_FLOATS; idx += blockDim.x) {
        float v = 0.f;
        if (idx < QSUB * UT_LD) {
            const int cl = idx / UT_LD, rem = idx % UT_LD;
            const int p = rem / UT_PART, k = rem % UT_PART;
            const int c = S * QSUB + cl, col = QCPT * p + k;
            if (k < QCPT && c < bw && col > c && col < bw)
                v = U[static_cast<int64_t>(j0 + c) * d_in + j0 + col];
        } else {
            const int i = idx - QSUB * UT_LD;
            const int c = S * QSUB + i / 2;
            if (i % 2 == 0) {
                if (c < bw) v = 1.f / U[static_cast<int64_t>(j0 + c) * d_in + j0 + c];
            } else if (c + 1 < bw) {
                v = U[static_cast<int64_t>(j0 + c) * d_in + j0 + c + 1];
            }
        }
        out[idx] = v;
    }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void grid_from_range(float mn, float mx, float maxq, float& s, float& z)
{
    if (mn == mx) {
        mn = -1.f;
        mx = 1.f;
    }
    s = __fdiv_rn(mx - mn, maxq);
    z = rintf(__fdiv_rn(-mn, s));
}

// rint(w / s) with w / s correctly rounded, from the product t = w * rs (rs the
// correctly rounded 1 / s).  t is within 2^-23 relative of w / s, so the two
// round to the same integer unless t lies that close to a half-integer; only
// then is the division carried out.
__device__ __forceinline__ float rint_div(float w, float s, float rs)
{
    const float t = w * rs;
    const float r = rintf(t);
    const float thr = fmaf(-4.8e-7f, fmaxf(fabsf(t), 1.f), 0.5f);
    if (fabsf(t - r) >= thr) return rintf(__fdiv_rn(w, s));
    return r;
}

// Scale and zero of the group starting at in-block column c, from the row's
// current values: each part reduces its registers whose column lies in
// [c, c + gs) and below bw, then the row's QTPR parts combine.
__device__ __forceinline__ void group_grid(const float (&w)[QCPT], int part, int c, int gs, int bw,
                                           float maxq, float& s, float& z)
{
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int k = 0; k < QCPT; ++k) {
        const int col = QCPT * part + k;
        const bool in = col >= c && col < c + gs && col < bw;
        const float v = in ? w[k] : 0.f;
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
// Per column c every lane of the row knows the row's current value through
// `nxt` (column c+1 fetched one step early with a shuffle from its owner and
// corrected by this step's error), computes the same q and e, writes e, the
// code and w^ to global memory, and corrects its own registers with U row c.
// Columns at and before c have coefficient 0 in the laid-out U rows, so the
// register file is updated whole and stays compile-time indexed; a 16-step
// sub-block is unrolled (the half of the 32-register window it sits in is
// chosen by a select).
// kGroupsInStep: a group may start inside a 16-column sub-block (group sizes
// that are not multiples of 16); otherwise groups start at sub-block starts.
template <bool kGroupsInStep>
__global__ void __launch_bounds__(QTHREADS, 1) gptq_block_kernel(QArgs a)
{
    extern __shared__ __align__(128) uint8_t qsm_raw[];
    float* Ut = reinterpret_cast<float*>(qsm_raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(qsm_raw + QNSUB * UCH_BYTES);
    int* abort_flag = reinterpret_cast<int*>(bars + QNSUB);
    const int tid = threadIdx.x;
    const int j0 = a.j0, bw = a.bw, d_in = a.d_in;
    const int nsub = (bw + QSUB - 1) / QSUB;
    const int nch_blk = (a.block + QSUB - 1) / QSUB;

    if (tid == 0) {
        for (int S = 0; S < QNSUB; ++S) mbar_init(&bars[S], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const float* src = a.Ul + static_cast<int64_t>(j0 / a.block) * nch_blk * UCH_FLOATS;
        for (int S = 0; S < nsub; ++S) {
            mbar_arrive_expect_tx(&bars[S], UCH_BYTES);
            bulk_load(qsm_raw + S * UCH_BYTES, src + S * UCH_FLOATS, UCH_BYTES, &bars[S]);
        }
    }

    const int lrow = tid / QTPR, part = tid % QTPR;
    const int r = blockIdx.x * QROWS + lrow;
    const bool valid = r < a.d_out;
    const int lane = tid & 31;
    const int lane_base = lane & ~(QTPR - 1);
    const float maxq = static_cast<float>((1 << a.bits) - 1);
    const int64_t rowoff = static_cast<int64_t>(valid ? r : 0) * d_in;

    float w[QCPT];
#pragma unroll
    for (int m = 0; m < QCPT / 4; ++m) {
        const int col = QCPT * part + 4 * m;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid && col < bw) v = *reinterpret_cast<const float4*>(a.Wp + rowoff + j0 + col);
        w[4 * m] = v.x;
        w[4 * m + 1] = v.y;
        w[4 * m + 2] = v.z;
        w[4 * m + 3] = v.w;
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

    float* e_out = a.E + static_cast<int64_t>(valid ? r : 0) * kOuterMax + a.e_off;
    uint8_t* q_out = a.codes_p + rowoff + j0;
    float* w_out = a.Wp + rowoff + j0;

    float errsum = 0.f;
    float nxt = __shfl_sync(0xffffffffu, w[0], lane_base);   // column 0 (part 0)

#pragma unroll 1
    for (int S = 0; S < nsub; ++S) {
        const bool got = mbar_wait_bounded(&bars[S], 0, abort_flag, a.status);
        if (!__syncthreads_and(got)) break;
        const float* ub = Ut + S * UCH_FLOATS;
        const float2* pairs = reinterpret_cast<const float2*>(ub + QSUB * UT_LD);
        const bool hi = (S & 1) != 0;                 // sub-block sits in registers 16..31
        const int src_in = lane_base | (S >> 1);      // owner of columns 16S .. 16S+15
        const int src_next = lane_base | min((S + 1) >> 1, QTPR - 1);
        const int cbase = S * QSUB;
        if (!kGroupsInStep && cbase == next_group) {
            group_grid(w, part, cbase, gs_in, bw, maxq, s, z);
            rs = 1.f / s;
            if (valid && part == 0) {
                const int g = (j0 + cbase) / gs_in;
                a.scales[static_cast<int64_t>(r) * a.n_groups + g] = s;
                a.zeros[static_cast<int64_t>(r) * a.n_groups + g] = z;
            }
            next_group += gs_in;
        }
#pragma unroll
        for (int cl = 0; cl < QSUB; ++cl) {
            const int c = cbase + cl;
            const float* urow = ub + cl * UT_LD + part * UT_PART;
            float u[QCPT];
#pragma unroll
            for (int k = 0; k < QCPT; k += 4) {
                const float4 u4 = *reinterpret_cast<const float4*>(urow + k);
                u[k] = u4.x;
                u[k + 1] = u4.y;
                u[k + 2] = u4.z;
                u[k + 3] = u4.w;
            }
            const float2 rn = pairs[cl];   // (1 / U[c][c], U[c][c+1])
            // column c+1 after the corrections of steps < c, from its owner
            const float cand = hi ? w[(QSUB + 1 + cl) & (QCPT - 1)] : w[cl + 1];
            const float pre = __shfl_sync(0xffffffffu, cand, cl + 1 < QSUB ? src_in : src_next);
            if (kGroupsInStep && c == next_group && c < bw) {
                group_grid(w, part, c, gs_in, bw, maxq, s, z);
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
            const float e = (wc - what) * rn.x;
            nxt = fmaf(-e, rn.y, pre);
            errsum = fmaf(e, e, errsum);
            if (valid && c < bw) {
                e_out[c] = e;
                q_out[c] = static_cast<uint8_t>(q);
                w_out[c] = what;
            }
#pragma unroll
            for (int k = 0; k < QCPT; ++k) w[k] = fmaf(-e, u[k], w[k]);
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

// Sub-block chunks of the U layout for any block width 8..128: each block of
// width bw has ceil(bw / 16) <= bw / 8 chunks, plus one for a ragged last block.
inline size_t u_layout_bytes(int64_t d_in)
{
    return static_cast<size_t>(d_in / 8 + 16) * UCH_BYTES;
}

size_t quantize_workspace_bytes(int64_t d_out, int64_t d_in)
{
    const size_t n = static_cast<size_t>(d_out) * static_cast<size_t>(d_in);
    return 256 + up256(n * sizeof(float)) + up256(n) +
           up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float)) +
           up256(static_cast<size_t>(d_in) * sizeof(int32_t)) + up256(u_layout_bytes(d_in));
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
    float* Ul = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(inv) +
                                         up256(static_cast<size_t>(d_in) * sizeof(int32_t)));
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

    const int nch_blk = (block + QSUB - 1) / QSUB;
    const int n_blocks = (d_in + block - 1) / block;
    u_layout_kernel<<<n_blocks * nch_blk, 256, 0, stream>>>(U, d_in, block, nch_blk, Ul);
    GPTQ_LAUNCH_CHECK();

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
            QArgs a{work, Ul, d_out, d_in, j0, bw, block, bits, gs, n_groups, scales, zeros,
                    codes_p, E, j0 - J0, err_sq, status};
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
