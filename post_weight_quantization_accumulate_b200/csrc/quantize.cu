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
// Rows are independent once U is known.  A lane holds two rows and 16 of
// their in-block columns in registers (part p of 8 lanes: columns 16p ..
// 16p+15), so each U value read from shared memory serves two rows.  Every
// lane of a row pair computes the same (q, e) for the current column of both
// rows and corrects its own registers with U row c.  The block's U rows are
// laid out once per call by u_layout_kernel and arrive in shared memory by
// bulk copies, one per 16-column sub-block.
#include "common.cuh"
#include "gemm.cuh"

#include <algorithm>
#include <mutex>
#include <vector>

namespace gptq {

namespace {

constexpr int QB = 128;           // largest block width
constexpr int kOuterMax = 1024;   // widest outer window of the two-level lazy batch
constexpr int QTPR = 8;           // lanes per row pair
constexpr int QCPT = QB / QTPR;   // 16 registers per row: part p holds columns 16p .. 16p+15
constexpr int QSUB = 16;          // columns per sub-block = one part's columns
constexpr int QNSUB = QB / QSUB;
constexpr int QPAIRS = 16;        // row pairs per CTA
constexpr int QROWS = 2 * QPAIRS;
constexpr int QTHREADS = QPAIRS * QTPR;
static_assert(QSUB == QCPT, "sub-block S is the register range of part S");
// U rows of a sub-block: [16 rows][8 parts][20] (16 coefficients + 4 pad, so
// the 8 parts of a row fall in distinct 16-byte bank groups), then 16 pairs
// (1 / U[c][c], U[c][c+1]).
constexpr int UT_PART = QCPT + 4;
constexpr int UT_LD = QTPR * UT_PART;
constexpr int UCH_FLOATS = QSUB * UT_LD + 2 * QSUB;
constexpr int UCH_BYTES = UCH_FLOATS * 4;          // 10368, a multiple of 16
constexpr size_t kBlockSmem = static_cast<size_t>(QNSUB) * UCH_BYTES + 128;
// Shared memory a column-loop launch asks for when its grid fits on the SMs
// at once: more than half of an SM's, so that one CTA holds an SM by itself.
// Two CTAs on one SM would each take longer, and every launch lasts as long as
// its slowest CTA; with programmatic dependent launches the early CTAs of a
// launch would otherwise double up on the few SMs the previous kernel leaves
// free.
constexpr size_t kBlockSmemLaunch = 116 * 1024;
static_assert(kBlockSmemLaunch >= kBlockSmem, "the launch covers the kernel's shared memory");
static_assert(UCH_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");

struct QArgs {
    float* Wp;            // [d_out][d_in] working weights, processing order
    const float* Ul;      // U blocks in sub-block layout (u_layout_kernel)
    int d_out, d_in, j0, bw, block, bits, gs, n_groups;
    float* scales;        // [d_out][n_groups]
    float* zeros;
    uint8_t* codes_p;     // [d_out][d_in], processing order
    float* E;             // [d_out][kOuterMax] errors of the current outer window
    float* E_lo;          // their low parts e - trunc_tf32(e) (tensor-core operand) or null
    int e_off;            // column of this block inside the outer window
    float* err_sq;        // [d_out] or null
    int* status;
    // two-level Q4_K grid (null otherwise): 6-bit scale and min per 32-column
    // block [d_out][d_in / 32], super-block scales [d_out][d_in / 256]
    uint8_t* sc6;
    uint8_t* m6;
    float* dsup;
    float* dmin;
    // span of this launch (two words preset to ~0 and 0; null when not timed):
    // atomicMin of the time the first CTA passes the dependency wait,
    // atomicMax of the time the last CTA ends (globaltimer, ns)
    unsigned long long* stamp;
};

// Sub-block layout of U's diagonal blocks: chunk (b, S) covers rows
// j0 + 16S .. j0 + 16S + 15 of block b (j0 = b * block, width bw).  Entry
// [cl][p][k] is U[j0+c][j0+16p+k] for in-block column 16p+k > c (zero on and
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

// Low part of x below its tf32 truncation (exact in float32): the tensor core
// reads an fp32 operand as tf32 by dropping the 13 low mantissa bits.
__device__ __forceinline__ float tf32_low(float x)
{
    return x - __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// U_lo[i][j] = tf32_low(U[i][j]) on and above the diagonal (the part the
// lazy-batch products read).
__global__ void u_low_kernel(const float* __restrict__ U, int d, float* __restrict__ U_lo)
{
    const int64_t n4 = static_cast<int64_t>(d) * d / 4;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int row = static_cast<int>((4 * i) / d), col = static_cast<int>((4 * i) % d);
        if (col + 3 < row) continue;
        const float4 v = reinterpret_cast<const float4*>(U)[i];
        reinterpret_cast<float4*>(U_lo)[i] = make_float4(tf32_low(v.x), tf32_low(v.y), tf32_low(v.z), tf32_low(v.w));
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

// w / s correctly rounded, without a division: t = w * rs with rs = RN(1 / s),
// then one correction with the exact residual fma(-t, s, w) (Markstein's
// correction step, P. Markstein, "IA-64 and Elementary Functions", 2000).
// Being free of branches it keeps the unrolled column steps one basic block.
// gptq_selftest_quotient compares it with IEEE division on the device.
__device__ __forceinline__ float div_rn(float w, float s, float rs)
{
    const float t = w * rs;
    return fmaf(fmaf(-t, s, w), rs, t);
}

// Operands of the quotient w / s for one group.  The correction above needs
// the residual w - t s exactly and a finite RN(1 / s); both hold while s and
// the residual stay clear of the subnormal range, i.e. for s >= 2^-100 (the
// residual's lowest bit is at least 2^-47 s when |w / s| >= 1/2, where the
// rounding is decided).  A group whose range is that tiny (1 / s overflows
// below 2^-128) has its scale and every quotient numerator lifted by 2^100:
// multiplying both by a power of two is exact and leaves w / s unchanged.
struct QuotOp {
    float f;    // 1 or 2^100
    float s;    // s * f
    float rs;   // RN(1 / (s * f))
};

__device__ __forceinline__ QuotOp quot_op(float s)
{
    const float f = s < 0x1p-60f ? 0x1p100f : 1.f;
    const float sf = s * f;
    return {f, sf, 1.f / sf};
}

__device__ __forceinline__ float quot(float w, const QuotOp& o) { return div_rn(w * o.f, o.s, o.rs); }

// Scale and zero of the group starting at in-block column c, from one row's
// current values: each part reduces its registers whose column lies in
// [c, c + gs) and below bw, then the QTPR parts of the row pair combine.
__device__ __forceinline__ void group_range(const float (&w)[QCPT], int part, int c, int gs, int bw,
                                            float& mn, float& mx)
{
    mn = 0.f;
    mx = 0.f;
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
}

__device__ __forceinline__ void group_grid(const float (&w)[QCPT], int part, int c, int gs, int bw,
                                           float maxq, float& s, float& z)
{
    float mn, mx;
    group_range(w, part, c, gs, bw, mn, mx);
    grid_from_range(mn, mx, maxq, s, z);
}

// Q4_K (torchao pull request "Add gguf q4_k quantization": w = q * block_scale
// + block_min, 6-bit block scales and mins under a super-block scale): the
// raw scale and offset of a 32-column block from its range (an all-zero
// range taking [-1, 1]).
__device__ __forceinline__ void q4k_raw(float mn, float mx, float& scale, float& off)
{
    if (mn == mx) {
        mn = -1.f;
        mx = 1.f;
    }
    scale = __fdiv_rn(mx - mn, 15.f);
    off = -mn;
}

// The block's 6-bit scale and min against the super-block's d and dmin, and
// the grid they give: w^ = s q - o, s = d sc, o = dmin m.
__device__ __forceinline__ void q4k_block_grid(float mn, float mx, float d, float dmin, float& s,
                                               float& o, float& sc, float& m)
{
    float scale, off;
    q4k_raw(mn, mx, scale, off);
    sc = fminf(fmaxf(rintf(__fdiv_rn(scale, d)), 1.f), 63.f);
    m = dmin > 0.f ? fminf(fmaxf(rintf(__fdiv_rn(off, dmin)), 0.f), 63.f) : 0.f;
    s = d * sc;
    o = dmin * m;
}

// One lazy-batch block [j0, j0 + bw) of the column loop for QROWS rows.
// Per column c every lane of a row pair knows both rows' current values
// through `nxt` (column c+1 fetched one step early with a shuffle from its
// owner and corrected by this step's error), computes the same q and e, and
// corrects its own registers with U row c.  Columns at and before c have
// coefficient 0 in the laid-out U rows, so the registers are updated whole
// and stay compile-time indexed.  Lane part p keeps the results of steps 2p
// and 2p+1 of a sub-block and writes them (e, w^, codes) with one vector
// store each when the sub-block ends.
// kGroupsInStep: a group may start inside a 16-column sub-block (group sizes
// that are not multiples of 16); otherwise groups start at sub-block starts
// and w^ is formed from the code at the store.
template <bool kGroupsInStep, bool kQ4K>
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
    // Under a programmatic dependent launch everything above (the U block is
    // laid out before the first block's launch) overlaps the previous kernel,
    // the lazy-batch product that corrects this block's columns; W is read
    // only after it completes.  The next product may start its set-up now.
    pdl_wait();
    pdl_trigger();
    if (a.stamp && tid == 0) atomicMin(a.stamp, globaltimer_ns());

    const int pair = tid / QTPR, part = tid % QTPR;
    const int lane = tid & 31;
    const int lane_base = lane & ~(QTPR - 1);
    const float maxq = static_cast<float>((1 << a.bits) - 1);
    int r[2];
    bool valid[2];
    int64_t rowoff[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        r[h] = blockIdx.x * QROWS + 2 * pair + h;
        valid[h] = r[h] < a.d_out;
        rowoff[h] = static_cast<int64_t>(valid[h] ? r[h] : 0) * d_in;
    }

    float w[2][QCPT];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < QCPT / 4; ++m) {
            const int col = QCPT * part + 4 * m;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (valid[h] && col < bw) v = *reinterpret_cast<const float4*>(a.Wp + rowoff[h] + j0 + col);
            w[h][4 * m] = v.x;
            w[h][4 * m + 1] = v.y;
            w[h][4 * m + 2] = v.z;
            w[h][4 * m + 3] = v.w;
        }

    // grid of the group in effect at the block start
    float s[2] = {1.f, 1.f}, z[2] = {0.f, 0.f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (a.gs < 0) {
            if (valid[h]) {
                s[h] = a.scales[r[h]];
                z[h] = a.zeros[r[h]];
            }
        } else if (a.gs > a.block) {
            const int g = j0 / a.gs;
            if (j0 % a.gs == 0) {
                float mn = 0.f, mx = 0.f;
                for (int k = part; k < a.gs; k += QTPR) {
                    const float v = valid[h] ? a.Wp[rowoff[h] + j0 + k] : 0.f;
                    mn = fminf(mn, v);
                    mx = fmaxf(mx, v);
                }
#pragma unroll
                for (int o = 1; o < QTPR; o <<= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                }
                grid_from_range(mn, mx, maxq, s[h], z[h]);
                if (valid[h] && part == 0) {
                    a.scales[static_cast<int64_t>(r[h]) * a.n_groups + g] = s[h];
                    a.zeros[static_cast<int64_t>(r[h]) * a.n_groups + g] = z[h];
                }
            } else if (valid[h]) {
                s[h] = a.scales[static_cast<int64_t>(r[h]) * a.n_groups + g];
                z[h] = a.zeros[static_cast<int64_t>(r[h]) * a.n_groups + g];
            }
        }
    }
    // Q4_K super-block scales: at a super-block's first block from the current
    // values of its 256 columns (this block's in registers, the next block's
    // in the working copy, already corrected by every earlier block), else
    // those the first block stored.  Part p holds columns 16p .. 16p + 15 of
    // a block, i.e. half of 32-column block p / 2.
    float qd[2] = {1.f, 1.f}, qdm[2] = {0.f, 0.f};
    if (kQ4K) {
        const int64_t sidx = j0 / 256;
        const int ns = d_in / 256;
        if (j0 % 256 == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float smax = 0.f, omax = 0.f;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[QCPT];
                    if (half == 0) {
#pragma unroll
                        for (int k = 0; k < QCPT; ++k) v[k] = w[h][k];
                    } else {
#pragma unroll
                        for (int m4 = 0; m4 < QCPT / 4; ++m4) {
                            float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (valid[h])
                                t4 = *reinterpret_cast<const float4*>(a.Wp + rowoff[h] + j0 + a.block +
                                                                      QCPT * part + 4 * m4);
                            v[4 * m4] = t4.x;
                            v[4 * m4 + 1] = t4.y;
                            v[4 * m4 + 2] = t4.z;
                            v[4 * m4 + 3] = t4.w;
                        }
                    }
                    float mn = 0.f, mx = 0.f;
#pragma unroll
                    for (int k = 0; k < QCPT; ++k) {
                        mn = fminf(mn, v[k]);
                        mx = fmaxf(mx, v[k]);
                    }
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));   // the block's other half
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    float scale, off;
                    q4k_raw(mn, mx, scale, off);
                    smax = fmaxf(smax, scale);
                    omax = fmaxf(omax, off);
                }
#pragma unroll
                for (int o = 2; o < QTPR; o <<= 1) {
                    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
                    omax = fmaxf(omax, __shfl_xor_sync(0xffffffffu, omax, o));
                }
                qd[h] = __fdiv_rn(smax, 63.f);
                qdm[h] = __fdiv_rn(omax, 63.f);
                if (valid[h] && part == 0) {
                    a.dsup[static_cast<int64_t>(r[h]) * ns + sidx] = qd[h];
                    a.dmin[static_cast<int64_t>(r[h]) * ns + sidx] = qdm[h];
                }
            }
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (valid[h]) {
                    qd[h] = a.dsup[static_cast<int64_t>(r[h]) * ns + sidx];
                    qdm[h] = a.dmin[static_cast<int64_t>(r[h]) * ns + sidx];
                }
        }
    }
    QuotOp qo[2] = {quot_op(s[0]), quot_op(s[1])};
    const int gs_in = (a.gs > 0 && a.gs <= a.block) ? a.gs : 0;
    int next_group = gs_in ? 0 : 1 << 30;

    float errsum[2] = {0.f, 0.f};
    float nxt[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) nxt[h] = __shfl_sync(0xffffffffu, w[h][0], lane_base);   // column 0

#pragma unroll 1
    for (int S = 0; S < nsub; ++S) {
        const bool got = mbar_wait_bounded(&bars[S], 0, abort_flag, a.status);
        if (!__syncthreads_and(got)) break;
        const float* ub = Ut + S * UCH_FLOATS;
        const float2* pairs = reinterpret_cast<const float2*>(ub + QSUB * UT_LD);
        const int src_in = lane_base | S;                          // owner of this sub-block
        const int src_next = lane_base | min(S + 1, QTPR - 1);     // owner of the next one
        const int cbase = S * QSUB;
        if (!kGroupsInStep && cbase == next_group) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float qsc = 0.f, qm = 0.f;
                if (kQ4K) {   // z holds the block's offset o
                    float mn, mx;
                    group_range(w[h], part, cbase, gs_in, bw, mn, mx);
                    q4k_block_grid(mn, mx, qd[h], qdm[h], s[h], z[h], qsc, qm);
                } else {
                    group_grid(w[h], part, cbase, gs_in, bw, maxq, s[h], z[h]);
                }
                qo[h] = quot_op(s[h]);
                if (valid[h] && part == 0) {
                    const int g = (j0 + cbase) / gs_in;
                    a.scales[static_cast<int64_t>(r[h]) * a.n_groups + g] = s[h];
                    a.zeros[static_cast<int64_t>(r[h]) * a.n_groups + g] = z[h];
                    if (kQ4K) {
                        a.sc6[static_cast<int64_t>(r[h]) * a.n_groups + g] = static_cast<uint8_t>(qsc);
                        a.m6[static_cast<int64_t>(r[h]) * a.n_groups + g] = static_cast<uint8_t>(qm);
                    }
                }
            }
            next_group += gs_in;
        }
        float ke[2][2], kq[2][2], kw[2][2];   // results of steps 2*part, 2*part + 1
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
            // column c+1 of both rows after the corrections of steps < c
            float pre[2];
#pragma unroll
            for (int h = 0; h < 2; ++h)
                pre[h] = __shfl_sync(0xffffffffu, w[h][(cl + 1) % QCPT], cl + 1 < QSUB ? src_in : src_next);
            if (kGroupsInStep && c == next_group && c < bw) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    group_grid(w[h], part, c, gs_in, bw, maxq, s[h], z[h]);
                    qo[h] = quot_op(s[h]);
                    if (valid[h] && part == 0) {
                        const int g = (j0 + c) / gs_in;
                        a.scales[static_cast<int64_t>(r[h]) * a.n_groups + g] = s[h];
                        a.zeros[static_cast<int64_t>(r[h]) * a.n_groups + g] = z[h];
                    }
                }
                next_group += gs_in;
            }
            const bool keep = part == cl / 2;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float wc = nxt[h];
                // q = clamp(rint(w / s) + z, 0, maxq) and w^ = s (q - z); with
                // integer-valued floats, q - z = clamp(rint(w / s), -z, maxq - z)
                float q, what;
                if (kQ4K) {   // q = clamp(rint((w + o) / s), 0, 15), w^ = s q - o
                    q = fminf(fmaxf(rintf(quot(wc + z[h], qo[h])), 0.f), 15.f);
                    what = fmaf(s[h], q, -z[h]);
                } else {
                    const float qz = fminf(fmaxf(rintf(quot(wc, qo[h])), -z[h]), maxq - z[h]);
                    q = qz + z[h];
                    what = s[h] * qz;
                }
                const float e = (wc - what) * rn.x;
                nxt[h] = fmaf(-e, rn.y, pre[h]);
                errsum[h] = fmaf(e, e, errsum[h]);
                if (keep) {
                    ke[h][cl % 2] = e;
                    kq[h][cl % 2] = q;
                    if (kGroupsInStep) kw[h][cl % 2] = what;
                }
                // the row's 16 columns, two per instruction (each lane of the
                // pair is fmaf(-e, u, w): the same bits as the scalar form)
                const float2 ne = make_float2(-e, -e);
#pragma unroll
                for (int k = 0; k < QCPT; k += 2) {
                    const float2 r2 = __ffma2_rn(ne, make_float2(u[k], u[k + 1]), make_float2(w[h][k], w[h][k + 1]));
                    w[h][k] = r2.x;
                    w[h][k + 1] = r2.y;
                }
            }
        }
        // this lane's two columns of the sub-block: e, w^ and the codes
        const int col = cbase + 2 * part;
        if (col < bw) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (!valid[h]) continue;
                if (!kGroupsInStep) {
                    if (kQ4K) {
                        kw[h][0] = fmaf(s[h], kq[h][0], -z[h]);
                        kw[h][1] = fmaf(s[h], kq[h][1], -z[h]);
                    } else {
                        kw[h][0] = s[h] * (kq[h][0] - z[h]);
                        kw[h][1] = s[h] * (kq[h][1] - z[h]);
                    }
                }
                const int64_t eo = static_cast<int64_t>(r[h]) * kOuterMax + a.e_off + col;
                *reinterpret_cast<float2*>(a.E + eo) = make_float2(ke[h][0], ke[h][1]);
                if (a.E_lo)
                    *reinterpret_cast<float2*>(a.E_lo + eo) = make_float2(tf32_low(ke[h][0]), tf32_low(ke[h][1]));
                *reinterpret_cast<float2*>(a.Wp + rowoff[h] + j0 + col) = make_float2(kw[h][0], kw[h][1]);
                const uint32_t q2 = static_cast<uint32_t>(kq[h][0]) | (static_cast<uint32_t>(kq[h][1]) << 8);
                *reinterpret_cast<uint16_t*>(a.codes_p + rowoff[h] + j0 + col) = static_cast<uint16_t>(q2);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
        if (valid[h] && a.err_sq && part == 0) a.err_sq[r[h]] += errsum[h];
    if (a.stamp) {
        __syncthreads();
        if (tid == 0) atomicMax(a.stamp + 1, globaltimer_ns());
    }
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

// inv[perm[k]] = k, with a range check of perm (inv starts as all -1, so a
// column that no entry of perm names stays -1 and finish_kernel reports it).
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

// Row-staged forms of the two column gathers of the act_order path, for rows
// of at most kRowStageMax columns: a CTA reads a whole row with coalesced
// 16-byte loads into shared memory, then writes the permuted row in order, so
// the scattered reads hit shared memory instead of pulling a 32-byte sector
// from L2 for every 4 useful bytes.
constexpr int kRowStageMax = 16384;
constexpr int kRowThreads = 512;

// Wp[r][k] = W[r][perm[k]]
__global__ void __launch_bounds__(kRowThreads)
    gather_cols_rows_kernel(const float* __restrict__ W, int d_out, int d_in,
                            const int32_t* __restrict__ perm, float* __restrict__ Wp)
{
    extern __shared__ __align__(16) float row[];
    for (int r = blockIdx.x; r < d_out; r += gridDim.x) {
        const float4* src = reinterpret_cast<const float4*>(W + static_cast<int64_t>(r) * d_in);
        __syncthreads();   // the previous row has been written out
        for (int i = threadIdx.x; i < d_in / 4; i += blockDim.x) reinterpret_cast<float4*>(row)[i] = src[i];
        __syncthreads();
        float* dst = Wp + static_cast<int64_t>(r) * d_in;
        for (int k = threadIdx.x; k < d_in; k += blockDim.x) {
            int p = perm[k];
            p = (p < 0 || p >= d_in) ? 0 : p;
            dst[k] = row[p];
        }
    }
}

// finish_kernel's work for a permuted layer, one staged row (W^ and codes in
// processing order) at a time: W^, codes and packed nibbles in original order.
__global__ void __launch_bounds__(kRowThreads)
    finish_rows_kernel(const uint8_t* __restrict__ codes_p, const float* __restrict__ Wp,
                       const int32_t* __restrict__ inv, int d_out, int d_in, float* __restrict__ W,
                       uint8_t* __restrict__ codes, uint8_t* __restrict__ packed, int* status)
{
    extern __shared__ __align__(16) float wrow[];
    uint8_t* crow = reinterpret_cast<uint8_t*>(wrow + d_in);
    const int half = d_in / 2;
    for (int r = blockIdx.x; r < d_out; r += gridDim.x) {
        const int64_t ro = static_cast<int64_t>(r) * d_in;
        __syncthreads();   // the previous row has been written out
        for (int i = threadIdx.x; i < d_in / 4; i += blockDim.x)
            reinterpret_cast<float4*>(wrow)[i] = reinterpret_cast<const float4*>(Wp + ro)[i];
        for (int i = threadIdx.x; i < d_in / 8; i += blockDim.x)
            reinterpret_cast<uint2*>(crow)[i] = reinterpret_cast<const uint2*>(codes_p + ro)[i];
        __syncthreads();
        for (int i = threadIdx.x; i < half; i += blockDim.x) {
            int k0 = inv[2 * i], k1 = inv[2 * i + 1];
            if (k0 < 0 || k0 >= d_in || k1 < 0 || k1 >= d_in) {   // a malformed permutation
                if (r == 0) record_status(status, GPTQ_ERR_INVALID_ARG);
                k0 = (k0 < 0 || k0 >= d_in) ? 0 : k0;
                k1 = (k1 < 0 || k1 >= d_in) ? 0 : k1;
            }
            const uint8_t q0 = crow[k0], q1 = crow[k1];
            if (codes) {   // byte stores: the caller's codes buffer has no alignment rule
                codes[ro + 2 * i] = q0;
                codes[ro + 2 * i + 1] = q1;
            }
            if (packed) packed[static_cast<int64_t>(r) * half + i] = static_cast<uint8_t>((q0 & 15) | ((q1 & 15) << 4));
            *reinterpret_cast<float2*>(W + ro + 2 * i) = make_float2(wrow[k0], wrow[k1]);
        }
    }
}

// Original-order outputs: codes, packed nibbles, and (with a permutation) W^.
// One thread per pair of original columns (2i, 2i+1).  A column missing from
// the permutation (perm not a bijection) records GPTQ_ERR_INVALID_ARG; its
// outputs are then unspecified, but every access stays in bounds.
__global__ void finish_kernel(const uint8_t* __restrict__ codes_p, const float* __restrict__ Wp,
                              const int32_t* __restrict__ inv, int d_out, int d_in,
                              float* __restrict__ W, uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ packed, int* status)
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
        if (k0 < 0 || k0 >= d_in || k1 < 0 || k1 >= d_in) {   // a malformed permutation
            if (r == 0) record_status(status, GPTQ_ERR_INVALID_ARG);
            k0 = (k0 < 0 || k0 >= d_in) ? 0 : k0;
            k1 = (k1 < 0 || k1 >= d_in) ? 0 : k1;
        }
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

// finish_kernel's work for a layer without a permutation (W^ is already in
// place), 8 columns per thread with 8-byte loads of the codes and 8- and
// 4-byte stores; the caller's codes and packed buffers must be 8- and 4-byte
// aligned (checked on the host).
__global__ void finish_noperm_kernel(const uint8_t* __restrict__ codes_p, int d_out, int d_in,
                                     uint8_t* __restrict__ codes, uint8_t* __restrict__ packed)
{
    const int per_row = d_in / 8;
    const int64_t n = static_cast<int64_t>(d_out) * per_row;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = idx / per_row;
        const int g = static_cast<int>(idx - r * per_row);
        const int64_t off = r * d_in + 8 * g;
        const uint2 q = *reinterpret_cast<const uint2*>(codes_p + off);
        if (codes) *reinterpret_cast<uint2*>(codes + off) = q;
        if (packed) {
            // bytes b0..b7 of q -> nibbles: byte k of the result = b(2k) | b(2k+1) << 4
            const uint32_t lo = q.x, hi = q.y;
            const uint32_t p0 = (lo & 0x0F) | ((lo >> 4) & 0xF0);                 // bytes 0, 1
            const uint32_t p1 = ((lo >> 16) & 0x0F) | ((lo >> 20) & 0xF0);        // bytes 2, 3
            const uint32_t p2 = (hi & 0x0F) | ((hi >> 4) & 0xF0);
            const uint32_t p3 = ((hi >> 16) & 0x0F) | ((hi >> 20) & 0xF0);
            *reinterpret_cast<uint32_t*>(packed + r * (d_in / 2) + 4 * g) = p0 | (p1 << 8) | (p2 << 16) | (p3 << 24);
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

// Counter-based test operands (splitmix64 finaliser) for the quotient check.
__device__ __forceinline__ uint32_t st_mix(uint64_t x)
{
    x ^= x >> 33;
    x *= 0xff51afd7ed558ccdULL;
    x ^= x >> 33;
    x *= 0xc4ceb9fe1a85ec53ULL;
    x ^= x >> 33;
    return static_cast<uint32_t>(x);
}

__device__ __forceinline__ float st_unif(uint64_t k) { return (st_mix(k) >> 8) * (1.0f / 16777216.0f); }

__device__ unsigned long long g_quotient_bad;   // mismatch count of the self-test

// The column loop's quotient (quot after quot_op) against IEEE division on
// four operand families: s log-uniform in [2^-40, 2^20] with |w / s| < 2^12,
// s with an all-ones significand, w within 4 ulps of (n + 1/2) s (quotients
// next to a rounding tie of rint), and tiny scales, s log-uniform in
// [2^-149, 2^-60] (subnormals included) with w within 4 ulps of (n + 1/2) s.
__global__ void quotient_selftest_kernel(uint64_t seed, int64_t n, unsigned long long* bad)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    unsigned long long local = 0;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
        const uint64_t k = (seed << 40) ^ (4 * static_cast<uint64_t>(i));
        const int mode = static_cast<int>(i % 4);
        float s, w;
        if (mode == 0) {
            s = exp2f(-40.f + 60.f * st_unif(k));
            w = s * (st_unif(k + 1) * 8192.f - 4096.f);
        } else if (mode == 1) {
            const int e = static_cast<int>(st_mix(k) % 60) - 40;
            const uint32_t m = 0x7FFFFFu - (st_mix(k + 2) & 7u);
            s = __uint_as_float((static_cast<uint32_t>(e + 127) << 23) | m);
            w = s * (st_unif(k + 1) * 600.f - 300.f);
        } else {
            s = mode == 2 ? exp2f(-20.f + 24.f * st_unif(k)) : exp2f(-149.f + 89.f * st_unif(k));
            const float m = floorf(st_unif(k + 1) * 600.f - 300.f);
            const float w0 = (m + 0.5f) * s;
            w = __uint_as_float(__float_as_uint(w0) + static_cast<int>(st_mix(k + 3) % 9) - 4);
        }
        // skip an ulp step below a zero numerator's bit pattern, and a scale
        // that came out as zero
        if (!isfinite(w) || !(s > 0.f)) continue;
        if (quot(w, quot_op(s)) != __fdiv_rn(w, s)) ++local;
    }
    if (local) atomicAdd(bad, local);
}

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

// Sub-block chunks of the U layout for any block width 8..128: each block of
// width bw has ceil(bw / 16) <= bw / 8 chunks, plus one for a ragged last block.
inline size_t u_layout_bytes(int64_t d_in)
{
    return static_cast<size_t>(d_in / 8 + 16) * UCH_BYTES;
}

// Workspace of the column loop, in this order: working weights Wp (d_out x d_in
// f32), codes (d_out x d_in u8), errors E (d_out x 1024 f32), the inverse
// permutation (d_in i32), the U block layout -- the minimum -- then the tf32
// low parts of E (d_out x 1024 f32) and of U (d_in x d_in f32).  With the low
// parts present the lazy-batch products skip their conversion pass.
size_t quantize_workspace_min_bytes(int64_t d_out, int64_t d_in)
{
    const size_t n = static_cast<size_t>(d_out) * static_cast<size_t>(d_in);
    return 256 + up256(n * sizeof(float)) + up256(n) +
           up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float)) +
           up256(static_cast<size_t>(d_in) * sizeof(int32_t)) + up256(u_layout_bytes(d_in));
}

size_t quantize_workspace_bytes(int64_t d_out, int64_t d_in)
{
    return quantize_workspace_min_bytes(d_out, d_in) +
           up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float)) +
           up256(static_cast<size_t>(d_in) * static_cast<size_t>(d_in) * sizeof(float));
}

// Timing of one enqueue (the diagnostic entry point): the column-loop
// kernels and the tensor-core lazy-batch products record their spans in a
// static device array, one pair of words per launch, tagged on the host with
// the launch's class (1 = column loop, 2 = lazy-batch product).  The launch
// sequence is the production one (programmatic dependent launches included).
constexpr int kMaxStamped = 8192;
__device__ unsigned long long g_stamps[2 * kMaxStamped];

__global__ void stamps_init_kernel(unsigned long long* st, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        st[2 * i] = ~0ull;
        st[2 * i + 1] = 0ull;
    }
}

struct QuantizeMarks {   // the launches of one timed enqueue and their span slots
    unsigned long long* stamps = nullptr;   // g_stamps
    std::vector<int> cls;
    unsigned long long* slot(int c)
    {
        if (cls.size() >= static_cast<size_t>(kMaxStamped)) return nullptr;
        cls.push_back(c);
        return stamps + 2 * (cls.size() - 1);
    }
};

static int enqueue_quantize(float* W, const float* U, const int32_t* perm, int64_t d_out64,
                            int64_t d_in64, int bits, int gs, int block, uint8_t* codes,
                            float* scales, float* zeros, uint8_t* packed, int32_t* g_idx,
                            float* err_sq, void* workspace, bool with_low_parts, cudaStream_t stream,
                            QuantizeMarks* marks = nullptr, const Q4KOut* q4k = nullptr)
{
    auto slot = [&](int c) { return marks ? marks->slot(c) : nullptr; };
    // The column-loop kernels and the lazy-batch products alternate on the
    // stream as programmatic dependent launches, each one's set-up overlapping
    // the previous one's tail.
    const bool pdl = true;
    const int d_out = static_cast<int>(d_out64), d_in = static_cast<int>(d_in64);
    const size_t n = static_cast<size_t>(d_out) * d_in;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* Wp = reinterpret_cast<float*>(ws + 256);
    uint8_t* codes_p = ws + 256 + up256(n * sizeof(float));
    const size_t e_bytes = up256(static_cast<size_t>(d_out) * kOuterMax * sizeof(float));
    float* E = reinterpret_cast<float*>(ws + 256 + up256(n * sizeof(float)) + up256(n));
    int32_t* inv = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(E) + e_bytes);
    float* Ul = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(inv) +
                                         up256(static_cast<size_t>(d_in) * sizeof(int32_t)));
    float* E_lo = nullptr;
    float* U_lo = nullptr;
    if (with_low_parts) {
        E_lo = reinterpret_cast<float*>(ws + quantize_workspace_min_bytes(d_out, d_in));
        U_lo = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(E_lo) + e_bytes);
    }
    const int nsm = sm_count();
    int* status = device_status_ptr();
    const int n_groups = gs > 0 ? d_in / gs : 1;

    static bool attr_set[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel<false, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmemLaunch)));
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel<true, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmemLaunch)));
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gptq_block_kernel<false, true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kBlockSmemLaunch)));
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gather_cols_rows_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRowStageMax * static_cast<int>(sizeof(float))));
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(finish_rows_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kRowStageMax * static_cast<int>(sizeof(float) + 1)));
        attr_set[dev] = true;
    }
    // groups start only at 16-column sub-block starts when group_size is a
    // multiple of 16 that fits the block (or there are no in-block groups)
    const bool groups_in_step = gs > 0 && gs <= block && (gs % QSUB) != 0;

    const int nch_blk = (block + QSUB - 1) / QSUB;
    const int n_blocks = (d_in + block - 1) / block;
    u_layout_kernel<<<n_blocks * nch_blk, 256, 0, stream>>>(U, d_in, block, nch_blk, Ul);
    GPTQ_LAUNCH_CHECK();
    if (with_low_parts) {
        u_low_kernel<<<nsm * 8, 256, 0, stream>>>(U, d_in, U_lo);
        GPTQ_LAUNCH_CHECK();
    }

    float* work = W;
    if (perm) {
        GPTQ_CUDA_CHECK(cudaMemsetAsync(inv, 0xFF, static_cast<size_t>(d_in) * sizeof(int32_t), stream));
        invert_perm_kernel<<<(d_in + 255) / 256, 256, 0, stream>>>(perm, d_in, inv, status);
        GPTQ_LAUNCH_CHECK();
        if (d_in <= kRowStageMax)
            gather_cols_rows_kernel<<<std::min(d_out, 2 * nsm), kRowThreads,
                                      static_cast<size_t>(d_in) * sizeof(float), stream>>>(W, d_out, d_in,
                                                                                          perm, Wp);
        else
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
    // one CTA per SM while the grid fits on the SMs at once; beyond that two
    // per SM (more warps to hide each other's step latency in every wave)
    const size_t block_smem = grid <= nsm ? kBlockSmemLaunch : kBlockSmem;
    for (int J0 = 0; J0 < d_in; J0 += outer) {
        const int J1 = (d_in - J0 < outer) ? d_in : J0 + outer;
        for (int j0 = J0; j0 < J1; j0 += block) {
            const int bw = (J1 - j0 < block) ? J1 - j0 : block;
            QArgs a{work, Ul, d_out, d_in, j0, bw, block, bits, gs, n_groups, scales, zeros,
                    codes_p, E, E_lo, j0 - J0, err_sq, status,
                    q4k ? q4k->sc6 : nullptr, q4k ? q4k->m6 : nullptr,
                    q4k ? q4k->dsup : nullptr, q4k ? q4k->dmin : nullptr, slot(1)};
            auto kern = q4k ? gptq_block_kernel<false, true>
                            : (groups_in_step ? gptq_block_kernel<true, false> : gptq_block_kernel<false, false>);
            GPTQ_CUDA_CHECK(launch_k(kern, dim3(grid), dim3(QTHREADS), block_smem, stream, pdl, a));
            GPTQ_LAUNCH_CHECK();
            const int rest_in = J1 - j0 - bw;
            if (rest_in > 0) {
                const int64_t uo = static_cast<int64_t>(j0) * d_in + j0 + bw;
                int rc = launch_sgemm(false, d_out, rest_in, bw, -1.f, E + (j0 - J0), kOuterMax, 0,
                                      U + uo, d_in, 0, 1.f, work + j0 + bw, d_in, 0, 1, 0, stream, 0,
                                      E_lo ? E_lo + (j0 - J0) : nullptr, U_lo ? U_lo + uo : nullptr,
                                      pdl, slot(2));
                if (rc) return rc;
            }
        }
        const int rest = d_in - J1;
        if (rest > 0) {
            const int64_t uo = static_cast<int64_t>(J0) * d_in + J1;
            int rc = launch_sgemm(false, d_out, rest, J1 - J0, -1.f, E, kOuterMax, 0, U + uo, d_in, 0,
                                  1.f, work + J1, d_in, 0, 1, 0, stream, 0, E_lo,
                                  U_lo ? U_lo + uo : nullptr, pdl, slot(2));
            if (rc) return rc;
        }
    }
    if (codes || packed || perm) {
        const bool vec_ok = (reinterpret_cast<uintptr_t>(codes) % 8 == 0) &&
                            (reinterpret_cast<uintptr_t>(packed) % 4 == 0);
        if (perm && d_in <= kRowStageMax)
            finish_rows_kernel<<<std::min(d_out, 2 * nsm), kRowThreads,
                                 static_cast<size_t>(d_in) * (sizeof(float) + 1), stream>>>(
                codes_p, Wp, inv, d_out, d_in, W, codes, packed, status);
        else if (!perm && vec_ok)
            finish_noperm_kernel<<<nsm * 8, 256, 0, stream>>>(codes_p, d_out, d_in, codes, packed);
        else
            finish_kernel<<<nsm * 8, 256, 0, stream>>>(codes_p, Wp, perm ? inv : nullptr, d_out, d_in,
                                                       W, codes, packed, status);
        GPTQ_LAUNCH_CHECK();
    }
    if (g_idx) {
        g_idx_kernel<<<(d_in + 255) / 256, 256, 0, stream>>>(perm, d_in, gs, g_idx);
        GPTQ_LAUNCH_CHECK();
    }
    return GPTQ_OK;
}

int run_quantize(float* W, const float* U, const int32_t* perm, int64_t d_out, int64_t d_in, int bits,
                 int gs, int block, uint8_t* codes, float* scales, float* zeros, uint8_t* packed,
                 int32_t* g_idx, float* err_sq, void* workspace, size_t ws_bytes, cudaStream_t stream,
                 bool graphed, const Q4KOut* q4k)
{
    const bool low = ws_bytes >= quantize_workspace_bytes(d_out, d_in);
    auto enq = [&](cudaStream_t s, int*) {
        return enqueue_quantize(W, U, perm, d_out, d_in, bits, gs, block, codes, scales, zeros,
                                packed, g_idx, err_sq, workspace, low, s, nullptr, q4k);
    };
    if (!graphed) return enq(stream, nullptr);
    auto P = [](const void* p) { return static_cast<uint64_t>(reinterpret_cast<uintptr_t>(p)); };
    const std::vector<uint64_t> key = {2, P(W), P(U), P(perm), static_cast<uint64_t>(d_out),
                                       static_cast<uint64_t>(d_in), static_cast<uint64_t>(bits),
                                       static_cast<uint64_t>(static_cast<int64_t>(gs)),
                                       static_cast<uint64_t>(block), P(codes), P(scales), P(zeros),
                                       P(packed), P(g_idx), P(err_sq), P(workspace),
                                       static_cast<uint64_t>(low), P(q4k ? q4k->sc6 : nullptr),
                                       P(q4k ? q4k->m6 : nullptr), P(q4k ? q4k->dsup : nullptr),
                                       P(q4k ? q4k->dmin : nullptr)};
    return run_graphed(key, false, enq, stream, nullptr);
}

int run_quantize_timed(float* W, const float* U, const int32_t* perm, int64_t d_out, int64_t d_in,
                       int bits, int gs, int block, uint8_t* codes, float* scales, float* zeros,
                       uint8_t* packed, int32_t* g_idx, float* err_sq, void* workspace,
                       size_t ws_bytes, cudaStream_t stream, float* ms_by_class)
{
    static std::mutex mu;   // one timed call at a time: they share g_stamps
    std::lock_guard<std::mutex> lk(mu);
    QuantizeMarks marks;
    void* p = nullptr;
    GPTQ_CUDA_CHECK(cudaGetSymbolAddress(&p, g_stamps));
    marks.stamps = static_cast<unsigned long long*>(p);
    stamps_init_kernel<<<(kMaxStamped + 255) / 256, 256, 0, stream>>>(marks.stamps, kMaxStamped);
    GPTQ_LAUNCH_CHECK();
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    GPTQ_CUDA_CHECK(cudaEventCreate(&e0));
    GPTQ_CUDA_CHECK(cudaEventCreate(&e1));
    const bool low = ws_bytes >= quantize_workspace_bytes(d_out, d_in);
    int rc = GPTQ_OK;
    if (cudaEventRecord(e0, stream) != cudaSuccess) rc = cuda_fail(cudaGetLastError());
    if (!rc)
        rc = enqueue_quantize(W, U, perm, d_out, d_in, bits, gs, block, codes, scales, zeros, packed,
                              g_idx, err_sq, workspace, low, stream, &marks);
    if (!rc && cudaEventRecord(e1, stream) != cudaSuccess) rc = cuda_fail(cudaGetLastError());
    if (!rc && cudaStreamSynchronize(stream) != cudaSuccess) rc = cuda_fail(cudaGetLastError());
    float total = 0.f;
    if (!rc && cudaEventElapsedTime(&total, e0, e1) != cudaSuccess) rc = cuda_fail(cudaGetLastError());
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (rc) return rc;
    std::vector<unsigned long long> h(2 * marks.cls.size());
    if (!h.empty())
        GPTQ_CUDA_CHECK(cudaMemcpyFromSymbol(h.data(), g_stamps, h.size() * sizeof(unsigned long long)));
    double by[3] = {0.0, 0.0, 0.0};
    for (size_t i = 0; i < marks.cls.size(); ++i)
        if (h[2 * i] != ~0ull && h[2 * i + 1] > h[2 * i]) by[marks.cls[i]] += 1e-6 * (h[2 * i + 1] - h[2 * i]);
    ms_by_class[1] = static_cast<float>(by[1]);
    ms_by_class[2] = static_cast<float>(by[2]);
    ms_by_class[0] = std::max(0.f, total - ms_by_class[1] - ms_by_class[2]);
    return GPTQ_OK;
}

int run_quotient_selftest(int64_t n, uint64_t seed, int64_t* mismatches)
{
    void* p = nullptr;
    GPTQ_CUDA_CHECK(cudaGetSymbolAddress(&p, g_quotient_bad));
    unsigned long long* d = static_cast<unsigned long long*>(p);
    GPTQ_CUDA_CHECK(cudaMemset(d, 0, sizeof(unsigned long long)));
    quotient_selftest_kernel<<<sm_count() * 8, 256>>>(seed, n, d);
    GPTQ_LAUNCH_CHECK();
    unsigned long long h = 0;
    GPTQ_CUDA_CHECK(cudaMemcpy(&h, d, sizeof h, cudaMemcpyDeviceToHost));
    *mismatches = static_cast<int64_t>(h);
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
