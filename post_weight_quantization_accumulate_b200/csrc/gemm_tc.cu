// gemm_tc.cu -- fp32-accurate matrix product on the sm_100a tensor cores.
//
// C = alpha * A * B + beta * C with float32 operands, computed as three
// tcgen05 kind::tf32 products (3xTF32): the tensor core reads a float32
// operand as tf32 by dropping its 13 low mantissa bits, so with hi = x as
// stored and lo = x - trunc_tf32(x) (exact)
//     A B ~= A_hi B_hi + A_hi B_lo + A_lo B_hi
// keeps about 2^-21 relative error per product, close to float32 (measured
// 1e-6 relative on K = 128 against float64).
//
// Used for the lazy-batch update of the column loop (W[:, j+B:] -= E U_blk),
// the trailing update of the blocked Cholesky (A22 -= L21 L21^T) and the
// accumulation of the factor's inverse.
//
// Two variants, persistent over output tiles x batch, 384 threads per CTA:
//  * 128 x 128 tiles, low parts formed in shared memory (three 64 KB stages:
//    A_hi, A_lo, B_hi, B_lo of 16 KB) -- for operands produced on the fly;
//  * 128 x 256 tiles with the low parts supplied by the caller as two more
//    matrices (two 96 KB stages) -- no conversion pass, and N = 256 MMAs read
//    A once per 256 columns: a third less shared-memory traffic per flop.
// Roles:
//   warp 0       TMA producer: fp32 tiles of A (K-major) and B (MN- or K-major)
//   warp 1       MMA issuer + TMEM owner (two fp32 accumulators of TN columns)
//   warps 4-7    converters (first variant): the low tf32 parts of a stage
//   warps 8-11   epilogue: TMEM -> registers -> global.  With beta = 1 each
//                warp stages alpha * acc for its 32 rows x 32 columns in
//                shared memory and a TMA reduce-add applies it to C in L2
//                (one rounding of C + alpha * acc, the same as the fma
//                below); with beta = 0 a TMA store writes it; other betas
//                (or a C that breaks the TMA rules) read C with plain loads.
// Plus 32 KB of epilogue staging.  All waits are bounded (mbar_wait_bounded).
#include "gemm.cuh"

#include <cstring>
#include <mutex>

namespace gptq {
namespace {

constexpr int TBM = 128, TBK = 32;              // 32 fp32 = 128 bytes = one swizzle row
constexpr int TTHREADS = 384;
constexpr int A_BYTES = TBM * TBK * 4;           // 16 KB
constexpr int CBUF_BYTES = 32 * 32 * 4;          // one warp's 32 x 32 chunk of C

template <int TN, bool PRELO>
struct GemmCfg {
    static constexpr int B_BYTES = TN * TBK * 4;
    static constexpr int STAGE_BYTES = 2 * (A_BYTES + B_BYTES);   // hi and lo of A and B
    static constexpr int STAGES = TN == 256 ? 2 : 3;
    static constexpr int TMEM_COLS = 2 * TN;
    static constexpr uint32_t TX_BYTES = PRELO ? 2 * (A_BYTES + B_BYTES) : A_BYTES + B_BYTES;
};

template <int TN, bool PRELO>
struct alignas(1024) GemmSmem {
    using C = GemmCfg<TN, PRELO>;
    uint8_t stage[C::STAGES][C::STAGE_BYTES];      // A_hi | A_lo | B_hi | B_lo
    uint8_t cbuf[4][2][CBUF_BYTES];                // per epilogue warp, double-buffered
    uint64_t full[C::STAGES];    // TMA landed
    uint64_t conv[C::STAGES];    // hi/lo split done (converter variant)
    uint64_t empty[C::STAGES];   // MMAs done reading
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
};
template <int TN, bool PRELO>
constexpr size_t gemm_smem_bytes()
{
    return sizeof(GemmSmem<TN, PRELO>) + 1024;
}
static_assert(gemm_smem_bytes<128, false>() <= 227 * 1024, "one CTA per SM");
static_assert(gemm_smem_bytes<256, true>() <= 227 * 1024, "one CTA per SM");
static_assert(gemm_smem_bytes<128, true>() <= 227 * 1024, "one CTA per SM");

enum CMode : int { kCPlain = 0, kCStore = 1, kCReduce = 2 };

struct GemmArgs {
    int M, N, K, batch, flags, trans_b, c_mode, tn;
    float alpha, beta;
    float* C;
    int64_t ldc, sC;
    int n_mt, n_nt;
    int* status;
    unsigned long long* stamp;   // span of this launch (see launch_sgemm) or null
};

// Low part of x below its tf32 truncation (exact in float32).
__device__ __forceinline__ float tf32_low(float x)
{
    return x - __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// C chunk from shared memory (128B-swizzled 32 x 32 fp32 box) to global:
// added to C (reduce) or written (store), by the TMA unit.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x, int y,
                                                  int z)
{
    asm volatile(
        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// at most one committed group may still be reading shared memory
__device__ __forceinline__ void bulk_wait_read_1()
{
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Unit u -> (batch, m-tile, n-tile) and its K range [k0, k1) (multiples of TBK);
// returns false for a tile the lower-triangular output flag skips.
__device__ __forceinline__ bool unit_info(const GemmArgs& g, int u, int& b, int& mt, int& nt, int& k0,
                                          int& k1)
{
    const int per = g.n_mt * g.n_nt;
    b = u / per;
    const int t = u % per;
    mt = t / g.n_nt;
    nt = t % g.n_nt;
    const int m0 = mt * TBM, n0 = nt * g.tn;
    if ((g.flags & kGemmLowerC) && n0 > m0 + TBM - 1) return false;
    k0 = 0;
    k1 = g.K;
    if (g.flags & kGemmLowerB) k0 = (n0 / TBK) * TBK;
    if (g.flags & kGemmLowerA) k1 = min(g.K, m0 + TBM);
    return true;
}

template <int TN, bool PRELO>
__global__ void __launch_bounds__(TTHREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const __grid_constant__ CUtensorMap mapAlo, const __grid_constant__ CUtensorMap mapBlo,
                   const __grid_constant__ CUtensorMap mapC, const GemmArgs g_param)
{
    // a register copy of the arguments: the parameter struct itself, reached
    // through a reference, would be reloaded with generic loads after every
    // asm statement with a memory clobber inside the loops
    const GemmArgs g = g_param;
    using Cfg = GemmCfg<TN, PRELO>;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int B_BYTES = Cfg::B_BYTES;
    extern __shared__ uint8_t smem_raw[];
    GemmSmem<TN, PRELO>& S = *reinterpret_cast<GemmSmem<TN, PRELO>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.conv[s], 4);
            mbar_init(&S.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S.tfull[a], 1);
            mbar_init(&S.tempty[a], 4);
        }
        S.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mapA);
        prefetch_tmap(&mapB);
        if (PRELO) {
            prefetch_tmap(&mapAlo);
            prefetch_tmap(&mapBlo);
        }
        if (g.c_mode != kCPlain) prefetch_tmap(&mapC);
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Under a programmatic dependent launch the set-up above overlaps the tail
    // of the previous kernel; its outputs (the A operand, C) are touched only
    // after this wait.  The next kernel may then start its own set-up.
    pdl_wait();
    pdl_trigger();
    if (g.stamp && threadIdx.x == 0) atomicMin(g.stamp, globaltimer_ns());
    const uint32_t tbase = S.tmem_base;
    volatile int* abort = &S.abort;
    int* status = g.status;
    const int n_units = g.n_mt * g.n_nt * g.batch;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                int b, mt, nt, k0, k1;
                if (!unit_info(g, u, b, mt, nt, k0, k1)) continue;
                for (int k = k0; k < k1; k += TBK, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&S.full[s], Cfg::TX_BYTES);
                    uint8_t* st = S.stage[s];
                    uint8_t* bh = st + 2 * A_BYTES;
                    tma_load_3d(st, &mapA, &S.full[s], k, mt * TBM, b);
                    if (PRELO) tma_load_3d(st + A_BYTES, &mapAlo, &S.full[s], k, mt * TBM, b);
                    if (g.trans_b) {
                        tma_load_3d(bh, &mapB, &S.full[s], k, nt * TN, b);
                        if (PRELO) tma_load_3d(bh + B_BYTES, &mapBlo, &S.full[s], k, nt * TN, b);
                    } else {
#pragma unroll
                        for (int q = 0; q < TN / 32; ++q) {   // 32-column x 32-row boxes
                            tma_load_3d(bh + q * (TBK * 32 * 4), &mapB, &S.full[s], nt * TN + q * 32, k, b);
                            if (PRELO)
                                tma_load_3d(bh + B_BYTES + q * (TBK * 32 * 4), &mapBlo, &S.full[s],
                                            nt * TN + q * 32, k, b);
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f32acc(2 /*tf32*/, 0 /*A K-major*/, g.trans_b ? 0u : 1u, TBM, TN);
            uint32_t it = 0, uc = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                int b, mt, nt, k0, k1;
                if (!unit_info(g, u, b, mt, nt, k0, k1)) continue;
                const int acc = uc & 1;
                const uint32_t aph = (uc >> 1) & 1;
                ++uc;
                if (!mbar_wait_bounded(&S.tempty[acc], aph ^ 1, abort, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dt = tbase + acc * TN;
                bool first = true;
                for (int k = k0; k < k1; k += TBK, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait_bounded(PRELO ? &S.full[s] : &S.conv[s], ph, abort, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ahi = smem_u32(S.stage[s]);
                    const uint32_t alo = ahi + A_BYTES;
                    const uint32_t bhi = ahi + 2 * A_BYTES;
                    const uint32_t blo = bhi + B_BYTES;
#pragma unroll
                    for (int k8 = 0; k8 < TBK / 8; ++k8) {
                        // A: K-major, 8 fp32 = 32 bytes further along the swizzled row
                        const uint64_t dah = sdesc_sw128(ahi + k8 * 32, 16, 1024);
                        const uint64_t dal = sdesc_sw128(alo + k8 * 32, 16, 1024);
                        uint64_t dbh, dbl;
                        if (g.trans_b) {
                            dbh = sdesc_sw128(bhi + k8 * 32, 16, 1024);
                            dbl = sdesc_sw128(blo + k8 * 32, 16, 1024);
                        } else {
                            // B: MN-major tf32 (128B swizzle, 32-byte atoms): 8 K-rows are
                            // 1024 bytes on, 4-row K groups 512 bytes apart, 32-column
                            // chunks TBK * 128 bytes apart
                            dbh = sdesc_sw128_base32b(bhi + k8 * 1024, TBK * 128, 512);
                            dbl = sdesc_sw128_base32b(blo + k8 * 1024, TBK * 128, 512);
                        }
                        umma_tf32(dt, dal, dbh, idesc, first ? 0u : 1u);
                        umma_tf32(dt, dah, dbl, idesc, 1u);
                        umma_tf32(dt, dah, dbh, idesc, 1u);
                        first = false;
                    }
                    umma_commit(&S.empty[s]);
                }
                if (!ok) break;
                umma_commit(&S.tfull[acc]);
            }
        }
        __syncwarp();
    } else if (!PRELO && warp >= 4 && warp < 8) {
        // converters: lo = x - trunc_tf32(x); hi is the loaded tile itself
        const int ct = threadIdx.x - 128;
        uint32_t it = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            int b, mt, nt, k0, k1;
            if (!unit_info(g, u, b, mt, nt, k0, k1)) continue;
            for (int k = k0; k < k1; k += TBK, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                const bool got = mbar_wait_bounded(&S.full[s], ph, abort, status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                float4* ah = reinterpret_cast<float4*>(S.stage[s]);
                float4* al = reinterpret_cast<float4*>(S.stage[s] + A_BYTES);
                float4* bh = reinterpret_cast<float4*>(S.stage[s] + 2 * A_BYTES);
                float4* bl = reinterpret_cast<float4*>(S.stage[s] + 2 * A_BYTES + B_BYTES);
#pragma unroll 4
                for (int i = ct; i < A_BYTES / 16; i += 128) {
                    const float4 xa = ah[i];
                    al[i] = make_float4(tf32_low(xa.x), tf32_low(xa.y), tf32_low(xa.z), tf32_low(xa.w));
                }
#pragma unroll 4
                for (int i = ct; i < B_BYTES / 16; i += 128) {
                    const float4 xb = bh[i];
                    bl[i] = make_float4(tf32_low(xb.x), tf32_low(xb.y), tf32_low(xb.z), tf32_low(xb.w));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.conv[s]);
            }
        }
    } else if (warp >= 8 && g.c_mode != kCPlain) {
        // epilogue through the TMA unit: warp w stages rows 32*(w % 4) .. +31
        // of a 32-column chunk (128B swizzle: 16-byte piece j of row r sits at
        // piece j ^ (r % 8)) and one lane issues the reduce-add or store
        const int q = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const bool lower = (g.flags & kGemmLowerC) != 0;
        uint32_t uc = 0, nbuf = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            int b, mt, nt, k0, k1;
            if (!unit_info(g, u, b, mt, nt, k0, k1)) continue;
            const int acc = uc & 1;
            const uint32_t aph = (uc >> 1) & 1;
            ++uc;
            const bool got = mbar_wait_bounded(&S.tfull[acc], aph, abort, status);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const bool have = k1 > k0;
            const int row0 = mt * TBM + q * 32;
#pragma unroll 1
            for (int c = 0; c < TN / 32; ++c) {
                const int col0 = nt * TN + c * 32;
                float v[32];
                tmem_ld_32x32b_x32(tbase + lane_addr + acc * TN + c * 32, v);
                tmem_ld_wait();
                // nothing of this chunk inside C (or, lower C, all above the diagonal)
                if (row0 >= g.M || col0 >= g.N || (lower && col0 > row0 + 31)) continue;
                uint8_t* buf = S.cbuf[q][nbuf & 1];
                ++nbuf;
                if (lane == 0) bulk_wait_read_1();
                __syncwarp();
                float4* rowp = reinterpret_cast<float4*>(buf + lane * 128);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float4 o;
                    o.x = have ? g.alpha * v[4 * j] : 0.f;
                    o.y = have ? g.alpha * v[4 * j + 1] : 0.f;
                    o.z = have ? g.alpha * v[4 * j + 2] : 0.f;
                    o.w = have ? g.alpha * v[4 * j + 3] : 0.f;
                    rowp[j ^ (lane & 7)] = o;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (g.c_mode == kCReduce)
                        tma_reduce_add_3d(&mapC, buf, col0, row0, b);
                    else
                        tma_store_3d(&mapC, buf, col0, row0, b);
                    bulk_commit();
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tempty[acc]);
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    } else if (warp >= 8) {
        // epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31 (= tile rows).  The
        // C values of a 32-column chunk are loaded one chunk ahead, the first
        // before the accumulator is ready, so the loads overlap the MMAs and
        // the previous chunk's arithmetic.
        const int q = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const bool lower = (g.flags & kGemmLowerC) != 0;
        const bool read_c = g.beta != 0.f;
        uint32_t uc = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            int b, mt, nt, k0, k1;
            if (!unit_info(g, u, b, mt, nt, k0, k1)) continue;
            const int acc = uc & 1;
            const uint32_t aph = (uc >> 1) & 1;
            ++uc;
            const int row = mt * TBM + q * 32 + lane;
            float* crow = g.C + b * g.sC + static_cast<int64_t>(row) * g.ldc;
            // chunk c takes the vector path when it lies inside C, above no
            // skipped (upper) element and 16-byte aligned
            auto vec_ok = [&](int c) {
                const int col0 = nt * TN + c * 32;
                return row < g.M && col0 + 32 <= g.N && !(lower && col0 + 31 > row) &&
                       (reinterpret_cast<uintptr_t>(crow + col0) & 15) == 0;
            };
            float4 cn[8];
            if (read_c && vec_ok(0)) {
                const float4* p = reinterpret_cast<const float4*>(crow + nt * TN);
#pragma unroll
                for (int m = 0; m < 8; ++m) cn[m] = p[m];
            }
            const bool got = mbar_wait_bounded(&S.tfull[acc], aph, abort, status);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const bool have = k1 > k0;   // an empty K range leaves the accumulator unwritten
#pragma unroll 1
            for (int c = 0; c < TN / 32; ++c) {
                float4 cc[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) cc[m] = cn[m];
                if (read_c && c + 1 < TN / 32 && vec_ok(c + 1)) {
                    const float4* p = reinterpret_cast<const float4*>(crow + nt * TN + (c + 1) * 32);
#pragma unroll
                    for (int m = 0; m < 8; ++m) cn[m] = p[m];
                }
                float v[32];
                __syncwarp();   // the loads above may diverge; tcgen05.ld is warp-aligned
                tmem_ld_32x32b_x32(tbase + lane_addr + acc * TN + c * 32, v);
                tmem_ld_wait();
                const int col0 = nt * TN + c * 32;
                if (row >= g.M || col0 >= g.N) continue;
                if (vec_ok(c)) {
                    float4* p = reinterpret_cast<float4*>(crow + col0);
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        float4 o = read_c ? cc[m] : make_float4(0.f, 0.f, 0.f, 0.f);
                        const float a0 = have ? v[4 * m] : 0.f, a1 = have ? v[4 * m + 1] : 0.f;
                        const float a2 = have ? v[4 * m + 2] : 0.f, a3 = have ? v[4 * m + 3] : 0.f;
                        o.x = fmaf(g.alpha, a0, g.beta * o.x);
                        o.y = fmaf(g.alpha, a1, g.beta * o.y);
                        o.z = fmaf(g.alpha, a2, g.beta * o.z);
                        o.w = fmaf(g.alpha, a3, g.beta * o.w);
                        p[m] = o;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 32; ++m) {
                        const int col = col0 + m;
                        if (col >= g.N || (lower && col > row)) continue;
                        const float a = have ? v[m] : 0.f;
                        const float old = read_c ? crow[col] : 0.f;
                        crow[col] = fmaf(g.alpha, a, g.beta * old);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (g.stamp && threadIdx.x == 0) atomicMax(g.stamp + 1, globaltimer_ns());
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, Cfg::TMEM_COLS);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D fp32 tensor map: inner dimension `cols` (contiguous), `rows` rows of
// pitch ld, `batch` matrices `bstride` elements apart; box box_c x box_r x 1.
int make_map_f32(CUtensorMap* map, const float* base, int64_t cols, int64_t rows, int64_t ld,
                 int batch, int64_t bstride, int box_c, int box_r, CUtensorMapSwizzle swz)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(batch)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 4,
                             static_cast<cuuint64_t>(batch > 1 ? bstride : ld * rows) * 4};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_r), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return GPTQ_OK;
}

}  // namespace

bool gemm_tc_supported(const float* A, int64_t lda, int64_t sA, const float* B, int64_t ldb,
                       int64_t sB, int batch)
{
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al16(A) || !al16(B) || (lda & 3) || (ldb & 3)) return false;
    if (batch > 1 && ((sA & 3) || (sB & 3))) return false;
    return true;
}

template <int TN, bool PRELO>
static int set_smem_attr()
{
    static bool attr_set[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gemm_tc_kernel<TN, PRELO>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(gemm_smem_bytes<TN, PRELO>())));
        attr_set[dev] = true;
    }
    return GPTQ_OK;
}

int launch_gemm_tc(bool trans_b, int M, int N, int K, float alpha, const float* A, int64_t lda,
                   int64_t sA, const float* B, int64_t ldb, int64_t sB, float beta, float* C,
                   int64_t ldc, int64_t sC, int batch, int flags, cudaStream_t stream, int max_ctas,
                   const float* A_lo, const float* B_lo, bool pdl, unsigned long long* stamp)
{
    if (M <= 0 || N <= 0 || batch <= 0) return GPTQ_OK;
    const bool prelo = A_lo && B_lo;
    // 128 x 256 tiles with supplied low parts, unless they would not fill one
    // wave of the SMs: then 128 x 128 tiles, twice as many CTAs with half the
    // MMA work each
    int tn = prelo ? 256 : 128;
    if (prelo && static_cast<int64_t>((M + TBM - 1) / TBM) * ((N + 255) / 256) * batch < sm_count())
        tn = 128;
    int rc = prelo ? (tn == 256 ? set_smem_attr<256, true>() : set_smem_attr<128, true>())
                   : set_smem_attr<128, false>();
    if (rc) return rc;
    const int Kp = K > 0 ? K : 1;
    CUtensorMap mA, mB, mAlo, mBlo, mC;
    memset(&mAlo, 0, sizeof mAlo);
    memset(&mBlo, 0, sizeof mBlo);
    int c_mode = kCPlain;
    const bool c_tma = (reinterpret_cast<uintptr_t>(C) & 15) == 0 && (ldc & 3) == 0 &&
                       (batch == 1 || (sC & 3) == 0);
    if (c_tma && (beta == 1.f || beta == 0.f)) {
        rc = make_map_f32(&mC, C, N, M, ldc, batch, sC, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc) return rc;
        c_mode = beta == 1.f ? kCReduce : kCStore;
    } else {
        memset(&mC, 0, sizeof mC);
    }
    // A: [M][K] K-major boxes of 32 x 128; B: [N][K] boxes 32 x tn (trans_b) or
    // [K][N] boxes of 32 columns x 32 rows
    auto map_a = [&](CUtensorMap* m, const float* p) {
        return make_map_f32(m, p, Kp, M, lda, batch, sA, TBK, TBM, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    auto map_b = [&](CUtensorMap* m, const float* p) {
        return trans_b ? make_map_f32(m, p, Kp, N, ldb, batch, sB, TBK, tn, CU_TENSOR_MAP_SWIZZLE_128B)
                       : make_map_f32(m, p, N, Kp, ldb, batch, sB, 32, TBK,
                                      CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
    };
    if ((rc = map_a(&mA, A)) || (rc = map_b(&mB, B))) return rc;
    if (prelo && ((rc = map_a(&mAlo, A_lo)) || (rc = map_b(&mBlo, B_lo)))) return rc;
    GemmArgs g;
    g.M = M;
    g.N = N;
    g.K = K;
    g.batch = batch;
    g.flags = flags;
    g.trans_b = trans_b ? 1 : 0;
    g.c_mode = c_mode;
    g.tn = tn;
    g.alpha = alpha;
    g.beta = beta;
    g.C = C;
    g.ldc = ldc;
    g.sC = sC;
    g.n_mt = (M + TBM - 1) / TBM;
    g.n_nt = (N + tn - 1) / tn;
    g.status = device_status_ptr();
    g.stamp = stamp;
    const int64_t units = static_cast<int64_t>(g.n_mt) * g.n_nt * batch;
    int64_t cap = sm_count();
    if (max_ctas > 0 && max_ctas < cap) cap = max_ctas;
    if (max_ctas < 0) cap = units;   // one CTA per tile
    const int grid = static_cast<int>(units < cap ? units : cap);
    if (prelo && tn == 256)
        GPTQ_CUDA_CHECK(launch_k(gemm_tc_kernel<256, true>, dim3(grid), dim3(TTHREADS),
                                 gemm_smem_bytes<256, true>(), stream, pdl, mA, mB, mAlo, mBlo, mC, g));
    else if (prelo)
        GPTQ_CUDA_CHECK(launch_k(gemm_tc_kernel<128, true>, dim3(grid), dim3(TTHREADS),
                                 gemm_smem_bytes<128, true>(), stream, pdl, mA, mB, mAlo, mBlo, mC, g));
    else
        GPTQ_CUDA_CHECK(launch_k(gemm_tc_kernel<128, false>, dim3(grid), dim3(TTHREADS),
                                 gemm_smem_bytes<128, false>(), stream, pdl, mA, mB, mAlo, mBlo, mC, g));
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

}  // namespace gptq
