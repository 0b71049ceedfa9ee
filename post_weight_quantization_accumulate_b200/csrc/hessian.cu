// hessian.cu -- H += 2 X^T X on the sm_100a tensor cores.
//
// GPTQ overview page, "Jak działa": the layer Hessian is H = 2 X X^T from the
// input activations (X there is d x N; here X is [N, d], so H = 2 X^T X);
// "Złożoność obliczeniowa": O(N_calib d^2), the dominant cost of the method
// for calibration sets much larger than d.
//
// Design (B200):
//  * H is symmetric, so only 256 x 256 output tiles (ti, tj) with tj >= ti
//    are computed; the strict lower triangle is written afterwards by a
//    transpose copy (mirror_upper_kernel), so H is bitwise symmetric.
//  * A tile is computed by a pair of CTAs (a cluster of two on neighbouring
//    SMs) with the pair form of the tensor-core MMA (M = 256, N = 256): CTA r
//    of the pair holds the 128 rows 256 ti + 128 r (its A operand) and the
//    128 columns 256 tj + 128 r (its half of B), and each SM keeps its 128 x
//    256 accumulator in its own tensor memory.  Per SM and token this moves
//    half of the B operand a single-CTA 128 x 256 tile would, which keeps the
//    shared-memory traffic (TMA writes + MMA reads) under the shared-memory
//    bandwidth at the full MMA rate.
//  * Both operands are slices of the same X rows: A = X[t, rows], B = X[t,
//    cols].  Their contraction index (tokens) is the outer dimension of X, so
//    both are MN-major; TMA brings 128-token x 64-column boxes with 128-byte
//    swizzle, the canonical MN-major SW128 layout tcgen05.mma reads.  Each CTA
//    loads its own boxes (no multicast); the loads of both CTAs complete on
//    the first CTA's barrier, whose thread issues the MMAs.
//  * Work units = (tile, token span of 4096 .. 32768 tokens, the longest that
//    still gives each pair about eight units).  A persistent grid of
//    one pair per two SMs walks the units span-major, so concurrently
//    running units read the same token rows of X (L2 reuse).
//  * Accumulation precision: the tensor core adds each MMA's result into the
//    fp32 TMEM accumulator with a rounding that is biased for long chains
//    (measured: sums of squares come out ~0.25 ulp low per MMA).  So a TMEM
//    chain covers only kChainTokens tokens (32 MMAs); the epilogue promotes
//    each chain into fp32 registers with round-to-nearest adds, and flushes
//    the span's sum into H with one fp32 red.add per element.
//  * Warp roles per CTA (384 threads, three warpgroups): warp 0 = TMA
//    producer, warp 1 = MMA issuer (first CTA of the pair) and TMEM owner
//    (warpgroup 0 gives its registers up to 64); warps 4-11 = epilogue (raised
//    to 216 registers); warps w and w+4 share TMEM lanes 32*(w%4)..+31 and
//    split the 256 columns in halves, 128 fp32 registers of running sum each.
//    128 x 64 + 256 x 216 = 63488 fits the launch budget 384 x 168.  A 3-stage
//    shared-memory ring (64 KB per stage: few, large TMA batches per barrier
//    round trip measured faster than more, smaller stages) and two TMEM chain
//    buffers (2 x 256
//    columns) let the promotion of one chain overlap the MMAs of the next.
//  * Flush order is fixed, so H is bitwise reproducible: the flush of span s
//    of a tile waits until the flushes of spans 0 .. s-1 of that tile have
//    landed (a turn counter per tile and CTA, counting epilogue-warp flushes).
//    The counters live in H itself, in the strictly lower triangle below the
//    first tile row (rows 256.., columns 0..255), which no tile flushes into
//    and which the mirror copy overwrites at the end of the call; each launch
//    zeroes the ones it uses.  A unit only ever waits on a unit with a smaller
//    index, and each pair walks its units in increasing order, so with every
//    pair resident the waits end.  A one-tile H (d <= 256) has no room for
//    counters and runs its tokens as one unit.
//  * Every mbarrier and counter wait is bounded; a time-out records
//    GPTQ_ERR_TIMEOUT (a timed-out turn wait still flushes, unordered); both
//    CTAs meet at a cluster barrier before the pair frees its tensor memory.
#include "common.cuh"

#include <algorithm>
#include <mutex>

namespace gptq {

namespace {

constexpr int kBM = 128;          // H rows per CTA (half of the pair's M = 256)
constexpr int kBN = 256;          // H cols per tile (MMA N)
constexpr int kTile = 256;        // tile edge
constexpr int kBK = 128;          // tokens per pipeline stage
constexpr int kStages = 3;
constexpr int kBoxCols = 64;      // 64 bf16 = 128 bytes = one swizzle row
constexpr int kBoxBytes = kBK * kBoxCols * 2;           // 16 KB
constexpr int kABytes = kBoxBytes * (kBM / kBoxCols);   // 32 KB: 128 rows of A
constexpr int kBBytes = kBoxBytes * (kBN / 2 / kBoxCols);  // 32 KB: this CTA's 128 columns of B
constexpr int kStageBytes = kABytes + kBBytes;          // 64 KB
constexpr int kThreads = 384;
constexpr int kEpiWarps = 8;
constexpr int kTmemCols = 512;    // two 256-column fp32 chain buffers
constexpr int kChainTokens = 512; // tokens per TMEM accumulation chain
constexpr int kSpanMax = 32768;   // tokens per work unit (one flush into H), at most
constexpr int kSpanMin = 4096;
constexpr uint32_t kIdesc = idesc_f32acc(1 /*bf16*/, 1, 1, 2 * kBM, kBN);

struct alignas(1024) HessSmem {
    uint8_t stage[kStages][kStageBytes];
    uint64_t full[kStages];     // first CTA: TMA bytes of both CTAs landed
    uint64_t empty[kStages];    // MMAs done reading the stage (both CTAs)
    uint64_t tfull[2];          // chain complete (both CTAs)
    uint64_t tempty[2];         // first CTA: both epilogues drained the buffer
    uint32_t tmem_base;
    int abort;
};
constexpr size_t kSmemBytes = sizeof(HessSmem) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "one CTA per SM");

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank)
{
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the
// barrier at cluster address `bar` (the first CTA's), pair form, no multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x,
                                                 int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on the barrier at this offset in both CTAs of the pair when
// the MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar)
{
    const uint16_t mask = 3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(mask)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Upper-triangle tile number -> (ti, tj), tj >= ti, in bands of kBand tile
// rows enumerated column by column: the pairs running at the same time (same
// token span, consecutive tile numbers) then cover a compact block of tiles
// and share both operand slices of X in L2, instead of one tile row sharing A
// and streaming a different B slice each.
constexpr int kBand = 8;
__device__ __forceinline__ void tile_coords(int tile, int n_t, int& ti, int& tj)
{
    int idx = tile;
    for (int b0 = 0; b0 < n_t; b0 += kBand) {
        const int b1 = min(b0 + kBand, n_t);
        for (int c = b0; c < n_t; ++c) {
            const int cnt = min(c + 1, b1) - b0;   // rows b0 .. min(c, b1-1)
            if (idx < cnt) {
                ti = b0 + idx;
                tj = c;
                return;
            }
            idx -= cnt;
        }
    }
    ti = n_t - 1;
    tj = n_t - 1;
}

// Turn counter of (tile, CTA rank) inside H's strictly lower triangle.
__device__ __forceinline__ int* turn_counter(float* H, int d, int tile, uint32_t rank)
{
    const int c = 2 * tile + static_cast<int>(rank);
    return reinterpret_cast<int*>(H + static_cast<int64_t>(kTile + c / kTile) * d + c % kTile);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Waits (lane 0 of the calling warp) until *ctr >= target; bounded like the
// mbarrier waits.  Returns false on a time-out (recorded in the status word).
__device__ __forceinline__ bool wait_turn(const int* ctr, int target, int* status)
{
    if (ld_acquire_gpu(ctr) >= target) return true;
    const long long t0 = clock64();
    while (ld_acquire_gpu(ctr) < target) {
        if (clock64() - t0 > kWaitLimitCycles) {
            record_status(status, GPTQ_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(256);
    }
    return true;
}

__global__ void zero_turns_kernel(float* H, int d, int n)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c < n) *reinterpret_cast<int*>(H + static_cast<int64_t>(kTile + c / kTile) * d + c % kTile) = 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap, float* __restrict__ H, int d,
                      int n_tokens, int n_t, int n_tiles, int n_split, int span, int* status)
{
    extern __shared__ uint8_t smem_raw[];
    HessSmem& S = *reinterpret_cast<HessSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.tfull[b], 1);
            mbar_init(&S.tempty[b], 2 * kEpiWarps);
        }
        S.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap);
    }
    if (warp == 1) {
        tmem_alloc_pair(&S.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers and tensor memory exist before any use
    tc_fence_after();
    const uint32_t tbase = S.tmem_base;
    volatile int* abort = &S.abort;
    const int n_units = n_tiles * n_split;

    if (warp < 4) {
        regs_dealloc<64>();
        if (warp == 0 && lane == 0) {
            uint32_t it = 0;
            for (int u = pair; u < n_units && !*abort; u += n_pairs) {
                int ti, tj;
                tile_coords(u % n_tiles, n_t, ti, tj);
                const int t0 = (u / n_tiles) * span;
                const int t1 = min(n_tokens, t0 + span);
                const int col_a = ti * kTile + static_cast<int>(rank) * kBM;
                const int col_b = tj * kTile + static_cast<int>(rank) * (kBN / 2);
                const bool diag = ti == tj;
                bool ok = true;
                for (int t = t0; t < t1 && ok; t += kBK, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, status)) { ok = false; break; }
                    // a diagonal tile's B half is this CTA's A rows: loaded once
                    if (leader) mbar_arrive_expect_tx(&S.full[s], 2 * (diag ? kABytes : kStageBytes));
                    const uint32_t fb = cluster_addr(&S.full[s], 0);
                    uint8_t* a = S.stage[s];
                    uint8_t* b = a + kABytes;
#pragma unroll
                    for (int m = 0; m < kBM / kBoxCols; ++m)
                        tma_load_2d_pair(a + m * kBoxBytes, &tmap, fb, col_a + m * kBoxCols, t);
                    if (!diag) {
#pragma unroll
                        for (int m = 0; m < kBN / 2 / kBoxCols; ++m)
                            tma_load_2d_pair(b + m * kBoxBytes, &tmap, fb, col_b + m * kBoxCols, t);
                    }
                }
                if (!ok) break;
            }
        } else if (warp == 1 && lane == 0 && leader) {
            uint32_t it = 0, ch = 0;
            bool ok = true;
            for (int u = pair; u < n_units && ok && !*abort; u += n_pairs) {
                const int t0 = (u / n_tiles) * span;
                const int t1 = min(n_tokens, t0 + span);
                int ti, tj;
                tile_coords(u % n_tiles, n_t, ti, tj);
                const uint32_t b_off = ti == tj ? 0u : static_cast<uint32_t>(kABytes);
                for (int c0 = t0; c0 < t1 && ok; c0 += kChainTokens, ++ch) {
                    const int b = ch & 1;
                    const uint32_t cph = (ch >> 1) & 1;
                    if (!mbar_wait_bounded(&S.tempty[b], cph ^ 1, abort, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t dt = tbase + b * kBN;
                    const int nk = (min(t1, c0 + kChainTokens) - c0 + kBK - 1) / kBK;
                    for (int kk = 0; kk < nk; ++kk, ++it) {
                        const int s = it % kStages;
                        const uint32_t ph = (it / kStages) & 1;
                        if (!mbar_wait_bounded(&S.full[s], ph, abort, status)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(S.stage[s]);
                        const uint32_t b0 = a0 + b_off;
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            // 16 tokens = two 8-row swizzle groups = 2048 bytes
                            const uint64_t ad = sdesc_sw128(a0 + k * 2048, kBoxBytes, 1024);
                            const uint64_t bd = sdesc_sw128(b0 + k * 2048, kBoxBytes, 1024);
                            umma_f16_pair(dt, ad, bd, kIdesc, (kk | k) != 0);
                        }
                        umma_commit_pair(&S.empty[s]);
                    }
                    if (ok) umma_commit_pair(&S.tfull[b]);
                }
            }
        }
        __syncwarp();
    } else {
        regs_alloc<216>();
        // epilogue: warp w reads TMEM lanes 32*(w % 4) .. +31, column half h
        const int q = warp & 3;
        const int h = (warp - 4) / 4;
        const int row_in_tile = static_cast<int>(rank) * kBM + q * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        uint32_t ch = 0;
        bool ok = true;
        for (int u = pair; u < n_units && ok; u += n_pairs) {
            const int t0 = (u / n_tiles) * span;
            const int t1 = min(n_tokens, t0 + span);
            float acc[kBN / 2];
#pragma unroll
            for (int i = 0; i < kBN / 2; ++i) acc[i] = 0.f;
            for (int c0 = t0; c0 < t1; c0 += kChainTokens, ++ch) {
                const int b = ch & 1;
                const uint32_t cph = (ch >> 1) & 1;
                // every lane waits, then the warp reconverges for tcgen05.ld
                const bool got = mbar_wait_bounded(&S.tfull[b], cph, abort, status);
                __syncwarp();
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                const uint32_t taddr = tbase + lane_addr + b * kBN + h * (kBN / 2);
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) {
                    float v[16];
                    tmem_ld_32x32b_x16(taddr + c * 16, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[c * 16 + i] += v[i];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(cluster_addr(&S.tempty[b], 0));
            }
            if (!ok) break;
            int ti, tj;
            tile_coords(u % n_tiles, n_t, ti, tj);
            const int row = ti * kTile + row_in_tile;
            int* turn = n_split > 1 ? turn_counter(H, d, u % n_tiles, rank) : nullptr;
            if (turn) {
                // the 8 epilogue warps of this CTA flushed every earlier span
                if (lane == 0) wait_turn(turn, (u / n_tiles) * kEpiWarps, status);
                __syncwarp();
            }
#pragma unroll
            for (int c = 0; c < kBN / 64; ++c) {
                const int col0 = tj * kTile + h * (kBN / 2) + c * 32;
                if (row < d && col0 < d && col0 + 31 >= row) {
                    float* dst = H + static_cast<int64_t>(row) * d + col0;
                    if (col0 + 32 <= d) {
#pragma unroll
                        for (int m = 0; m < 8; ++m)
                            atomicAdd(reinterpret_cast<float4*>(dst) + m,
                                      make_float4(2.f * acc[c * 32 + 4 * m], 2.f * acc[c * 32 + 4 * m + 1],
                                                  2.f * acc[c * 32 + 4 * m + 2], 2.f * acc[c * 32 + 4 * m + 3]));
                    } else {
#pragma unroll
                        for (int m = 0; m < 32; ++m)
                            if (m < d - col0) atomicAdd(dst + m, 2.f * acc[c * 32 + m]);
                    }
                }
            }
            if (turn) {
                __syncwarp();
                if (lane == 0) {
                    __threadfence();   // this warp's additions land before its turn is passed on
                    atomicAdd(turn, 1);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no MMA, commit or remote arrive of the pair is still in flight
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tbase, kTmemCols);
    }
}

// H[j][i] = H[i][j] for i < j: copies the upper triangle into the lower one
// through a 32 x 32 shared-memory transpose.
__global__ void mirror_upper_kernel(float* __restrict__ H, int d)
{
    __shared__ float t[32][33];
    const int bx = blockIdx.x, by = blockIdx.y;
    if (bx > by) return;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int i = bx * 32 + r, j = by * 32 + threadIdx.x;
        if (i < d && j < d) t[r][threadIdx.x] = H[static_cast<int64_t>(i) * d + j];
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int row = by * 32 + r, col = bx * 32 + threadIdx.x;
        if (row < d && col < d && row > col) H[static_cast<int64_t>(row) * d + col] = t[threadIdx.x][r];
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

}  // namespace

// Tensor map over X [n_rows, d] bf16 with 64 x 64 boxes, 128-byte swizzle;
// rows beyond n_rows read as zero.
int make_x_tmap(CUtensorMap* map, const uint16_t* X, int64_t n_rows, int64_t d)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n_rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[2] = {kBoxCols, kBK};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
    return GPTQ_OK;
}

// Accumulates the upper triangle of 2 X^T X (n_rows < 2^31) into H.
int launch_hessian_upper(float* H, const uint16_t* X, int64_t n_rows, int64_t d,
                         cudaStream_t stream)
{
    if (n_rows <= 0) return GPTQ_OK;
    static bool attr_set[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        GPTQ_CUDA_CHECK(cudaFuncSetAttribute(hessian_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes)));
        attr_set[dev] = true;
    }
    CUtensorMap map;
    int rc = make_x_tmap(&map, X, n_rows, d);
    if (rc) return rc;
    const int n_t = static_cast<int>((d + kTile - 1) / kTile);
    const int n_tiles = n_t * (n_t + 1) / 2;
    // the longest token span (fewest flushes of partial sums into H) that
    // still gives every pair about eight units
    const int64_t want = 8 * static_cast<int64_t>(sm_count() / 2);
    int span = kSpanMax;
    while (span > kSpanMin && n_tiles * ((n_rows + span - 1) / span) < want) span /= 2;
    if (n_t == 1) span = static_cast<int>(n_rows);   // no room for turn counters: one unit
    const int n_split = static_cast<int>((n_rows + span - 1) / span);
    if (n_split > 1) {
        // turn counters of this launch, inside H's strictly lower triangle
        const int n = 2 * n_tiles;
        zero_turns_kernel<<<(n + 255) / 256, 256, 0, stream>>>(H, static_cast<int>(d), n);
        GPTQ_LAUNCH_CHECK();
    }
    const int64_t units = static_cast<int64_t>(n_tiles) * n_split;
    // pairs that can be resident at once (a GPC with an odd number of free
    // SMs holds one pair less than half its SMs)
    static int resident_pairs[64] = {};
    int max_pairs = sm_count() / 2;
    if (dev < 64) {
        if (!resident_pairs[dev]) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * max_pairs);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = kSmemBytes;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, hessian_tc_kernel, &cfg) != cudaSuccess || n <= 0) {
                (void)cudaGetLastError();
                n = max_pairs;
            }
            resident_pairs[dev] = n;
        }
        max_pairs = std::min(max_pairs, resident_pairs[dev]);
    }
    const int pairs = static_cast<int>(units < max_pairs ? units : max_pairs);
    hessian_tc_kernel<<<2 * pairs, kThreads, kSmemBytes, stream>>>(
        map, H, static_cast<int>(d), static_cast<int>(n_rows), n_t, n_tiles, n_split, span,
        device_status_ptr());
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

int launch_mirror(float* H, int64_t d, cudaStream_t stream)
{
    const int nb = static_cast<int>((d + 31) / 32);
    mirror_upper_kernel<<<dim3(nb, nb), dim3(32, 8), 0, stream>>>(H, static_cast<int>(d));
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

}  // namespace gptq
