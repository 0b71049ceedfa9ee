// w4a16.cu -- the quantized linear at inference time: Y = X W^T with bf16
// activations X [M, K] and the packed 4-bit weights gptq_quantize writes
// (codes [N, K/2], two per byte, column 2i in the low nibble; fp32 scales and
// integer zeros per (row, group)).
//
// AutoGPTQ page, "Mixed Precision Scheme": the weights stay 4-bit in memory
// and are dequantized on the fly next to the compute unit; W^[n][k] =
// s (q - z) with the scale and zero of column k's group.  For a decode-sized
// batch (M up to a few dozen rows) the product is bound by reading the packed
// weights: N K / 2 bytes plus 8 bytes of (scale, zero) per row and group.
//
// Tensor-core path (groups contiguous along K: g = k / group_size):
//   Y[m][n] = sum_g s[n][g] * sum_{k in g} (q[n][k] - z[n][g]) x[m][k]
// The integer differences q - z (|q - z| <= 15) are exact in bf16, so the
// inner sums are bf16 x bf16 products accumulated in fp32 on tcgen05, one
// TMEM accumulator per group; the scale is applied once per group in the
// epilogue.  This is X W^T with W^ exactly as the quantizer defines it (no
// 16-bit rounding of s (q - z)), differing only in the order of the fp32
// additions.
//   * A tile is 128 weight rows (the MMA's M) by a K range.  Stages of 128
//     columns: TMA brings the packed bytes (128 x 64 B) and the X tile (M
//     padded to NP rows, 128B-swizzled).  Each converter thread reads its own
//     row's zero and scale through L1 (one 32-byte sector serves 8 groups).
//   * Eight converter warps turn a row's nibbles into bf16 pairs (128 + q
//     from the exponent trick, minus 128 + z) and store them with
//     tcgen05.st straight into tensor memory, which is the MMA's A operand:
//     the dequantized weights never touch shared memory.  Within each
//     8-column word the pairs come out as columns (i, i + 4); the converters
//     permute each 16-byte chunk of the X tile the same way.
//   * One thread issues kind::f16 MMAs, A from TMEM, B = X from shared memory,
//     D = the group's accumulator slot (NP columns; 128 / NP slots in a ring).
//     The group bookkeeping is done once per group; per 16-column step only
//     the MMA is issued (eight straight-line MMAs when a whole stage lies in
//     one group), because the issuing thread's own instruction count sets the
//     pace at these small MMA shapes.
//   * The converters read finished group accumulators one stage behind and
//     accumulate s * acc into registers.
//   * K is split over a cluster of up to 8 CTAs; the partial sums meet in
//     distributed shared memory and each CTA of the cluster adds a slice of
//     the tile in a fixed rank order (deterministic) and writes Y.
// Decode path (at most 4 activation rows, groups contiguous along K): the
// weights streamed once with 16-byte loads straight into registers, four
// weight rows per block sharing each read of the activations, (q - z) x in
// bf16 pairs and mixed-precision FMAs (see the kernel below).
// General path (g_idx given, or a group size or K the tiles do not fit): one
// warp per weight row on the SIMT pipes, W^ = s (q - z) in fp32.
#include "common.cuh"

#include <mutex>

namespace gptq {

namespace {

// ------------------------------------------------------------ general path
constexpr int kWThreads = 256;
constexpr int kMTile = 8;   // output rows per pass over the weights

// 8 bf16 (16 bytes) -> float
__device__ __forceinline__ void bf16x8(const uint16_t* p, float (&x)[8])
{
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// One warp per weight row; each lane takes 8 columns (one packed word) per
// step.  contiguous: no g_idx and group_size a multiple of 8 (or one group),
// so one (s, z) per word; otherwise each column looks up its group.
template <bool kContiguous>
__global__ void __launch_bounds__(kWThreads)
    w4a16_simt_kernel(float* __restrict__ Y, const uint16_t* __restrict__ X,
                      const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                      const float* __restrict__ zeros, const int32_t* __restrict__ g_idx, int M,
                      int N, int K, int gs, int ng, int m0)
{
    const int lane = threadIdx.x & 31;
    const int n_warps = (gridDim.x * kWThreads) >> 5;
    const int mt = min(kMTile, M - m0);
    const int units = K / 8;
    for (int n = (blockIdx.x * kWThreads + threadIdx.x) >> 5; n < N; n += n_warps) {
        float acc[kMTile];
#pragma unroll
        for (int m = 0; m < kMTile; ++m) acc[m] = 0.f;
        const uint32_t* prow =
            reinterpret_cast<const uint32_t*>(packed + static_cast<int64_t>(n) * (K / 2));
        const float* srow = scales + static_cast<int64_t>(n) * ng;
        const float* zrow = zeros + static_cast<int64_t>(n) * ng;
        for (int u = lane; u < units; u += 32) {
            const uint32_t q8 = prow[u];   // columns 8u .. 8u+7, even column in the low nibble
            float w[8];
            if (kContiguous) {
                const int g = gs > 0 ? (8 * u) / gs : 0;
                const float s = srow[g], z = zrow[g];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    w[i] = s * (static_cast<float>((q8 >> (4 * i)) & 15u) - z);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int k = 8 * u + i;
                    const int g = g_idx ? g_idx[k] : (gs > 0 ? k / gs : 0);
                    w[i] = srow[g] * (static_cast<float>((q8 >> (4 * i)) & 15u) - zrow[g]);
                }
            }
#pragma unroll
            for (int m = 0; m < kMTile; ++m) {
                if (m < mt) {
                    float x[8];
                    bf16x8(X + static_cast<int64_t>(m0 + m) * K + 8 * u, x);
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[m] = fmaf(w[i], x[i], acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < kMTile; ++m) {
#pragma unroll
            for (int o = 16; o; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
        }
        if (lane == 0) {
#pragma unroll
            for (int m = 0; m < kMTile; ++m)
                if (m < mt) Y[static_cast<int64_t>(m0 + m) * N + n] = acc[m];
        }
    }
}

// ------------------------------------------------------------ decode path
// For at most four rows of activations the product is a matrix-vector
// product per row: about 2 M flops per half-byte of weights, so the issue
// rate of the SIMT pipes, not the tensor cores, decides whether the weights
// stream at HBM speed.  The packed bytes are read once with 16-byte loads
// and never staged.  Work unit: a block of kGvWarps warps owns kGvRows
// weight rows; lane l of warp w takes the 32-column chunks
// c = l + 32 w, l + 32 (w + kGvWarps), ... of all kGvRows rows, so one read of
// the chunk's activations (64 bytes per activation row, from L1) serves
// kGvRows weight rows.  Per 8-column word: four bf16 pairs 128 + q from the
// exponent trick (columns (i, i + 4)), minus the pair 128 + z (exact: q - z
// is an integer of at most 15 in magnitude), then one mixed-precision FMA per
// column, bf16 (q - z) times bf16 x accumulated in fp32 (the product is
// exact in fp32).  The chunk's sum is scaled once: acc += s * dot.  Lanes
// and then warps are reduced in a fixed order (deterministic).  Needs
// K % 32 == 0 and groups of a multiple of 32 columns (or one group per row),
// contiguous along K, zeros integer-valued in 0..15.
constexpr int kGvRows = 4;
constexpr int kGvWarps = 4;

__device__ __forceinline__ float fma_f32_bf16(uint32_t a, uint32_t b, float c)
{
    // a, b: bf16 in the low 16 bits
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;"
        : "=f"(d)
        : "h"(static_cast<uint16_t>(a)), "h"(static_cast<uint16_t>(b)), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int MM>
__global__ void __launch_bounds__(kGvWarps * 32)
    w4a16_gemv_kernel(float* __restrict__ Y, const uint16_t* __restrict__ X,
                      const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                      const float* __restrict__ zeros, int N, int K, int gs, int ng)
{
    __shared__ float red[kGvWarps][kGvRows * MM];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int chunks = K >> 5;
    const int64_t row_bytes = K / 2;
    for (int n0 = blockIdx.x * kGvRows; n0 < N; n0 += gridDim.x * kGvRows) {
        float acc[kGvRows][MM];
#pragma unroll
        for (int r = 0; r < kGvRows; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[r][m] = 0.f;
#pragma unroll(MM <= 2 ? 2 : 1)
        for (int c = lane + 32 * warp; c < chunks; c += 32 * kGvWarps) {
            const int g = gs > 0 ? (32 * c) / gs : 0;
            uint4 q4[kGvRows];
            float s[kGvRows];
            uint32_t zb[kGvRows];
#pragma unroll
            for (int r = 0; r < kGvRows; ++r) {
                const int n = min(n0 + r, N - 1);   // rows past N repeat row N - 1 and are not stored
                q4[r] = __ldcs(reinterpret_cast<const uint4*>(packed + n * row_bytes) + c);
                s[r] = __ldg(scales + static_cast<int64_t>(n) * ng + g);
                zb[r] = 0x43004300u + static_cast<uint32_t>(__ldg(zeros + static_cast<int64_t>(n) * ng + g)) * 0x00010001u;
            }
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                const uint4* xp = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K + 32 * c);
                uint4 xv[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) xv[v] = __ldg(xp + v);   // 8 bf16: columns 32c + 8v .. + 7
#pragma unroll
                for (int r = 0; r < kGvRows; ++r) {
                    const uint32_t qw[4] = {q4[r].x, q4[r].y, q4[r].z, q4[r].w};
                    float dot = 0.f;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const uint32_t w = qw[v];
                        const uint32_t xw[4] = {xv[v].x, xv[v].y, xv[v].z, xv[v].w};
                        // (q - z) pairs for columns (0, 4), (1, 5), (2, 6), (3, 7) of the word
                        const uint32_t p0 = sub_bf16x2((w & 0x000F000Fu) | 0x43004300u, zb[r]);
                        const uint32_t p1 = sub_bf16x2(((w >> 4) & 0x000F000Fu) | 0x43004300u, zb[r]);
                        const uint32_t p2 = sub_bf16x2(((w >> 8) & 0x000F000Fu) | 0x43004300u, zb[r]);
                        const uint32_t p3 = sub_bf16x2(((w >> 12) & 0x000F000Fu) | 0x43004300u, zb[r]);
                        dot = fma_f32_bf16(p0, xw[0], dot);
                        dot = fma_f32_bf16(p1, xw[0] >> 16, dot);
                        dot = fma_f32_bf16(p2, xw[1], dot);
                        dot = fma_f32_bf16(p3, xw[1] >> 16, dot);
                        dot = fma_f32_bf16(p0 >> 16, xw[2], dot);
                        dot = fma_f32_bf16(p1 >> 16, xw[2] >> 16, dot);
                        dot = fma_f32_bf16(p2 >> 16, xw[3], dot);
                        dot = fma_f32_bf16(p3 >> 16, xw[3] >> 16, dot);
                    }
                    acc[r][m] = fmaf(s[r], dot, acc[r][m]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kGvRows; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m)
#pragma unroll
                for (int o = 16; o; o >>= 1) acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], o);
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < kGvRows; ++r)
#pragma unroll
                for (int m = 0; m < MM; ++m) red[warp][r * MM + m] = acc[r][m];
        }
        __syncthreads();
        if (threadIdx.x < kGvRows * MM) {
            const int r = threadIdx.x / MM, m = threadIdx.x % MM;
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < kGvWarps; ++w) t += red[w][threadIdx.x];
            if (n0 + r < N) Y[static_cast<int64_t>(m) * N + n0 + r] = t;
        }
        __syncthreads();
    }
}

template <int MM>
int launch_gemv(float* Y, const uint16_t* X, const uint8_t* packed, const float* scales,
                const float* zeros, int N, int K, int gs, int ng, cudaStream_t stream)
{
    const int64_t tiles = (static_cast<int64_t>(N) + kGvRows - 1) / kGvRows;
    const int blocks = static_cast<int>(std::min<int64_t>(tiles, int64_t(1) << 30));
    w4a16_gemv_kernel<MM><<<blocks, kGvWarps * 32, 0, stream>>>(Y, X, packed, scales, zeros, N, K, gs, ng);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
}

// ------------------------------------------------------- tensor-core path
constexpr int kRows = 128;          // weight rows per tile = MMA M
constexpr int kStageCols = 128;     // K columns per stage
constexpr int kMaxStages = 6;
// pipeline depth per accumulator width: two CTAs fit on an SM for NP <= 32
template <int NP>
__host__ __device__ constexpr int stages_for()
{
    return NP <= 16 ? 6 : (NP <= 32 ? 5 : 4);
}
constexpr int kTcThreads = 320;     // warp 0 loads, warp 1 issues MMAs, 2..9 convert
constexpr int kConvWarps = 8;
constexpr int kTmemCols = 256;      // 2 A buffers of 64 columns + 128 accumulator columns
constexpr int kAcols = 64;          // TMEM columns of one stage's A (128 bf16 per lane)
constexpr int kWBytes = kRows * kStageCols / 2;   // packed bytes of a stage
constexpr int kMinSmem = 78 * 1024;  // at most two CTAs per SM (TMEM holds two)
// sleeps between polls of a barrier (ns): waiting warps give their issue slots
// to the converters and to the MMA thread
constexpr unsigned kSleepLoad = 200, kSleepMma = 20, kSleepConv = 60;

struct TcArgs {
    float* Y;
    const float* scales;
    const float* zeros;
    int* status;
    int M, N, K;
    int m0;       // first X row of this pass
    int gs;       // group length along K (K for one group per row)
    int gs_shift; // log2(gs) when gs is a power of two, else -1
    int ng;       // row length of scales / zeros
    int stage_bytes;
    int splits;   // CTAs along K (the cluster)
};

struct TcShared {
    uint64_t full[kMaxStages];  // TMA bytes
    uint64_t empty[kMaxStages]; // MMA commit
    uint64_t a_full[2];         // 8 converter warps
    uint64_t a_empty[2];        // MMA commit
    uint64_t slot_full[8];      // MMA commit after a group's last K step
    uint64_t slot_empty[8];     // 8 converter warps
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&v)[8])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16 with bf16 operands.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_l1(const void* p)
{
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint32_t cta_rank_in_cluster()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank)
{
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight packed columns -> four bf16 pairs (q_i - z, q_{i+4} - z), i = 0..3.
// 0x4300 | q is the bf16 of 128 + q; zz holds 128 + z twice.
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t zz, uint32_t* out)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = bf16x2_sub(((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u, zz);
}

// Group of column c (a shift when the group length is a power of two).
__device__ __forceinline__ int group_of(int c, int gs, int gs_shift)
{
    return gs_shift >= 0 ? c >> gs_shift : c / gs;
}

// Column range and groups of stage `t` (local index) of a CTA whose K range
// is [kb, ke).
struct StageGroups {
    int c0, ce;      // columns
    int g0, count;   // first group touching the stage, groups touching it
    int fin;         // groups that end inside the stage (the first `fin` of them)
};

__device__ __forceinline__ StageGroups stage_groups(int t, int kb, int ke, int gs, int gs_shift)
{
    StageGroups r;
    r.c0 = kb + t * kStageCols;
    r.ce = min(r.c0 + kStageCols, ke);
    r.g0 = group_of(r.c0, gs, gs_shift);
    if (gs <= kStageCols) {   // gs divides the stage width: every group ends inside
        r.count = group_of(r.ce - r.c0 + gs - 1, gs, gs_shift);
        r.fin = r.count;
    } else {                  // one group spans the stage
        r.count = 1;
        r.fin = (r.ce == min((r.g0 + 1) * gs, ke)) ? 1 : 0;
    }
    return r;
}

template <int NP>
__global__ void __launch_bounds__(kTcThreads, 1)
    w4a16_tc_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapX,
                    const TcArgs a)
{
    constexpr int R = 128 / NP;                 // accumulator slots
    constexpr int kStages = stages_for<NP>();
    constexpr int XBOX = NP * 128;              // bytes of one 64-column X box
    constexpr int XBYTES = 2 * XBOX;
    constexpr uint32_t kIdesc = idesc_f32acc(1 /*bf16*/, 0, 0, kRows, NP);
    // the arguments as scalars: the kernel never reads the parameter struct
    // through a reference, which after each asm statement with a memory
    // clobber would be reloaded with generic loads inside the loops
    const int K = a.K, N = a.N, M = a.M, m0 = a.m0, gs = a.gs, gs_shift = a.gs_shift;
    const int ng = a.ng, splits = a.splits, stage_bytes = a.stage_bytes;
    float* const Yout = a.Y;
    const float* const scales = a.scales;
    const float* const zeros = a.zeros;
    int* const status = a.status;
    __shared__ TcShared S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    // stage layout: X tile (1024-aligned) | packed weights
    auto xs = [base, stage_bytes](int s) { return base + s * stage_bytes; };
    auto ws = [base, stage_bytes](int s) { return base + s * stage_bytes + XBYTES; };
    float* red = reinterpret_cast<float*>(base + kStages * stage_bytes);   // [NP][128]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank_in_cluster();
    const int n0 = blockIdx.y * kRows;
    // this CTA's stages of the K range
    const int T = (K + kStageCols - 1) / kStageCols;
    const int t_begin = static_cast<int>((static_cast<int64_t>(T) * rank) / splits);
    const int t_end = static_cast<int>((static_cast<int64_t>(T) * (rank + 1)) / splits);
    const int nt = t_end - t_begin;
    const int kb = t_begin * kStageCols;
    const int ke = min(t_end * kStageCols, K);
    const int g_first = group_of(kb, gs, gs_shift);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.a_full[b], kConvWarps);
            mbar_init(&S.a_empty[b], 1);
        }
        for (int r = 0; r < R; ++r) {
            mbar_init(&S.slot_full[r], 1);
            mbar_init(&S.slot_empty[r], kConvWarps);
        }
        S.abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mapW);
        prefetch_tmap(&mapX);
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tA = S.tmem_base;              // A buffers: columns 0..127
    const uint32_t tAcc = S.tmem_base + 2 * kAcols;   // accumulator slots: 128..255
    volatile int* abort = &S.abort;
    float y[NP / 2];
#pragma unroll
    for (int j = 0; j < NP / 2; ++j) y[j] = 0.f;

    if (warp == 0) {
        // ---- loads: TMA for X and the packed weights
        if (lane == 0) {
            int issued = 0;
            for (int t = 0; t < nt; ++t) {
                const int s = t % kStages;
                if (!mbar_wait_bounded(&S.empty[s], ((t / kStages) & 1) ^ 1, abort, status, kWaitLimitCycles, kSleepLoad)) break;
                const int c0 = kb + t * kStageCols;
                mbar_arrive_expect_tx(&S.full[s], XBYTES + kWBytes);
                tma_load_2d(xs(s), &mapX, &S.full[s], c0, m0);
                tma_load_2d(xs(s) + XBOX, &mapX, &S.full[s], c0 + 64, m0);
                tma_load_2d(ws(s), &mapW, &S.full[s], c0 / 2, n0);
                ++issued;
            }
            // after a time-out, let the copies already issued land before the
            // CTA's shared memory goes away
            if (*abort) {
                for (int t = max(0, issued - kStages); t < issued; ++t)
                    mbar_wait_bounded(&S.full[t % kStages], (t / kStages) & 1, abort, nullptr,
                                      kWaitLimitCycles / 16);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issue
        if (lane == 0) {
            bool ok = true;
            for (int t = 0; t < nt && ok; ++t) {
                const int s = t % kStages;
                const int b = t & 1;
                if (!mbar_wait_bounded(&S.a_full[b], (t >> 1) & 1, abort, status, kWaitLimitCycles, kSleepMma)) break;
                tc_fence_after();
                const StageGroups sg = stage_groups(t, kb, ke, gs, gs_shift);
                const int nk = (sg.ce - sg.c0) >> 4;              // K steps in the stage
                // B descriptor of K step 0; step j starts (j / 4) boxes and
                // (j % 4) * 32 bytes further (address field in 16-byte units)
                const uint64_t bdesc0 = sdesc_sw128(smem_u32(xs(s)), 16, 1024);
                const uint32_t a0 = tA + b * kAcols;
                int j = 0;
                // the groups touching the stage, in order; per K step only the
                // MMA itself is issued
                for (int gi = 0; gi < sg.count && ok; ++gi) {
                    const int g = sg.g0 + gi;
                    const int gstart = max(g * gs, kb);        // group's first column in this CTA
                    const int gend = min((g + 1) * gs, ke);
                    const int j1 = min(nk, (gend - sg.c0) >> 4);
                    const int u = g - g_first;
                    const int slot = u % R;
                    const int jfirst = gstart >= sg.c0 ? (gstart - sg.c0) >> 4 : -1;
                    if (jfirst >= 0 && u >= R) {
                        if (!mbar_wait_bounded(&S.slot_empty[slot], ((u / R) - 1) & 1, abort, status,
                                               kWaitLimitCycles, kSleepMma)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    const uint32_t d = tAcc + slot * NP;
                    if (j == 0 && j1 == kStageCols / 16) {
                        // a whole stage inside one group: eight MMAs, straight line
#pragma unroll
                        for (int jj = 0; jj < kStageCols / 16; ++jj)
                            umma_f16_ts(d, a0 + 8 * jj,
                                        bdesc0 + static_cast<uint64_t>(((jj >> 2) * XBOX + (jj & 3) * 32) >> 4),
                                        kIdesc, jj == jfirst ? 0u : 1u);
                        j = j1;
                    }
#pragma unroll 1
                    for (; j < j1; ++j) {
                        const uint64_t bdesc =
                            bdesc0 + static_cast<uint64_t>(((j >> 2) * XBOX + (j & 3) * 32) >> 4);
                        umma_f16_ts(d, a0 + 8 * j, bdesc, kIdesc, j == jfirst ? 0u : 1u);
                    }
                    if (gend <= sg.ce) umma_commit(&S.slot_full[slot]);
                }
                if (!ok) break;
                umma_commit(&S.a_empty[b]);
                umma_commit(&S.empty[s]);
            }
        }
        __syncwarp();
    } else {
        // ---- converters and epilogue: warp w owns TMEM lanes 32 (w % 4) ..
        // +31 (= tile rows) and half h of each stage's K steps and of each
        // accumulator slot's columns
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const int rl = q * 32 + lane;                  // tile row
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        const int ct = threadIdx.x - 64;               // 0..255
        // this row's scales and zeros (rows past N read row N - 1; unused)
        const int64_t roff = static_cast<int64_t>(min(n0 + rl, N - 1)) * ng;
        const float* srow = scales + roff;
        const float* zrow = zeros + roff;

        // epilogue of the groups that end in stage tp (local index)
        auto drain = [&](int tp) -> bool {
            const StageGroups sg = stage_groups(tp, kb, ke, gs, gs_shift);
            for (int gi = 0; gi < sg.fin; ++gi) {
                const int u = sg.g0 + gi - g_first;
                const int slot = u % R;
                if (!mbar_wait_warp(&S.slot_full[slot], (u / R) & 1, abort, status, kWaitLimitCycles, kSleepConv)) return false;
                tc_fence_after();
                const float sv = __ldg(srow + sg.g0 + gi);
#pragma unroll
                for (int c8 = 0; c8 < NP / 16; ++c8) {
                    float v[8];
                    tmem_ld_32x32b_x8(tAcc + lane_addr + slot * NP + h * (NP / 2) + 8 * c8, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[8 * c8 + i] = fmaf(sv, v[i], y[8 * c8 + i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.slot_empty[slot]);
            }
            return true;
        };

        bool ok = true;
        prefetch_l1(zrow + g_first);
        prefetch_l1(srow + g_first);
        for (int t = 0; t < nt; ++t) {
            const int s = t % kStages;
            const int b = t & 1;
            {   // the next stage's zero and scale, into L1 ahead of use
                const int gn = min(group_of(kb + (t + 1) * kStageCols, gs, gs_shift), ng - 1);
                prefetch_l1(zrow + gn);
                prefetch_l1(srow + gn);
            }
            bool got = mbar_wait_warp(&S.full[s], (t / kStages) & 1, abort, status, kWaitLimitCycles, kSleepConv);
            if (got && t >= 2) got = mbar_wait_warp(&S.a_empty[b], ((t >> 1) - 1) & 1, abort, status, kWaitLimitCycles, kSleepConv);
            if (!got) { ok = false; break; }
            tc_fence_after();
            const StageGroups sg = stage_groups(t, kb, ke, gs, gs_shift);
            // X tile: within each 16-byte chunk (8 columns) order the columns
            // (0, 4, 1, 5, 2, 6, 3, 7) like the converted weight pairs
            uint4* xc = reinterpret_cast<uint4*>(xs(s));
            for (int i = ct; i < XBYTES / 16; i += 32 * kConvWarps) {
                const uint4 v = xc[i];
                uint4 o;
                o.x = __byte_perm(v.x, v.z, 0x5410);
                o.y = __byte_perm(v.x, v.z, 0x7632);
                o.z = __byte_perm(v.y, v.w, 0x5410);
                o.w = __byte_perm(v.y, v.w, 0x7632);
                xc[i] = o;
            }
            fence_async_smem();
            // weights: this warp's 4 K steps (64 columns = 32 bytes of the row)
            const uint8_t* wrow = ws(s) + rl * (kStageCols / 2) + h * 32;
            // neighbouring row pairs read the two 16-byte halves in opposite
            // order, which halves the bank conflicts of each read
            const int rot = (lane >> 1) & 1;
            const uint4 r0 = *reinterpret_cast<const uint4*>(wrow + 16 * rot);
            const uint4 r1 = *reinterpret_cast<const uint4*>(wrow + 16 * (rot ^ 1));
            const uint4 wv0 = rot ? r1 : r0;
            const uint4 wv1 = rot ? r0 : r1;
            // this warp's 64 columns lie in one group when the stage is whole
            // and groups are at least 64 columns long: one zero, no checks
            if (sg.ce - sg.c0 == kStageCols && gs >= 64) {
                const float zf = 128.f + __ldg(zrow + group_of(sg.c0 + 64 * h, gs, gs_shift));
                const uint32_t zb = __float_as_uint(zf) >> 16;   // exact: 128 + z, z in 0..15
                const uint32_t zz = zb | (zb << 16);
                const uint32_t wq[8] = {wv0.x, wv0.y, wv0.z, wv0.w, wv1.x, wv1.y, wv1.z, wv1.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t v[8];
                    dequant_word(wq[2 * jj], zz, v);
                    dequant_word(wq[2 * jj + 1], zz, v + 4);
                    tmem_st_32x32b_x8(tA + lane_addr + b * kAcols + 8 * (4 * h + jj), v);
                }
            } else {
                int gz = -1;
                float zf = 0.f;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = 4 * h + jj;
                    const int c = sg.c0 + 16 * j;
                    if (c >= sg.ce) break;   // warp-uniform
                    const int g = group_of(c, gs, gs_shift);
                    if (g != gz) {           // warp-uniform
                        zf = 128.f + __ldg(zrow + g);
                        gz = g;
                    }
                    const uint32_t zb = __float_as_uint(zf) >> 16;   // exact: 128 + z, z in 0..15
                    const uint32_t zz = zb | (zb << 16);
                    const uint32_t w0 = jj < 2 ? (jj == 0 ? wv0.x : wv0.z) : (jj == 2 ? wv1.x : wv1.z);
                    const uint32_t w1 = jj < 2 ? (jj == 0 ? wv0.y : wv0.w) : (jj == 2 ? wv1.y : wv1.w);
                    uint32_t v[8];
                    dequant_word(w0, zz, v);
                    dequant_word(w1, zz, v + 4);
                    tmem_st_32x32b_x8(tA + lane_addr + b * kAcols + 8 * j, v);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.a_full[b]);
            if (t >= 1 && !drain(t - 1)) { ok = false; break; }
        }
        if (ok && nt >= 1) drain(nt - 1);
        // partial sums of this CTA: red[m][row]
#pragma unroll
        for (int j = 0; j < NP / 2; ++j) red[(h * (NP / 2) + j) * kRows + rl] = y[j];
    }

    // ---- split-K sum over the cluster, fixed rank order
    __syncthreads();
    cluster_barrier();
    {
        const int mv = min(NP, M - m0);
        const int E = mv * kRows;
        const int e0 = static_cast<int>((static_cast<int64_t>(E) * rank) / splits);
        const int e1 = static_cast<int>((static_cast<int64_t>(E) * (rank + 1)) / splits);
        for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += kTcThreads) {
            const int m = e / kRows, r = e % kRows;
            if (n0 + r >= N) continue;
            float v = 0.f;
            for (int p = 0; p < splits; ++p) v += ld_cluster_f32(red + e, static_cast<uint32_t>(p));
            Yout[static_cast<int64_t>(m0 + m) * N + n0 + r] = v;
        }
    }
    cluster_barrier();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(S.tmem_base, kTmemCols);
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

int make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, int64_t cols,
                int64_t rows, int64_t pitch_bytes, int box_c, int box_r, CUtensorMapSwizzle swz)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(pitch_bytes)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_r)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cuda_fail_msg("w4a16: tensor map encoding", cudaErrorInvalidValue);
    return GPTQ_OK;
}

template <int NP>
int launch_tc(float* Y, const uint16_t* X, const uint8_t* packed, const float* scales,
              const float* zeros, int M, int N, int K, int gs_e, int ng, cudaStream_t stream)
{
    const int stage_bytes = 2 * NP * 128 + kWBytes;
    const int smem = std::max(1024 + stages_for<NP>() * stage_bytes + NP * kRows * 4, kMinSmem);
    // the opt-in limit is raised to what this call needs (once per size and device)
    static int attr_bytes[64] = {};
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev >= 64 || attr_bytes[dev] < smem) {
        cudaError_t e = cudaFuncSetAttribute(w4a16_tc_kernel<NP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail_msg("w4a16: shared-memory attribute", e);
        if (dev < 64) attr_bytes[dev] = smem;
    }
    CUtensorMap mapW, mapX;
    int rc = make_map_2d(&mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, K / 2, N, K / 2,
                         kStageCols / 2, kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    rc = make_map_2d(&mapX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, static_cast<int64_t>(K) * 2, 64,
                     NP, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;

    const int tiles = (N + kRows - 1) / kRows;
    const int T = (K + kStageCols - 1) / kStageCols;
    // two CTAs per SM when both fit (each also holds 1 KB the system reserves)
    const int per_sm = 2 * (smem + static_cast<int>(sizeof(TcShared)) + 1024) <= 228 * 1024 ? 2 : 1;
    int splits = (per_sm * sm_count()) / tiles;
    splits = std::max(1, std::min({splits, 8, T}));

    TcArgs args;
    args.Y = Y;
    args.scales = scales;
    args.zeros = zeros;
    args.status = device_status_ptr();
    args.M = M;
    args.N = N;
    args.K = K;
    args.gs = gs_e;
    args.gs_shift = (gs_e & (gs_e - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(gs_e)) : -1;
    args.ng = ng;
    args.stage_bytes = stage_bytes;
    args.splits = splits;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, tiles, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    for (int m0 = 0; m0 < M; m0 += NP) {
        args.m0 = m0;
        cudaError_t e = cudaLaunchKernelEx(&cfg, w4a16_tc_kernel<NP>, mapW, mapX, args);
        if (e != cudaSuccess) return cuda_fail_msg("w4a16: cluster launch", e);
        GPTQ_LAUNCH_CHECK();
    }
    return GPTQ_OK;
}

}  // namespace

// The tensor-core path takes groups contiguous along K whose length divides
// the 128-column stage or is a multiple of it (or one group per row), K a
// multiple of 32 (16-byte rows of packed codes) and 16-byte aligned operands.
bool gemv_supported(const int32_t* g_idx, int64_t M, int64_t K, int gs)
{
    return !g_idx && M >= 1 && M <= 4 && K % 32 == 0 && (gs <= 0 || gs % 32 == 0);
}

bool w4a16_tc_supported(const uint16_t* X, const uint8_t* packed, const int32_t* g_idx,
                        int64_t K, int gs)
{
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (g_idx || K % 32 != 0 || !al16(X) || !al16(packed)) return false;
    const int64_t gs_e = gs > 0 ? gs : K;
    if (gs_e % 16 != 0 && gs_e != K) return false;
    return (gs_e <= kStageCols && kStageCols % gs_e == 0) || gs_e % kStageCols == 0 || gs_e == K;
}

int run_w4a16(float* Y, const uint16_t* X, const uint8_t* packed, const float* scales,
              const float* zeros, const int32_t* g_idx, int64_t M, int64_t N, int64_t K, int gs,
              int path, cudaStream_t stream)
{
    const int ng = gs > 0 ? static_cast<int>(K / gs) : 1;
    if (path == 3 || (path == 0 && gemv_supported(g_idx, M, K, gs))) {
        const int Ni = static_cast<int>(N), Ki = static_cast<int>(K);
        switch (M) {
            case 1: return launch_gemv<1>(Y, X, packed, scales, zeros, Ni, Ki, gs, ng, stream);
            case 2: return launch_gemv<2>(Y, X, packed, scales, zeros, Ni, Ki, gs, ng, stream);
            case 3: return launch_gemv<3>(Y, X, packed, scales, zeros, Ni, Ki, gs, ng, stream);
            default: return launch_gemv<4>(Y, X, packed, scales, zeros, Ni, Ki, gs, ng, stream);
        }
    }
    const bool tc = path == 1 || (path == 0 && w4a16_tc_supported(X, packed, g_idx, K, gs));
    if (tc) {
        const int gs_e = gs > 0 ? gs : static_cast<int>(K);
        const int Mi = static_cast<int>(M), Ni = static_cast<int>(N), Ki = static_cast<int>(K);
        if (M <= 16) return launch_tc<16>(Y, X, packed, scales, zeros, Mi, Ni, Ki, gs_e, ng, stream);
        if (M <= 32) return launch_tc<32>(Y, X, packed, scales, zeros, Mi, Ni, Ki, gs_e, ng, stream);
        return launch_tc<64>(Y, X, packed, scales, zeros, Mi, Ni, Ki, gs_e, ng, stream);
    }
    const bool contiguous = !g_idx && (gs <= 0 || gs % 8 == 0);
    int blocks = static_cast<int>((N * 32 + kWThreads - 1) / kWThreads);
    blocks = std::min(blocks, sm_count() * 8);
    for (int64_t m0 = 0; m0 < M; m0 += kMTile) {
        if (contiguous)
            w4a16_simt_kernel<true><<<blocks, kWThreads, 0, stream>>>(
                Y, X, packed, scales, zeros, g_idx, static_cast<int>(M), static_cast<int>(N),
                static_cast<int>(K), gs, ng, static_cast<int>(m0));
        else
            w4a16_simt_kernel<false><<<blocks, kWThreads, 0, stream>>>(
                Y, X, packed, scales, zeros, g_idx, static_cast<int>(M), static_cast<int>(N),
                static_cast<int>(K), gs, ng, static_cast<int>(m0));
        GPTQ_LAUNCH_CHECK();
    }
    return GPTQ_OK;
}

}  // namespace gptq
