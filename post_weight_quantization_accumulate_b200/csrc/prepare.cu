// prepare.cu -- damping, activation order, and the Cholesky factor of the
// inverse Hessian.
//
// GPTQ overview page: "Hiperparametry" (a value added to the Hessian
// diagonal for numerical stability; columns quantized in order of activation
// importance) and "Komponenty" / "Jak działa" (a Cholesky decomposition of
// the inverse Hessian gives stability on large layers).
//
// Route: with P the processing order and J the index reversal,
//   A   = J P^T (H + delta I) P J          (one gather pass, delta = damp * mean diag H)
//   M   = chol_lower(A)                    (blocked, right-looking, fp32)
//   U   = J M^{-1} J                       (upper; U^T U = (P^T H_d P)^{-1})
// which needs one Cholesky and one triangular inverse (2/3 d^3 flops) instead
// of inverse + Cholesky of the inverse.  M^{-1} is accumulated alongside the
// factorisation, as forward elimination of [A | I]: once panel k is factored,
// row block k of M^{-1} is M_kk^{-1} (E_k - sum_{j<k} M_kj (M^{-1})_j), and the
// rows below receive -M_ik (M^{-1})_k right-looking, like the trailing update.
#include "common.cuh"
#include "gemm.cuh"

#include <algorithm>
#include <cstring>
#include <mutex>

namespace gptq {

struct PrepHeader {
    int status;
    float mean;
    float delta;
    int pad;
};

constexpr int kNB = 64;  // panel width of the blocked Cholesky / leaf of the inverse
constexpr int kPanelMaxCtas = 64;

size_t prepare_workspace_bytes(int64_t d)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t dd = static_cast<size_t>(d) * static_cast<size_t>(d) * sizeof(float);
    return 256 + up(dd) /*A,M*/ + up(dd) /*Minv*/;
}

namespace {

// mean(diag H) in double, delta = damp * mean (float); diagonal sanity.
__global__ void diag_mean_kernel(const float* __restrict__ H, int d, float damp, PrepHeader* hdr)
{
    __shared__ double part[32];
    __shared__ int bad[1];
    if (threadIdx.x == 0) bad[0] = 0;
    __syncthreads();
    double s = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        const float v = H[static_cast<int64_t>(i) * d + i];
        if (!isfinite(v)) bad[0] = 1;
        s += v;
    }
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
        const float mean = static_cast<float>(t / d);
        hdr->mean = mean;
        hdr->delta = damp * mean;
        if (bad[0])
            hdr->status = GPTQ_ERR_NONFINITE;
        else if (!(mean > 0.f))
            hdr->status = GPTQ_ERR_NOT_PD;
    }
}

// perm[rank(i)] = i with rank by descending diag(H), ties by lower index.
__global__ void act_order_kernel(const float* __restrict__ H, int d, int act_order,
                                 int32_t* __restrict__ perm)
{
    __shared__ float key[1024];
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (!act_order) {
        if (i < d) perm[i] = i;
        return;
    }
    const float ki = (i < d) ? H[static_cast<int64_t>(i) * d + i] : 0.f;
    int rank = 0;
    for (int j0 = 0; j0 < d; j0 += 1024) {
        __syncthreads();
        for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
            const int j = j0 + t;
            key[t] = (j < d) ? H[static_cast<int64_t>(j) * d + j] : 0.f;
        }
        __syncthreads();
        const int jn = min(1024, d - j0);
        for (int t = 0; t < jn; ++t) {
            const float kj = key[t];
            rank += (kj > ki) || (kj == ki && j0 + t < i);
        }
    }
    if (i < d) perm[rank] = i;
}

// A[a][b] = H[q(a)][q(b)] + (a == b ? delta : 0), q(a) = perm[d-1-a]; the
// reversed order q staged once per CTA and one row of H at a time, both in
// shared memory (2 d floats, d <= kGatherSmemMax); rows read and written with
// 16-byte accesses when d % 4 == 0 and H is 16-byte aligned.
constexpr int kGatherSmemMax = 16384;
__global__ void gather_rev_kernel(const float* __restrict__ H, int d,
                                  const int32_t* __restrict__ perm, const PrepHeader* hdr,
                                  float* __restrict__ A)
{
    extern __shared__ float gsm[];
    float* rowbuf = gsm;
    int* q = reinterpret_cast<int*>(gsm + d);
    const float delta = hdr->delta;
    const bool vec = (d % 4) == 0 && (reinterpret_cast<uintptr_t>(H) & 15) == 0;
    for (int b = threadIdx.x; b < d; b += blockDim.x) q[b] = perm[d - 1 - b];
    for (int a = blockIdx.x; a < d; a += gridDim.x) {
        __syncthreads();   // q staged; the previous row's reads of rowbuf done
        const float* src = H + static_cast<int64_t>(q[a]) * d;
        if (vec) {
            for (int j = threadIdx.x; j < d / 4; j += blockDim.x)
                reinterpret_cast<float4*>(rowbuf)[j] = reinterpret_cast<const float4*>(src)[j];
        } else {
            for (int j = threadIdx.x; j < d; j += blockDim.x) rowbuf[j] = src[j];
        }
        __syncthreads();
        float* dst = A + static_cast<int64_t>(a) * d;
        if (vec) {
            for (int j = threadIdx.x; j < d / 4; j += blockDim.x) {
                const int b = 4 * j;
                float4 v = make_float4(rowbuf[q[b]], rowbuf[q[b + 1]], rowbuf[q[b + 2]], rowbuf[q[b + 3]]);
                if (a == b) v.x += delta;
                if (a == b + 1) v.y += delta;
                if (a == b + 2) v.z += delta;
                if (a == b + 3) v.w += delta;
                reinterpret_cast<float4*>(dst)[j] = v;
            }
        } else {
            for (int b = threadIdx.x; b < d; b += blockDim.x) {
                float v = rowbuf[q[b]];
                if (b == a) v += delta;
                dst[b] = v;
            }
        }
    }
}

__global__ void gather_rev_direct_kernel(const float* __restrict__ H, int d,
                                         const int32_t* __restrict__ perm, const PrepHeader* hdr,
                                         float* __restrict__ A)
{
    const float delta = hdr->delta;
    const int64_t n = static_cast<int64_t>(d) * d;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int a = static_cast<int>(idx / d), b = static_cast<int>(idx % d);
        float v = H[static_cast<int64_t>(perm[d - 1 - a]) * d + perm[d - 1 - b]];
        if (a == b) v += delta;
        A[idx] = v;
    }
}

// Without a reordering (perm = identity) the gather is a reversed copy:
// A[a][b] = H[d-1-a][d-1-b] (+ delta on the diagonal), four columns per
// thread with 16-byte loads and stores (d % 4 == 0, H and A 16-byte aligned).
__global__ void reverse_copy_kernel(const float* __restrict__ H, int d, const PrepHeader* hdr,
                                    float* __restrict__ A)
{
    const float delta = hdr->delta;
    const int q = d / 4;
    const int64_t n = static_cast<int64_t>(d) * q;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int a = static_cast<int>(idx / q), b = 4 * static_cast<int>(idx % q);
        const float4 h = *reinterpret_cast<const float4*>(H + static_cast<int64_t>(d - 1 - a) * d + (d - 4 - b));
        float4 v = make_float4(h.w, h.z, h.y, h.x);   // columns b .. b+3 of A
        if (a == b) v.x += delta;
        if (a == b + 1) v.y += delta;
        if (a == b + 2) v.z += delta;
        if (a == b + 3) v.w += delta;
        *reinterpret_cast<float4*>(A + static_cast<int64_t>(a) * d + b) = v;
    }
}

// One panel step of the blocked Cholesky, fused:
//   every CTA factors the kb x kb diagonal block at (k0, k0) (redundantly, so
//   no other launch has to wait for it); CTA 0 writes L_kk^{-1} (the solve
//   with the identity) into M^{-1}; CTA b in 1..n_trsm solves the panel rows
//   k0+kb+64(b-1) .. +63:  L[r][k0:k0+kb] = A[r][k0:k0+kb] L_kk^{-T};
//   CTA n_trsm+1+c finishes column block c < k0/64 of row block k of M^{-1}:
//   Y_k = L_kk^{-1} (Y~_k - L_k,k-1 Y_{k-1}), Y~_k holding the updates of the
//   panels before k-1 (applied in memory by the side stream).
// Factorisation of the 64 x 64 block in shared memory, in 16 strips of 4
// columns: warp 0 factors the strip with shuffles (lane l holds rows 4P+l and
// 4P+l+32), then all warps subtract its rank-4 product from the trailing
// lower triangle (thread (ty, tx) owns the 4 x 4 tile rows 4ty.., cols 4tx..).
// The factor is then used through triangular solves, never inverted as a
// whole: the panel rows P solve P L^T = T and the row block of M^{-1} solves
// L X = T (as X^T L^T = T^T), by blocked substitution (solve_rows: 16 columns
// at a time by one thread per row, then the block's product subtracted from
// the later columns by all threads).  The diagonal block of M^{-1} is the
// solve with T = I.
// The previous panel's rows enter every product of the kernel as its k index
// (the 64 columns of that panel), so they are kept k-major: KTile[k][r] with
// 16-byte aligned rows, read four rows (or columns) of the product at a time.
typedef float Tile64[kNB + 1];
constexpr int kLTld = kNB + 4;   // row pitch of k-major tiles: 16-byte aligned rows
typedef float KTile[kLTld];
constexpr size_t kPanelSmem = (2 * kNB * (kNB + 1) + 3 * kNB * kLTld + kNB + 2 * 4 * kLTld) * sizeof(float) + 16;
static_assert((2 * kNB * (kNB + 1) * sizeof(float)) % 16 == 0, "the k-major tiles start 16-byte aligned");

// 4-byte asynchronous copy global -> shared; `valid` false writes a zero.
__device__ __forceinline__ void cp_async4(void* dst, const float* src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 4 : 0)
                 : "memory");
}

// 64 x 64 tile of A (rows r_begin.., columns c_begin..) into smem by
// asynchronous copies (one commit group); rows >= nrows or columns >= ncols
// read as 0.  Completes at cp.async.wait_group.
__device__ __forceinline__ void load_tile_async(Tile64* dst, const float* A, int d, int r_begin, int nrows,
                                                int c_begin, int ncols)
{
    const int tid = threadIdx.x;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        const bool valid = i < nrows && j < ncols;
        cp_async4(&dst[i][j], valid ? A + static_cast<int64_t>(r_begin + i) * d + c_begin + j : A, valid);
    }
}

// 64 x 64 tile of A into a k-major tile, asynchronously: transposed
// (dst[j][i] = A[r_begin + i][c_begin + j]) or as it is (dst[i][j]).
__device__ __forceinline__ void load_ktile_async(KTile* dst, const float* A, int d, int r_begin, int nrows,
                                                 int c_begin, int ncols, bool transpose)
{
    const int tid = threadIdx.x;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        const bool valid = i < nrows && j < ncols;
        float* slot = transpose ? &dst[j][i] : &dst[i][j];
        cp_async4(slot, valid ? A + static_cast<int64_t>(r_begin + i) * d + c_begin + j : A, valid);
    }
}

__device__ __forceinline__ void load_ktile(KTile* dst, const float* A, int d, int r_begin, int nrows,
                                           int c_begin, int ncols, bool transpose)
{
    const int tid = threadIdx.x;
    float tv[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        tv[t] = (i < nrows && j < ncols) ? A[static_cast<int64_t>(r_begin + i) * d + c_begin + j] : 0.f;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        if (transpose)
            dst[j][i] = tv[t];
        else
            dst[i][j] = tv[t];
    }
}

// acc[i][j] (tile rows r0.., cols c0..) -= sum_k X[k][r0 + i] Y[k][c0 + j], X
// and Y k-major: per k one 16-byte load of each, 16 fmas as 8 paired fmas
// (two independent IEEE fmas each, the bits of 16 fmaf).
__device__ __forceinline__ void tile_minus_kmajor(float (&acc)[4][4], const KTile* X, const KTile* Y,
                                                  int r0, int c0)
{
#pragma unroll 4
    for (int k = 0; k < kNB; ++k) {
        const float4 xv = *reinterpret_cast<const float4*>(&X[k][r0]);
        const float4 yv = *reinterpret_cast<const float4*>(&Y[k][c0]);
        const float xs[4] = {-xv.x, -xv.y, -xv.z, -xv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 nx = make_float2(xs[i], xs[i]);
            float2 a = make_float2(acc[i][0], acc[i][1]);
            float2 b = make_float2(acc[i][2], acc[i][3]);
            a = __ffma2_rn(nx, make_float2(yv.x, yv.y), a);
            b = __ffma2_rn(nx, make_float2(yv.z, yv.w), b);
            acc[i][0] = a.x;
            acc[i][1] = a.y;
            acc[i][2] = b.x;
            acc[i][3] = b.y;
        }
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The first nrows x ncols entries of a tile back to A (rows r_begin..,
// columns c_begin..), coalesced.
__device__ __forceinline__ void store_tile(const Tile64* src, float* A, int d, int r_begin, int nrows,
                                           int c_begin, int ncols)
{
    const int tid = threadIdx.x;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        if (i < nrows && j < ncols) A[static_cast<int64_t>(r_begin + i) * d + c_begin + j] = src[i][j];
    }
}

// The same for a tile that holds the block transposed: A[r_begin + i][c_begin
// + j] = src[j][i].
__device__ __forceinline__ void store_tile_t(const Tile64* src, float* A, int d, int r_begin, int nrows,
                                             int c_begin, int ncols)
{
    const int tid = threadIdx.x;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        if (i < nrows && j < ncols) A[static_cast<int64_t>(r_begin + i) * d + c_begin + j] = src[j][i];
    }
}

// 64 x 64 tile of A (rows r_begin.., columns c_begin..c_begin+ncols) into smem;
// rows >= d or columns >= ncols read as `pad` on the diagonal, 0 elsewhere
// (lower_only: entries above the diagonal read as 0 too).
__device__ __forceinline__ void load_tile(Tile64* dst, const float* A, int d, int r_begin, int nrows,
                                          int c_begin, int ncols, bool lower_only, bool pad_identity)
{
    const int tid = threadIdx.x;
    float tv[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        float v = (pad_identity && i == j) ? 1.f : 0.f;
        if (i < nrows && j < ncols && (!lower_only || j <= i))
            v = A[static_cast<int64_t>(r_begin + i) * d + c_begin + j];
        tv[t] = v;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        dst[idx / kNB][idx % kNB] = tv[t];
    }
}

// The 64 rows of S (a 64 x 64 right-hand side in shared memory) solved in
// place against the panel's factor: row r becomes p with p L^T = S[r], i.e.
// for s = 0 .. 63, p[s] = S[r][s] / L[s][s] and S[r][e] -= p[s] L[e][s] for
// e > s.  LT is L transposed (LT[s][e] = L[e][s], kLTld floats per row),
// rls[s] = 1 / L[s][s].  Blocked by 16 columns: one thread per row solves a
// block's 16 columns step by step (its entries in registers, L's entries by
// broadcast loads), then all 256 threads subtract the block's product from
// the columns to its right, 4 x 4 entries each.  Called by every thread.
__device__ __forceinline__ void solve_rows(Tile64* S, const float* __restrict__ LT,
                                           const float* __restrict__ rls)
{
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
#pragma unroll 1
    for (int b = 0; b < kNB / 16; ++b) {
        const int b0 = 16 * b;
        if (tid < kNB) {
            float t[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = S[tid][b0 + e];
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const float v = t[s] * rls[b0 + s];
                t[s] = v;
                const float* lt = LT + (b0 + s) * kLTld + b0;
#pragma unroll
                for (int e = s + 1; e < 16; ++e) t[e] = fmaf(-v, lt[e], t[e]);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) S[tid][b0 + e] = t[e];
        }
        __syncthreads();
        const int c0 = b0 + 16 + 4 * tx;   // 4 x 4 entries: rows 4 ty .., columns c0 ..
        if (c0 < kNB) {
            const int r0 = 4 * ty;
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = S[r0 + i][c0 + j];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float4 l4 = *reinterpret_cast<const float4*>(LT + (b0 + k) * kLTld + c0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float p = S[r0 + i][b0 + k];
                    acc[i][0] = fmaf(-p, l4.x, acc[i][0]);
                    acc[i][1] = fmaf(-p, l4.y, acc[i][1]);
                    acc[i][2] = fmaf(-p, l4.z, acc[i][2]);
                    acc[i][3] = fmaf(-p, l4.w, acc[i][3]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) S[r0 + i][c0 + j] = acc[i][j];
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(256)
    chol_panel_kernel(float* __restrict__ A, int d, int k0, int kb, int pk0,
                      float* __restrict__ Minv, PrepHeader* hdr)
{
    extern __shared__ __align__(16) float psm[];
    Tile64* As = reinterpret_cast<Tile64*>(psm);
    Tile64* Ts = As + kNB;       // this CTA's operand tile (panel rows, or a block of M^{-1})
    KTile* Pd = reinterpret_cast<KTile*>(Ts + kNB);   // previous panel, rows of this diagonal block, k-major
    KTile* Pr = Pd + kNB;        // previous panel's rows of this CTA's panel block (k-major), or Y_{k-1}
    float* LT = reinterpret_cast<float*>(Pr + kNB);   // the factor transposed, [kNB][kLTld]
    float* rls = LT + kNB * kLTld;                     // 1 / L[i][i]
    float* LsT = rls + kNB;      // a strip's 4 columns of L, k-major, two buffers of [4][kLTld]
    int& bad_any = *reinterpret_cast<int*>(LsT + 2 * 4 * kLTld);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ty = tid >> 4, tx = tid & 15;
    const int r0 = 4 * ty, c0 = 4 * tx;
    // Second-phase work items: n_trsm blocks of 64 panel rows, then (from the
    // second panel on) k0/64 column blocks of M^{-1}'s row block; CTA b >= 1
    // takes items b-1, b-1 + (G-1), ...
    const int n_trsm = (d - k0 - kb + kNB - 1) / kNB;
    const int n_items = n_trsm + (pk0 >= 0 ? k0 / kNB : 0);
    const int stride = static_cast<int>(gridDim.x) - 1;
    auto fetch_item = [&](int it, bool async) {
        if (it >= n_trsm) {
            const int cb = (it - n_trsm) * kNB;
            if (async) {
                load_tile_async(Ts, Minv, d, k0, kb, cb, kNB);              // Y~_k
                load_ktile_async(Pr, Minv, d, pk0, kNB, cb, kNB, false);    // Y_{k-1}, [k][c]
            } else {
                load_tile(Ts, Minv, d, k0, kb, cb, kNB, false, false);
                load_ktile(Pr, Minv, d, pk0, kNB, cb, kNB, false);
            }
        } else {
            const int pr0 = k0 + kb + it * kNB;
            const int prn = min(kNB, d - pr0);
            if (async) {
                load_tile_async(Ts, A, d, pr0, prn, k0, kb);
                if (pk0 >= 0) load_ktile_async(Pr, A, d, pr0, prn, pk0, kNB, true);
            } else {
                load_tile(Ts, A, d, pr0, prn, k0, kb, false, false);
                if (pk0 >= 0) load_ktile(Pr, A, d, pr0, prn, pk0, kNB, true);
            }
        }
    };

    // The diagonal block (lower part; padding beyond kb is the identity) and
    // the previous panel's rows of it are read first, in one round trip; the
    // operand tiles of the first item do not depend on the diagonal block, so
    // they are fetched asynchronously afterwards, while it is factored.
    float ta[16], tp[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        float v = (i == j) ? 1.f : 0.f;
        if (i < kb && j <= i) v = A[static_cast<int64_t>(k0 + i) * d + k0 + j];
        ta[t] = v;
        tp[t] = (pk0 >= 0 && i < kb) ? A[static_cast<int64_t>(k0 + i) * d + pk0 + j] : 0.f;
    }
    if (blockIdx.x > 0 && static_cast<int>(blockIdx.x) - 1 < n_items) fetch_item(blockIdx.x - 1, true);
    cp_async_commit();
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int idx = tid + t * 256;
        const int i = idx / kNB, j = idx % kNB;
        As[i][j] = ta[t];
        Pd[j][i] = tp[t];   // k-major
    }
    if (tid == 0) bad_any = 0;
    __syncthreads();
    // This thread's 4 x 4 tile of the diagonal block (tiles on and below the
    // diagonal) stays in registers through the previous panel's correction
    // and every strip's update; it is written back to shared memory once, at
    // the strip before the one that needs its columns, and not re-read in
    // between.
    const bool own = ty >= tx;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = As[r0 + i][c0 + j];
    // A_kk -= P_prev,kk P_prev,kk^T: the previous panel's correction of this
    // block column, applied here rather than in memory
    if (pk0 >= 0 && own) tile_minus_kmajor(acc, Pd, Pd, r0, c0);
    auto flush = [&]() {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) As[r0 + i][c0 + j] = acc[i][j];
    };
    if (own && tx <= 1) flush();   // the columns of strips 0 and 1
    __syncthreads();
    bool bad = false;

    // Strips of 4 columns with look-ahead: while warps 1-7 subtract strip P's
    // rank-4 product from their tiles right of strip P+1, warp 0 applies it to
    // strip P+1 itself and factors that strip, so each strip costs one barrier
    // and the long update is off the chain.  Warp 0 keeps rows 4P+l and
    // 4P+l+32 of a strip in registers (lane l), and publishes the strip's L
    // both in As (for the solves later) and k-major in LsT (for the updates).
    // Every lane factors the strip's 4 x 4 diagonal block itself, from the
    // lower entries it gathers with independent shuffles, then its own rows
    // with the same steps (so lanes 0-3, the block's rows, match it bit for
    // bit): no shuffle waits on the previous column.
    auto factor_strip = [&](int cb, float (&x)[4], float (&y)[4], float* ls) {
        float D[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j <= i; ++j) D[i][j] = __shfl_sync(0xffffffffu, x[j], i);
        float rs[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float piv = D[c][c];
            if (!(piv > 0.f) || !isfinite(piv)) {
                bad = true;
                piv = 1.f;
            }
            rs[c] = rsqrtf(piv);
#pragma unroll
            for (int i = c; i < 4; ++i) D[i][c] = D[i][c] * rs[c];
#pragma unroll
            for (int j = c + 1; j < 4; ++j)
#pragma unroll
                for (int i = j; i < 4; ++i) D[i][j] = fmaf(-D[i][c], D[j][c], D[i][j]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float lx = x[c] * rs[c], ly = y[c] * rs[c];
            x[c] = lx;
            y[c] = ly;
#pragma unroll
            for (int j = c + 1; j < 4; ++j) {
                x[j] = fmaf(-lx, D[j][c], x[j]);
                y[j] = fmaf(-ly, D[j][c], y[j]);
            }
        }
        const int ra = cb + lane, rb = cb + lane + 32;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            if (ra < kNB) {
                As[ra][cb + t] = x[t];
                ls[t * kLTld + ra] = x[t];
            }
            if (rb < kNB) {
                As[rb][cb + t] = y[t];
                ls[t * kLTld + rb] = y[t];
            }
        }
    };
    if (warp == 0) {
        float x[4], y[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            x[t] = As[lane][t];
            y[t] = As[lane + 32][t];
        }
        factor_strip(0, x, y, LsT);
    }
    __syncthreads();
    for (int P = 0; P < kNB / 4; ++P) {
        const int cb = 4 * P;
        const float* lcur = LsT + (P & 1) * 4 * kLTld;   // strip P, k-major
        if (warp == 0) {
            if (P + 1 < kNB / 4) {
                const int nb = cb + 4;
                const int ra = nb + lane, rb = nb + lane + 32;
                float lstrip[4][4];   // L[nb + t][cb + u]
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int u = 0; u < 4; ++u) lstrip[t][u] = lcur[u * kLTld + nb + t];
                float x[4], y[4], la[4], lb[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    la[u] = ra < kNB ? lcur[u * kLTld + ra] : 0.f;
                    lb[u] = rb < kNB ? lcur[u * kLTld + rb] : 0.f;
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    float xa = ra < kNB ? As[ra][nb + t] : 0.f;
                    float ya = rb < kNB ? As[rb][nb + t] : 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        xa = fmaf(-la[u], lstrip[t][u], xa);
                        ya = fmaf(-lb[u], lstrip[t][u], ya);
                    }
                    x[t] = xa;
                    y[t] = ya;
                }
                factor_strip(nb, x, y, LsT + ((P + 1) & 1) * 4 * kLTld);
            }
        } else if (own && tx > P + 1) {
            float li[4][4], lj[4][4];   // L[r0 + i][cb + t], L[c0 + j][cb + t]
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float4 a4 = *reinterpret_cast<const float4*>(lcur + t * kLTld + r0);
                const float4 b4 = *reinterpret_cast<const float4*>(lcur + t * kLTld + c0);
                li[0][t] = a4.x;
                li[1][t] = a4.y;
                li[2][t] = a4.z;
                li[3][t] = a4.w;
                lj[0][t] = b4.x;
                lj[1][t] = b4.y;
                lj[2][t] = b4.z;
                lj[3][t] = b4.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int t = 0; t < 4; ++t) acc[i][j] = fmaf(-li[i][t], lj[j][t], acc[i][j]);
            if (tx == P + 2) flush();   // warp 0 reads these columns next strip
        }
        __syncthreads();
    }

    // the factor transposed for the solves, and the reciprocals of its diagonal
    for (int idx = tid; idx < kNB * kNB; idx += 256) {
        const int sj = idx / kNB, e = idx % kNB;
        LT[sj * kLTld + e] = (e >= sj) ? As[e][sj] : 0.f;
    }
    if (tid < kNB) rls[tid] = 1.f / As[tid][tid];
    if (bad) bad_any = 1;
    __syncthreads();
    if (bad_any && tid == 0 && blockIdx.x == 0) atomicCAS(&hdr->status, 0, GPTQ_ERR_NOT_PD);


    if (blockIdx.x == 0) {
        // diagonal block of M^{-1}: L^{-1}, the solve L X = I column by column
        // (L_kk itself is not needed later -- the trailing updates use the
        // off-diagonal panels -- and the other CTAs of this launch may still be
        // reading the diagonal block of A, so only M^{-1} is written)
        // (the transposed problem: rows of X^T solve X^T L^T = I)
        for (int idx = tid; idx < kNB * kNB; idx += 256) Ts[idx / kNB][idx % kNB] = (idx / kNB == idx % kNB) ? 1.f : 0.f;
        __syncthreads();
        solve_rows(Ts, LT, rls);
        store_tile_t(Ts, Minv, d, k0, kb, k0, kb);
        return;
    }
    cp_async_wait_all();
    for (int it = blockIdx.x - 1; it < n_items; it += stride) {
        if (it != static_cast<int>(blockIdx.x) - 1) {
            __syncthreads();   // the previous item is done with Ts, Pr and As
            fetch_item(it, false);
        }
        __syncthreads();
        if (it >= n_trsm) {
            // column block cb of row block k of M^{-1} (pk0 >= 0 here):
            // T = Y~_k - L_k,k-1 Y_{k-1}, then X = L_kk^{-1} T
            const int cb = (it - n_trsm) * kNB;
            float t4[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) t4[i][j] = Ts[r0 + i][c0 + j];
            tile_minus_kmajor(t4, Pd, Pr, r0, c0);
            // T transposed into As (the factor lives on in LT): the rows of
            // X^T solve X^T L^T = T^T
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) As[c0 + j][r0 + i] = t4[i][j];
            __syncthreads();
            solve_rows(As, LT, rls);
            store_tile_t(As, Minv, d, k0, kb, cb, kNB);
            continue;
        }
        // panel rows: T = A[rows][block] - P_prev[rows] P_prev,kk^T, then
        // P solves P L^T = T
        const int pr0 = k0 + kb + it * kNB;
        if (pk0 >= 0) {
            float t4[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) t4[i][j] = Ts[r0 + i][c0 + j];
            tile_minus_kmajor(t4, Pr, Pd, r0, c0);
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) Ts[r0 + i][c0 + j] = t4[i][j];
            __syncthreads();
        }
        solve_rows(Ts, LT, rls);
        store_tile(Ts, A, d, pr0, min(kNB, d - pr0), k0, kb);
    }
}

// U[i][j] = Minv[d-1-i][d-1-j] for i <= j, 0 below the diagonal.
__global__ void reverse_upper_kernel(const float* __restrict__ Minv, int d, float* __restrict__ U)
{
    const int64_t n = static_cast<int64_t>(d) * d;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(idx / d), j = static_cast<int>(idx % d);
        U[idx] = (i <= j) ? Minv[static_cast<int64_t>(d - 1 - i) * d + (d - 1 - j)] : 0.f;
    }
}

}  // namespace

// Side streams of the factorisation (one set per device, created on first
// use) with their events; the caller's stream forks to them and joins them.
struct SideStream {
    static constexpr int kRing = 4;
    cudaStream_t sp = nullptr;         // the chain of panel kernels
    cudaStream_t s = nullptr;          // narrow and band updates of A
    cudaStream_t s2 = nullptr;         // narrow and band updates of M^{-1}
    cudaStream_t s3 = nullptr;         // far updates of A
    cudaStream_t s4 = nullptr;         // far updates of M^{-1}
    cudaEvent_t fork = nullptr, join = nullptr, join2 = nullptr, join3 = nullptr, join4 = nullptr;
    cudaEvent_t ready = nullptr, join_p = nullptr, done_panel = nullptr, cleared = nullptr;
    cudaEvent_t ev[kRing] = {}, ev2[kRing] = {};     // narrow/band work of a panel done
    cudaEvent_t far[kRing] = {}, far2[kRing] = {};   // far update of a batch done
};

static int side_stream(SideStream** out)
{
    static SideStream streams[64];
    static std::mutex mu;
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return GPTQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(mu);
    SideStream& st = streams[dev];
    if (!st.s) {
        // the panel chain and the products it waits for at the highest
        // priority, the far updates at the lowest: when a far product's CTA
        // retires, a waiting CTA of the chain takes the SM first
        int lo = 0, hi = 0;
        GPTQ_CUDA_CHECK(cudaDeviceGetStreamPriorityRange(&lo, &hi));
        GPTQ_CUDA_CHECK(cudaStreamCreateWithPriority(&st.sp, cudaStreamNonBlocking, hi));
        GPTQ_CUDA_CHECK(cudaStreamCreateWithPriority(&st.s, cudaStreamNonBlocking, hi));
        GPTQ_CUDA_CHECK(cudaStreamCreateWithPriority(&st.s2, cudaStreamNonBlocking, hi));
        GPTQ_CUDA_CHECK(cudaStreamCreateWithPriority(&st.s3, cudaStreamNonBlocking, lo));
        GPTQ_CUDA_CHECK(cudaStreamCreateWithPriority(&st.s4, cudaStreamNonBlocking, lo));
        for (cudaEvent_t* e : {&st.fork, &st.join, &st.join2, &st.join3, &st.join4, &st.ready,
                               &st.join_p, &st.done_panel, &st.cleared})
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
        for (int i = 0; i < SideStream::kRing; ++i) {
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&st.ev[i], cudaEventDisableTiming));
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&st.ev2[i], cudaEventDisableTiming));
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&st.far[i], cudaEventDisableTiming));
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&st.far2[i], cudaEventDisableTiming));
        }
    }
    *out = &st;
    return GPTQ_OK;
}

// Enqueues the whole factorisation on `stream`; the status word of the run
// is copied into the pinned word status_host.
static int enqueue_prepare(const float* H, int64_t d64, float damp, int act_order, int32_t* perm,
                           float* U, void* workspace, cudaStream_t stream, int* status_host)
{
    const int d = static_cast<int>(d64);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t dd = static_cast<size_t>(d) * d * sizeof(float);
    PrepHeader* hdr = reinterpret_cast<PrepHeader*>(ws);
    float* A = reinterpret_cast<float*>(ws + 256);
    float* Minv = reinterpret_cast<float*>(ws + 256 + up(dd));
    const int nsm = sm_count();

    SideStream* side = nullptr;
    int rc = side_stream(&side);
    if (rc) return rc;
    // M^{-1} starts as zeros (its row blocks are accumulated in place); the
    // clear runs on the second side stream next to the gather
    GPTQ_CUDA_CHECK(cudaEventRecord(side->fork, stream));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s, side->fork, 0));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s2, side->fork, 0));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s3, side->fork, 0));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s4, side->fork, 0));
    GPTQ_CUDA_CHECK(cudaMemsetAsync(Minv, 0, dd, side->s2));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->cleared, side->s2));

    GPTQ_CUDA_CHECK(cudaMemsetAsync(hdr, 0, sizeof(PrepHeader), stream));
    diag_mean_kernel<<<1, 1024, 0, stream>>>(H, d, damp, hdr);
    GPTQ_LAUNCH_CHECK();
    act_order_kernel<<<(d + 255) / 256, 256, 0, stream>>>(H, d, act_order, perm);
    GPTQ_LAUNCH_CHECK();
    if (!act_order && d % 4 == 0 && (reinterpret_cast<uintptr_t>(H) & 15) == 0) {
        const int64_t n4 = static_cast<int64_t>(d) * (d / 4);
        reverse_copy_kernel<<<static_cast<int>(std::min<int64_t>((n4 + 255) / 256, nsm * 8)), 256, 0,
                              stream>>>(H, d, hdr, A);
    } else if (d <= kGatherSmemMax) {
        const size_t sm = 2 * static_cast<size_t>(d) * sizeof(float);
        static bool attr[64] = {};   // per device: the attribute is set per context
        int dev = 0;
        GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
        if (dev < 0 || dev >= 64) return GPTQ_ERR_UNSUPPORTED;
        if (!attr[dev]) {
            GPTQ_CUDA_CHECK(cudaFuncSetAttribute(gather_rev_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 2 * kGatherSmemMax * static_cast<int>(sizeof(float))));
            attr[dev] = true;
        }
        // CTAs per SM that fit next to each other, about two rows each
        const int per_sm = std::max(1, static_cast<int>((220u * 1024u) / (sm + 1024)));
        gather_rev_kernel<<<std::min(d, nsm * per_sm), 256, sm, stream>>>(H, d, perm, hdr, A);
    } else {
        gather_rev_direct_kernel<<<nsm * 8, 256, 0, stream>>>(H, d, perm, hdr, A);
    }
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->cleared, 0));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->ready, stream));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->sp, side->ready, 0));

    // Blocked right-looking Cholesky, A = M M^T (lower), with look-ahead:
    // panel k+1 applies panel k's correction to its own block column (and to
    // its row block of M^{-1}) on the fly.  The corrections below block k+1
    // are split by distance.  Panels form batches of kBatch (256 columns);
    // for panel q of batch b, with E_b = (kBatch (b + 2)) kNB:
    //   narrow(q)  K = 64: columns [(q + 2) kNB, E_b) of A and the same row
    //              blocks of M^{-1}, right after panel q; panel q + 2 waits
    //              for it;
    //   band(b)    K = 256, after the batch's last panel, on the narrow
    //              streams: the batch's correction of columns (row blocks of
    //              M^{-1}) [E_b, E_b + 256), which narrow(q') of the next
    //              batch writes as well, so it goes first;
    //   far(b)     K = 256: everything from E_b + 256 on, on streams of its
    //              own, overlapping the next panels: first the head (the
    //              256 columns band(b + 1) writes as well, so band(b + 1)
    //              waits for it), then the tail, which band(b + 2) meets only
    //              behind far(b + 1)'s head on the same stream.
    // Every region thus receives its corrections in one fixed order (the
    // factorisation is bitwise reproducible), and the bulk of the trailing
    // work runs as K = 256 products: a quarter of the HBM traffic of
    // rank-64 updates, which bound the factorisation at d = 11008.  The
    // critical path is the chain of panel kernels (stream sp).  The far
    // products run one CTA per tile at the lowest priority: they fill the
    // SMs the chain leaves and give them back tile by tile.
    constexpr int kBatch = 8;
    constexpr int kBW = kBatch * kNB;
    constexpr int kBatchMinDim = 7168;
    const int n_panels = (d + kNB - 1) / kNB;
    {
        static bool attr_panel[64] = {};
        int dev = 0;
        GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
        if (dev < 64 && !attr_panel[dev]) {
            GPTQ_CUDA_CHECK(cudaFuncSetAttribute(chol_panel_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kPanelSmem)));
            attr_panel[dev] = true;
        }
    }
    // CTA caps of a pair of products (A, M^{-1}) sharing `sms` SMs in
    // proportion to their flops
    auto split = [](int sms, double f_a, double f_inv, int* c_a, int* c_inv) {
        const double t = f_a + f_inv;
        *c_a = std::max(8, static_cast<int>(sms * (t > 0 ? f_a / t : 0.5) + 0.5));
        *c_inv = std::max(8, sms - *c_a);
    };
    for (int p = 0; p < n_panels; ++p) {
        const int k0 = p * kNB;
        const int kb = std::min(kNB, d - k0);
        const int rest = d - k0 - kb;
        const int n_trsm = (rest + kNB - 1) / kNB;
        // CTA 0 writes L_kk^{-1}; the others share the panel's work items, at
        // most kPanelMaxCtas of them so the side products keep enough SMs
        const int n_cta = std::min(1 + n_trsm + p, kPanelMaxCtas);
        const int free_sm = std::max(16, nsm - n_cta);
        if (p >= 2) {
            GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->sp, side->ev[(p - 2) % SideStream::kRing], 0));
            GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->sp, side->ev2[(p - 2) % SideStream::kRing], 0));
        }
        chol_panel_kernel<<<n_cta, 256, kPanelSmem, side->sp>>>(A, d, k0, kb, p > 0 ? k0 - kNB : -1,
                                                                Minv, hdr);
        GPTQ_LAUNCH_CHECK();
        GPTQ_CUDA_CHECK(cudaEventRecord(side->done_panel, side->sp));
        GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s, side->done_panel, 0));
        GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s2, side->done_panel, 0));
        const int b = p / kBatch;
        // below kBatchMinDim every correction is narrow: columns [r0, d)
        const int64_t e_b = d >= kBatchMinDim ? static_cast<int64_t>(kBatch) * (b + 2) * kNB : d;
        const bool batch_end = p % kBatch == kBatch - 1 && e_b < d;
        const bool has_far = batch_end && e_b + kBW < d;
        const int r0 = k0 + kb + kNB;   // first row/column below block k+1
        const int c1 = static_cast<int>(std::min<int64_t>(e_b, d));
        if (r0 < c1) {
            const int m = d - r0, n = c1 - r0;
            int ca = 0, ci = 0;
            split(free_sm, 0.5 * n * n + double(m - n) * n, double(n) * (k0 + kb), &ca, &ci);
            float* P = A + static_cast<int64_t>(r0) * d + k0;
            rc = launch_sgemm(true, m, n, kb, -1.f, P, d, 0, P, d, 0, 1.f,
                              A + static_cast<int64_t>(r0) * d + r0, d, 0, 1, kGemmLowerC, side->s, ca);
            if (rc) return rc;
            // (M^{-1})[r0 : c1][0 : k0+kb] -= M[r0 : c1][k] (M^{-1})_k
            rc = launch_sgemm(false, n, k0 + kb, kb, -1.f, P, d, 0, Minv + static_cast<int64_t>(k0) * d, d,
                              0, 1.f, Minv + static_cast<int64_t>(r0) * d, d, 0, 1, 0, side->s2, ci);
            if (rc) return rc;
        }
        if (batch_end) {
            const int c0 = (p + 1) * kNB - kBW;   // first column of the batch
            const int e = static_cast<int>(e_b);
            const int m = d - e, n = std::min(kBW, d - e);
            float* P = A + static_cast<int64_t>(e) * d + c0;
            int ca = 0, ci = 0;
            split(free_sm, 0.5 * n * n + double(m - n) * n, double(n) * (c0 + kBW), &ca, &ci);
            if (b >= 1) {   // far(b - 1) wrote these columns / row blocks
                GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s, side->far[(b - 1) % SideStream::kRing], 0));
                GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s2, side->far2[(b - 1) % SideStream::kRing], 0));
            }
            rc = launch_sgemm(true, m, n, kBW, -1.f, P, d, 0, P, d, 0, 1.f,
                              A + static_cast<int64_t>(e) * d + e, d, 0, 1, kGemmLowerC, side->s, ca);
            if (rc) return rc;
            rc = launch_sgemm(false, n, c0 + kBW, kBW, -1.f, P, d, 0, Minv + static_cast<int64_t>(c0) * d, d,
                              0, 1.f, Minv + static_cast<int64_t>(e) * d, d, 0, 1, 0, side->s2, ci);
            if (rc) return rc;
            if (has_far) {
                // head: the 256 columns band(b + 1) writes next, then the tail
                const int f = e + kBW, mf = d - f, hb = std::min(kBW, mf);
                GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s3, side->done_panel, 0));
                GPTQ_CUDA_CHECK(cudaStreamWaitEvent(side->s4, side->done_panel, 0));
                for (int part = 0; part < 2; ++part) {
                    const int g0 = part == 0 ? f : f + hb;   // first row/column of the part
                    const int mg = d - g0, ng = part == 0 ? hb : mg;
                    if (mg <= 0) break;
                    float* Pf = A + static_cast<int64_t>(g0) * d + c0;
                    rc = launch_sgemm(true, mg, ng, kBW, -1.f, Pf, d, 0, Pf, d, 0, 1.f,
                                      A + static_cast<int64_t>(g0) * d + g0, d, 0, 1, kGemmLowerC,
                                      side->s3, -1);
                    if (rc) return rc;
                    rc = launch_sgemm(false, ng, c0 + kBW, kBW, -1.f, Pf, d, 0,
                                      Minv + static_cast<int64_t>(c0) * d, d, 0, 1.f,
                                      Minv + static_cast<int64_t>(g0) * d, d, 0, 1, 0, side->s4, -1);
                    if (rc) return rc;
                    if (part == 0) {
                        GPTQ_CUDA_CHECK(cudaEventRecord(side->far[b % SideStream::kRing], side->s3));
                        GPTQ_CUDA_CHECK(cudaEventRecord(side->far2[b % SideStream::kRing], side->s4));
                    }
                }
            }
        }
        GPTQ_CUDA_CHECK(cudaEventRecord(side->ev[p % SideStream::kRing], side->s));
        GPTQ_CUDA_CHECK(cudaEventRecord(side->ev2[p % SideStream::kRing], side->s2));
    }
    GPTQ_CUDA_CHECK(cudaEventRecord(side->join_p, side->sp));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->join_p, 0));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->join, side->s));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->join, 0));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->join2, side->s2));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->join2, 0));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->join3, side->s3));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->join3, 0));
    GPTQ_CUDA_CHECK(cudaEventRecord(side->join4, side->s4));
    GPTQ_CUDA_CHECK(cudaStreamWaitEvent(stream, side->join4, 0));

    reverse_upper_kernel<<<nsm * 8, 256, 0, stream>>>(Minv, d, U);
    GPTQ_LAUNCH_CHECK();

    GPTQ_CUDA_CHECK(cudaMemcpyAsync(status_host, &hdr->status, sizeof(int), cudaMemcpyDeviceToHost,
                                    stream));
    return GPTQ_OK;
}

// One factorisation in flight per device: the calls of a device share its
// side streams and events (and, when graphs are off or the caller's stream is
// being captured, enqueue on them directly), so a second call -- another host
// thread, another stream -- waits here until the first has synchronised.
static std::mutex& prepare_mutex()
{
    static std::mutex mu[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    return mu[dev];
}

// host_status != nullptr: synchronises the stream and stores the status there.
// Otherwise the status word is copied to async_status in stream order and the
// call returns without waiting.
int run_prepare(const float* H, int64_t d, float damp, int act_order, int32_t* perm, float* U,
                void* workspace, cudaStream_t stream, int* host_status, bool graphed,
                int* async_status)
{
    std::lock_guard<std::mutex> one_in_flight(prepare_mutex());
    uint32_t damp_bits = 0;
    static_assert(sizeof damp_bits == sizeof damp, "float is 32-bit");
    memcpy(&damp_bits, &damp, sizeof damp);
    const std::vector<uint64_t> key = {1,
                                       reinterpret_cast<uintptr_t>(H),
                                       static_cast<uint64_t>(d),
                                       damp_bits,
                                       static_cast<uint64_t>(act_order),
                                       reinterpret_cast<uintptr_t>(perm),
                                       reinterpret_cast<uintptr_t>(U),
                                       reinterpret_cast<uintptr_t>(workspace)};
    auto enq = [&](cudaStream_t s, int* st) {
        return enqueue_prepare(H, d, damp, act_order, perm, U, workspace, s, st);
    };
    int* st = nullptr;
    int rc = graphed ? run_graphed(key, true, enq, stream, &st) : GPTQ_OK;
    if (!graphed) {
        static thread_local int* direct = nullptr;
        if (!direct) GPTQ_CUDA_CHECK(cudaMallocHost(&direct, sizeof(int)));
        st = direct;
        rc = enq(stream, st);
    }
    if (rc) return rc;
    if (!host_status) {
        const PrepHeader* hdr = reinterpret_cast<const PrepHeader*>(workspace);
        GPTQ_CUDA_CHECK(cudaMemcpyAsync(async_status, &hdr->status, sizeof(int), cudaMemcpyDefault, stream));
        // launched directly (no graph) on the shared side streams: they must be
        // idle before the next call of the device may use them
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        GPTQ_CUDA_CHECK(cudaStreamIsCapturing(stream, &cs));
        int dev = 0;
        GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
        const bool direct = !graphed || !graphs_enabled() || dev < 0 || dev >= 64;
        if (direct && cs == cudaStreamCaptureStatusNone) GPTQ_CUDA_CHECK(cudaStreamSynchronize(stream));
        return GPTQ_OK;
    }
    GPTQ_CUDA_CHECK(cudaStreamSynchronize(stream));
    *host_status = *st;
    return GPTQ_OK;
}

}  // namespace gptq
