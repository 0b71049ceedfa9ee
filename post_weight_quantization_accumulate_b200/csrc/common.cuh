// common.cuh -- shared helpers of libgptq.so (sm_100a): status word, launch
// accounting, and thin inline-PTX wrappers for mbarrier, TMA and tcgen05.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gptq.h"

#include <algorithm>
#include <functional>
#include <vector>

namespace gptq {

// ---------------------------------------------------------------- host side
// Records a launch (for gptq_launch_count) and checks the launch error.
void note_launch();
void note_launches(uint64_t n);     // a graph replay of n launches
void unnote_launches(uint64_t n);   // launches recorded into a graph, not run
uint64_t launch_count();            // launches recorded by the calling thread

// Runs enqueue(stream, status_host) directly on `stream`, or replays a CUDA
// graph captured from it for the same `key` (every argument that shapes the
// launch sequence).  With want_status, *status_out is a pinned word that holds
// the run's status after `stream` is synchronised.
// false when GPTQ_GRAPHS=0 asks for direct launches instead of cached graphs
bool graphs_enabled();
int run_graphed(const std::vector<uint64_t>& key, bool want_status,
                const std::function<int(cudaStream_t, int*)>& enqueue, cudaStream_t stream,
                int** status_out);
int cuda_fail(cudaError_t e);          // stores the message, returns GPTQ_ERR_CUDA
int cuda_fail_msg(const char* where, cudaError_t e);   // same, naming the failing step
int* device_status_ptr();              // status word of the current device (device memory)
int sm_count();                        // SMs of the current device
int check_device();                    // GPTQ_ERR_UNSUPPORTED unless the current device is sm_100

// Launches kernel `k` on `stream`; with `pdl` as a programmatic dependent
// launch: the kernel may start while the previous kernel on the stream is
// still running, once every CTA of that kernel has executed pdl_trigger(), and
// must call pdl_wait() before it touches anything the previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     bool pdl, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

#define GPTQ_LAUNCH_CHECK()                                   \
    do {                                                      \
        ::gptq::note_launch();                                \
        cudaError_t _e = cudaGetLastError();                  \
        if (_e != cudaSuccess) return ::gptq::cuda_fail(_e);  \
    } while (0)

#define GPTQ_CUDA_CHECK(x)                                    \
    do {                                                      \
        cudaError_t _e = (x);                                 \
        if (_e != cudaSuccess) return ::gptq::cuda_fail(_e);  \
    } while (0)

// Outputs of the two-level Q4_K grid (gptq_quantize_q4k).
struct Q4KOut {
    uint8_t* sc6;    // [d_out][d_in / 32] 6-bit block scales
    uint8_t* m6;     // [d_out][d_in / 32] 6-bit block mins
    float* dsup;     // [d_out][d_in / 256] super-block scale of the scales
    float* dmin;     // [d_out][d_in / 256] super-block scale of the mins
};

// Upper bound on one device-side wait, in SM clock cycles (about 1 s).
constexpr long long kWaitLimitCycles = 2000000000LL;

// -------------------------------------------------------------- device side
__device__ __forceinline__ void record_status(int* status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of `bar` with the given parity.  Gives up when *abort
// becomes non-zero or after `limit` cycles; on a time-out it raises *abort
// and records GPTQ_ERR_TIMEOUT.  Returns false when it gave up.  The abort
// flag and the clock are read once per 32 polls of the barrier: waiting warps
// share the SM's issue slots and load/store queues with the working ones.
// With sleep_ns > 0 the waiting warp sleeps that long between polls and
// leaves its scheduler's issue slots to the warps that have work.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int* status,
                                                  long long limit = kWaitLimitCycles,
                                                  unsigned sleep_ns = 0)
{
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            if (mbar_try_wait(bar, parity)) return true;
            if (sleep_ns) __nanosleep(sleep_ns);
        }
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            record_status(status, GPTQ_ERR_TIMEOUT);
            return false;
        }
    }
}

// mbar_wait_bounded for a whole warp (all 32 lanes call it): lane 0 polls and
// the others wait at the warp barrier, which also orders what lane 0 observed
// before their own accesses.  Polls from every lane of many waiting warps
// fill the SM's shared-memory pipe that the working warps' loads, special-
// function and tcgen05 instructions go through as well.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               int* status, long long limit = kWaitLimitCycles,
                                               unsigned sleep_ns = 0)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait_bounded(bar, parity, abort, status, limit, sleep_ns) ? 1 : 0;
    __syncwarp();
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// 2-D tiled TMA load into shared memory, completing on `bar` (tx bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Programmatic dependent launch, device side.  pdl_wait: returns once the
// previous kernel on the stream has completed and its writes are visible (at
// once for a kernel launched without the attribute).  pdl_trigger: this CTA
// lets the next kernel start; the next kernel's CTAs may occupy free SMs and
// run their prologue while this grid still runs.
// Device-wide nanosecond clock (the same on every SM), for the spans the
// timing entry points record.
__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 (5th-generation tensor core, accumulators in tensor memory)
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warpgroup register re-allocation (all 4 warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void regs_dealloc()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_alloc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16/f16 in, f32 acc).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A * B, kind::tf32 (tf32 in, f32 acc).
__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives the
// 32 columns of TMEM lane (lane base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma, SWIZZLE_128B canonical
// layout.  For an MN-major operand: lbo = bytes between consecutive 64-element
// (128-byte) MN chunks, sbo = bytes between consecutive 8-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
    return d;
}

// Shared-memory descriptor for an MN-major 32-bit (tf32) operand, the
// SWIZZLE_128B_BASE32B layout (32-byte chunks swizzled within 128-byte rows,
// period 4 rows) that TMA writes with CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B:
// lbo = bytes between consecutive 32-element MN chunks, sbo = bytes between
// consecutive 4-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128_base32b(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
    d |= static_cast<uint64_t>(1) << 61;  // SWIZZLE_128B_BASE32B
    return d;
}

// Instruction descriptor for kind::f16 / kind::tf32 with f32 accumulation.
// fmt: 0 = f16, 1 = bf16, 2 = tf32 (both operands); a_mn/b_mn: operand is
// MN-major (1) or K-major (0).
__host__ __device__ constexpr uint32_t idesc_f32acc(uint32_t fmt, uint32_t a_mn, uint32_t b_mn,
                                                    uint32_t M, uint32_t N)
{
    return (1u << 4)                 // D format f32
           | (fmt << 7) | (fmt << 10)  // A, B formats
           | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

}  // namespace gptq
