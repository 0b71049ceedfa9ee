// noalloc.cu -- gptq_quantize for callers that must not allocate device memory.
//
// Some callers cannot hand this library a workspace: a plugin inside another
// engine that only receives input and output pointers and has no allocator to
// ask; a serving loop that must not pay cudaMalloc's implicit device-wide
// synchronisation in the middle of its work; or a process that has reserved
// all of the GPU's memory up front for its own pool.  For them this entry
// point takes its scratch from a fixed array in the library's own device
// memory, which exists from the moment the library's device code is loaded
// until the process exits.
#include "common.cuh"

#include <mutex>

namespace gptq {
size_t quantize_workspace_min_bytes(int64_t d_out, int64_t d_in);
}

namespace {

// The scratch array.  Its size is GPTQ_STATIC_SCRATCH_BYTES (gptq.h).
static __device__ __align__(256) unsigned char g_quantize_scratch[GPTQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name only stands for the variable; its device address has to be
// looked up once per device, with that device current.  CUDA loads a module's
// device code lazily, so on each device this lookup is also the moment the
// array itself is created: it can fail for lack of device memory, which is
// reported as GPTQ_ERR_NO_MEMORY (and the runtime's error is cleared, so it
// does not surface in the caller's next CUDA call).
int scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return gptq::cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_quantize_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            const int rc = gptq::cuda_fail_msg("creating the static scratch", e);
            return e == cudaErrorMemoryAllocation ? GPTQ_ERR_NO_MEMORY : rc;
        }
        if (!p) return GPTQ_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return GPTQ_OK;
}

}  // namespace

namespace gptq {
int quantize_entry(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                   int64_t d_in, int bits, int group_size, int block_size, uint8_t* codes,
                   float* scales, float* zeros, uint8_t* packed_int4, int32_t* g_idx,
                   float* err_sq, void* workspace, size_t ws_bytes, void* stream, bool graphed,
                   float* ms_by_class);
}

extern "C" int gptq_quantize_static_scratch(float* W, const float* Hinv_chol,
                                            const int32_t* perm, int64_t d_out, int64_t d_in,
                                            int bits, int group_size, int block_size,
                                            uint8_t* codes, float* scales, float* zeros,
                                            uint8_t* packed_int4, int32_t* g_idx,
                                            float* err_sq, void* stream)
{
    if (d_out <= 0 || d_in <= 0) return GPTQ_ERR_INVALID_ARG;
    // A layer whose working set does not fit the fixed array is refused
    // before anything touches the device.
    if (gptq::quantize_workspace_min_bytes(d_out, d_in) > GPTQ_STATIC_SCRATCH_BYTES)
        return GPTQ_ERR_WORKSPACE;
    // the device check comes before the lookup: on a GPU this library has no
    // code for, the lookup itself would fail with a less telling error
    int rc = gptq::check_device();
    if (rc != GPTQ_OK) return rc;
    void* scratch = nullptr;
    rc = scratch_address(&scratch);
    if (rc != GPTQ_OK) return rc;
    // Nothing in the scratch has to start at zero: every byte gptq_quantize
    // reads from its workspace is written earlier in the same call.  The
    // launches are enqueued directly (no graph is instantiated for this path).
    return gptq::quantize_entry(W, Hinv_chol, perm, d_out, d_in, bits, group_size, block_size,
                                codes, scales, zeros, packed_int4, g_idx, err_sq, scratch,
                                GPTQ_STATIC_SCRATCH_BYTES, stream, false, nullptr);
}
