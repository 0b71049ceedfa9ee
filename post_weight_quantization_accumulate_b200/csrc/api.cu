// api.cu -- extern "C" entry points of libgptq.so: argument validation on the
// host, then the stream-ordered launches of hessian.cu, prepare.cu and
// quantize.cu.  No call allocates device memory.
#include "common.cuh"

#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

namespace gptq {

int launch_hessian_upper(float* H, const uint16_t* X, int64_t n_rows, int64_t d, cudaStream_t s);
int launch_mirror(float* H, int64_t d, cudaStream_t s);
size_t prepare_workspace_bytes(int64_t d);
size_t quantize_workspace_bytes(int64_t d_out, int64_t d_in);
size_t quantize_workspace_min_bytes(int64_t d_out, int64_t d_in);
int run_prepare(const float* H, int64_t d, float damp, int act_order, int32_t* perm, float* U,
                void* ws, cudaStream_t s, int* host_status, bool graphed, int* async_status = nullptr);
int run_quantize(float* W, const float* U, const int32_t* perm, int64_t d_out, int64_t d_in,
                 int bits, int gs, int block, uint8_t* codes, float* scales, float* zeros,
                 uint8_t* packed, int32_t* g_idx, float* err_sq, void* ws, size_t ws_bytes,
                 cudaStream_t s, bool graphed, const Q4KOut* q4k = nullptr);
int run_bf16_to_f32(float* dst, const uint16_t* src, int64_t n, cudaStream_t s);
int run_quotient_selftest(int64_t n, uint64_t seed, int64_t* mismatches);
size_t hessian_f32_workspace_bytes(int64_t d, int64_t chunk);
int run_hessian_f32(float* H, const float* X, int64_t n, int64_t d, int64_t chunk, void* ws,
                    cudaStream_t s);
bool w4a16_tc_supported(const uint16_t* X, const uint8_t* packed, const int32_t* g_idx,
                        int64_t K, int gs);
bool gemv_supported(const int32_t* g_idx, int64_t M, int64_t K, int gs);
int run_w4a16(float* Y, const uint16_t* X, const uint8_t* packed, const float* scales,
              const float* zeros, const int32_t* g_idx, int64_t M, int64_t N, int64_t K, int gs,
              int path, cudaStream_t stream);
int run_quantize_timed(float* W, const float* U, const int32_t* perm, int64_t d_out, int64_t d_in,
                       int bits, int gs, int block, uint8_t* codes, float* scales, float* zeros,
                       uint8_t* packed, int32_t* g_idx, float* err_sq, void* workspace,
                       size_t ws_bytes, cudaStream_t stream, float* ms_by_class);

namespace {
std::atomic<uint64_t> g_launches{0};
thread_local char g_last_error[256] = "";
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::mutex g_dev_mutex;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Valid for 64-bit problem sizes that fit the kernels' 32-bit indexing.
constexpr int64_t kMaxDim = 65536;

struct StreamPair {
    cudaStream_t copy = nullptr;
    cudaEvent_t ev_ready[2] = {nullptr, nullptr};
    cudaEvent_t ev_done[2] = {nullptr, nullptr};
    cudaEvent_t ev_start = nullptr;
    const void* last_staging = nullptr;   // staging buffer of the previous call
    size_t last_bytes = 0;
};
StreamPair g_streams[kMaxDevices];
}  // namespace

namespace {
thread_local uint64_t t_launches = 0;   // this thread's launches (graph capture accounting)
}

void note_launch()
{
    g_launches.fetch_add(1, std::memory_order_relaxed);
    ++t_launches;
}
void note_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
void unnote_launches(uint64_t n) { g_launches.fetch_sub(n, std::memory_order_relaxed); }
uint64_t launch_count() { return t_launches; }

int cuda_fail(cudaError_t e)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return GPTQ_ERR_CUDA;
}

int cuda_fail_msg(const char* where, cudaError_t e)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s: %s", where, cudaGetErrorName(e),
             cudaGetErrorString(e));
    return GPTQ_ERR_CUDA;
}

int* device_status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    return g_status_ptr[dev];
}

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lk(g_dev_mutex);
    if (!g_sm_count[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

int check_device()
{
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    int major = 0;
    GPTQ_CUDA_CHECK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    if (major != 10) return GPTQ_ERR_UNSUPPORTED;
    if (dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
    return GPTQ_OK;
}

static int hessian_device(float* H, const uint16_t* X, int64_t n, int64_t d, cudaStream_t s)
{
    // TMA row coordinates are 32-bit: feed at most 2^30 rows per launch.
    const int64_t kRows = int64_t(1) << 30;
    for (int64_t t = 0; t < n; t += kRows) {
        const int64_t rows = (n - t < kRows) ? n - t : kRows;
        int rc = launch_hessian_upper(H, X + t * d, rows, d, s);
        if (rc) return rc;
    }
    return GPTQ_OK;
}

// One thread waits, through the same bounded-wait helper the tensor-core
// kernels use, on an mbarrier that nothing completes, with a limit of
// `limit_cycles`; the wait gives up, records GPTQ_ERR_TIMEOUT and returns.
__global__ void bounded_wait_selftest_kernel(long long limit_cycles, int* status)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, status, limit_cycles);
    __syncthreads();
}

// Argument checks and the column loop; `graphed` replays a cached CUDA graph
// of the launch sequence (the allocation-free entry point enqueues directly).
int quantize_entry(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                   int64_t d_in, int bits, int group_size, int block_size, uint8_t* codes,
                   float* scales, float* zeros, uint8_t* packed_int4, int32_t* g_idx,
                   float* err_sq, void* workspace, size_t ws_bytes, void* stream, bool graphed,
                   float* ms_by_class = nullptr)
{
    if (!W || !Hinv_chol || !scales || !zeros || d_out <= 0 || d_in <= 0 || d_in > kMaxDim ||
        d_out > (int64_t(1) << 31) / 2 || d_in % 8 != 0 || bits < 1 || bits > 8 ||
        block_size < 8 || block_size > 128 || block_size % 8 != 0 || !aligned(W, 16))
        return GPTQ_ERR_INVALID_ARG;
    if (group_size != -1) {
        if (group_size <= 0 || d_in % group_size != 0) return GPTQ_ERR_INVALID_ARG;
        if (group_size % block_size != 0 && block_size % group_size != 0)
            return GPTQ_ERR_INVALID_ARG;
    }
    if (packed_int4 && bits > 4) return GPTQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(d_out) * d_in >= (int64_t(1) << 40)) return GPTQ_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < quantize_workspace_min_bytes(d_out, d_in))
        return GPTQ_ERR_WORKSPACE;
    int rc = check_device();
    if (rc) return rc;
    if (ms_by_class)
        return run_quantize_timed(W, Hinv_chol, perm, d_out, d_in, bits, group_size, block_size,
                                  codes, scales, zeros, packed_int4, g_idx, err_sq, workspace,
                                  ws_bytes, static_cast<cudaStream_t>(stream), ms_by_class);
    return run_quantize(W, Hinv_chol, perm, d_out, d_in, bits, group_size, block_size, codes,
                        scales, zeros, packed_int4, g_idx, err_sq, workspace, ws_bytes,
                        static_cast<cudaStream_t>(stream), graphed);
}

}  // namespace gptq

using namespace gptq;

extern "C" {

const char* gptq_status_string(int status)
{
    switch (status) {
        case GPTQ_OK: return "ok";
        case GPTQ_ERR_INVALID_ARG: return "invalid argument";
        case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
        case GPTQ_ERR_NONFINITE: return "non-finite value in the Hessian";
        case GPTQ_ERR_CUDA: return "CUDA error";
        case GPTQ_ERR_TIMEOUT: return "device-side wait timed out";
        case GPTQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case GPTQ_ERR_UNSUPPORTED: return "device is not sm_100 (B200)";
        case GPTQ_ERR_NO_MEMORY: return "device memory for the library's static scratch could not be created";
        default: return "unknown status";
    }
}

const char* gptq_last_cuda_error(void) { return g_last_error; }

int gptq_version(void) { return 100; }

uint64_t gptq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int gptq_device_status(void)
{
    int* p = device_status_ptr();
    if (!p) return GPTQ_ERR_CUDA;
    GPTQ_CUDA_CHECK(cudaDeviceSynchronize());
    int v = 0;
    GPTQ_CUDA_CHECK(cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost));
    const int zero = 0;
    GPTQ_CUDA_CHECK(cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice));
    return v;
}

size_t gptq_workspace_bytes(int64_t d_out, int64_t d_in, int block_size)
{
    if (d_in <= 0 || d_in > kMaxDim || d_out < 0 || d_out > (int64_t(1) << 31) / 2 ||
        block_size < 0)
        return 0;
    size_t a = prepare_workspace_bytes(d_in);
    size_t b = quantize_workspace_bytes(d_out, d_in);
    return a > b ? a : b;
}

size_t gptq_workspace_min_bytes(int64_t d_out, int64_t d_in, int block_size)
{
    if (d_in <= 0 || d_in > kMaxDim || d_out < 0 || d_out > (int64_t(1) << 31) / 2 ||
        block_size < 0)
        return 0;
    size_t a = prepare_workspace_bytes(d_in);
    size_t b = quantize_workspace_min_bytes(d_out, d_in);
    return a > b ? a : b;
}

int gptq_hessian_accumulate(float* H, const uint16_t* X, int64_t n_tokens, int64_t d_in,
                            void* stream)
{
    if (!H || (!X && n_tokens > 0) || n_tokens < 0 || d_in <= 0 || d_in > kMaxDim ||
        d_in % 8 != 0 || !aligned(H, 16) || !aligned(X, 16))
        return GPTQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return GPTQ_OK;
    int rc = check_device();
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = hessian_device(H, X, n_tokens, d_in, s);
    if (rc) return rc;
    return launch_mirror(H, d_in, s);
}

size_t gptq_hessian_f32_workspace_bytes(int64_t d_in, int64_t chunk_tokens)
{
    if (d_in <= 0 || d_in > kMaxDim / 2 || d_in % 8 != 0 || chunk_tokens <= 0 ||
        chunk_tokens > (int64_t(1) << 30))
        return 0;
    return hessian_f32_workspace_bytes(d_in, chunk_tokens);
}

int gptq_hessian_accumulate_f32(float* H, const float* X, int64_t n_tokens, int64_t d_in,
                                int64_t chunk_tokens, void* workspace, size_t ws_bytes,
                                void* stream)
{
    if (!H || (!X && n_tokens > 0) || n_tokens < 0 || d_in <= 0 || d_in > kMaxDim / 2 ||
        d_in % 8 != 0 || chunk_tokens <= 0 || chunk_tokens > (int64_t(1) << 30) ||
        !aligned(H, 16) || !aligned(X, 16))
        return GPTQ_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) ||
        ws_bytes < hessian_f32_workspace_bytes(d_in, chunk_tokens))
        return GPTQ_ERR_WORKSPACE;
    if (n_tokens == 0) return GPTQ_OK;
    int rc = check_device();
    if (rc) return rc;
    return run_hessian_f32(H, X, n_tokens, d_in, chunk_tokens, workspace,
                           static_cast<cudaStream_t>(stream));
}

int gptq_hessian_accumulate_host(float* H, const uint16_t* X_host, int64_t n_tokens,
                                 int64_t d_in, uint16_t* staging, int64_t chunk_tokens,
                                 void* stream)
{
    if (!H || (!X_host && n_tokens > 0) || !staging || n_tokens < 0 || chunk_tokens <= 0 ||
        chunk_tokens > (int64_t(1) << 30) || d_in <= 0 || d_in > kMaxDim || d_in % 8 != 0 ||
        !aligned(H, 16) || !aligned(staging, 16))
        return GPTQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return GPTQ_OK;
    int rc = check_device();
    if (rc) return rc;
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    StreamPair& sp = g_streams[dev];
    {
        std::lock_guard<std::mutex> lk(g_dev_mutex);
        if (!sp.copy) {
            GPTQ_CUDA_CHECK(cudaStreamCreateWithFlags(&sp.copy, cudaStreamNonBlocking));
            for (int i = 0; i < 2; ++i) {
                GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&sp.ev_ready[i], cudaEventDisableTiming));
                GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&sp.ev_done[i], cudaEventDisableTiming));
            }
            GPTQ_CUDA_CHECK(cudaEventCreateWithFlags(&sp.ev_start, cudaEventDisableTiming));
        }
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    GPTQ_CUDA_CHECK(cudaStreamIsCapturing(s, &cs));
    const size_t staging_bytes = 2 * static_cast<size_t>(chunk_tokens) * static_cast<size_t>(d_in) * 2;
    const bool same_staging = sp.last_staging == staging && sp.last_bytes == staging_bytes;
    if (cs != cudaStreamCaptureStatusNone || !same_staging) {
        // captured (the copy stream joins the capture through `stream`), or a
        // staging buffer this function has not used last (it may hold memory
        // that earlier work on `stream` still reads): wait for that work
        GPTQ_CUDA_CHECK(cudaEventRecord(sp.ev_start, s));
        GPTQ_CUDA_CHECK(cudaStreamWaitEvent(sp.copy, sp.ev_start, 0));
    } else {
        // the same buffers as the previous call: their last readers are that
        // call's accumulations
        for (int i = 0; i < 2; ++i) GPTQ_CUDA_CHECK(cudaStreamWaitEvent(sp.copy, sp.ev_done[i], 0));
    }
    sp.last_staging = staging;
    sp.last_bytes = staging_bytes;
    const size_t chunk_elems = static_cast<size_t>(chunk_tokens) * static_cast<size_t>(d_in);
    int64_t c = 0;
    for (int64_t t = 0; t < n_tokens; t += chunk_tokens, ++c) {
        const int b = static_cast<int>(c & 1);
        const int64_t rows = (n_tokens - t < chunk_tokens) ? n_tokens - t : chunk_tokens;
        uint16_t* buf = staging + b * chunk_elems;
        if (c >= 2) GPTQ_CUDA_CHECK(cudaStreamWaitEvent(sp.copy, sp.ev_done[b], 0));
        GPTQ_CUDA_CHECK(cudaMemcpyAsync(buf, X_host + static_cast<size_t>(t) * d_in,
                                        static_cast<size_t>(rows) * d_in * sizeof(uint16_t),
                                        cudaMemcpyHostToDevice, sp.copy));
        GPTQ_CUDA_CHECK(cudaEventRecord(sp.ev_ready[b], sp.copy));
        GPTQ_CUDA_CHECK(cudaStreamWaitEvent(s, sp.ev_ready[b], 0));
        rc = launch_hessian_upper(H, buf, rows, d_in, s);
        if (rc) return rc;
        GPTQ_CUDA_CHECK(cudaEventRecord(sp.ev_done[b], s));
    }
    return launch_mirror(H, d_in, s);
}

int gptq_prepare(const float* H, int64_t d_in, float damp, int act_order, int32_t* perm,
                 float* Hinv_chol, void* workspace, size_t ws_bytes, void* stream)
{
    if (!H || !perm || !Hinv_chol || d_in <= 0 || d_in > kMaxDim || !(damp >= 0.f) ||
        !(damp < 1e30f))
        return GPTQ_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < prepare_workspace_bytes(d_in))
        return GPTQ_ERR_WORKSPACE;
    int rc = check_device();
    if (rc) return rc;
    int st = 0;
    rc = run_prepare(H, d_in, damp, act_order ? 1 : 0, perm, Hinv_chol, workspace,
                     static_cast<cudaStream_t>(stream), &st, true);
    if (rc) return rc;
    return st;
}

int gptq_prepare_async(const float* H, int64_t d_in, float damp, int act_order, int32_t* perm,
                       float* Hinv_chol, void* workspace, size_t ws_bytes, int* status, void* stream)
{
    if (!H || !perm || !Hinv_chol || !status || d_in <= 0 || d_in > kMaxDim || !(damp >= 0.f) ||
        !(damp < 1e30f) || !aligned(status, 4))
        return GPTQ_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < prepare_workspace_bytes(d_in))
        return GPTQ_ERR_WORKSPACE;
    int rc = check_device();
    if (rc) return rc;
    return run_prepare(H, d_in, damp, act_order ? 1 : 0, perm, Hinv_chol, workspace,
                       static_cast<cudaStream_t>(stream), nullptr, true, status);
}

int gptq_quantize(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                  int64_t d_in, int bits, int group_size, int block_size, uint8_t* codes,
                  float* scales, float* zeros, uint8_t* packed_int4, int32_t* g_idx,
                  float* err_sq, void* workspace, size_t ws_bytes, void* stream)
{
    return quantize_entry(W, Hinv_chol, perm, d_out, d_in, bits, group_size, block_size, codes,
                          scales, zeros, packed_int4, g_idx, err_sq, workspace, ws_bytes, stream,
                          true);
}

int gptq_quantize_timed(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                        int64_t d_in, int bits, int group_size, int block_size, uint8_t* codes,
                        float* scales, float* zeros, uint8_t* packed_int4, int32_t* g_idx,
                        float* err_sq, void* workspace, size_t ws_bytes, void* stream,
                        float* loop_ms, float* update_ms, float* other_ms)
{
    if (!loop_ms || !update_ms || !other_ms) return GPTQ_ERR_INVALID_ARG;
    float ms[3] = {0.f, 0.f, 0.f};
    const int rc = quantize_entry(W, Hinv_chol, perm, d_out, d_in, bits, group_size, block_size,
                                  codes, scales, zeros, packed_int4, g_idx, err_sq, workspace,
                                  ws_bytes, stream, false, ms);
    *other_ms = ms[0];
    *loop_ms = ms[1];
    *update_ms = ms[2];
    return rc;
}

int gptq_selftest_bounded_wait(int64_t limit_cycles)
{
    if (limit_cycles <= 0 || limit_cycles > kWaitLimitCycles) return GPTQ_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc) return rc;
    int* status = device_status_ptr();
    if (!status) return GPTQ_ERR_CUDA;
    bounded_wait_selftest_kernel<<<1, 32>>>(limit_cycles, status);
    GPTQ_LAUNCH_CHECK();
    return gptq_device_status();
}

int gptq_selftest_quotient(int64_t n_pairs, uint64_t seed, int64_t* mismatches)
{
    if (n_pairs <= 0 || !mismatches) return GPTQ_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc) return rc;
    return run_quotient_selftest(n_pairs, seed, mismatches);
}

int gptq_w4a16_gemm(float* Y, const uint16_t* X, const uint8_t* packed, const float* scales,
                    const float* zeros, const int32_t* g_idx, int64_t M, int64_t N, int64_t K,
                    int group_size, int path, void* stream)
{
    if (M < 0 || N < 0 || K <= 0 || K % 8 != 0 || K > (int64_t(1) << 30) ||
        M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || M * N > (int64_t(1) << 40) ||
        path < GPTQ_W4A16_AUTO || path > GPTQ_W4A16_DECODE)
        return GPTQ_ERR_INVALID_ARG;
    if (group_size != -1 && (group_size <= 0 || K % group_size != 0)) return GPTQ_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return GPTQ_OK;
    if (!Y || !X || !packed || !scales || !zeros || !aligned(X, 16) || !aligned(packed, 16) ||
        !aligned(Y, 4) || !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(g_idx, 4))
        return GPTQ_ERR_INVALID_ARG;
    if (path == GPTQ_W4A16_TENSOR_CORE && !w4a16_tc_supported(X, packed, g_idx, K, group_size))
        return GPTQ_ERR_INVALID_ARG;
    if (path == GPTQ_W4A16_DECODE && !gemv_supported(g_idx, M, K, group_size)) return GPTQ_ERR_INVALID_ARG;
    int rc = check_device();
    if (rc) return rc;
    return run_w4a16(Y, X, packed, scales, zeros, g_idx, M, N, K, group_size, path,
                     static_cast<cudaStream_t>(stream));
}

int gptq_quantize_q4k(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                      int64_t d_in, uint8_t* codes, uint8_t* sc6, uint8_t* m6, float* dsup,
                      float* dmin, float* scales, float* offsets, uint8_t* packed_int4,
                      int32_t* g_idx, float* err_sq, void* workspace, size_t ws_bytes, void* stream)
{
    if (!W || !Hinv_chol || !sc6 || !m6 || !dsup || !dmin || !scales || !offsets || d_out <= 0 ||
        d_in <= 0 || d_in > kMaxDim || d_in % 256 != 0 || d_out > (int64_t(1) << 31) / 2 ||
        !aligned(W, 16) || static_cast<int64_t>(d_out) * d_in >= (int64_t(1) << 40))
        return GPTQ_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < quantize_workspace_min_bytes(d_out, d_in))
        return GPTQ_ERR_WORKSPACE;
    int rc = check_device();
    if (rc) return rc;
    const Q4KOut q4k{sc6, m6, dsup, dmin};
    return run_quantize(W, Hinv_chol, perm, d_out, d_in, 4, 32, 128, codes, scales, offsets,
                        packed_int4, g_idx, err_sq, workspace, ws_bytes,
                        static_cast<cudaStream_t>(stream), true, &q4k);
}

int gptq_bf16_to_f32(float* dst, const uint16_t* src, int64_t n, void* stream)
{
    if (n < 0 || (n > 0 && (!dst || !src))) return GPTQ_ERR_INVALID_ARG;
    if (n == 0) return GPTQ_OK;
    int rc = check_device();
    if (rc) return rc;
    return run_bf16_to_f32(dst, src, n, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
