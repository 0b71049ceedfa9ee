// graph.cu -- replay of the factorisation and of the column loop as CUDA
// graphs.  A call's launch sequence depends only on its arguments (sizes,
// options, pointers), so it is captured once into a graph, instantiated, and
// replayed on the caller's stream for every later call with the same
// arguments: one launch from the host instead of a few hundred, and the
// device resolves the dependencies between the streams of the factorisation
// without waiting on the host.
#include "common.cuh"

#include <cstdlib>
#include <list>
#include <mutex>
#include <vector>

namespace gptq {

namespace {

struct Entry {
    int dev;
    std::vector<uint64_t> key;
    cudaGraphExec_t exec;
    int* status_host;      // pinned word the graph copies the status into (or null)
    uint64_t launches;     // kernel launches the graph holds
};

constexpr size_t kMaxEntries = 16;
std::mutex g_mu;
std::list<Entry> g_cache;   // most recently used first
cudaStream_t g_capture[64] = {};

void drop(Entry& e)
{
    cudaGraphExecDestroy(e.exec);
    if (e.status_host) cudaFreeHost(e.status_host);
}

}  // namespace

bool graphs_enabled()
{
    static const bool on = [] {
        const char* v = std::getenv("GPTQ_GRAPHS");
        return !(v && v[0] == '0');
    }();
    return on;
}

// Runs enqueue(stream, status_host) either directly on `stream` or through a
// cached graph.  status_host (when want_status) receives the device status
// word of the run once the caller synchronises `stream`.
int run_graphed(const std::vector<uint64_t>& key, bool want_status,
                const std::function<int(cudaStream_t, int*)>& enqueue, cudaStream_t stream,
                int** status_out)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    GPTQ_CUDA_CHECK(cudaStreamIsCapturing(stream, &cs));
    int dev = 0;
    GPTQ_CUDA_CHECK(cudaGetDevice(&dev));
    if (!graphs_enabled() || cs != cudaStreamCaptureStatusNone || dev < 0 || dev >= 64) {
        static thread_local int* direct_status = nullptr;
        if (want_status && !direct_status) GPTQ_CUDA_CHECK(cudaMallocHost(&direct_status, sizeof(int)));
        if (status_out) *status_out = direct_status;
        return enqueue(stream, want_status ? direct_status : nullptr);
    }
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto it = g_cache.begin(); it != g_cache.end(); ++it) {
        if (it->dev == dev && it->key == key) {
            g_cache.splice(g_cache.begin(), g_cache, it);
            Entry& e = g_cache.front();
            GPTQ_CUDA_CHECK(cudaGraphLaunch(e.exec, stream));
            note_launches(e.launches);
            if (status_out) *status_out = e.status_host;
            return GPTQ_OK;
        }
    }
    if (!g_capture[dev]) GPTQ_CUDA_CHECK(cudaStreamCreateWithFlags(&g_capture[dev], cudaStreamNonBlocking));
    cudaStream_t cap = g_capture[dev];
    Entry e{dev, key, nullptr, nullptr, 0};
    if (want_status) GPTQ_CUDA_CHECK(cudaMallocHost(&e.status_host, sizeof(int)));
    const uint64_t before = launch_count();
    cudaError_t ce = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
    if (ce != cudaSuccess) {
        if (e.status_host) cudaFreeHost(e.status_host);
        return cuda_fail(ce);
    }
    const int rc = enqueue(cap, e.status_host);
    cudaGraph_t graph = nullptr;
    ce = cudaStreamEndCapture(cap, &graph);
    e.launches = launch_count() - before;
    if (rc || ce != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        if (e.status_host) cudaFreeHost(e.status_host);
        return rc ? rc : cuda_fail(ce);
    }
    ce = cudaGraphInstantiate(&e.exec, graph, cudaGraphInstantiateFlagUseNodePriority);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) {
        if (e.status_host) cudaFreeHost(e.status_host);
        return cuda_fail(ce);
    }
    // the captured launches were counted while recording; the replay counts them
    unnote_launches(e.launches);
    g_cache.push_front(e);
    if (g_cache.size() > kMaxEntries) {
        drop(g_cache.back());
        g_cache.pop_back();
    }
    Entry& f = g_cache.front();
    GPTQ_CUDA_CHECK(cudaGraphLaunch(f.exec, stream));
    note_launches(f.launches);
    if (status_out) *status_out = f.status_host;
    return GPTQ_OK;
}

}  // namespace gptq
