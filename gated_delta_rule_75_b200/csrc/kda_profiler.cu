// Per-kernel launch counting and CUDA-event timing of the library's own
// launches.  Every launch site opens a LaunchScope; while the profiler is
// enabled the scope records a start and a stop event on the launching stream,
// so durations are measured on the stream the kernel runs on.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "kda.h"
#include "kda_internal.h"

namespace kda {

static const char* const kKernelNames[K_KERNEL_COUNT] = {
    "chunk_offsets", "chunk_prep_simt", "chunk_state_simt", "decode_step",
    "chunk_prep_tc", "chunk_state_tc", "chunk_state_seg_tc", "affine_prefix", "fill",
    "bwd_state", "bwd_dense1", "bwd_dense2", "bwd_param", "chunk_fused_tc",
};

namespace {
struct Rec {
    int id;
    cudaEvent_t start, stop;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free;
std::atomic<int64_t> g_launches[K_KERNEL_COUNT];

cudaEvent_t take_event()
{
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

LaunchScope::LaunchScope(cudaStream_t st, KernelId id) : st_(st), id_(id)
{
    g_launches[id].fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_on) return;
    start_ = take_event();
    stop_ = take_event();
    if (start_ && stop_ && cudaEventRecord((cudaEvent_t)start_, st) == cudaSuccess) return;
    if (start_) g_free.push_back((cudaEvent_t)start_);
    if (stop_) g_free.push_back((cudaEvent_t)stop_);
    start_ = stop_ = nullptr;
}

LaunchScope::~LaunchScope()
{
    if (!start_) return;
    std::lock_guard<std::mutex> lock(g_mu);
    if (cudaEventRecord((cudaEvent_t)stop_, st_) == cudaSuccess) {
        g_recs.push_back({(int)id_, (cudaEvent_t)start_, (cudaEvent_t)stop_});
    } else {
        g_free.push_back((cudaEvent_t)start_);
        g_free.push_back((cudaEvent_t)stop_);
    }
}

}  // namespace kda

using namespace kda;

extern "C" {

void kda_profiler_enable(int on)
{
    std::lock_guard<std::mutex> lock(g_mu);
    g_on = on != 0;
}

int kda_profiler_read(kda_kernel_stat_t* out, int max_entries, int reset)
{
    double ms[K_KERNEL_COUNT] = {};
    int64_t timed[K_KERNEL_COUNT] = {};
    std::vector<Rec> recs;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        recs.swap(g_recs);
    }
    int rc = 0;
    for (const Rec& r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess ||
            cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
            rc = -1;
        } else {
            ms[r.id] += t;
            timed[r.id] += 1;
        }
    }
    {
        std::lock_guard<std::mutex> lock(g_mu);
        for (const Rec& r : recs) {
            g_free.push_back(r.start);
            g_free.push_back(r.stop);
        }
    }
    int n = 0;
    for (int i = 0; i < K_KERNEL_COUNT && n < max_entries; ++i) {
        const int64_t launches = reset ? g_launches[i].exchange(0) : g_launches[i].load();
        if (out) {
            out[n].name = kKernelNames[i];
            out[n].launches = launches;
            out[n].timed_launches = timed[i];
            out[n].total_ms = ms[i];
        }
        ++n;
    }
    return rc < 0 ? rc : n;
}

}  // extern "C"
