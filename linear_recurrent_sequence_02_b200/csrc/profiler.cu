// Per-kernel device timing: CUDA events recorded around each launch when
// enabled (off by default).  Used by the benchmark to time the dominant
// kernel live, on the stream it runs on, inside the timed region.
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"

namespace retnet {

namespace {
struct Pending {
    std::string name;
    cudaEvent_t start, stop;
    bool captured;       // recorded by a graph node: never handed out again
};
struct Totals {
    double ms = 0.0;
    unsigned long long launches = 0;
};
std::mutex g_mu;
bool g_enabled = false;
std::string g_only;          // time only this kernel when not empty
std::vector<cudaEvent_t> g_pool;
std::vector<Pending> g_pending;
std::map<std::string, Totals> g_totals;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Folds finished event pairs into the totals (caller holds the lock).
cudaError_t resolve_pending() {
    cudaError_t first = cudaSuccess;
    for (auto &p : g_pending) {
        cudaError_t e = cudaEventSynchronize(p.stop);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.start, p.stop);
        if (e == cudaSuccess) {
            Totals &t = g_totals[p.name];
            t.ms += ms;
            t.launches += 1;
        } else if (first == cudaSuccess) {
            first = e;
        }
        if (!p.captured) {
            g_pool.push_back(p.start);
            g_pool.push_back(p.stop);
        }
    }
    g_pending.clear();
    return first;
}
}  // namespace

namespace {
bool capturing(cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(s, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive;
}
// Inside a capture an ordinary record only marks a dependency; an external
// record becomes a node that takes a timestamp whenever the graph runs.
void record(cudaEvent_t e, cudaStream_t s, bool captured) {
    if (captured)
        cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else
        cudaEventRecord(e, s);
}
}  // namespace

KernelTimer::KernelTimer(const char *name, cudaStream_t stream) : stream_(stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_enabled || (!g_only.empty() && g_only != name)) return;
    captured_ = capturing(stream_);
    if (captured_) {                       // fresh events: the graph keeps using them
        cudaEvent_t a = nullptr, b = nullptr;
        if (cudaEventCreate(&a) != cudaSuccess) return;
        if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
        start_ = a;
        stop_ = b;
    } else {
        start_ = take_event();
        stop_ = take_event();
        if (!start_ || !stop_) return;
    }
    name_ = name;
    record((cudaEvent_t)start_, stream_, captured_);
}

KernelTimer::~KernelTimer() {
    if (!name_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    record((cudaEvent_t)stop_, stream_, captured_);
    g_pending.push_back({name_, (cudaEvent_t)start_, (cudaEvent_t)stop_, captured_});
}

}  // namespace retnet

using namespace retnet;

extern "C" {

retnet_status retnet_profiler_enable(int on) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_enabled = on != 0;
    return RETNET_OK;
}

retnet_status retnet_profiler_select(const char *name) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_only = name ? std::string(name) : std::string();
    return RETNET_OK;
}

retnet_status retnet_profiler_reset(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    cudaError_t e = resolve_pending();
    g_totals.clear();
    return e == cudaSuccess ? RETNET_OK : RETNET_ERR_CUDA;
}

retnet_status retnet_profiler_read(int index, char *name, size_t name_len, double *total_ms,
                                   unsigned long long *launches) {
    if (index < 0 || !name || name_len == 0 || !total_ms || !launches)
        return RETNET_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    if (resolve_pending() != cudaSuccess) return RETNET_ERR_CUDA;
    if (index >= (int)g_totals.size()) return RETNET_ERR_INVALID_ARG;
    auto it = g_totals.begin();
    std::advance(it, index);
    std::strncpy(name, it->first.c_str(), name_len - 1);
    name[name_len - 1] = '\0';
    *total_ms = it->second.ms;
    *launches = it->second.launches;
    return RETNET_OK;
}

}  // extern "C"
