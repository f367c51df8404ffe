// Launch accounting and optional per-kernel device timing.
//
// Every launcher brackets each kernel it enqueues with trace_begin/trace_end
// (the CSA_LAUNCH macro). trace_end counts the launch (csa_launch_count).
// While tracing is enabled (csa_trace_enable), the pair also records CUDA
// events on the launching stream, so csa_trace_read can report each
// kernel's device time as seen on its own stream. Disabled (the default),
// the cost is one atomic increment per launch.
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "kernels.h"

namespace csa {

namespace {
struct Rec {
    cudaEvent_t a, b;
    const char* name;
};
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_on{0};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

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
}  // namespace

int trace_begin(cudaStream_t st) {
    if (!g_on.load(std::memory_order_relaxed)) return -1;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t a = take_event();
    if (!a) return -1;
    cudaEventRecord(a, st);
    g_recs.push_back(Rec{a, nullptr, nullptr});
    return (int)g_recs.size() - 1;
}

void trace_end(int tok, cudaStream_t st, const char* name) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (tok < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (tok >= (int)g_recs.size()) return;
    cudaEvent_t b = take_event();
    if (!b) return;
    cudaEventRecord(b, st);
    g_recs[tok].b = b;
    g_recs[tok].name = name;
}

uint64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

void trace_enable(int on) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& r : g_recs) {
        if (r.a) g_pool.push_back(r.a);
        if (r.b) g_pool.push_back(r.b);
    }
    g_recs.clear();
    g_on.store(on ? 1 : 0);
}

int trace_read(int max_kernels, char* names, double* total_ms, int* counts, int* n_out) {
    std::lock_guard<std::mutex> lk(g_mu);
    int n = 0;
    for (auto& r : g_recs) {
        if (!r.b) continue;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e != cudaSuccess) return (int)e;
        float ms = 0.f;
        e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess) return (int)e;
        int j = 0;
        while (j < n && strncmp(names + (size_t)j * 64, r.name, 63) != 0) ++j;
        if (j == n) {
            if (n == max_kernels) continue;
            strncpy(names + (size_t)n * 64, r.name, 63);
            names[(size_t)n * 64 + 63] = 0;
            total_ms[n] = 0.0;
            counts[n] = 0;
            ++n;
        }
        total_ms[j] += ms;
        counts[j] += 1;
    }
    *n_out = n;
    return 0;
}

}  // namespace csa
