// Per-kernel timing with CUDA events, and a process-wide launch counter.
//
// When tracing is enabled, every entry point records one event on its stream when it
// starts and one after each kernel it launches, from a fixed pool created by
// hs2_trace_enable (no device memory is allocated).  hs2_trace_collect waits for the
// recorded events, turns consecutive pairs into per-kernel durations, sums them per
// kernel name, and clears the record.  Host-side state is process-global and not
// thread-safe; it is meant for benchmarking and profiling runs.
#include <atomic>
#include <cstring>
#include <vector>

#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr int kPool = 8192;

struct Mark {
    const char* name;  // nullptr marks the start of a call
    cudaEvent_t ev;
};

struct TraceState {
    bool enabled = false;
    std::vector<cudaEvent_t> pool;
    std::vector<Mark> marks;
    bool overflow = false;
};

TraceState& state() {
    static TraceState s;
    return s;
}

std::atomic<uint64_t> g_launches{0};

void record(const char* name, cudaStream_t st) {
    TraceState& s = state();
    if (!s.enabled) return;
    if (s.marks.size() >= s.pool.size()) {
        s.overflow = true;
        return;
    }
    cudaEvent_t ev = s.pool[s.marks.size()];
    if (cudaEventRecord(ev, st) == cudaSuccess) s.marks.push_back(Mark{name, ev});
}

}  // namespace

void trace_call_begin(cudaStream_t st) { record(nullptr, st); }

void trace_mark(const char* name, cudaStream_t st, bool kernel) {
    if (kernel) g_launches.fetch_add(1, std::memory_order_relaxed);
    record(name, st);
}

}  // namespace hs2

using namespace hs2;

extern "C" {

hs2_status hs2_trace_enable(int enable) {
    TraceState& s = state();
    if (enable && s.pool.empty()) {
        s.pool.resize(kPool);
        for (auto& e : s.pool)
            if (cudaEventCreate(&e) != cudaSuccess) {
                s.pool.clear();
                return HS2_ERR_CUDA;
            }
    }
    s.enabled = enable != 0;
    s.marks.clear();
    s.overflow = false;
    return HS2_OK;
}

int hs2_trace_collect(const char** names, double* total_ms, int64_t* launches, int max_entries) {
    TraceState& s = state();
    int n = 0;
    if (!s.marks.empty() && cudaEventSynchronize(s.marks.back().ev) != cudaSuccess) {
        s.marks.clear();
        return -1;
    }
    for (size_t i = 1; i < s.marks.size(); ++i) {
        const Mark& m = s.marks[i];
        if (!m.name) continue;  // a call boundary: no kernel between the previous mark and this one
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, s.marks[i - 1].ev, m.ev) != cudaSuccess) continue;
        int e = 0;
        while (e < n && std::strcmp(names[e], m.name) != 0) ++e;
        if (e == n) {
            if (n >= max_entries) continue;
            names[n] = m.name;
            total_ms[n] = 0.0;
            launches[n] = 0;
            ++n;
        }
        total_ms[e] += ms;
        launches[e] += 1;
    }
    s.marks.clear();
    const bool ovf = s.overflow;
    s.overflow = false;
    return ovf ? -n - 1 : n;
}

uint64_t hs2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
