// Kernel timing instrumentation (include/kata_profile.h): CUDA events recorded
// on the launching stream around each kernel launch while enabled.
#include <mutex>
#include <string.h>
#include <vector>

#include "../../include/kata_profile.h"
#include "kata_internal.cuh"

namespace kata {
namespace {

constexpr int kMaxRecords = 65536;

struct Record {
    const char *name;
    int ev;  // index of the start event; stop is ev + 1
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<cudaEvent_t> events;
    std::vector<Record> records;
    int dropped = 0;
    // aggregated results
    std::vector<const char *> names;
    std::vector<int> launches;
    std::vector<double> total_ms;
};

Profiler &prof() {
    static Profiler p;
    return p;
}

}  // namespace

int prof_begin(const char *name, cudaStream_t st) {
    Profiler &p = prof();
    if (!p.on) return -1;
    std::lock_guard<std::mutex> lk(p.mu);
    if ((int)p.records.size() >= kMaxRecords) {
        ++p.dropped;
        return -1;
    }
    const int ev = 2 * (int)p.records.size();
    while ((int)p.events.size() < ev + 2) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return -1;
        p.events.push_back(e);
    }
    p.records.push_back({name, ev});
    cudaEventRecord(p.events[ev], st);
    return ev;
}

void prof_end(int ev, cudaStream_t st) {
    if (ev < 0) return;
    Profiler &p = prof();
    cudaEventRecord(p.events[ev + 1], st);
}

}  // namespace kata

using kata::prof;

extern "C" {

kata_status kata_profile_enable(int enable) {
    kata::Profiler &p = prof();
    std::lock_guard<std::mutex> lk(p.mu);
    if (enable) {
        p.records.clear();
        p.names.clear();
        p.launches.clear();
        p.total_ms.clear();
        p.dropped = 0;
    }
    p.on = enable != 0;
    return KATA_OK;
}

int kata_profile_kernel_count(void) {
    kata::Profiler &p = prof();
    std::lock_guard<std::mutex> lk(p.mu);
    p.names.clear();
    p.launches.clear();
    p.total_ms.clear();
    for (const kata::Record &r : p.records) {
        if (cudaEventSynchronize(p.events[r.ev + 1]) != cudaSuccess) return -1;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.events[r.ev], p.events[r.ev + 1]) != cudaSuccess) return -1;
        size_t i = 0;
        while (i < p.names.size() && strcmp(p.names[i], r.name) != 0) ++i;
        if (i == p.names.size()) {
            p.names.push_back(r.name);
            p.launches.push_back(0);
            p.total_ms.push_back(0.0);
        }
        p.launches[i] += 1;
        p.total_ms[i] += ms;
    }
    return (int)p.names.size();
}

kata_status kata_profile_kernel(int idx, const char **name, int *launches, double *total_ms) {
    kata::Profiler &p = prof();
    std::lock_guard<std::mutex> lk(p.mu);
    if (idx < 0 || idx >= (int)p.names.size()) return KATA_ERR_INVALID_ARG;
    if (name) *name = p.names[idx];
    if (launches) *launches = p.launches[idx];
    if (total_ms) *total_ms = p.total_ms[idx];
    return KATA_OK;
}

int kata_profile_dropped(void) { return prof().dropped; }

}  // extern "C"
