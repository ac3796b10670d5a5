// Per-kernel timing with CUDA events (tracing aid, off by default).
//
// While enabled, every kernel the library launches is bracketed by a pair of
// events recorded on the launch stream.  laplex_profile_report synchronises on
// those events and returns, per kernel name, the number of launches and the sum
// of their device durations.  Events come from a pool that grows on demand and
// is reused after every report.
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "laplex.h"
#include "laplex_internal.h"

namespace laplex {

namespace {

struct Mark {
    const char* name;
    cudaEvent_t start, stop;
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<cudaEvent_t> pool;
    size_t used = 0;
    std::vector<Mark> marks;

    cudaEvent_t take() {
        if (used == pool.size()) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            pool.push_back(e);
        }
        return pool[used++];
    }
};

Profiler& prof() {
    static Profiler p;
    return p;
}

}  // namespace

bool profiling() { return prof().on; }

void* profile_begin(const char* name, cudaStream_t st) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.on) return nullptr;
    Mark m{name, p.take(), p.take()};
    if (!m.start || !m.stop) return nullptr;
    cudaEventRecord(m.start, st);
    p.marks.push_back(m);
    return (void*)(p.marks.size());  // 1-based index
}

void profile_end(void* token, cudaStream_t st) {
    if (token == nullptr) return;
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    const size_t i = (size_t)token - 1;
    if (i < p.marks.size()) cudaEventRecord(p.marks[i].stop, st);
}

}  // namespace laplex

using namespace laplex;

extern "C" {

void laplex_profile_enable(int on) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    p.on = (on != 0);
    p.marks.clear();
    p.used = 0;
}

int laplex_profile_report(int max_kernels, char* names, int name_len, int* launches, double* total_ms) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    std::vector<std::string> keys;
    std::vector<int> cnt;
    std::vector<double> ms;
    for (const Mark& m : p.marks) {
        if (cudaEventSynchronize(m.stop) != cudaSuccess) return -1;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, m.start, m.stop) != cudaSuccess) return -1;
        size_t k = 0;
        while (k < keys.size() && keys[k] != m.name) ++k;
        if (k == keys.size()) {
            keys.push_back(m.name);
            cnt.push_back(0);
            ms.push_back(0.0);
        }
        cnt[k] += 1;
        ms[k] += t;
    }
    const int nk = (int)keys.size();
    for (int k = 0; k < nk && k < max_kernels; ++k) {
        if (names && name_len > 0) {
            std::strncpy(names + (size_t)k * name_len, keys[k].c_str(), name_len - 1);
            names[(size_t)k * name_len + name_len - 1] = '\0';
        }
        if (launches) launches[k] = cnt[k];
        if (total_ms) total_ms[k] = ms[k];
    }
    p.marks.clear();
    p.used = 0;
    return nk;
}

}  // extern "C"
