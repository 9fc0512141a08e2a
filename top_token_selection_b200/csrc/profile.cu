// profile.cu -- optional per-launch kernel timing and launch counting.
//
// When timing is on, every kernel the library launches is bracketed by two
// CUDA events recorded on the launch's own stream, together with the
// algorithmic work of that launch (indexer pairs for the scans, entries for
// the selection, bytes for the memory-bound kernels).  Reading the totals
// waits on the recorded events.  Launch counting is always on and costs one
// atomic increment per launch.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace pivot {

namespace {

struct Record {
    int kernel;
    cudaEvent_t a, b;
    double work;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Record> g_pending;
std::vector<cudaEvent_t> g_pool;
std::atomic<long long> g_launches{0};
long long g_count[PK_COUNT] = {0};
double g_ms[PK_COUNT] = {0};
double g_work[PK_COUNT] = {0};

cudaEvent_t get_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

void resolve_pending() {
    for (const Record& r : g_pending) {
        float ms = 0.0f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            g_count[r.kernel] += 1;
            g_ms[r.kernel] += ms;
            g_work[r.kernel] += r.work;
        }
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_pending.clear();
}

}  // namespace

bool prof_begin(int kernel, cudaStream_t s, cudaEvent_t* a, cudaEvent_t* b) {
    (void)kernel;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on) return false;
    *a = get_event();
    *b = get_event();
    cudaEventRecord(*a, s);
    return true;
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void prof_end(int kernel, cudaStream_t s, cudaEvent_t a, cudaEvent_t b, double work) {
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_mu);
    g_pending.push_back(Record{kernel, a, b, work});
}

}  // namespace pivot

using namespace pivot;

extern "C" {

pivot_status_t pivot_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_mu);
    resolve_pending();
    if (on) {   // a new measurement starts from zero; turning off keeps the totals
        for (int k = 0; k < PK_COUNT; ++k) {
            g_count[k] = 0;
            g_ms[k] = 0.0;
            g_work[k] = 0.0;
        }
    }
    g_on = on != 0;
    return PIVOT_OK;
}

pivot_status_t pivot_profile_read(int32_t kernel, int64_t* launches, double* total_ms,
                                  double* work) {
    if (kernel < 0 || kernel >= PK_COUNT) return PIVOT_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    resolve_pending();
    if (launches) *launches = g_count[kernel];
    if (total_ms) *total_ms = g_ms[kernel];
    if (work) *work = g_work[kernel];
    return PIVOT_OK;
}

int64_t pivot_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
