// profile.cu -- opt-in per-kernel timing with CUDA events (tracing aid).
//
// When enabled, every kernel launch of the library is bracketed by two CUDA events recorded on
// the launching stream. lnq_profile_read() waits for those events and returns, per kernel name,
// the number of launches and their summed device time. Events are host/driver objects; no device
// memory is allocated.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "profile.cuh"

namespace lnq {

namespace {
struct Record {
    const char *name;
    cudaEvent_t start, stop;
};
std::atomic<int> g_enabled{0};
std::mutex g_mu;
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event()
{
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess)
        return nullptr;
    return e;
}
}  // namespace

KernelTimer::KernelTimer(const char *name, cudaStream_t s) : name_(name), stream_(s)
{
    if (g_enabled.load(std::memory_order_relaxed) == 0)
        return;
    std::lock_guard<std::mutex> lk(g_mu);
    start_ = take_event();
    stop_ = take_event();
    if (start_ == nullptr || stop_ == nullptr || cudaEventRecord(start_, s) != cudaSuccess) {
        start_ = stop_ = nullptr;
        return;
    }
    active_ = true;
}

KernelTimer::~KernelTimer()
{
    if (!active_)
        return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (cudaEventRecord(stop_, stream_) == cudaSuccess)
        g_records.push_back({name_, start_, stop_});
}

}  // namespace lnq

extern "C" {

LNQ_API void lnq_profile_enable(int on) { lnq::g_enabled.store(on ? 1 : 0); }

LNQ_API int lnq_profile_read(int max_kernels, const char **names, double *total_ms,
                             int64_t *launches)
{
    using namespace lnq;
    std::lock_guard<std::mutex> lk(g_mu);
    int count = 0;
    for (const Record &r : g_records) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess ||
            cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
            ms = -1.f;
        int slot = -1;
        for (int k = 0; k < count; ++k)
            if (std::strcmp(names[k], r.name) == 0)
                slot = k;
        if (slot < 0 && count < max_kernels) {
            slot = count++;
            names[slot] = r.name;
            total_ms[slot] = 0.0;
            launches[slot] = 0;
        }
        if (slot >= 0) {
            total_ms[slot] += ms;
            launches[slot] += 1;
        }
        g_pool.push_back(r.start);
        g_pool.push_back(r.stop);
    }
    g_records.clear();
    return count;
}

}  // extern "C"
