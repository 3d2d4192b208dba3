// oal_prof.cuh -- launch accounting and optional per-kernel CUDA-event tracing.
//
// Every kernel launch of the library goes through a LaunchScope: it counts the launch, and
// while tracing is enabled (oal_profile_enable) records a CUDA event pair around it on the
// launching stream, taking the events from a pool created when tracing was switched on (no
// event creation on the launch path).  oal_profile_read turns the pairs into per-kernel
// totals and returns the events to the pool.  Host only.
#pragma once

#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

namespace oal {

struct TraceRecord {
    const char* name;
    cudaEvent_t start, stop;
};

struct Tracer {
    std::atomic<unsigned long long> launches{0};
    std::atomic<int> enabled{0};
    std::mutex mu;
    std::vector<TraceRecord> records;    // recorded, not yet read
    std::vector<cudaEvent_t> pool;       // free events
    int device = -1;                     // device the pool's events belong to
    static constexpr size_t kPoolPairs = 4096;
};

inline Tracer& tracer()
{
    static Tracer t;
    return t;
}

// Creates the event pool on the current device (called with the mutex held).
inline bool tracer_fill_pool(Tracer& t)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (t.device != dev) {
        for (cudaEvent_t e : t.pool) cudaEventDestroy(e);
        t.pool.clear();
        t.device = dev;
    }
    while (t.pool.size() < 2 * Tracer::kPoolPairs) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return false;
        t.pool.push_back(e);
    }
    return true;
}

class LaunchScope {
  public:
    LaunchScope(const char* name, cudaStream_t st) : name_(name), st_(st)
    {
        Tracer& t = tracer();
        t.launches.fetch_add(1, std::memory_order_relaxed);
        if (!t.enabled.load(std::memory_order_relaxed)) return;
        std::lock_guard<std::mutex> g(t.mu);
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || dev != t.device || t.pool.size() < 2) return;
        stop_ = t.pool.back();
        t.pool.pop_back();
        start_ = t.pool.back();
        t.pool.pop_back();
        active_ = cudaEventRecord(start_, st_) == cudaSuccess;
        if (!active_) {
            t.pool.push_back(start_);
            t.pool.push_back(stop_);
        }
    }
    ~LaunchScope()
    {
        if (!active_) return;
        Tracer& t = tracer();
        cudaEventRecord(stop_, st_);
        std::lock_guard<std::mutex> g(t.mu);
        t.records.push_back({name_, start_, stop_});
    }
    LaunchScope(const LaunchScope&) = delete;
    LaunchScope& operator=(const LaunchScope&) = delete;

  private:
    const char* name_;
    cudaStream_t st_;
    cudaEvent_t start_{}, stop_{};
    bool active_ = false;
};

}  // namespace oal
