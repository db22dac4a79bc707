// launch_timer.cuh -- optional per-launch timing of the library's kernels with CUDA events.
//
// While timing is on (gdn_timing_start .. gdn_timing_stop), every kernel launch the library
// makes is bracketed by a pair of events recorded on the launch's own stream, so a caller can
// split the device time of a multi-kernel entry point (gdn_chunk_fwd launches two kernels)
// into per-kernel durations without a profiler.  The events come from a pool created when
// timing starts; launches beyond the pool, or made on another device, run untimed.
#pragma once

#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <vector>

namespace gdn {

struct LaunchTimer {
    std::mutex mu;
    bool on = false;
    int device = -1;
    unsigned generation = 0;
    std::vector<cudaEvent_t> pool;      // 2 events per timed launch
    std::vector<const char*> names;     // kernel name of each timed launch (static strings)
};

inline LaunchTimer& launch_timer() {
    static LaunchTimer t;
    return t;
}

// Records the start event in the constructor and the end event in the destructor; put one
// around each launch (the launch's error check may sit inside the scope).
class LaunchScope {
  public:
    LaunchScope(cudaStream_t st, const char* name) : st_(st) {
        LaunchTimer& t = launch_timer();
        std::lock_guard<std::mutex> lock(t.mu);
        if (!t.on || 2 * (t.names.size() + 1) > t.pool.size()) return;
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || dev != t.device) return;
        const size_t i = t.names.size();
        if (cudaEventRecord(t.pool[2 * i], st) != cudaSuccess) return;
        t.names.push_back(name);
        idx_ = (long)i;
        gen_ = t.generation;
    }
    ~LaunchScope() {
        if (idx_ < 0) return;
        LaunchTimer& t = launch_timer();
        std::lock_guard<std::mutex> lock(t.mu);
        if (t.generation == gen_ && (size_t)idx_ < t.names.size())
            cudaEventRecord(t.pool[2 * idx_ + 1], st_);
    }
    LaunchScope(const LaunchScope&) = delete;
    LaunchScope& operator=(const LaunchScope&) = delete;

  private:
    cudaStream_t st_;
    long idx_ = -1;
    unsigned gen_ = 0;
};

}  // namespace gdn
