// profile.cuh -- optional per-launch timing: CUDA events recorded around every kernel launch of
// the library, on the launch's own stream, while recording is switched on.  Host-side only; the
// events are created on first use and reused (no device memory is allocated).
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <string>
#include <vector>

namespace kda {

struct ProfRecord {
    const char* name;
    cudaEvent_t start, stop;
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<ProfRecord> recs;   // recorded this session
    std::vector<cudaEvent_t> pool;  // reusable events
    size_t used = 0;

    cudaEvent_t take()
    {
        if (used < pool.size()) return pool[used++];
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        pool.push_back(e);
        ++used;
        return e;
    }
};

inline Profiler& profiler()
{
    static Profiler p;
    return p;
}

// RAII scope around one launch.
struct LaunchScope {
    ProfRecord rec{nullptr, nullptr, nullptr};
    cudaStream_t stream;
    LaunchScope(const char* name, cudaStream_t s) : stream(s)
    {
        Profiler& p = profiler();
        std::lock_guard<std::mutex> g(p.mu);
        if (!p.on) return;
        rec.name = name;
        rec.start = p.take();
        rec.stop = p.take();
        if (rec.start) cudaEventRecord(rec.start, stream);
    }
    ~LaunchScope()
    {
        if (!rec.name || !rec.start || !rec.stop) return;
        cudaEventRecord(rec.stop, stream);
        Profiler& p = profiler();
        std::lock_guard<std::mutex> g(p.mu);
        p.recs.push_back(rec);
    }
};

}  // namespace kda
