// Diagnostic kernel timing: CUDA events around each launch while enabled,
// summed per kernel kind when read.  Host code only; nothing here runs unless
// a caller turns it on (ckv_kernel_timing), so the normal path pays one
// atomic load per launch.
#include <atomic>
#include <mutex>
#include <vector>

#include "ckv_internal.cuh"

namespace ckv {
namespace {

struct Mark {
    int kind;
    cudaEvent_t start, end;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<cudaEvent_t> g_pool;  // events free for reuse
std::vector<Mark> g_done;         // recorded, not yet read
thread_local cudaEvent_t t_open = nullptr;
thread_local int t_open_kind = -1;

cudaError_t take_event(cudaEvent_t* ev) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_pool.empty()) {
            *ev = g_pool.back();
            g_pool.pop_back();
            return cudaSuccess;
        }
    }
    return cudaEventCreate(ev);
}

}  // namespace

bool timing_enabled() { return g_on.load(std::memory_order_relaxed); }

cudaError_t timing_mark(int kind, bool start, cudaStream_t st) {
    cudaEvent_t ev = nullptr;
    cudaError_t e = take_event(&ev);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(ev, st);
    if (e != cudaSuccess) return e;
    if (start) {
        if (t_open) {  // a launch failed after its start mark: reuse that event
            std::lock_guard<std::mutex> lk(g_mu);
            g_pool.push_back(t_open);
        }
        t_open = ev;
        t_open_kind = kind;
        return cudaSuccess;
    }
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (t_open && t_open_kind == kind) {
            g_done.push_back(Mark{kind, t_open, ev});
        } else {  // no matching start: nothing to time
            if (t_open) g_pool.push_back(t_open);
            g_pool.push_back(ev);
        }
    }
    t_open = nullptr;
    t_open_kind = -1;
    return cudaSuccess;
}

void timing_set(bool on) { g_on.store(on, std::memory_order_relaxed); }

// Waits for every recorded pair, adds its duration to total_ms[kind] and one
// launch to launches[kind], and returns the events to the pool.
cudaError_t timing_read(float* total_ms, int32_t* launches) {
    std::vector<Mark> done;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        done.swap(g_done);
    }
    for (int k = 0; k < KK_COUNT; ++k) {
        total_ms[k] = 0.f;
        launches[k] = 0;
    }
    cudaError_t err = cudaSuccess;
    for (const Mark& m : done) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(m.end);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, m.start, m.end);
        if (e == cudaSuccess) {
            total_ms[m.kind] += ms;
            launches[m.kind] += 1;
        } else if (err == cudaSuccess) {
            err = e;
        }
    }
    std::lock_guard<std::mutex> lk(g_mu);
    for (const Mark& m : done) {
        g_pool.push_back(m.start);
        g_pool.push_back(m.end);
    }
    return err;
}

}  // namespace ckv
