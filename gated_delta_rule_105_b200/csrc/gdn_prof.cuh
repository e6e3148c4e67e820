// Optional per-kernel device timing of the library's own launches (host side).  Off by default; while on,
// each launch is bracketed by two CUDA events recorded on the launching stream, and gdn_profile_take()
// later waits for them and reports launches and device milliseconds per kernel.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

namespace gdn {

enum ProfKernel : int {
    PK_SIMT = 0, PK_TC_WY = 1, PK_TC_MAIN = 2, PK_TC2_PREP = 3, PK_TC2_MAIN = 4, PK_DECODE = 5, PK_PRELUDE = 6,
    PK_OUT_GATE = 7, PK_BWD = 8, PK_COUNT = 9
};

struct ProfState {
    std::atomic<bool> on{false};
    std::mutex mu;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[PK_COUNT];
    std::vector<cudaEvent_t> pool;
};
inline ProfState& prof_state() {
    static ProfState s;
    return s;
}
inline cudaEvent_t prof_event_locked(ProfState& s) {
    if (!s.pool.empty()) {
        cudaEvent_t e = s.pool.back();
        s.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Brackets one launch: construct before it, call done() after it.
class ProfScope {
   public:
    ProfScope(int kernel, cudaStream_t stream) : kernel_(kernel), stream_(stream) {
        ProfState& s = prof_state();
        if (!s.on.load()) return;
        std::lock_guard<std::mutex> lock(s.mu);
        begin_ = prof_event_locked(s);
        end_ = prof_event_locked(s);
        if (begin_ && end_ && cudaEventRecord(begin_, stream_) != cudaSuccess) begin_ = nullptr;
    }
    void done() {
        if (!begin_ || !end_) return;
        ProfState& s = prof_state();
        std::lock_guard<std::mutex> lock(s.mu);
        if (cudaEventRecord(end_, stream_) == cudaSuccess) s.pending[kernel_].push_back({begin_, end_});
        begin_ = end_ = nullptr;
    }

   private:
    int kernel_;
    cudaStream_t stream_;
    cudaEvent_t begin_ = nullptr, end_ = nullptr;
};

// Waits for the recorded launches of `kernel`, returns their count and total device time, and forgets them.
inline bool prof_take(int kernel, int* launches, double* total_ms) {
    ProfState& s = prof_state();
    std::lock_guard<std::mutex> lock(s.mu);
    int n = 0;
    double ms = 0.0;
    bool ok = true;
    for (auto& pr : s.pending[kernel]) {
        float t = 0.f;
        if (cudaEventSynchronize(pr.second) != cudaSuccess || cudaEventElapsedTime(&t, pr.first, pr.second) != cudaSuccess)
            ok = false;
        ms += t;
        ++n;
        s.pool.push_back(pr.first);
        s.pool.push_back(pr.second);
    }
    s.pending[kernel].clear();
    *launches = n;
    *total_ms = ms;
    return ok;
}

}  // namespace gdn
