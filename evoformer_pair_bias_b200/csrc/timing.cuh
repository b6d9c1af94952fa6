// timing.cuh -- optional per-kernel timing with CUDA events on the launch stream.
//
// Off by default.  When switched on, every call brackets its main kernel (and
// the backward as a whole) with a pair of events recorded on the stream the
// kernels go to, so the device time of each phase can be read back after the
// work has run.  Events come from a per-device pool that collect() refills,
// so steady-state calls create none.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "evo_attn.h"

namespace evo {
namespace timing {

struct Rec {
    int phase;
    int dev;
    cudaEvent_t a, b;
};

struct State {
    std::mutex mu;
    bool on = false;
    std::vector<std::pair<int, cudaEvent_t>> pool;   // (device, event)
    std::vector<Rec> pending;
};

inline State& state() {
    static State s;
    return s;
}

inline cudaEvent_t take(State& s, int dev) {
    for (size_t i = s.pool.size(); i-- > 0;) {
        if (s.pool[i].first == dev) {
            cudaEvent_t e = s.pool[i].second;
            s.pool.erase(s.pool.begin() + (long)i);
            return e;
        }
    }
    cudaEvent_t e = nullptr;
    return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
}

// Brackets one phase on `stream`.  Does nothing while timing is off or when an
// event cannot be had; never fails the call it wraps.
class Scope {
  public:
    Scope(int phase, cudaStream_t stream) : stream_(stream) {
        State& s = state();
        std::lock_guard<std::mutex> lock(s.mu);
        if (!s.on || cudaGetDevice(&rec_.dev) != cudaSuccess) return;
        rec_.phase = phase;
        rec_.a = take(s, rec_.dev);
        rec_.b = take(s, rec_.dev);
        if (!rec_.a || !rec_.b || cudaEventRecord(rec_.a, stream_) != cudaSuccess) {
            if (rec_.a) s.pool.emplace_back(rec_.dev, rec_.a);
            if (rec_.b) s.pool.emplace_back(rec_.dev, rec_.b);
            rec_.a = rec_.b = nullptr;
        }
    }
    ~Scope() {
        if (!rec_.a) return;
        State& s = state();
        std::lock_guard<std::mutex> lock(s.mu);
        if (cudaEventRecord(rec_.b, stream_) == cudaSuccess) {
            s.pending.push_back(rec_);
        } else {
            s.pool.emplace_back(rec_.dev, rec_.a);
            s.pool.emplace_back(rec_.dev, rec_.b);
        }
    }
    Scope(const Scope&) = delete;
    Scope& operator=(const Scope&) = delete;

  private:
    cudaStream_t stream_;
    Rec rec_{0, 0, nullptr, nullptr};
};

inline evo_status_t enable(int on) {
    State& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    s.on = on != 0;
    return EVO_OK;
}

// Waits for every recorded phase, sums its device time into `out` and returns
// the events to the pool.
inline evo_status_t collect(evo_timing_t* out) {
    if (!out) return EVO_ERR_INVALID_ARG;
    *out = evo_timing_t{};
    State& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    evo_status_t st = EVO_OK;
    for (const Rec& r : s.pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            st = EVO_ERR_CUDA;
        } else if (r.phase >= 0 && r.phase < EVO_TIMING_PHASES) {
            out->calls[r.phase] += 1;
            out->ms[r.phase] += ms;
        }
        s.pool.emplace_back(r.dev, r.a);
        s.pool.emplace_back(r.dev, r.b);
    }
    s.pending.clear();
    return st;
}

}  // namespace timing
}  // namespace evo
