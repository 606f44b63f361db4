// Launch counting and per-kernel CUDA-event timing for measurement.
//
// Every kernel launch of the library goes through Launch::before / after.
// Launches are always counted.  When a kernel name is selected with
// ca_profile_start, each launch of that kernel is bracketed by two CUDA
// events recorded on the launching stream; ca_profile_stop synchronizes on
// the recorded events and returns the summed durations.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

namespace ca {

struct ProfileState {
    std::mutex mu;
    std::atomic<long long> launches{0};
    std::string selected;  // empty: time nothing
    bool active = false;
    struct Pair {
        cudaEvent_t a, b;
        double bytes;
    };
    std::vector<Pair> pairs;
    std::vector<cudaEvent_t> pool;

    cudaEvent_t get_event() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
};

inline ProfileState &profile() {
    static ProfileState s;
    return s;
}

// Brackets one launch.  Usage: Launch pl("name", stream, bytes); kernel<<<...>>>; pl.after();
struct Launch {
    const char *name;
    cudaStream_t st;
    double bytes;
    cudaEvent_t a = nullptr;
    Launch(const char *n, cudaStream_t s, double alg_bytes) : name(n), st(s), bytes(alg_bytes) {
        ProfileState &p = profile();
        p.launches.fetch_add(1, std::memory_order_relaxed);
        if (p.active) {
            std::lock_guard<std::mutex> g(p.mu);
            if (p.active && p.selected == name) {
                a = p.get_event();
                cudaEventRecord(a, st);
            }
        }
    }
    void after() {
        if (!a) return;
        ProfileState &p = profile();
        std::lock_guard<std::mutex> g(p.mu);
        cudaEvent_t b = p.get_event();
        cudaEventRecord(b, st);
        p.pairs.push_back({a, b, bytes});
        a = nullptr;
    }
};

}  // namespace ca
