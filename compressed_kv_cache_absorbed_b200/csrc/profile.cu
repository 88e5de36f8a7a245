// Optional per-kernel device timing of the library's own launches: when enabled, every
// launch is bracketed by two CUDA events recorded on the launching stream.
#include <stdio.h>
#include <string.h>

#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "mla.h"

namespace {

struct Rec {
    const char* name;
    cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_open;            // recorded, not yet read
std::vector<cudaEvent_t> g_pool;    // free events
std::map<std::string, std::pair<long long, double>> g_acc;  // name -> (launches, total ms)
const char* g_pending = nullptr;
cudaEvent_t g_pending_ev = nullptr;

cudaEvent_t take() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

void drain() {
    for (auto& r : g_open) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            auto& v = g_acc[r.name];
            v.first += 1;
            v.second += ms;
        }
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_open.clear();
}

}  // namespace

namespace mla {

void prof_begin(cudaStream_t s, const char* name) {
    if (!g_on) return;
    std::lock_guard<std::mutex> g(g_mu);
    g_pending = name;
    g_pending_ev = take();
    cudaEventRecord(g_pending_ev, s);
}

void prof_end(cudaStream_t s) {
    if (!g_on) return;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_pending) return;
    cudaEvent_t b = take();
    cudaEventRecord(b, s);
    g_open.push_back({g_pending, g_pending_ev, b});
    g_pending = nullptr;
    if (g_open.size() > 4096) drain();
}

}  // namespace mla

extern "C" void mla_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> g(g_mu);
    g_on = on != 0;
}

extern "C" int32_t mla_profile_report(char* buf, size_t cap, int32_t reset) {
    std::lock_guard<std::mutex> g(g_mu);
    drain();
    std::string out;
    char line[256];
    for (auto& kv : g_acc) {
        snprintf(line, sizeof line, "%s %lld %.6f\n", kv.first.c_str(), kv.second.first, kv.second.second);
        out += line;
    }
    if (buf && cap) {
        strncpy(buf, out.c_str(), cap - 1);
        buf[cap - 1] = 0;
    }
    const int32_t n = (int32_t)g_acc.size();
    if (reset) g_acc.clear();
    return n;
}
