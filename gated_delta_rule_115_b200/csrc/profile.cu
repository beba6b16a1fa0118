// profile.cu -- opt-in per-kernel CUDA-event timing (see include/muir_profile.h).
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/muir_profile.h"
#include "profile.h"

namespace muir {
namespace prof {
namespace {

struct Pending {
    int id;
    cudaEvent_t start, stop;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<std::string> g_names;
std::vector<double> g_ms;
std::vector<long long> g_count;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;

cudaEvent_t take_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

int name_id(const char* n) {
    for (size_t i = 0; i < g_names.size(); ++i)
        if (g_names[i] == n) return (int)i;
    g_names.emplace_back(n);
    g_ms.push_back(0.0);
    g_count.push_back(0);
    return (int)g_names.size() - 1;
}

}  // namespace

bool enabled() { return g_on.load(std::memory_order_relaxed); }

int begin(const char* name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    Pending p;
    p.id = name_id(name);
    p.start = take_event();
    p.stop = take_event();
    if (!p.start || !p.stop) return -1;
    cudaEventRecord(p.start, st);
    g_pending.push_back(p);
    return (int)g_pending.size() - 1;
}

void end(int ticket, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (ticket >= 0 && ticket < (int)g_pending.size()) cudaEventRecord(g_pending[ticket].stop, st);
}

}  // namespace prof
}  // namespace muir

using namespace muir::prof;

extern "C" {

void muir_profile_enable(int on) { g_on.store(on != 0); }

void muir_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (auto& p : g_pending) {
        cudaEventSynchronize(p.stop);
        g_free.push_back(p.start);
        g_free.push_back(p.stop);
    }
    g_pending.clear();
    g_names.clear();
    g_ms.clear();
    g_count.clear();
}

int muir_profile_collect(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int rc = 0;
    for (auto& p : g_pending) {
        cudaError_t e = cudaEventSynchronize(p.stop);
        float ms = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.start, p.stop);
        if (e == cudaSuccess) {
            g_ms[p.id] += ms;
            g_count[p.id] += 1;
        } else if (rc == 0) {
            rc = (int)e;
        }
        g_free.push_back(p.start);
        g_free.push_back(p.stop);
    }
    g_pending.clear();
    return rc;
}

int muir_profile_count(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    return (int)g_names.size();
}

const char* muir_profile_name(int i) {
    std::lock_guard<std::mutex> lk(g_mu);
    return (i >= 0 && i < (int)g_names.size()) ? g_names[i].c_str() : nullptr;
}

double muir_profile_total_ms(int i) {
    std::lock_guard<std::mutex> lk(g_mu);
    return (i >= 0 && i < (int)g_ms.size()) ? g_ms[i] : 0.0;
}

long long muir_profile_launches(int i) {
    std::lock_guard<std::mutex> lk(g_mu);
    return (i >= 0 && i < (int)g_count.size()) ? g_count[i] : 0;
}

}  // extern "C"
