// profile.cu — optional per-kernel timing: when enabled, every launch of the
// library is bracketed by two CUDA events recorded on the launching stream;
// moe_profile_collect() waits for them and sums the elapsed times per kernel.
// Off by default; when off, the launchers record nothing.
#include <mutex>
#include <vector>

#include "internal.h"

namespace moe {

namespace {

struct Rec {
    int id;
    cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

ProfScope::ProfScope(int id, cudaStream_t s) : id_(id), s_(s), a_(nullptr) {
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_on) return;
    a_ = take_event();
    if (a_) cudaEventRecord(static_cast<cudaEvent_t>(a_), s_);
}

ProfScope::~ProfScope() {
    if (!a_) return;
    std::lock_guard<std::mutex> g(g_mu);
    cudaEvent_t b = take_event();
    if (!b) {
        g_pool.push_back(static_cast<cudaEvent_t>(a_));
        return;
    }
    cudaEventRecord(b, s_);
    g_recs.push_back(Rec{id_, static_cast<cudaEvent_t>(a_), b});
}

}  // namespace moe

extern "C" {

MOE_API int moe_profile_enable(int on) {
    std::lock_guard<std::mutex> g(moe::g_mu);
    moe::g_on = on != 0;
    return MOE_OK;
}

MOE_API int moe_profile_collect(double* total_ms, int64_t* launches) {
    if (!total_ms || !launches) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(moe::g_mu);
    for (int i = 0; i < MOE_K_COUNT; ++i) {
        total_ms[i] = 0.0;
        launches[i] = 0;
    }
    int st = MOE_OK;
    for (const auto& r : moe::g_recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            st = MOE_ERR_CUDA;
        if (r.id >= 0 && r.id < MOE_K_COUNT) {
            total_ms[r.id] += ms;
            launches[r.id] += 1;
        }
        moe::g_pool.push_back(r.a);
        moe::g_pool.push_back(r.b);
    }
    moe::g_recs.clear();
    return st;
}

}  // extern "C"
