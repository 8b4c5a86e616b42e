// Optional kernel timing for benchmarks: when enabled, CUDA event pairs are
// recorded on the launch stream around the library's kernels, grouped by kind;
// qlora_timing_read synchronizes on the recorded events and reports the launch
// count and total device milliseconds per kind.  Disabled by default, in which
// case a TimerScope costs one relaxed atomic load.
#include <atomic>
#include <mutex>
#include <vector>

#include "qlora_internal.cuh"
#include "timing.cuh"

namespace qlora {
namespace {

std::atomic<int> g_enabled{0};
std::mutex g_mu;

struct Pending { int kind; cudaEvent_t a, b; };
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;
uint64_t g_count[QLORA_TIMER_KINDS] = {};
double g_ms[QLORA_TIMER_KINDS] = {};

cudaEvent_t get_event() {
    if (!g_free.empty()) { cudaEvent_t e = g_free.back(); g_free.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

qlora_status drain() {
    qlora_status st = QLORA_OK;
    for (const Pending& p : g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) {
            st = QLORA_ERR_CUDA;
        } else {
            g_count[p.kind] += 1;
            g_ms[p.kind] += ms;
        }
        g_free.push_back(p.a);
        g_free.push_back(p.b);
    }
    g_pending.clear();
    return st;
}

}  // namespace

TimerScope::TimerScope(int kind, cudaStream_t s) : kind_(kind), stream_(s), a_(nullptr), b_(nullptr) {
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_mu);
    a_ = get_event();
    b_ = get_event();
    if (a_ && b_) cudaEventRecord(a_, stream_);
}

TimerScope::~TimerScope() {
    if (!a_ || !b_) return;
    std::lock_guard<std::mutex> lock(g_mu);
    cudaEventRecord(b_, stream_);
    g_pending.push_back({kind_, a_, b_});
}

}  // namespace qlora

extern "C" {

qlora_status qlora_timing_enable(int32_t on) {
    qlora::g_enabled.store(on ? 1 : 0);
    return QLORA_OK;
}

qlora_status qlora_timing_read(int32_t kind, uint64_t* launches, double* total_ms, int32_t reset) {
    if (kind < 0 || kind >= QLORA_TIMER_KINDS) return QLORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(qlora::g_mu);
    const qlora_status st = qlora::drain();
    if (launches) *launches = qlora::g_count[kind];
    if (total_ms) *total_ms = qlora::g_ms[kind];
    if (reset) {
        for (int k = 0; k < QLORA_TIMER_KINDS; ++k) { qlora::g_count[k] = 0; qlora::g_ms[k] = 0.0; }
    }
    return st;
}

}  // extern "C"
