// timing.cu -- optional CUDA-event timing of the library's own launches.
#include <mutex>
#include <vector>

#include "hsa_internal.cuh"

namespace hsa {

namespace {
struct Rec {
    int kind;
    int nlaunch;
    cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free;
double g_ms[HSA_K_COUNT];
int64_t g_launches[HSA_K_COUNT];

cudaEvent_t get_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// fold finished records into the totals (caller holds the lock)
cudaError_t drain() {
    for (Rec &r : g_recs) {
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e != cudaSuccess) return e;
        float ms = 0.f;
        e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess) return e;
        g_ms[r.kind] += ms;
        g_launches[r.kind] += r.nlaunch;
        g_free.push_back(r.a);
        g_free.push_back(r.b);
    }
    g_recs.clear();
    return cudaSuccess;
}
}  // namespace

TimedLaunch::TimedLaunch(int kind, int nlaunch, cudaStream_t st) : kind_(kind), nlaunch_(nlaunch), st_(st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on || kind < 0 || kind >= HSA_K_COUNT) return;
    a_ = get_event();
    b_ = get_event();
    if (a_ && b_ && cudaEventRecord(a_, st_) == cudaSuccess) active_ = true;
}

TimedLaunch::~TimedLaunch() {
    if (!active_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (cudaEventRecord(b_, st_) == cudaSuccess) g_recs.push_back({kind_, nlaunch_, a_, b_});
}

namespace {
std::mutex g_attr_mu;
std::vector<std::pair<const void *, size_t>> g_attr;
}  // namespace

cudaError_t set_smem_once(const void *func, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    std::lock_guard<std::mutex> lk(g_attr_mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // key on (function, device) by folding the device into the size slot's high bits
    const size_t key = bytes | ((size_t)dev << 48);
    for (auto &p : g_attr)
        if (p.first == func && (p.second >> 48) == (size_t)dev && (p.second & ((1ull << 48) - 1)) >= bytes)
            return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) g_attr.push_back({func, key});
    return e;
}

}  // namespace hsa

extern "C" {

hsa_status_t hsa_timing_enable(int on) {
    using namespace hsa;
    std::lock_guard<std::mutex> lk(g_mu);
    if (on) {
        if (drain() != cudaSuccess) return HSA_ERR_CUDA;
        for (int i = 0; i < HSA_K_COUNT; ++i) { g_ms[i] = 0.0; g_launches[i] = 0; }
    }
    g_on = on != 0;
    return HSA_OK;
}

hsa_status_t hsa_timing_read(int kind, double *total_ms, int64_t *launches) {
    using namespace hsa;
    if (kind < 0 || kind >= HSA_K_COUNT || !total_ms || !launches) return HSA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    if (drain() != cudaSuccess) return HSA_ERR_CUDA;
    *total_ms = g_ms[kind];
    *launches = g_launches[kind];
    return HSA_OK;
}

}  // extern "C"
