// zha_profile.cu -- launch counting and optional per-launch CUDA-event timing.
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "zha_common.cuh"

namespace zha {

namespace {

struct Rec {
    const char *name;
    cudaEvent_t a, b;
};

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_enabled{0};
std::mutex g_mu;
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

ProfScope::ProfScope(const char *name, cudaStream_t s) : slot(-1), st(s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Rec r{name, take_event(), take_event()};
    if (!r.a || !r.b) return;
    cudaEventRecord(r.a, st);
    g_recs.push_back(r);
    slot = (int)g_recs.size() - 1;
}

ProfScope::~ProfScope() {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (slot < (int)g_recs.size()) cudaEventRecord(g_recs[slot].b, st);
}

}  // namespace zha

extern "C" {

uint64_t zha_launch_count(void) { return zha::g_launches.load(); }

zha_status zha_profile_enable(int32_t on) {
    zha::g_enabled.store(on ? 1 : 0);
    return ZHA_OK;
}

int32_t zha_profile_read(char *names, int32_t names_len, double *ms, int64_t *launches,
                         int32_t max_kernels) {
    using namespace zha;
    std::lock_guard<std::mutex> lk(g_mu);
    std::map<std::string, std::pair<double, int64_t>> agg;
    std::vector<std::string> order;
    for (const Rec &r : g_recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            return -1;
        auto it = agg.find(r.name);
        if (it == agg.end()) {
            order.push_back(r.name);
            agg[r.name] = {t, 1};
        } else {
            it->second.first += t;
            it->second.second += 1;
        }
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_recs.clear();
    int n = 0;
    std::string all;
    for (const std::string &k : order) {
        if (n >= max_kernels) break;
        if (ms) ms[n] = agg[k].first;
        if (launches) launches[n] = agg[k].second;
        all += k;
        all += '\n';
        ++n;
    }
    if (names && names_len > 0) {
        size_t m = all.size() < (size_t)(names_len - 1) ? all.size() : (size_t)(names_len - 1);
        memcpy(names, all.data(), m);
        names[m] = 0;
    }
    return n;
}

}  // extern "C"
