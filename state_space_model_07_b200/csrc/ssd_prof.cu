// ssd_prof.cu -- per-kernel launch counters and CUDA-event durations.
#include <atomic>
#include <mutex>
#include <string.h>
#include <vector>

#include "ssd.h"
#include "ssd_prof.h"

namespace ssd {
namespace {

const char* const kNames[K_COUNT] = {
    "seq_bounds", "seq_table", "simt_chunk_state", "simt_state_pass", "simt_chunk_out",
    "state_update", "tc_prep", "tc_scan", "selftest_wait", "scan_bwd", "bwd_cast",
    "segment_logdecay", "state_chain", "state_out", "tile_logdecay", "group_norm", "quant_allreduce", "bwd_pass", "bwd_grads",
};

struct Pending {
    int id;
    cudaEvent_t e0, e1;
};

std::atomic<int> g_enabled{0};
std::atomic<long long> g_launches[K_COUNT];
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
long long g_timed[K_COUNT];
double g_ms[K_COUNT];

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

ProfScope::ProfScope(KernelId id, cudaStream_t st) : id_(id), st_(st) {
    g_launches[id].fetch_add(1, std::memory_order_relaxed);
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    e0_ = take_event();
    e1_ = take_event();
    if (e0_ && e1_) cudaEventRecord(e0_, st_);
}

ProfScope::~ProfScope() {
    if (!e0_ || !e1_) return;
    cudaEventRecord(e1_, st_);
    std::lock_guard<std::mutex> lk(g_mu);
    g_pending.push_back({(int)id_, e0_, e1_});
}

}  // namespace ssd

extern "C" {

int ssd_profile_enable(int on) { return ssd::g_enabled.exchange(on ? 1 : 0); }

int ssd_profile_read(ssd_kernel_stat* out, int max_entries, int reset) {
    using namespace ssd;
    std::lock_guard<std::mutex> lk(g_mu);
    int rc = 0;
    for (const Pending& p : g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.e1) != cudaSuccess ||
            cudaEventElapsedTime(&ms, p.e0, p.e1) != cudaSuccess) {
            rc = -SSD_ERR_CUDA;
        } else {
            g_timed[p.id] += 1;
            g_ms[p.id] += ms;
        }
        g_pool.push_back(p.e0);
        g_pool.push_back(p.e1);
    }
    g_pending.clear();
    if (rc) return rc;
    int n = 0;
    for (int k = 0; k < K_COUNT && n < max_entries; ++k) {
        long long l = g_launches[k].load();
        if (l == 0) continue;
        if (out) {
            memset(&out[n], 0, sizeof(out[n]));
            strncpy(out[n].name, kNames[k], sizeof(out[n].name) - 1);
            out[n].launches = l;
            out[n].timed = g_timed[k];
            out[n].total_ms = g_ms[k];
        }
        ++n;
    }
    if (reset) {
        for (int k = 0; k < K_COUNT; ++k) {
            g_launches[k].store(0);
            g_timed[k] = 0;
            g_ms[k] = 0.0;
        }
    }
    return n;
}

}  // extern "C"
