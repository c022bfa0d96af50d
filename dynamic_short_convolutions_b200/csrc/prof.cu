// prof.cu -- per-kernel device timing with CUDA events recorded on the launch stream.
//
// When enabled, every kernel launch of the library is bracketed by two events
// on the stream it is launched on; dynconv_profile_read() waits for them and
// reports, per kernel, the number of launches and the summed device time.
// Disabled (the default), a launch costs one relaxed atomic load.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dynconv.h"
#include "prof.h"

namespace dynconv {
namespace {

struct Pending {
    int id;
    cudaEvent_t a, b;
};

std::atomic<int> g_enabled{0};
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
double g_ms[kKernelCount];
int64_t g_launches[kKernelCount];

const char* kNames[kKernelCount] = {
    "simt_gen", "simt_widen", "simt_conv_fwd", "simt_conv_bwd", "simt_dB", "simt_hTX", "simt_dh",
    "check_seqlens", "tc_gen", "tc_lowrank_fwd", "tc_lowrank_bwd", "tc_gen_bwd", "tc_reduce",
    "tc_headwise_fwd", "tc_headwise_bwd", "tc_prep", "decode_gen", "decode_conv", "simt_rope",
};

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

ProfScope::ProfScope(int id, cudaStream_t st) : id_(id), st_(st), a_(nullptr) {
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    a_ = take_event();
    if (a_ && cudaEventRecord(a_, st_) != cudaSuccess) {
        g_pool.push_back(a_);
        a_ = nullptr;
    }
}

ProfScope::~ProfScope() {
    if (!a_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEvent_t b = take_event();
    if (b && cudaEventRecord(b, st_) == cudaSuccess) {
        g_pending.push_back({id_, a_, b});
    } else {
        g_pool.push_back(a_);
        if (b) g_pool.push_back(b);
    }
}

const char* kernel_name(int id) { return (id >= 0 && id < kKernelCount) ? kNames[id] : "?"; }

}  // namespace dynconv

using namespace dynconv;

extern "C" {

int dynconv_profile_enable(int enable) { return g_enabled.exchange(enable ? 1 : 0); }

int dynconv_profile_read(dynconv_profile_entry* entries, int max_entries, int reset) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const Pending& p : g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
            g_ms[p.id] += ms;
            g_launches[p.id] += 1;
        }
        g_pool.push_back(p.a);
        g_pool.push_back(p.b);
    }
    g_pending.clear();
    int n = 0;
    for (int i = 0; i < kKernelCount; ++i) {
        if (g_launches[i] == 0) continue;
        if (entries && n < max_entries) {
            std::memset(entries[n].name, 0, sizeof(entries[n].name));
            std::strncpy(entries[n].name, kNames[i], sizeof(entries[n].name) - 1);
            entries[n].launches = g_launches[i];
            entries[n].total_ms = g_ms[i];
        }
        ++n;
    }
    if (reset) {
        std::memset(g_ms, 0, sizeof(g_ms));
        std::memset(g_launches, 0, sizeof(g_launches));
    }
    return n;
}

}  // extern "C"
