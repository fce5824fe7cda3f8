// Launch accounting and optional per-kernel timing for libcsa.
//
// Every kernel launch site holds a LaunchScope.  The scope always bumps a process-wide
// launch counter; when timing is enabled it also records a CUDA event pair around the
// launch on the launching stream.  csa_profile_collect() waits for the recorded events
// and returns, per kernel, the number of timed launches and their total device time.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "launchers.cuh"

namespace csa {

namespace {
std::atomic<long long> g_launches{0};
std::atomic<int> g_timing{0};
std::mutex g_mu;
struct Pending {
    int kernel;
    cudaEvent_t start, stop;
};
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
long long g_count[kKernelKinds];
double g_ms[kKernelKinds];

// Inside a stream capture an event record only orders work within the graph unless it is
// recorded as an external node, which timestamps on every replay.
void record(cudaEvent_t ev, cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, stream);
}

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

const char* kernel_name(int kind) {
    static const char* names[kKernelKinds] = {"compress", "topk_radix",
                                              "attn_simt", "indexer_score_tc", "attn_tc",
                                              "attn_combine", "attn576_tc", "topk_merge",
                                              "cp_candidates", "cp_pack_rows",
                                              "indexer_score_fp4", "cache_append"};
    return (kind >= 0 && kind < kKernelKinds) ? names[kind] : "?";
}

LaunchScope::LaunchScope(int kind, cudaStream_t stream) : kind_(kind), stream_(stream) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_timing.load(std::memory_order_relaxed)) {
        std::lock_guard<std::mutex> lk(g_mu);
        start_ = take_event();
        stop_ = take_event();
        if (start_ && stop_) record(start_, stream_);
    }
}

LaunchScope::~LaunchScope() {
    if (start_ && stop_) {
        record(stop_, stream_);
        std::lock_guard<std::mutex> lk(g_mu);
        g_pending.push_back({kind_, start_, stop_});
    }
}

}  // namespace csa

extern "C" {

long long csa_launch_count(void) { return csa::g_launches.load(); }

void csa_profile_enable(int on) { csa::g_timing.store(on ? 1 : 0); }

int csa_profile_collect(csa_kernel_time_t* out, int max_entries, int keep_pending) {
    std::lock_guard<std::mutex> lk(csa::g_mu);
    for (const auto& p : csa::g_pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.stop) == cudaSuccess &&
            cudaEventElapsedTime(&ms, p.start, p.stop) == cudaSuccess) {
            csa::g_count[p.kernel] += 1;
            csa::g_ms[p.kernel] += ms;
        }
        if (!keep_pending) {
            csa::g_pool.push_back(p.start);
            csa::g_pool.push_back(p.stop);
        }
    }
    if (!keep_pending) csa::g_pending.clear();
    int n = 0;
    for (int k = 0; k < csa::kKernelKinds && n < max_entries; k++) {
        if (csa::g_count[k] == 0) continue;
        std::memset(&out[n], 0, sizeof(out[n]));
        std::strncpy(out[n].name, csa::kernel_name(k), sizeof(out[n].name) - 1);
        out[n].launches = csa::g_count[k];
        out[n].total_ms = csa::g_ms[k];
        n++;
    }
    for (int k = 0; k < csa::kKernelKinds; k++) {
        csa::g_count[k] = 0;
        csa::g_ms[k] = 0.0;
    }
    return n;
}

}  // extern "C"
