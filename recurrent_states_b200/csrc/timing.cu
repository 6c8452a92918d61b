// Opt-in kernel timing for benchmarks.  When enabled on a host thread, each
// kernel this library launches from that thread is bracketed by two CUDA
// events recorded on the launch stream; taylor_attn_timing_read() waits for
// them and returns per-kernel launch counts and total device milliseconds.
// Disabled (the default) it costs one thread-local branch per launch.
#include <string.h>

#include <string>
#include <vector>

#include "../../include/taylor_attn.h"
#include "internal.h"

namespace ta {
namespace timing {

namespace {

struct Rec {
    const char* name;
    cudaEvent_t start, stop;
};

thread_local bool g_on = false;
thread_local std::vector<Rec> g_recs;
// Events are created once and reused, so that enabling the timing adds only
// two event records per launch to the host's enqueue path.
thread_local std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

}  // namespace

bool enabled() { return g_on; }

// Every begin() pushes one record, so that end() always closes the record of
// its own launch; a launch whose events could not be had keeps a record with
// null events, which end() and taylor_attn_timing_read() skip.
void begin(cudaStream_t s, const char* name) {
    if (!g_on) return;
    Rec r{name, take_event(), take_event()};
    if (!r.start || !r.stop) {
        if (r.start) g_pool.push_back(r.start);
        if (r.stop) g_pool.push_back(r.stop);
        r.start = r.stop = nullptr;
    } else {
        cudaEventRecord(r.start, s);
    }
    g_recs.push_back(r);
}

void end(cudaStream_t s) {
    if (!g_on || g_recs.empty() || !g_recs.back().stop) return;
    cudaEventRecord(g_recs.back().stop, s);
}

}  // namespace timing
}  // namespace ta

extern "C" {

int taylor_attn_timing_enable(int on) {
    ta::timing::g_on = on != 0;
    // pre-create a pool so the first timed launches do not pay for creation
    while (on && ta::timing::g_pool.size() < 256) {
        cudaEvent_t e = nullptr;
        if (cudaEventCreate(&e) != cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_CUDA;
        }
        ta::timing::g_pool.push_back(e);
    }
    return TAYLOR_OK;
}

int taylor_attn_timing_read(int max_kernels, char* names, int* launches, float* total_ms) {
    using ta::timing::g_recs;
    if (max_kernels < 0 || (max_kernels > 0 && (!names || !launches || !total_ms)))
        return TAYLOR_ERR_INVALID_ARG;
    std::vector<std::string> keys;
    std::vector<int> cnt;
    std::vector<double> ms;
    int rc = TAYLOR_OK;
    for (auto& r : g_recs) {
        if (!r.start || !r.stop) {  // no events could be had for this launch
            rc = TAYLOR_ERR_CUDA;
            continue;
        }
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
            cudaGetLastError();
            rc = TAYLOR_ERR_CUDA;
        }
        size_t i = 0;
        while (i < keys.size() && keys[i] != r.name) ++i;
        if (i == keys.size()) {
            keys.push_back(r.name);
            cnt.push_back(0);
            ms.push_back(0.0);
        }
        cnt[i] += 1;
        ms[i] += t;
        ta::timing::g_pool.push_back(r.start);
        ta::timing::g_pool.push_back(r.stop);
    }
    g_recs.clear();
    if (rc != TAYLOR_OK) return rc;
    const int n = (int)keys.size() < max_kernels ? (int)keys.size() : max_kernels;
    for (int i = 0; i < n; ++i) {
        strncpy(names + 64 * i, keys[i].c_str(), 63);
        names[64 * i + 63] = 0;
        launches[i] = cnt[i];
        total_ms[i] = (float)ms[i];
    }
    return (int)keys.size();
}

}  // extern "C"
