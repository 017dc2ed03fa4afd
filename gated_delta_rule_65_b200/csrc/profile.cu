// profile.cu -- opt-in per-kernel timing with CUDA events on the launching stream.
//
// When enabled (gdr2_profile_enable(1)), every kernel launch made through GDR2_LAUNCH is bracketed by
// two CUDA events recorded on the launch stream. gdr2_profile_collect() waits for those events and
// returns, per kernel name, the number of launches and their summed device time. Events come from a
// fixed pool created on first use; launches beyond the pool are counted as dropped, never blocked.
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "gdr2.h"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int kPool = 8192;

struct Rec {
    const char *name;
    int slot;
};

std::mutex g_mu;
bool g_on = false;
std::vector<cudaEvent_t> g_ev;  // 2 * kPool events
std::vector<Rec> g_recs;
int g_dropped = 0;

}  // namespace

int prof_begin(const char *name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on) return -1;
    if (g_ev.empty()) {
        g_ev.resize(2 * kPool);
        for (auto &e : g_ev)
            if (cudaEventCreate(&e) != cudaSuccess) { g_ev.clear(); g_on = false; return -1; }
    }
    if ((int)g_recs.size() >= kPool) { ++g_dropped; return -1; }
    const int slot = (int)g_recs.size();
    g_recs.push_back(Rec{name, slot});
    cudaEventRecord(g_ev[2 * slot], st);
    return slot;
}

void prof_end(int slot, cudaStream_t st) {
    if (slot < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEventRecord(g_ev[2 * slot + 1], st);
}

}  // namespace gdr2

extern "C" {

GDR2_API int gdr2_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(gdr2::g_mu);
    gdr2::g_on = on != 0;
    return GDR2_OK;
}

GDR2_API int gdr2_profile_collect(char *names, int name_stride, int *launches, double *ms, int max_entries,
                                  int *dropped) {
    std::lock_guard<std::mutex> lk(gdr2::g_mu);
    if (max_entries < 0 || (max_entries > 0 && (!names || !launches || !ms || name_stride < 2)))
        return -GDR2_ERR_INVALID_ARG;
    int n = 0;
    for (const auto &r : gdr2::g_recs) {
        float t = 0.f;
        if (cudaEventSynchronize(gdr2::g_ev[2 * r.slot + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&t, gdr2::g_ev[2 * r.slot], gdr2::g_ev[2 * r.slot + 1]) != cudaSuccess)
            return -GDR2_ERR_CUDA;
        int i = 0;
        for (; i < n; ++i)
            if (strncmp(names + (size_t)i * name_stride, r.name, name_stride - 1) == 0) break;
        if (i == n) {
            if (n >= max_entries) continue;
            snprintf(names + (size_t)n * name_stride, name_stride, "%s", r.name);
            launches[n] = 0;
            ms[n] = 0.0;
            ++n;
        }
        launches[i] += 1;
        ms[i] += t;
    }
    if (dropped) *dropped = gdr2::g_dropped;
    gdr2::g_recs.clear();
    gdr2::g_dropped = 0;
    return n;
}

}  // extern "C"
