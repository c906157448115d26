// ssd_profile.cu -- launch counter and opt-in per-kernel event timing (see ssd_profile.h).
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/ssd_mixer.h"
#include "ssd_profile.h"

namespace ssd {
namespace {

struct Rec {
    const char* name;
    cudaEvent_t a, b;
    int launches;
};

std::atomic<long long> g_launches{0};
std::atomic<int> g_enabled{0};
std::mutex g_mu;
std::vector<Rec> g_recs;

}  // namespace

void profile_begin(const char* name, cudaStream_t st, void** token, int launches)
{
    g_launches.fetch_add(launches, std::memory_order_relaxed);
    *token = nullptr;
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    Rec* r = new Rec{name, nullptr, nullptr, launches};
    if (cudaEventCreate(&r->a) != cudaSuccess) {
        delete r;
        return;
    }
    if (cudaEventCreate(&r->b) != cudaSuccess || cudaEventRecord(r->a, st) != cudaSuccess) {
        cudaEventDestroy(r->a);
        if (r->b) cudaEventDestroy(r->b);
        delete r;
        return;
    }
    *token = r;
}

void profile_end(void* token, cudaStream_t st)
{
    if (!token) return;
    Rec* r = (Rec*)token;
    cudaEventRecord(r->b, st);
    std::lock_guard<std::mutex> lk(g_mu);
    g_recs.push_back(*r);
    delete r;
}

}  // namespace ssd

extern "C" {

long long ssd_mixer_launch_count(void) { return ssd::g_launches.load(); }

void ssd_mixer_profile_enable(int on) { ssd::g_enabled.store(on ? 1 : 0); }

int ssd_mixer_profile_read(const char** names, double* total_ms, int* launches, int max_entries)
{
    std::vector<ssd::Rec> recs;
    {
        std::lock_guard<std::mutex> lk(ssd::g_mu);
        recs.swap(ssd::g_recs);
    }
    int n = 0;
    for (const ssd::Rec& r : recs) {
        float ms = 0.0f;
        const bool timed =
            cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
        int k = 0;
        while (k < n && strcmp(names[k], r.name) != 0) ++k;
        if (k == n) {
            if (n >= max_entries) continue;
            names[n] = r.name;
            total_ms[n] = 0.0;
            launches[n] = 0;
            ++n;
        }
        if (timed) total_ms[k] += ms;   // a pair that could not be timed still counts as a launch
        launches[k] += r.launches;
    }
    return n;
}

}  // extern "C"
