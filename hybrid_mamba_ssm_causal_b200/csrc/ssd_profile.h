// ssd_profile.h -- launch accounting and optional per-kernel CUDA-event timing.
//
// Every kernel launch of the library goes through a LaunchScope. It always counts the
// launch; when profiling is switched on (ssd_mixer_profile_enable), it also records a
// CUDA event pair around the launch on the launching stream, so a caller can read
// each kernel's device time over a region without an external profiler.
#pragma once

#include <cuda_runtime.h>

namespace ssd {

void profile_begin(const char* name, cudaStream_t st, void** token, int launches);
void profile_end(void* token, cudaStream_t st);

// `launches`: the kernel launches the scope encloses (a series of launches that may overlap,
// such as the pieces of one prefill call, is timed as one span with no events between them).
struct LaunchScope {
    void* token = nullptr;
    cudaStream_t st;
    LaunchScope(const char* name, cudaStream_t s, int launches = 1) : st(s) { profile_begin(name, s, &token, launches); }
    ~LaunchScope() { profile_end(token, st); }
};

}  // namespace ssd
