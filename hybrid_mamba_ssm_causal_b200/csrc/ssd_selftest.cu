// ssd_selftest.cu -- the bounded-wait path of the library's kernels, exercised on its own.
//
// Every spin in the tensor-core kernels (an mbarrier wait on a TMA load, a peer's copy or a
// tensor-core commit) gives up after a limit of clock cycles, sets the status word at the
// start of the caller's workspace and stops waiting; ssd_mixer_workspace_status then reports
// SSD_ERR_TIMEOUT. Forcing that inside the prefill kernel on purpose is not safe (a CTA that
// stops waiting may leave while copies still target its shared memory), so this entry point
// runs the same wait helper alone: one thread waits on an mbarrier that nothing arrives on
// (or, with `arrive`, on one it has already arrived on), with a limit the caller sets.
#include "../../include/ssd_mixer.h"
#include "ssd_internal.h"
#include "ssd_profile.h"
#include "ssd_tc_util.cuh"

namespace ssd {
namespace {

using namespace tc;

__global__ void selftest_wait_kernel(int* status, long long limit, int arrive)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    if (arrive) mbar_arrive_local(b);
    if (!mbar_wait_bounded(b, 0, limit)) set_device_status(status, kDevTimeout);
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_mixer_selftest_wait(void* workspace, long long limit_cycles, int arrive, void* stream)
{
    if (!workspace || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (limit_cycles < 0 || limit_cycles > 4000000000LL) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (ssd::clear_device_status((int*)workspace, st) != cudaSuccess) return SSD_ERR_CUDA;
    ssd::LaunchScope ls("selftest_wait", st);
    ssd::selftest_wait_kernel<<<1, 32, 0, st>>>((int*)workspace, limit_cycles, arrive ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
