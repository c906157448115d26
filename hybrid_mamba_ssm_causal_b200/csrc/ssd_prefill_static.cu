// ssd_prefill_static.cu -- ssd_mixer_prefill_static: the prefill with its scratch in a
// fixed device array, for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: a plugin slot in a host
// framework that passes only tensors and a stream, or a serving process whose device
// memory is entirely reserved up front by its own pool, where an extra cudaMalloc would
// fail or would stall every stream in the middle of the serving loop. This entry point
// takes the same arguments as ssd_mixer_prefill minus the workspace and uses a
// file-scope device array of SSD_MIXER_STATIC_WORKSPACE_BYTES instead.
//
// The array is a __device__ variable: in host code its name is only a host-side
// stand-in, so the device address is fetched once per device with cudaGetSymbolAddress
// (on the first call on that device, with that device current) and cached. Every call
// on a device shares the array; the prefill kernels write every scratch byte they read
// in the same call and reset the status word themselves, so no clearing is needed, but
// two calls whose work overlaps on the GPU (different streams, no ordering) race on it.
#include <mutex>

#include "../../include/ssd_mixer.h"
#include "ssd_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[SSD_MIXER_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device (looked up once per device).
cudaError_t static_workspace(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ws_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess) return e;
        g_ws_ptr[dev] = p;
    }
    *out = g_ws_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ssd_status ssd_mixer_prefill_static(
    const ssd_dims* d, const void* x, int64_t x_ld, const void* z, int64_t z_ld, const void* B,
    int64_t B_ld, const void* C, int64_t C_ld, const void* dt, int64_t dt_ld, const float* A,
    const float* D, const float* conv_w, const float* conv_b, const float* dt_bias,
    const float* norm_w, const float* init_ssm_state, const void* init_conv_state, void* y,
    int64_t y_ld, float* final_ssm_state, void* final_conv_state, void* stream)
{
    const size_t need = ssd_mixer_prefill_workspace_size(d);
    if (need == 0) {
        // invalid or unsupported dims: let the regular entry point name the error
        return ssd_mixer_prefill(d, x, x_ld, z, z_ld, B, B_ld, C, C_ld, dt, dt_ld, A, D, conv_w,
                                 conv_b, dt_bias, norm_w, init_ssm_state, init_conv_state, y, y_ld,
                                 final_ssm_state, final_conv_state, nullptr, 0, stream);
    }
    if (need > (size_t)SSD_MIXER_STATIC_WORKSPACE_BYTES) return SSD_ERR_TOO_LARGE;
    void* ws = nullptr;
    if (static_workspace(&ws) != cudaSuccess) return SSD_ERR_CUDA;
    return ssd_mixer_prefill(d, x, x_ld, z, z_ld, B, B_ld, C, C_ld, dt, dt_ld, A, D, conv_w, conv_b,
                             dt_bias, norm_w, init_ssm_state, init_conv_state, y, y_ld,
                             final_ssm_state, final_conv_state, ws,
                             (size_t)SSD_MIXER_STATIC_WORKSPACE_BYTES, stream);
}
