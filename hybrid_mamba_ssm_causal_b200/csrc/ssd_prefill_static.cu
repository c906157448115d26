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
// stand-in, so its device address is fetched with cudaGetSymbolAddress while the caller's
// context is current, on the first call in that context, and cached under the context's
// unique ID (cuCtxGetId never hands out an ID twice in a process, so a context created
// after cudaDeviceReset, or a caller's own non-primary context, gets its own entry).
// Every call in a context shares the array; the prefill clears the array's status word
// on its stream before its first kernel, and its kernels write every other scratch byte
// they read in the same call, so no other clearing is needed, but two calls whose work
// overlaps on the GPU (different streams, no ordering) race on it.
#include <cuda.h>

#include <mutex>

#include "../../include/ssd_mixer.h"
#include "ssd_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[SSD_MIXER_STATIC_WORKSPACE_BYTES];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct DriverFns {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

// The two driver calls, fetched once through the runtime (no link-time libcuda dependency).
const DriverFns& driver_fns()
{
    static DriverFns fns = []() {
        DriverFns f;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_id = reinterpret_cast<CtxGetIdFn>(p);
        return f;
    }();
    return fns;
}

constexpr int kMaxContexts = 256;
struct CacheEntry {
    unsigned long long ctx_id;
    void* ptr;
};
std::mutex g_mu;
CacheEntry g_cache[kMaxContexts];
int g_ncache = 0;

// ID of the context current on this thread; the runtime's primary context is made current
// first if none is.
cudaError_t current_context_id(unsigned long long* id)
{
    const DriverFns& f = driver_fns();
    if (!f.get_current || !f.get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    if (!ctx) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaSetDevice(dev);   // initialises and binds the primary context
        if (e != cudaSuccess) return e;
        if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    }
    return f.get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of g_static_workspace in the current context (looked up once per context).
cudaError_t static_workspace(void** out)
{
    unsigned long long id = 0;
    cudaError_t e = current_context_id(&id);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < g_ncache; ++i) {
        if (g_cache[i].ctx_id == id) {
            *out = g_cache[i].ptr;
            return cudaSuccess;
        }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    if (g_ncache < kMaxContexts) g_cache[g_ncache++] = CacheEntry{id, p};   // else: looked up each call
    *out = p;
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

extern "C" ssd_status ssd_mixer_prefill_static_status(void* stream)
{
    void* ws = nullptr;
    if (static_workspace(&ws) != cudaSuccess) return SSD_ERR_CUDA;
    return ssd_mixer_workspace_status(ws, stream);
}
