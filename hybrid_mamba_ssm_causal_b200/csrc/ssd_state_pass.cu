// ssd_state_pass.cu -- state passing between the pieces of a sequence split across devices.
//
// A prefill's final state is linear in its initial state: the state after a piece equals its
// decay exp(A * sum(delta)) times the state before it plus the piece's own final state from a
// zero start. So the state entering piece r follows from the pieces before it:
//   H_in(0) = H0,  H_in(j+1) = a_j * H_in(j) + S_j
// (the state passing across a split sequence that the Modalities PR #459 tests, section
// "Testing", and that its long-context next step needs, section "Next steps for production at
// scale"). Memory-bound: each state element is read once per earlier piece and written once.
#include "ssd_internal.h"
#include "ssd_profile.h"

namespace ssd {
namespace {

__global__ void __launch_bounds__(256) state_pass_kernel(int64_t n4, int64_t per_head4, int64_t bh, int r,
                                                         const float* __restrict__ decay,
                                                         const float4* __restrict__ state,
                                                         const float4* __restrict__ init, float4* __restrict__ out)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const int64_t head = i / per_head4;   // (row, head) index
    float4 h = init ? init[i] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int j = 0; j < r; ++j) {
        const float a = decay[j * bh + head];
        const float4 s = state[j * n4 + i];
        h = make_float4(fmaf(a, h.x, s.x), fmaf(a, h.y, s.y), fmaf(a, h.z, s.z), fmaf(a, h.w, s.w));
    }
    out[i] = h;
}

}  // namespace

cudaError_t launch_state_pass(int64_t b, int H, int P, int N, int r, const float* decay, const float* state,
                              const float* init, float* out, cudaStream_t st)
{
    const int64_t n4 = b * H * (int64_t)P * N / 4;
    if (n4 == 0) return cudaSuccess;
    LaunchScope ls("state_pass", st);
    state_pass_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(
        n4, (int64_t)P * N / 4, b * H, r, decay, reinterpret_cast<const float4*>(state),
        reinterpret_cast<const float4*>(init), reinterpret_cast<float4*>(out));
    return cudaGetLastError();
}

}  // namespace ssd
