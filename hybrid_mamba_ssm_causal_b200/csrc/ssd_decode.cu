// ssd_decode.cu -- single-token decode step of the SSD mixer, in place on state slots.
//
// One token per sequence, continuing from the state in the sequence's slot (the
// one-token-at-a-time decode of gllm PR #86, section "Validation"). The step is
// memory-bound: the fp32 SSM state [H][P][N] of every stepped sequence is read once and
// written once, which is almost all of the bytes. One CTA owns one (sequence, group): the group's x
// channels (r = H/G heads), its B and C channels and its norm group, so the conv state
// of every channel is updated by exactly one thread and the gated RMSNorm needs no
// cross-CTA exchange.
//
// Per CTA:
//   1. conv: for each owned channel, v = conv_b + w0 s0 + w1 s1 + w2 s2 + w3 u, x' = SiLU(v),
//      and the conv state shifts to [s1, s2, u] (same thread reads, then writes).
//   2. delta = softplus(dt + dt_bias) for the group's heads.
//   3. state rows (h, p): N/4 lanes each hold one float4 of the row;
//        h[p][:] = exp(delta A) h[p][:] + delta x'[p] B'[:];  y[p] = h[p][:] . C'[:] + D x'[p]
//      each lane group loads two rows before using either; 16 warps per CTA and three CTAs
//      per SM keep the rest of the bytes in flight.
//   4. gated RMSNorm over the group's r*P channels; y written in the activation dtype.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"

namespace ssd {
namespace {

// 512 threads and two state rows in flight per lane group keep the kernel at about 40
// registers, three CTAs per SM. Measured on decode_bf16 (B200): 389 us per step, against
// 418 us with 256 threads (six CTAs per SM), 492 us with 128, and 445 / 526 / 477 us with
// 256 threads and four / eight / one rows in flight.
constexpr int kThreads = 512;
constexpr int kRowsInFlight = 2;

template <typename T, int N>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(DecodeParams p)
{
    constexpr int LPR = N / 4;             // lanes per state row (one float4 each)
    constexpr int RPW = 32 / LPR;          // rows per warp per pass
    constexpr int kWarps = kThreads / 32;
    extern __shared__ __align__(16) float sm[];

    const int g = blockIdx.x;
    const int64_t i = blockIdx.y;
    const int64_t slot = p.slot_idx ? (int64_t)p.slot_idx[i] : i;
    const int r = p.H / p.G, P = p.P;
    const int gw = r * P;                          // channels of the group's heads
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    float* xa = sm;                                // [gw]
    float* ba = xa + gw;                           // [N]
    float* ca = ba + N;                            // [N]
    float* yb = ca + N;                            // [gw]
    float* dl = yb + gw;                           // [r]
    float* red = dl + r;                           // [kWarps]

    // 1. conv over the owned channels, conv state updated in place
    const int nch = gw + 2 * N;
    for (int k = threadIdx.x; k < nch; k += kThreads) {
        int64_t ch;
        float u;
        if (k < gw) {
            ch = (int64_t)g * gw + k;
            u = ld_f<T>((const T*)p.x + i * p.x_ld + ch);
        } else if (k < gw + N) {
            ch = HP + (int64_t)g * N + (k - gw);
            u = ld_f<T>((const T*)p.B + i * p.B_ld + (int64_t)g * N + (k - gw));
        } else {
            ch = HP + GN + (int64_t)g * N + (k - gw - N);
            u = ld_f<T>((const T*)p.C + i * p.C_ld + (int64_t)g * N + (k - gw - N));
        }
        T* st = (T*)p.conv_state + (slot * Cc + ch) * 3;
        const float s0 = ld_f<T>(st), s1 = ld_f<T>(st + 1), s2 = ld_f<T>(st + 2);
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        const float v = p.conv_b[ch] + w.x * s0 + w.y * s1 + w.z * s2 + w.w * u;
        st[0] = st[1];
        st[1] = st[2];
        st[2] = Act<T>::from_f(u);
        const float a = silu(v);
        if (k < gw) xa[k] = a;
        else if (k < gw + N) ba[k - gw] = a;
        else ca[k - gw - N] = a;
    }
    for (int k = threadIdx.x; k < r; k += kThreads) {
        const int h = g * r + k;
        dl[k] = softplus(ld_f<T>((const T*)p.dt + i * p.dt_ld + h) + p.dt_bias[h]);
    }
    __syncthreads();

    // 3. stream the group's state rows
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, ln = lane % LPR;   // row within the warp's pass, float4 index
    const float4 bv = *reinterpret_cast<const float4*>(ba + 4 * ln);
    const float4 cv = *reinterpret_cast<const float4*>(ca + 4 * ln);
    float* state = p.ssm_state + (slot * p.H + (int64_t)g * r) * (int64_t)P * N;
    const int rows_per_pass = kWarps * RPW;
    for (int base = 0; base < gw; base += rows_per_pass * kRowsInFlight) {
        float4 hv[kRowsInFlight];
        int row[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            row[u] = base + (u * kWarps + warp) * RPW + sub;
            if (row[u] < gw) hv[u] = *reinterpret_cast<const float4*>(state + (int64_t)row[u] * N + 4 * ln);
        }
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            float part = 0.0f;
            if (row[u] < gw) {
                const int hh = row[u] / P;
                const float d = dl[hh];
                const float a = expf(d * p.A[g * r + hh]);
                const float dx = d * xa[row[u]];
                float4 h4 = hv[u];
                h4.x = a * h4.x + dx * bv.x;
                h4.y = a * h4.y + dx * bv.y;
                h4.z = a * h4.z + dx * bv.z;
                h4.w = a * h4.w + dx * bv.w;
                *reinterpret_cast<float4*>(state + (int64_t)row[u] * N + 4 * ln) = h4;
                part = h4.x * cv.x + h4.y * cv.y + h4.z * cv.z + h4.w * cv.w;
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (ln == 0 && row[u] < gw) {
                const int hh = row[u] / P;
                yb[row[u]] = part + p.D[g * r + hh] * xa[row[u]];
            }
        }
    }
    __syncthreads();

    // 4. gated RMSNorm over the group
    const T* z = (const T*)p.z + i * p.z_ld + (int64_t)g * gw;
    float ss = 0.0f;
    for (int k = threadIdx.x; k < gw; k += kThreads) {
        const float gt = yb[k] * silu(ld_f<T>(z + k));
        yb[k] = gt;
        ss += gt * gt;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += red[w];
    const float inv = rsqrtf(tot / (float)gw + p.eps);
    T* y = (T*)p.y + i * p.y_ld + (int64_t)g * gw;
    for (int k = threadIdx.x; k < gw; k += kThreads)
        y[k] = Act<T>::from_f(yb[k] * inv * p.norm_w[(int64_t)g * gw + k]);
}

template <typename T>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t st)
{
    const int r = p.H / p.G;
    const size_t smem = sizeof(float) * (size_t)(2 * r * p.P + 2 * p.N + r + kThreads / 32);
    const dim3 grid((unsigned)p.G, (unsigned)p.b);
#define SSD_DEC_CASE(NN)                                                                          \
    if (p.N == NN) {                                                                              \
        cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<T, NN>,                           \
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                           \
        LaunchScope ls("decode_step", st);                                                        \
        decode_step_kernel<T, NN><<<grid, kThreads, smem, st>>>(p);                               \
        return cudaGetLastError();                                                                \
    }
    SSD_DEC_CASE(16) SSD_DEC_CASE(32) SSD_DEC_CASE(64) SSD_DEC_CASE(128)
#undef SSD_DEC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

bool decode_supported(int P, int N)
{
    return (P % 4 == 0) && (N == 16 || N == 32 || N == 64 || N == 128);
}

cudaError_t launch_decode_step(const DecodeParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    if (p.act == 1) return launch_t<__nv_bfloat16>(p, stream);
    return launch_t<float>(p, stream);
}

}  // namespace ssd
