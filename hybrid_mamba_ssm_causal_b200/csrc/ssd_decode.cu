// ssd_decode.cu -- single-token decode step of the SSD mixer, in place on state slots.
//
// One token per sequence, continuing from the state in the sequence's slot (the
// one-token-at-a-time decode of gllm PR #86, section "Validation"). The step is
// memory-bound: the fp32 SSM state [H][P][N] of every stepped sequence is read once and
// written once, which is almost all of the bytes. One CTA owns one (sequence, group), or, when
// so few sequences step that most SMs would idle, a cluster of S CTAs owns it and each CTA
// takes r/S of the group's r heads. The CTAs of a cluster exchange their partial sums of
// squares of the gated norm through distributed shared memory; every conv state channel is
// still shifted by exactly one thread.
//
// Per CTA:
//   1. conv: for each of its x channels and for the group's B and C channels,
//      v = conv_b + w0 s0 + w1 s1 + w2 s2 + w3 u, x' = SiLU(v); the conv state shifts to
//      [s1, s2, u] (same thread reads, then writes). In a cluster every CTA computes B', C' and
//      rank 0 shifts their state after a cluster barrier, once every CTA has read it.
//   2. delta = softplus(dt + dt_bias) for its heads.
//   3. state rows (h, p): N/4 lanes each hold one float4 of the row;
//        h[p][:] = exp(delta A) h[p][:] + delta x'[p] B'[:];  y[p] = h[p][:] . C'[:] + D x'[p]
//      each lane group loads two rows before using either; 16 warps per CTA and three CTAs
//      per SM keep the rest of the bytes in flight.
//   4. gated RMSNorm over the group's r*P channels; y written in the activation dtype.
#include <cooperative_groups.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"

namespace cg = cooperative_groups;

namespace ssd {
namespace {

// 512 threads and two state rows in flight per lane group keep the kernel at about 40
// registers, three CTAs per SM. Measured on decode_bf16 (B200): 389 us per step, against
// 418 us with 256 threads (six CTAs per SM), 492 us with 128, and 445 / 526 / 477 us with
// 256 threads and four / eight / one rows in flight.
// A cluster CTA has few rows (r/S heads), so it keeps eight in flight per lane group: its rows
// then take two rounds of loads instead of eight.
constexpr int kThreads = 512;
constexpr int kMaxCluster = 8;

// S = CTAs per (sequence, group): 1, or the cluster that splits the group's heads. RIF = state
// rows in flight per lane group.
template <typename T, int N, int RIF>
__global__ void __launch_bounds__(kThreads) decode_step_kernel(DecodeParams p, int S)
{
    constexpr int LPR = N / 4;             // lanes per state row (one float4 each)
    constexpr int RPW = 32 / LPR;          // rows per warp per pass
    constexpr int kWarps = kThreads / 32;
    extern __shared__ __align__(16) float sm[];
    cg::cluster_group cluster = cg::this_cluster();

    const int q = S > 1 ? (int)cluster.block_rank() : 0;
    const int g = blockIdx.x / S;
    const int64_t i = blockIdx.y;
    const int64_t slot = p.slot_idx ? (int64_t)p.slot_idx[i] : i;
    const int r = p.H / p.G, ro = r / S, P = p.P;
    const int gw = r * P;                          // channels of the norm group
    const int gwo = ro * P;                        // this CTA's channels: heads h0 .. h0+ro-1
    const int h0 = g * r + q * ro;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    float* xa = sm;                                // [gwo]
    float* ba = xa + gwo;                          // [N]
    float* ca = ba + N;                            // [N]
    float* yb = ca + N;                            // [gwo]
    float* dl = yb + gwo;                          // [ro]
    float* red = dl + ro;                          // [kWarps]
    float* cred = red + kWarps;                    // [kMaxCluster] partial sums of the cluster

    // 1. conv over this CTA's x channels and the group's B, C channels
    const int nch = gwo + 2 * N;
    for (int k = threadIdx.x; k < nch; k += kThreads) {
        int64_t ch;
        float u;
        if (k < gwo) {
            ch = (int64_t)h0 * P + k;
            u = ld_f<T>((const T*)p.x + i * p.x_ld + ch);
        } else if (k < gwo + N) {
            ch = HP + (int64_t)g * N + (k - gwo);
            u = ld_f<T>((const T*)p.B + i * p.B_ld + (int64_t)g * N + (k - gwo));
        } else {
            ch = HP + GN + (int64_t)g * N + (k - gwo - N);
            u = ld_f<T>((const T*)p.C + i * p.C_ld + (int64_t)g * N + (k - gwo - N));
        }
        T* st = (T*)p.conv_state + (slot * Cc + ch) * 3;
        const float s0 = ld_f<T>(st), s1 = ld_f<T>(st + 1), s2 = ld_f<T>(st + 2);
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        const float v = p.conv_b[ch] + w.x * s0 + w.y * s1 + w.z * s2 + w.w * u;
        if (k < gwo || S == 1) {
            st[0] = st[1];
            st[1] = st[2];
            st[2] = Act<T>::from_f(u);
        }
        const float a = silu(v);
        if (k < gwo) xa[k] = a;
        else if (k < gwo + N) ba[k - gwo] = a;
        else ca[k - gwo - N] = a;
    }
    for (int k = threadIdx.x; k < ro; k += kThreads) {
        const int h = h0 + k;
        dl[k] = softplus(ld_f<T>((const T*)p.dt + i * p.dt_ld + h) + p.dt_bias[h]);
    }
    if (S > 1) {
        cluster.sync();   // every CTA of the cluster has read the B/C conv state
        if (q == 0) {
            for (int k = threadIdx.x; k < 2 * N; k += kThreads) {
                const bool isC = k >= N;
                const int64_t ch = HP + (isC ? GN : 0) + (int64_t)g * N + (k % N);
                const T* src = (const T*)(isC ? p.C : p.B) + i * (isC ? p.C_ld : p.B_ld) + (int64_t)g * N + (k % N);
                T* st = (T*)p.conv_state + (slot * Cc + ch) * 3;
                st[0] = st[1];
                st[1] = st[2];
                st[2] = *src;
            }
        }
    } else {
        __syncthreads();
    }

    // 3. stream this CTA's state rows
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / LPR, ln = lane % LPR;   // row within the warp's pass, float4 index
    const float4 bv = *reinterpret_cast<const float4*>(ba + 4 * ln);
    const float4 cv = *reinterpret_cast<const float4*>(ca + 4 * ln);
    float* state = p.ssm_state + (slot * p.H + (int64_t)h0) * (int64_t)P * N;
    const int rows_per_pass = kWarps * RPW;
    for (int base = 0; base < gwo; base += rows_per_pass * RIF) {
        float4 hv[RIF];
        int row[RIF];
#pragma unroll
        for (int u = 0; u < RIF; ++u) {
            row[u] = base + (u * kWarps + warp) * RPW + sub;
            if (row[u] < gwo) hv[u] = *reinterpret_cast<const float4*>(state + (int64_t)row[u] * N + 4 * ln);
        }
#pragma unroll
        for (int u = 0; u < RIF; ++u) {
            float part = 0.0f;
            if (row[u] < gwo) {
                const int hh = row[u] / P;
                const float d = dl[hh];
                const float a = expf(d * p.A[h0 + hh]);
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
            if (ln == 0 && row[u] < gwo) {
                const int hh = row[u] / P;
                yb[row[u]] = part + p.D[h0 + hh] * xa[row[u]];
            }
        }
    }
    __syncthreads();

    // 4. gated RMSNorm over the group: this CTA's channels, the sums of squares of all of them
    const T* z = (const T*)p.z + i * p.z_ld + (int64_t)h0 * P;
    float ss = 0.0f;
    for (int k = threadIdx.x; k < gwo; k += kThreads) {
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
    if (S > 1) {
        // this CTA's partial into slot q of every CTA of the cluster, then the cluster's total
        if (threadIdx.x < (unsigned)S) cluster.map_shared_rank(cred, (unsigned)threadIdx.x)[q] = tot;
        cluster.sync();
        tot = 0.0f;
        for (int j = 0; j < S; ++j) tot += cred[j];
    }
    const float inv = rsqrtf(tot / (float)gw + p.eps);
    T* y = (T*)p.y + i * p.y_ld + (int64_t)h0 * P;
    for (int k = threadIdx.x; k < gwo; k += kThreads)
        y[k] = Act<T>::from_f(yb[k] * inv * p.norm_w[(int64_t)h0 * P + k]);
}

// CTAs per (sequence, group): the largest cluster of 2, 4 or 8 that divides the group's heads
// while the grid stays within two CTAs per SM; 1 when the sequences alone fill the GPU.
int decode_cluster(const DecodeParams& p)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;
    const int r = p.H / p.G;
    for (int c = kMaxCluster; c >= 2; c /= 2)
        if (r % c == 0 && p.b * p.G * c <= 2 * (int64_t)sms) return c;
    return 1;
}

template <typename T>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t st)
{
    const int S = decode_cluster(p);
    const int ro = p.H / p.G / S;
    const size_t smem = sizeof(float) * (size_t)(2 * ro * p.P + 2 * p.N + ro + kThreads / 32 + kMaxCluster);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.G * S), (unsigned)p.b);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = S > 1 ? 1 : 0;
#define SSD_DEC_CASE(NN, RIF)                                                                     \
    if (p.N == NN) {                                                                              \
        cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<T, NN, RIF>,                      \
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                           \
        LaunchScope ls("decode_step", st);                                                        \
        return cudaLaunchKernelEx(&cfg, decode_step_kernel<T, NN, RIF>, p, S);                     \
    }
    if (S == 1) {
        SSD_DEC_CASE(16, 2) SSD_DEC_CASE(32, 2) SSD_DEC_CASE(64, 2) SSD_DEC_CASE(128, 2)
    } else {
        SSD_DEC_CASE(16, 8) SSD_DEC_CASE(32, 8) SSD_DEC_CASE(64, 8) SSD_DEC_CASE(128, 8)
    }
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
