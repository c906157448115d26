// ssd_backward.cu -- backward pass (vector-Jacobian product) of the SSD mixer core, on CUDA
// cores in fp32.
//
// The mixer is trained through its scan, and gradient flow through the scan is one of the
// checks the pages run on it (Modalities PR #459, sections "Testing" and "Caveats"). Given
// the forward's inputs and the gradient dout of a scalar loss with respect to y (and,
// optionally, with respect to the final SSM and conv states), one call computes the
// gradients with respect to x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w and both
// initial states. Nothing is saved from the training forward: it is recomputed.
//
// Schedule (all on the caller's stream):
//   forward    the CUDA-core prefill with 64-token chunks, into the workspace: xBC',
//              delta, the state entering every chunk, the pre-norm y
//   norm_gate  one warp per (token, group): dy (gradient of y before the gate) and dz from
//              dout through the gated RMSNorm; dnorm_w summed per block in shared memory,
//              then added atomically
//   scan       one CTA per (row, head, 16 state rows p); each thread owns four elements
//              H[p][n] of one column n. For each chunk, last to first, it steps the state
//              entering the chunk to the start of each 16-token sub-chunk; for each
//              sub-chunk, last to first, it recomputes the sub-chunk's 16 states
//              (registers), then runs the recurrence backwards with G the gradient of the
//              state after token t:
//                G += dy_t (x) C'_t,  dC'_t = H_t^T dy_t,  dx'_t = delta_t G B'_t + D dy_t,
//                dB'_t = delta_t G^T x'_t,  ddelta_t = A a_t <G, H_{t-1}> + <G, x'_t (x) B'_t>,
//                dA += delta_t a_t <G, H_{t-1}>,  G <- a_t G       (a_t = exp(delta_t A)).
//              dB' and dC' leave as partial sums per (head, row block), ddelta per row block;
//              G after the first token is the initial state's gradient
//   conv       one thread per (row, channel, 32 tokens): dv = dxBC' SiLU'(v) with v
//              recomputed, the conv's transpose for the raw inputs and the initial conv
//              state (plus the final conv state's gradient on the last three positions),
//              dconv_w and dconv_b per thread, then added atomically
//   dt         ddt = ddelta sigmoid(dt + dt_bias); ddt_bias per block, added atomically
// Every element of an activation or state gradient is written by exactly one thread;
// parameter gradients are fp32 sums whose order of addition is not fixed.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"

namespace ssd {
namespace {

constexpr int kQf = kBackwardForwardChunk;   // tokens per chunk of the recompute forward
constexpr int kQb = kBackwardChunk;   // tokens per recompute sub-chunk (states in registers)
constexpr int kSub = kQf / kQb;       // sub-chunks per chunk
constexpr int kRows = kBackwardRows;  // state rows per scan CTA
constexpr int kE = 4;                 // state rows per scan thread (four row groups of four)
constexpr int kConvSeg = 32;          // tokens per conv-backward thread
constexpr int kNormRows = 64;         // token rows per norm-backward CTA

__device__ __forceinline__ float sigmoid_f(float u) { return 1.0f / (1.0f + expf(-u)); }

// d/du [u sigmoid(u)] = sigmoid(u) (1 + u (1 - sigmoid(u)))
__device__ __forceinline__ float dsilu(float u)
{
    const float s = sigmoid_f(u);
    return s * (1.0f + u * (1.0f - s));
}

// ------------------------------------------------------------------ gated RMSNorm backward
// out = g r w with g = y SiLU(z), r = (mean_group g^2 + eps)^(-1/2):
//   dg_c = r w_c dout_c - (r^3 / gs) g_c sum_i w_i dout_i g_i,  dy = dg SiLU(z),
//   dz = dg y SiLU'(z),  dw_c = sum over tokens of dout_c g_c r.
// One CTA of 8 warps per (64 token rows, group); warp w takes rows w, w + 8, ...
template <typename T>
__global__ void __launch_bounds__(256) bwd_norm_gate_kernel(BackwardParams p, int smem_acc)
{
    extern __shared__ float acc[];   // [gs] this CTA's share of dnorm_w (when it fits)
    const PrefillParams& f = p.f;
    const int64_t HP = f.HP(), gs = HP / f.G;
    const int g = blockIdx.y;
    const int64_t c0 = (int64_t)g * gs;
    const int64_t rows = f.b * f.L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* dw = smem_acc ? acc : p.dnorm_w + c0;
    if (smem_acc) {
        for (int64_t c = threadIdx.x; c < gs; c += blockDim.x) acc[c] = 0.0f;
        __syncthreads();
    }
    const int64_t r0 = (int64_t)blockIdx.x * kNormRows;
    const int64_t r1 = min(rows, r0 + kNormRows);
    for (int64_t row = r0 + warp; row < r1; row += 8) {
        const float* yp = f.ypre + row * HP + c0;
        const T* z = (const T*)f.z + row * f.z_ld + c0;
        const T* dout = (const T*)p.dout + row * p.dout_ld + c0;
        const float* nw = f.norm_w + c0;
        float ss = 0.0f, dot = 0.0f;
        for (int64_t c = lane; c < gs; c += 32) {
            const float gt = yp[c] * silu(ld_f<T>(z + c));
            ss += gt * gt;
            dot += nw[c] * ld_f<T>(dout + c) * gt;
        }
        ss = warp_sum(ss);
        dot = warp_sum(dot);
        const float r = rsqrtf(ss / (float)gs + f.eps);
        const float k3 = r * r * r / (float)gs * dot;
        float* dy = p.dy + row * HP + c0;
        T* dz = (T*)p.dz + row * p.dz_ld + c0;
        for (int64_t c = lane; c < gs; c += 32) {
            const float zc = ld_f<T>(z + c), yc = yp[c], sc = silu(zc), gt = yc * sc;
            const float dc = ld_f<T>(dout + c);
            const float dg = r * nw[c] * dc - k3 * gt;
            dy[c] = dg * sc;
            dz[c] = Act<T>::from_f(dg * yc * dsilu(zc));
            atomicAdd(dw + c, dc * gt * r);
        }
    }
    if (smem_acc) {
        __syncthreads();
        for (int64_t c = threadIdx.x; c < gs; c += blockDim.x) atomicAdd(p.dnorm_w + c0 + c, acc[c]);
    }
}

// ------------------------------------------------------------------ scan backward
template <int N>
struct BwdScanSmem {
    static constexpr int NT = 4 * N;
    static constexpr int NW = N >= 32 ? N / 32 : 1;   // warps per row group
    static constexpr int NWARPS = NT / 32;
    float x[kQf][kRows];        // x' of the chunk's tokens, this CTA's rows
    float dy[kQf][kRows];       // dy, same
    float b[kQf][N];            // B' of the head's group
    float c[kQf][N];            // C'
    float dl[kQf], al[kQf];     // delta and exp(delta A); 0 and 1 past the end of the row
    float entry[kSub][kE][NT];  // each thread's state entering each 16-token sub-chunk
    float rc[kQb][4][N];        // per row group: dC' summed over its four rows
    float rb[kQb][4][N];        // per row group: dB' summed over its four rows
    float rx[kQb][kRows][NW];   // dx' summed over one warp's columns
    float rd[kQb][NWARPS];      // ddelta summed over one warp's elements
    float red[2][32];
};

// Thread tid: column n = tid % N, row group rg = tid / N (rows rg*4 .. rg*4+3 of the CTA's 16).
// Per 64-token chunk of the forward (last to first): stage it, step the state entering it
// through the chunk to get the state entering each 16-token sub-chunk, then for each
// sub-chunk (last to first) recompute its 16 states and run the recurrence backwards.
template <typename T, int P, int N>
__global__ void __launch_bounds__(4 * N) bwd_scan_kernel(BackwardParams p)
{
    constexpr int NT = 4 * N, NB = P / kRows;
    using S = BwdScanSmem<N>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    S& s = *reinterpret_cast<S*>(smem_raw);
    const PrefillParams& f = p.f;
    const int pb = blockIdx.x, h = blockIdx.y;
    const int64_t bi = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = tid % N, rg = tid / N;
    const int g = h / (f.H / f.G);
    const int64_t HP = f.HP(), GN = f.GN(), Cc = f.Cc(), L = f.L, PN = (int64_t)P * N;
    const float A = f.A[h], Dh = f.D[h];
    const int pr = pb * kRows;          // first row of the CTA
    const int p0 = pr + rg * kE;        // first of this thread's rows
    const T* xbc = (const T*)f.xbc;

    float G[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e)
        G[e] = p.dfinal_ssm ? p.dfinal_ssm[((bi * f.H + h) * P + p0 + e) * N + n] : 0.0f;
    float accA = 0.0f, accD = 0.0f;

    for (int64_t ck = f.nc - 1; ck >= 0; --ck) {
        const int64_t t0 = ck * kQf;
        const int len = (int)min((int64_t)kQf, L - t0);
        __syncthreads();   // the previous chunk's partial sums have been written out
        // stage the chunk; zeros (delta 0, a 1) past the end of the row make those steps no-ops
        for (int i = tid; i < kQf * kRows; i += NT) {
            const int t = i / kRows, r = i % kRows;
            const bool in = t < len;
            const int64_t row = bi * L + t0 + t;
            s.x[t][r] = in ? ld_f<T>(xbc + row * Cc + (int64_t)h * P + pr + r) : 0.0f;
            s.dy[t][r] = in ? p.dy[row * HP + (int64_t)h * P + pr + r] : 0.0f;
        }
        for (int i = tid; i < kQf * N; i += NT) {
            const int t = i / N, m = i % N;
            const bool in = t < len;
            const int64_t row = bi * L + t0 + t;
            s.b[t][m] = in ? ld_f<T>(xbc + row * Cc + HP + (int64_t)g * N + m) : 0.0f;
            s.c[t][m] = in ? ld_f<T>(xbc + row * Cc + HP + GN + (int64_t)g * N + m) : 0.0f;
        }
        for (int t = tid; t < kQf; t += NT) {
            const float dl = t < len ? f.delta[(bi * f.H + h) * L + t0 + t] : 0.0f;
            s.dl[t] = dl;
            s.al[t] = expf(dl * A);
        }
        float hc[kE];
        const float* st = f.states + ((bi * f.nc + ck) * f.H + h) * PN;
#pragma unroll
        for (int e = 0; e < kE; ++e) hc[e] = st[(int64_t)(p0 + e) * N + n];
        __syncthreads();
        // the state entering each 16-token sub-chunk (each thread keeps its own four elements)
        for (int j = 0; j < kSub; ++j) {
#pragma unroll
            for (int e = 0; e < kE; ++e) s.entry[j][e][tid] = hc[e];
#pragma unroll
            for (int t = j * kQb; t < (j + 1) * kQb; ++t) {
                const float a = s.al[t], db = s.dl[t] * s.b[t][n];
#pragma unroll
                for (int e = 0; e < kE; ++e) hc[e] = a * hc[e] + db * s.x[t][rg * kE + e];
            }
        }
        for (int j = kSub - 1; j >= 0; --j) {
            const int tj = j * kQb;                       // first token of the sub-chunk in the chunk
            const int lj = min(kQb, len - tj);            // its tokens in the row (uniform over the CTA)
            if (lj <= 0) continue;
            float hin[kE];
#pragma unroll
            for (int e = 0; e < kE; ++e) hin[e] = s.entry[j][e][tid];
            // the sub-chunk's states, recomputed from the state entering it
            float hs[kQb][kE];
#pragma unroll
            for (int t = 0; t < kQb; ++t) {
                const float a = s.al[tj + t], db = s.dl[tj + t] * s.b[tj + t][n];
#pragma unroll
                for (int e = 0; e < kE; ++e)
                    hs[t][e] = a * (t ? hs[t - 1][e] : hin[e]) + db * s.x[tj + t][rg * kE + e];
            }
            // the recurrence backwards
#pragma unroll
            for (int t = kQb - 1; t >= 0; --t) {
                const int u = tj + t;
                const float a = s.al[u], dl = s.dl[u], bn = s.b[u][n], cn = s.c[u][n];
                float pc = 0.0f, gh = 0.0f, gx = 0.0f, px[kE];
#pragma unroll
                for (int e = 0; e < kE; ++e) {
                    const float dyv = s.dy[u][rg * kE + e], xv = s.x[u][rg * kE + e];
                    G[e] += dyv * cn;
                    pc += dyv * hs[t][e];
                    gh += G[e] * (t ? hs[t - 1][e] : hin[e]);
                    gx += G[e] * xv;
                    px[e] = dl * G[e] * bn;
                }
                accA += dl * a * gh;
                s.rc[t][rg][n] = pc;
                s.rb[t][rg][n] = dl * gx;
                {   // dx': the four rows' sums over the row group's columns, reduce-scattered over a
                    // segment of min(N, 32) lanes. After the two halving steps a lane keeps one row
                    // (slot 2 hiA + hiB), summed over its segment by the remaining steps.
                    constexpr int SEG = N < 32 ? N : 32, O1 = SEG / 2, O2 = SEG / 4;
                    const bool hiA = (lane & O1) != 0, hiB = (lane & O2) != 0;
                    float k0 = hiA ? px[2] : px[0], k1 = hiA ? px[3] : px[1];
                    const float s0 = hiA ? px[0] : px[2], s1 = hiA ? px[1] : px[3];
                    k0 += __shfl_xor_sync(0xffffffffu, s0, O1);
                    k1 += __shfl_xor_sync(0xffffffffu, s1, O1);
                    float k = hiB ? k1 : k0;
                    k += __shfl_xor_sync(0xffffffffu, hiB ? k0 : k1, O2);
#pragma unroll
                    for (int o = O2 / 2; o > 0; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
                    if ((lane & (O2 - 1)) == 0) s.rx[t][rg * kE + (hiA ? 2 : 0) + (hiB ? 1 : 0)][n / 32] = k;
                }
                const float dd = warp_sum(A * a * gh + bn * gx);
                if (lane == 0) s.rd[t][warp] = dd;
#pragma unroll
                for (int e = 0; e < kE; ++e) G[e] *= a;
            }
            __syncthreads();
            // the sub-chunk's sums out: dC', dB' per (head, row block); dx' complete; ddelta per row block
            const int64_t r0 = bi * L + t0 + tj;          // its first token row
            for (int i = tid; i < lj * N; i += NT) {
                const int t = i / N, m = i % N;
                const int64_t o = (((r0 + t) * f.H + h) * NB + pb) * N + m;
                p.dCp[o] = (s.rc[t][0][m] + s.rc[t][1][m]) + (s.rc[t][2][m] + s.rc[t][3][m]);
                p.dBp[o] = (s.rb[t][0][m] + s.rb[t][1][m]) + (s.rb[t][2][m] + s.rb[t][3][m]);
            }
            for (int i = tid; i < lj * kRows; i += NT) {
                const int t = i / kRows, r = i % kRows;
                float v = Dh * s.dy[tj + t][r];
#pragma unroll
                for (int w = 0; w < S::NW; ++w) v += s.rx[t][r][w];
                p.dxs[(r0 + t) * HP + (int64_t)h * P + pr + r] = v;
                accD += s.dy[tj + t][r] * s.x[tj + t][r];
            }
            if (tid < lj) {
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < S::NWARPS; ++w) v += s.rd[tid][w];
                p.ddp[((bi * f.H + h) * NB + pb) * L + t0 + tj + tid] = v;
            }
            __syncthreads();   // before the next sub-chunk overwrites the partial sums
        }
    }
    if (p.dinit_ssm) {
#pragma unroll
        for (int e = 0; e < kE; ++e) p.dinit_ssm[((bi * f.H + h) * P + p0 + e) * N + n] = G[e];
    }
    accA = warp_sum(accA);
    accD = warp_sum(accD);
    if (lane == 0) {
        s.red[0][warp] = accA;
        s.red[1][warp] = accD;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.0f, d = 0.0f;
        for (int w = 0; w < S::NWARPS; ++w) {
            a += s.red[0][w];
            d += s.red[1][w];
        }
        atomicAdd(p.dA + h, a);
        atomicAdd(p.dD + h, d);
    }
}

// ------------------------------------------------------------------ conv + SiLU backward
// v_t = conv_b + sum_k w_k s_{t+k} over s = [init_conv ; raw inputs], xBC' = SiLU(v), and the
// final conv state is s_{L..L+2}. With dv = dxBC' SiLU'(v):
//   ds_j = sum_k w_k dv_{j-k} (+ dfinal_conv_{j-L} for j >= L),
// raw input t gets ds_{t+3}, the initial conv state ds_{0..2};
//   dconv_w_k = sum_t dv_t s_{t+k},  dconv_b = sum_t dv_t.
template <typename T>
__global__ void __launch_bounds__(128) bwd_conv_kernel(BackwardParams p)
{
    const PrefillParams& f = p.f;
    const int64_t HP = f.HP(), GN = f.GN(), Cc = f.Cc(), L = f.L;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= Cc) return;
    const int64_t bi = blockIdx.z;
    const int64_t tb = (int64_t)blockIdx.y * kConvSeg, te = min(L, tb + kConvSeg);
    const int NB = f.P / kRows, r = f.H / f.G;
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = f.conv_w[c * 4 + k];
    const float bias = f.conv_b[c];
    // channel c's raw inputs and its gradient's destination
    const T* src;
    T* dst;
    int64_t ld, dld, col;
    if (c < HP) {
        src = (const T*)f.x; ld = f.x_ld; dst = (T*)p.dx; dld = p.dx_ld; col = c;
    } else if (c < HP + GN) {
        src = (const T*)f.B; ld = f.B_ld; dst = (T*)p.dB; dld = p.dB_ld; col = c - HP;
    } else {
        src = (const T*)f.C; ld = f.C_ld; dst = (T*)p.dC; dld = p.dC_ld; col = c - HP - GN;
    }
    // s_{t+3}: raw input t, or (t < 0) the initial conv state, zeros without one
    auto raw = [&](int64_t t) -> float {
        if (t >= 0) return ld_f<T>(src + (bi * L + t) * ld + col);
        return f.init_conv ? ld_f<T>((const T*)f.init_conv + (bi * Cc + c) * 3 + (t + 3)) : 0.0f;
    };
    // the gradient reaching xBC' of channel c at token t (B', C': summed over the group's
    // heads and row blocks)
    auto dxbc = [&](int64_t t) -> float {
        if (c < HP) return p.dxs[(bi * L + t) * HP + c];
        const bool isC = c >= HP + GN;
        const int64_t j = isC ? c - HP - GN : c - HP;
        const int gg = (int)(j / f.N), m = (int)(j % f.N);
        const float* part = isC ? p.dCp : p.dBp;
        float v = 0.0f;
        for (int hh = gg * r; hh < (gg + 1) * r; ++hh)
            for (int q = 0; q < NB; ++q) v += part[(((bi * L + t) * f.H + hh) * NB + q) * f.N + m];
        return v;
    };
    auto dv_at = [&](int64_t t) -> float {
        if (t < 0 || t >= L) return 0.0f;
        float v = bias;
#pragma unroll
        for (int k = 0; k < 4; ++k) v += w[k] * raw(t - 3 + k);
        return dxbc(t) * dsilu(v);
    };
    const float* dfc = p.dfinal_conv ? p.dfinal_conv + (bi * Cc + c) * 3 : nullptr;
    float dv[4];   // dv at tokens t .. t+3
#pragma unroll
    for (int k = 0; k < 4; ++k) dv[k] = dv_at(tb + k);
    if (tb == 0 && p.dinit_conv) {   // s_0 .. s_2, the initial conv state
        for (int j = 0; j < 3; ++j) {
            float v = 0.0f;
            for (int k = 0; k <= j; ++k) v += w[k] * dv[j - k];
            if (dfc && j >= L) v += dfc[j - L];
            p.dinit_conv[(bi * Cc + c) * 3 + j] = v;
        }
    }
    float dw[4] = {0.0f, 0.0f, 0.0f, 0.0f}, db = 0.0f;
    for (int64_t t = tb; t < te; ++t) {
        float du = w[0] * dv[3] + w[1] * dv[2] + w[2] * dv[1] + w[3] * dv[0];   // ds_{t+3}
        if (dfc && t + 3 >= L) du += dfc[t + 3 - L];
        dst[(bi * L + t) * dld + col] = Act<T>::from_f(du);
#pragma unroll
        for (int k = 0; k < 4; ++k) dw[k] += dv[0] * raw(t - 3 + k);
        db += dv[0];
        dv[0] = dv[1];
        dv[1] = dv[2];
        dv[2] = dv[3];
        dv[3] = dv_at(t + 4);
    }
    if (te > tb) {
#pragma unroll
        for (int k = 0; k < 4; ++k) atomicAdd(p.dconv_w + c * 4 + k, dw[k]);
        atomicAdd(p.dconv_b + c, db);
    }
}

// ------------------------------------------------------------------ softplus backward
// ddt = ddelta sigmoid(dt + dt_bias); one CTA per (256 tokens, head, row).
template <typename T>
__global__ void __launch_bounds__(256) bwd_dt_kernel(BackwardParams p)
{
    __shared__ float red[8];
    const PrefillParams& f = p.f;
    const int h = blockIdx.y;
    const int64_t bi = blockIdx.z;
    const int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int NB = f.P / kRows;
    float v = 0.0f;
    if (t < f.L) {
        float dd = 0.0f;
        for (int q = 0; q < NB; ++q) dd += p.ddp[((bi * f.H + h) * NB + q) * f.L + t];
        const float u = ld_f<T>((const T*)f.dt + (bi * f.L + t) * f.dt_ld + h) + f.dt_bias[h];
        v = dd * sigmoid_f(u);
        ((T*)p.ddt)[(bi * f.L + t) * p.ddt_ld + h] = Act<T>::from_f(v);
    }
    v = warp_sum(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.0f;
        for (int w = 0; w < 8; ++w) sum += red[w];
        atomicAdd(p.ddt_bias + h, sum);
    }
}

template <typename T, int P, int N>
cudaError_t launch_scan(const BackwardParams& p, cudaStream_t st)
{
    const size_t smem = sizeof(BwdScanSmem<N>);
    cudaError_t e = cudaFuncSetAttribute(bwd_scan_kernel<T, P, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope ls("bwd_scan", st);
    bwd_scan_kernel<T, P, N><<<dim3(P / kRows, p.f.H, (unsigned)p.f.b), 4 * N, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_all(const BackwardParams& p, cudaStream_t st)
{
    const PrefillParams& f = p.f;
    const int64_t HP = f.HP(), Cc = f.Cc();
    // parameter gradients are sums over rows and tokens: start them from zero
    const struct { float* ptr; int64_t n; } zero[] = {{p.dA, f.H}, {p.dD, f.H}, {p.dconv_w, Cc * 4},
                                                       {p.dconv_b, Cc}, {p.ddt_bias, f.H}, {p.dnorm_w, HP}};
    for (const auto& z : zero) {
        const cudaError_t e = cudaMemsetAsync(z.ptr, 0, (size_t)z.n * sizeof(float), st);
        if (e != cudaSuccess) return e;
    }
    if (f.b == 0) return cudaSuccess;
    cudaError_t e = launch_prefill_simt(f, st);
    if (e != cudaSuccess) return e;
    if (f.L > 0) {
        const int64_t gs = HP / f.G;
        const int smem_acc = gs * 4 <= 48 * 1024;
        LaunchScope ls("bwd_norm_gate", st);
        bwd_norm_gate_kernel<T><<<dim3((unsigned)((f.b * f.L + kNormRows - 1) / kNormRows), f.G), 256,
                                  smem_acc ? (size_t)gs * 4 : 0, st>>>(p, smem_acc);
    }
    e = cudaErrorInvalidValue;
#define SSD_BWD_CASE(PP, NN) \
    if (f.P == PP && f.N == NN) e = launch_scan<T, PP, NN>(p, st);
    SSD_BWD_CASE(16, 16) SSD_BWD_CASE(16, 32) SSD_BWD_CASE(16, 64) SSD_BWD_CASE(16, 128)
    SSD_BWD_CASE(32, 16) SSD_BWD_CASE(32, 32) SSD_BWD_CASE(32, 64) SSD_BWD_CASE(32, 128)
    SSD_BWD_CASE(64, 16) SSD_BWD_CASE(64, 32) SSD_BWD_CASE(64, 64) SSD_BWD_CASE(64, 128)
#undef SSD_BWD_CASE
    if (e != cudaSuccess) return e;
    {
        const int64_t segs = f.L > 0 ? (f.L + kConvSeg - 1) / kConvSeg : 1;
        LaunchScope ls("bwd_conv", st);
        bwd_conv_kernel<T><<<dim3((unsigned)((Cc + 127) / 128), (unsigned)segs, (unsigned)f.b), 128, 0, st>>>(p);
    }
    if (f.L > 0) {
        LaunchScope ls("bwd_dt", st);
        bwd_dt_kernel<T><<<dim3((unsigned)((f.L + 255) / 256), f.H, (unsigned)f.b), 256, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

bool backward_supported(int P, int N) { return prefill_simt_supported(P, N) && P % kBackwardRows == 0; }

cudaError_t launch_backward(const BackwardParams& p, cudaStream_t stream)
{
    if (p.f.act == 1) return launch_all<__nv_bfloat16>(p, stream);
    return launch_all<float>(p, stream);
}

}  // namespace ssd
