// ssd_prefill_simt.cu -- the CUDA-core (FFMA, fp32) prefill path of the SSD mixer.
//
// Five kernels, one pass each, enqueued on the caller's stream:
//   conv_silu     causal depthwise conv (K = 4) + bias + SiLU over the x|B|C channels
//                 (the "CausalConv1D" op of the Nemotron-H Mamba-2 mixer; gllm PR #86,
//                 section "2. feat(model): Nemotron-H on the CPU"), 16-byte loads, a
//                 sliding window of the last three raw inputs kept in registers.
//   conv_state    the last K-1 raw inputs of every channel -> final conv state.
//   chunk_state   per (row, chunk, head): delta = softplus(dt + dt_bias), the chunk's
//                 inclusive cumsum lam of delta*A, and the chunk's own state
//                 S[p][n] = sum_j exp(lam_end - lam_j) delta_j x'_j[p] B'_j[n]
//                 (the per-chunk state of the chunk-parallel SSD decomposition,
//                 Modalities PR #459, ssd.py notes).
//   state_pass    sequential over chunks: H_{c+1} = exp(lam_end(c)) H_c + S_c, keeps
//                 the state entering every chunk, writes the final SSM state.
//   chunk_scan    per (row, chunk, head, 64-row tile):
//                 y_i = sum_{j<=i} (C'_i.B'_j) exp(lam_i - lam_j) delta_j x'_j
//                       + exp(lam_i) C'_i . H_c + D x'_i
//   gated_norm    g = y * SiLU(z); out = g / sqrt(mean_group(g^2) + eps) * norm_w.
// This path carries the fp32 workloads (a 1e-4 relative bound that TF32 or bf16
// operands cannot meet) and serves as the plain reference schedule for the
// tensor-core path.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"

namespace ssd {
namespace {

constexpr int kConvTokens = 16;  // tokens per thread in conv_silu
constexpr int kTile = 64;        // row / column tile of chunk_scan

template <typename T>
__global__ void __launch_bounds__(128) conv_silu_kernel(PrefillParams p)
{
    constexpr int V = Act<T>::kVec;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    const int64_t cv = ((int64_t)blockIdx.y * blockDim.x + threadIdx.x) * V;
    if (cv >= Cc) return;
    const int64_t bi = blockIdx.z;
    const int64_t t0 = (int64_t)blockIdx.x * kConvTokens;
    if (t0 >= p.L) return;

    const T* src;
    int64_t ld, col;
    if (cv < HP) { src = (const T*)p.x; ld = p.x_ld; col = cv; }
    else if (cv < HP + GN) { src = (const T*)p.B; ld = p.B_ld; col = cv - HP; }
    else { src = (const T*)p.C; ld = p.C_ld; col = cv - HP - GN; }
    const T* base = src + bi * p.L * ld + col;

    float w[V][4], bias[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const float4 wv = *reinterpret_cast<const float4*>(p.conv_w + (cv + i) * 4);
        w[i][0] = wv.x; w[i][1] = wv.y; w[i][2] = wv.z; w[i][3] = wv.w;
        bias[i] = p.conv_b[cv + i];
    }
    // win[k] = raw input at token t-3+k (k = 0..2)
    float win[3][V];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int64_t tt = t0 - 3 + k;
        if (tt >= 0) {
            load_vec<T>(base + tt * ld, win[k]);
        } else {
#pragma unroll
            for (int i = 0; i < V; ++i)
                win[k][i] = p.init_conv
                                ? ld_f<T>((const T*)p.init_conv + (bi * Cc + cv + i) * 3 + (tt + 3))
                                : 0.0f;
        }
    }
    T* out = (T*)p.xbc + bi * p.L * Cc + cv;
    const int64_t t1 = min(t0 + kConvTokens, p.L);
    for (int64_t t = t0; t < t1; ++t) {
        float u[V], o[V];
        load_vec<T>(base + t * ld, u);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const float v = bias[i] + w[i][0] * win[0][i] + w[i][1] * win[1][i] +
                            w[i][2] * win[2][i] + w[i][3] * u[i];
            o[i] = silu(v);
            win[0][i] = win[1][i];
            win[1][i] = win[2][i];
            win[2][i] = u[i];
        }
        store_vec<T>(out + t * Cc, o);
    }
}

// final_conv[c][k] = s[L + k], s = [init_conv[c][0..2], raw[0..L-1]]. Runs after
// conv_silu, and each thread reads its channel's three old taps before writing, so the
// final state may share memory with the initial one.
template <typename T>
__global__ void conv_state_kernel(PrefillParams p)
{
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= p.b * Cc) return;
    const int64_t bi = idx / Cc, c = idx % Cc;
    const T* src;
    int64_t ld, col;
    if (c < HP) { src = (const T*)p.x; ld = p.x_ld; col = c; }
    else if (c < HP + GN) { src = (const T*)p.B; ld = p.B_ld; col = c - HP; }
    else { src = (const T*)p.C; ld = p.C_ld; col = c - HP - GN; }
    T v[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int64_t s = p.L + k;  // index into s
        if (s >= 3) v[k] = src[(bi * p.L + (s - 3)) * ld + col];
        else v[k] = p.init_conv ? ((const T*)p.init_conv)[idx * 3 + s] : Act<T>::from_f(0.0f);
    }
    T* fc = (T*)p.final_conv + idx * 3;
#pragma unroll
    for (int k = 0; k < 3; ++k) fc[k] = v[k];
}

// Inclusive scan of one value per thread over a block of up to 256 threads.
__device__ float block_inclusive_scan(float v, float* warp_tot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_tot[wid] = v;
    __syncthreads();
    float off = 0.0f;
    for (int w = 0; w < wid; ++w) off += warp_tot[w];
    return v + off;
}

template <typename T, int P, int N>
__global__ void __launch_bounds__(256) chunk_state_kernel(PrefillParams p)
{
    constexpr int JT = 32;               // tokens per smem stage
    constexpr int RP = P / 16, RN = N / 16;
    __shared__ float s_dl[256], s_w[256], s_wt[8];
    __shared__ float xs[JT][P];
    __shared__ float bs[JT][N + 1];

    const int c = blockIdx.x, h = blockIdx.y;
    const int64_t bi = blockIdx.z;
    const int r = p.H / p.G, g = h / r;
    const int64_t t0 = (int64_t)c * p.Q;
    const int len = (int)min((int64_t)p.Q, p.L - t0);
    const int tid = threadIdx.x;
    const int64_t Cc = p.Cc(), HP = p.HP();

    // delta and the within-chunk inclusive cumsum of delta * A
    float dl = 0.0f, a = 0.0f;
    if (tid < len) {
        const float u = ld_f<T>((const T*)p.dt + (bi * p.L + t0 + tid) * p.dt_ld + h) + p.dt_bias[h];
        dl = softplus(u);
        a = dl * p.A[h];
    }
    const float lam = block_inclusive_scan(a, s_wt);
    if (tid < len) {
        const int64_t o = (bi * p.H + h) * p.L + t0 + tid;
        p.delta[o] = dl;
        p.lam[o] = lam;
        s_dl[tid] = dl;
    }
    __shared__ float s_lam_end;
    if (tid == len - 1) s_lam_end = lam;
    __syncthreads();
    if (tid < len) s_w[tid] = expf(s_lam_end - lam) * s_dl[tid];
    __syncthreads();

    const int ty = tid / 16, tx = tid % 16;
    float acc[RP][RN];
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int k = 0; k < RN; ++k) acc[i][k] = 0.0f;

    const T* xbc = (const T*)p.xbc + (bi * p.L + t0) * Cc;
    for (int j0 = 0; j0 < len; j0 += JT) {
        for (int e = tid; e < JT * P; e += 256) {
            const int jj = e / P, pp = e % P;
            xs[jj][pp] = (j0 + jj < len) ? s_w[j0 + jj] * ld_f<T>(xbc + (int64_t)(j0 + jj) * Cc + (int64_t)h * P + pp) : 0.0f;
        }
        for (int e = tid; e < JT * N; e += 256) {
            const int jj = e / N, nn = e % N;
            bs[jj][nn] = (j0 + jj < len) ? ld_f<T>(xbc + (int64_t)(j0 + jj) * Cc + HP + (int64_t)g * N + nn) : 0.0f;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < JT; ++jj) {
            float xv[RP], bv[RN];
#pragma unroll
            for (int i = 0; i < RP; ++i) xv[i] = xs[jj][ty + 16 * i];
#pragma unroll
            for (int k = 0; k < RN; ++k) bv[k] = bs[jj][tx + 16 * k];
#pragma unroll
            for (int i = 0; i < RP; ++i)
#pragma unroll
                for (int k = 0; k < RN; ++k) acc[i][k] += xv[i] * bv[k];
        }
        __syncthreads();
    }
    float* S = p.states + (((bi * p.nc + c) * p.H + h) * (int64_t)P) * N;
    if (!SSD_IN_BOUNDS(p.status, bi < p.b && c < p.nc && h < p.H)) return;
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int k = 0; k < RN; ++k) S[(ty + 16 * i) * N + tx + 16 * k] = acc[i][k];
}

// Sequential pass over chunks; each thread owns 4 consecutive state elements of one
// (row, head). Reads the initial state and writes the final one in the same thread.
__global__ void __launch_bounds__(256) state_pass_kernel(PrefillParams p)
{
    const int64_t PN = (int64_t)p.P * p.N;
    const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (e >= PN) return;
    const int h = blockIdx.y;
    const int64_t bi = blockIdx.z;
    float4 H = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.init_ssm) H = *reinterpret_cast<const float4*>(p.init_ssm + (bi * p.H + h) * PN + e);
    const float* lam = p.lam + (bi * p.H + h) * p.L;
    for (int64_t c = 0; c < p.nc; ++c) {
        float4* slot = reinterpret_cast<float4*>(p.states + ((bi * p.nc + c) * p.H + h) * PN + e);
        const float4 S = *slot;
        *slot = H;
        const float a = expf(lam[min((c + 1) * p.Q, p.L) - 1]);
        H.x = a * H.x + S.x; H.y = a * H.y + S.y; H.z = a * H.z + S.z; H.w = a * H.w + S.w;
    }
    *reinterpret_cast<float4*>(p.final_ssm + (bi * p.H + h) * PN + e) = H;
}

template <int P, int N>
struct ScanSmem {
    float cs[kTile][N];          // C' rows of the output tile
    float bs[kTile][N + 1];      // B' rows of the current column tile
    float m[kTile][kTile + 1];   // decay-masked (C'B'^T) tile
    float xs[kTile][P];          // x' rows of the current column tile
    float hs[P][N + 1];          // state entering the chunk
    float lam[256], dl[256];
};

template <typename T, int P, int N>
__global__ void __launch_bounds__(256) chunk_scan_kernel(PrefillParams p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ScanSmem<P, N>& s = *reinterpret_cast<ScanSmem<P, N>*>(smem_raw);
    constexpr int RQ = P / 16;
    const int tiles = (p.Q + kTile - 1) / kTile;
    const int64_t c = blockIdx.x / tiles;
    const int it = (int)(blockIdx.x % tiles);
    const int64_t bi = blockIdx.z;
    const int h = blockIdx.y, r = p.H / p.G, g = h / r;
    const int64_t t0 = (int64_t)c * p.Q;
    const int len = (int)min((int64_t)p.Q, p.L - t0);
    const int i0 = it * kTile;
    if (i0 >= len) return;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int64_t Cc = p.Cc(), HP = p.HP(), GN = p.GN();
    const T* xbc = (const T*)p.xbc + (bi * p.L + t0) * Cc;

    for (int e = tid; e < len; e += 256) {
        s.lam[e] = p.lam[(bi * p.H + h) * p.L + t0 + e];
        s.dl[e] = p.delta[(bi * p.H + h) * p.L + t0 + e];
    }
    for (int e = tid; e < kTile * N; e += 256) {
        const int ii = e / N, nn = e % N;
        s.cs[ii][nn] = (i0 + ii < len) ? ld_f<T>(xbc + (int64_t)(i0 + ii) * Cc + HP + GN + (int64_t)g * N + nn) : 0.0f;
    }
    float acc[4][RQ];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < RQ; ++q) acc[a][q] = 0.0f;

    for (int j0 = 0; j0 <= i0; j0 += kTile) {
        __syncthreads();
        for (int e = tid; e < kTile * N; e += 256) {
            const int jj = e / N, nn = e % N;
            s.bs[jj][nn] = (j0 + jj < len) ? ld_f<T>(xbc + (int64_t)(j0 + jj) * Cc + HP + (int64_t)g * N + nn) : 0.0f;
        }
        for (int e = tid; e < kTile * P; e += 256) {
            const int jj = e / P, pp = e % P;
            s.xs[jj][pp] = (j0 + jj < len) ? ld_f<T>(xbc + (int64_t)(j0 + jj) * Cc + (int64_t)h * P + pp) : 0.0f;
        }
        __syncthreads();
        // masked, decayed C'B'^T tile
        float cb[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) cb[a][bq] = 0.0f;
        for (int n = 0; n < N; ++n) {
            float cv[4], bv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) cv[a] = s.cs[ty + 16 * a][n];
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) bv[bq] = s.bs[tx + 16 * bq][n];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int bq = 0; bq < 4; ++bq) cb[a][bq] += cv[a] * bv[bq];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
                const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * bq;
                float v = 0.0f;
                if (j <= i && i < len && j < len) v = cb[a][bq] * expf(s.lam[i] - s.lam[j]) * s.dl[j];
                s.m[ty + 16 * a][tx + 16 * bq] = v;
            }
        __syncthreads();
        for (int jj = 0; jj < kTile; ++jj) {
            float mv[4], xv[RQ];
#pragma unroll
            for (int a = 0; a < 4; ++a) mv[a] = s.m[ty + 16 * a][jj];
#pragma unroll
            for (int q = 0; q < RQ; ++q) xv[q] = s.xs[jj][tx + 16 * q];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < RQ; ++q) acc[a][q] += mv[a] * xv[q];
        }
    }
    // contribution of the state entering the chunk
    __syncthreads();
    const float* Hc = p.states + ((bi * p.nc + c) * p.H + h) * (int64_t)P * N;
    for (int e = tid; e < P * N; e += 256) s.hs[e / N][e % N] = Hc[e];
    __syncthreads();
    float ch[4][RQ];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < RQ; ++q) ch[a][q] = 0.0f;
    for (int n = 0; n < N; ++n) {
        float cv[4], hv[RQ];
#pragma unroll
        for (int a = 0; a < 4; ++a) cv[a] = s.cs[ty + 16 * a][n];
#pragma unroll
        for (int q = 0; q < RQ; ++q) hv[q] = s.hs[tx + 16 * q][n];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int q = 0; q < RQ; ++q) ch[a][q] += cv[a] * hv[q];
    }
    const float Dh = p.D[h];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + ty + 16 * a;
        if (i >= len || !SSD_IN_BOUNDS(p.status, t0 + i < p.L)) continue;
        const float el = expf(s.lam[i]);
        float* yo = p.ypre + (bi * p.L + t0 + i) * HP + (int64_t)h * P;
#pragma unroll
        for (int q = 0; q < RQ; ++q) {
            const int pp = tx + 16 * q;
            const float xv = ld_f<T>(xbc + (int64_t)i * Cc + (int64_t)h * P + pp);
            yo[pp] = acc[a][q] + el * ch[a][q] + Dh * xv;
        }
    }
}

// One warp per (row, token, group): out = g / sqrt(mean(g^2) + eps) * norm_w.
template <typename T>
__global__ void __launch_bounds__(256) gated_norm_kernel(PrefillParams p)
{
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = p.b * p.L;
    if (w >= rows * p.G) return;
    const int64_t row = w / p.G;
    const int g = (int)(w % p.G);
    const int64_t HP = p.HP(), gs = HP / p.G, c0 = (int64_t)g * gs;
    const float* yp = p.ypre + row * HP + c0;
    const T* z = (const T*)p.z + row * p.z_ld + c0;
    float ss = 0.0f;
    for (int64_t c = lane; c < gs; c += 32) {
        const float gt = yp[c] * silu(ld_f<T>(z + c));
        ss += gt * gt;
    }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)gs + p.eps);
    T* y = (T*)p.y + row * p.y_ld + c0;
    for (int64_t c = lane; c < gs; c += 32) {
        const float gt = yp[c] * silu(ld_f<T>(z + c));
        y[c] = Act<T>::from_f(gt * inv * p.norm_w[c0 + c]);
    }
}

template <typename T, int P, int N>
cudaError_t launch_scan_kernels(const PrefillParams& p, cudaStream_t st)
{
    {
        LaunchScope ls("simt_chunk_state", st);
        chunk_state_kernel<T, P, N><<<dim3((unsigned)p.nc, p.H, (unsigned)p.b), 256, 0, st>>>(p);
    }
    const int64_t PN = (int64_t)P * N;
    {
        LaunchScope ls("simt_state_pass", st);
        state_pass_kernel<<<dim3((unsigned)((PN / 4 + 255) / 256), p.H, (unsigned)p.b), 256, 0, st>>>(p);
    }
    const size_t smem = sizeof(ScanSmem<P, N>);
    cudaError_t e = cudaFuncSetAttribute(chunk_scan_kernel<T, P, N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.Q + kTile - 1) / kTile;
    LaunchScope ls("simt_chunk_scan", st);
    chunk_scan_kernel<T, P, N><<<dim3((unsigned)(tiles * p.nc), p.H, (unsigned)p.b), 256, smem, st>>>(p);
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_all(const PrefillParams& p, cudaStream_t st)
{
    constexpr int V = Act<T>::kVec;
    const int64_t Cc = p.Cc();
    if (p.b == 0) return cudaSuccess;
    if (p.L > 0) {
        LaunchScope ls("conv_silu", st);
        conv_silu_kernel<T><<<dim3((unsigned)((p.L + kConvTokens - 1) / kConvTokens),
                                   (unsigned)((Cc / V + 127) / 128), (unsigned)p.b), 128, 0, st>>>(p);
    }
    {
        LaunchScope ls("conv_state", st);
        conv_state_kernel<T><<<(unsigned)((p.b * Cc + 255) / 256), 256, 0, st>>>(p);
    }
    if (p.L == 0) {  // no tokens: the final SSM state is the initial one
        const int64_t PN = (int64_t)p.P * p.N;
        LaunchScope ls("simt_state_pass", st);
        state_pass_kernel<<<dim3((unsigned)((PN / 4 + 255) / 256), p.H, (unsigned)p.b), 256, 0, st>>>(p);
        return cudaGetLastError();
    }
    cudaError_t e = cudaErrorInvalidValue;
#define SSD_SIMT_CASE(PP, NN) \
    if (p.P == PP && p.N == NN) e = launch_scan_kernels<T, PP, NN>(p, st);
    SSD_SIMT_CASE(16, 16) SSD_SIMT_CASE(16, 32) SSD_SIMT_CASE(16, 64) SSD_SIMT_CASE(16, 128)
    SSD_SIMT_CASE(32, 16) SSD_SIMT_CASE(32, 32) SSD_SIMT_CASE(32, 64) SSD_SIMT_CASE(32, 128)
    SSD_SIMT_CASE(64, 16) SSD_SIMT_CASE(64, 32) SSD_SIMT_CASE(64, 64) SSD_SIMT_CASE(64, 128)
#undef SSD_SIMT_CASE
    if (e != cudaSuccess) return e;
    const int64_t warps = p.b * p.L * p.G;
    {
        LaunchScope ls("gated_norm", st);
        gated_norm_kernel<T><<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

bool prefill_simt_supported(int P, int N)
{
    const bool okP = P == 16 || P == 32 || P == 64;
    const bool okN = N == 16 || N == 32 || N == 64 || N == 128;
    return okP && okN;
}

cudaError_t launch_prefill_simt(const PrefillParams& p, cudaStream_t stream)
{
    if (p.act == 1) return launch_all<__nv_bfloat16>(p, stream);
    return launch_all<float>(p, stream);
}

}  // namespace ssd
