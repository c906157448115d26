// ssd_prefill_tc.cu -- the tensor-core (tcgen05) prefill of the SSD mixer for bf16
// activations, head dim 64 and state dim 128.
//
// One kernel does the whole core: causal conv + SiLU, softplus, the chunked SSD scan
// with the state kept on chip, the D skip and the gated group RMSNorm. Each CTA owns one
// head of one batch row and walks the sequence in 128-token blocks, so the state never
// leaves the SM: no chunk states are written to memory and there is no separate state
// pass. The r heads of a group form a thread-block cluster: every CTA convolves 1/r of
// the group's B and C channels and stores its slice into every peer's shared memory
// (DSMEM), and the norm's per-token sums of squares are exchanged the same way, so the
// normalisation over the group's r*64 channels happens in the same pass.
//
// Per 128-token block (Modalities PR #459, ssd.py notes: the chunk-parallel SSD block
// decomposition with a within-chunk segment sum):
//   lam_i  = inclusive sum of delta*A over the block (log2 units here)
//   CB     = C' B'^T                                  (MMA, 128x128, K = 128)
//   Ys     = C' H^T                                   (MMA, 128x64,  K = 128)
//   S^T    = B'^T (x' * w),  w_j = exp(lam_end - lam_j) delta_j   (MMA, 128x64, K = 128)
//   M_ij   = CB_ij exp(lam_i - lam_j) delta_j  (j <= i, else 0), rounded to bf16
//   Yi     = M x'                                     (MMA, 128x64,  K = 128)
//   y_i    = Yi_i + exp(lam_i) Ys_i + D x'_i ;  g = y SiLU(z) ; out = g / rms_group(g) * norm_w
//   H     <- exp(lam_end) H + S                       (fp32, in registers)
// The result equals the chunked form with 128-token chunks, which equals the sequential
// recurrence up to rounding for any chunk length.
//
// Threads: 256. Thread t owns TMEM lane / row (t % 128) and column half (t / 128).
// Thread 0 issues the MMAs; mbarriers signal their completion (bounded waits).
#include <cooperative_groups.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"
#include "ssd_tc_util.cuh"

namespace cg = cooperative_groups;

namespace ssd {
namespace {

using namespace tc;

constexpr int kT = 128;       // tokens per block
constexpr int kP = 64;        // head dim
constexpr int kN = 128;       // state dim
constexpr int kThreads = 256;
constexpr int kStageRows = kT + 3;   // 3 halo rows (raw inputs before the block) + the block

// TMEM columns
constexpr uint32_t kColCB = 0, kColYi = 128, kColYs = 192, kColS = 256, kTmemCols = 512;

// shared memory map (bytes)
constexpr uint32_t OFF_C = 0;          // C'   [128 tok][128 n]  bf16 canonical
constexpr uint32_t OFF_B = 32768;      // B'   [128 tok][128 n]
constexpr uint32_t OFF_M = 65536;      // M    [128 i][128 j]
constexpr uint32_t OFF_X = 98304;      // x'   [128 tok][64 p]
constexpr uint32_t OFF_XW = 114688;    // x'*w [128 tok][64 p]
constexpr uint32_t OFF_H = 131072;     // H^T  [128 n][64 p]
constexpr uint32_t OFF_STAGE = 147456; // raw staging, 8-channel vectors: [SROW/8][131 rows] x 16 B

constexpr long long kWaitLimit = 4000000000LL;  // ~2 s at 2 GHz

template <int R>
struct Layout {
    static constexpr int NS = kN / R;                // B/C channels convolved by one CTA
    static constexpr int SROW = kP + 2 * NS;         // staged channels per row
    static constexpr int NV = SROW / 8;              // staged 8-channel vectors
    static constexpr uint32_t STAGE_BYTES = (uint32_t)kStageRows * SROW * 2;
    static constexpr uint32_t OFF_MISC = OFF_STAGE + ((STAGE_BYTES + 127) / 128) * 128;
    // misc floats
    static constexpr uint32_t F_LAM = 0, F_DL = 128, F_V = 256, F_SCAN = 384, F_RED = 392,
                              F_CW = F_RED + R * 256, F_CB = F_CW + SROW * 4, F_NW = F_CB + SROW,
                              F_END = F_NW + kP;
    static constexpr uint32_t OFF_BAR = OFF_MISC + ((F_END * 4 + 15) / 16) * 16;
    static constexpr uint32_t TOTAL = OFF_BAR + 32;
};

__device__ __forceinline__ float scan128(float v, float* tot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tot[wid] = v;
    __syncthreads();
    float off = 0.0f;
    for (int w = 0; w < wid; ++w) off += tot[w];
    return v + off;
}

// R = CTAs per cluster (heads per cluster). SPLIT: the group has more heads than one
// cluster holds (H/G > R); each CTA then writes the gated values and its per-token sums
// of squares, and norm_finish_kernel applies the group RMSNorm.
template <int R, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1) ssd_prefill_tc_kernel(PrefillParams p)
{
    using Lo = Layout<R>;
    constexpr int NS = Lo::NS, SROW = Lo::SROW;
    extern __shared__ __align__(1024) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int q = (int)cluster.block_rank();            // head within the cluster
    const int rpg = p.H / p.G;                           // heads per group
    const int ncl = rpg / R;                             // clusters per group
    const int64_t cid = blockIdx.x / R;                  // (batch row, group, cluster)
    const int64_t bi = cid / ((int64_t)p.G * ncl);
    const int g = (int)((cid / ncl) % p.G);
    const int h = g * rpg + (int)(cid % ncl) * R + q;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, half = tid >> 7;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    float* mf = reinterpret_cast<float*>(smem + Lo::OFF_MISC);
    float* s_lam = mf + Lo::F_LAM;     // log2-domain inclusive cumsum of delta*A
    float* s_dl = mf + Lo::F_DL;
    float* s_v = mf + Lo::F_V;         // column factors of the decay mask (see the M build)
    float* s_scan = mf + Lo::F_SCAN;
    float* s_red = mf + Lo::F_RED;     // [R][2][128] per-(head, half) sums of g^2, pushed by every peer
    float* s_cw = mf + Lo::F_CW;       // [SROW][4] conv taps of the staged channels
    float* s_cb = mf + Lo::F_CB;       // [SROW]
    float* s_nw = mf + Lo::F_NW;       // [64] norm weights of this head
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lo::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::OFF_BAR + 16);
    // stage[v * kStageRows + r]: channels 8v..8v+7 of staged row r (row r = token t0 + r - 3).
    // Vector-major, so threads on consecutive rows read consecutive 16-byte words.
    uint4* stage = reinterpret_cast<uint4*>(smem + OFF_STAGE);

    const uint32_t s_base = smem_u32(smem);
    const uint32_t aC = s_base + OFF_C, aB = s_base + OFF_B, aM = s_base + OFF_M;
    const uint32_t aX = s_base + OFF_X, aXW = s_base + OFF_XW, aH = s_base + OFF_H;
    const uint32_t bar0 = smem_u32(&bars[0]), bar1 = smem_u32(&bars[1]);

    // channel index (in xBC) of staged column c
    auto staged_channel = [&](int c) -> int64_t {
        if (c < kP) return (int64_t)h * kP + c;
        if (c < kP + NS) return HP + (int64_t)g * kN + (int64_t)q * NS + (c - kP);
        return HP + GN + (int64_t)g * kN + (int64_t)q * NS + (c - kP - NS);
    };

    // ---- set-up: parameters, initial conv taps, barriers, TMEM, initial state
    if (blockIdx.x == 0 && tid == 0) *p.status = 0;  // this call's status word starts clean
    for (int c = tid; c < SROW; c += kThreads) {
        const int64_t ch = staged_channel(c);
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        s_cw[c * 4 + 0] = w.x; s_cw[c * 4 + 1] = w.y; s_cw[c * 4 + 2] = w.z; s_cw[c * 4 + 3] = w.w;
        s_cb[c] = p.conv_b[ch];
    }
    if (tid < kP) s_nw[tid] = p.norm_w[(int64_t)h * kP + tid];
    for (int e = tid; e < 3 * SROW; e += kThreads) {
        const int k = e / SROW, c = e % SROW;
        __nv_bfloat16 v = __float2bfloat16_rn(0.0f);
        if (p.init_conv) v = ((const __nv_bfloat16*)p.init_conv)[(bi * Cc + staged_channel(c)) * 3 + k];
        reinterpret_cast<__nv_bfloat16*>(stage + (c / 8) * kStageRows + k)[c % 8] = v;
    }
    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    // state H^T[n][p]: thread (n = row, half) keeps p in [half*32, half*32 + 32) in fp32
    float H[32];
    {
        const float* h0 = p.init_ssm ? p.init_ssm + (bi * p.H + h) * (int64_t)kP * kN : nullptr;
#pragma unroll
        for (int i = 0; i < 32; ++i) H[i] = h0 ? h0[(int64_t)(half * 32 + i) * kN + row] : 0.0f;
        unsigned char* sH = smem + OFF_H;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
            u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
            *reinterpret_cast<uint4*>(sH + canon_off(row, half * 32 + 8 * v, kP)) = u;
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const float A2 = p.A[h] * 1.4426950408889634f;  // A in log2 units
    const float Dh = p.D[h];
    const float bias = p.dt_bias[h];
    bool ok = true;

    const int64_t nblk = (p.L + kT - 1) / kT;
    const __nv_bfloat16* gx = (const __nv_bfloat16*)p.x;
    const __nv_bfloat16* gB = (const __nv_bfloat16*)p.B;
    const __nv_bfloat16* gC = (const __nv_bfloat16*)p.C;
    const __nv_bfloat16* gz = (const __nv_bfloat16*)p.z;
    const __nv_bfloat16* gdt = (const __nv_bfloat16*)p.dt;
    __nv_bfloat16* gy = (__nv_bfloat16*)p.y;

    // issue the raw loads of block k into staging rows 3..3+len-1
    auto load_block = [&](int64_t k, int t0i, int nthr) {
        const int64_t t0 = k * kT;
        const int len = (int)min((int64_t)kT, p.L - t0);
        constexpr int CPR = SROW / 8;  // 16-byte chunks per staged row
        for (int e = t0i; e < len * CPR; e += nthr) {
            const int r = e / CPR, c8 = (e % CPR) * 8;
            const int64_t tok = bi * p.L + t0 + r;
            const __nv_bfloat16* src;
            if (c8 < kP) src = gx + tok * p.x_ld + (int64_t)h * kP + c8;
            else if (c8 < kP + NS) src = gB + tok * p.B_ld + (int64_t)g * kN + (int64_t)q * NS + (c8 - kP);
            else src = gC + tok * p.C_ld + (int64_t)g * kN + (int64_t)q * NS + (c8 - kP - NS);
            cp_async16(smem_u32(stage + (c8 / 8) * kStageRows + r + 3), src);
        }
        cp_async_commit();
    };

    if (nblk > 0) load_block(0, tid, kThreads);
    float dt_next = 0.0f;
    if (nblk > 0 && tid < kT && tid < p.L)
        dt_next = __bfloat162float(gdt[(bi * p.L + tid) * p.dt_ld + h]);

    int len = 0;
    for (int64_t k = 0; k < nblk; ++k) {
        const int64_t t0 = k * kT;
        len = (int)min((int64_t)kT, p.L - t0);
        const uint32_t par = (uint32_t)(k & 1);
        cp_async_wait_all();
        __syncthreads();

        // ---- delta and its within-block cumsum (log2 units)
        float dl = 0.0f, a2 = 0.0f;
        if (tid < len) {
            dl = softplus(dt_next + bias);
            a2 = dl * A2;
        }
        const float lam = scan128(a2, s_scan);
        if (tid < kT) { s_lam[tid] = lam; s_dl[tid] = dl; }
        __syncthreads();
        const float lam_end = s_lam[kT - 1];
        // exp2(lam_i - lam_j) = u_i * v_j with u_i = exp2(lam_i) and v_j = exp2(-lam_j): exact
        // up to rounding while the factors (and v_j times delta_j) stay normal fp32 numbers.
        // lam is non-increasing from <= 0, so for a row i with lam_i > -96 every j <= i has
        // v_j <= 2^96; rows past that decay take exp2 per element. The choice for row i
        // depends on tokens up to i only, so the result stays causal bit for bit.
        if (tid < kT) s_v[tid] = (lam > -96.0f) ? ex2(-lam) * dl : 0.0f;

        // ---- conv + SiLU of the staged channels: this head's x channels -> x' and x'*w in
        //      shared memory; this CTA's slice of B and C -> every peer's B' and C'.
        //      Work item (v, i): 8 channels of row i; consecutive threads take consecutive rows.
        {
            unsigned char* sX = smem + OFF_X;
            unsigned char* sXW = smem + OFF_XW;
            for (int e = tid; e < Lo::NV * kT; e += kThreads) {
                const int i = e % kT, v = e / kT;
                const int c0 = v * 8;
                float o[8];
                if (i < len) {
                    float u[4][8];
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) unpack_bf16x8(stage[v * kStageRows + i + kk], u[kk]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float* w = s_cw + (c0 + j) * 4;
                        const float vv = s_cb[c0 + j] + w[0] * u[0][j] + w[1] * u[1][j] + w[2] * u[2][j] + w[3] * u[3][j];
                        o[j] = silu_fast(vv);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = 0.0f;
                }
                uint4 u8;
                u8.x = pack_bf16x2(o[0], o[1]); u8.y = pack_bf16x2(o[2], o[3]);
                u8.z = pack_bf16x2(o[4], o[5]); u8.w = pack_bf16x2(o[6], o[7]);
                if (c0 < kP) {
                    const float wgt = (i < len) ? ex2(lam_end - s_lam[i]) * s_dl[i] : 0.0f;
                    uint4 uw;
                    uw.x = pack_bf16x2(o[0] * wgt, o[1] * wgt); uw.y = pack_bf16x2(o[2] * wgt, o[3] * wgt);
                    uw.z = pack_bf16x2(o[4] * wgt, o[5] * wgt); uw.w = pack_bf16x2(o[6] * wgt, o[7] * wgt);
                    *reinterpret_cast<uint4*>(sX + canon_off(i, c0, kP)) = u8;
                    *reinterpret_cast<uint4*>(sXW + canon_off(i, c0, kP)) = uw;
                } else {
                    const bool isC = c0 >= kP + NS;
                    const int n0 = q * NS + (isC ? c0 - kP - NS : c0 - kP);
                    uint4* dst = reinterpret_cast<uint4*>(smem + (isC ? OFF_C : OFF_B) + canon_off(i, n0, kN));
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) *cluster.map_shared_rank(dst, rr) = u8;
                }
            }
        }
        fence_async_smem();
        fence_async_cluster();
        fence_before_sync();
        cluster.sync();
        fence_after_sync();

        // ---- MMAs on C'B'^T, C'H^T and B'^T(x'w)
        if (tid == 0) {
            fence_async_smem();
            const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_ys = idesc_bf16(128, 64, 0, 1);
            const uint32_t id_s = idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColCB, sdesc(aC + kk * 256, 128, 2048), sdesc(aB + kk * 256, 128, 2048), id_cb, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColYs, sdesc(aC + kk * 256, 128, 2048), sdesc(aH + kk * 2048, 1024, 128), id_ys, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColS, sdesc(aB + kk * 4096, 2048, 128), sdesc(aXW + kk * 2048, 1024, 128), id_s, kk > 0);
            mma_commit(bar0);
        }
        // raw data of the next block: warps 1..7 keep its three halo rows, then start its
        // loads, while warp 0 issues the MMAs (the conv of every thread finished before the
        // cluster barrier above, so the staging rows are free)
        if (k + 1 < nblk && warp > 0) {
            for (int e = tid - 32; e < 3 * Lo::NV; e += kThreads - 32) {
                const int r = e % 3, v = e / 3;
                stage[v * kStageRows + r] = stage[v * kStageRows + kT + r];
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kThreads - 32) : "memory");
            load_block(k + 1, tid - 32, kThreads - 32);
        }
        if (k + 1 < nblk && tid < kT && (k + 1) * kT + tid < p.L)
            dt_next = __bfloat162float(gdt[(bi * p.L + (k + 1) * kT + tid) * p.dt_ld + h]);
        // z of this block for the gate, loaded early
        uint4 zr[4];
        {
            const int i = row;
            if (i < len) {
                const uint4* zs = reinterpret_cast<const uint4*>(gz + (bi * p.L + t0 + i) * p.z_ld + (int64_t)h * kP + half * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) zr[v] = zs[v];
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) zr[v] = make_uint4(0, 0, 0, 0);
            }
        }

        // ---- wait for CB, Ys, S
        if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
        fence_after_sync();
        // masked, decayed M = CB * exp(lam_i - lam_j) * delta_j (j <= i), bf16, K-major
        {
            const int i = row;
            float cb[64];
            tmem_ld32(tmem + lane_base + kColCB + half * 64, cb);
            tmem_ld32(tmem + lane_base + kColCB + half * 64 + 32, cb + 32);
            tmem_wait_ld();
            const float li = s_lam[i];
            const bool fac = li > -96.0f;
            const float ui = ex2(li);
            unsigned char* sM = smem + OFF_M;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                float m[8];
                if (fac) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = half * 64 + v * 8 + e;
                        m[e] = (j <= i) ? cb[v * 8 + e] * (ui * s_v[j]) : 0.0f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = half * 64 + v * 8 + e;
                        m[e] = (j <= i) ? cb[v * 8 + e] * ex2(li - s_lam[j]) * s_dl[j] : 0.0f;
                    }
                }
                uint4 u;
                u.x = pack_bf16x2(m[0], m[1]); u.y = pack_bf16x2(m[2], m[3]);
                u.z = pack_bf16x2(m[4], m[5]); u.w = pack_bf16x2(m[6], m[7]);
                *reinterpret_cast<uint4*>(sM + canon_off(i, half * 64 + v * 8, kT)) = u;
            }
        }
        // state update H <- exp(lam_end) H + S, and its bf16 copy for the next block
        {
            float s[32];
            tmem_ld32(tmem + lane_base + kColS + half * 32, s);
            tmem_wait_ld();
            const float aend = ex2(lam_end);
#pragma unroll
            for (int i = 0; i < 32; ++i) H[i] = fmaf(aend, H[i], s[i]);
            unsigned char* sH = smem + OFF_H;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint4 u;
                u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
                u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
                *reinterpret_cast<uint4*>(sH + canon_off(row, half * 32 + 8 * v, kP)) = u;
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_yi = idesc_bf16(128, 64, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColYi, sdesc(aM + kk * 256, 128, 2048), sdesc(aX + kk * 2048, 1024, 128), id_yi, kk > 0);
            mma_commit(bar1);
        }
        if (ok && !mbar_wait_bounded(bar1, par, kWaitLimit)) ok = false;
        fence_after_sync();

        // ---- epilogue: y = Yi + exp(lam_i) Ys + D x', gate, group RMSNorm
        float gt[32];
        {
            const int i = row;
            float yi[32], ys[32];
            tmem_ld32(tmem + lane_base + kColYi + half * 32, yi);
            tmem_ld32(tmem + lane_base + kColYs + half * 32, ys);
            tmem_wait_ld();
            const float el = ex2(s_lam[i]);
            const unsigned char* sX = smem + OFF_X;
            float ss = 0.0f;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                float xv[8], zv[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(sX + canon_off(i, half * 32 + 8 * v, kP)), xv);
                unpack_bf16x8(zr[v], zv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = 8 * v + e;
                    const float y = fmaf(el, ys[c], yi[c]) + Dh * xv[e];
                    const float gg = y * silu_fast(zv[e]);
                    gt[c] = gg;
                    ss = fmaf(gg, gg, ss);
                }
            }
            if constexpr (SPLIT) {
                if (i < len) p.ssp[((bi * p.L + t0 + i) * p.H + h) * 2 + half] = ss;
            } else {
#pragma unroll
                for (int rr = 0; rr < R; ++rr) *cluster.map_shared_rank(s_red + (q * 2 + half) * 128 + i, rr) = ss;
            }
        }
        fence_before_sync();
        // also orders every peer's MMAs on B' and C' of this block before the next block's
        // conv writes into them
        cluster.sync();
        if constexpr (SPLIT) {
            if (row < len) {
                uint4* yo = reinterpret_cast<uint4*>(gy + (bi * p.L + t0 + row) * p.y_ld + (int64_t)h * kP + half * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 u;
                    u.x = pack_bf16x2(gt[8 * v + 0], gt[8 * v + 1]); u.y = pack_bf16x2(gt[8 * v + 2], gt[8 * v + 3]);
                    u.z = pack_bf16x2(gt[8 * v + 4], gt[8 * v + 5]); u.w = pack_bf16x2(gt[8 * v + 6], gt[8 * v + 7]);
                    yo[v] = u;
                }
            }
        } else {
            const int i = row;
            float tot = 0.0f;
#pragma unroll
            for (int rr = 0; rr < 2 * R; ++rr) tot += s_red[rr * 128 + i];
            const float inv = rsqrtf(tot / (float)(R * kP) + p.eps);
            if (i < len) {
                uint4* yo = reinterpret_cast<uint4*>(gy + (bi * p.L + t0 + i) * p.y_ld + (int64_t)h * kP + half * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float* nw = s_nw + half * 32 + 8 * v;
                    uint4 u;
                    u.x = pack_bf16x2(gt[8 * v + 0] * inv * nw[0], gt[8 * v + 1] * inv * nw[1]);
                    u.y = pack_bf16x2(gt[8 * v + 2] * inv * nw[2], gt[8 * v + 3] * inv * nw[3]);
                    u.z = pack_bf16x2(gt[8 * v + 4] * inv * nw[4], gt[8 * v + 5] * inv * nw[5]);
                    u.w = pack_bf16x2(gt[8 * v + 6] * inv * nw[6], gt[8 * v + 7] * inv * nw[7]);
                    yo[v] = u;
                }
            }
        }
    }

    // ---- final states: SSM state of this head, conv taps of the staged channels
    {
        float* fs = p.final_ssm + (bi * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < 32; ++i) fs[(int64_t)(half * 32 + i) * kN + row] = H[i];
    }
    __syncthreads();
    for (int e = tid; e < 3 * SROW; e += kThreads) {
        const int kk = e / SROW, c = e % SROW;
        // staging row len + kk holds the raw input kk - 3 tokens before the end
        ((__nv_bfloat16*)p.final_conv)[(bi * Cc + staged_channel(c)) * 3 + kk] =
            reinterpret_cast<const __nv_bfloat16*>(stage + (c / 8) * kStageRows + len + kk)[c % 8];
    }
    if (!ok && tid == 0) atomicExch(p.status, 1);
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Group RMSNorm of the gated values written by the SPLIT kernel: one warp per
// (batch row, token, group) sums the 2 * (H/G) partial sums of squares, then rescales the
// group's H/G * 64 channels in place.
__global__ void __launch_bounds__(256) norm_finish_kernel(PrefillParams p)
{
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= p.b * p.L * p.G) return;
    const int64_t row = w / p.G;
    const int g = (int)(w % p.G);
    const int rpg = p.H / p.G, gs = rpg * kP;
    const float* sp = p.ssp + (row * p.H + (int64_t)g * rpg) * 2;
    float s = 0.0f;
    for (int k = lane; k < 2 * rpg; k += 32) s += sp[k];
    s = warp_sum(s);
    const float inv = rsqrtf(s / (float)gs + p.eps);
    __nv_bfloat16* y = (__nv_bfloat16*)p.y + row * p.y_ld + (int64_t)g * gs;
    const float* nw = p.norm_w + (int64_t)g * gs;
    for (int c = lane * 8; c < gs; c += 256) {
        float v[8];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(y + c), v);
        uint4 u;
        u.x = pack_bf16x2(v[0] * inv * nw[c + 0], v[1] * inv * nw[c + 1]);
        u.y = pack_bf16x2(v[2] * inv * nw[c + 2], v[3] * inv * nw[c + 3]);
        u.z = pack_bf16x2(v[4] * inv * nw[c + 4], v[5] * inv * nw[c + 5]);
        u.w = pack_bf16x2(v[6] * inv * nw[c + 6], v[7] * inv * nw[c + 7]);
        *reinterpret_cast<uint4*>(y + c) = u;
    }
}

template <int R, bool SPLIT>
cudaError_t launch_r(const PrefillParams& p, cudaStream_t st)
{
    const uint32_t smem = Layout<R>::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(ssd_prefill_tc_kernel<R, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.b * p.H));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        LaunchScope ls("tc_prefill", st);
        e = cudaLaunchKernelEx(&cfg, ssd_prefill_tc_kernel<R, SPLIT>, p);
        if (e != cudaSuccess) return e;
    }
    if (SPLIT && p.L > 0) {
        LaunchScope ls("tc_norm_finish", st);
        const int64_t warps = p.b * p.L * p.G;
        norm_finish_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

bool prefill_tc_supported(int act, int P, int N, int H, int G)
{
    const int r = H / G;
    return act == 1 && P == kP && N == kN && (r == 2 || r == 4 || r == 8 || (r % 8 == 0 && r <= 256));
}

bool prefill_tc_split(int H, int G) { return H / G > 8; }

cudaError_t launch_prefill_tc(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    switch (p.H / p.G) {
    case 2: return launch_r<2, false>(p, stream);
    case 4: return launch_r<4, false>(p, stream);
    case 8: return launch_r<8, false>(p, stream);
    }
    return launch_r<8, true>(p, stream);
}

}  // namespace ssd
