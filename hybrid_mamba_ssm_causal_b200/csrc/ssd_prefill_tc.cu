// ssd_prefill_tc.cu -- the tensor-core (tcgen05) prefill of the SSD mixer for bf16
// activations, head dim 64 and state dim 128.
//
// One kernel does the whole core: causal conv + SiLU, softplus, the chunked SSD scan
// with the state kept on chip, the D skip and the gated group RMSNorm. Each CTA owns one
// head of one batch row and walks the sequence in 128-token blocks, so the state never
// leaves the SM: no chunk states are written to memory and there is no separate state
// pass. The r heads of a group form a thread-block cluster: every CTA convolves a slice
// of the group's B and C channels and copies it into every peer's shared memory (DSMEM
// bulk copies), and the norm's per-token sums of squares are exchanged through DSMEM
// too, so the normalisation over the group's r*64 channels happens in the same pass.
// When the batch has too few heads to fill the GPU, each head is split over PS = 2 CTAs
// that own 32 of its 64 head-dim columns each (the block's C'B'^T is computed by both).
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
// Threads: 512. Thread t owns TMEM lane / row (t % 128) and column quarter (t / 128).
// Head-dim columns owned by a CTA: kP / PS.
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
constexpr int kThreads = 512;
constexpr int kQ = kThreads / 128;    // column slices: thread t owns row t % 128, slice t / 128
constexpr int kTC = kT / kQ;          // token columns of C'B'^T per thread (32)
constexpr int kStageRows = kT + 3;   // 3 halo rows (raw inputs before the block) + the block

constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitLimit = 4000000000LL;  // ~2 s at 2 GHz

// Per-configuration layout. R heads per cluster, PS CTAs per head.
//   shared memory: C', B', M (128x128 bf16 each), x', x'w (128 x PL), H^T (128 x PL),
//   raw staging (8-channel vectors x 131 rows), then small fp32 arrays and the barriers.
//   TMEM columns: C'B'^T [0,128), then Yi, Ys and S^T (PL columns each).
template <int R, int PS>
struct Layout {
    static constexpr int CL = R * PS;                // CTAs per cluster
    static constexpr int PL = kP / PS;               // head-dim columns of one CTA
    static constexpr int PC = PL / kQ;               // head-dim columns per thread
    static constexpr int NS = kN / CL;               // B/C channels convolved by one CTA
    static constexpr int SROW = PL + 2 * NS;         // staged channels per row
    static constexpr int NV = SROW / 8;              // staged 8-channel vectors
    static constexpr uint32_t RBX = (PL / 8) * 128;  // row-block stride of the x', x'w, H^T tiles
    static constexpr uint32_t OFF_C = 0, OFF_B = 32768, OFF_M = 65536, OFF_X = 98304,
                              OFF_XW = OFF_X + 128 * PL * 2, OFF_H = OFF_XW + 128 * PL * 2,
                              OFF_STAGE = OFF_H + 128 * PL * 2;
    static constexpr uint32_t STAGE_BYTES = (uint32_t)kStageRows * SROW * 2;
    static constexpr uint32_t OFF_MISC = OFF_STAGE + ((STAGE_BYTES + 127) / 128) * 128;
    // misc floats
    static constexpr uint32_t F_LAM = 0, F_DL = 256, F_V = 512, F_SCAN = 768, F_RED = 768 + kThreads / 32,
                              F_CW = F_RED + CL * kQ * 128, F_CB = F_CW + SROW * 4, F_NW = F_CB + SROW,
                              F_END = F_NW + PL;
    static constexpr uint32_t OFF_BAR = OFF_MISC + ((F_END * 4 + 15) / 16) * 16;
    static constexpr uint32_t TOTAL = OFF_BAR + 32;   // bar0, bar1, barX, tmem slot
    static constexpr uint32_t kColCB = 0, kColYi = 128, kColYs = 128 + PL, kColS = 128 + 2 * PL;
};

// Inclusive scan over threads 0..127 (warps 0..3 only; named barrier 2).
__device__ __forceinline__ float scan128(float v, float* tot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tot[wid] = v;
    asm volatile("bar.sync 2, 128;" ::: "memory");
    float off = 0.0f;
    for (int w = 0; w < wid; ++w) off += tot[w];
    return v + off;
}

// R heads per cluster, PS CTAs per head (cluster of R * PS CTAs). SPLIT: the group has
// more heads than one cluster holds (H/G > R); each CTA then writes the gated values and
// its per-token sums of squares, and norm_finish_kernel applies the group RMSNorm.
template <int R, int PS, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1) ssd_prefill_tc_kernel(PrefillParams p)
{
    using Lo = Layout<R, PS>;
    constexpr int CL = Lo::CL, PL = Lo::PL, PC = Lo::PC, NS = Lo::NS, SROW = Lo::SROW;
    constexpr uint32_t RBX = Lo::RBX;
    constexpr uint32_t kColCB = Lo::kColCB, kColYi = Lo::kColYi, kColYs = Lo::kColYs, kColS = Lo::kColS;
    extern __shared__ __align__(1024) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int q = (int)cluster.block_rank();            // CTA within the cluster
    const int qh = q / PS, ps = q % PS;                  // head within the cluster, column half
    const int rpg = p.H / p.G;                           // heads per group
    const int ncl = rpg / R;                             // clusters per group
    const int64_t cid = blockIdx.x / CL;                 // (batch row, group, cluster)
    const int64_t bi = cid / ((int64_t)p.G * ncl);
    const int g = (int)((cid / ncl) % p.G);
    const int h = g * rpg + (int)(cid % ncl) * R + qh;
    const int p0 = ps * PL;                              // first head-dim column of this CTA
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & 127, cq = tid >> 7;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

    float* mf = reinterpret_cast<float*>(smem + Lo::OFF_MISC);
    float* s_lam = mf + Lo::F_LAM;     // [2][128] log2-domain inclusive cumsum of delta*A
    float* s_dl = mf + Lo::F_DL;       // [2][128] delta
    float* s_v = mf + Lo::F_V;         // [2][128] column factors of the decay mask
    float* s_scan = mf + Lo::F_SCAN;
    float* s_red = mf + Lo::F_RED;     // [CL][kQ][128] per-(CTA, slice) sums of g^2, pushed by every peer
    float* s_cw = mf + Lo::F_CW;       // [SROW][4] conv taps of the staged channels
    float* s_cb = mf + Lo::F_CB;       // [SROW]
    float* s_nw = mf + Lo::F_NW;       // [PL] norm weights of this CTA's columns
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lo::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::OFF_BAR + 24);
    // stage[v * kStageRows + r]: channels 8v..8v+7 of staged row r (row r = token t0 + r - 3).
    // Vector-major, so threads on consecutive rows read consecutive 16-byte words.
    uint4* stage = reinterpret_cast<uint4*>(smem + Lo::OFF_STAGE);

    const uint32_t s_base = smem_u32(smem);
    const uint32_t aC = s_base + Lo::OFF_C, aB = s_base + Lo::OFF_B, aM = s_base + Lo::OFF_M;
    const uint32_t aX = s_base + Lo::OFF_X, aXW = s_base + Lo::OFF_XW, aH = s_base + Lo::OFF_H;
    const uint32_t bar0 = smem_u32(&bars[0]), bar1 = smem_u32(&bars[1]);
    const uint32_t barX = smem_u32(&bars[2]);   // peers' B'/C' slices have landed

    // channel index (in xBC) of staged column c
    auto staged_channel = [&](int c) -> int64_t {
        if (c < PL) return (int64_t)h * kP + p0 + c;
        if (c < PL + NS) return HP + (int64_t)g * kN + (int64_t)q * NS + (c - PL);
        return HP + GN + (int64_t)g * kN + (int64_t)q * NS + (c - PL - NS);
    };

    // ---- set-up: parameters, initial conv taps, barriers, TMEM, initial state
    if (blockIdx.x == 0 && tid == 0) *p.status = 0;  // this call's status word starts clean
    for (int c = tid; c < SROW; c += kThreads) {
        const int64_t ch = staged_channel(c);
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        s_cw[c * 4 + 0] = w.x; s_cw[c * 4 + 1] = w.y; s_cw[c * 4 + 2] = w.z; s_cw[c * 4 + 3] = w.w;
        s_cb[c] = p.conv_b[ch];
    }
    if (tid < PL) s_nw[tid] = p.norm_w[(int64_t)h * kP + p0 + tid];
    for (int e = tid; e < 3 * SROW; e += kThreads) {
        const int k = e / SROW, c = e % SROW;
        __nv_bfloat16 v = __float2bfloat16_rn(0.0f);
        if (p.init_conv) v = ((const __nv_bfloat16*)p.init_conv)[(bi * Cc + staged_channel(c)) * 3 + k];
        reinterpret_cast<__nv_bfloat16*>(stage + (c / 8) * kStageRows + k)[c % 8] = v;
    }
    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        mbar_init(barX, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    // state H^T[n][p]: thread (n = row, cq) keeps this CTA's columns p0 + [cq*PC, cq*PC + PC)
    float H[PC];
    {
        const float* h0 = p.init_ssm ? p.init_ssm + (bi * p.H + h) * (int64_t)kP * kN : nullptr;
#pragma unroll
        for (int i = 0; i < PC; ++i) H[i] = h0 ? h0[(int64_t)(p0 + cq * PC + i) * kN + row] : 0.0f;
        unsigned char* sH = smem + Lo::OFF_H;
#pragma unroll
        for (int v = 0; v < PC / 8; ++v) {
            uint4 u;
            u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
            u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
            *reinterpret_cast<uint4*>(sH + canon_off(row, cq * PC + 8 * v, PL)) = u;
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
            if (c8 < PL) src = gx + tok * p.x_ld + (int64_t)h * kP + p0 + c8;
            else if (c8 < PL + NS) src = gB + tok * p.B_ld + (int64_t)g * kN + (int64_t)q * NS + (c8 - PL);
            else src = gC + tok * p.C_ld + (int64_t)g * kN + (int64_t)q * NS + (c8 - PL - NS);
            cp_async16(smem_u32(stage + (c8 / 8) * kStageRows + r + 3), src);
        }
        cp_async_commit();
    };

    // delta, its within-block cumsum lam (log2 units) and the column factors of the decay
    // mask for one block, into double-buffer slot `buf`. Threads 0..127 (warps 0..3) only.
    // exp2(lam_i - lam_j) = u_i * v_j with u_i = exp2(lam_i) and v_j = exp2(-lam_j): exact up
    // to rounding while the factors (and v_j times delta_j) stay normal fp32 numbers. lam is
    // non-increasing from <= 0, so for a row i with lam_i > -96 every j <= i has v_j <= 2^96;
    // rows past that decay take exp2 per element. The choice for row i depends on tokens up
    // to i only, so the result stays causal bit for bit.
    auto block_scan = [&](int blen, float dt_in, int buf) {
        float dl = 0.0f, a2 = 0.0f;
        if (tid < blen) {
            dl = softplus(dt_in + bias);
            a2 = dl * A2;
        }
        const float lam = scan128(a2, s_scan);
        s_lam[buf * kT + tid] = lam;
        s_dl[buf * kT + tid] = dl;
        s_v[buf * kT + tid] = (lam > -96.0f) ? ex2(-lam) * dl : 0.0f;
    };

    float dt_next = 0.0f;
    if (nblk > 0) {
        load_block(0, tid, kThreads);
        if (tid < kT) {
            if (tid < p.L) dt_next = __bfloat162float(gdt[(bi * p.L + tid) * p.dt_ld + h]);
            block_scan((int)min((int64_t)kT, p.L), dt_next, 0);
        }
    }
    constexpr uint32_t kSliceBytes = (uint32_t)NS * kT * 2;     // one CTA's B' (or C') slice
    const uint32_t slice_off = (uint32_t)q * kSliceBytes;

    int len = 0;
    for (int64_t k = 0; k < nblk; ++k) {
        const int64_t t0 = k * kT;
        len = (int)min((int64_t)kT, p.L - t0);
        const uint32_t par = (uint32_t)(k & 1);
        const float* lamb = s_lam + (k & 1) * kT;
        const float* dlb = s_dl + (k & 1) * kT;
        const float* vb = s_v + (k & 1) * kT;
        cp_async_wait_all();
        if (tid == 0) mbar_arrive_expect_tx(barX, (uint32_t)(CL - 1) * 2 * kSliceBytes);
        __syncthreads();   // raw rows of this block and its scan are visible to every thread
        const float lam_end = lamb[kT - 1];

        // ---- conv + SiLU of the staged channels: this CTA's x channels -> x' and x'*w;
        //      its slice of B and C -> its own B'/C' slice (sent to the peers below).
        //      Work item (v, i): 8 channels of row i; consecutive threads take consecutive rows.
        {
            unsigned char* sX = smem + Lo::OFF_X;
            unsigned char* sXW = smem + Lo::OFF_XW;
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
                if (c0 < PL) {
                    const float wgt = (i < len) ? ex2(lam_end - lamb[i]) * dlb[i] : 0.0f;
                    uint4 uw;
                    uw.x = pack_bf16x2(o[0] * wgt, o[1] * wgt); uw.y = pack_bf16x2(o[2] * wgt, o[3] * wgt);
                    uw.z = pack_bf16x2(o[4] * wgt, o[5] * wgt); uw.w = pack_bf16x2(o[6] * wgt, o[7] * wgt);
                    *reinterpret_cast<uint4*>(sX + canon_off(i, c0, PL)) = u8;
                    *reinterpret_cast<uint4*>(sXW + canon_off(i, c0, PL)) = uw;
                } else {
                    const bool isC = c0 >= PL + NS;
                    const int n0 = q * NS + (isC ? c0 - PL - NS : c0 - PL);
                    *reinterpret_cast<uint4*>(smem + (isC ? Lo::OFF_C : Lo::OFF_B) + canon_koff(i, n0, kT)) = u8;
                }
            }
        }
        fence_async_smem();
        __syncthreads();   // x', x'w and this CTA's B'/C' slice are complete

        // ---- send this CTA's slices to the peers, wait for theirs, then the MMAs on C'B'^T,
        //      C'H^T and B'^T(x'w). B'/C' have their column blocks outermost (K-major: SBO 128,
        //      LBO 2048; B' as the MN-major A of B'^T: SBO 2048, LBO 128).
        if (tid == 0) {
#pragma unroll
            for (int rr = 0; rr < CL; ++rr) {
                if (rr == q) continue;
                const uint32_t mb = cluster_map(barX, (uint32_t)rr);
                bulk_copy_to_peer(cluster_map(aB + slice_off, (uint32_t)rr), aB + slice_off, kSliceBytes, mb);
                bulk_copy_to_peer(cluster_map(aC + slice_off, (uint32_t)rr), aC + slice_off, kSliceBytes, mb);
            }
            if (ok && !mbar_wait_bounded(barX, par, kWaitLimit)) ok = false;
            fence_after_sync();
            const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_ys = idesc_bf16(128, PL, 0, 1);
            const uint32_t id_s = idesc_bf16(128, PL, 1, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColCB, sdesc(aC + kk * 4096, 2048, 128), sdesc(aB + kk * 4096, 2048, 128), id_cb, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColYs, sdesc(aC + kk * 4096, 2048, 128), sdesc(aH + kk * 2 * RBX, RBX, 128), id_ys, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColS, sdesc(aB + kk * 256, 128, 2048), sdesc(aXW + kk * 2 * RBX, RBX, 128), id_s, kk > 0);
            mma_commit(bar0);
        }
        // raw data of the next block: warps 1.. keep its three halo rows, then start its
        // loads, while thread 0 sends the slices and issues the MMAs (the conv of every
        // thread finished before the barrier above, so the staging rows are free)
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
        uint4 zr[PC / 8];
        {
            const int i = row;
            if (i < len) {
                const uint4* zs = reinterpret_cast<const uint4*>(gz + (bi * p.L + t0 + i) * p.z_ld + (int64_t)h * kP + p0 + cq * PC);
#pragma unroll
                for (int v = 0; v < PC / 8; ++v) zr[v] = zs[v];
            } else {
#pragma unroll
                for (int v = 0; v < PC / 8; ++v) zr[v] = make_uint4(0, 0, 0, 0);
            }
        }

        // ---- wait for CB, Ys, S
        if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
        fence_after_sync();
        // masked, decayed M = CB * exp(lam_i - lam_j) * delta_j (j <= i), bf16, K-major
        {
            const int i = row;
            float cb[kTC];
            tmem_ld32(tmem + lane_base + kColCB + cq * kTC, cb);
            tmem_wait_ld();
            const float li = lamb[i];
            const bool fac = li > -96.0f;
            const float ui = ex2(li);
            unsigned char* sM = smem + Lo::OFF_M;
#pragma unroll
            for (int v = 0; v < kTC / 8; ++v) {
                float m[8];
                if (fac) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = cq * kTC + v * 8 + e;
                        m[e] = (j <= i) ? cb[v * 8 + e] * (ui * vb[j]) : 0.0f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = cq * kTC + v * 8 + e;
                        m[e] = (j <= i) ? cb[v * 8 + e] * ex2(li - lamb[j]) * dlb[j] : 0.0f;
                    }
                }
                uint4 u;
                u.x = pack_bf16x2(m[0], m[1]); u.y = pack_bf16x2(m[2], m[3]);
                u.z = pack_bf16x2(m[4], m[5]); u.w = pack_bf16x2(m[6], m[7]);
                *reinterpret_cast<uint4*>(sM + canon_off(i, cq * kTC + v * 8, kT)) = u;
            }
        }
        // state update H <- exp(lam_end) H + S, and its bf16 copy for the next block
        {
            float s_[PC];
            tmem_ld_cols<PC>(tmem + lane_base + kColS + cq * PC, s_);
            tmem_wait_ld();
            const float aend = ex2(lam_end);
#pragma unroll
            for (int i = 0; i < PC; ++i) H[i] = fmaf(aend, H[i], s_[i]);
            unsigned char* sH = smem + Lo::OFF_H;
#pragma unroll
            for (int v = 0; v < PC / 8; ++v) {
                uint4 u;
                u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
                u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
                *reinterpret_cast<uint4*>(sH + canon_off(row, cq * PC + 8 * v, PL)) = u;
            }
        }
        fence_async_smem();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_yi = idesc_bf16(128, PL, 0, 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kColYi, sdesc(aM + kk * 256, 128, 2048), sdesc(aX + kk * 2 * RBX, RBX, 128), id_yi, kk > 0);
            mma_commit(bar1);
        }
        if (ok && !mbar_wait_bounded(bar1, par, kWaitLimit)) ok = false;
        fence_after_sync();

        // ---- epilogue: y = Yi + exp(lam_i) Ys + D x', gate, group RMSNorm
        float gt[PC];
        {
            const int i = row;
            float yi[PC], ys[PC];
            tmem_ld_cols<PC>(tmem + lane_base + kColYi + cq * PC, yi);
            tmem_ld_cols<PC>(tmem + lane_base + kColYs + cq * PC, ys);
            tmem_wait_ld();
            const float el = ex2(lamb[i]);
            const unsigned char* sX = smem + Lo::OFF_X;
            float ss = 0.0f;
#pragma unroll
            for (int v = 0; v < PC / 8; ++v) {
                float xv[8], zv[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(sX + canon_off(i, cq * PC + 8 * v, PL)), xv);
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
                if (i < len) p.ssp[((bi * p.L + t0 + i) * p.H + h) * (PS * kQ) + ps * kQ + cq] = ss;
            } else {
#pragma unroll
                for (int rr = 0; rr < CL; ++rr) *cluster.map_shared_rank(s_red + (q * kQ + cq) * 128 + i, rr) = ss;
            }
        }
        // delta and lam of the next block (its dt was loaded above)
        if (k + 1 < nblk && tid < kT) block_scan((int)min((int64_t)kT, p.L - (k + 1) * kT), dt_next, (int)((k + 1) & 1));
        fence_before_sync();
        // also orders every peer's MMAs on B' and C' of this block before the next block's
        // slices are copied into them
        cluster.sync();
        if (row < len) {
            float scale = 1.0f;
            if constexpr (!SPLIT) {
                float tot = 0.0f;
#pragma unroll
                for (int rr = 0; rr < kQ * CL; ++rr) tot += s_red[rr * 128 + row];
                scale = rsqrtf(tot / (float)(R * kP) + p.eps);
            }
            uint4* yo = reinterpret_cast<uint4*>(gy + (bi * p.L + t0 + row) * p.y_ld + (int64_t)h * kP + p0 + cq * PC);
#pragma unroll
            for (int v = 0; v < PC / 8; ++v) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = SPLIT ? gt[8 * v + e] : gt[8 * v + e] * scale * s_nw[cq * PC + 8 * v + e];
                uint4 u;
                u.x = pack_bf16x2(o[0], o[1]); u.y = pack_bf16x2(o[2], o[3]);
                u.z = pack_bf16x2(o[4], o[5]); u.w = pack_bf16x2(o[6], o[7]);
                yo[v] = u;
            }
        }
    }

    // ---- final states: SSM state of this CTA's columns, conv taps of the staged channels
    {
        float* fs = p.final_ssm + (bi * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < PC; ++i) fs[(int64_t)(p0 + cq * PC + i) * kN + row] = H[i];
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
    const float* sp = p.ssp + (row * p.H + (int64_t)g * rpg) * kQ;
    float s = 0.0f;
    for (int k = lane; k < kQ * rpg; k += 32) s += sp[k];
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

template <int R, int PS, bool SPLIT>
cudaError_t launch_r(const PrefillParams& p, cudaStream_t st)
{
    using Lo = Layout<R, PS>;
    const uint32_t smem = Lo::TOTAL;
    cudaError_t e = cudaFuncSetAttribute(ssd_prefill_tc_kernel<R, PS, SPLIT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.b * p.H * PS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Lo::CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        LaunchScope ls("tc_prefill", st);
        e = cudaLaunchKernelEx(&cfg, ssd_prefill_tc_kernel<R, PS, SPLIT>, p);
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
    return act == 1 && P == kP && N == kN && (r == 2 || (r % 4 == 0 && r <= 256));
}

bool prefill_tc_split(int H, int G) { return H / G > 4; }

int prefill_tc_partials_per_head() { return kQ; }

// Cluster shapes. A cluster of 8 one-CTA-per-SM CTAs must fit inside one GPC, and at most
// 15 such clusters are resident on a B200, against 37 clusters of 4: so groups of up to
// 4 heads run as one cluster per group (fused norm), and wider groups run as clusters of
// 4 heads with the norm finished by norm_finish_kernel. The head-dim split (PS = 2) is
// kept for shapes whose clusters stay small; it doubles CTAs per cluster, so it is only
// used for groups of 2 heads on batches too small to fill the GPU.
cudaError_t launch_prefill_tc(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    switch (p.H / p.G) {
    case 2: return (p.b * p.H <= 148) ? launch_r<2, 2, false>(p, stream) : launch_r<2, 1, false>(p, stream);
    case 4: return launch_r<4, 1, false>(p, stream);
    }
    return launch_r<4, 1, true>(p, stream);
}

}  // namespace ssd
