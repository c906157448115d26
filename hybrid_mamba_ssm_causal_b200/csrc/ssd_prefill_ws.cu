// ssd_prefill_ws.cu -- warp-specialised, software-pipelined tensor-core prefill of the SSD
// mixer (bf16 activations, head dim 64, state dim 128).
//
// Same arithmetic as one block of the chunked SSD decomposition (Modalities PR #459,
// ssd.py notes on the chunk-parallel block decomposition) with the state kept on chip:
// per 128-token block of one head,
//   lam_i = inclusive sum of delta*A (log2 units), CB = C' B'^T, Ys = C' H^T,
//   S^T = B'^T (x' w) with w_j = exp(lam_end - lam_j) delta_j,
//   M_ij = CB_ij exp(lam_i - lam_j) delta_j (j <= i), Yi = M x',
//   y = Yi + exp(lam_i) Ys + D x',  g = y SiLU(z),  out = g / rms_group(g) * norm_w,
//   H <- exp(lam_end) H + S.
// Each CTA owns one head of one sequence; the heads of a cluster share the B/C conv (each
// CTA convolves a slice and bulk-copies it into every peer) and, when the cluster holds the
// whole group, the norm's per-token sums of squares (st.async into every peer).
//
// Data movement: the raw x, B and C rows of a block (with the 3-token conv halo) arrive by
// TMA, one box per kind of channel; z is read and y written through 128-byte-swizzled TMA
// tiles; the decay-masked M goes from registers into TMEM and feeds M x' as the TMEM
// A operand.
//
// Roles (512 threads):
//   producer warps 0..7  : for block k, the conv + SiLU of this CTA's B'/C' slice, then one
//                          duty per warp (warp 1 the TMA refill of the next raw B/C rows,
//                          warps 2.. one slice copy each to a peer), the conv + SiLU of x' and
//                          x'w, and (thread 0) the MMAs C'B'^T, C'H^T and B'^T(x'w) once the
//                          peers' slices are in; warps 4..7 then the softplus + cumsum of
//                          block k+1;
//   consumer warps 8..15 : for block k-1 meanwhile: the masked decay product M, the state
//                          update, (thread 256) the MMA M x', the epilogue, and the group
//                          norm of block k-2.
// Variants: packed variable-length sequences on state slots (a CTA reads its sequence's
// rows, length and slot from device arrays), and STATE_ONLY (final states and decay only).
// Hand-offs use mbarriers (all waits bounded):
//   bar0   MMA1-3 of a block done (tensor-core commit)     bar1  MMA4 done
//   barX   the peers' B'/C' slices of a block have landed (bulk-copy transaction bytes)
//   barP   producer: this block's x', x'w and cumsum are in shared memory (arrived just
//          before MMA1-3 are issued)
//   barC   consumer: C'B'^T and S^T read from TMEM, H^T of the next block written
//   barE2  consumer: a block's x' and cumsum buffers are free again (2 slots by parity)
//   barF2  every CTA of the cluster: its MMA1-3 of a block are done (2 slots; one arrival per
//          CTA, multicast by its tensor-core commit). Once all have arrived, no CTA reads its
//          B'/C' of that block any more and every slice copy of it has landed, so the next
//          block's slice may be written and sent.
//   barN3  the sums of squares of a block from every CTA of the cluster have landed
//          (st.async transaction bytes; 3 slots)
//   barTB, barTX, barZ: TMA of the raw B/C rows, the raw x rows, the z tile
// Barriers waited two blocks back use two slots, so a waiter never meets a barrier that
// has moved two phases past the one it expects. The group norm of block k is finished one
// block late (its gated values wait in TMEM), while the MMA of block k+1 runs; a peer can
// be at most two blocks ahead of that finish, hence three slots for the sums of squares.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <type_traits>

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
constexpr int kProd = 256;    // producer threads (warps 0..7)
// Raw staging of one 8-channel vector: tokens t0-8 .. t0+127 of a block, so rows 5..7 hold
// the conv halo and rows 8..135 the block's tokens; 2176 bytes, a multiple of 128, so every
// vector starts 128-byte aligned. One TMA box fills several consecutive vectors.
constexpr int kStageRows = 136, kStageTok = 8;
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitLimit = 4000000000LL;  // ~2 s at 2 GHz

// TMEM columns: C'B'^T, Ys (two slots), S^T, Yi, the gated values of a block awaiting its norm,
// and the masked decay matrix M (bf16 pairs; the A operand of M x')
constexpr uint32_t kColCB = 0, kColYs0 = 128, kColS = 256, kColYi = 320, kColG = 384, kColM = 448;

// named barriers
constexpr int kBarProd = 1, kBarCons = 2, kBarScan = 3;

template <int R>
struct WsLayout {
    static constexpr int NS = kN / R;                // B/C channels convolved by one CTA
    static constexpr int SROW = kP + 2 * NS;
    // z and y tiles of a block: [128 tokens][64 channels] bf16, 16-byte chunks swizzled by token % 8
    static constexpr uint32_t OFF_C = 0, OFF_B = 32768, OFF_Z = 65536, OFF_Y = 81920, OFF_X = 98304,   // x' [2]
                              OFF_XW = OFF_X + 2 * 16384, OFF_H = OFF_XW + 16384, OFF_STAGE = OFF_H + 16384;
    static constexpr uint32_t STAGE_BYTES = (uint32_t)kStageRows * SROW * 2;   // SROW/8 vectors
    static constexpr uint32_t OFF_MISC = OFF_STAGE + ((STAGE_BYTES + 127) / 128) * 128;
    // fp32 arrays: lam, delta, v (2 slots each), scan scratch, sums of squares [3][R][2][128],
    // conv taps and biases of the staged channels, norm weights
    static constexpr uint32_t F_LAM = 0, F_DL = 256, F_V = 512, F_SCAN = 768, F_RED = 784,
                              F_CW = F_RED + 3 * R * 2 * 128, F_CB = F_CW + SROW * 4, F_NW = F_CB + SROW,
                              F_END = F_NW + kP;
    static constexpr uint32_t OFF_BAR = OFF_MISC + ((F_END * 4 + 15) / 16) * 16;
    static constexpr int NBAR = 15;  // bar0 bar1 barX barP barC barE2[2] barF2[2] barN3[3] barTB barTX barZ
    static constexpr uint32_t OFF_TSLOT = OFF_BAR + NBAR * 8;
    static constexpr uint32_t TOTAL = OFF_TSLOT + 16;
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// 4-byte store into a peer's shared memory that completes 4 transaction bytes on the
// peer's mbarrier (both shared::cluster addresses).
__device__ __forceinline__ void st_async_f32(uint32_t dst_cluster, float v, uint32_t mbar_cluster)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(dst_cluster),
                 "r"(__float_as_uint(v)), "r"(mbar_cluster)
                 : "memory");
}

// Bounded wait whose acquire covers cluster scope (peers' arrivals and DSMEM stores).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t mbar, uint32_t parity, long long limit)
{
    const long long t0 = clock64();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// Inclusive scan over the 128 threads of warps 4..7 (named barrier kBarScan).
__device__ __forceinline__ float scan128(float v, float* tot)
{
    const int lane = threadIdx.x & 31, wid = (threadIdx.x >> 5) - 4;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) tot[wid] = v;
    named_sync(kBarScan, 128);
    float off = 0.0f;
    for (int w = 0; w < wid; ++w) off += tot[w];
    return v + off;
}

// Tensor maps of x, B and C viewed as [b][vector][token][8 channels] (bf16; a vector is 8
// consecutive channels), boxes of 136 tokens x several vectors; of z and y as [b][L][channels],
// boxes of 64 channels x 128 tokens with 128-byte swizzling.
struct WsMaps {
    CUtensorMap x, B, C, z, y;
};

// STATE_ONLY: the state-only pass (final states and decay of a prefill, no output rows): the
// conv of x and B, B'^T(x'w) and the state recurrence; C's raw rows only for the conv state.
template <int R, bool SPLIT, bool STATE_ONLY>
__global__ void __launch_bounds__(kThreads, 1) ssd_prefill_ws_kernel(PrefillParams p, const __grid_constant__ WsMaps maps)
{
    using Lo = WsLayout<R>;
    constexpr int NS = Lo::NS, SROW = Lo::SROW;
    extern __shared__ __align__(1024) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int q = (int)cluster.block_rank();
    const int rpg = p.H / p.G;
    const int ncl = rpg / R;
    const int64_t cid = blockIdx.x / R;
    const int64_t bi = cid / ((int64_t)p.G * ncl);
    const int g = (int)((cid / ncl) % p.G);
    const int h = g * rpg + (int)(cid % ncl) * R + q;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    // this CTA's sequence: its first token row, length, state slot, and whether it starts from
    // the states given (packed variable-length calls read them from their slot arrays)
    const bool varlen = p.cu_seqlens != nullptr;
    const int64_t row0 = varlen ? (int64_t)p.cu_seqlens[bi] : bi * p.L;
    const int64_t seqlen = varlen ? (int64_t)p.cu_seqlens[bi + 1] - row0 : p.L;
    const int64_t sidx = varlen && p.slot_idx ? (int64_t)p.slot_idx[bi] : bi;
    const bool cont = varlen ? (!p.has_init || p.has_init[bi] != 0) : true;
    const bool init_ssm = cont && p.init_ssm != nullptr, init_conv = cont && p.init_conv != nullptr;
    // coordinates of token 0 in the tensor maps (token, sequence)
    const int tmap_t0 = varlen ? (int)row0 : 0, tmap_b = varlen ? 0 : (int)bi;

    float* mf = reinterpret_cast<float*>(smem + Lo::OFF_MISC);
    float* s_lam = mf + Lo::F_LAM;
    float* s_dl = mf + Lo::F_DL;
    float* s_v = mf + Lo::F_V;
    float* s_scan = mf + Lo::F_SCAN;
    float* s_red = mf + Lo::F_RED;     // [3 slots][R CTAs][2 halves][128 rows]
    float* s_cw = mf + Lo::F_CW;
    float* s_cb = mf + Lo::F_CB;
    float* s_nw = mf + Lo::F_NW;
    uint4* stage = reinterpret_cast<uint4*>(smem + Lo::OFF_STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lo::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::OFF_TSLOT);

    const uint32_t s_base = smem_u32(smem);
    const uint32_t aC = s_base + Lo::OFF_C, aB = s_base + Lo::OFF_B, aZ = s_base + Lo::OFF_Z, aY = s_base + Lo::OFF_Y;
    const uint32_t aX = s_base + Lo::OFF_X, aXW = s_base + Lo::OFF_XW, aH = s_base + Lo::OFF_H;
    const uint32_t bar0 = smem_u32(&bars[0]), bar1 = smem_u32(&bars[1]), barX = smem_u32(&bars[2]);
    const uint32_t barP = smem_u32(&bars[3]), barC = smem_u32(&bars[4]);
    const uint32_t barE2 = smem_u32(&bars[5]), barF2 = smem_u32(&bars[7]), barN3 = smem_u32(&bars[9]);
    const uint32_t barTB = smem_u32(&bars[12]), barTX = smem_u32(&bars[13]);   // raw B/C rows, raw x rows
    const uint32_t barZ = smem_u32(&bars[14]);                                      // z tile

    auto staged_channel = [&](int c) -> int64_t {
        if (c < kP) return (int64_t)h * kP + c;
        if (c < kP + NS) return HP + (int64_t)g * kN + (int64_t)q * NS + (c - kP);
        return HP + GN + (int64_t)g * kN + (int64_t)q * NS + (c - kP - NS);
    };

    // ---- set-up
    // the swizzled TMA tiles need a 1024-byte aligned base; every CTA sees the same base, so
    // all of them leave here together (before any barrier) if it is not
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_device_status(p.status, kDevSmemMisaligned);
        return;
    }
    for (int c = tid; c < SROW; c += kThreads) {
        const int64_t ch = staged_channel(c);
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        float* cw = s_cw + (c / 2) * 8 + (c % 2);   // taps of channel pairs: [pair][tap][2]
        cw[0] = w.x; cw[2] = w.y; cw[4] = w.z; cw[6] = w.w;
        s_cb[c] = p.conv_b[ch];
    }
    if (!STATE_ONLY && tid < kP) s_nw[tid] = p.norm_w[(int64_t)h * kP + tid];
    if (tid == 0) {
        mbar_init(bar0, 1);
        mbar_init(bar1, 1);
        mbar_init(barX, 1);
        mbar_init(barP, 1);
        mbar_init(barC, 1);
        mbar_init(barE2, 1);
        mbar_init(barE2 + 8, 1);
        mbar_init(barF2, R);
        mbar_init(barF2 + 8, R);
        mbar_init(barN3, 1);
        mbar_init(barN3 + 8, 1);
        mbar_init(barN3 + 16, 1);
        mbar_init(barTB, 1);
        mbar_init(barTX, 1);
        mbar_init(barZ, 1);
        fence_mbar_init();
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.B);
        prefetch_tmap(&maps.C);
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);

    // consumer state: thread (n = row, half) keeps H^T[n][half*32 .. half*32+32) in fp32
    const bool consumer = tid >= kProd;
    const int crow = tid & 127, chalf = (tid - kProd) >> 7;   // consumer row and column half
    float H[32];
    if (consumer) {
        const float* h0 = init_ssm ? p.init_ssm + (sidx * p.H + h) * (int64_t)kP * kN : nullptr;
#pragma unroll
        for (int i = 0; i < 32; ++i) H[i] = h0 ? h0[(int64_t)(chalf * 32 + i) * kN + crow] : 0.0f;
        unsigned char* sH = smem + Lo::OFF_H;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
            u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
            *reinterpret_cast<uint4*>(sH + canon_off(crow, chalf * 32 + 8 * v, kP)) = u;
        }
        fence_async_smem();
    }
    fence_before_sync();
    __syncthreads();
    cluster.sync();   // every peer's barriers are initialised before any remote arrival or copy
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const float A2 = p.A[h] * 1.4426950408889634f;
    const float Dh = STATE_ONLY ? 0.0f : p.D[h];
    const float bias = p.dt_bias[h];
    bool ok = true;

    const int64_t nblk = (seqlen + kT - 1) / kT;
    const __nv_bfloat16* gdt = (const __nv_bfloat16*)p.dt;
    constexpr uint32_t kSliceBytes = (uint32_t)NS * kT * 2;
    const uint32_t slice_off = (uint32_t)q * kSliceBytes;
    auto blen = [&](int64_t k) { return (int)min((int64_t)kT, seqlen - k * kT); };

    if (!consumer) {
        // =========================== producer (warps 0..7) ===========================
        constexpr int kVX = kP / 8, kVBC = 2 * NS / 8;   // x vectors, then this CTA's B and C vectors
        // raw rows t0-8 .. t0+127 of block kb (TMA): one box for the head's x vectors on barTX, one
        // each for this CTA's B and C vectors on barTB; rows outside the sequence read as zeros
        auto load_bc = [&](int64_t kb) {
            mbar_arrive_expect_tx(barTB, (uint32_t)kVBC * kStageRows * 16);
            const int t0 = tmap_t0 + (int)(kb * kT) - kStageTok, vb = (g * kN + q * NS) / 8;
            tma_load_4d(smem_u32(stage + kVX * kStageRows), &maps.B, 0, t0, vb, tmap_b, barTB);
            tma_load_4d(smem_u32(stage + (kVX + NS / 8) * kStageRows), &maps.C, 0, t0, vb, tmap_b, barTB);
        };
        auto load_x = [&](int64_t kb) {
            mbar_arrive_expect_tx(barTX, (uint32_t)kVX * kStageRows * 16);
            tma_load_4d(smem_u32(stage), &maps.x, 0, tmap_t0 + (int)(kb * kT) - kStageTok, h * kVX, tmap_b, barTX);
        };
        // softplus and cumsum of block kb into its slot (warps 4..7, token tid - 128), then dt of
        // block kb + 1, a whole block ahead of its use
        float dt_next = 0.0f;
        const int tok = tid - 128;
        auto scan_block = [&](int64_t kb) {
            const int slb = (int)(kb & 1);
            float dl = 0.0f, a2 = 0.0f;
            if (tok < blen(kb)) {
                dl = softplus(dt_next + bias);
                a2 = dl * A2;
            }
            if (kb + 1 < nblk && (kb + 1) * kT + tok < seqlen)
                dt_next = __bfloat162float(gdt[(row0 + (kb + 1) * kT + tok) * p.dt_ld + h]);
            const float lam = scan128(a2, s_scan);
            s_lam[slb * kT + tok] = lam;
            s_dl[slb * kT + tok] = dl;
            // exp2(lam_i - lam_j) = exp2(lam_i) * exp2(-lam_j) while every factor stays a
            // normal fp32 number (rows with lam_i > -96); chosen per row from its past only
            s_v[slb * kT + tok] = (lam > -96.0f) ? ex2(-lam) * dl : 0.0f;
        };
        if (nblk > 0) {
            if (tid == 0) {
                load_bc(0);
                load_x(0);
            }
            if (warp >= 4) {
                if (tok < seqlen) dt_next = __bfloat162float(gdt[(row0 + tok) * p.dt_ld + h]);
                scan_block(0);
            }
        }
        // the three rows before the sequence hold the initial conv state (zeros without one), not
        // the TMA's fill or a neighbouring packed sequence: written once block 0's rows have landed
        if (nblk == 0 || init_conv || varlen) {
            if (nblk > 0) {
                if (ok && !mbar_wait_bounded(barTB, 0, kWaitLimit)) ok = false;
                if (ok && !mbar_wait_bounded(barTX, 0, kWaitLimit)) ok = false;
            }
            for (int e = tid; e < 3 * SROW; e += kProd) {
                const int kk = e / SROW, c = e % SROW;
                __nv_bfloat16 v = __float2bfloat16_rn(0.0f);
                if (init_conv) v = ((const __nv_bfloat16*)p.init_conv)[(sidx * Cc + staged_channel(c)) * 3 + kk];
                reinterpret_cast<__nv_bfloat16*>(stage + (c / 8) * kStageRows + kStageTok - 3 + kk)[c % 8] = v;
            }
        }
        for (int64_t k = 0; k < nblk; ++k) {
            const int len = blen(k);
            const int sl = (int)(k & 1);
            // buffers of this block: x'[sl] was last read by the consumer in block k-2, B'/C'/x'w
            // by the MMAs of block k-1. Every CTA of the cluster has finished those: this CTA's
            // B'/C' are no longer read, its own copies of block k-1's slice have landed in every
            // peer (a peer's MMAs start only once they have), and every peer's B'/C' may take
            // this block's slice. The cumsum of this block is already in its slot.
            if (tid == 0) {
                if (k >= 1 && ok &&
                    !mbar_wait_cluster(barF2 + 8 * (uint32_t)((k - 1) & 1), (uint32_t)(((k - 1) >> 1) & 1), kWaitLimit))
                    ok = false;
                if (k >= 2 && ok && !mbar_wait_bounded(barE2 + 8 * sl, (uint32_t)(((k - 2) >> 1) & 1), kWaitLimit)) ok = false;
                mbar_arrive_expect_tx(barX, (uint32_t)(R - 1) * (STATE_ONLY ? 1 : 2) * kSliceBytes);
            }
            // this block's raw B/C rows (its x rows may still be in flight)
            if (ok && !mbar_wait_bounded(barTB, (uint32_t)(k & 1), kWaitLimit)) ok = false;
            named_sync(kBarProd, kProd);
            const float* lamb = s_lam + sl * kT;
            const float* dlb = s_dl + sl * kT;
            const float lam_end = lamb[kT - 1];
            // conv + SiLU of the staged 8-channel vectors [vbeg, vbeg + VC): x' and x'w of this
            // head, or this CTA's slice of B' and C'. TPV threads per vector, each taking rows
            // i = t % TPV + TPV m, so a warp reads consecutive staged rows and writes
            // consecutive canonical rows (conflict-free); a thread keeps its taps in registers.
            auto conv_vectors = [&](auto vbeg_c, auto vc_c) {
                constexpr int VBEG = decltype(vbeg_c)::value, VC = decltype(vc_c)::value;
                constexpr int TPV = kProd / VC;
                static_assert(kProd % VC == 0 && kT % (2 * TPV) == 0, "conv work split");
                unsigned char* sX = smem + Lo::OFF_X + sl * 16384;
                unsigned char* sXW = smem + Lo::OFF_XW;
                const int v = VBEG + tid / TPV;
                const int c0 = v * 8;
                float2 wr[4][4], br[4];
                {
                    const float2* cw2 = reinterpret_cast<const float2*>(s_cw) + (c0 / 2) * 4;
                    const float2* cb2 = reinterpret_cast<const float2*>(s_cb) + c0 / 2;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        br[j] = cb2[j];
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) wr[j][kk] = cw2[j * 4 + kk];
                    }
                }
                const bool is_x = c0 < kP;
                const bool isC = c0 >= kP + NS;
                const int n0 = q * NS + (isC ? c0 - kP - NS : c0 - kP);
                unsigned char* dstBC = smem + (isC ? Lo::OFF_C : Lo::OFF_B);
#pragma unroll 1
                for (int m = 0; m < kT / TPV; m += 2) {
                    int ii[2];
                    uint4 raw[2][4];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        ii[u] = (tid % TPV) + TPV * (m + u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) raw[u][kk] = stage[v * kStageRows + kStageTok - 3 + ii[u] + kk];
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int i = ii[u];
                        float2 o[4];
                        if (i < len) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {   // channel pair (c0 + 2j, c0 + 2j + 1)
                                float2 vv = fma2(wr[j][0], bf2_to_f2((&raw[u][0].x)[j]), br[j]);
                                vv = fma2(wr[j][1], bf2_to_f2((&raw[u][1].x)[j]), vv);
                                vv = fma2(wr[j][2], bf2_to_f2((&raw[u][2].x)[j]), vv);
                                vv = fma2(wr[j][3], bf2_to_f2((&raw[u][3].x)[j]), vv);
                                o[j] = silu2(vv);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[j] = make_float2(0.0f, 0.0f);
                        }
                        const uint4 u8 = make_uint4(pack_f2(o[0]), pack_f2(o[1]), pack_f2(o[2]), pack_f2(o[3]));
                        if (is_x) {
                            const float2 wgt = splat2((i < len) ? ex2(lam_end - lamb[i]) * dlb[i] : 0.0f);
                            const uint4 uw = make_uint4(pack_f2(mul2(o[0], wgt)), pack_f2(mul2(o[1], wgt)),
                                                        pack_f2(mul2(o[2], wgt)), pack_f2(mul2(o[3], wgt)));
                            *reinterpret_cast<uint4*>(sX + canon_off(i, c0, kP)) = u8;
                            *reinterpret_cast<uint4*>(sXW + canon_off(i, c0, kP)) = uw;
                        } else {
                            *reinterpret_cast<uint4*>(dstBC + canon_koff(i, n0, kT)) = u8;
                        }
                    }
                }
            };
            // this CTA's slice of B' and C' first, so its copies to the peers overlap the x' conv
            conv_vectors(std::integral_constant<int, kVX>{}, std::integral_constant<int, STATE_ONLY ? NS / 8 : kVBC>{});
            fence_async_smem();
            named_sync(kBarProd, kProd);
            // one duty per warp (lane 0), so that none lags the x' conv by more than one TMA or
            // bulk-copy issue: warp 1 refills the raw B/C rows (these are consumed), warps 2.. each
            // send one copy of this CTA's slice of B'/C' to a peer
            if ((tid & 31) == 0) {
                if (warp == 1) {
                    if (k + 1 < nblk) load_bc(k + 1);
                } else if (warp >= 2 && warp - 2 < (STATE_ONLY ? 1 : 2) * (R - 1)) {
                    const int idx = warp - 2, nm = STATE_ONLY ? 1 : 2;   // matrices sent (B, or B and C)
                    const uint32_t rr = (uint32_t)((q + 1 + idx / nm) % R);
                    const uint32_t src = (idx % nm ? aC : aB) + slice_off;
                    bulk_copy_to_peer(cluster_map(src, rr), src, kSliceBytes, cluster_map(barX, rr));
                }
            }
            // this block's raw x rows (the next block's B/C rows may be in flight)
            if (ok && !mbar_wait_bounded(barTX, (uint32_t)(k & 1), kWaitLimit)) ok = false;
            conv_vectors(std::integral_constant<int, 0>{}, std::integral_constant<int, kVX>{});
            fence_async_smem();
            named_sync(kBarProd, kProd);
            if (tid == 0) {
                if (ok && !mbar_wait_bounded(barX, (uint32_t)(k & 1), kWaitLimit)) ok = false;
                // the consumer has read C'B'^T and S^T of block k-1 and written H^T for this block
                if (k >= 1 && ok && !mbar_wait_bounded(barC, (uint32_t)((k - 1) & 1), kWaitLimit)) ok = false;
                mbar_arrive_local(barP);   // this block's cumsum and x' are in place
                fence_after_sync();
                const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
                const uint32_t id_ys = idesc_bf16(128, 64, 0, 1);
                const uint32_t id_s = idesc_bf16(128, 64, 1, 1);
                const uint32_t colYs = kColYs0 + 64 * (uint32_t)sl;
                if constexpr (!STATE_ONLY) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + kColCB, sdesc(aC + kk * 4096, 2048, 128), sdesc(aB + kk * 4096, 2048, 128), id_cb, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + colYs, sdesc(aC + kk * 4096, 2048, 128), sdesc(aH + kk * 2048, 1024, 128), id_ys, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + kColS, sdesc(aB + kk * 256, 128, 2048), sdesc(aXW + kk * 2048, 1024, 128), id_s, kk > 0);
                mma_commit(bar0);
                // once these MMAs are done, this CTA's B'/C' may be overwritten: every peer is told
                mma_commit_cluster(barF2 + 8 * (uint32_t)sl, (uint16_t)((1u << R) - 1));
            }
            // while thread 0 issues the MMAs: x raw rows of the next block (thread 32) and its
            // softplus and cumsum (warps 4..7, once the consumer has released that slot in block k-1)
            if (k + 1 < nblk) {
                if (tid == 32) {
                    load_x(k + 1);
                } else if (warp >= 4) {
                    if (k >= 1 && tid == 128 && ok &&
                        !mbar_wait_bounded(barE2 + 8 * ((k + 1) & 1), (uint32_t)(((k - 1) >> 1) & 1), kWaitLimit))
                        ok = false;
                    named_sync(kBarScan, 128);
                    scan_block(k + 1);
                }
            }
        }
        // final conv state: the last three raw inputs of the staged channels
        const int len_last = nblk > 0 ? blen(nblk - 1) : 0;
        named_sync(kBarProd, kProd);
        // B/C channels of a group wider than one cluster: several clusters hold the same values
        // and may run at different times, so the first cluster of the group stages them and a
        // later kernel writes them out (an in-place final state must not be overwritten before
        // every cluster has read it as its initial state)
        const bool first_cluster = (cid % ncl) == 0;
        for (int e = tid; e < 3 * SROW; e += kProd) {
            const int kk = e / SROW, c = e % SROW;
            const __nv_bfloat16 v =
                reinterpret_cast<const __nv_bfloat16*>(stage + (c / 8) * kStageRows + kStageTok - 3 + len_last + kk)[c % 8];
            if (SPLIT && c >= kP) {
                if (first_cluster)
                    ((__nv_bfloat16*)p.bc_conv)[(bi * 2 * GN + staged_channel(c) - HP) * 3 + kk] = v;
            } else {
                ((__nv_bfloat16*)p.final_conv)[(sidx * Cc + staged_channel(c)) * 3 + kk] = v;
            }
        }
    } else if constexpr (STATE_ONLY) {
        // ================= consumer of the state-only pass (warps 8..15) =================
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float lam_tot = 0.0f;   // sum of delta*A over the row, log2 units
        for (int64_t k = 0; k < nblk; ++k) {
            const int sl = (int)(k & 1);
            const uint32_t par = (uint32_t)(k & 1);
            if (ok && !mbar_wait_bounded(barP, par, kWaitLimit)) ok = false;
            if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
            fence_after_sync();
            const float lam_end = s_lam[sl * kT + kT - 1];
            lam_tot += lam_end;
            float s_[32];
            tmem_ld32(tmem + lane_base + kColS + chalf * 32, s_);
            tmem_wait_ld();
            const float2 aend = splat2(ex2(lam_end));
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float2 hv = fma2(aend, make_float2(H[i], H[i + 1]), make_float2(s_[i], s_[i + 1]));
                H[i] = hv.x;
                H[i + 1] = hv.y;
            }
            fence_before_sync();
            named_sync(kBarCons, kThreads - kProd);
            if (tid == kProd) {
                mbar_arrive_local(barC);             // S^T read: the next block's MMA may overwrite it
                mbar_arrive_local(barE2 + 8 * sl);   // the cumsum slot is free
            }
        }
        float* fs = p.final_ssm + (sidx * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < 32; ++i) fs[(int64_t)(chalf * 32 + i) * kN + crow] = H[i];
        if (tid == kProd && p.decay) p.decay[bi * p.H + h] = ex2(lam_tot);
    } else {
        // =========================== consumer (warps 8..15) ===========================
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        // byte offset of 16-byte chunk c of token row r in a swizzled z/y tile
        auto zy_off = [](int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); };
        auto load_z = [&](int64_t kb) {   // thread kProd
            mbar_arrive_expect_tx(barZ, (uint32_t)kT * kP * 2);
            tma_load_3d(aZ, &maps.z, h * kP, tmap_t0 + (int)(kb * kT), tmap_b, barZ);
        };
        // this thread's 32 output channels of token crow into the y tile, then (thread kProd,
        // after every consumer thread) one TMA store of the block's [128 x 64] box; the tile is
        // free again once the previous store has been read out (waited before the named barrier
        // that precedes every call)
        // The last, shorter block of a packed sequence is stored row by row instead: a box would
        // also write the first rows of the next sequence.
        auto store_y = [&](int64_t kb, const float* gv, float scale, bool norm) {
            const bool rows_only = varlen && blen(kb) < kT;
            unsigned char* ty = smem + Lo::OFF_Y;
            uint4* yrow = reinterpret_cast<uint4*>((__nv_bfloat16*)p.y + (row0 + kb * kT + crow) * p.y_ld + h * kP + chalf * 32);
            const float2* nw2 = reinterpret_cast<const float2*>(s_nw + chalf * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 gg = make_float2(gv[8 * v + 2 * e], gv[8 * v + 2 * e + 1]);
                    w[e] = pack_f2(norm ? mul2(mul2(gg, splat2(scale)), nw2[4 * v + e]) : gg);
                }
                if (!rows_only) *reinterpret_cast<uint4*>(ty + zy_off(crow, chalf * 4 + v)) = make_uint4(w[0], w[1], w[2], w[3]);
                else if (crow < blen(kb)) yrow[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (rows_only) return;
            fence_async_smem();
            named_sync(kBarCons, kThreads - kProd);
            if (tid == kProd) {
                tma_store_3d(&maps.y, aY, h * kP, tmap_t0 + (int)(kb * kT), tmap_b);
                bulk_commit();
            }
        };
        // group RMSNorm of block kb: every CTA's sums of squares, the gated values from TMEM
        auto finish_norm = [&](int64_t kb) {
            const uint32_t nsl = (uint32_t)(kb % 3);
            if (ok && !mbar_wait_cluster(barN3 + 8 * nsl, (uint32_t)((kb / 3) & 1), kWaitLimit)) ok = false;
            float tot = 0.0f;
#pragma unroll
            for (int rr = 0; rr < 2 * R; ++rr) tot += s_red[(nsl * R * 2 + rr) * 128 + crow];
            const float scale = rsqrtf(tot / (float)(R * kP) + p.eps);
            float gv[32];
            tmem_ld32(tmem + lane_base + kColG + chalf * 32, gv);
            tmem_wait_ld();
            store_y(kb, gv, scale, true);
        };
        if (nblk > 0 && tid == kProd) load_z(0);
        for (int64_t k = 0; k < nblk; ++k) {
            const int64_t t0 = k * kT;
            const int len = blen(k);
            const int sl = (int)(k & 1);
            const uint32_t par = (uint32_t)(k & 1);
            if (ok && !mbar_wait_bounded(barP, par, kWaitLimit)) ok = false;
            if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
            fence_after_sync();
            // expect the peers' sums of squares of block k (2 floats per row from every CTA)
            if constexpr (!SPLIT) {
                if (tid == kProd) mbar_arrive_expect_tx(barN3 + 8 * (uint32_t)(k % 3), (uint32_t)(R * 2 * 128 * 4));
            }
            const float* lamb = s_lam + sl * kT;
            const float* dlb = s_dl + sl * kT;
            const float* vb = s_v + sl * kT;
            const float lam_end = lamb[kT - 1];
            // masked, decayed M (row crow, columns chalf*64 .. +64) as bf16 pairs into TMEM
            {
                const int i = crow;
                const float li = lamb[i];
                const bool fac = li > -96.0f;
                const float ui = ex2(li);
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float cb[32];
                    tmem_ld32(tmem + lane_base + kColCB + chalf * 64 + part * 32, cb);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int j0 = chalf * 64 + part * 32 + v * 8;
                        if (j0 > i) {                 // above the diagonal: all zero
#pragma unroll
                            for (int e = 0; e < 4; ++e) w[4 * v + e] = 0u;
                        } else if (fac) {
                            const float2* v2 = reinterpret_cast<const float2*>(vb + j0);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float2 m = mul2(make_float2(cb[v * 8 + 2 * e], cb[v * 8 + 2 * e + 1]), mul2(splat2(ui), v2[e]));
                                if (j0 + 2 * e > i) m.x = 0.0f;
                                if (j0 + 2 * e + 1 > i) m.y = 0.0f;
                                w[4 * v + e] = pack_f2(m);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = j0 + 2 * e;
                                const float mx = (j <= i) ? cb[v * 8 + 2 * e] * ex2(li - lamb[j]) * dlb[j] : 0.0f;
                                const float my = (j + 1 <= i) ? cb[v * 8 + 2 * e + 1] * ex2(li - lamb[j + 1]) * dlb[j + 1] : 0.0f;
                                w[4 * v + e] = pack_bf16x2(mx, my);
                            }
                        }
                    }
                    tmem_st16(tmem + lane_base + kColM + chalf * 32 + part * 16, w);
                }
            }
            // state update H <- exp(lam_end) H + S and its bf16 copy for the next block
            {
                float s_[32];
                tmem_ld32(tmem + lane_base + kColS + chalf * 32, s_);
                tmem_wait_ld();
                const float2 aend = splat2(ex2(lam_end));
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float2 hv = fma2(aend, make_float2(H[i], H[i + 1]), make_float2(s_[i], s_[i + 1]));
                    H[i] = hv.x;
                    H[i + 1] = hv.y;
                }
                unsigned char* sH = smem + Lo::OFF_H;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 u;
                    u.x = pack_bf16x2(H[8 * v + 0], H[8 * v + 1]); u.y = pack_bf16x2(H[8 * v + 2], H[8 * v + 3]);
                    u.z = pack_bf16x2(H[8 * v + 4], H[8 * v + 5]); u.w = pack_bf16x2(H[8 * v + 6], H[8 * v + 7]);
                    *reinterpret_cast<uint4*>(sH + canon_off(crow, chalf * 32 + 8 * v, kP)) = u;
                }
            }
            tmem_wait_st();
            fence_async_smem();
            fence_before_sync();
            if (tid == kProd) bulk_wait_read_all();   // the previous y store has left the y tile
            named_sync(kBarCons, kThreads - kProd);
            if (tid == kProd) {
                fence_after_sync();
                const uint32_t id_yi = idesc_bf16(128, 64, 0, 1);
                const uint32_t aXs = aX + 16384 * (uint32_t)sl;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + kColYi, tmem + kColM + kk * 8, sdesc(aXs + kk * 2048, 1024, 128), id_yi, kk > 0);
                mma_commit(bar1);
                // C'B'^T and S^T read, H^T of block k+1 written; the producer's next MMAs queue
                // behind M x'
                mbar_arrive_local(barC);
            }
            if constexpr (!SPLIT) {
                if (k >= 1) finish_norm(k - 1);   // overlaps the MMA M x' of this block
            }
            if (ok && !mbar_wait_bounded(bar1, par, kWaitLimit)) ok = false;
            if (ok && !mbar_wait_bounded(barZ, par, kWaitLimit)) ok = false;
            fence_after_sync();
            // epilogue: y = Yi + exp(lam_i) Ys + D x', gate
            float gt[32];
            {
                const int i = crow;
                float yi[32], ys[32];
                tmem_ld32(tmem + lane_base + kColYi + chalf * 32, yi);
                tmem_ld32(tmem + lane_base + kColYs0 + 64 * sl + chalf * 32, ys);
                tmem_wait_ld();
                const float2 el = splat2(ex2(lamb[i])), d2 = splat2(Dh);
                const unsigned char* sX = smem + Lo::OFF_X + sl * 16384;
                const unsigned char* tz = smem + Lo::OFF_Z;
                float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 xw = *reinterpret_cast<const uint4*>(sX + canon_off(i, chalf * 32 + 8 * v, kP));
                    const uint4 zv = *reinterpret_cast<const uint4*>(tz + zy_off(i, chalf * 4 + v));
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 8 * v + 2 * e;
                        float2 y = fma2(el, make_float2(ys[c], ys[c + 1]), make_float2(yi[c], yi[c + 1]));
                        y = fma2(d2, bf2_to_f2((&xw.x)[e]), y);
                        const float2 gg = mul2(y, silu2(bf2_to_f2((&zv.x)[e])));
                        gt[c] = gg.x;
                        gt[c + 1] = gg.y;
                        ss2 = fma2(gg, gg, ss2);
                    }
                }
                const float ss = ss2.x + ss2.y;
                if constexpr (SPLIT) {
                    if (i < len) p.ssp[((row0 + t0 + i) * p.H + h) * 2 + chalf] = ss;
                } else {
                    const uint32_t nsl = (uint32_t)(k % 3);
                    const uint32_t dst = smem_u32(s_red + ((nsl * R + q) * 2 + chalf) * 128 + i);
#pragma unroll
                    for (int rr = 0; rr < R; ++rr)
                        st_async_f32(cluster_map(dst, (uint32_t)rr), ss, cluster_map(barN3 + 8 * nsl, (uint32_t)rr));
                    tmem_st32(tmem + lane_base + kColG + chalf * 32, gt);
                    tmem_wait_st();
                }
            }
            fence_before_sync();
            if constexpr (SPLIT) {
                if (tid == kProd) bulk_wait_read_all();
            }
            named_sync(kBarCons, kThreads - kProd);
            if (tid == kProd) {
                mbar_arrive_local(barE2 + 8 * sl);   // x'[sl] and the cumsum slot are free
                if (k + 1 < nblk) load_z(k + 1);     // the z tile is free
            }
            if constexpr (SPLIT) store_y(k, gt, 1.0f, false);
        }
        if constexpr (!SPLIT) {
            if (nblk >= 1) {
                if (tid == kProd) bulk_wait_read_all();
                named_sync(kBarCons, kThreads - kProd);
                finish_norm(nblk - 1);
            }
        }
        if (tid == kProd) bulk_wait_all();   // the y stores have completed
        // final SSM state of this head
        float* fs = p.final_ssm + (sidx * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < 32; ++i) fs[(int64_t)(chalf * 32 + i) * kN + crow] = H[i];
    }

    if (!ok) set_device_status(p.status, kDevTimeout);
    fence_before_sync();
    __syncthreads();
    cluster.sync();   // no peer still copies into or arrives on this CTA's shared memory
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Group RMSNorm of the gated values written by the SPLIT kernel (2 partial sums per head).
__global__ void __launch_bounds__(256) ws_norm_finish_kernel(PrefillParams p)
{
    const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (w >= p.rows() * p.G) return;
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

// cuTensorMapEncodeTiled, fetched once through the runtime (no link-time libcuda dependency).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn()
{
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// [b][L][width] bf16 rows of `ld` elements viewed as [b][width/8 vectors][L][8]; boxes of
// 8 channels x kStageRows tokens x `nvec` vectors x 1 sequence land as [vector][token][8].
bool encode_rows(CUtensorMap* m, const void* base, int64_t width, int64_t ld, int64_t L, int64_t b, int nvec)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {8, (cuuint64_t)L, (cuuint64_t)(width / 8), (cuuint64_t)b};
    const cuuint64_t strides[3] = {(cuuint64_t)(ld * 2), 16, (cuuint64_t)(L * ld * 2)};
    const cuuint32_t box[4] = {8, (cuuint32_t)kStageRows, (cuuint32_t)nvec, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [b][L][width] bf16 rows of `ld` elements; boxes of 64 channels x 128 tokens x 1 sequence,
// 128-byte swizzled in shared memory.
bool encode_tile(CUtensorMap* m, const void* base, int64_t width, int64_t ld, int64_t L, int64_t b)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)L, (cuuint64_t)b};
    const cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(L * ld * 2)};
    const cuuint32_t box[3] = {(cuuint32_t)kP, (cuuint32_t)kT, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The staged B/C part of the final conv state, into each sequence's slot.
__global__ void __launch_bounds__(256) ws_bc_conv_out_kernel(PrefillParams p)
{
    const int64_t per = 2 * p.GN() * 3;
    const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (e >= p.b * per) return;
    const int64_t bi = e / per, r = e % per;
    const int64_t sidx = p.cu_seqlens && p.slot_idx ? (int64_t)p.slot_idx[bi] : bi;
    ((__nv_bfloat16*)p.final_conv)[(sidx * p.Cc() + p.HP()) * 3 + r] = ((const __nv_bfloat16*)p.bc_conv)[e];
}

template <int R, bool SPLIT, bool STATE_ONLY = false>
cudaError_t launch_ws(const PrefillParams& p, cudaStream_t st)
{
    using Lo = WsLayout<R>;
    WsMaps maps;
    memset(&maps, 0, sizeof(maps));
    // packed sequences: one row of all the packed tokens
    const int64_t mL = p.L, mb = p.cu_seqlens ? 1 : p.b;
    if (p.L > 0) {   // no block, no load: the maps stay unused
        if (!encode_rows(&maps.x, p.x, p.HP(), p.x_ld, mL, mb, kP / 8) ||
            !encode_rows(&maps.B, p.B, p.GN(), p.B_ld, mL, mb, Lo::NS / 8) ||
            !encode_rows(&maps.C, p.C, p.GN(), p.C_ld, mL, mb, Lo::NS / 8))
            return cudaErrorInvalidValue;
        if (!STATE_ONLY &&
            (!encode_tile(&maps.z, p.z, p.HP(), p.z_ld, mL, mb) || !encode_tile(&maps.y, p.y, p.HP(), p.y_ld, mL, mb)))
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(ssd_prefill_ws_kernel<R, SPLIT, STATE_ONLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Lo::TOTAL);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.b * p.H));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Lo::TOTAL;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        LaunchScope ls(STATE_ONLY ? "tc_prefill_state" : "tc_prefill", st);
        e = cudaLaunchKernelEx(&cfg, ssd_prefill_ws_kernel<R, SPLIT, STATE_ONLY>, p, maps);
        if (e != cudaSuccess) return e;
    }
    if (SPLIT && !STATE_ONLY && p.rows() > 0) {
        LaunchScope ls("tc_norm_finish", st);
        const int64_t warps = p.rows() * p.G;
        ws_norm_finish_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (SPLIT) {
        LaunchScope ls("tc_bc_conv_out", st);
        const int64_t n = p.b * 2 * p.GN() * 3;
        ws_bc_conv_out_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

// Groups of 2 or 4 heads: one cluster per group (fused norm); wider groups: clusters of 4
// heads and the norm finished by ws_norm_finish_kernel.
cudaError_t launch_prefill_state_ws(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    switch (p.H / p.G) {
    case 2: return launch_ws<2, false, true>(p, stream);
    case 4: return launch_ws<4, false, true>(p, stream);
    }
    return launch_ws<4, true, true>(p, stream);
}

cudaError_t launch_prefill_ws(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    switch (p.H / p.G) {
    case 2: return launch_ws<2, false>(p, stream);
    case 4: return launch_ws<4, false>(p, stream);
    }
    return launch_ws<4, true>(p, stream);
}

int prefill_ws_partials_per_head() { return 2; }

bool prefill_tc_supported(int act, int P, int N, int H, int G)
{
    const int r = H / G;
    return act == 1 && P == kP && N == kN && (r == 2 || (r % 4 == 0 && r <= 256));
}

bool prefill_tc_split(int H, int G) { return H / G > 4; }



}  // namespace ssd
