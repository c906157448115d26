// ssd_prefill_ws.cu -- warp-specialised, software-pipelined tensor-core prefill of the SSD
// mixer (bf16 activations, head dim 64, state dim 128).
//
// Same arithmetic as one block of the chunked SSD decomposition (Modalities PR #459,
// ssd.py notes on the chunk-parallel block decomposition) with the state kept on chip:
// per 128-token block of one head,
//   lam_i = inclusive sum of delta*A (log2 units), CB = C' B'^T, Ys = C' H^T,
//   S^T = B'^T (x' w) with w_j = exp(lam_end - lam_j) delta_j,
//   M_ij = CB_ij exp(lam_i - lam_j) delta_j (j <= i), Yi = M x',
//   y = Yi + exp(lam_i) Ys + D x',  g = y SiLU(z),  out = g / rms_group(g) * norm_w
//   (for groups held by a cluster D sits on M's diagonal, so Yi already holds D x'),
//   H <- exp(lam_end) H + S.
//
// Two kernels per call (three when the norm group is wider than a cluster):
//   bc_conv       SiLU(conv) of the B and C channels, once for all heads of a group (every
//                 head reads the same B', C'), into the workspace as one 32 KB chunk per
//                 (128-token block, matrix, group), already in the MMA operand layout;
//   ssd_prefill_ws_kernel  one CTA per (sequence, head): the x conv, the scan, the chunked SSD
//                 on tensor cores, the D skip and the gated norm. When a thread-block cluster
//                 holds the whole group (2 or 4 heads), the norm's per-token sums of squares go
//                 to every peer with st.async; wider groups write gated values and partial sums
//                 and a light pass finishes the norm.
//
// Data movement: the raw x rows of a block (with the 3-token conv halo) arrive by TMA as one
// 128-byte-swizzled box, double-buffered; the block's B', C' by two contiguous bulk copies; z is
// brought into L2 by a TMA prefetch a block ahead and read into registers (64 contiguous bytes
// per consumer thread) during the state update; y leaves through a TMA store of a
// 128-byte-swizzled tile; the decay-masked M goes from registers into TMEM and feeds M x' as the
// TMEM A operand. Every copy moves rows of at least 128 bytes: the copy engine of an SM handles
// requests at a limited rate, and 16-byte pieces (8 channels) left it the slowest stage.
//
// Roles (512 threads). A tcgen05.mma issue holds its thread about as long as the MMAs take,
// so one thread that does nothing else issues them all, in the order the consumer needs them:
// M x' of block k-1, then C'B'^T of block k (so the consumer's M of block k never waits for the
// state-dependent products), then C'H^T and B'^T(x'w) of block k:
//   producer warps 0..6  : the softplus + cumsum (warps 3..6) and the conv + SiLU of x' and
//                          x'w of block k+1 while the MMAs of block k run;
//   control warp 7       : (one lane) the copies of B'/C', M x' of block k-1 once the consumer
//                          has written M, C'B'^T of block k once B', C' are in, C'H^T and
//                          B'^T(x'w) of block k once x'w and H^T are in;
//   consumer warps 8..15 : for block k: the masked decay product M (then M x' may start), the
//                          state update while M x' runs, the group norm of block k-1, then the
//                          epilogue of block k.
// Variants: packed variable-length sequences on state slots (a CTA reads its sequence's
// rows, length and slot from device arrays), and STATE_ONLY (final states and decay only).
// Rows of fixed length may run as pieces over a series of launches (WsPieces), when whole rows
// would leave the last wave of CTAs part-empty.
// Hand-offs use mbarriers (all waits bounded):
//   barCB  C'B'^T of a block done     bar0  C'H^T and B'^T(x'w) done     bar1  M x' done
//   (tensor-core commits)
//   barBC  B' and C' of a block have landed (bulk copies)
//   barP   producer: block k's x', x'w and cumsum are in shared memory (3 slots: the producer
//          may arrive for blocks k+1 and k+2 before a slow consumer waits for k)
//   barM   consumer (one arrival per warp): C'B'^T of block k read, M of block k in TMEM
//   barH   consumer (one arrival per warp): phase 0, H^T of block 0 written; phase k+1, S^T of
//          block k read and H^T of block k+1 written to shared memory, so the MMAs of block
//          k+1 may start
//   barE2  consumer: a block's x' and cumsum slots are free again (3 slots: x' and the cumsum
//          live until the epilogue, so they rotate through three buffers)
//   barW   the MMAs of a block are done, so its x'w slot is free again (2 slots: x'w is read
//          only by the MMA B'^T(x'w), so two buffers suffice)
//   barN3  the sums of squares of a block from every CTA of the cluster have landed
//          (st.async transaction bytes; 3 slots)
//   barTX  TMA of the raw x rows (one per stage)
// Barriers waited two blocks back use two slots, so a waiter never meets a barrier that
// has moved two phases past the one it expects. The group norm of block k is finished one
// block late (its gated values wait in TMEM); a peer can be at most two blocks ahead of
// that finish, hence three slots for the sums of squares.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
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
constexpr int kProd = 224;    // producer threads (warps 0..6)
constexpr int kCtl = 224;     // the control thread (warp 7, lane 0)
constexpr int kCons = 256;    // first consumer thread (warps 8..15)
constexpr int kConsWarps = (kThreads - kCons) / 32;
constexpr int kScan0 = 96;    // the cumsum runs on producer threads 96..223 (warps 3..6)
// Raw staging of the head's x channels: tokens t0-3 .. t0+127 of a block, so rows 0..2 hold the
// conv halo and rows 3..130 the block's tokens; one TMA box of 131 rows of 128 bytes, 128-byte
// swizzled (16-byte piece v of row r at piece v ^ (r % 8)), 1024-byte aligned.
constexpr int kStageRows = 131, kStageTok = 3, kVX = kP / 8;
__device__ __forceinline__ int stage_u4(int r, int v) { return r * 8 + (v ^ (r & 7)); }
constexpr uint32_t kTmemCols = 512;
constexpr long long kWaitLimit = 4000000000LL;  // ~2 s at 2 GHz

// TMEM columns: C'B'^T, Ys (two slots), S^T, Yi, the gated values of a block awaiting its norm,
// and the masked decay matrix M (bf16 pairs; the A operand of M x')
constexpr uint32_t kColCB = 0, kColYs0 = 128, kColS = 256, kColYi = 320, kColG = 384, kColM = 448;

// named barriers
constexpr int kBarProd = 1, kBarCons = 2, kBarScan = 3;

// R = CTAs of the cluster that share the group norm (1: no cluster, the norm is finished by a
// later pass or not computed).
template <int R>
struct WsLayout {
    // B', C' of a block: [16 vectors of 8 channels][128 tokens][8] bf16 (the MMA operand
    // layout); y tile [128 tokens][64 channels] bf16, 16-byte chunks swizzled by token % 8
    // (1024-byte aligned); x' three slots, x'w two; the bf16 copy of H^T
    static constexpr uint32_t OFF_C = 0, OFF_B = 32768, OFF_Y = 65536, OFF_X = 81920,
                              OFF_XW = OFF_X + 3 * 16384, OFF_H = OFF_XW + 2 * 16384, OFF_STAGE = OFF_H + 16384;
    static constexpr uint32_t STAGE_BYTES = (uint32_t)kStageRows * kP * 2;
    static constexpr uint32_t STAGE_PITCH = ((STAGE_BYTES + 1023) / 1024) * 1024;   // swizzle atoms
    // two raw x stages (the rows of block k+1 arrive while block k is convolved) where shared
    // memory allows; one for clusters of 4, whose exchange buffer for the norm sums is larger
    static constexpr int XBUF = R <= 2 ? 2 : 1;
    static_assert(OFF_STAGE % 1024 == 0, "the swizzled x stage needs 1024-byte alignment");
    static constexpr uint32_t OFF_MISC = OFF_STAGE + XBUF * STAGE_PITCH;
    // fp32 arrays: lam, delta, v, the segment factors g (3 slots each), scan scratch, sums of
    // squares [3][R][2][128], conv taps and biases of the head's x channels, norm weights
    static constexpr uint32_t F_LAM = 0, F_DL = 384, F_V = 768, F_G = 1152, F_SCAN = 1536, F_RED = 1552,
                              F_CW = F_RED + 3 * R * 2 * 128, F_CB = F_CW + kP * 4, F_NW = F_CB + kP,
                              F_END = F_NW + kP;
    static constexpr uint32_t OFF_BAR = OFF_MISC + ((F_END * 4 + 15) / 16) * 16;
    static constexpr int NBAR = 19;  // bar0 bar1 barBC barP[3] barM barE2[3] barW[2] barN3[3] barTX[2] barH barCB
    static constexpr uint32_t OFF_TSLOT = OFF_BAR + NBAR * 8;
    static constexpr uint32_t TOTAL = OFF_TSLOT + 16;
    static_assert(TOTAL <= 232448, "dynamic shared memory above the 227 KB a CTA may use");
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

// Inclusive scan over the 128 threads kScan0 .. kScan0+127 (named barrier kBarScan).
__device__ __forceinline__ float scan128(float v, float* tot)
{
    const int lane = threadIdx.x & 31, wid = (threadIdx.x - kScan0) >> 5;
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

// SiLU(conv) of the B and C channels (the first nch of the 2*G*N), once per token for all the
// heads that read them, into the workspace as one 32 KB chunk per (128-token block of a
// sequence, matrix, group) in the MMA operand layout (prefill_bc_blocks), so the main kernel
// fetches each with one contiguous copy. One CTA per (block slot, 64 channels): the block's raw
// rows and its 3-row halo (the sequence's initial conv state before its first token, zeros
// without one) are loaded with coalesced 16-byte loads into a padded tile, and each 8-channel
// vector's [128 tokens][8] slab is written as one contiguous 2 KB run, zeros past the end of
// the sequence.
constexpr int kBcRows = kT + 3, kBcPitch = 9;   // tile rows (block + halo), 16-byte pieces per row
__global__ void __launch_bounds__(256) bc_conv_kernel(PrefillParams p, int nch)
{
    __shared__ uint4 tile[kBcRows * kBcPitch];
    __shared__ float4 wsm[64];
    __shared__ float bsm[64];
    const int64_t GN = p.GN(), HP = p.HP(), Cc = p.Cc();
    const int64_t slot_blk = blockIdx.x;
    const int64_t c0 = (int64_t)blockIdx.y * 64;   // first channel within [B | C]
    const int tid = threadIdx.x;
    // the sequence whose blocks hold this slot: the last s with s + start_s / 128 <= slot_blk
    auto start_of = [&](int64_t s) { return p.cu_seqlens ? (int64_t)p.cu_seqlens[s] : s * p.L; };
    int64_t lo = 0, hi = p.b - 1;
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) / 2;
        if (mid + start_of(mid) / kT <= slot_blk) lo = mid;
        else hi = mid - 1;
    }
    const int64_t s = lo, start = start_of(s);
    const int64_t len = p.cu_seqlens ? (int64_t)p.cu_seqlens[s + 1] - start : p.L;
    const int64_t k = slot_blk - (s + start / kT);
    if (k < 0 || k * kT >= len) return;   // a slot no block of any sequence uses
    const int64_t slot = p.cu_seqlens && p.slot_idx ? (int64_t)p.slot_idx[s] : s;
    const bool init = p.init_conv != nullptr && (!p.cu_seqlens || !p.has_init || p.has_init[s] != 0);
    const bool isC = c0 >= GN;
    const __nv_bfloat16* src = (const __nv_bfloat16*)(isC ? p.C : p.B) + (isC ? c0 - GN : c0);
    const int64_t ld = isC ? p.C_ld : p.B_ld;
    if (tid < 64) {
        wsm[tid] = *reinterpret_cast<const float4*>(p.conv_w + (HP + c0 + tid) * 4);
        bsm[tid] = p.conv_b[HP + c0 + tid];
    }
    // tile row r holds token k*128 + r - 3 of the sequence; every load of a thread is issued
    // before the first one is stored
    constexpr int kLoads = (kBcRows * 8 + 255) / 256;
    uint4 val[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int e = tid + 256 * i;
        const int r = e / 8, v = e % 8;
        const int64_t tok = k * kT + r - 3;
        val[i] = make_uint4(0u, 0u, 0u, 0u);
        if (e < kBcRows * 8 && tok >= 0 && tok < len && SSD_IN_BOUNDS(p.status, start + tok < p.rows()))
            val[i] = *reinterpret_cast<const uint4*>(src + (start + tok) * ld + v * 8);
    }
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
        const int e = tid + 256 * i;
        const int r = e / 8, v = e % 8;
        const int64_t tok = k * kT + r - 3;
        if (e < kBcRows * 8 && tok < 0 && init) {   // the initial conv state, oldest first
            __nv_bfloat16 hv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                hv[q] = ((const __nv_bfloat16*)p.init_conv)[(slot * Cc + HP + c0 + v * 8 + q) * 3 + (tok + 3)];
            val[i] = *reinterpret_cast<const uint4*>(hv);
        }
        if (e < kBcRows * 8) tile[r * kBcPitch + v] = val[i];
    }
    __syncthreads();
    const int64_t mat = isC ? 1 : 0, cw = isC ? c0 - GN : c0;   // channel within its matrix
    __nv_bfloat16* chunk = (__nv_bfloat16*)p.bcp + ((slot_blk * 2 + mat) * p.G + cw / kN) * (int64_t)(kT * kN);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int o = tid + 256 * i;
        const int v = o / kT, t = o % kT;   // consecutive threads: consecutive tokens of one vector
        float out[8];
        if (k * kT + t < len) {
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = bsm[v * 8 + q];
#pragma unroll
            for (int j = 0; j < 4; ++j) {   // tap j multiplies token t - 3 + j (tile row t + j)
                float in[8];
                unpack_bf16x8(tile[(t + j) * kBcPitch + v], in);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf((&wsm[v * 8 + q].x)[j], in[q], acc[q]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) out[q] = tc::silu_fast(acc[q]);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) out[q] = 0.0f;
        }
        if (SSD_IN_BOUNDS(p.status, (slot_blk * 2 + mat) * p.G + cw / kN < (int64_t)prefill_bc_blocks(p.b, p.rows()) * 2 * p.G))
            store_vec<__nv_bfloat16>(chunk + (((cw % kN) / 8 + v) * kT + t) * 8, out);
    }
}

// Tensor maps of x, y and z as [b][L][channels] (bf16), boxes of one head's 64 channels (128
// bytes) with 128-byte swizzling: 131 tokens for x (a block and its conv halo), 128 for y and z
// (z only to prefetch a block into L2 a block ahead of the epilogue that reads it).
struct WsMaps {
    CUtensorMap x, y, z;
};

// Rows split into pieces (runs of whole blocks), run as a series of launches: launch `round`
// takes positions round * per_round ... of the queue [piece 0 of every (sequence, cluster),
// piece 1 of every one, ...]. A piece's predecessor sits one queue length (the number of
// (sequence, cluster) pairs, at least per_round) earlier, so it ran in an earlier launch; it
// left the state in final_ssm, which the piece continues from. npieces = 1: one launch, one
// whole row per cluster.
struct WsPieces {
    int round, per_round, npieces, piece_blocks;
};

// STATE_ONLY: the state-only pass (final states and decay of a prefill, no output rows): the
// conv of x, B'^T(x'w) and the state recurrence.
template <int R, bool SPLIT, bool STATE_ONLY>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_prefill_ws_kernel(PrefillParams p, const __grid_constant__ WsMaps maps, WsPieces pc)
{
    using Lo = WsLayout<R>;
    extern __shared__ __align__(1024) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();

    const int q = (int)cluster.block_rank();
    const int rpg = p.H / p.G;
    const int ncl = rpg / R;
    // this cluster's (sequence, head group) and, for a row split into pieces, the first block
    // of its piece (pieces only for fixed-length rows, in the one-CTA full pass)
    int64_t cid = blockIdx.x / R, k0 = 0;
    if constexpr (R == 1 && !STATE_ONLY) {
        if (pc.npieces > 1) {
            const int64_t jobs = p.b * p.G * ncl;
            const int64_t pos = (int64_t)pc.round * pc.per_round + cid;
            cid = pos % jobs;
            k0 = (pos / jobs) * pc.piece_blocks;
        }
    }
    const int64_t bi = cid / ((int64_t)p.G * ncl);
    const int g = (int)((cid / ncl) % p.G);
    const int h = g * rpg + (int)(cid % ncl) * R + q;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t HP = p.HP(), GN = p.GN(), Cc = p.Cc();
    // this CTA's sequence: its first token row, length, state slot, and whether it starts from
    // the states given (packed variable-length calls read them from their slot arrays)
    const bool varlen = p.cu_seqlens != nullptr;
    const int64_t row0 = varlen ? (int64_t)p.cu_seqlens[bi] : bi * p.L + k0 * kT;
    const int64_t seqlen = varlen ? (int64_t)p.cu_seqlens[bi + 1] - row0
                                  : min(p.L - k0 * kT, pc.npieces > 1 ? (int64_t)pc.piece_blocks * kT : p.L);
    // a piece after the row's first continues from the state its predecessor left in final_ssm,
    // and its conv halo is the row's own preceding tokens
    const bool piece_cont = k0 > 0;
    const int64_t sidx = varlen && p.slot_idx ? (int64_t)p.slot_idx[bi] : bi;
    const bool cont = varlen ? (!p.has_init || p.has_init[bi] != 0) : true;
    const bool init_ssm = piece_cont || (cont && p.init_ssm != nullptr);
    const bool init_conv = !piece_cont && cont && p.init_conv != nullptr;
    // coordinates of token 0 in the tensor maps (token, sequence)
    const int tmap_t0 = varlen ? (int)row0 : (int)(k0 * kT), tmap_b = varlen ? 0 : (int)bi;

    float* mf = reinterpret_cast<float*>(smem + Lo::OFF_MISC);
    float* s_lam = mf + Lo::F_LAM;
    float* s_dl = mf + Lo::F_DL;
    float* s_v = mf + Lo::F_V;
    float* s_g = mf + Lo::F_G;
    float* s_scan = mf + Lo::F_SCAN;
    float* s_red = mf + Lo::F_RED;     // [3 slots][R CTAs][2 halves][128 rows]
    float* s_cw = mf + Lo::F_CW;
    float* s_cb = mf + Lo::F_CB;
    float* s_nw = mf + Lo::F_NW;
    uint4* stage = reinterpret_cast<uint4*>(smem + Lo::OFF_STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lo::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lo::OFF_TSLOT);

    const uint32_t s_base = smem_u32(smem);
    const uint32_t aC = s_base + Lo::OFF_C, aB = s_base + Lo::OFF_B;
    const uint32_t aX = s_base + Lo::OFF_X, aXW = s_base + Lo::OFF_XW, aH = s_base + Lo::OFF_H;
    const uint32_t bar0 = smem_u32(&bars[0]), bar1 = smem_u32(&bars[1]), barBC = smem_u32(&bars[2]);
    const uint32_t barP = smem_u32(&bars[3]), barM = smem_u32(&bars[6]);
    const uint32_t barE2 = smem_u32(&bars[7]), barW = smem_u32(&bars[10]), barN3 = smem_u32(&bars[12]);
    const uint32_t barTX = smem_u32(&bars[15]), barH = smem_u32(&bars[17]), barCB = smem_u32(&bars[18]);
    constexpr int XBUF = Lo::XBUF;
    constexpr int kStageU4 = (int)(Lo::STAGE_PITCH / 16);   // one raw x stage, in 16-byte units
    // ring slots of block k: x', the cumsum and barP/barE2 rotate by 3, x'w and barW by 2
    auto s3 = [](int64_t k) { return (uint32_t)(k % 3); };
    auto p3 = [](int64_t k) { return (uint32_t)((k / 3) & 1); };

    // ---- set-up
    // the swizzled y tile needs a 1024-byte aligned base; every CTA sees the same base, so
    // all of them leave here together (before any barrier) if it is not
    if (smem_u32(smem) & 1023u) {
        if (tid == 0) set_device_status(p.status, kDevSmemMisaligned);
        return;
    }
    for (int c = tid; c < kP; c += kThreads) {
        const int64_t ch = (int64_t)h * kP + c;
        const float4 w = *reinterpret_cast<const float4*>(p.conv_w + ch * 4);
        float* cw = s_cw + (c / 2) * 8 + (c % 2);   // taps of channel pairs: [pair][tap][2]
        cw[0] = w.x; cw[2] = w.y; cw[4] = w.z; cw[6] = w.w;
        s_cb[c] = p.conv_b[ch];
    }
    if (!STATE_ONLY && tid < kP) s_nw[tid] = p.norm_w[(int64_t)h * kP + tid];
    if (tid == 0) {
        for (int i = 0; i < Lo::NBAR; ++i) mbar_init(smem_u32(&bars[i]), (i == 6 || i == 17) ? kConsWarps : 1);
        fence_mbar_init();
        prefetch_tmap(&maps.x);
        if (!STATE_ONLY) prefetch_tmap(&maps.z);
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);

    // consumer state: thread (n = row, half) keeps H^T[n][half*32 .. half*32+32) in fp32
    const bool consumer = tid >= kCons;
    const int crow = tid & 127, chalf = (tid - kCons) >> 7;   // consumer row and column half
    float H[32];
    fence_before_sync();
    __syncthreads();
    cluster.sync();   // every peer's barriers are initialised before any remote arrival
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const float A2 = p.A[h] * 1.4426950408889634f;
    const float Dh = STATE_ONLY ? 0.0f : p.D[h];
    const float bias = p.dt_bias[h];
    bool ok = true;
    // a launch of a series of pieces lets the next launch start on the SMs its CTAs free; that
    // launch waits for this one (griddepcontrol.wait) only where it reads what this one wrote
    if (pc.npieces > 1 && tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // consumer: the state entering the first block (fp32 in registers, thread (n = row, half)
    // keeps H^T[n][half*32 .. half*32+32)) and its bf16 copy for C'H^T; then the per-warp
    // arrival on barH that lets block 0's products start. A continuing piece first waits for the
    // earlier launches, whose last one wrote the state it continues from.
    auto init_state = [&]() {
        if (piece_cont) asm volatile("griddepcontrol.wait;" ::: "memory");
        const float* h0 = init_ssm ? (piece_cont ? p.final_ssm : p.init_ssm) + (sidx * p.H + h) * (int64_t)kP * kN : nullptr;
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
        fence_before_sync();
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive_local(barH);
    };

    const int64_t nblk = (seqlen + kT - 1) / kT;
    auto blen = [&](int64_t k) { return (int)min((int64_t)kT, seqlen - k * kT); };

    if (tid < kProd) {
        // =========================== producer (warps 0..6) ===========================
        // raw x rows t0-8 .. t0+127 of block kb (TMA, one box of the head's 8 vectors) into stage
        // kb % XBUF; rows outside the sequence read as zeros
        auto load_x = [&](int64_t kb) {
            const uint32_t bx = barTX + 8 * (uint32_t)(kb % XBUF);
            mbar_arrive_expect_tx(bx, Lo::STAGE_BYTES);
            tma_load_3d(smem_u32(stage + (kb % XBUF) * kStageU4), &maps.x, h * kP, tmap_t0 + (int)(kb * kT) - kStageTok,
                        tmap_b, bx);
        };
        auto wait_x = [&](int64_t kb) {
            return mbar_wait_bounded(barTX + 8 * (uint32_t)(kb % XBUF), (uint32_t)((kb / XBUF) & 1), kWaitLimit);
        };
        // softplus and cumsum of block kb into its slot (threads kScan0.., token tid - kScan0),
        // then dt of block kb + 1, a whole block ahead of its use
        // raw bf16 bits of the next block's dt, widened only when used, so the load's latency is
        // not waited for until a block later
        uint32_t dt_next = 0u;
        const unsigned short* gdt16 = reinterpret_cast<const unsigned short*>(p.dt);
        const int tok = tid - kScan0;
        auto scan_block = [&](int64_t kb) {
            const int slb = (int)s3(kb);
            float dl = 0.0f, a2 = 0.0f;
            if (tok < blen(kb)) {
                dl = softplus(__uint_as_float(dt_next << 16) + bias);
                a2 = dl * A2;
            }
            if (kb + 1 < nblk && (kb + 1) * kT + tok < seqlen &&
                SSD_IN_BOUNDS(p.status, row0 + (kb + 1) * kT + tok < p.rows()))
                dt_next = gdt16[(row0 + (kb + 1) * kT + tok) * p.dt_ld + h];
            const float lam = scan128(a2, s_scan);
            s_lam[slb * kT + tok] = lam;
            s_dl[slb * kT + tok] = dl;
            // exp2(lam_i - lam_j) = exp2(lam_i) * exp2(-lam_j) while every factor stays a
            // normal fp32 number (rows with lam_i > -96); chosen per row from its past only
            s_v[slb * kT + tok] = (lam > -96.0f) ? ex2(-lam) * dl : 0.0f;
            // for rows past that range: exp2(lam_i - lam_j) = exp2(lam_i - lam_s) * exp2(lam_s - lam_j)
            // with s the first token of j's 8-token segment; g_j = exp2(lam_s - lam_j) * delta_j
            const float lam_s = __shfl_sync(0xffffffffu, lam, (tid & 31) & ~7);
            s_g[slb * kT + tok] = ex2(lam_s - lam) * dl;
        };
        // conv + SiLU of the head's 8 staged x vectors of block kb into x' and x'w. Thread t takes
        // vector t / TPV and run t % TPV of its 128 tokens (4 or 5 consecutive tokens), sliding a
        // window of three widened raw rows along the run, so each raw row is read and widened
        // about 1.7 times instead of once per tap. A quarter warp covers 8 runs of one vector:
        // its staged rows (131-row pitch) and its x' rows fall in distinct shared-memory banks.
        auto conv_x = [&](int64_t kb) {
            constexpr int TPV = kProd / kVX;
            static_assert(kProd % kVX == 0 && 4 * TPV <= kT && kT <= 5 * TPV, "runs of 4 or 5 tokens");
            const int len = blen(kb);
            const int slb = (int)s3(kb);
            const float* lamb = s_lam + slb * kT;
            const float* dlb = s_dl + slb * kT;
            const float lam_end = lamb[kT - 1];
            unsigned char* sX = smem + Lo::OFF_X + slb * 16384;
            unsigned char* sXW = smem + Lo::OFF_XW + (uint32_t)(kb & 1) * 16384;
            const int v = tid / TPV, run = tid % TPV;
            const int r0 = (kT * run) / TPV, r1 = (kT * (run + 1)) / TPV;
            const int c0 = v * 8;
            // staged rows of tokens r0-3 .. r0+4 (the last only for runs of five)
            const uint4* stg = stage + (kb % XBUF) * kStageU4;
            const int rr0 = kStageTok - 3 + r0;
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
            float2 win[3][4];   // widened raw rows of tokens i-3, i-2, i-1 (channel pairs)
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                const uint4 r = stg[stage_u4(rr0 + e, v)];
#pragma unroll
                for (int j = 0; j < 4; ++j) win[e][j] = bf2_to_f2((&r.x)[j]);
            }
#pragma unroll
            for (int st = 0; st < 5; ++st) {
                const int i = r0 + st;
                if (st == 4 && i >= r1) break;
                float2 cur[4];
                {
                    const uint4 r = stg[stage_u4(rr0 + 3 + st, v)];
#pragma unroll
                    for (int j = 0; j < 4; ++j) cur[j] = bf2_to_f2((&r.x)[j]);
                }
                float2 o[4];
                if (i < len) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {   // channel pair (c0 + 2j, c0 + 2j + 1)
                        float2 vv = fma2(wr[j][0], win[0][j], br[j]);
                        vv = fma2(wr[j][1], win[1][j], vv);
                        vv = fma2(wr[j][2], win[2][j], vv);
                        vv = fma2(wr[j][3], cur[j], vv);
                        o[j] = silu2(vv);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[j] = make_float2(0.0f, 0.0f);
                }
                const float2 wgt = splat2((i < len) ? ex2(lam_end - lamb[i]) * dlb[i] : 0.0f);
                const uint4 u8 = make_uint4(pack_f2(o[0]), pack_f2(o[1]), pack_f2(o[2]), pack_f2(o[3]));
                const uint4 uw = make_uint4(pack_f2(mul2(o[0], wgt)), pack_f2(mul2(o[1], wgt)),
                                            pack_f2(mul2(o[2], wgt)), pack_f2(mul2(o[3], wgt)));
                *reinterpret_cast<uint4*>(sX + canon_off(i, c0, kP)) = u8;
                *reinterpret_cast<uint4*>(sXW + canon_off(i, c0, kP)) = uw;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    win[0][j] = win[1][j];
                    win[1][j] = win[2][j];
                    win[2][j] = cur[j];
                }
            }
        };
        if (nblk > 0) {
            if (tid == 0) {
                for (int64_t kb = 0; kb < XBUF && kb < nblk; ++kb) load_x(kb);
            }
            if (tid >= kScan0) {
                if (tok < seqlen && SSD_IN_BOUNDS(p.status, row0 + tok < p.rows())) dt_next = gdt16[(row0 + tok) * p.dt_ld + h];
                scan_block(0);
            }
        }
        // the three rows before the sequence hold the initial conv state (zeros without one), not
        // the TMA's fill or a neighbouring packed sequence: written once block 0's rows have landed
        if (nblk == 0 || init_conv || varlen) {
            if (nblk > 0 && ok && !wait_x(0)) ok = false;
            for (int e = tid; e < 3 * kP; e += kProd) {
                const int kk = e / kP, c = e % kP;
                __nv_bfloat16 v = __float2bfloat16_rn(0.0f);
                if (init_conv) v = ((const __nv_bfloat16*)p.init_conv)[(sidx * Cc + (int64_t)h * kP + c) * 3 + kk];
                reinterpret_cast<__nv_bfloat16*>(stage + stage_u4(kStageTok - 3 + kk, c / 8))[c % 8] = v;
            }
        }
        // x' and x'w of block 0 (the cumsum of block 0 is in its slot)
        if (nblk > 0) {
            if (ok && !wait_x(0)) ok = false;
            named_sync(kBarProd, kProd);
            conv_x(0);
            fence_async_smem();
            named_sync(kBarProd, kProd);
            if (tid == 32 && XBUF < nblk) load_x(XBUF);   // stage 0 has been read
            if (tid == 0) mbar_arrive_local(barP);
        }
        // while the MMAs of earlier blocks run: the cumsum, x' and x'w of block m, into the x' and
        // cumsum slots the consumer released after block m-3 and the x'w slot the MMAs of block
        // m-2 have finished with
        for (int64_t m = 1; m < nblk; ++m) {
            if (tid >= kScan0) {
                if (m >= 3 && tid == kScan0 && ok && !mbar_wait_bounded(barE2 + 8 * s3(m), p3(m - 3), kWaitLimit))
                    ok = false;
                named_sync(kBarScan, 128);
                scan_block(m);
            }
            if (tid == 0) {
                if (m >= 3 && ok && !mbar_wait_bounded(barE2 + 8 * s3(m), p3(m - 3), kWaitLimit)) ok = false;
                if (m >= 2 && ok && !mbar_wait_bounded(barW + 8 * (uint32_t)(m & 1), (uint32_t)(((m - 2) >> 1) & 1), kWaitLimit))
                    ok = false;
            }
            if (ok && !wait_x(m)) ok = false;
            named_sync(kBarProd, kProd);
            conv_x(m);
            fence_async_smem();
            named_sync(kBarProd, kProd);
            if (tid == 32 && m + XBUF < nblk) load_x(m + XBUF);   // its stage has been read
            if (tid == 0) mbar_arrive_local(barP + 8 * s3(m));
        }
        // final conv state of the head's x channels: the last three raw inputs. Of a row run as
        // pieces only the last piece writes it, and only once the earlier launches are done: a
        // short piece's producer can finish before them, and a first piece may still have to read
        // the initial conv state that the final one overwrites in place.
        const int len_last = nblk > 0 ? blen(nblk - 1) : 0;
        const bool row_end = pc.npieces == 1 || k0 * kT + seqlen >= p.L;
        if (pc.npieces > 1 && row_end) asm volatile("griddepcontrol.wait;" ::: "memory");
        named_sync(kBarProd, kProd);
        for (int e = tid; e < 3 * kP && row_end; e += kProd) {
            const int kk = e / kP, c = e % kP;
            const uint4* stl = stage + (nblk > 0 ? ((nblk - 1) % XBUF) * kStageU4 : 0);
            const __nv_bfloat16 v =
                reinterpret_cast<const __nv_bfloat16*>(stl + stage_u4(kStageTok - 3 + len_last + kk, c / 8))[c % 8];
            ((__nv_bfloat16*)p.final_conv)[(sidx * Cc + (int64_t)h * kP + c) * 3 + kk] = v;
        }
        // the group's first head also writes the B/C part: the last three raw inputs (with the
        // initial state in front when the sequence is shorter than three tokens). The B/C pass
        // has read the initial state before this kernel started, and each thread reads its
        // channel's three values before writing them, so the final state may share memory with
        // the initial one.
        if (h == g * rpg && row_end) {
            for (int c = tid; c < 2 * kN; c += kProd) {
                const bool isC = c >= kN;
                const int64_t ch = (isC ? GN : 0) + (int64_t)g * kN + (c % kN);   // within [B | C]
                const __nv_bfloat16* src = (const __nv_bfloat16*)(isC ? p.C : p.B) + (ch - (isC ? GN : 0));
                const int64_t ld = isC ? p.C_ld : p.B_ld;
                const __nv_bfloat16* ic = (const __nv_bfloat16*)p.init_conv + (sidx * Cc + HP + ch) * 3;
                __nv_bfloat16 v3[3];
#pragma unroll
                for (int kk = 0; kk < 3; ++kk) {
                    const int64_t idx = seqlen + kk;   // into [initial state (3) ; tokens]
                    if (idx < 3 && !piece_cont) v3[kk] = init_conv ? ic[idx] : __float2bfloat16_rn(0.0f);
                    else v3[kk] = src[(row0 + idx - 3) * ld];
                }
                __nv_bfloat16* fc = (__nv_bfloat16*)p.final_conv + (sidx * Cc + HP + ch) * 3;
#pragma unroll
                for (int kk = 0; kk < 3; ++kk) fc[kk] = v3[kk];
            }
        }
    } else if (!consumer) {
        // ============ control (warp 7, one lane): B'/C' by TMA and every MMA ============
        if (tid == kCtl) {
            const uint32_t id_cb = idesc_bf16(128, 128, 0, 0);
            const uint32_t id_ys = idesc_bf16(128, 64, 0, 1);
            const uint32_t id_s = idesc_bf16(128, 64, 1, 1);
            const uint32_t id_yi = idesc_bf16(128, 64, 0, 1);
            // B' (and C') of block kb: [16 vectors][128 tokens][8] each, straight into the operand
            // layout; tokens past the end of the call read as zeros
            // (the B/C pass wrote each as one contiguous chunk of the workspace; rows past the
            // sequence's end are zeros there)
            auto load_bc = [&](int64_t kb) {
                constexpr uint32_t kChunk = (uint32_t)kT * kN * 2;
                mbar_arrive_expect_tx(barBC, (STATE_ONLY ? 1u : 2u) * kChunk);
                const int64_t ci = ((bi + row0 / kT + kb) * 2) * p.G + g;
                const unsigned char* cB = (const unsigned char*)p.bcp + ci * (int64_t)kChunk;
                if (SSD_IN_BOUNDS(p.status, ci + p.G < (int64_t)prefill_bc_blocks(p.b, p.rows()) * 2 * p.G)) {
                    bulk_load(aB, cB, kChunk, barBC);
                    if (!STATE_ONLY) bulk_load(aC, cB + (int64_t)p.G * kChunk, kChunk, barBC);
                } else {   // nothing lands: complete the expected bytes so no wait is left hanging
                    mbar_arrive_expect_tx(barBC, 0u);
                }
            };
            if (nblk > 0) load_bc(0);
            // M x' of block kb, once every consumer warp has written its rows of M
            auto mma_yi = [&](int64_t kb) {
                if (ok && !mbar_wait_bounded(barM, (uint32_t)(kb & 1), kWaitLimit)) ok = false;
                fence_after_sync();
                const uint32_t aXs = aX + 16384 * s3(kb);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + kColYi, tmem + kColM + kk * 8, sdesc(aXs + kk * 2048, 1024, 128), id_yi, kk > 0);
                mma_commit(bar1);
            };
            for (int64_t k = 0; k < nblk; ++k) {
                const int sl = (int)(k & 1);
                const uint32_t par = (uint32_t)(k & 1);
                if constexpr (!STATE_ONLY) {
                    if (k >= 1) mma_yi(k - 1);   // also: C'B'^T of block k-1 has been read
                    // C'B'^T of this block as soon as its B' and C' are in
                    if (ok && !mbar_wait_bounded(barBC, par, kWaitLimit)) ok = false;
                    fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + kColCB, sdesc(aC + kk * 4096, 2048, 128), sdesc(aB + kk * 4096, 2048, 128), id_cb, kk > 0);
                    mma_commit(barCB);
                } else {
                    if (ok && !mbar_wait_bounded(barBC, par, kWaitLimit)) ok = false;
                }
                // this block's x'w (barP); the consumer has read S^T of block k-1 and written H^T
                // for this block (barH)
                if (ok && !mbar_wait_bounded(barP + 8 * s3(k), p3(k), kWaitLimit)) ok = false;
                if (ok && !mbar_wait_bounded(barH, (uint32_t)(k & 1), kWaitLimit)) ok = false;
                fence_after_sync();
                const uint32_t colYs = kColYs0 + 64 * (uint32_t)sl;
                const uint32_t aXWs = aXW + 16384 * (uint32_t)sl;
                if constexpr (!STATE_ONLY) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16(tmem + colYs, sdesc(aC + kk * 4096, 2048, 128), sdesc(aH + kk * 2048, 1024, 128), id_ys, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + kColS, sdesc(aB + kk * 256, 128, 2048), sdesc(aXWs + kk * 2048, 1024, 128), id_s, kk > 0);
                mma_commit(bar0);
                mma_commit(barW + 8 * (uint32_t)sl);   // x'w of this block is free once they are done
                // B'/C' are free once all three products of this block are done (a commit covers
                // every earlier MMA of this thread): the next block's come in meanwhile
                if (k + 1 < nblk) {
                    if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
                    load_bc(k + 1);
                }
            }
            if constexpr (!STATE_ONLY) {
                if (nblk > 0) mma_yi(nblk - 1);
            }
        }
    } else if constexpr (STATE_ONLY) {
        // ================= consumer of the state-only pass (warps 8..15) =================
        init_state();
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float lam_tot = 0.0f;   // sum of delta*A over the row, log2 units
        for (int64_t k = 0; k < nblk; ++k) {
            const uint32_t par = (uint32_t)(k & 1);
            if (ok && !mbar_wait_bounded(barP + 8 * s3(k), p3(k), kWaitLimit)) ok = false;
            if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
            fence_after_sync();
            const float lam_end = s_lam[s3(k) * kT + kT - 1];
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
            named_sync(kBarCons, kThreads - kCons);
            if ((tid & 31) == 0) mbar_arrive_local(barH);   // S^T read: the next block's MMA may overwrite it
            if (tid == kCons) mbar_arrive_local(barE2 + 8 * s3(k));   // the cumsum slot is free
        }
        float* fs = p.final_ssm + (sidx * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < 32; ++i) fs[(int64_t)(chalf * 32 + i) * kN + crow] = H[i];
        if (tid == kCons && p.decay) p.decay[bi * p.H + h] = ex2(lam_tot);
    } else {
        // =========================== consumer (warps 8..15) ===========================
        init_state();
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t aY = s_base + Lo::OFF_Y;
        // byte offset of 16-byte chunk c of token row r in the swizzled y tile
        auto ty_off = [](int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); };
        // this thread's 32 channels of z for token crow of block kb: 16-byte loads nv of its four
        // pieces from v0 on, issued well before the epilogue uses them (rows past the block's end
        // read as zeros)
        auto load_z = [&](int64_t kb, uint4* zr, int v0, int nv) {
            if (crow < blen(kb) && SSD_IN_BOUNDS(p.status, row0 + kb * kT + crow < p.rows())) {
                const uint4* zrow = reinterpret_cast<const uint4*>((const __nv_bfloat16*)p.z +
                                                                   (row0 + kb * kT + crow) * p.z_ld + h * kP + chalf * 32);
#pragma unroll
                for (int v = 0; v < nv; ++v) zr[v0 + v] = zrow[v0 + v];
            } else {
#pragma unroll
                for (int v = 0; v < nv; ++v) zr[v0 + v] = make_uint4(0u, 0u, 0u, 0u);
            }
        };
        // this thread's 32 output channels of token crow into the y tile, then (thread kCons,
        // after every consumer thread) one TMA store of the block's [128 x 64] box. The tile is
        // free again once the previous store has read it out, which thread kCons waits for
        // before a named barrier that precedes every call.
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
                if (!rows_only) *reinterpret_cast<uint4*>(ty + ty_off(crow, chalf * 4 + v)) = make_uint4(w[0], w[1], w[2], w[3]);
                else if (crow < blen(kb) && SSD_IN_BOUNDS(p.status, row0 + kb * kT + crow < p.rows()))
                    yrow[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (rows_only) return;
            fence_async_smem();
            named_sync(kBarCons, kThreads - kCons);
            if (tid == kCons) {
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
        if (tid == kCons && nblk > 0) tma_prefetch_3d(&maps.z, h * kP, tmap_t0, tmap_b);
        for (int64_t k = 0; k < nblk; ++k) {
            const int64_t t0 = k * kT;
            const int len = blen(k);
            const int sl = (int)(k & 1);
            const uint32_t par = (uint32_t)(k & 1);
            // z of the next block into L2 now, so that its loads below do not wait on HBM
            if (tid == kCons && k + 1 < nblk) tma_prefetch_3d(&maps.z, h * kP, tmap_t0 + (int)((k + 1) * kT), tmap_b);
            if (ok && !mbar_wait_bounded(barP + 8 * s3(k), p3(k), kWaitLimit)) ok = false;
            if (ok && !mbar_wait_bounded(barCB, par, kWaitLimit)) ok = false;
            fence_after_sync();
            // expect the peers' sums of squares of block k (2 floats per row from every CTA)
            if constexpr (!SPLIT) {
                if (tid == kCons) mbar_arrive_expect_tx(barN3 + 8 * (uint32_t)(k % 3), (uint32_t)(R * 2 * 128 * 4));
            }
            const float* lamb = s_lam + s3(k) * kT;
            const float* dlb = s_dl + s3(k) * kT;
            const float* vb = s_v + s3(k) * kT;
            const float lam_end = lamb[kT - 1];
            uint4 zr[4];
            // masked, decayed M (row crow, columns chalf*64 .. +64) as bf16 pairs into TMEM. Every
            // 8-column vector takes the same arithmetic (the causal mask is applied afterwards, to
            // the vectors on or above the diagonal only), so the warps that hold the diagonal do
            // not run several paths one after another.
            {
                const int i = crow;
                const float li = lamb[i];
                // rows with lam_i > -96: exp2(lam_i - lam_j) = exp2(lam_i) * exp2(-lam_j), every
                // factor a normal fp32 number; the choice uses only the row's own past, so outputs
                // stay causal bit for bit
                const bool fac = li > -96.0f;
                const float2 u2 = splat2(ex2(li));
                const float* gb = s_g + s3(k) * kT;
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    float cb[32];
                    tmem_ld32(tmem + lane_base + kColCB + chalf * 64 + part * 32, cb);
                    tmem_wait_ld();
                    uint32_t w[16];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int j0 = chalf * 64 + part * 32 + v * 8;
                        float2 m[4];
                        if (fac) {
                            const float2* v2 = reinterpret_cast<const float2*>(vb + j0);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                m[e] = mul2(make_float2(cb[v * 8 + 2 * e], cb[v * 8 + 2 * e + 1]), mul2(u2, v2[e]));
                        } else if (lamb[j0] - lamb[j0 + 7] < 100.0f) {
                            // by 8-token segments: one exp2 per segment (it overflows only above the
                            // diagonal, which the mask clears)
                            const float2 sg = splat2(ex2(li - lamb[j0]));
                            const float2* g2 = reinterpret_cast<const float2*>(gb + j0);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                m[e] = mul2(make_float2(cb[v * 8 + 2 * e], cb[v * 8 + 2 * e + 1]), mul2(sg, g2[e]));
                        } else {
                            // a segment whose own decay leaves the fp32 range: element by element
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = j0 + 2 * e;
                                m[e] = make_float2(cb[v * 8 + 2 * e] * ex2(li - lamb[j]) * dlb[j],
                                                   cb[v * 8 + 2 * e + 1] * ex2(li - lamb[j + 1]) * dlb[j + 1]);
                            }
                        }
                        if (j0 + 7 > i) {   // on or above the diagonal
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                if (j0 + 2 * e > i) m[e].x = 0.0f;
                                if (j0 + 2 * e + 1 > i) m[e].y = 0.0f;
                                // groups held by a cluster: the D skip rides on the diagonal, so M x'
                                // gives D x'_i too and the epilogue reads no x' (the wide-group variant
                                // is at its register limit and keeps D x' in the epilogue)
                                if constexpr (!SPLIT) {
                                    if (j0 + 2 * e == i) m[e].x += Dh;
                                    if (j0 + 2 * e + 1 == i) m[e].y += Dh;
                                }
                            }
                        } else if (!SPLIT && j0 + 7 == i) {
                            m[3].y += Dh;
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) w[4 * v + e] = pack_f2(m[e]);
                    }
                    tmem_st16(tmem + lane_base + kColM + chalf * 32 + part * 16, w);
                }
            }
            // this warp's rows of M are in TMEM and its C'B'^T rows read: once all eight warps have
            // arrived the control thread issues M x', which runs during the state update
            tmem_wait_st();
            fence_before_sync();
            __syncwarp();
            if ((tid & 31) == 0) mbar_arrive_local(barM);
            load_z(k, zr, 0, 4);   // from L2 (prefetched a block ahead), in flight through the state update
            // S^T of this block is in TMEM, and C'H^T of this block has read H^T
            if (ok && !mbar_wait_bounded(bar0, par, kWaitLimit)) ok = false;
            fence_after_sync();

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
            // S^T read and H^T of block k+1 written (generic stores made visible to the tensor
            // cores): the next block's MMAs may start
            fence_async_smem();
            fence_before_sync();
            __syncwarp();
            if ((tid & 31) == 0) mbar_arrive_local(barH);
            if constexpr (!SPLIT) {
                if (k >= 1) finish_norm(k - 1);   // overlaps the MMA M x' of this block
            }
            if (ok && !mbar_wait_bounded(bar1, par, kWaitLimit)) ok = false;
            fence_after_sync();
            // epilogue: y = Yi + exp(lam_i) Ys + D x', gate; two halves of 16 columns
            float gt[32];
            {
                const int i = crow;
                const float2 el = splat2(ex2(lamb[i])), d2 = splat2(SPLIT ? Dh : 0.0f);
                const unsigned char* sX = smem + Lo::OFF_X + s3(k) * 16384;
                float2 ss2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float yi[16], ys[16];
                    tmem_ld16(tmem + lane_base + kColYi + chalf * 32 + hf * 16, yi);
                    tmem_ld16(tmem + lane_base + kColYs0 + 64 * sl + chalf * 32 + hf * 16, ys);
                    tmem_wait_ld();
#pragma unroll
                    for (int vv = 0; vv < 2; ++vv) {
                        const int v = hf * 2 + vv;
                        const uint4 xw = SPLIT ? *reinterpret_cast<const uint4*>(sX + canon_off(i, chalf * 32 + 8 * v, kP))
                                               : make_uint4(0u, 0u, 0u, 0u);
                        const uint4 zv = zr[v];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 8 * vv + 2 * e;
                            float2 y = fma2(el, make_float2(ys[c], ys[c + 1]), make_float2(yi[c], yi[c + 1]));
                            if constexpr (SPLIT) y = fma2(d2, bf2_to_f2((&xw.x)[e]), y);
                            const float2 gg = mul2(y, silu2(bf2_to_f2((&zv.x)[e])));
                            gt[8 * v + 2 * e] = gg.x;
                            gt[8 * v + 2 * e + 1] = gg.y;
                            ss2 = fma2(gg, gg, ss2);
                        }
                    }
                }
                const float ss = ss2.x + ss2.y;
                if constexpr (SPLIT) {
                    if (i < len && SSD_IN_BOUNDS(p.status, row0 + t0 + i < p.rows()))
                        p.ssp[((row0 + t0 + i) * p.H + h) * 2 + chalf] = ss;
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
            if (tid == kCons) bulk_wait_read_all();   // the last y store has left the y tile
            named_sync(kBarCons, kThreads - kCons);
            if (tid == kCons) mbar_arrive_local(barE2 + 8 * s3(k));   // the x' and cumsum slots are free
            if constexpr (SPLIT) store_y(k, gt, 1.0f, false);
        }
        if constexpr (!SPLIT) {
            if (nblk >= 1) {
                if (tid == kCons) bulk_wait_read_all();
                named_sync(kBarCons, kThreads - kCons);
                finish_norm(nblk - 1);
            }
        }
        if (tid == kCons) bulk_wait_all();   // the y stores have completed
        // final SSM state of this head
        float* fs = p.final_ssm + (sidx * p.H + h) * (int64_t)kP * kN;
#pragma unroll
        for (int i = 0; i < 32; ++i) fs[(int64_t)(chalf * 32 + i) * kN + crow] = H[i];
    }

    if (!ok) set_device_status(p.status, kDevTimeout);
    // a launch of pieces completes only after the launch before it, so a piece whose predecessor
    // ran several launches back still finds its state written
    if (pc.npieces > 1 && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    cluster.sync();   // no peer still arrives on this CTA's shared memory
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Group RMSNorm of the gated values written by the SPLIT kernel (2 partial sums per head):
// one warp per (token, group), each lane streaming 16-byte pieces of the group's row, four in
// flight at a time.
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
    const bool nw16 = ((uintptr_t)nw & 15u) == 0;
    constexpr int kU = 4;
    for (int c0 = lane * 8; c0 < gs; c0 += 256 * kU) {
        uint4 raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (c0 + u * 256 < gs) raw[u] = *reinterpret_cast<const uint4*>(y + c0 + u * 256);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int c = c0 + u * 256;
            if (c >= gs) break;
            float v[8], wv[8];
            unpack_bf16x8(raw[u], v);
            if (nw16) {
                const float4 a = *reinterpret_cast<const float4*>(nw + c), b = *reinterpret_cast<const float4*>(nw + c + 4);
                wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w; wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) wv[e] = nw[c + e];
            }
            uint4 o;
            o.x = pack_bf16x2(v[0] * inv * wv[0], v[1] * inv * wv[1]);
            o.y = pack_bf16x2(v[2] * inv * wv[2], v[3] * inv * wv[3]);
            o.z = pack_bf16x2(v[4] * inv * wv[4], v[5] * inv * wv[5]);
            o.w = pack_bf16x2(v[6] * inv * wv[6], v[7] * inv * wv[7]);
            *reinterpret_cast<uint4*>(y + c) = o;
        }
    }
}

// The group RMS scale of every (token, group) from the SPLIT kernel's partial sums, for a
// caller that applies the norm itself (the out_proj prologue of the mixer layer):
// scale[row][g] = 1 / sqrt(mean over the group of g^2 + eps).
__global__ void __launch_bounds__(256) ws_norm_scale_kernel(PrefillParams p, float* scale)
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
    if (lane == 0) scale[w] = rsqrtf(s / (float)gs + p.eps);
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

// [b][L][width] bf16 rows of `ld` elements; boxes of 64 channels x `rows` tokens x 1 sequence,
// 128-byte swizzled in shared memory.
bool encode_tile(CUtensorMap* m, const void* base, int64_t width, int64_t ld, int64_t L, int64_t b, int rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)L, (cuuint64_t)b};
    const cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(L * ld * 2)};
    const cuuint32_t box[3] = {(cuuint32_t)kP, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The B/C conv pass (the main kernel reads only the x part of the initial conv state).
cudaError_t launch_bc_conv(const PrefillParams& p, int nch, cudaStream_t st)
{
    const int64_t rows = p.rows();
    if (rows == 0) return cudaSuccess;
    LaunchScope ls("tc_bc_conv", st);
    const dim3 grid((unsigned)prefill_bc_blocks(p.b, rows), (unsigned)(nch / 64));
    bc_conv_kernel<<<grid, 256, 0, st>>>(p, nch);
    return cudaGetLastError();
}

// Pieces per row for `jobs` rows of `nblk` blocks, one CTA per SM on `sms` SMs: whole rows
// leave the last wave part-empty (256 rows on 148 SMs run as two waves, the second 108 wide).
// The plan minimises launches x (blocks per piece + about 1.5 blocks for the fill and drain of
// a launch's pipelines); with fewer rows than SMs it keeps rows whole. The environment
// variable SSD_MIXER_PREFILL_PIECES (read once; 1 .. 64) fixes the number of pieces instead.
WsPieces plan_pieces(int64_t jobs, int64_t nblk, int sms)
{
    static const int forced = [] {
        const char* v = getenv("SSD_MIXER_PREFILL_PIECES");
        const int n = v ? atoi(v) : 0;
        return n >= 1 && n <= 64 ? n : 0;
    }();
    const WsPieces whole{0, (int)jobs, 1, (int)nblk};   // one launch, every row whole
    if (nblk < 2 || (!forced && jobs < sms)) return whole;
    WsPieces pc{0, (int)std::min((int64_t)sms, jobs), 1, (int)nblk};
    double best = 0.0;
    for (int n = forced ? forced : 1; n <= (forced ? forced : 8) && n <= nblk; ++n) {
        const int64_t pb = (nblk + n - 1) / n, np = (nblk + pb - 1) / pb;
        const int64_t launches = (jobs * np + sms - 1) / sms;
        const double cost = (double)launches * ((double)pb + 1.5);
        if (n == (forced ? forced : 1) || cost < best) {
            best = cost;
            pc.npieces = (int)np;
            pc.piece_blocks = (int)pb;
        }
    }
    return pc.npieces > 1 ? pc : whole;
}

int sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        return 148;
    return sms;
}

template <int R, bool SPLIT, bool STATE_ONLY = false>
cudaError_t launch_ws(const PrefillParams& p, cudaStream_t st)
{
    using Lo = WsLayout<R>;
    cudaError_t e = launch_bc_conv(p, STATE_ONLY ? (int)p.GN() : (int)(2 * p.GN()), st);
    if (e != cudaSuccess) return e;
    WsMaps maps;
    memset(&maps, 0, sizeof(maps));
    // packed sequences: one row of all the packed tokens
    const int64_t mL = p.L, mb = p.cu_seqlens ? 1 : p.b;
    if (p.L > 0) {   // no block, no load: the maps stay unused
        if (!encode_tile(&maps.x, p.x, p.HP(), p.x_ld, mL, mb, kStageRows)) return cudaErrorInvalidValue;
        if (!STATE_ONLY && (!encode_tile(&maps.y, p.y, p.HP(), p.y_ld, mL, mb, kT) ||
                            !encode_tile(&maps.z, p.z, p.HP(), p.z_ld, mL, mb, kT)))
            return cudaErrorInvalidValue;
    }
    e = cudaFuncSetAttribute(ssd_prefill_ws_kernel<R, SPLIT, STATE_ONLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Lo::TOTAL);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.b * p.H));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Lo::TOTAL;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one CTA per SM (R = 1, no cluster): rows of fixed length may run as pieces, each launch
    // after the first allowed to start while the one before it finishes
    const int64_t jobs = p.b * p.H / R;
    WsPieces pc{0, (int)jobs, 1, 0};
    if (R == 1 && !STATE_ONLY && !p.cu_seqlens) pc = plan_pieces(jobs, (p.L + kT - 1) / kT, sm_count());
    const int64_t total = jobs * pc.npieces;
    {
        LaunchScope ls(STATE_ONLY ? "tc_prefill_state" : "tc_prefill", st, (int)((total + pc.per_round - 1) / pc.per_round));
        for (pc.round = 0; (int64_t)pc.round * pc.per_round < total; ++pc.round) {
            cfg.gridDim = dim3((unsigned)(R * std::min((int64_t)pc.per_round, total - (int64_t)pc.round * pc.per_round)));
            cfg.numAttrs = pc.round > 0 ? 2 : 1;
            e = cudaLaunchKernelEx(&cfg, ssd_prefill_ws_kernel<R, SPLIT, STATE_ONLY>, p, maps, pc);
            if (e != cudaSuccess) return e;
        }
    }
    if (SPLIT && !STATE_ONLY && p.rows() > 0 && !p.defer_norm) {
        LaunchScope ls("tc_norm_finish", st);
        const int64_t warps = p.rows() * p.G;
        ws_norm_finish_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace

// The state-only pass needs no norm and so no cluster.
cudaError_t launch_prefill_state_ws(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    return launch_ws<1, false, true>(p, stream);
}

PrefillPlan prefill_ws_plan(int64_t b, int64_t L, int H, int G, int sms)
{
    const int r = H / G, R = (r == 2 || r == 4) ? r : 1;
    const int64_t jobs = b * H / R, nblk = (L + kT - 1) / kT;
    const WsPieces pc = R == 1 ? plan_pieces(jobs, nblk, sms) : WsPieces{0, (int)jobs, 1, (int)nblk};
    const int64_t total = jobs * pc.npieces;
    return PrefillPlan{(int)((total + pc.per_round - 1) / std::max(1, pc.per_round)), pc.npieces, pc.piece_blocks,
                       pc.per_round * R};
}

int device_sm_count() { return sm_count(); }

// Groups of 2 or 4 heads: one cluster per group, the norm fused; wider groups: no cluster,
// the norm finished by ws_norm_finish_kernel.
cudaError_t launch_prefill_ws(const PrefillParams& p, cudaStream_t stream)
{
    if (p.b == 0) return cudaSuccess;
    switch (p.H / p.G) {
    case 2: return launch_ws<2, false>(p, stream);
    case 4: return launch_ws<4, false>(p, stream);
    }
    return launch_ws<1, true>(p, stream);
}

int prefill_ws_partials_per_head() { return 2; }

cudaError_t launch_norm_scale(const PrefillParams& p, float* scale, cudaStream_t stream)
{
    if (p.rows() == 0) return cudaSuccess;
    LaunchScope ls("tc_norm_scale", stream);
    const int64_t warps = p.rows() * p.G;
    ws_norm_scale_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(p, scale);
    return cudaGetLastError();
}

bool prefill_tc_supported(int act, int P, int N, int H, int G)
{
    const int r = H / G;
    return act == 1 && P == kP && N == kN && (r == 2 || (r % 4 == 0 && r <= 256));
}

bool prefill_tc_split(int H, int G) { return H / G > 4; }

}  // namespace ssd
