// ssd_gemm.cu -- the mixer layer's projections on tcgen05: C[M][N] = A[M][K] . W[N][K]^T in
// bf16 with fp32 accumulation, bf16 out (in_proj: hidden -> [z | x | B | C | dt]; out_proj:
// y -> model width; the layer of gllm PR #86, section "2. feat(model): Nemotron-H on the
// CPU", mixer row M, "in_proj ... out_proj").
//
// Persistent and warp-specialised, one CTA per SM, 128 x 256 output tiles walked N-fastest
// (consecutive tiles share their A rows, and the whole weight matrix stays in L2):
//   warp 0 (one lane) TMA of A [128][64] and W [256][64] K-blocks into a 4-stage ring, landing
//                     in the 128-byte swizzled K-major operand layout (128-byte rows);
//   warp 1 (one lane) tcgen05.mma 128x256x16 into one of two TMEM accumulators (256 columns
//                     each), so the epilogue of a tile overlaps the MMAs of the next;
//   warps 2..5        the epilogue: a TMEM lane (one output row) per thread, 64 columns at a
//                     time into a 128-byte-swizzled staging tile, stored by TMA (double
//                     buffered; rows and columns past the matrix are clipped by the store).
//   warps 6..13       (with a prologue on A only) every A element of row t and column k times
//                     row_scale[t][k / scale_group] and col_scale[k], in shared memory, before
//                     its MMAs (out_proj of a group norm finished late); the K-block's column
//                     scales are staged once in shared memory.
// All waits are bounded; a wait that gives up sets the status word and stops waiting.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_profile.h"
#include "ssd_tc_util.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kGemmThreads = 192, kGemmThreadsScaled = 448;
constexpr uint32_t kABytes = kBM * kBK * 2, kWBytes = kBN * kBK * 2, kStageBytes = kABytes + kWBytes;
constexpr uint32_t kOutChunk = 64;                     // columns per staged store
constexpr uint32_t kOutBytes = kBM * kOutChunk * 2;    // 16 KB
constexpr uint32_t kOffOut = kStages * kStageBytes;    // 2 staging tiles
constexpr uint32_t kOffColScale = kOffOut + 2 * kOutBytes;   // [kStages][64] fp32
constexpr uint32_t kOffBar = kOffColScale + kStages * kBK * 4;
// full[4] empty[4] scaled[4] acc_full[2] acc_empty[2]
constexpr int kNBar = 3 * kStages + 4;
constexpr uint32_t kOffTmem = kOffBar + kNBar * 8;
constexpr uint32_t kGemmSmem = kOffTmem + 16;
static_assert(kGemmSmem <= 232448, "GEMM shared memory above 227 KB");
constexpr long long kGemmWait = 4000000000LL;   // ~2 s at 2 GHz

struct GemmMaps {
    CUtensorMap a, w, c;
};

struct GemmArgs {
    int M, N, K;
    int* status;
    const float* row_scale;   // [M][K / scale_group] or nullptr
    int scale_group;
    int64_t scale_ld;
    const float* col_scale;   // [K] or nullptr (with row_scale only)
};

__device__ __forceinline__ void gemm_named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <bool SCALE>
__global__ void __launch_bounds__(SCALE ? kGemmThreadsScaled : kGemmThreads, 1)
    gemm_bf16_tn_kernel(GemmArgs g, const __grid_constant__ GemmMaps maps)
{
    extern __shared__ __align__(1024) unsigned char smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
    const uint32_t sb = smem_u32(smem);
    auto full = [&](int s) { return smem_u32(&bars[s]); };
    auto empty = [&](int s) { return smem_u32(&bars[kStages + s]); };
    auto scaled = [&](int s) { return smem_u32(&bars[2 * kStages + s]); };
    auto acc_full = [&](int b) { return smem_u32(&bars[3 * kStages + b]); };
    auto acc_empty = [&](int b) { return smem_u32(&bars[3 * kStages + 2 + b]); };

    if (sb & 1023u) {   // the swizzled staging tiles need a 1024-byte aligned base
        if (tid == 0) set_device_status(g.status, kDevSmemMisaligned);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
            mbar_init(scaled(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 1);
        }
        fence_mbar_init();
        prefetch_tmap(&maps.a);
        prefetch_tmap(&maps.w);
        prefetch_tmap(&maps.c);
    }
    if (warp == 0) tmem_alloc(smem_u32(tmem_slot), 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    const int tiles_m = (g.M + kBM - 1) / kBM, tiles_n = (g.N + kBN - 1) / kBN;
    const int ntiles = tiles_m * tiles_n;
    const int nk = (g.K + kBK - 1) / kBK;

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        if (lane == 0) {
            int it = 0;   // K-blocks loaded so far, over all tiles
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
                const int tm = t / tiles_n, tn = t % tiles_n;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && ok && !mbar_wait_bounded(empty(s), (uint32_t)(((it / kStages) - 1) & 1), kGemmWait))
                        ok = false;
                    mbar_arrive_expect_tx(full(s), kStageBytes);
                    const uint32_t dst = sb + (uint32_t)s * kStageBytes;
                    tma_load_3d(dst, &maps.a, kb * kBK, tm * kBM, 0, full(s));
                    tma_load_3d(dst + kABytes, &maps.w, kb * kBK, tn * kBN, 0, full(s));
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer -------------------------------
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kBM, kBN, 0, 0);
            int it = 0, lt = 0;   // K-blocks consumed, tiles done by this CTA
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                // the epilogue has read this accumulator's previous tile
                if (lt >= 2 && ok && !mbar_wait_bounded(acc_empty(b), (uint32_t)(((lt >> 1) - 1) & 1), kGemmWait)) ok = false;
                fence_after_sync();
                const uint32_t d = tmem + (uint32_t)b * kBN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t par = (uint32_t)((it / kStages) & 1);
                    if (ok && !mbar_wait_bounded(SCALE ? scaled(s) : full(s), par, kGemmWait)) ok = false;
                    fence_after_sync();
                    const uint32_t aa = sb + (uint32_t)s * kStageBytes, ww = aa + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16(d, sdesc_sw128(aa + kk * 32), sdesc_sw128(ww + kk * 32), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(empty(s));   // the stage is free once these MMAs are done
                }
                mma_commit(acc_full(b));
            }
        }
    } else if (warp >= 6) {
        // ------------------------------- A prologue (warps 6..13) -------------------------------
        if constexpr (SCALE) {
            const int sid = tid - 192;
            const int r = sid & 127;            // A row of the tile, and which half of its 8 chunks
            const int vh = sid >> 7;
            float* s_cs = reinterpret_cast<float*>(smem + kOffColScale);
            // every global read is issued well before its use: the column scales one K-block
            // ahead, the row's group scale one group ahead
            auto colv = [&](int kcol) { return (sid < kBK && g.col_scale && kcol + sid < g.K) ? g.col_scale[kcol + sid] : 1.0f; };
            const int ngrp = (g.K + g.scale_group - 1) / g.scale_group;
            int it = 0;
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
                const int tm = t / tiles_n;
                const int64_t grow = (int64_t)tm * kBM + r;
                const float* rs = g.row_scale + grow * g.scale_ld;
                auto rowv = [&](int grp) { return (grow < g.M && grp < ngrp) ? rs[grp] : 0.0f; };
                int cur_grp = 0;
                float cur_sc = rowv(0), next_sc = rowv(1);
                float ncs = colv(0);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t par = (uint32_t)((it / kStages) & 1);
                    const int kcol = kb * kBK;
                    float* cs = s_cs + s * kBK;
                    if (sid < kBK) cs[sid] = ncs;
                    if (kb + 1 < nk) ncs = colv(kcol + kBK);
                    const int grp = kcol / g.scale_group;
                    if (grp != cur_grp) {
                        cur_grp = grp;
                        cur_sc = next_sc;
                        next_sc = rowv(grp + 1);
                    }
                    const float sc = cur_sc;
                    if (ok && !mbar_wait_bounded(full(s), par, kGemmWait)) ok = false;
                    gemm_named_sync(2, 256);
                    unsigned char* a = smem + (size_t)s * kStageBytes;
#pragma unroll
                    for (int vv = 0; vv < kBK / 16; ++vv) {   // 16-byte chunk v of row r (128-byte swizzle)
                        const int v = vh * (kBK / 16) + vv;
                        uint4* p = reinterpret_cast<uint4*>(a + r * 128 + ((v ^ (r & 7)) << 4));
                        const float4 c0 = *reinterpret_cast<const float4*>(cs + v * 8);
                        const float4 c1 = *reinterpret_cast<const float4*>(cs + v * 8 + 4);
                        float f[8];
                        unpack_bf16x8(*p, f);
                        *p = make_uint4(pack_bf16x2(f[0] * sc * c0.x, f[1] * sc * c0.y), pack_bf16x2(f[2] * sc * c0.z, f[3] * sc * c0.w),
                                        pack_bf16x2(f[4] * sc * c1.x, f[5] * sc * c1.y), pack_bf16x2(f[6] * sc * c1.z, f[7] * sc * c1.w));
                    }
                    fence_async_smem();
                    gemm_named_sync(2, 256);
                    if (sid == 0) mbar_arrive_local(scaled(s));
                }
            }
        }
    } else {
        // ------------------------------- epilogue (warps 2..5) -------------------------------
        const int q = warp & 3;                 // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;          // output row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int etid = tid - 64;              // 0..127
        int lt = 0, nst = 0;                    // tiles stored, staged chunks issued
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const int tm = t / tiles_n, tn = t % tiles_n;
            const int b = lt & 1;
            if (ok && !mbar_wait_bounded(acc_full(b), (uint32_t)((lt >> 1) & 1), kGemmWait)) ok = false;
            fence_after_sync();
            for (int c = 0; c < kBN / (int)kOutChunk; ++c, ++nst) {
                const int n0 = tn * kBN + c * (int)kOutChunk;
                if (n0 >= g.N) break;
                unsigned char* st = smem + kOffOut + (nst & 1) * kOutBytes;
                // the store issued two chunks ago has read this staging tile
                if (etid == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                gemm_named_sync(1, 128);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float v[32];
                    tmem_ld32(tmem + lane_base + (uint32_t)b * kBN + c * kOutChunk + h * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {   // 16-byte chunk (h * 4 + j) of the row, swizzled by row % 8
                        const uint4 u = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                                   pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
                        const int ch = h * 4 + j;
                        *reinterpret_cast<uint4*>(st + row * 128 + ((ch ^ (row & 7)) << 4)) = u;
                    }
                }
                fence_async_smem();
                gemm_named_sync(1, 128);
                if (etid == 0) {
                    tma_store_3d(&maps.c, smem_u32(st), n0, tm * kBM, 0);
                    bulk_commit();
                }
            }
            // every lane of this accumulator has been read: the MMAs of the tile after next may use it
            fence_before_sync();
            gemm_named_sync(1, 128);
            if (etid == 0) mbar_arrive_local(acc_empty(b));
        }
        if (etid == 0) bulk_wait_all();
    }
    if (!ok) set_device_status(g.status, kDevTimeout);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn gemm_encode_fn()
{
    static EncodeFn fn = []() -> EncodeFn {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeFn>(f);
    }();
    return fn;
}

// A row-major [rows][K] bf16 operand; a box of 64 K x `box_rows` rows lands as 128-byte rows
// with 128-byte swizzling, the K-major operand layout of sdesc_sw128.
bool encode_operand(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int64_t ld, int box_rows)
{
    EncodeFn enc = gemm_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, 1};
    const cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(rows * ld * 2)};
    const cuuint32_t box[3] = {(cuuint32_t)kBK, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The output [M][N] bf16 (row stride ld) for 64-column x 128-row stores, 128-byte swizzled.
bool encode_output(CUtensorMap* m, void* base, int64_t M, int64_t N, int64_t ld)
{
    EncodeFn enc = gemm_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, 1};
    const cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(M * ld * 2)};
    const cuuint32_t box[3] = {kOutChunk, kBM, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

int sm_count()
{
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    }
    return n;
}

}  // namespace

bool gemm_supported(int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldw, int64_t ldc)
{
    return M > 0 && N > 0 && K > 0 && K % 8 == 0 && lda % 8 == 0 && ldw % 8 == 0 && ldc % 8 == 0 && lda >= K &&
           ldw >= K && ldc >= N && M < (1LL << 31) && N < (1LL << 31) && K < (1LL << 31);
}

cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, const void* W, int64_t ldw,
                             void* C, int64_t ldc, const float* row_scale, int scale_group, int64_t scale_ld,
                             const float* col_scale, int* status, cudaStream_t st)
{
    GemmMaps maps;
    memset(&maps, 0, sizeof(maps));
    if (!encode_operand(&maps.a, A, M, K, lda, kBM) || !encode_operand(&maps.w, W, N, K, ldw, kBN) ||
        !encode_output(&maps.c, C, M, N, ldc))
        return cudaErrorInvalidValue;
    GemmArgs g{};
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.status = status;
    g.row_scale = row_scale;
    g.scale_group = scale_group > 0 ? scale_group : 1;
    g.scale_ld = scale_ld;
    g.col_scale = col_scale;
    const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
    if (row_scale) {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
        if (e != cudaSuccess) return e;
        LaunchScope ls("tc_gemm_scaled", st);
        gemm_bf16_tn_kernel<true><<<grid, kGemmThreadsScaled, kGemmSmem, st>>>(g, maps);
    } else {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem);
        if (e != cudaSuccess) return e;
        LaunchScope ls("tc_gemm", st);
        gemm_bf16_tn_kernel<false><<<grid, kGemmThreads, kGemmSmem, st>>>(g, maps);
    }
    return cudaGetLastError();
}

}  // namespace ssd
