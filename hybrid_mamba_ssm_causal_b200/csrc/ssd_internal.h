// ssd_internal.h -- launch parameters shared by the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define SSD_HD __host__ __device__
#else
#define SSD_HD
#endif

namespace ssd {

// Values of the device status word at the start of a prefill workspace. The host clears it
// (cudaMemsetAsync on the call's stream) before the call's first kernel; a kernel that meets
// a failure records its code with set_device_status, and the first failure of a call is kept.
enum DeviceStatus : int {
    kDevOk = 0,
    kDevTimeout = 1,          // a bounded wait (mbarrier, peer copy, tensor-core commit) gave up
    kDevSmemMisaligned = 2,   // the dynamic shared memory base lacked the alignment the kernel needs
    kDevBounds = 3,           // (bounds-checked build) an index fell outside its buffer; access skipped
};
#ifdef __CUDACC__
__device__ __forceinline__ void set_device_status(int* status, int code) { atomicCAS(status, 0, code); }
// SSD_IN_BOUNDS(status, cond): in the bounds-checked build (compiled with -DSSD_DEBUG_BOUNDS,
// libssd_mixer_debug.so) a false cond records kDevBounds in the status word and the guarded
// access is skipped, so a bad index is reported instead of faulting; in the normal build it is
// `true` and cond is not evaluated.
#ifdef SSD_DEBUG_BOUNDS
__device__ __forceinline__ bool ssd_in_bounds(int* status, bool ok)
{
    if (!ok) set_device_status(status, kDevBounds);
    return ok;
}
#define SSD_IN_BOUNDS(status, cond) ::ssd::ssd_in_bounds((status), (cond))
#else
#define SSD_IN_BOUNDS(status, cond) true
#endif
#endif
// Clears the status word of a call's workspace on its stream.
inline cudaError_t clear_device_status(int* status, cudaStream_t st)
{
    return cudaMemsetAsync(status, 0, sizeof(int), st);
}

// Everything one prefill call needs, validated by the ABI layer.
struct PrefillParams {
    int64_t b, L;        // batch rows, tokens per row
    int H, P, G, N, K, Q;
    float eps;
    int act;             // 0 = fp32, 1 = bf16
    int64_t nc;          // chunks per row = ceil(L / Q)
    const void *x, *z, *B, *C, *dt;
    int64_t x_ld, z_ld, B_ld, C_ld, dt_ld;
    const float *A, *D, *conv_w, *conv_b, *dt_bias, *norm_w;
    const float* init_ssm;   // [b][H][P][N] or nullptr
    const void* init_conv;   // [b][Cc][K-1] or nullptr
    void* y;
    int64_t y_ld;
    float* final_ssm;
    void* final_conv;
    // workspace regions (carved by the ABI layer)
    int* status;     // device status word
    void* xbc;       // [b][L][Cc] activated x|B|C, activation dtype
    float* delta;    // [b][H][L]
    float* lam;      // [b][H][L] within-chunk inclusive cumsum of delta*A
    float* states;   // [b][nc][H][P][N] chunk states, then states entering each chunk
    float* ypre;     // [b][L][HP] y before the gate and norm
    float* ssp;      // tensor-core path, groups wider than one cluster: [rows][H][parts] sums of g^2
    void* bcp;       // tensor-core path: SiLU(conv) of the B and C channels, bf16, blocked (see
                     // prefill_bc_blocks)
    // Packed variable-length sequences on state slots (cu_seqlens != nullptr): b sequences,
    // L = total packed tokens, sequence i owns rows cu_seqlens[i] .. cu_seqlens[i+1]-1; its
    // states are the slot slot_idx[i] (identity when null) of init_ssm/init_conv, which
    // alias final_ssm/final_conv; has_init[i] == 0 starts it from zero states.
    const int32_t* cu_seqlens;
    const int32_t* slot_idx;
    const uint8_t* has_init;
    // state-only pass (ssd_mixer_prefill_state): exp(sum_t delta_t * A) per (row, head), [b][H]
    float* decay;
    // tensor-core path, groups wider than one cluster: leave y gated but not normalised and keep
    // the partial sums of squares in the workspace (the caller finishes the norm)
    bool defer_norm;

    SSD_HD int64_t HP() const { return (int64_t)H * P; }
    SSD_HD int64_t GN() const { return (int64_t)G * N; }
    SSD_HD int64_t Cc() const { return HP() + 2 * GN(); }
    SSD_HD int64_t rows() const { return cu_seqlens ? L : b * L; }   // token rows of x, z, y, ...
};

struct DecodeParams {
    int64_t b;
    int H, P, G, N, K;
    float eps;
    int act;
    const void *x, *z, *B, *C, *dt;
    int64_t x_ld, z_ld, B_ld, C_ld, dt_ld;
    const float *A, *D, *conv_w, *conv_b, *dt_bias, *norm_w;
    float* ssm_state;
    void* conv_state;
    const int32_t* slot_idx;
    void* y;
    int64_t y_ld;

    SSD_HD int64_t HP() const { return (int64_t)H * P; }
    SSD_HD int64_t GN() const { return (int64_t)G * N; }
    SSD_HD int64_t Cc() const { return HP() + 2 * GN(); }
};

// Workspace layout of one prefill call; offsets in bytes, each 256-byte aligned.
struct WorkspaceLayout {
    size_t status, xbc, delta, lam, states, ypre, ssp, bcp, total;
};
// rows = token rows of one call (b*L, or the packed total of a variable-length call).
WorkspaceLayout prefill_workspace_layout(int64_t b, int64_t L, int64_t rows, int H, int P, int G, int N,
                                         int Q, int act);
// The CUDA-core path's layout (every intermediate in the workspace), whatever the shape.
WorkspaceLayout simt_workspace_layout(int64_t b, int64_t L, int H, int P, int G, int N, int Q, int act);

// ---- backward pass (ssd_backward.cu)
// The backward reruns the CUDA-core forward with 64-token chunks (the state entering each one
// is kept in the workspace); its scan recomputes the states of a chunk 16 tokens at a time.
constexpr int kBackwardForwardChunk = 64;
constexpr int kBackwardChunk = 16;
// State rows p handled by one CTA of the backward scan (so P / 16 row blocks per head).
constexpr int kBackwardRows = 16;

struct BackwardParams {
    PrefillParams f;              // the forward's inputs; its workspace regions (chunk Q = 64)
    const void* dout;             // [b][L][HP] gradient of y, activation dtype
    int64_t dout_ld;
    const float* dfinal_ssm;      // [b][H][P][N] or nullptr
    const float* dfinal_conv;     // [b][Cc][K-1] or nullptr
    void *dx, *dz, *dB, *dC, *ddt;   // activation dtype, row strides below
    int64_t dx_ld, dz_ld, dB_ld, dC_ld, ddt_ld;
    float *dA, *dD, *dconv_w, *dconv_b, *ddt_bias, *dnorm_w;   // written (zeroed, then summed into)
    float* dinit_ssm;             // [b][H][P][N] or nullptr
    float* dinit_conv;            // [b][Cc][K-1] or nullptr
    // workspace
    float* dy;                    // [b][L][HP] gradient of y before the gate
    float* dxs;                   // [b][L][HP] gradient of x'
    float* dBp;                   // [b][L][H][P/16][N] partial gradients of B' (per head, row block)
    float* dCp;                   // [b][L][H][P/16][N] partial gradients of C'
    float* ddp;                   // [b][H][P/16][L] partial gradients of delta
};

struct BackwardLayout {
    WorkspaceLayout fwd;          // the recompute forward's regions
    size_t y, final_ssm, final_conv;   // the recompute forward's outputs (not returned)
    size_t dy, dxs, dBp, dCp, ddp, total;
};
BackwardLayout backward_workspace_layout(int64_t b, int64_t L, int H, int P, int G, int N, int act);
bool backward_supported(int P, int N);
cudaError_t launch_backward(const BackwardParams& p, cudaStream_t stream);

// Tensor-core path (ssd_prefill_ws.cu): bf16 activations, P = 64, N = 128, 2 or a multiple
// of 4 heads per group. Its workspace holds the status word, SiLU(conv) of the B and C
// channels (computed once for all heads of a group), and per-(token, head) partial sums of
// squares when the group is wider than one cluster (prefill_tc_split).
bool prefill_tc_supported(int act, int P, int N, int H, int G);
bool prefill_tc_split(int H, int G);
// scale[row][g] of the group norm from the partial sums a deferred-norm prefill left in p.ssp.
cudaError_t launch_norm_scale(const PrefillParams& p, float* scale, cudaStream_t stream);

// The layer's projections (ssd_gemm.cu): C[M][N] = A[M][K] . W[N][K]^T, bf16 in and out, fp32
// accumulation. With row_scale, A[t][k] is first multiplied by row_scale[t][k / scale_group]
// (and by col_scale[k] when given), scale_group a multiple of 64.
bool gemm_supported(int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldw, int64_t ldc);
cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, const void* W, int64_t ldw,
                             void* C, int64_t ldc, const float* row_scale, int scale_group, int64_t scale_ld,
                             const float* col_scale, int* status, cudaStream_t st);
// The state-only pass on the tensor-core path: final states and decay, no output rows.
cudaError_t launch_prefill_state_ws(const PrefillParams& p, cudaStream_t stream);
cudaError_t launch_prefill_ws(const PrefillParams& p, cudaStream_t stream);
// How the tensor-core main kernel runs a fixed-length call of b rows of L tokens on `sms` SMs:
// launches per call, pieces per (sequence, head) row, 128-token blocks per piece (the last
// piece of a row may be shorter), CTAs per launch (the last launch may have fewer).
struct PrefillPlan {
    int launches, pieces, piece_blocks, ctas_per_launch;
};
PrefillPlan prefill_ws_plan(int64_t b, int64_t L, int H, int G, int sms);
int device_sm_count();
// The tensor-core path keeps SiLU(conv) of B and C in the workspace as 32 KB chunks, one per
// (128-token block of a sequence, matrix B or C, group): chunk ((s + floor(start_s / 128) + k) * 2
// + matrix) * G + group holds block k of sequence s (first packed row start_s) in the MMA operand
// layout [16 vectors of 8 channels][128 tokens][8]. Sequences never share a chunk, and
// prefill_bc_blocks(b, rows) = b + rows / 128 + 1 bounds the block index.
constexpr int64_t kBcBlockTokens = 128;
SSD_HD inline size_t prefill_bc_blocks(int64_t b, int64_t rows) { return (size_t)(b + rows / kBcBlockTokens + 1); }
int prefill_ws_partials_per_head();

// H_in(r) of a sequence split into pieces: init (NULL = zeros) carried through pieces 0..r-1.
cudaError_t launch_state_pass(int64_t b, int H, int P, int N, int r, const float* decay, const float* state,
                              const float* init, float* out, cudaStream_t stream);

bool prefill_simt_supported(int P, int N);
cudaError_t launch_prefill_simt(const PrefillParams& p, cudaStream_t stream);

bool decode_supported(int P, int N);
cudaError_t launch_decode_step(const DecodeParams& p, cudaStream_t stream);

}  // namespace ssd
