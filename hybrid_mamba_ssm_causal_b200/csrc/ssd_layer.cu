// ssd_layer.cu -- the whole Mamba-2 mixer layer on one stream: in_proj, the mixer core and
// out_proj, with the layer's GEMMs on tcgen05 (ssd_gemm.cu).
//
// in_proj emits one packed row per token, split [z | x | B | C | dt] (gllm PR #86, section
// "2. feat(model): Nemotron-H on the CPU", "Supporting changes", on the in_proj output
// [z | xBC | dt]; Modalities PR #459, commit notes on mamba2.py, on the packed [z, x, B, C, dt]
// projection). The core reads x, z, B, C and dt as column slices of that row (its ABI takes a
// row stride for each), so nothing is copied between the GEMM and the core. When the core's
// norm group is wider than a thread-block cluster, the norm is finished either by the core's own
// pass over y (the default), or, on request, inside out_proj: the core leaves y gated but not
// normalised and the group RMS scale of every (token, group) and the norm weights are applied
// to out_proj's A tiles in shared memory before their MMAs. The second way saves the pass over y
// but routes every A tile through shared memory twice more, which costs more than it saves on a
// B200 at the shapes measured, so it is not the default.
#include <cuda_bf16.h>

#include "../../include/ssd_mixer.h"
#include "ssd_internal.h"

namespace ssd {
ssd_status prefill_call(const ssd_dims* d, const void* x, int64_t x_ld, const void* z, int64_t z_ld, const void* B,
                        int64_t B_ld, const void* C, int64_t C_ld, const void* dt, int64_t dt_ld, const float* A,
                        const float* D, const float* conv_w, const float* conv_b, const float* dt_bias,
                        const float* norm_w, const float* init_ssm_state, const void* init_conv_state, void* y,
                        int64_t y_ld, float* final_ssm_state, void* final_conv_state, void* workspace,
                        size_t workspace_bytes, void* stream, bool defer_norm, bool keep_status, PrefillParams* out);
}  // namespace ssd

namespace {

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Layer workspace: the core's workspace first (its status word at offset 0 is the layer's),
// then the packed in_proj output, y, and the group scales of a norm finished in out_proj.
struct LayerLayout {
    size_t core, zxbcdt, y, scale, total;
};

LayerLayout layer_layout(const ssd_dims* d, size_t core_bytes)
{
    const int64_t rows = d->batch * d->seqlen;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    const int64_t width = 2 * HP + 2 * GN + d->nheads;
    LayerLayout l{};
    size_t off = align256(core_bytes);
    l.core = 0;
    l.zxbcdt = off; off = align256(off + (size_t)rows * (size_t)width * 2);
    l.y = off;      off = align256(off + (size_t)rows * (size_t)HP * 2);
    l.scale = off;  off = align256(off + (size_t)rows * (size_t)d->ngroups * 4);
    l.total = off;
    return l;
}

bool layer_dims_ok(const ssd_dims* d, int64_t d_model)
{
    if (!d || d->act != SSD_BF16 || d_model <= 0 || d_model % 8 != 0) return false;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    const int64_t width = 2 * HP + 2 * GN + d->nheads;
    const int64_t rows = d->batch * d->seqlen;
    return width % 8 == 0 && ssd_mixer_prefill_workspace_size(d) > 0 &&
           (rows == 0 || (ssd::gemm_supported(rows, width, d_model, d_model, d_model, width) &&
                          ssd::gemm_supported(rows, d_model, HP, HP, HP, d_model)));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

ssd_status ssd_mixer_projection(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, const void* W,
                                int64_t ldw, void* C, int64_t ldc, void* workspace, void* stream)
{
    if (M < 0 || N <= 0 || K <= 0 || !workspace || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (M == 0) return SSD_OK;
    if (!A || !W || !C) return SSD_ERR_INVALID_ARG;
    if (!ssd::gemm_supported(M, N, K, lda, ldw, ldc) || !aligned16(A) || !aligned16(W) || !aligned16(C))
        return SSD_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
    int* status = (int*)workspace;
    if (ssd::clear_device_status(status, st) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::launch_gemm_bf16(M, N, K, A, lda, W, ldw, C, ldc, nullptr, 0, 0, nullptr, status, st) != cudaSuccess)
        return SSD_ERR_CUDA;
    return SSD_OK;
}

size_t ssd_mixer_layer_workspace_size(const ssd_dims* d, int64_t d_model)
{
    if (!layer_dims_ok(d, d_model)) return 0;
    return layer_layout(d, ssd_mixer_prefill_workspace_size(d)).total;
}

ssd_status ssd_mixer_layer_prefill(const ssd_dims* d, int64_t d_model, const void* hidden, int64_t hidden_ld,
                                   const void* W_in, const void* W_out, const float* A, const float* D,
                                   const float* conv_w, const float* conv_b, const float* dt_bias,
                                   const float* norm_w, const float* init_ssm_state, const void* init_conv_state,
                                   void* out, int64_t out_ld, float* final_ssm_state, void* final_conv_state,
                                   int norm_in_out_proj, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!d) return SSD_ERR_INVALID_ARG;
    if (!layer_dims_ok(d, d_model)) return SSD_ERR_UNSUPPORTED;
    const size_t core_bytes = ssd_mixer_prefill_workspace_size(d);
    const LayerLayout l = layer_layout(d, core_bytes);
    if (!workspace || workspace_bytes < l.total || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (!W_in || !W_out || !aligned16(W_in) || !aligned16(W_out)) return SSD_ERR_INVALID_ARG;
    const int64_t rows = d->batch * d->seqlen;
    if (rows > 0) {
        if (!hidden || !out) return SSD_ERR_INVALID_ARG;
        if (!aligned16(hidden) || !aligned16(out) || hidden_ld < d_model || out_ld < d_model || hidden_ld % 8 ||
            out_ld % 8)
            return SSD_ERR_UNSUPPORTED;
    }
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    const int64_t width = 2 * HP + 2 * GN + d->nheads;
    char* ws = (char*)workspace;
    __nv_bfloat16* zx = (__nv_bfloat16*)(ws + l.zxbcdt);
    __nv_bfloat16* y = (__nv_bfloat16*)(ws + l.y);
    float* scale = (float*)(ws + l.scale);
    int* status = (int*)(ws + l.core);   // the core's status word
    cudaStream_t st = (cudaStream_t)stream;
    if (ssd::clear_device_status(status, st) != cudaSuccess) return SSD_ERR_CUDA;
    // in_proj: the packed [z | x | B | C | dt] row of every token
    if (rows > 0 && ssd::launch_gemm_bf16(rows, width, d_model, hidden, hidden_ld, W_in, d_model, zx, width, nullptr, 0, 0,
                                          nullptr, status, st) != cudaSuccess)
        return SSD_ERR_CUDA;
    // the core, on column slices of that row
    ssd::PrefillParams p{};
    const ssd_status cs = ssd::prefill_call(d, zx + HP, width, zx, width, zx + 2 * HP, width, zx + 2 * HP + GN, width,
                                            zx + 2 * HP + 2 * GN, width, A, D, conv_w, conv_b, dt_bias, norm_w,
                                            init_ssm_state, init_conv_state, y, HP, final_ssm_state, final_conv_state,
                                            ws + l.core, core_bytes, stream, norm_in_out_proj != 0, true, &p);
    if (cs != SSD_OK) return cs;
    if (rows == 0) return SSD_OK;
    // out_proj; a norm left to it is applied to its A tiles (group scale and norm weights)
    cudaError_t e;
    if (p.defer_norm) {
        if (ssd::launch_norm_scale(p, scale, st) != cudaSuccess) return SSD_ERR_CUDA;
        e = ssd::launch_gemm_bf16(rows, d_model, HP, y, HP, W_out, HP, out, out_ld, scale, (int)(HP / d->ngroups),
                                  d->ngroups, norm_w, status, st);
    } else {
        e = ssd::launch_gemm_bf16(rows, d_model, HP, y, HP, W_out, HP, out, out_ld, nullptr, 0, 0, nullptr, status, st);
    }
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // extern "C"
