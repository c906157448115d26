// ssd_api.cu -- the C ABI of include/ssd_mixer.h: argument checks, workspace carving
// and kernel dispatch. No allocation, no host synchronisation (except the explicit
// status read), no state kept between calls.
#include <string.h>

#include "../../include/ssd_mixer.h"
#include "ssd_internal.h"

namespace ssd {

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

WorkspaceLayout prefill_workspace_layout(int64_t b, int64_t L, int64_t rows, int H, int P, int G, int N,
                                         int Q, int act)
{
    WorkspaceLayout w{};
    if (prefill_tc_supported(act, P, N, H, G)) {   // the scan's intermediates stay on chip
        w.status = 0;
        w.xbc = w.delta = w.lam = w.states = w.ypre = 256;
        w.bcp = 256;
        size_t off = align256(256 + prefill_bc_blocks(b, rows) * (size_t)(2 * G * N) * kBcBlockTokens * 2);
        w.ssp = off;
        if (prefill_tc_split(H, G)) off = align256(off + (size_t)(rows * H) * (size_t)prefill_ws_partials_per_head() * 4);
        w.total = off;
        return w;
    }
    return simt_workspace_layout(b, L, H, P, G, N, Q, act);
}

WorkspaceLayout simt_workspace_layout(int64_t b, int64_t L, int H, int P, int G, int N, int Q, int act)
{
    WorkspaceLayout w{};
    const size_t es = act == SSD_BF16 ? 2 : 4;
    const int64_t HP = (int64_t)H * P, Cc = HP + 2 * (int64_t)G * N;
    const int64_t nc = Q > 0 ? (L + Q - 1) / Q : 0;
    size_t off = 0;
    w.status = off; off = align256(off + 256);
    w.xbc = off;    off = align256(off + (size_t)(b * L * Cc) * es);
    w.delta = off;  off = align256(off + (size_t)(b * H * L) * 4);
    w.lam = off;    off = align256(off + (size_t)(b * H * L) * 4);
    w.states = off; off = align256(off + (size_t)(b * nc * H) * (size_t)P * N * 4);
    w.ypre = off;   off = align256(off + (size_t)(b * L * HP) * 4);
    w.ssp = w.bcp = off;
    w.total = off;
    return w;
}

BackwardLayout backward_workspace_layout(int64_t b, int64_t L, int H, int P, int G, int N, int act)
{
    BackwardLayout w{};
    w.fwd = simt_workspace_layout(b, L, H, P, G, N, kBackwardForwardChunk, act);
    const size_t es = act == SSD_BF16 ? 2 : 4;
    const int64_t HP = (int64_t)H * P, Cc = HP + 2 * (int64_t)G * N, NB = P / kBackwardRows;
    size_t off = w.fwd.total;
    w.y = off;          off = align256(off + (size_t)(b * L * HP) * es);
    w.final_ssm = off;  off = align256(off + (size_t)(b * H) * (size_t)P * N * 4);
    w.final_conv = off; off = align256(off + (size_t)(b * Cc) * 3 * es);
    w.dy = off;         off = align256(off + (size_t)(b * L * HP) * 4);
    w.dxs = off;        off = align256(off + (size_t)(b * L * HP) * 4);
    w.dBp = off;        off = align256(off + (size_t)(b * L * H * NB) * (size_t)N * 4);
    w.dCp = off;        off = align256(off + (size_t)(b * L * H * NB) * (size_t)N * 4);
    w.ddp = off;        off = align256(off + (size_t)(b * H * NB) * (size_t)L * 4);
    w.total = off;
    return w;
}

}  // namespace ssd

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Shape checks common to prefill and decode. Returns SSD_OK or the error.
ssd_status check_dims(const ssd_dims* d, bool decode)
{
    if (!d) return SSD_ERR_INVALID_ARG;
    if (d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->headdim <= 0 || d->ngroups <= 0 ||
        d->dstate <= 0 || !(d->eps > 0.0f))
        return SSD_ERR_INVALID_ARG;
    if (d->act != SSD_F32 && d->act != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (d->nheads % d->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (d->dconv != 4) return SSD_ERR_UNSUPPORTED;
    if (!pow2_in(d->headdim, 16, 128) || !pow2_in(d->dstate, 16, 128)) return SSD_ERR_UNSUPPORTED;
    if (d->nheads > 65535 || d->batch > 65535) return SSD_ERR_UNSUPPORTED;
    if (decode) {
        if (d->seqlen != 1) return SSD_ERR_INVALID_ARG;
        if (!ssd::decode_supported(d->headdim, d->dstate)) return SSD_ERR_UNSUPPORTED;
        // the group's channels and vectors live in shared memory
        const int64_t r = d->nheads / d->ngroups;
        if ((2 * r * d->headdim + 2 * d->dstate + r + 8) * 4 > 200 * 1024) return SSD_ERR_UNSUPPORTED;
    } else {
        if (d->chunk < 16 || d->chunk > 256 || d->chunk % 16 != 0) return SSD_ERR_UNSUPPORTED;
        if (!ssd::prefill_simt_supported(d->headdim, d->dstate) &&
            !ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups))
            return SSD_ERR_UNSUPPORTED;
        const int64_t nc = (d->seqlen + d->chunk - 1) / d->chunk;
        if (nc * ((d->chunk + 63) / 64) > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    }
    return SSD_OK;
}

// Row-layout checks for one activation operand (16-byte vector access unless scalar).
bool row_ok(const void* p, int64_t ld, int64_t width, size_t es, bool vector)
{
    if (!p || ld < width) return false;
    if (vector) return aligned16(p) && ((size_t)ld * es) % 16 == 0;
    return ((uintptr_t)p % es) == 0;
}

}  // namespace

extern "C" {

size_t ssd_mixer_prefill_workspace_size(const ssd_dims* d)
{
    if (check_dims(d, false) != SSD_OK) return 0;
    return ssd::prefill_workspace_layout(d->batch, d->seqlen, d->batch * d->seqlen, d->nheads, d->headdim,
                                         d->ngroups, d->dstate, d->chunk, d->act)
        .total;
}

}  // extern "C"

namespace ssd {

// The prefill behind ssd_mixer_prefill. With defer_norm, a tensor-core call whose norm group is
// wider than a cluster leaves y gated but not normalised and returns, in *out, the parameters
// whose ssp holds the partial sums of squares; with keep_status the status word is not cleared
// (the caller cleared it before an earlier kernel of its own).
ssd_status prefill_call(const ssd_dims* d, const void* x, int64_t x_ld, const void* z, int64_t z_ld, const void* B,
                        int64_t B_ld, const void* C, int64_t C_ld, const void* dt, int64_t dt_ld, const float* A,
                        const float* D, const float* conv_w, const float* conv_b, const float* dt_bias,
                        const float* norm_w, const float* init_ssm_state, const void* init_conv_state, void* y,
                        int64_t y_ld, float* final_ssm_state, void* final_conv_state, void* workspace,
                        size_t workspace_bytes, void* stream, bool defer_norm, bool keep_status, PrefillParams* out)
{
    const ssd_status ds = check_dims(d, false);
    if (ds != SSD_OK) return ds;
    const size_t es = d->act == SSD_BF16 ? 2 : 4;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    if (!A || !D || !conv_w || !conv_b || !dt_bias || !norm_w || !final_ssm_state || !final_conv_state)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(conv_w) || !aligned16(final_ssm_state) ||
        (init_ssm_state && !aligned16(init_ssm_state)))
        return SSD_ERR_UNSUPPORTED;
    if ((init_conv_state && ((uintptr_t)init_conv_state % es)) || ((uintptr_t)final_conv_state % es))
        return SSD_ERR_UNSUPPORTED;
    const ssd::WorkspaceLayout wl = ssd::prefill_workspace_layout(d->batch, d->seqlen, d->batch * d->seqlen, d->nheads,
                                                                  d->headdim, d->ngroups, d->dstate, d->chunk, d->act);
    if (!workspace || workspace_bytes < wl.total || ((uintptr_t)workspace & 255u))
        return SSD_ERR_INVALID_ARG;
    if (d->seqlen > 0 && d->batch > 0) {
        if (!x || !z || !B || !C || !dt || !y) return SSD_ERR_INVALID_ARG;
        if (!row_ok(x, x_ld, HP, es, true) || !row_ok(z, z_ld, HP, es, true) ||
            !row_ok(B, B_ld, GN, es, true) || !row_ok(C, C_ld, GN, es, true) ||
            !row_ok(y, y_ld, HP, es, true) || !row_ok(dt, dt_ld, d->nheads, es, false))
            return SSD_ERR_UNSUPPORTED;
    }
    ssd::PrefillParams p{};
    p.b = d->batch; p.L = d->seqlen;
    p.H = d->nheads; p.P = d->headdim; p.G = d->ngroups; p.N = d->dstate; p.K = d->dconv;
    p.Q = d->chunk; p.eps = d->eps; p.act = d->act;
    p.nc = (p.L + p.Q - 1) / p.Q;
    p.x = x; p.z = z; p.B = B; p.C = C; p.dt = dt;
    p.x_ld = x_ld; p.z_ld = z_ld; p.B_ld = B_ld; p.C_ld = C_ld; p.dt_ld = dt_ld;
    p.A = A; p.D = D; p.conv_w = conv_w; p.conv_b = conv_b; p.dt_bias = dt_bias; p.norm_w = norm_w;
    p.init_ssm = init_ssm_state; p.init_conv = init_conv_state;
    p.y = y; p.y_ld = y_ld; p.final_ssm = final_ssm_state; p.final_conv = final_conv_state;
    char* ws = (char*)workspace;
    p.status = (int*)(ws + wl.status);
    p.xbc = ws + wl.xbc;
    p.delta = (float*)(ws + wl.delta);
    p.lam = (float*)(ws + wl.lam);
    p.states = (float*)(ws + wl.states);
    p.ypre = (float*)(ws + wl.ypre);
    p.ssp = (float*)(ws + wl.ssp);
    p.bcp = ws + wl.bcp;
    cudaStream_t st = (cudaStream_t)stream;

    const bool tc = ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups);
    p.defer_norm = defer_norm && tc && ssd::prefill_tc_split(d->nheads, d->ngroups);
    if (!keep_status && ssd::clear_device_status(p.status, st) != cudaSuccess) return SSD_ERR_CUDA;
    if ((tc ? ssd::launch_prefill_ws(p, st) : ssd::launch_prefill_simt(p, st)) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (out) *out = p;
    return SSD_OK;
}

}  // namespace ssd

extern "C" {

ssd_status ssd_mixer_prefill(const ssd_dims* d, const void* x, int64_t x_ld, const void* z,
                             int64_t z_ld, const void* B, int64_t B_ld, const void* C, int64_t C_ld,
                             const void* dt, int64_t dt_ld, const float* A, const float* D,
                             const float* conv_w, const float* conv_b, const float* dt_bias,
                             const float* norm_w, const float* init_ssm_state,
                             const void* init_conv_state, void* y, int64_t y_ld,
                             float* final_ssm_state, void* final_conv_state, void* workspace,
                             size_t workspace_bytes, void* stream)
{
    return ssd::prefill_call(d, x, x_ld, z, z_ld, B, B_ld, C, C_ld, dt, dt_ld, A, D, conv_w, conv_b, dt_bias, norm_w,
                             init_ssm_state, init_conv_state, y, y_ld, final_ssm_state, final_conv_state, workspace,
                             workspace_bytes, stream, false, false, nullptr);
}

int ssd_mixer_prefill_path(const ssd_dims* d)
{
    if (check_dims(d, false) != SSD_OK) return SSD_PATH_NONE;
    return ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups) ? SSD_PATH_TENSOR_CORES
                                                                                           : SSD_PATH_CUDA_CORES;
}

ssd_status ssd_mixer_prefill_plan(const ssd_dims* d, int sms, int* launches, int* pieces, int* piece_blocks,
                                  int* ctas_per_launch)
{
    if (ssd_mixer_prefill_path(d) != SSD_PATH_TENSOR_CORES) return SSD_ERR_UNSUPPORTED;
    if (!launches || !pieces || !piece_blocks || !ctas_per_launch || sms < 0) return SSD_ERR_INVALID_ARG;
    const ssd::PrefillPlan pl =
        ssd::prefill_ws_plan(d->batch, d->seqlen, d->nheads, d->ngroups, sms > 0 ? sms : ssd::device_sm_count());
    *launches = d->batch > 0 && d->seqlen > 0 ? pl.launches : 0;
    *pieces = pl.pieces;
    *piece_blocks = pl.piece_blocks;
    *ctas_per_launch = pl.ctas_per_launch;
    return SSD_OK;
}

ssd_status ssd_mixer_prefill_stage_offsets(const ssd_dims* d, size_t* xbc_act, size_t* delta, size_t* y_pre)
{
    if (ssd_mixer_prefill_path(d) != SSD_PATH_CUDA_CORES) return SSD_ERR_UNSUPPORTED;
    if (!xbc_act || !delta || !y_pre) return SSD_ERR_INVALID_ARG;
    const ssd::WorkspaceLayout wl = ssd::simt_workspace_layout(d->batch, d->seqlen, d->nheads, d->headdim,
                                                               d->ngroups, d->dstate, d->chunk, d->act);
    *xbc_act = wl.xbc;
    *delta = wl.delta;
    *y_pre = wl.ypre;
    return SSD_OK;
}

size_t ssd_mixer_prefill_state_workspace_size(const ssd_dims* d)
{
    if (check_dims(d, false) != SSD_OK ||
        !ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups))
        return 0;
    return ssd::prefill_workspace_layout(d->batch, d->seqlen, d->batch * d->seqlen, d->nheads, d->headdim,
                                         d->ngroups, d->dstate, d->chunk, d->act)
        .total;
}

ssd_status ssd_mixer_prefill_state(const ssd_dims* d, const void* x, int64_t x_ld, const void* B, int64_t B_ld,
                                   const void* C, int64_t C_ld, const void* dt, int64_t dt_ld, const float* A,
                                   const float* conv_w, const float* conv_b, const float* dt_bias,
                                   const float* init_ssm_state, const void* init_conv_state,
                                   float* final_ssm_state, void* final_conv_state, float* decay,
                                   void* workspace, size_t workspace_bytes, void* stream)
{
    const ssd_status ds = check_dims(d, false);
    if (ds != SSD_OK) return ds;
    if (!ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups))
        return SSD_ERR_UNSUPPORTED;
    const size_t es = 2;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    if (!A || !conv_w || !conv_b || !dt_bias || !final_ssm_state || !final_conv_state) return SSD_ERR_INVALID_ARG;
    if (!aligned16(conv_w) || !aligned16(final_ssm_state) || (init_ssm_state && !aligned16(init_ssm_state)) ||
        (init_conv_state && ((uintptr_t)init_conv_state % es)) || ((uintptr_t)final_conv_state % es) ||
        (decay && ((uintptr_t)decay & 3u)))
        return SSD_ERR_UNSUPPORTED;
    const ssd::WorkspaceLayout wl = ssd::prefill_workspace_layout(d->batch, d->seqlen, d->batch * d->seqlen, d->nheads,
                                                                  d->headdim, d->ngroups, d->dstate, d->chunk, d->act);
    if (!workspace || workspace_bytes < wl.total || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (d->seqlen > 0 && d->batch > 0) {
        if (!x || !B || !C || !dt) return SSD_ERR_INVALID_ARG;
        if (!row_ok(x, x_ld, HP, es, true) || !row_ok(B, B_ld, GN, es, true) || !row_ok(C, C_ld, GN, es, true) ||
            !row_ok(dt, dt_ld, d->nheads, es, false))
            return SSD_ERR_UNSUPPORTED;
    }
    ssd::PrefillParams p{};
    p.b = d->batch; p.L = d->seqlen;
    p.H = d->nheads; p.P = d->headdim; p.G = d->ngroups; p.N = d->dstate; p.K = d->dconv;
    p.Q = d->chunk; p.eps = d->eps; p.act = d->act;
    p.nc = (p.L + p.Q - 1) / p.Q;
    p.x = x; p.B = B; p.C = C; p.dt = dt;
    p.x_ld = x_ld; p.B_ld = B_ld; p.C_ld = C_ld; p.dt_ld = dt_ld;
    p.A = A; p.conv_w = conv_w; p.conv_b = conv_b; p.dt_bias = dt_bias;
    p.init_ssm = init_ssm_state; p.init_conv = init_conv_state;
    p.final_ssm = final_ssm_state; p.final_conv = final_conv_state; p.decay = decay;
    char* ws = (char*)workspace;
    p.status = (int*)(ws + wl.status);
    p.ssp = (float*)(ws + wl.ssp);
    p.bcp = ws + wl.bcp;
    if (ssd::clear_device_status(p.status, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::launch_prefill_state_ws(p, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
}

ssd_status ssd_mixer_state_pass(int64_t batch, int32_t nheads, int32_t headdim, int32_t dstate, int32_t r,
                                const float* decay, const float* state, const float* init, float* out,
                                void* stream)
{
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || r < 0) return SSD_ERR_INVALID_ARG;
    if (((int64_t)headdim * dstate) % 4 != 0) return SSD_ERR_UNSUPPORTED;
    if (!out || (r > 0 && (!decay || !state))) return SSD_ERR_INVALID_ARG;
    if (!aligned16(out) || (state && !aligned16(state)) || (init && !aligned16(init)) ||
        (decay && ((uintptr_t)decay & 3u)))
        return SSD_ERR_UNSUPPORTED;
    if (ssd::launch_state_pass(batch, nheads, headdim, dstate, r, decay, state, init, out, (cudaStream_t)stream) !=
        cudaSuccess)
        return SSD_ERR_CUDA;
    return SSD_OK;
}

size_t ssd_mixer_prefill_varlen_workspace_size(const ssd_dims* d)
{
    if (check_dims(d, false) != SSD_OK ||
        !ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups))
        return 0;
    return ssd::prefill_workspace_layout(d->batch, d->seqlen, d->seqlen, d->nheads, d->headdim, d->ngroups,
                                         d->dstate, d->chunk, d->act)
        .total;
}

ssd_status ssd_mixer_prefill_varlen(const ssd_dims* d, const int32_t* cu_seqlens, const int32_t* slot_idx,
                                    const uint8_t* has_init, const void* x, int64_t x_ld, const void* z,
                                    int64_t z_ld, const void* B, int64_t B_ld, const void* C, int64_t C_ld,
                                    const void* dt, int64_t dt_ld, const float* A, const float* D,
                                    const float* conv_w, const float* conv_b, const float* dt_bias,
                                    const float* norm_w, float* ssm_state, void* conv_state, void* y,
                                    int64_t y_ld, void* workspace, size_t workspace_bytes, void* stream)
{
    const ssd_status ds = check_dims(d, false);
    if (ds != SSD_OK) return ds;
    if (!ssd::prefill_tc_supported(d->act, d->headdim, d->dstate, d->nheads, d->ngroups))
        return SSD_ERR_UNSUPPORTED;
    if (d->seqlen > 0x7fffff00LL) return SSD_ERR_UNSUPPORTED;   // token rows are int32 (cu_seqlens)
    const size_t es = 2;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    if (!A || !D || !conv_w || !conv_b || !dt_bias || !norm_w || !ssm_state || !conv_state || !cu_seqlens)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(conv_w) || !aligned16(ssm_state) || ((uintptr_t)conv_state % es) ||
        ((uintptr_t)cu_seqlens & 3u) || (slot_idx && ((uintptr_t)slot_idx & 3u)))
        return SSD_ERR_UNSUPPORTED;
    const ssd::WorkspaceLayout wl = ssd::prefill_workspace_layout(d->batch, d->seqlen, d->seqlen, d->nheads,
                                                                  d->headdim, d->ngroups, d->dstate, d->chunk, d->act);
    if (!workspace || workspace_bytes < wl.total || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (d->seqlen > 0) {
        if (!x || !z || !B || !C || !dt || !y) return SSD_ERR_INVALID_ARG;
        if (!row_ok(x, x_ld, HP, es, true) || !row_ok(z, z_ld, HP, es, true) ||
            !row_ok(B, B_ld, GN, es, true) || !row_ok(C, C_ld, GN, es, true) ||
            !row_ok(y, y_ld, HP, es, true) || !row_ok(dt, dt_ld, d->nheads, es, false))
            return SSD_ERR_UNSUPPORTED;
    }
    if (d->batch == 0) return SSD_OK;
    ssd::PrefillParams p{};
    p.b = d->batch; p.L = d->seqlen;
    p.H = d->nheads; p.P = d->headdim; p.G = d->ngroups; p.N = d->dstate; p.K = d->dconv;
    p.Q = d->chunk; p.eps = d->eps; p.act = d->act;
    p.nc = (p.L + p.Q - 1) / p.Q;
    p.x = x; p.z = z; p.B = B; p.C = C; p.dt = dt;
    p.x_ld = x_ld; p.z_ld = z_ld; p.B_ld = B_ld; p.C_ld = C_ld; p.dt_ld = dt_ld;
    p.A = A; p.D = D; p.conv_w = conv_w; p.conv_b = conv_b; p.dt_bias = dt_bias; p.norm_w = norm_w;
    p.init_ssm = ssm_state; p.init_conv = conv_state;
    p.final_ssm = ssm_state; p.final_conv = conv_state;
    p.y = y; p.y_ld = y_ld;
    p.cu_seqlens = cu_seqlens; p.slot_idx = slot_idx; p.has_init = has_init;
    char* ws = (char*)workspace;
    p.status = (int*)(ws + wl.status);
    p.ssp = (float*)(ws + wl.ssp);
    p.bcp = ws + wl.bcp;
    if (ssd::clear_device_status(p.status, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    if (ssd::launch_prefill_ws(p, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
}

ssd_status ssd_mixer_decode_step(const ssd_dims* d, const void* x, int64_t x_ld, const void* z,
                                 int64_t z_ld, const void* B, int64_t B_ld, const void* C,
                                 int64_t C_ld, const void* dt, int64_t dt_ld, const float* A,
                                 const float* D, const float* conv_w, const float* conv_b,
                                 const float* dt_bias, const float* norm_w, float* ssm_state,
                                 void* conv_state, const int32_t* slot_idx, void* y, int64_t y_ld,
                                 void* stream)
{
    const ssd_status ds = check_dims(d, true);
    if (ds != SSD_OK) return ds;
    if (d->batch == 0) return SSD_OK;
    const size_t es = d->act == SSD_BF16 ? 2 : 4;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    if (!A || !D || !conv_w || !conv_b || !dt_bias || !norm_w || !ssm_state || !conv_state ||
        !x || !z || !B || !C || !dt || !y)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(conv_w) || !aligned16(ssm_state) || ((uintptr_t)conv_state % es) ||
        (slot_idx && ((uintptr_t)slot_idx & 3u)))
        return SSD_ERR_UNSUPPORTED;
    if (!row_ok(x, x_ld, HP, es, false) || !row_ok(z, z_ld, HP, es, false) ||
        !row_ok(B, B_ld, GN, es, false) || !row_ok(C, C_ld, GN, es, false) ||
        !row_ok(y, y_ld, HP, es, false) || !row_ok(dt, dt_ld, d->nheads, es, false))
        return SSD_ERR_UNSUPPORTED;
    ssd::DecodeParams p{};
    p.b = d->batch;
    p.H = d->nheads; p.P = d->headdim; p.G = d->ngroups; p.N = d->dstate; p.K = d->dconv;
    p.eps = d->eps; p.act = d->act;
    p.x = x; p.z = z; p.B = B; p.C = C; p.dt = dt;
    p.x_ld = x_ld; p.z_ld = z_ld; p.B_ld = B_ld; p.C_ld = C_ld; p.dt_ld = dt_ld;
    p.A = A; p.D = D; p.conv_w = conv_w; p.conv_b = conv_b; p.dt_bias = dt_bias; p.norm_w = norm_w;
    p.ssm_state = ssm_state; p.conv_state = conv_state; p.slot_idx = slot_idx;
    p.y = y; p.y_ld = y_ld;
    if (ssd::launch_decode_step(p, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
}

size_t ssd_mixer_backward_workspace_size(const ssd_dims* d)
{
    if (check_dims(d, false) != SSD_OK || !ssd::backward_supported(d->headdim, d->dstate)) return 0;
    return ssd::backward_workspace_layout(d->batch, d->seqlen, d->nheads, d->headdim, d->ngroups, d->dstate, d->act)
        .total;
}

ssd_status ssd_mixer_backward(const ssd_dims* d, const void* x, int64_t x_ld, const void* z, int64_t z_ld,
                              const void* B, int64_t B_ld, const void* C, int64_t C_ld, const void* dt,
                              int64_t dt_ld, const float* A, const float* D, const float* conv_w,
                              const float* conv_b, const float* dt_bias, const float* norm_w,
                              const float* init_ssm_state, const void* init_conv_state, const void* dy,
                              int64_t dy_ld, const float* dfinal_ssm_state, const float* dfinal_conv_state,
                              void* dx, int64_t dx_ld, void* dz, int64_t dz_ld, void* dB, int64_t dB_ld, void* dC,
                              int64_t dC_ld, void* ddt, int64_t ddt_ld, float* dA, float* dD, float* dconv_w,
                              float* dconv_b, float* ddt_bias, float* dnorm_w, float* dinit_ssm_state,
                              float* dinit_conv_state, void* workspace, size_t workspace_bytes, void* stream)
{
    const ssd_status ds = check_dims(d, false);
    if (ds != SSD_OK) return ds;
    if (!ssd::backward_supported(d->headdim, d->dstate)) return SSD_ERR_UNSUPPORTED;
    if (d->seqlen > 65535LL * 32) return SSD_ERR_UNSUPPORTED;   // token segments of the conv backward
    const size_t es = d->act == SSD_BF16 ? 2 : 4;
    const int64_t HP = (int64_t)d->nheads * d->headdim, GN = (int64_t)d->ngroups * d->dstate;
    if (!A || !D || !conv_w || !conv_b || !dt_bias || !norm_w) return SSD_ERR_INVALID_ARG;
    if (!dA || !dD || !dconv_w || !dconv_b || !ddt_bias || !dnorm_w) return SSD_ERR_INVALID_ARG;
    if (!aligned16(conv_w) || (init_ssm_state && !aligned16(init_ssm_state)) ||
        (init_conv_state && ((uintptr_t)init_conv_state % es)))
        return SSD_ERR_UNSUPPORTED;
    const ssd::BackwardLayout wl = ssd::backward_workspace_layout(d->batch, d->seqlen, d->nheads, d->headdim,
                                                                  d->ngroups, d->dstate, d->act);
    if (!workspace || workspace_bytes < wl.total || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    if (d->seqlen > 0 && d->batch > 0) {
        if (!x || !z || !B || !C || !dt || !dy || !dx || !dz || !dB || !dC || !ddt) return SSD_ERR_INVALID_ARG;
        if (!row_ok(x, x_ld, HP, es, true) || !row_ok(z, z_ld, HP, es, true) ||
            !row_ok(B, B_ld, GN, es, true) || !row_ok(C, C_ld, GN, es, true) ||
            !row_ok(dt, dt_ld, d->nheads, es, false) || !row_ok(dy, dy_ld, HP, es, false) ||
            !row_ok(dx, dx_ld, HP, es, false) || !row_ok(dz, dz_ld, HP, es, false) ||
            !row_ok(dB, dB_ld, GN, es, false) || !row_ok(dC, dC_ld, GN, es, false) ||
            !row_ok(ddt, ddt_ld, d->nheads, es, false))
            return SSD_ERR_UNSUPPORTED;
    }
    ssd::BackwardParams p{};
    ssd::PrefillParams& f = p.f;
    f.b = d->batch; f.L = d->seqlen;
    f.H = d->nheads; f.P = d->headdim; f.G = d->ngroups; f.N = d->dstate; f.K = d->dconv;
    f.Q = ssd::kBackwardForwardChunk; f.eps = d->eps; f.act = d->act;
    f.nc = (f.L + f.Q - 1) / f.Q;
    f.x = x; f.z = z; f.B = B; f.C = C; f.dt = dt;
    f.x_ld = x_ld; f.z_ld = z_ld; f.B_ld = B_ld; f.C_ld = C_ld; f.dt_ld = dt_ld;
    f.A = A; f.D = D; f.conv_w = conv_w; f.conv_b = conv_b; f.dt_bias = dt_bias; f.norm_w = norm_w;
    f.init_ssm = init_ssm_state; f.init_conv = init_conv_state;
    char* ws = (char*)workspace;
    f.status = (int*)(ws + wl.fwd.status);
    if (ssd::clear_device_status(f.status, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    f.xbc = ws + wl.fwd.xbc;
    f.delta = (float*)(ws + wl.fwd.delta);
    f.lam = (float*)(ws + wl.fwd.lam);
    f.states = (float*)(ws + wl.fwd.states);
    f.ypre = (float*)(ws + wl.fwd.ypre);
    f.ssp = (float*)(ws + wl.fwd.ssp);
    f.bcp = ws + wl.fwd.bcp;
    f.y = ws + wl.y; f.y_ld = HP;
    f.final_ssm = (float*)(ws + wl.final_ssm);
    f.final_conv = ws + wl.final_conv;
    p.dout = dy; p.dout_ld = dy_ld;
    p.dfinal_ssm = dfinal_ssm_state; p.dfinal_conv = dfinal_conv_state;
    p.dx = dx; p.dz = dz; p.dB = dB; p.dC = dC; p.ddt = ddt;
    p.dx_ld = dx_ld; p.dz_ld = dz_ld; p.dB_ld = dB_ld; p.dC_ld = dC_ld; p.ddt_ld = ddt_ld;
    p.dA = dA; p.dD = dD; p.dconv_w = dconv_w; p.dconv_b = dconv_b; p.ddt_bias = ddt_bias; p.dnorm_w = dnorm_w;
    p.dinit_ssm = dinit_ssm_state; p.dinit_conv = dinit_conv_state;
    p.dy = (float*)(ws + wl.dy);
    p.dxs = (float*)(ws + wl.dxs);
    p.dBp = (float*)(ws + wl.dBp);
    p.dCp = (float*)(ws + wl.dCp);
    p.ddp = (float*)(ws + wl.ddp);
    if (ssd::launch_backward(p, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
}

ssd_status ssd_mixer_workspace_status(const void* workspace, void* stream)
{
    if (!workspace || ((uintptr_t)workspace & 255u)) return SSD_ERR_INVALID_ARG;
    int v = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    switch (v) {
    case ssd::kDevOk: return SSD_OK;
    case ssd::kDevTimeout: return SSD_ERR_TIMEOUT;
    default: return SSD_ERR_DEVICE;
    }
}

const char* ssd_status_string(ssd_status s)
{
    switch (s) {
    case SSD_OK: return "ok";
    case SSD_ERR_INVALID_ARG: return "invalid argument";
    case SSD_ERR_UNSUPPORTED: return "unsupported shape, alignment or dtype";
    case SSD_ERR_CUDA: return "CUDA launch or runtime error";
    case SSD_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case SSD_ERR_TOO_LARGE: return "problem needs more scratch than the fixed static workspace holds";
    case SSD_ERR_DEVICE:
        return "a kernel could not start its work (its shared memory base was misaligned), or, in the "
               "bounds-checked build, an index fell outside its buffer";
    }
    return "unknown status";
}

int ssd_mixer_version(void) { return 100; }

}  // extern "C"
