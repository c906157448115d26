/*
 * ssd_mixer.h -- C ABI of a B200 (sm_100a) library for the core of the Mamba-2
 * mixer in Nemotron-H hybrid models: everything between in_proj and out_proj.
 *
 * The mixer projects its input (in_proj), runs a causal depthwise conv, the
 * selective SSM scan and a gated RMSNorm, and projects back (out_proj); the
 * recurrent state of each sequence lives in an engine slot (gllm PR #86 "feat(model): Nemotron-H hybrid (Mamba2 + attention + MoE) on the
 * CPU", section "2. feat(model): Nemotron-H on the CPU", mixer table row M). The
 * scan is the chunked "structured state-space duality" (SSD) form of the Mamba-2
 * recurrence (openNemo model card, section "Architecture"; Modalities PR #459,
 * section "Testing" and the ssd.py notes on the chunk-parallel block
 * decomposition and the GatedRMSNorm semantics).
 *
 * Notation: b batch rows, L tokens per row, H heads, P head dim, G groups sharing
 * B and C, N state dim, K conv width (4), HP = H*P, GN = G*N, Cc = HP + 2*GN (the
 * xBC channels), r = H/G heads per group; head h reads group h / r.
 *
 * What every call computes, per batch row, for t = 0..L-1:
 *   xBC' = SiLU(causal depthwise conv_K([x|B|C]) + conv_b), the conv running over
 *          the K-1 stored raw inputs followed by this call's inputs;
 *   delta_t[h] = softplus(dt_t[h] + dt_bias[h]);
 *   h_t = exp(delta_t[h] * A[h]) * h_{t-1} + delta_t[h] * x'_t[h] (outer) B'_t[g];
 *   y_t[h] = h_t . C'_t[g] + D[h] * x'_t[h];
 *   out_t  = RMSNorm over each contiguous group of HP/G channels of
 *            (y_t * SiLU(z_t)), times norm_w, with eps.
 * The prefill evaluates the scan chunk by chunk (chunk = Q tokens): exact up to
 * rounding, whatever Q is.
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers owned by the caller, except `dims`, which is a
 *    host pointer read during the call only. The library allocates nothing, keeps
 *    no pointer after the call returns and never synchronises the stream.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and runs asynchronously. Results are ready when the stream is.
 *  - Activations (x, z, B, C, dt, y and the conv state) have dtype dims->act: fp32
 *    or bf16. Parameters (A, D, conv_w, conv_b, dt_bias, norm_w) and the SSM state
 *    are always fp32. Arithmetic is fp32 throughout; bf16 activations feed the
 *    tensor-core contractions as bf16 with fp32 accumulation.
 *  - Row layouts: token t of batch row i of x starts at x + (i*L + t) * x_ld
 *    elements (likewise z, B, C, dt, y with their own ld), so the five inputs may
 *    be column slices of one packed in_proj output. x, z, B, C and y must be
 *    16-byte aligned with ld*elem_size a multiple of 16 bytes; dt needs only
 *    element alignment. x and y must not overlap.
 *  - Parameter layouts: A, D, dt_bias [H] (A negative); conv_w [Cc][K] with tap K-1
 *    on the current token; conv_b [Cc]; norm_w [HP]; channel order of Cc is x
 *    (HP), then B (GN), then C (GN).
 *  - State layouts: SSM state [slots or b][H][P][N] fp32, N contiguous; conv state
 *    [slots or b][Cc][K-1] in the activation dtype, oldest raw input first.
 *  - Errors: argument errors return SSD_ERR_INVALID_ARG or SSD_ERR_UNSUPPORTED
 *    before anything is launched; a failed launch returns SSD_ERR_CUDA. Nothing
 *    is written when an error is returned before the launch.
 */
#ifndef SSD_MIXER_H
#define SSD_MIXER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,  /* null pointer, bad size, workspace too small */
    SSD_ERR_UNSUPPORTED = 2,  /* shape/alignment/dtype the library does not run */
    SSD_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed */
    SSD_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up (status word) */
    SSD_ERR_TOO_LARGE = 5,    /* needs more scratch than the fixed static workspace */
    SSD_ERR_DEVICE = 6,       /* a kernel could not start its work, or (bounds-checked build)
                                 an index fell outside its buffer (status word) */
} ssd_status;

typedef enum ssd_dtype {
    SSD_F32 = 0,
    SSD_BF16 = 1,
} ssd_dtype;

/* Problem dimensions (a plain struct; every field is read, none is kept). */
typedef struct ssd_dims {
    int64_t batch;    /* b: batch rows (prefill) or sequences stepped (decode) */
    int64_t seqlen;   /* L: tokens per row in this call (decode: must be 1)     */
    int32_t nheads;   /* H */
    int32_t headdim;  /* P: 16, 32, 64 or 128 */
    int32_t ngroups;  /* G: divides H */
    int32_t dstate;   /* N: 16, 32, 64 or 128 */
    int32_t dconv;    /* K: must be 4 */
    int32_t chunk;    /* Q: prefill chunk length, 16..256 and a multiple of 16 */
    float eps;        /* RMSNorm epsilon (> 0) */
    int32_t act;      /* ssd_dtype of the activations */
} ssd_dims;

/* Bytes of device workspace ssd_mixer_prefill needs for `dims`; 0 when the dims
 * are invalid or unsupported (call ssd_mixer_prefill to learn which). The size
 * grows linearly with batch * seqlen. */
SSD_API size_t ssd_mixer_prefill_workspace_size(const ssd_dims* dims);

/* Prefill: run L tokens of b independent rows through the mixer core.
 *
 * Inputs: x, z [b][L][HP]; B, C [b][L][GN]; dt [b][L][H] (raw, before the bias);
 * parameters as above; init_ssm_state [b][H][P][N] and init_conv_state [b][Cc][K-1]
 * (either may be NULL = zeros). To continue a sequence that arrives in several
 * pieces, pass the previous call's final states as this call's initial states (the
 * split-prefill case of gllm PR #86, section "Validation").
 * Outputs: y [b][L][HP] (gated, normalised; y_ld), final_ssm_state, final_conv_state
 * (same layouts as the inits). A final state may be the same buffer as its init.
 * workspace: device scratch of at least ssd_mixer_prefill_workspace_size(dims)
 * bytes, 256-byte aligned, not shared with a concurrently running call.
 * L = 0 is allowed: y is untouched and the final states equal the initial ones. */
SSD_API ssd_status ssd_mixer_prefill(const ssd_dims* dims,
                             const void* x, int64_t x_ld,
                             const void* z, int64_t z_ld,
                             const void* B, int64_t B_ld,
                             const void* C, int64_t C_ld,
                             const void* dt, int64_t dt_ld,
                             const float* A, const float* D,
                             const float* conv_w, const float* conv_b,
                             const float* dt_bias, const float* norm_w,
                             const float* init_ssm_state, const void* init_conv_state,
                             void* y, int64_t y_ld,
                             float* final_ssm_state, void* final_conv_state,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/* Which kernels ssd_mixer_prefill runs for `dims` (a host-side query; nothing is launched):
 * SSD_PATH_TENSOR_CORES for bf16 activations with P = 64, N = 128 and 2 or a multiple of 4
 * heads per group (one fused tcgen05 kernel; intermediates stay on chip, dims->chunk is not
 * used: the chunked form is evaluated in 128-token blocks); SSD_PATH_CUDA_CORES for the other
 * supported shapes (fp32 FFMA kernels with dims->chunk-token chunks, intermediates in the
 * workspace); SSD_PATH_NONE when the dims are invalid or unsupported. */
typedef enum ssd_path {
    SSD_PATH_NONE = 0,
    SSD_PATH_CUDA_CORES = 1,
    SSD_PATH_TENSOR_CORES = 2,
} ssd_path;
SSD_API int ssd_mixer_prefill_path(const ssd_dims* dims);

/* How ssd_mixer_prefill runs the tensor-core main kernel for `dims` (a host-side query;
 * nothing is launched; no counterpart in the pages). Each (sequence, head) row is a walk over
 * its 128-token blocks, one CTA per SM. When the rows of a group wider than a cluster outnumber
 * the SMs, whole rows would leave the last wave of CTAs part-empty. The call then splits every
 * row into pieces of whole blocks and runs them as a series of launches. Each piece continues
 * from the state its predecessor left in final_ssm_state, written by an earlier launch.
 * sms: the SM count to plan for, 0 = the current device's (148 when none can be queried).
 * Writes the launches per call (0 for an empty call), the pieces per row, the blocks per piece
 * (the last piece of a row may be shorter) and the CTAs per launch (the last launch may have
 * fewer). The environment variable SSD_MIXER_PREFILL_PIECES (read once per process, 1 .. 64)
 * fixes the piece count. Returns SSD_ERR_UNSUPPORTED unless the dims take the tensor-core path
 * (ssd_mixer_prefill_path), SSD_ERR_INVALID_ARG for a NULL output or a negative sms. */
SSD_API ssd_status ssd_mixer_prefill_plan(const ssd_dims* dims, int sms, int* launches, int* pieces,
                                          int* piece_blocks, int* ctas_per_launch);

/* Where a CUDA-core prefill (SSD_PATH_CUDA_CORES) leaves its intermediates in its workspace,
 * for checking each stage on its own: byte offsets from the workspace start of
 *   xbc_act [b][L][Cc] activation dtype: SiLU(conv) of [x|B|C];
 *   delta   [b][H][L] fp32: softplus(dt + dt_bias), head-major;
 *   y_pre   [b][L][HP] fp32: y = C'.h + D x' before the gate and the norm.
 * They hold the values of the last call that used the workspace. Returns SSD_OK, or
 * SSD_ERR_UNSUPPORTED for dims that run on the tensor cores (nothing of this is kept there)
 * or are invalid; host pointers, written only on SSD_OK. */
SSD_API ssd_status ssd_mixer_prefill_stage_offsets(const ssd_dims* dims, size_t* xbc_act, size_t* delta,
                                                   size_t* y_pre);

/* Bytes of device workspace ssd_mixer_prefill_state needs for `dims`; 0 when the dims are
 * invalid or the shape is one the state-only pass does not run. */
SSD_API size_t ssd_mixer_prefill_state_workspace_size(const ssd_dims* dims);

/* State-only prefill: the final states of ssd_mixer_prefill, without the output rows, plus
 * the decay of each row's whole piece. A piece of a long sequence then hands its state to the
 * next piece without computing its own outputs first, which is the state passing that a
 * sequence split across devices needs (Modalities PR #459, section "Next steps for
 * production at scale", item "MTP and long-context", on splitting long sequences across
 * GPUs; section "Testing", on a state carried across the parts of a split sequence). With S_r the final state of piece r computed from a zero initial state and a_r
 * its decay, the state entering piece r+1 is a_r * (state entering piece r) + S_r.
 *
 * Same inputs and state layouts as ssd_mixer_prefill, without z, D and norm_w (C is read
 * only for its final conv state). Outputs: final_ssm_state, final_conv_state, and decay
 * [b][H] fp32 (NULL = not wanted): exp(A[h] * sum over the row's tokens of delta_t[h]).
 * Runs the tensor-core kernel only (bf16, P = 64, N = 128, 2 or a multiple of 4 heads per
 * group); other shapes return SSD_ERR_UNSUPPORTED. Final states may alias initial ones. */
SSD_API ssd_status ssd_mixer_prefill_state(const ssd_dims* dims,
                                   const void* x, int64_t x_ld,
                                   const void* B, int64_t B_ld,
                                   const void* C, int64_t C_ld,
                                   const void* dt, int64_t dt_ld,
                                   const float* A, const float* conv_w, const float* conv_b,
                                   const float* dt_bias,
                                   const float* init_ssm_state, const void* init_conv_state,
                                   float* final_ssm_state, void* final_conv_state,
                                   float* decay,
                                   void* workspace, size_t workspace_bytes,
                                   void* stream);

/* State passing between the pieces of a split sequence (the companion of
 * ssd_mixer_prefill_state; same citations): writes the state entering piece r,
 *   H_in(0) = init,  H_in(j+1) = decay[j] * H_in(j) + state[j],  j < r,
 * where state[j] is piece j's final SSM state from a zero initial state and decay[j] its
 * decay. decay [npieces][batch][nheads] fp32; state [npieces][batch][nheads][headdim][dstate]
 * fp32 (only pieces 0..r-1 are read); init [batch][nheads][headdim][dstate] or NULL = zeros;
 * out the same shape (may alias init). Device pointers, 16-byte aligned (decay: 4). */
SSD_API ssd_status ssd_mixer_state_pass(int64_t batch, int32_t nheads, int32_t headdim, int32_t dstate,
                                int32_t r, const float* decay, const float* state,
                                const float* init, float* out, void* stream);

/* Bytes of device workspace ssd_mixer_prefill_varlen needs for `dims` (dims->batch
 * sequences, dims->seqlen packed tokens in total); 0 when the dims are invalid or the
 * shape is one the packed entry point does not run. */
SSD_API size_t ssd_mixer_prefill_varlen_workspace_size(const ssd_dims* dims);

/* Prefill of packed variable-length sequences on state slots: b sequences of any
 * lengths, their tokens back to back in one token dimension, each continuing from (or
 * starting afresh on) the state slot it owns. This is the engine case of gllm PR #86,
 * section "Validation": several sequences in one batch, each Mamba layer picking up the
 * recurrent state of its own slot, of which one may be prefilling while another decodes
 * (a one-token sequence here runs the same arithmetic as ssd_mixer_decode_step).
 *
 * dims->batch = b sequences; dims->seqlen = T, the total number of packed tokens;
 * dims->chunk as for ssd_mixer_prefill.
 * cu_seqlens [b+1] int32 (device): sequence i owns packed rows cu_seqlens[i] ..
 *   cu_seqlens[i+1]-1, with cu_seqlens[0] = 0, non-decreasing, cu_seqlens[b] = T. A
 *   length may be 0: the final states are then the initial ones (the slot's own, or
 *   zeros where has_init is 0).
 * slot_idx [b] int32 (device; NULL = sequence i uses slot i): distinct, in range.
 * has_init [b] uint8 (device; NULL = all nonzero): nonzero = the sequence continues from
 *   the states in its slot; 0 = it starts from zero states (a new prompt).
 * x, z [T][HP]; B, C [T][GN]; dt [T][H]; y [T][HP]: packed rows with the strides given,
 *   same alignment rules as ssd_mixer_prefill.
 * ssm_state [nslots][H][P][N] fp32 and conv_state [nslots][Cc][K-1]: read as the initial
 *   states where has_init says so, and overwritten in place with the final states.
 * workspace: ssd_mixer_prefill_varlen_workspace_size(dims) bytes, 256-byte aligned.
 * Runs the tensor-core kernel only: bf16 activations, P = 64, N = 128 and 2 or a multiple
 * of 4 heads per group; other shapes return SSD_ERR_UNSUPPORTED. The library cannot check
 * device-resident cu_seqlens, slot_idx or has_init. */
SSD_API ssd_status ssd_mixer_prefill_varlen(const ssd_dims* dims,
                                    const int32_t* cu_seqlens, const int32_t* slot_idx,
                                    const uint8_t* has_init,
                                    const void* x, int64_t x_ld,
                                    const void* z, int64_t z_ld,
                                    const void* B, int64_t B_ld,
                                    const void* C, int64_t C_ld,
                                    const void* dt, int64_t dt_ld,
                                    const float* A, const float* D,
                                    const float* conv_w, const float* conv_b,
                                    const float* dt_bias, const float* norm_w,
                                    float* ssm_state, void* conv_state,
                                    void* y, int64_t y_ld,
                                    void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Decode step: advance b sequences by one token each, in place on their state
 * slots (the one-token-at-a-time decode of gllm PR #86, section "Validation", where
 * each Mamba layer picks up from the state held in the sequence's slot).
 *
 * dims->seqlen must be 1 and dims->chunk is ignored. x, z [b][HP]; B, C [b][GN];
 * dt [b][H] with row strides x_ld ... dt_ld between sequences.
 * ssm_state [nslots][H][P][N] fp32 and conv_state [nslots][Cc][K-1] are read and
 * rewritten in place for the slots named by slot_idx [b] (int32, device; NULL =
 * sequence i uses slot i). Slot indices must be distinct and in range; the library
 * cannot check device-resident indices. y [b][HP] (y_ld) receives the output. */
SSD_API ssd_status ssd_mixer_decode_step(const ssd_dims* dims,
                                 const void* x, int64_t x_ld,
                                 const void* z, int64_t z_ld,
                                 const void* B, int64_t B_ld,
                                 const void* C, int64_t C_ld,
                                 const void* dt, int64_t dt_ld,
                                 const float* A, const float* D,
                                 const float* conv_w, const float* conv_b,
                                 const float* dt_bias, const float* norm_w,
                                 float* ssm_state, void* conv_state,
                                 const int32_t* slot_idx,
                                 void* y, int64_t y_ld,
                                 void* stream);

/* Size of the fixed device scratch array used by ssd_mixer_prefill_static. */
#define SSD_MIXER_STATIC_WORKSPACE_BYTES (64u * 1024u * 1024u)

/* Prefill without a caller-supplied workspace (no counterpart in the pages: this is a
 * library convenience). For callers that cannot allocate device memory -- a plugin
 * slot that receives only tensors and a stream, or a process whose device memory is
 * wholly reserved by its own pool so that a cudaMalloc would fail or would stall the
 * device mid-loop. Same arguments and results as ssd_mixer_prefill, minus the
 * workspace: the scratch is a file-scope device array of
 * SSD_MIXER_STATIC_WORKSPACE_BYTES that every GPU loading this library holds until the
 * process exits. The library allocates nothing here either.
 *  - Calls needing more scratch than that (ssd_mixer_prefill_workspace_size(dims) >
 *    SSD_MIXER_STATIC_WORKSPACE_BYTES) return SSD_ERR_TOO_LARGE and launch nothing.
 *  - The first call in a CUDA context (with that context current) looks up the array's
 *    device address and caches it under the context's unique ID, so a caller's own
 *    non-primary context, or a context created after cudaDeviceReset, gets its own
 *    lookup; make the first call in a context before any stream capture.
 *  - All calls in a context share the one array, which keeps the last call's contents.
 *    Calls that overlap on the GPU (other streams, no ordering between them) race on it
 *    and give wrong results: order them on one stream or with events.
 *  - A bounded device-side wait that gives up is recorded in the array's status word, not
 *    in the return value: read it with ssd_mixer_prefill_static_status. */
SSD_API ssd_status ssd_mixer_prefill_static(const ssd_dims* dims,
                                    const void* x, int64_t x_ld,
                                    const void* z, int64_t z_ld,
                                    const void* B, int64_t B_ld,
                                    const void* C, int64_t C_ld,
                                    const void* dt, int64_t dt_ld,
                                    const float* A, const float* D,
                                    const float* conv_w, const float* conv_b,
                                    const float* dt_bias, const float* norm_w,
                                    const float* init_ssm_state, const void* init_conv_state,
                                    void* y, int64_t y_ld,
                                    float* final_ssm_state, void* final_conv_state,
                                    void* stream);

/* Status word of the fixed array that ssd_mixer_prefill_static uses, in the current
 * context (no counterpart in the pages, like the entry point it serves): the same reading
 * as ssd_mixer_workspace_status, for the last static call enqueued in this context.
 * Synchronises `stream`; call it on the stream of that prefill. Returns SSD_OK,
 * SSD_ERR_TIMEOUT or SSD_ERR_DEVICE as ssd_mixer_workspace_status does, or SSD_ERR_CUDA if
 * the array's address cannot be looked up. */
SSD_API ssd_status ssd_mixer_prefill_static_status(void* stream);

/* One projection of the mixer layer on the tensor cores: C[M][N] = A[M][K] . W[N][K]^T, bf16
 * inputs and output with fp32 accumulation (in_proj maps the block's hidden state to the packed
 * [z | x | B | C | dt] row, out_proj maps y back to the model width: gllm PR #86 "feat(model):
 * Nemotron-H hybrid (Mamba2 + attention + MoE) on the CPU", section "2. feat(model): Nemotron-H
 * on the CPU", mixer table row M). A [M][K] with row stride lda, W [N][K] (the row-major weight
 * of an N-output linear map) with row stride ldw, C [M][N] with row stride ldc, all in elements;
 * K and the strides multiples of 8, pointers 16-byte aligned; M, N, K below 2^31. workspace:
 * 256 device bytes, 256-byte aligned, for the status word (ssd_mixer_workspace_status). Returns
 * SSD_ERR_UNSUPPORTED for other sizes or alignments. Device pointers owned by the caller; C must
 * not overlap A or W. */
SSD_API ssd_status ssd_mixer_projection(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                                        const void* W, int64_t ldw, void* C, int64_t ldc,
                                        void* workspace, void* stream);

/* Bytes of device workspace ssd_mixer_layer_prefill needs; 0 when the dims or d_model are
 * invalid or unsupported. */
SSD_API size_t ssd_mixer_layer_workspace_size(const ssd_dims* dims, int64_t d_model);

/* The whole mixer layer for a prefill: out = out_proj(core(in_proj(hidden))), the pages'
 * in_proj -> CausalConv1D -> SSMScan -> GatedRMSNorm -> out_proj (gllm PR #86, section "2.
 * feat(model): Nemotron-H on the CPU", mixer table row M). in_proj emits one packed row per token,
 * split [z | x | B | C | dt] (gllm PR #86, "Supporting changes"; Modalities PR #459, commit notes
 * on mamba2.py); the core then runs on column slices of that row with nothing copied.
 *
 * hidden [b][L][d_model] bf16 (row stride hidden_ld); W_in [2HP + 2GN + H][d_model] bf16 and
 * W_out [d_model][HP] bf16, row-major, 16-byte aligned; the core's parameters and states as for
 * ssd_mixer_prefill; out [b][L][d_model] bf16 (row stride out_ld). bf16 activations only;
 * d_model, the strides and 2HP + 2GN + H multiples of 8; the core's shape rules as for
 * ssd_mixer_prefill. workspace: ssd_mixer_layer_workspace_size bytes, 256-byte aligned; it holds
 * the packed in_proj output and y, and its status word is read by ssd_mixer_workspace_status.
 * norm_in_out_proj: when the core's norm group is wider than one cluster of the tensor-core
 * kernel (more than 4 heads per group), 0 finishes the norm with the core's own pass over y, and
 * nonzero finishes it inside out_proj instead (the group RMS scale and norm_w applied to
 * out_proj's input tiles in shared memory before their MMAs; no second pass over y, but more
 * shared-memory traffic per tile, measured slower on a B200). Ignored for other shapes. */
SSD_API ssd_status ssd_mixer_layer_prefill(const ssd_dims* dims, int64_t d_model,
                                           const void* hidden, int64_t hidden_ld,
                                           const void* W_in, const void* W_out,
                                           const float* A, const float* D,
                                           const float* conv_w, const float* conv_b,
                                           const float* dt_bias, const float* norm_w,
                                           const float* init_ssm_state, const void* init_conv_state,
                                           void* out, int64_t out_ld,
                                           float* final_ssm_state, void* final_conv_state,
                                           int norm_in_out_proj,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream);

/* Bytes of device workspace ssd_mixer_backward needs for `dims`; 0 when the dims are
 * invalid or the shape is one the backward does not run. About (b L (4 HP + Cc + 2 H
 * (P/16) N + H (P/16) + 2 H) + b (L/64) H P N) * 4 bytes: the recompute forward's
 * intermediates (the state entering every 64-token chunk among them) and the gradient
 * partial sums. */
SSD_API size_t ssd_mixer_backward_workspace_size(const ssd_dims* dims);

/* Backward pass of the mixer core: the vector-Jacobian product of ssd_mixer_prefill.
 * The pages train the Mamba-2 mixer through this scan and test gradient flow through it
 * (Modalities PR #459, sections "Testing" and "Caveats"). For a scalar loss whose
 * gradients with respect to the prefill's outputs are dy (for y), dfinal_ssm_state and
 * dfinal_conv_state, this writes the gradients with respect to every input, parameter and
 * initial state of a prefill with the same inputs. The forward is recomputed inside the
 * call (nothing is saved from the training forward); dims->chunk is checked as for
 * ssd_mixer_prefill but not used.
 *
 * Inputs: as ssd_mixer_prefill (same shapes, dtypes, strides and alignment rules; NULL
 *   initial states are zeros), plus
 *   dy [b][L][HP] activation dtype, row stride dy_ld;
 *   dfinal_ssm_state [b][H][P][N] fp32 and dfinal_conv_state [b][Cc][K-1] fp32, or NULL
 *   when the loss does not depend on the final states.
 * Outputs (written, not added to):
 *   dx, dz [b][L][HP], dB, dC [b][L][GN], ddt [b][L][H]: activation dtype, row strides;
 *   dA, dD, ddt_bias [H], dconv_w [Cc][K], dconv_b [Cc], dnorm_w [HP]: fp32;
 *   dinit_ssm_state [b][H][P][N] fp32 and dinit_conv_state [b][Cc][K-1] fp32, or NULL
 *   when not wanted (computed whether or not the initial states were given).
 * workspace: ssd_mixer_backward_workspace_size(dims) bytes, 256-byte aligned.
 * Runs on CUDA cores in fp32 for fp32 and bf16 activations, P in {16, 32, 64} and N in
 * {16, 32, 64, 128}; other shapes return SSD_ERR_UNSUPPORTED, as do rows longer than
 * 2,097,120 tokens. The parameter gradients are fp32 sums whose order of addition is not
 * fixed, so they may differ from call to call in the last bits. Outputs must not overlap
 * inputs or one another. All pointers are device pointers owned by the caller. */
SSD_API ssd_status ssd_mixer_backward(const ssd_dims* dims,
                              const void* x, int64_t x_ld,
                              const void* z, int64_t z_ld,
                              const void* B, int64_t B_ld,
                              const void* C, int64_t C_ld,
                              const void* dt, int64_t dt_ld,
                              const float* A, const float* D,
                              const float* conv_w, const float* conv_b,
                              const float* dt_bias, const float* norm_w,
                              const float* init_ssm_state, const void* init_conv_state,
                              const void* dy, int64_t dy_ld,
                              const float* dfinal_ssm_state, const float* dfinal_conv_state,
                              void* dx, int64_t dx_ld,
                              void* dz, int64_t dz_ld,
                              void* dB, int64_t dB_ld,
                              void* dC, int64_t dC_ld,
                              void* ddt, int64_t ddt_ld,
                              float* dA, float* dD, float* dconv_w, float* dconv_b,
                              float* ddt_bias, float* dnorm_w,
                              float* dinit_ssm_state, float* dinit_conv_state,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/* Reads the device status word that the prefill kernels keep at the start of
 * `workspace` (the last call that used it clears it on its stream before its first kernel,
 * and its kernels record the first failure). Synchronises `stream`. Returns SSD_OK;
 * SSD_ERR_TIMEOUT if a bounded device-side wait gave up; SSD_ERR_DEVICE if a kernel found
 * its dynamic shared memory base misaligned and did no work, or, in the bounds-checked build
 * (libssd_mixer_debug.so), an index fell outside its buffer and its access was skipped. In
 * every error case that call's outputs are invalid. */
SSD_API ssd_status ssd_mixer_workspace_status(const void* workspace, void* stream);

/* Self-test of the failure path that every bounded device-side wait in the library takes
 * (the tensor-core kernels wait on mbarriers for TMA loads, peer copies and tensor-core
 * commits; each wait gives up after a limit of clock cycles, sets the status word at the
 * start of the workspace and stops waiting). One thread waits on an mbarrier that nothing
 * arrives on (arrive = 0) or that it has already arrived on itself (arrive != 0), giving up
 * after limit_cycles SM clock cycles (0 .. 4e9). Afterwards ssd_mixer_workspace_status on
 * the same workspace reports SSD_ERR_TIMEOUT (gave up) or SSD_OK. workspace: at least 256
 * bytes, 256-byte aligned, device memory owned by the caller; only its status word is
 * written. Launches one single-CTA kernel on `stream`; the context stays usable. */
SSD_API ssd_status ssd_mixer_selftest_wait(void* workspace, long long limit_cycles, int arrive, void* stream);

/* Number of kernels this library has launched in the process so far (all entry
 * points, all devices). A caller reads it before and after a region to count the
 * library's launches in that region. Not a compute call; thread-safe. */
SSD_API long long ssd_mixer_launch_count(void);

/* Switch per-kernel timing on (1) or off (0). While on, every kernel launch is
 * bracketed by a pair of CUDA events recorded on the launching stream (a few
 * microseconds of host overhead per launch; the kernels themselves are unchanged). The
 * launches of one prefill call whose rows run as pieces may overlap one another, so they
 * share one pair: one span, counted as that many launches. Off by default. */
SSD_API void ssd_mixer_profile_enable(int on);

/* Collects the event pairs recorded since the last read: waits for each to complete
 * and sums their elapsed times per kernel name. Writes up to max_entries rows into
 * names (static strings owned by the library), total_ms and launches; returns the
 * number of rows. Host arrays owned by the caller. */
SSD_API int ssd_mixer_profile_read(const char** names, double* total_ms, int* launches,
                                   int max_entries);

/* Static description of a status code (never NULL). */
SSD_API const char* ssd_status_string(ssd_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
SSD_API int ssd_mixer_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_MIXER_H */
