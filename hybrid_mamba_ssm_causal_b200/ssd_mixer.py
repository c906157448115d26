"""Thin Python binding of the C ABI in include/ssd_mixer.h (argument marshalling only).

Every step of the mixer runs in libssd_mixer.so; this module only turns torch tensors
into device pointers, leading dimensions and the current CUDA stream. There is no
fallback: if the library is missing or the tensors are not on a CUDA device, the call
raises.

The entry points keep the C names:
  ssd_mixer_prefill_workspace_size(dims) -> int
  ssd_mixer_prefill(dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                    init_ssm_state, init_conv_state, y, final_ssm_state, final_conv_state,
                    workspace, stream=None)
  ssd_mixer_decode_step(dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                        ssm_state, conv_state, slot_idx, y, stream=None)
  ssd_mixer_backward(dims, <prefill inputs>, dy, dfinal_ssm_state, dfinal_conv_state,
                     <gradients>, workspace, stream=None)
plus :func:`prefill` / :func:`decode_step` / :func:`backward`, which allocate the outputs
and workspace with torch and call the entry points above.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# the library the binding opens: libssd_mixer.so, or another build of it (the bounds-checked
# libssd_mixer_debug.so) named by SSD_MIXER_LIBRARY
LIB_PATH = os.environ.get("SSD_MIXER_LIBRARY") or os.path.join(HERE, "libssd_mixer.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT, SSD_ERR_TOO_LARGE, SSD_ERR_DEVICE = range(7)
SSD_MIXER_STATIC_WORKSPACE_BYTES = 64 * 1024 * 1024
SSD_F32, SSD_BF16 = 0, 1
SYMBOLS = ("ssd_mixer_prefill_workspace_size", "ssd_mixer_prefill", "ssd_mixer_decode_step",
           "ssd_mixer_workspace_status", "ssd_status_string", "ssd_mixer_version",
           "ssd_mixer_launch_count", "ssd_mixer_profile_enable", "ssd_mixer_profile_read",
           "ssd_mixer_prefill_static", "ssd_mixer_prefill_varlen_workspace_size", "ssd_mixer_prefill_varlen",
           "ssd_mixer_prefill_state_workspace_size", "ssd_mixer_prefill_state", "ssd_mixer_state_pass",
           "ssd_mixer_backward_workspace_size", "ssd_mixer_backward", "ssd_mixer_selftest_wait",
           "ssd_mixer_prefill_static_status", "ssd_mixer_prefill_path", "ssd_mixer_prefill_plan",
           "ssd_mixer_prefill_stage_offsets",
           "ssd_mixer_projection", "ssd_mixer_layer_workspace_size", "ssd_mixer_layer_prefill")
SSD_PATH_NONE, SSD_PATH_CUDA_CORES, SSD_PATH_TENSOR_CORES = range(3)


class SsdError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class _CDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int32), ("headdim", ctypes.c_int32),
                ("ngroups", ctypes.c_int32), ("dstate", ctypes.c_int32),
                ("dconv", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("eps", ctypes.c_float), ("act", ctypes.c_int32)]


@dataclass(frozen=True)
class Dims:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    chunk: int = 128
    dconv: int = 4
    eps: float = 1e-5
    act: str = "bf16"

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def xbc_channels(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.dstate

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.act == "bf16" else torch.float32

    def c(self) -> _CDims:
        return _CDims(self.batch, self.seqlen, self.nheads, self.headdim, self.ngroups,
                      self.dstate, self.dconv, self.chunk, self.eps,
                      SSD_BF16 if self.act == "bf16" else SSD_F32)


_lib = None


def load_library(path: str = LIB_PATH):
    """Open libssd_mixer.so (raises if it is absent: build it with
    ``python -m hybrid_mamba_ssm_causal_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run python -m hybrid_mamba_ssm_causal_b200.build)")
    lib = ctypes.CDLL(path)
    V, I64, P = ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p
    FP = ctypes.c_void_p
    lib.ssd_mixer_prefill_workspace_size.argtypes = [ctypes.POINTER(_CDims)]
    lib.ssd_mixer_prefill_workspace_size.restype = ctypes.c_size_t
    lib.ssd_mixer_prefill.argtypes = ([ctypes.POINTER(_CDims)] + [P, I64] * 5 + [FP] * 6 +
                                      [FP, P, P, I64, FP, P, P, ctypes.c_size_t, V])
    lib.ssd_mixer_prefill.restype = ctypes.c_int
    lib.ssd_mixer_decode_step.argtypes = ([ctypes.POINTER(_CDims)] + [P, I64] * 5 + [FP] * 6 +
                                          [FP, P, P, P, I64, V])
    lib.ssd_mixer_decode_step.restype = ctypes.c_int
    lib.ssd_mixer_prefill_static.argtypes = ([ctypes.POINTER(_CDims)] + [P, I64] * 5 + [FP] * 6 +
                                             [FP, P, P, I64, FP, P, V])
    lib.ssd_mixer_prefill_static.restype = ctypes.c_int
    lib.ssd_mixer_projection.argtypes = [I64, I64, I64, P, I64, P, I64, P, I64, P, V]
    lib.ssd_mixer_projection.restype = ctypes.c_int
    lib.ssd_mixer_layer_workspace_size.argtypes = [ctypes.POINTER(_CDims), I64]
    lib.ssd_mixer_layer_workspace_size.restype = ctypes.c_size_t
    lib.ssd_mixer_layer_prefill.argtypes = ([ctypes.POINTER(_CDims), I64, P, I64, P, P] + [FP] * 6 +
                                            [FP, P, P, I64, FP, P, ctypes.c_int, P, ctypes.c_size_t, V])
    lib.ssd_mixer_layer_prefill.restype = ctypes.c_int
    lib.ssd_mixer_prefill_path.argtypes = [ctypes.POINTER(_CDims)]
    lib.ssd_mixer_prefill_path.restype = ctypes.c_int
    IP = ctypes.POINTER(ctypes.c_int)
    lib.ssd_mixer_prefill_plan.argtypes = [ctypes.POINTER(_CDims), ctypes.c_int, IP, IP, IP, IP]
    lib.ssd_mixer_prefill_plan.restype = ctypes.c_int
    SZP = ctypes.POINTER(ctypes.c_size_t)
    lib.ssd_mixer_prefill_stage_offsets.argtypes = [ctypes.POINTER(_CDims), SZP, SZP, SZP]
    lib.ssd_mixer_prefill_stage_offsets.restype = ctypes.c_int
    lib.ssd_mixer_prefill_static_status.argtypes = [V]
    lib.ssd_mixer_prefill_static_status.restype = ctypes.c_int
    lib.ssd_mixer_prefill_varlen_workspace_size.argtypes = [ctypes.POINTER(_CDims)]
    lib.ssd_mixer_prefill_varlen_workspace_size.restype = ctypes.c_size_t
    lib.ssd_mixer_prefill_varlen.argtypes = ([ctypes.POINTER(_CDims), P, P, P] + [P, I64] * 5 + [FP] * 6 +
                                             [FP, P, P, I64, P, ctypes.c_size_t, V])
    lib.ssd_mixer_prefill_varlen.restype = ctypes.c_int
    lib.ssd_mixer_prefill_state_workspace_size.argtypes = [ctypes.POINTER(_CDims)]
    lib.ssd_mixer_prefill_state_workspace_size.restype = ctypes.c_size_t
    lib.ssd_mixer_prefill_state.argtypes = ([ctypes.POINTER(_CDims)] + [P, I64] * 4 + [FP] * 4 +
                                            [FP, P, FP, P, FP, P, ctypes.c_size_t, V])
    lib.ssd_mixer_prefill_state.restype = ctypes.c_int
    lib.ssd_mixer_state_pass.argtypes = [I64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                         FP, FP, FP, FP, V]
    lib.ssd_mixer_state_pass.restype = ctypes.c_int
    lib.ssd_mixer_backward_workspace_size.argtypes = [ctypes.POINTER(_CDims)]
    lib.ssd_mixer_backward_workspace_size.restype = ctypes.c_size_t
    lib.ssd_mixer_backward.argtypes = ([ctypes.POINTER(_CDims)] + [P, I64] * 5 + [FP] * 6 + [FP, P] +
                                       [P, I64, FP, FP] + [P, I64] * 5 + [FP] * 8 + [P, ctypes.c_size_t, V])
    lib.ssd_mixer_backward.restype = ctypes.c_int
    lib.ssd_mixer_selftest_wait.argtypes = [P, ctypes.c_longlong, ctypes.c_int, V]
    lib.ssd_mixer_selftest_wait.restype = ctypes.c_int
    lib.ssd_mixer_workspace_status.argtypes = [P, V]
    lib.ssd_mixer_workspace_status.restype = ctypes.c_int
    lib.ssd_status_string.argtypes = [ctypes.c_int]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_mixer_version.argtypes = []
    lib.ssd_mixer_version.restype = ctypes.c_int
    lib.ssd_mixer_launch_count.argtypes = []
    lib.ssd_mixer_launch_count.restype = ctypes.c_longlong
    lib.ssd_mixer_profile_enable.argtypes = [ctypes.c_int]
    lib.ssd_mixer_profile_enable.restype = None
    lib.ssd_mixer_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    lib.ssd_mixer_profile_read.restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != SSD_OK:
        raise SsdError(status, f"{what}: {load_library().ssd_status_string(status).decode()}")


def _dev(t, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    return t.data_ptr()


def _rows(t: torch.Tensor, name: str, rows: int, width: int):
    """Pointer and leading dimension of a [.., rows, width]-shaped activation view whose
    consecutive rows (tokens) are ``ld`` elements apart and whose last dim is unit-stride."""
    if t.dim() < 2 or t.shape[-1] != width:
        raise ValueError(f"{name}: expected last dim {width}, got {tuple(t.shape)}")
    if t.numel() // width != rows:
        raise ValueError(f"{name}: expected {rows} rows, got {t.numel() // width}")
    if rows == 0:          # nothing is read or written; any strides will do
        return _dev(t, name), width
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: last dim must have unit stride")
    ld = t.stride(-2)
    # all leading dims must be an even tiling by ld (token t of row i at (i*L + t) * ld)
    expect = ld
    for d in range(t.dim() - 2, -1, -1):
        if t.shape[d] > 1 and t.stride(d) != expect:
            raise ValueError(f"{name}: rows must be evenly strided")
        expect *= t.shape[d]
    return _dev(t, name), ld


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def ssd_mixer_prefill_workspace_size(dims: Dims) -> int:
    cd = dims.c()
    return int(load_library().ssd_mixer_prefill_workspace_size(ctypes.byref(cd)))


def ssd_mixer_prefill(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                      init_ssm_state, init_conv_state, y, final_ssm_state, final_conv_state,
                      workspace, stream=None) -> None:
    lib = load_library()
    rows = dims.batch * dims.seqlen
    HP, GN = dims.d_inner, dims.ngroups * dims.dstate
    args = []
    for t, name, w in ((x, "x", HP), (z, "z", HP), (B, "B", GN), (C, "C", GN), (dt, "dt", dims.nheads)):
        args += list(_rows(t, name, rows, w))
    py, y_ld = _rows(y, "y", rows, HP)
    cd = dims.c()
    st = lib.ssd_mixer_prefill(
        ctypes.byref(cd), *args, _dev(A, "A"), _dev(D, "D"), _dev(conv_w, "conv_w"),
        _dev(conv_b, "conv_b"), _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"),
        _dev(init_ssm_state, "init_ssm_state"), _dev(init_conv_state, "init_conv_state"),
        py, y_ld, _dev(final_ssm_state, "final_ssm_state"), _dev(final_conv_state, "final_conv_state"),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_mixer_prefill")


def ssd_mixer_prefill_static(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                             init_ssm_state, init_conv_state, y, final_ssm_state, final_conv_state,
                             stream=None) -> int:
    """The prefill with its scratch in the library's fixed device array (for callers that
    cannot allocate device memory); returns the C status instead of raising."""
    lib = load_library()
    rows = dims.batch * dims.seqlen
    HP, GN = dims.d_inner, dims.ngroups * dims.dstate
    args = []
    for t, name, w in ((x, "x", HP), (z, "z", HP), (B, "B", GN), (C, "C", GN), (dt, "dt", dims.nheads)):
        args += list(_rows(t, name, rows, w))
    py, y_ld = _rows(y, "y", rows, HP)
    cd = dims.c()
    return int(lib.ssd_mixer_prefill_static(
        ctypes.byref(cd), *args, _dev(A, "A"), _dev(D, "D"), _dev(conv_w, "conv_w"),
        _dev(conv_b, "conv_b"), _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"),
        _dev(init_ssm_state, "init_ssm_state"), _dev(init_conv_state, "init_conv_state"),
        py, y_ld, _dev(final_ssm_state, "final_ssm_state"), _dev(final_conv_state, "final_conv_state"),
        _stream(stream)))


def ssd_mixer_projection(A, W, C, workspace, stream=None) -> None:
    """C = A . W^T on the tensor cores: A [M, K], W [N, K], C [M, N], bf16 (row strides from the
    tensors; last dims unit-stride). workspace: >= 256 bytes for the status word."""
    M, K = A.shape[-2], A.shape[-1]
    N = W.shape[0]
    for t, nm in ((A, "A"), (W, "W"), (C, "C")):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError(f"{nm}: bf16 with unit-stride rows expected")
    st = load_library().ssd_mixer_projection(M, N, K, _dev(A, "A"), A.stride(-2), _dev(W, "W"), W.stride(-2),
                                             _dev(C, "C"), C.stride(-2), _dev(workspace, "workspace"), _stream(stream))
    _check(st, "ssd_mixer_projection")


def ssd_mixer_layer_workspace_size(dims: Dims, d_model: int) -> int:
    cd = dims.c()
    return int(load_library().ssd_mixer_layer_workspace_size(ctypes.byref(cd), d_model))


def layer_prefill(dims: Dims, hidden, W_in, W_out, A, D, conv_w, conv_b, dt_bias, norm_w,
                  init_ssm_state=None, init_conv_state=None, workspace=None, out=None, norm_in_out_proj=False,
                  stream=None):
    """The whole mixer layer (in_proj, the core, out_proj) through ssd_mixer_layer_prefill.
    hidden [b, L, d_model] bf16; W_in [2HP + 2GN + H, d_model]; W_out [d_model, HP].
    norm_in_out_proj: finish a wide group's norm inside out_proj instead of in the core.
    Returns (out [b, L, d_model], final_ssm_state, final_conv_state)."""
    lib = load_library()
    d_model = hidden.shape[-1]
    rows = dims.batch * dims.seqlen
    ph, hld = _rows(hidden, "hidden", rows, d_model)
    dev = hidden.device
    if workspace is None:
        n = ssd_mixer_layer_workspace_size(dims, d_model)
        if n == 0:
            raise SsdError(SSD_ERR_UNSUPPORTED, "ssd_mixer_layer_workspace_size: unsupported dims")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    if out is None:
        y = torch.empty(dims.batch, dims.seqlen, d_model, dtype=torch.bfloat16, device=dev)
        fs = torch.empty(dims.batch, dims.nheads, dims.headdim, dims.dstate, dtype=torch.float32, device=dev)
        fc = torch.empty(dims.batch, dims.d_inner + 2 * dims.ngroups * dims.dstate, dims.dconv - 1,
                         dtype=torch.bfloat16, device=dev)
    else:
        y, fs, fc = out
    py, yld = _rows(y, "out", rows, d_model)
    cd = dims.c()
    st = lib.ssd_mixer_layer_prefill(
        ctypes.byref(cd), d_model, ph, hld, _dev(W_in, "W_in"), _dev(W_out, "W_out"), _dev(A, "A"), _dev(D, "D"),
        _dev(conv_w, "conv_w"), _dev(conv_b, "conv_b"), _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"),
        _dev(init_ssm_state, "init_ssm_state"), _dev(init_conv_state, "init_conv_state"), py, yld,
        _dev(fs, "final_ssm_state"), _dev(fc, "final_conv_state"), 1 if norm_in_out_proj else 0,
        _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_mixer_layer_prefill")
    return y, fs, fc


def ssd_mixer_prefill_path(dims: Dims) -> int:
    """SSD_PATH_TENSOR_CORES, SSD_PATH_CUDA_CORES or SSD_PATH_NONE: which kernels a prefill of
    these dims runs (a host-side query)."""
    cd = dims.c()
    return int(load_library().ssd_mixer_prefill_path(ctypes.byref(cd)))


def ssd_mixer_prefill_plan(dims: Dims, sms: int = 0) -> dict:
    """How the tensor-core main kernel runs a prefill of these dims on ``sms`` SMs (0 = this
    device's): launches per call, pieces per (sequence, head) row, blocks per piece, CTAs per
    launch (a host-side query)."""
    cd = dims.c()
    out = [ctypes.c_int(0) for _ in range(4)]
    st = load_library().ssd_mixer_prefill_plan(ctypes.byref(cd), sms, *[ctypes.byref(o) for o in out])
    _check(st, "ssd_mixer_prefill_plan")
    return dict(zip(("launches", "pieces", "piece_blocks", "ctas_per_launch"), (o.value for o in out)))


def prefill_uses_tensor_cores(dims: Dims) -> bool:
    return ssd_mixer_prefill_path(dims) == SSD_PATH_TENSOR_CORES


def ssd_mixer_prefill_stage_offsets(dims: Dims) -> dict:
    """Byte offsets of xbc_act, delta and y_pre in the workspace of a CUDA-core prefill."""
    cd = dims.c()
    o = [ctypes.c_size_t(0) for _ in range(3)]
    _check(load_library().ssd_mixer_prefill_stage_offsets(ctypes.byref(cd), *[ctypes.byref(v) for v in o]),
           "ssd_mixer_prefill_stage_offsets")
    return {"xbc_act": o[0].value, "delta": o[1].value, "y_pre": o[2].value}


def ssd_mixer_prefill_static_status(stream=None) -> int:
    """Status word of the fixed array that ssd_mixer_prefill_static uses (synchronises the stream)."""
    return int(load_library().ssd_mixer_prefill_static_status(_stream(stream)))


def ssd_mixer_prefill_varlen_workspace_size(dims: Dims) -> int:
    cd = dims.c()
    return int(load_library().ssd_mixer_prefill_varlen_workspace_size(ctypes.byref(cd)))


def ssd_mixer_prefill_varlen(dims: Dims, cu_seqlens, slot_idx, has_init, x, z, B, C, dt, A, D, conv_w,
                             conv_b, dt_bias, norm_w, ssm_state, conv_state, y, workspace,
                             stream=None) -> None:
    """Packed variable-length prefill on state slots: dims.batch sequences, dims.seqlen packed
    tokens in total (x ... y are [T, width] row views); cu_seqlens int32 [b+1], slot_idx int32
    [b] or None, has_init uint8 [b] or None, all on the device."""
    lib = load_library()
    rows = dims.seqlen
    HP, GN = dims.d_inner, dims.ngroups * dims.dstate
    if cu_seqlens.dtype != torch.int32 or (slot_idx is not None and slot_idx.dtype != torch.int32):
        raise TypeError("cu_seqlens and slot_idx must be int32")
    if has_init is not None and has_init.dtype != torch.uint8:
        raise TypeError("has_init must be uint8")
    args = []
    for t, name, w in ((x, "x", HP), (z, "z", HP), (B, "B", GN), (C, "C", GN), (dt, "dt", dims.nheads)):
        args += list(_rows(t, name, rows, w))
    py, y_ld = _rows(y, "y", rows, HP)
    cd = dims.c()
    st = lib.ssd_mixer_prefill_varlen(
        ctypes.byref(cd), _dev(cu_seqlens, "cu_seqlens"), _dev(slot_idx, "slot_idx"), _dev(has_init, "has_init"),
        *args, _dev(A, "A"), _dev(D, "D"), _dev(conv_w, "conv_w"), _dev(conv_b, "conv_b"),
        _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"), _dev(ssm_state, "ssm_state"),
        _dev(conv_state, "conv_state"), py, y_ld, _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_mixer_prefill_varlen")


def ssd_mixer_prefill_state_workspace_size(dims: Dims) -> int:
    cd = dims.c()
    return int(load_library().ssd_mixer_prefill_state_workspace_size(ctypes.byref(cd)))


def ssd_mixer_prefill_state(dims: Dims, x, B, C, dt, A, conv_w, conv_b, dt_bias, init_ssm_state,
                            init_conv_state, final_ssm_state, final_conv_state, decay, workspace,
                            stream=None) -> None:
    """State-only prefill: final states and the per-(row, head) decay, no output rows."""
    lib = load_library()
    rows = dims.batch * dims.seqlen
    GN = dims.ngroups * dims.dstate
    args = []
    for t, name, w in ((x, "x", dims.d_inner), (B, "B", GN), (C, "C", GN), (dt, "dt", dims.nheads)):
        args += list(_rows(t, name, rows, w))
    cd = dims.c()
    st = lib.ssd_mixer_prefill_state(
        ctypes.byref(cd), *args, _dev(A, "A"), _dev(conv_w, "conv_w"), _dev(conv_b, "conv_b"),
        _dev(dt_bias, "dt_bias"), _dev(init_ssm_state, "init_ssm_state"), _dev(init_conv_state, "init_conv_state"),
        _dev(final_ssm_state, "final_ssm_state"), _dev(final_conv_state, "final_conv_state"), _dev(decay, "decay"),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_mixer_prefill_state")


def ssd_mixer_state_pass(r: int, decay, state, init, out, stream=None) -> None:
    """State entering piece r of a split sequence: decay [npieces, b, H], state
    [npieces, b, H, P, N] (zero-start final states of the pieces), init [b, H, P, N] or None."""
    b, H, P, N = out.shape
    st = load_library().ssd_mixer_state_pass(b, H, P, N, r, _dev(decay, "decay"), _dev(state, "state"),
                                             _dev(init, "init"), _dev(out, "out"), _stream(stream))
    _check(st, "ssd_mixer_state_pass")


def ssd_mixer_decode_step(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                          ssm_state, conv_state, slot_idx, y, stream=None) -> None:
    lib = load_library()
    HP, GN = dims.d_inner, dims.ngroups * dims.dstate
    args = []
    for t, name, w in ((x, "x", HP), (z, "z", HP), (B, "B", GN), (C, "C", GN), (dt, "dt", dims.nheads)):
        args += list(_rows(t, name, dims.batch, w))
    py, y_ld = _rows(y, "y", dims.batch, HP)
    if slot_idx is not None and slot_idx.dtype != torch.int32:
        raise TypeError("slot_idx must be int32")
    cd = dims.c()
    st = lib.ssd_mixer_decode_step(
        ctypes.byref(cd), *args, _dev(A, "A"), _dev(D, "D"), _dev(conv_w, "conv_w"),
        _dev(conv_b, "conv_b"), _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"),
        _dev(ssm_state, "ssm_state"), _dev(conv_state, "conv_state"), _dev(slot_idx, "slot_idx"),
        py, y_ld, _stream(stream))
    _check(st, "ssd_mixer_decode_step")


def ssd_mixer_backward_workspace_size(dims: Dims) -> int:
    cd = dims.c()
    return int(load_library().ssd_mixer_backward_workspace_size(ctypes.byref(cd)))


def ssd_mixer_backward(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                       init_ssm_state, init_conv_state, dy, dfinal_ssm_state, dfinal_conv_state,
                       dx, dz, dB, dC, ddt, dA, dD, dconv_w, dconv_b, ddt_bias, dnorm_w,
                       dinit_ssm_state, dinit_conv_state, workspace, stream=None) -> None:
    lib = load_library()
    rows = dims.batch * dims.seqlen
    HP, GN, H = dims.d_inner, dims.ngroups * dims.dstate, dims.nheads
    ins = []
    for t, name, w in ((x, "x", HP), (z, "z", HP), (B, "B", GN), (C, "C", GN), (dt, "dt", H)):
        ins += list(_rows(t, name, rows, w))
    outs = []
    for t, name, w in ((dx, "dx", HP), (dz, "dz", HP), (dB, "dB", GN), (dC, "dC", GN), (ddt, "ddt", H)):
        outs += list(_rows(t, name, rows, w))
    pdy, dy_ld = _rows(dy, "dy", rows, HP)
    cd = dims.c()
    st = lib.ssd_mixer_backward(
        ctypes.byref(cd), *ins, _dev(A, "A"), _dev(D, "D"), _dev(conv_w, "conv_w"), _dev(conv_b, "conv_b"),
        _dev(dt_bias, "dt_bias"), _dev(norm_w, "norm_w"), _dev(init_ssm_state, "init_ssm_state"),
        _dev(init_conv_state, "init_conv_state"), pdy, dy_ld, _dev(dfinal_ssm_state, "dfinal_ssm_state"),
        _dev(dfinal_conv_state, "dfinal_conv_state"), *outs, _dev(dA, "dA"), _dev(dD, "dD"),
        _dev(dconv_w, "dconv_w"), _dev(dconv_b, "dconv_b"), _dev(ddt_bias, "ddt_bias"), _dev(dnorm_w, "dnorm_w"),
        _dev(dinit_ssm_state, "dinit_ssm_state"), _dev(dinit_conv_state, "dinit_conv_state"),
        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "ssd_mixer_backward")


def ssd_mixer_selftest_wait(workspace, limit_cycles: int, arrive: bool, stream=None) -> None:
    st = load_library().ssd_mixer_selftest_wait(_dev(workspace, "workspace"), int(limit_cycles), int(bool(arrive)),
                                                _stream(stream))
    _check(st, "ssd_mixer_selftest_wait")


def ssd_mixer_workspace_status(workspace, stream=None) -> int:
    return int(load_library().ssd_mixer_workspace_status(_dev(workspace, "workspace"), _stream(stream)))


def alloc_workspace(dims: Dims, device="cuda") -> torch.Tensor:
    n = ssd_mixer_prefill_workspace_size(dims)
    if n == 0:
        raise SsdError(SSD_ERR_UNSUPPORTED, "ssd_mixer_prefill_workspace_size: unsupported dims")
    return torch.empty(n, dtype=torch.uint8, device=device)


def prefill(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
            init_ssm_state=None, init_conv_state=None, workspace=None, out=None, stream=None):
    """Allocate y, the final states and (if not given) the workspace, then run
    :func:`ssd_mixer_prefill`. Returns (y, final_ssm_state, final_conv_state)."""
    dev = x.device
    b, L, H, P, N = dims.batch, dims.seqlen, dims.nheads, dims.headdim, dims.dstate
    if out is None:
        y = torch.empty(b, L, dims.d_inner, dtype=dims.torch_dtype, device=dev)
        fs = torch.empty(b, H, P, N, dtype=torch.float32, device=dev)
        fc = torch.empty(b, dims.xbc_channels, dims.dconv - 1, dtype=dims.torch_dtype, device=dev)
    else:
        y, fs, fc = out
    ws = workspace if workspace is not None else alloc_workspace(dims, dev)
    ssd_mixer_prefill(dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                      init_ssm_state, init_conv_state, y, fs, fc, ws, stream)
    return y, fs, fc


def backward(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w, dy,
             init_ssm_state=None, init_conv_state=None, dfinal_ssm_state=None, dfinal_conv_state=None,
             workspace=None, stream=None) -> dict:
    """Allocate the gradients and (if not given) the workspace, then run
    :func:`ssd_mixer_backward`. Returns a dict of gradients keyed like the inputs (x, z, B, C,
    dt, A, D, conv_w, conv_b, dt_bias, norm_w, init_ssm, init_conv)."""
    dev = x.device
    b, L, H, P, N, Cc = dims.batch, dims.seqlen, dims.nheads, dims.headdim, dims.dstate, dims.xbc_channels
    HP, GN, act = dims.d_inner, dims.ngroups * dims.dstate, dims.torch_dtype
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"x": torch.empty(b, L, HP, dtype=act, device=dev), "z": torch.empty(b, L, HP, dtype=act, device=dev),
         "B": torch.empty(b, L, GN, dtype=act, device=dev), "C": torch.empty(b, L, GN, dtype=act, device=dev),
         "dt": torch.empty(b, L, H, dtype=act, device=dev), "A": torch.empty(H, **f32), "D": torch.empty(H, **f32),
         "conv_w": torch.empty(Cc, dims.dconv, **f32), "conv_b": torch.empty(Cc, **f32),
         "dt_bias": torch.empty(H, **f32), "norm_w": torch.empty(HP, **f32),
         "init_ssm": torch.empty(b, H, P, N, **f32), "init_conv": torch.empty(b, Cc, dims.dconv - 1, **f32)}
    if workspace is None:
        n = ssd_mixer_backward_workspace_size(dims)
        if n == 0:
            raise SsdError(SSD_ERR_UNSUPPORTED, "ssd_mixer_backward_workspace_size: unsupported dims")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    ssd_mixer_backward(dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w, init_ssm_state,
                       init_conv_state, dy, dfinal_ssm_state, dfinal_conv_state, g["x"], g["z"], g["B"], g["C"],
                       g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"], g["dt_bias"], g["norm_w"],
                       g["init_ssm"], g["init_conv"], workspace, stream)
    return g


def decode_step(dims: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                ssm_state, conv_state, slot_idx=None, y=None, stream=None):
    """Run :func:`ssd_mixer_decode_step` (states updated in place); returns y."""
    if y is None:
        y = torch.empty(dims.batch, dims.d_inner, dtype=dims.torch_dtype, device=x.device)
    ssd_mixer_decode_step(dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                          ssm_state, conv_state, slot_idx, y, stream)
    return y
