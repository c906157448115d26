"""fp64 CPU oracle of the Mamba-2 mixer core (TEST INFRASTRUCTURE ONLY).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package. The CUDA library never imports it, and it
never imports the CUDA library.

Contents
  ssd_oracle.c   the oracle proper: sequential Mamba-2 recurrence in fp64, with the
                 causal conv + SiLU, softplus(dt + dt_bias) and the SiLU(z)-gated
                 group RMSNorm (built to liboracle_ssd.so by :func:`build`).
  forms.py       two further, separately written fp64 forms of the scan (the chunked
                 SSD decomposition and the quadratic "dual" matrix form), used only to
                 pin the oracle, and the chunked form of the scan's backward.
  backward.py    the backward pass (vector-Jacobian product) of the mixer core in fp64,
                 pinned against finite differences of the compiled oracle.
  layer.py       the whole mixer layer (in_proj, the core, out_proj) in fp64: the
                 computation that fusing the projections with the core must reproduce.

Pins: every function here is checked in tests/test_oracle_*.py against closed forms,
invariants and brute force. The mapping conventions that no page fixes (tap order,
head -> group map, gate-then-normalise order) are readings, not pins: parity
unpinned against the real model for those conventions only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_ssd.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c with the host C compiler (IEEE fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int32), ("headdim", ctypes.c_int32),
                ("ngroups", ctypes.c_int32), ("dstate", ctypes.c_int32),
                ("dconv", ctypes.c_int32), ("eps", ctypes.c_double)]


def _open(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.ssd_oracle_prefill.argtypes = [ctypes.POINTER(_Dims)] + [P] * 19 + [ctypes.c_int]
    lib.ssd_oracle_prefill.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _open(_LIB)
    return _lib


class use_library:
    """Context manager that points the oracle at another build of ssd_oracle.c (used by
    the mutation tests, which compile deliberately broken copies on the CPU)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _open(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


@dataclass(frozen=True)
class Dims:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    dconv: int = 4
    eps: float = 1e-5

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def xbc_channels(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.dstate


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def prefill(d: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
            init_ssm=None, init_conv=None, stages: bool = False, nthreads: int | None = None):
    """Run the oracle over a whole batch. Inputs of any float dtype are upcast exactly.

    Shapes: x, z [b, L, H*P]; B, C [b, L, G*N]; dt [b, L, H]; A, D, dt_bias [H];
    conv_w [Cc, K]; conv_b [Cc]; norm_w [H*P]; init_ssm [b, H, P, N]; init_conv [b, Cc, K-1].
    Returns dict(y, final_ssm, final_conv) and, if ``stages``, xbc_act, delta, y_pre.
    """
    lib = _load()
    b, L, H, P, G, N, K = d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv
    Cc = d.xbc_channels
    args = [_f64(a) for a in (x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w)]
    shapes = [(b, L, H * P), (b, L, H * P), (b, L, G * N), (b, L, G * N), (b, L, H), (H,), (H,),
              (Cc, K), (Cc,), (H,), (H * P,)]
    for a, s in zip(args, shapes):
        if a.shape != s:
            raise ValueError(f"oracle: shape {a.shape} != {s}")
    i_ssm, i_conv = _f64(init_ssm), _f64(init_conv)
    if i_ssm is not None and i_ssm.shape != (b, H, P, N):
        raise ValueError("oracle: init_ssm shape")
    if i_conv is not None and i_conv.shape != (b, Cc, K - 1):
        raise ValueError("oracle: init_conv shape")
    out = {
        "y": np.empty((b, L, H * P)),
        "final_ssm": np.empty((b, H, P, N)),
        "final_conv": np.empty((b, Cc, K - 1)),
    }
    if stages:
        out["xbc_act"] = np.empty((b, L, Cc))
        out["delta"] = np.empty((b, L, H))
        out["y_pre"] = np.empty((b, L, H * P))
    dims = _Dims(b, L, H, P, G, N, K, float(d.eps))
    rc = lib.ssd_oracle_prefill(
        ctypes.byref(dims), *[_ptr(a) for a in args], _ptr(i_ssm), _ptr(i_conv),
        _ptr(out["y"]), _ptr(out["final_ssm"]), _ptr(out["final_conv"]),
        _ptr(out.get("xbc_act")), _ptr(out.get("delta")), _ptr(out.get("y_pre")),
        int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return out


def group_subproblem(d: Dims, g: int, inputs: dict, batch_rows=None):
    """Slice the self-contained sub-problem of one group (its heads, x/z/y channels,
    B and C channels, conv taps and norm weights), optionally for some batch rows.

    The mixer core separates exactly by (batch row, group): nothing outside the group
    enters its outputs. Returns (sub_dims, sub_inputs, channel_slice, head_slice).
    """
    H, P, G, N = d.nheads, d.headdim, d.ngroups, d.dstate
    r = H // G
    HP, GN = H * P, G * N
    xs = slice(g * r * P, (g + 1) * r * P)
    hs = slice(g * r, (g + 1) * r)
    bs = slice(g * N, (g + 1) * N)
    conv_idx = np.concatenate([np.arange(xs.start, xs.stop), HP + np.arange(bs.start, bs.stop),
                               HP + GN + np.arange(bs.start, bs.stop)])
    rows = slice(None) if batch_rows is None else batch_rows
    sub = {
        "x": inputs["x"][rows, :, xs], "z": inputs["z"][rows, :, xs],
        "B": inputs["B"][rows, :, bs], "C": inputs["C"][rows, :, bs],
        "dt": inputs["dt"][rows, :, hs], "A": inputs["A"][hs], "D": inputs["D"][hs],
        "conv_w": inputs["conv_w"][conv_idx], "conv_b": inputs["conv_b"][conv_idx],
        "dt_bias": inputs["dt_bias"][hs], "norm_w": inputs["norm_w"][xs],
        "init_ssm": None if inputs.get("init_ssm") is None else inputs["init_ssm"][rows, hs],
        "init_conv": None if inputs.get("init_conv") is None else inputs["init_conv"][rows][:, conv_idx],
    }
    nb = sub["x"].shape[0]
    sd = Dims(nb, d.seqlen, r, P, 1, N, d.dconv, d.eps)
    return sd, sub, xs, hs, conv_idx


def prefill_dict(d: Dims, inp: dict, **kw):
    """:func:`prefill` with the inputs passed as a dict (keys as in :func:`group_subproblem`)."""
    return prefill(d, inp["x"], inp["z"], inp["B"], inp["C"], inp["dt"], inp["A"], inp["D"],
                   inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"],
                   inp.get("init_ssm"), inp.get("init_conv"), **kw)


def decay(dt, A, dt_bias):
    """exp(A[h] * sum_t delta_t[h]) per (row, head), delta = softplus(dt + dt_bias): the product
    of the per-token factors exp(delta_t A) of the state recurrence, i.e. the factor by which
    a prefill over these tokens carries its initial SSM state into its final one.
    dt [b, L, H]; returns [b, H]."""
    u = np.asarray(dt, np.float64) + np.asarray(dt_bias, np.float64)
    # softplus(u) = log(1 + e^u) written as max(u, 0) + log1p(e^-|u|): exact for every u, no cutoff
    delta = np.maximum(u, 0.0) + np.log1p(np.exp(-np.abs(u)))
    return np.exp(np.asarray(A, np.float64) * delta.sum(axis=1))


def prefill_varlen(d: Dims, cu_seqlens, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                   ssm_state, conv_state, slot_idx=None, has_init=None, nthreads: int | None = None):
    """Packed variable-length prefill on state slots. Sequence i owns packed rows
    cu_seqlens[i] .. cu_seqlens[i+1]-1 of x, z, B, C, dt ([T, width]); it is an independent
    prefill that starts from the states of its slot (or from zeros where has_init[i] == 0)
    and leaves its final states in that slot (several sequences in one engine batch, each on
    its own slot: gllm PR #86, section "Validation"). ``d.batch`` and ``d.seqlen`` are not
    used. Returns y [T, H*P] and NEW state arrays; inputs are not modified."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nseq = len(cu) - 1
    slots = np.arange(nseq) if slot_idx is None else np.asarray(slot_idx)
    init = np.ones(nseq, dtype=bool) if has_init is None else np.asarray(has_init) != 0
    ssm_state = np.array(ssm_state, dtype=np.float64, copy=True)
    conv_state = np.array(conv_state, dtype=np.float64, copy=True)
    x, z, B, C, dt = (np.asarray(a) for a in (x, z, B, C, dt))
    y = np.zeros((x.shape[0], d.nheads * d.headdim))
    for i in range(nseq):
        s0, s1 = int(cu[i]), int(cu[i + 1])
        di = Dims(1, s1 - s0, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
        k = slots[i]
        out = prefill(di, x[None, s0:s1], z[None, s0:s1], B[None, s0:s1], C[None, s0:s1], dt[None, s0:s1],
                      A, D, conv_w, conv_b, dt_bias, norm_w,
                      ssm_state[k][None] if init[i] else None, conv_state[k][None] if init[i] else None,
                      nthreads=nthreads)
        y[s0:s1] = out["y"][0]
        ssm_state[k] = out["final_ssm"][0]
        conv_state[k] = out["final_conv"][0]
    return y, ssm_state, conv_state


def decode_step(d: Dims, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w,
                ssm_state, conv_state, slot_idx=None, nthreads: int | None = None):
    """One single-token decode step on state slots (returns y [b, H*P] and NEW state
    arrays; inputs are not modified). A decode step is the prefill of one token that
    starts from the slot's states and leaves its final states in the slot (the
    one-token-at-a-time decode case of gllm PR #86, section "Validation")."""
    b = np.asarray(x).shape[0]
    slots = np.arange(b) if slot_idx is None else np.asarray(slot_idx)
    d1 = Dims(b, 1, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    ssm_state = np.array(ssm_state, dtype=np.float64, copy=True)
    conv_state = np.array(conv_state, dtype=np.float64, copy=True)
    out = prefill(d1, np.asarray(x)[:, None], np.asarray(z)[:, None], np.asarray(B)[:, None],
                  np.asarray(C)[:, None], np.asarray(dt)[:, None], A, D, conv_w, conv_b, dt_bias,
                  norm_w, ssm_state[slots], conv_state[slots], nthreads=nthreads)
    ssm_state[slots] = out["final_ssm"]
    conv_state[slots] = out["final_conv"]
    return out["y"][:, 0], ssm_state, conv_state
