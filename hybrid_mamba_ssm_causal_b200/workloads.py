"""Seeded synthetic inputs for the SSD mixer core (shared by tests, bench and smoke).

This module holds only the input recipe: shapes, seeds, value distributions and the
rounding of draws to the activation dtype. It holds none of the mixer's arithmetic.

No page prints a dataset or a benchmark for this path, so every input is synthetic.
Distributions (one recipe for all workloads): x, z, B, C, dt_raw ~ N(0, 1);
dt_bias = softplus^-1(u) with u log-uniform on [1e-3, 1e-1]; A = -exp(U[0, ln 16]);
D ~ U[0, 1]; conv_w ~ U[-0.5, 0.5]; conv_b ~ U[-0.1, 0.1]; norm_w = 1 + N(0, 0.1);
eps = 1e-5. N(mu, s) takes s as the standard deviation. Draw order is fixed: x, z, B,
C, dt_raw, dt_bias, A, D, conv_w, conv_b, norm_w, then the initial states. Workload i
draws from ``numpy.random.default_rng(seed)`` with seed = i unless overridden. For
bf16 workloads every activation (and conv_w, conv_b, norm_w) is rounded to the
nearest bf16 value (ties to even) and carried as float32, so both sides see the same
numbers; A, D and dt_bias stay float32. Parameters are drawn before the initial
states, so changing batch or seqlen for a smaller test case keeps the same recipe.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    act: str            # "f32" or "bf16": dtype of x, z, B, C, dt, y and the conv state
    batch: int
    seqlen: int          # tokens per prefill call (decode: 1)
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    chunk: int
    dconv: int = 4
    eps: float = 1e-5
    init_ssm_std: float = 0.0     # 0 = zero initial SSM state
    init_conv_std: float = 0.0    # 0 = zero initial conv state
    calls: int = 1                # prefill calls chained through the returned states
    steps: int = 0                # decode steps (decode workload only)
    seed: int = 0

    @property
    def d_inner(self) -> int:
        return self.nheads * self.headdim

    @property
    def xbc_channels(self) -> int:
        return self.d_inner + 2 * self.ngroups * self.dstate

    @property
    def total_seqlen(self) -> int:
        return self.seqlen * self.calls

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of this library's test and benchmark plan.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", "f32", 1, 256, 4, 16, 1, 16, 64, seed=0),
    "small_bf16": Workload("small_bf16", "bf16", 2, 2048, 32, 64, 8, 128, 128, seed=1),
    "mid_bf16": Workload("mid_bf16", "bf16", 8, 4096, 64, 64, 8, 128, 128,
                         init_ssm_std=0.1, init_conv_std=1.0, seed=2),
    "long_bf16": Workload("long_bf16", "bf16", 1, 16384, 256, 64, 8, 128, 256, calls=2, seed=3),
    "decode_bf16": Workload("decode_bf16", "bf16", 256, 1, 128, 64, 8, 128, 128,
                            init_ssm_std=0.1, init_conv_std=0.1, steps=1000, seed=4),
}
WORKLOAD_ORDER = ["tiny_f32", "small_bf16", "mid_bf16", "long_bf16", "decode_bf16"]


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even); returns float32.
    NaN stays NaN (the rounding carry would otherwise turn a low-payload NaN into Inf)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32)
    # in 32-bit arithmetic: only NaN bit patterns can wrap, and those are put back below
    out = ((bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000))
    out = out.view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out = np.where(nan, a, out)
    return out


def _act(w: Workload, a: np.ndarray) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_bf16(a) if w.act == "bf16" else a


def _normal(rng, shape, std=1.0):
    return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)


def make_params(w: Workload, rng) -> dict:
    H, Cc, K = w.nheads, w.xbc_channels, w.dconv
    u = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=H))
    p = {
        "dt_bias": np.log(np.expm1(u)).astype(np.float32),
        "A": (-np.exp(rng.uniform(0.0, np.log(16.0), size=H))).astype(np.float32),
        "D": rng.uniform(0.0, 1.0, size=H).astype(np.float32),
        "conv_w": _act(w, rng.uniform(-0.5, 0.5, size=(Cc, K))),
        "conv_b": _act(w, rng.uniform(-0.1, 0.1, size=Cc)),
        "norm_w": _act(w, 1.0 + 0.1 * rng.standard_normal(size=w.d_inner)),
    }
    return p


def make_prefill_inputs(w: Workload, seed: int | None = None) -> dict:
    """All inputs of a prefill workload over its total sequence (``calls * seqlen``).

    Returns float32 numpy arrays: x, z [b, T, H*P]; B, C [b, T, G*N]; dt [b, T, H];
    parameters; init_ssm [b, H, P, N] and init_conv [b, Cc, K-1] (None when zero)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    b, T, HP, GN, H = w.batch, w.total_seqlen, w.d_inner, w.ngroups * w.dstate, w.nheads
    inp = {
        "x": _act(w, _normal(rng, (b, T, HP))),
        "z": _act(w, _normal(rng, (b, T, HP))),
        "B": _act(w, _normal(rng, (b, T, GN))),
        "C": _act(w, _normal(rng, (b, T, GN))),
        "dt": _act(w, _normal(rng, (b, T, H))),
    }
    inp.update(make_params(w, rng))
    inp["init_ssm"] = (_normal(rng, (b, H, w.headdim, w.dstate), w.init_ssm_std)
                       if w.init_ssm_std > 0 else None)
    inp["init_conv"] = (_act(w, _normal(rng, (b, w.xbc_channels, w.dconv - 1), w.init_conv_std))
                        if w.init_conv_std > 0 else None)
    return inp


def make_decode_inputs(w: Workload, steps: int, seed: int | None = None) -> dict:
    """Parameters, initial slot states and ``steps`` per-step token inputs of a decode
    workload: x, z [steps, b, H*P]; B, C [steps, b, G*N]; dt [steps, b, H]."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    b, HP, GN, H = w.batch, w.d_inner, w.ngroups * w.dstate, w.nheads
    inp = make_params(w, rng)
    inp["init_ssm"] = _normal(rng, (b, H, w.headdim, w.dstate), w.init_ssm_std)
    inp["init_conv"] = _act(w, _normal(rng, (b, w.xbc_channels, w.dconv - 1), w.init_conv_std))
    inp["x"] = _act(w, _normal(rng, (steps, b, HP)))
    inp["z"] = _act(w, _normal(rng, (steps, b, HP)))
    inp["B"] = _act(w, _normal(rng, (steps, b, GN)))
    inp["C"] = _act(w, _normal(rng, (steps, b, GN)))
    inp["dt"] = _act(w, _normal(rng, (steps, b, H)))
    return inp
