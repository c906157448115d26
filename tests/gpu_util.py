"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run the C ABI
through the binding, compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import Workload

SEQ_KEYS = ("x", "z", "B", "C", "dt")
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dims_of(w: Workload, seqlen=None, batch=None, chunk=None) -> sm.Dims:
    return sm.Dims(batch if batch is not None else w.batch,
                   seqlen if seqlen is not None else w.seqlen, w.nheads, w.headdim, w.ngroups,
                   w.dstate, chunk or w.chunk, w.dconv, w.eps, w.act)


def oracle_dims(d: sm.Dims) -> oracle.Dims:
    return oracle.Dims(d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)


def to_dev(inp: dict, act: str, device="cuda") -> dict:
    """float32 numpy inputs (already rounded to the activation dtype) -> device tensors."""
    adt = torch.bfloat16 if act == "bf16" else torch.float32
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
            continue
        t = torch.from_numpy(np.ascontiguousarray(v))
        if k in SEQ_KEYS or k == "init_conv":
            t = t.to(adt)
        out[k] = t.to(device)
    return out


def gpu_prefill(d: sm.Dims, dv: dict, init_ssm="init_ssm", init_conv="init_conv", **kw):
    return sm.prefill(d, dv["x"], dv["z"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["D"],
                      dv["conv_w"], dv["conv_b"], dv["dt_bias"], dv["norm_w"],
                      dv.get(init_ssm) if isinstance(init_ssm, str) else init_ssm,
                      dv.get(init_conv) if isinstance(init_conv, str) else init_conv, **kw)


def slice_seq(inp: dict, t0: int, t1: int) -> dict:
    """Tokens t0..t1 of every row, as contiguous arrays (the ABI's row layout puts token t of
    row i at (i*L + t) * ld, which a sequence slice of a multi-row batch does not have)."""
    out = {}
    for k, v in inp.items():
        if k in SEQ_KEYS and v is not None:
            v = v[:, t0:t1]
            v = v.contiguous() if isinstance(v, torch.Tensor) else np.ascontiguousarray(v)
        out[k] = v
    return out


def relerr(got, ref) -> float:
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    return float(np.max(np.abs(got - ref)) / max(float(np.max(np.abs(ref))), 1e-30))


def assert_close(name, got, ref, tol):
    e = relerr(got, ref)
    assert e <= tol, f"{name}: max|err|/max|ref| = {e:.3e} > {tol:.1e}"
    return e
