"""GPU parity of the backward pass (ssd_mixer_backward) with the fp64 backward oracle
(oracle/backward.py, pinned against finite differences of the forward oracle).

Every gradient (x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w, both initial states)
is compared as max|err| / max|ref| <= 1e-4 for fp32 activations and <= 2e-2 for bf16, on
shapes that span several 16-token recompute chunks with ragged tails, rows shorter than the
conv window, zero tokens, one and several heads per group, and with and without initial
states and final-state gradients. The small_bf16 workload's shape is checked on one group
over both rows (the backward separates by group like the forward, so the group's
gradients, its heads' and channels' parameter gradients included, are those of its
sub-problem).
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs, round_bf16
from oracle.backward import prefill_vjp
from tests.gpu_util import TOL, assert_close, dims_of, oracle_dims, to_dev

pytestmark = pytest.mark.gpu

GRADS = ("x", "z", "B", "C", "dt", "A", "D", "conv_w", "conv_b", "dt_bias", "norm_w", "init_ssm", "init_conv")


def workload(act, b, L, H, P, G, N, init, seed):
    base = WORKLOADS["tiny_f32"] if act == "f32" else WORKLOADS["small_bf16"]
    return base.with_(batch=b, seqlen=L, nheads=H, headdim=P, ngroups=G, dstate=N, chunk=64,
                      init_ssm_std=0.1 if init else 0.0, init_conv_std=1.0 if init else 0.0, seed=seed)


def cotangents(w, final_grads, seed):
    rng = np.random.default_rng(seed)
    rnd = (lambda *s: round_bf16(rng.standard_normal(s))) if w.act == "bf16" else (lambda *s: rng.standard_normal(s))
    dout = rnd(w.batch, w.seqlen, w.d_inner).astype(np.float32)
    dfs = rng.standard_normal((w.batch, w.nheads, w.headdim, w.dstate)).astype(np.float32) if final_grads else None
    dfc = rng.standard_normal((w.batch, w.xbc_channels, 3)).astype(np.float32) if final_grads else None
    return dout, dfs, dfc


def run_gpu(w, inp, dout, dfs, dfc):
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    adt = torch.bfloat16 if w.act == "bf16" else torch.float32
    dy = torch.from_numpy(dout).to(adt).cuda()
    cuda = lambda a: None if a is None else torch.from_numpy(a).cuda()
    g = sm.backward(d, dv["x"], dv["z"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["D"], dv["conv_w"], dv["conv_b"],
                    dv["dt_bias"], dv["norm_w"], dy, dv.get("init_ssm"), dv.get("init_conv"), cuda(dfs), cuda(dfc))
    torch.cuda.synchronize()
    return g


def check(name, w, g, ref, keys=GRADS, index=None):
    tol = TOL[w.act]
    for k in keys:
        r = ref[k]
        if np.size(r) == 0:
            continue
        got = g[k] if index is None else index(k, g[k])
        assert_close(f"{name}: d{k}", got, r, tol)


CASES = [
    # act, b, L, H, P, G, N, initial states, final-state gradients
    ("f32", 2, 77, 4, 16, 2, 32, True, True),      # ragged: 4 chunks + 13 tokens
    ("f32", 1, 100, 4, 64, 1, 64, False, False),   # four heads per group, dout only
    ("f32", 1, 45, 8, 32, 1, 16, True, True),      # eight heads per group
    ("f32", 1, 0, 2, 16, 1, 16, True, True),       # no tokens: the states' gradients pass through
    ("bf16", 2, 300, 8, 64, 2, 128, True, True),   # the tensor-core forward's shape class
    ("bf16", 1, 2, 4, 64, 2, 128, True, True),     # shorter than the conv window
    ("bf16", 2, 33, 4, 16, 4, 16, False, True),    # one head per group
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(case):
    act, b, L, H, P, G, N, init, fg = case
    w = workload(act, b, L, H, P, G, N, init, seed=300 + L + H)
    inp = make_prefill_inputs(w)
    dout, dfs, dfc = cotangents(w, fg, seed=400 + L)
    ref = prefill_vjp(oracle_dims(dims_of(w)), inp, dout, dfs, dfc)
    g = run_gpu(w, inp, dout, dfs, dfc)
    check("-".join(map(str, case)), w, g, ref)


def test_backward_small_bf16_workload_one_group():
    """small_bf16 (b2 L2048 H32xP64 G8 N128) on the GPU; group 5 over both rows against the
    oracle's backward of that group's sub-problem."""
    w = WORKLOADS["small_bf16"]
    inp = make_prefill_inputs(w)
    dout, dfs, dfc = cotangents(w, True, seed=501)
    g = run_gpu(w, inp, dout, dfs, dfc)
    d = oracle_dims(dims_of(w))
    grp = 5
    sd, sub, xs, hs, conv_idx = oracle.group_subproblem(d, grp, inp)
    HP, GN, N = w.d_inner, w.ngroups * w.dstate, w.dstate
    bs = slice(grp * N, (grp + 1) * N)
    ref = prefill_vjp(sd, sub, dout[:, :, xs], dfs[:, hs], dfc[:, conv_idx])
    pick = {"x": lambda t: t[:, :, xs], "z": lambda t: t[:, :, xs], "B": lambda t: t[:, :, bs],
            "C": lambda t: t[:, :, bs], "dt": lambda t: t[:, :, hs], "A": lambda t: t[hs], "D": lambda t: t[hs],
            "conv_w": lambda t: t[torch.as_tensor(conv_idx, device=t.device)],
            "conv_b": lambda t: t[torch.as_tensor(conv_idx, device=t.device)], "dt_bias": lambda t: t[hs],
            "norm_w": lambda t: t[xs], "init_ssm": lambda t: t[:, hs],
            "init_conv": lambda t: t[:, torch.as_tensor(conv_idx, device=t.device)]}
    check("small_bf16 group 5", w, g, ref, index=lambda k, t: pick[k](t))
