"""Pins of the fp64 backward oracle (oracle/backward.py) against things other than itself
(CPU only).

- Its forward restatement equals the compiled oracle (oracle.prefill) to rounding.
- Every gradient equals central finite differences of the compiled oracle along a random
  direction: d/de L(theta + e V) at e = 0 with L = sum(dout y) + sum(dfinal_ssm final_ssm)
  + sum(dfinal_conv final_conv), for every input, parameter and initial state, with and
  without gradients on the final states, for groups of one and several heads, and for
  rows shorter than the conv window.
- Closed forms: dnorm_w = sum over tokens of dout * out / norm_w (out taken from the
  compiled oracle); with dout = 0 the gradient reaching the initial SSM state is the
  decay exp(A sum delta) times dfinal_ssm (oracle.decay), and the one reaching the
  initial conv state is dfinal_conv shifted by the row length.
"""
import numpy as np
import pytest

import oracle
from oracle.backward import forward_saved, prefill_vjp
from tests.test_oracle_pins import rand_problem

KEYS = ("x", "z", "B", "C", "dt", "A", "D", "conv_w", "conv_b", "dt_bias", "norm_w", "init_ssm", "init_conv")


def loss(d, inp, dout, dfs=None, dfc=None):
    o = oracle.prefill_dict(d, inp, nthreads=1)
    val = float(np.sum(dout * o["y"]))
    if dfs is not None:
        val += float(np.sum(dfs * o["final_ssm"]))
    if dfc is not None:
        val += float(np.sum(dfc * o["final_conv"]))
    return val


def directional_fd(d, inp, key, V, dout, dfs, dfc, eps=1e-6):
    plus, minus = dict(inp), dict(inp)
    plus[key] = inp[key] + eps * V
    minus[key] = inp[key] - eps * V
    return (loss(d, plus, dout, dfs, dfc) - loss(d, minus, dout, dfs, dfc)) / (2 * eps)


def cotangents(rng, d, final_grads):
    b, L, H, P, G, N = d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate
    dout = rng.standard_normal((b, L, H * P))
    dfs = rng.standard_normal((b, H, P, N)) if final_grads else None
    dfc = rng.standard_normal((b, d.xbc_channels, 3)) if final_grads else None
    return dout, dfs, dfc


def check_all_gradients(d, inp, dout, dfs, dfc, rng, vjp=prefill_vjp):
    """Every gradient against the finite difference along one random direction. Missing
    initial states are checked as zeros (the same forward)."""
    grads = vjp(d, inp, dout, dfs, dfc)
    full = dict(inp)
    b, H, P, N, Cc = d.batch, d.nheads, d.headdim, d.dstate, d.xbc_channels
    if full.get("init_ssm") is None:
        full["init_ssm"] = np.zeros((b, H, P, N))
    if full.get("init_conv") is None:
        full["init_conv"] = np.zeros((b, Cc, 3))
    for k in KEYS:
        V = rng.standard_normal(np.shape(full[k]))
        an = float(np.sum(grads[k] * V))
        fd = directional_fd(d, full, k, V, dout, dfs, dfc)
        bound = 1e-7 * (np.linalg.norm(grads[k]) * np.linalg.norm(V) + 1.0)
        assert abs(an - fd) <= bound, f"d/d{k}: vjp {an!r} vs finite difference {fd!r}"


@pytest.mark.parametrize("init", [True, False])
@pytest.mark.parametrize("L", [0, 1, 2, 5, 23])
def test_forward_restatement_equals_compiled_oracle(L, init):
    rng = np.random.default_rng(100 + L)
    d, inp = rand_problem(rng, b=2, L=L, H=4, P=3, G=2, N=5, init=init)
    ref = oracle.prefill_dict(d, inp)
    f = forward_saved(d, inp["x"], inp["z"], inp["B"], inp["C"], inp["dt"], inp["A"], inp["D"], inp["conv_w"],
                      inp["conv_b"], inp["dt_bias"], inp["norm_w"], inp["init_ssm"], inp["init_conv"])
    for ours, theirs in (("out", "y"), ("final_ssm", "final_ssm"), ("final_conv", "final_conv")):
        if ref[theirs].size:
            assert np.max(np.abs(f[ours] - ref[theirs])) <= 1e-12 * max(1.0, np.max(np.abs(ref[theirs])))


@pytest.mark.parametrize("b,L,H,P,G,N,init,final_grads", [
    (2, 11, 4, 3, 2, 5, True, True),      # two heads per group, every cotangent
    (2, 11, 4, 3, 2, 5, True, False),     # dout only
    (1, 9, 3, 2, 3, 4, False, True),      # one head per group, no initial states
    (1, 2, 2, 2, 1, 3, True, True),       # shorter than the conv window
    (1, 1, 2, 2, 1, 2, True, True),       # one token
    (1, 19, 4, 2, 1, 3, True, True),      # four heads sharing B and C
])
def test_gradients_match_finite_differences(b, L, H, P, G, N, init, final_grads):
    rng = np.random.default_rng(b * 1000 + L * 10 + H + 7 * init)
    d, inp = rand_problem(rng, b=b, L=L, H=H, P=P, G=G, N=N, init=init)
    dout, dfs, dfc = cotangents(rng, d, final_grads)
    check_all_gradients(d, inp, dout, dfs, dfc, rng)


def test_norm_weight_gradient_closed_form():
    """out = (normalised gate) * norm_w, so dL/dnorm_w = sum over tokens of dout * out / norm_w."""
    rng = np.random.default_rng(211)
    d, inp = rand_problem(rng, b=2, L=17, H=4, P=3, G=2, N=5)
    dout = rng.standard_normal((2, 17, 12))
    out = oracle.prefill_dict(d, inp)["y"]
    g = prefill_vjp(d, inp, dout)["norm_w"]
    ref = np.sum(dout * out, axis=(0, 1)) / inp["norm_w"]
    assert np.max(np.abs(g - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_state_gradients_closed_form_without_output_gradient():
    """With dout = 0 the loss sees the initial SSM state only through final = a H0 + (terms
    free of H0), a = exp(A sum delta) per (row, head). With dout = 0 and dfinal_ssm = 0 it
    sees the initial conv state only through the final conv state, the last three entries
    of s = [init_conv ; raw inputs]: final_conv[i] = init_conv[L + i] while L + i < 3."""
    rng = np.random.default_rng(212)
    for L in (0, 1, 2, 3, 8):
        d, inp = rand_problem(rng, b=2, L=L, H=4, P=3, G=2, N=5)
        dfs = rng.standard_normal((2, 4, 3, 5))
        dfc = rng.standard_normal((2, d.xbc_channels, 3))
        dout = np.zeros((2, L, 12))
        g = prefill_vjp(d, inp, dout, dfs, dfc)
        a = oracle.decay(inp["dt"], inp["A"], inp["dt_bias"])
        assert np.max(np.abs(g["init_ssm"] - a[:, :, None, None] * dfs)) <= 1e-14 * np.max(np.abs(dfs))
        for k in ("norm_w", "D", "z"):    # none of these reaches the final states
            assert not np.any(g[k])
        g = prefill_vjp(d, inp, dout, np.zeros_like(dfs), dfc)
        want = np.zeros_like(dfc)
        if L < 3:
            want[:, :, L:] = dfc[:, :, :3 - L]
        assert np.array_equal(g["init_conv"], want)


def test_backward_separates_by_group():
    """The gradients of one group's inputs, of its heads' parameters and of its channels'
    conv and norm weights are those of the group's own sub-problem (the forward separates by
    group). The full-size GPU test relies on this to check one group of a large workload."""
    rng = np.random.default_rng(213)
    d, inp = rand_problem(rng, b=2, L=23, H=4, P=3, G=2, N=5)
    dout = rng.standard_normal((2, 23, 12))
    dfs = rng.standard_normal((2, 4, 3, 5))
    dfc = rng.standard_normal((2, d.xbc_channels, 3))
    full = prefill_vjp(d, inp, dout, dfs, dfc)
    for g in range(d.ngroups):
        sd, sub, xs, hs, conv_idx = oracle.group_subproblem(d, g, inp)
        part = prefill_vjp(sd, sub, dout[:, :, xs], dfs[:, hs], dfc[:, conv_idx])
        bs = slice(g * d.dstate, (g + 1) * d.dstate)
        pick = {"x": lambda a: a[:, :, xs], "z": lambda a: a[:, :, xs], "B": lambda a: a[:, :, bs],
                "C": lambda a: a[:, :, bs], "dt": lambda a: a[:, :, hs], "A": lambda a: a[hs], "D": lambda a: a[hs],
                "conv_w": lambda a: a[conv_idx], "conv_b": lambda a: a[conv_idx], "dt_bias": lambda a: a[hs],
                "norm_w": lambda a: a[xs], "init_ssm": lambda a: a[:, hs], "init_conv": lambda a: a[:, conv_idx]}
        for k in KEYS:
            want = pick[k](full[k])
            assert np.max(np.abs(part[k] - want)) <= 1e-12 * max(1.0, np.max(np.abs(want))), (g, k)


@pytest.mark.parametrize("Q", [1, 3, 8, 16, 64])
def test_chunked_backward_form_matches_the_sequential_one(Q):
    """The scan's backward written in the chunked block form (oracle/forms.py) agrees with
    the step-by-step backward of the recurrence for every chunk length, ragged tails
    included: two separately written forms of the same derivative."""
    from oracle.backward import scan_vjp
    from oracle.forms import chunked_scan_vjp
    rng = np.random.default_rng(300 + Q)
    L, H, P, G, N = 37, 4, 3, 2, 5
    d, inp = rand_problem(rng, b=1, L=L, H=H, P=P, G=G, N=N)
    f = forward_saved(d, inp["x"], inp["z"], inp["B"], inp["C"], inp["dt"], inp["A"], inp["D"], inp["conv_w"],
                      inp["conv_b"], inp["dt_bias"], inp["norm_w"], inp["init_ssm"], inp["init_conv"])
    r = H // G
    dy = rng.standard_normal((1, L, H, P))
    dHf = rng.standard_normal((1, H, P, N))
    seq = scan_vjp(f["Hs"], f["xs"], f["Bh"], f["Ch"], f["delta"], inp["A"], inp["D"], dy, dHf)
    dxs, dBh, dCh, ddelta, dA, dD, dH0 = seq
    want = {"x": dxs[0], "B": dBh[0].reshape(L, G, r, N).sum(axis=2), "C": dCh[0].reshape(L, G, r, N).sum(axis=2),
            "delta": ddelta[0], "A": dA, "D": dD, "H0": dH0[0]}
    got = chunked_scan_vjp(f["xs"][0], f["Bh"][0][:, ::r], f["Ch"][0][:, ::r], f["delta"][0], inp["A"], inp["D"],
                           inp["init_ssm"][0], dy[0], dHf[0], Q)
    for k, g in zip(("x", "B", "C", "delta", "A", "D", "H0"), got):
        assert np.max(np.abs(g - want[k])) <= 1e-10 * np.max(np.abs(want[k])), (Q, k)
