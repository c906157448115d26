"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test pins one part of oracle/ssd_oracle.c: closed forms, hand-computed cases,
two separately written forms of the scan (chunked SSD, quadratic dual matrix),
invariants (zero step, split-and-chain, causality, separability by group) and the
decode step. The scan's math follows the Mamba-2 recurrence that the Modalities PR
#459 ("feat(model): add Nemotron-3 Nano hybrid Mamba-Transformer MoE architecture",
section "Testing") validates its chunked scan against, and that gllm PR #86
("feat(model): Nemotron-H hybrid (Mamba2 + attention + MoE) on the CPU", paragraph
"Reference quirk") runs as its scan.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import Dims
from oracle.forms import chunked_scan, quadratic_scan

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(rng, b=2, L=40, H=4, P=4, G=2, N=8, K=4, init=True, dt_shift=0.0):
    d = Dims(b, L, H, P, G, N, K, 1e-5)
    Cc = d.xbc_channels
    inp = dict(
        x=rng.standard_normal((b, L, H * P)), z=rng.standard_normal((b, L, H * P)),
        B=rng.standard_normal((b, L, G * N)), C=rng.standard_normal((b, L, G * N)),
        dt=rng.standard_normal((b, L, H)) + dt_shift,
        A=-np.exp(rng.uniform(0, np.log(16), H)), D=rng.uniform(0, 1, H),
        conv_w=rng.uniform(-0.5, 0.5, (Cc, K)), conv_b=rng.uniform(-0.1, 0.1, Cc),
        dt_bias=np.log(np.expm1(np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H)))),
        norm_w=1 + 0.1 * rng.standard_normal(H * P),
        init_ssm=0.1 * rng.standard_normal((b, H, P, N)) if init else None,
        init_conv=rng.standard_normal((b, Cc, K - 1)) if init else None,
    )
    return d, inp


def run(d, inp, **kw):
    return oracle.prefill_dict(d, inp, **kw)


def scan_inputs(d, out, bi):
    """The scan's own inputs for batch row ``bi``, taken from the oracle's stage outputs."""
    H, P, G, N = d.nheads, d.headdim, d.ngroups, d.dstate
    HP, GN = H * P, G * N
    xa = out["xbc_act"][bi, :, :HP].reshape(d.seqlen, H, P)
    Ba = out["xbc_act"][bi, :, HP:HP + GN].reshape(d.seqlen, G, N)
    Ca = out["xbc_act"][bi, :, HP + GN:].reshape(d.seqlen, G, N)
    return xa, Ba, Ca, out["delta"][bi]


def rel(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- softplus, SiLU, conv

def identity_conv(d):
    w = np.zeros((d.xbc_channels, d.dconv))
    w[:, -1] = 1.0
    return w


def test_softplus_closed_forms():
    d = Dims(1, 5, 1, 1, 1, 1, 4, 1e-5)
    u = np.array([0.0, math.log(math.e - 1.0), -1e4, 50.0, -30.0])
    inp = dict(x=np.zeros((1, 5, 1)), z=np.zeros((1, 5, 1)), B=np.zeros((1, 5, 1)),
               C=np.zeros((1, 5, 1)), dt=(u - 0.25).reshape(1, 5, 1), A=[-1.0], D=[0.0],
               conv_w=identity_conv(d), conv_b=np.zeros(3), dt_bias=[0.25], norm_w=[1.0])
    delta = run(d, inp, stages=True)["delta"][0, :, 0]
    # softplus(0) = ln 2; softplus(ln(e-1)) = 1; e^-1e4 underflows: exactly 0;
    # softplus(50) = 50 + ln(1 + e^-50); softplus(-30) = ln(1 + e^-30) ~ e^-30.
    assert delta[0] == pytest.approx(math.log(2.0), rel=1e-15)
    assert delta[1] == pytest.approx(1.0, rel=1e-15)
    assert delta[2] == 0.0
    assert delta[3] == pytest.approx(50.0, rel=1e-15)
    assert delta[4] == pytest.approx(math.exp(-30.0), rel=1e-12)


def test_silu_closed_forms():
    d = Dims(1, 4, 1, 1, 1, 1, 4, 1e-5)
    v = np.array([0.0, math.log(3.0), -math.log(3.0), 40.0])
    inp = dict(x=v.reshape(1, 4, 1), z=np.zeros((1, 4, 1)), B=np.zeros((1, 4, 1)),
               C=np.zeros((1, 4, 1)), dt=np.zeros((1, 4, 1)), A=[-1.0], D=[0.0],
               conv_w=identity_conv(d), conv_b=np.zeros(3), dt_bias=[0.0], norm_w=[1.0])
    act = run(d, inp, stages=True)["xbc_act"][0, :, 0]
    # SiLU(v) = v * sigma(v): sigma(ln 3) = 3/4, sigma(-ln 3) = 1/4, sigma(40) = 1 - ~4e-18.
    assert act[0] == 0.0
    assert act[1] == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    assert act[2] == pytest.approx(-0.25 * math.log(3.0), rel=1e-15)
    assert act[3] == pytest.approx(40.0, rel=1e-15)


def test_conv_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "conv_hand_L4.json")))["cases"]
    for case in cases:
        L = len(case["u"])
        d = Dims(1, L, 1, 1, 1, 1, 4, 1e-5)
        w = np.zeros((3, 4))
        w[0] = case["w"]
        bvec = np.array([case["b"], 0.0, 0.0])
        init_conv = np.zeros((1, 3, 3))
        init_conv[0, 0] = case["state"]
        inp = dict(x=np.array(case["u"]).reshape(1, L, 1), z=np.zeros((1, L, 1)),
                   B=np.zeros((1, L, 1)), C=np.zeros((1, L, 1)), dt=np.zeros((1, L, 1)),
                   A=[-1.0], D=[0.0], conv_w=w, conv_b=bvec, dt_bias=[0.0], norm_w=[1.0],
                   init_conv=init_conv)
        out = run(d, inp, stages=True)
        v = np.array(case["v"])
        silu_v = v / (1.0 + np.exp(-v))
        np.testing.assert_allclose(out["xbc_act"][0, :, 0], silu_v, rtol=1e-15, err_msg=case["name"])
        np.testing.assert_array_equal(out["final_conv"][0, 0], case["final_state"])


# ---------------------------------------------------------------- the scan

def test_recurrence_closed_form_constant_inputs():
    """Constant delta, A, x', B', C': h_t = a^(t+1) h0 + delta x B^T (1 - a^(t+1)) / (1 - a),
    a = exp(delta A) (a geometric series), y_t = h_t C + D x."""
    L, P, N = 30, 3, 5
    d = Dims(1, L, 1, P, 1, N, 4, 1e-5)
    rng = np.random.default_rng(7)
    xv, Bv, Cv = rng.standard_normal(P), rng.standard_normal(N), rng.standard_normal(N)
    h0 = rng.standard_normal((P, N))
    Ah, Dh, dtv = -1.7, 0.6, 0.3
    inp = dict(x=np.tile(xv, (1, L, 1)), z=np.zeros((1, L, P)), B=np.tile(Bv, (1, L, 1)),
               C=np.tile(Cv, (1, L, 1)), dt=np.full((1, L, 1), dtv), A=[Ah], D=[Dh],
               conv_w=identity_conv(d), conv_b=np.zeros(P + 2 * N), dt_bias=[0.0],
               norm_w=np.ones(P), init_ssm=h0[None, None], init_conv=None)
    out = run(d, inp, stages=True)
    xa = out["xbc_act"][0, 0, :P]
    Ba = out["xbc_act"][0, 0, P:P + N]
    Ca = out["xbc_act"][0, 0, P + N:]
    delta = out["delta"][0, 0, 0]
    # identity taps with a zero initial conv state: token 0..L-1 all see v = u
    assert np.all(out["xbc_act"][0] == out["xbc_act"][0, :1])
    a = math.exp(delta * Ah)
    for t in [0, 1, 2, 17, L - 1]:
        geo = (1.0 - a ** (t + 1)) / (1.0 - a)
        ht = a ** (t + 1) * h0 + delta * np.outer(xa, Ba) * geo
        np.testing.assert_allclose(out["y_pre"][0, t], ht @ Ca + Dh * xa, rtol=1e-12, atol=1e-14)
    hL = a ** L * h0 + delta * np.outer(xa, Ba) * (1.0 - a ** L) / (1.0 - a)
    np.testing.assert_allclose(out["final_ssm"][0, 0], hL, rtol=1e-12, atol=1e-14)


def test_brute_force_by_hand_L3():
    """H = G = P = N = 1, L = 3, every step by hand with exp(delta A) = 1/2.
    x' = B' = C' are fixed by the identity conv; delta = ln 2 via dt + bias = 0 ...
    use A = -1 so a = exp(-ln 2) = 1/2. Raw x = [1, 2, 3] -> x' = SiLU(x)."""
    d = Dims(1, 3, 1, 1, 1, 1, 4, 1e-5)
    u = np.array([1.0, 2.0, 3.0])
    bu = np.array([0.5, -1.0, 2.0])
    cu = np.array([1.5, 0.25, -0.5])
    inp = dict(x=u.reshape(1, 3, 1), z=np.zeros((1, 3, 1)), B=bu.reshape(1, 3, 1),
               C=cu.reshape(1, 3, 1), dt=np.zeros((1, 3, 1)), A=[-1.0], D=[0.25],
               conv_w=identity_conv(d), conv_b=np.zeros(3), dt_bias=[0.0], norm_w=[1.0],
               init_ssm=np.full((1, 1, 1, 1), 2.0))
    out = run(d, inp, stages=True)
    s = lambda v: v / (1.0 + math.exp(-v))
    xs, bs, cs = [s(v) for v in u], [s(v) for v in bu], [s(v) for v in cu]
    dl = math.log(2.0)
    h = 2.0
    ys = []
    h = 0.5 * h + dl * xs[0] * bs[0]; ys.append(h * cs[0] + 0.25 * xs[0])
    h = 0.5 * h + dl * xs[1] * bs[1]; ys.append(h * cs[1] + 0.25 * xs[1])
    h = 0.5 * h + dl * xs[2] * bs[2]; ys.append(h * cs[2] + 0.25 * xs[2])
    np.testing.assert_allclose(out["y_pre"][0, :, 0], ys, rtol=1e-14)
    assert out["final_ssm"][0, 0, 0, 0] == pytest.approx(h, rel=1e-14)


@pytest.mark.parametrize("Q", [1, 3, 8, 16, 64, 256])
def test_sequential_matches_chunked_form(Q):
    rng = np.random.default_rng(100 + Q)
    d, inp = rand_problem(rng, b=2, L=157, H=4, P=8, G=2, N=16)
    out = run(d, inp, stages=True)
    for bi in range(d.batch):
        xa, Ba, Ca, dl = scan_inputs(d, out, bi)
        y, Hf = chunked_scan(xa, Ba, Ca, dl, inp["A"], inp["D"], inp["init_ssm"][bi], Q)
        yo = out["y_pre"][bi].reshape(d.seqlen, d.nheads, d.headdim)
        assert rel(yo, y) <= 1e-10
        assert rel(out["final_ssm"][bi], Hf) <= 1e-10
        # the positions where each chunk after the first begins (where a pure-torch
        # fallback is reported to err) must agree just as well
        ks = np.arange(Q, d.seqlen, Q)
        if len(ks):
            assert rel(yo[ks], y[ks]) <= 1e-10


def test_sequential_matches_quadratic_form():
    rng = np.random.default_rng(5)
    d, inp = rand_problem(rng, b=2, L=19, H=4, P=3, G=2, N=5)
    out = run(d, inp, stages=True)
    for bi in range(d.batch):
        xa, Ba, Ca, dl = scan_inputs(d, out, bi)
        y, Hf = quadratic_scan(xa, Ba, Ca, dl, inp["A"], inp["D"], inp["init_ssm"][bi])
        assert rel(out["y_pre"][bi].reshape(d.seqlen, d.nheads, d.headdim), y) <= 1e-10
        assert rel(out["final_ssm"][bi], Hf) <= 1e-10


def test_quadratic_and_chunked_forms_catch_swapped_B_C():
    """A transposed operand (B and C exchanged) must not go unnoticed by the pins."""
    rng = np.random.default_rng(9)
    d, inp = rand_problem(rng, b=1, L=12, H=2, P=2, G=1, N=3)
    out = run(d, inp, stages=True)
    xa, Ba, Ca, dl = scan_inputs(d, out, 0)
    y_ok, _ = quadratic_scan(xa, Ba, Ca, dl, inp["A"], inp["D"], inp["init_ssm"][0])
    y_sw, _ = quadratic_scan(xa, Ca, Ba, dl, inp["A"], inp["D"], inp["init_ssm"][0])
    assert rel(y_sw, y_ok) > 1e-3


def test_zero_step_leaves_state_and_gives_readout():
    """delta = 0 (dt + bias = -1e4 underflows to exactly 0): the state is unchanged bit for
    bit and y' = C' . h0 + D x'."""
    rng = np.random.default_rng(11)
    d, inp = rand_problem(rng, b=2, L=33, H=4, P=4, G=2, N=8)
    inp["dt"] = np.full_like(inp["dt"], -1e4)
    out = run(d, inp, stages=True)
    assert np.all(out["delta"] == 0.0)
    np.testing.assert_array_equal(out["final_ssm"], inp["init_ssm"])
    for bi in range(d.batch):
        xa, Ba, Ca, _ = scan_inputs(d, out, bi)
        r = d.nheads // d.ngroups
        for h in range(d.nheads):
            expect = Ca[:, h // r, :] @ inp["init_ssm"][bi, h].T + inp["D"][h] * xa[:, h, :]
            got = out["y_pre"][bi].reshape(d.seqlen, d.nheads, d.headdim)[:, h]
            np.testing.assert_allclose(got, expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("L1", [1, 2, 3, 5, 64, 100])
def test_split_and_chain_equals_one_call(L1):
    rng = np.random.default_rng(200 + L1)
    d, inp = rand_problem(rng, b=2, L=130, H=4, P=4, G=2, N=8)
    full = run(d, inp)
    d1 = Dims(d.batch, L1, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    d2 = Dims(d.batch, d.seqlen - L1, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    seq = ("x", "z", "B", "C", "dt")
    p1 = {k: (v[:, :L1] if k in seq else v) for k, v in inp.items()}
    o1 = run(d1, p1)
    p2 = {k: (v[:, L1:] if k in seq else v) for k, v in inp.items()}
    p2["init_ssm"], p2["init_conv"] = o1["final_ssm"], o1["final_conv"]
    o2 = run(d2, p2)
    y = np.concatenate([o1["y"], o2["y"]], axis=1)
    assert rel(y, full["y"]) <= 1e-12
    assert rel(o2["final_ssm"], full["final_ssm"]) <= 1e-12
    np.testing.assert_array_equal(o2["final_conv"], full["final_conv"])


def test_causality():
    rng = np.random.default_rng(13)
    d, inp = rand_problem(rng, b=1, L=80, H=4, P=4, G=2, N=8)
    base = run(d, inp)
    tstar = 37
    pert = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
    for k in ("x", "z", "B", "C", "dt"):
        pert[k][:, tstar:] += rng.standard_normal(pert[k][:, tstar:].shape)
    out = run(d, pert)
    np.testing.assert_array_equal(out["y"][:, :tstar], base["y"][:, :tstar])
    assert np.max(np.abs(out["y"][:, tstar:] - base["y"][:, tstar:])) > 1e-3


# ---------------------------------------------------------------- gated norm, groups

def test_gated_norm_single_channel_groups():
    """Norm group of one channel: out = g * w / sqrt(g^2 + eps), g = y' * SiLU(z)."""
    rng = np.random.default_rng(17)
    d, inp = rand_problem(rng, b=1, L=10, H=2, P=1, G=2, N=4)
    out = run(d, inp, stages=True)
    z = inp["z"][0]
    g = out["y_pre"][0] * z / (1.0 + np.exp(-z))
    expect = g * inp["norm_w"][None, :] / np.sqrt(g * g + d.eps)
    np.testing.assert_allclose(out["y"][0], expect, rtol=1e-13)


def test_gated_norm_two_channel_group_by_hand():
    """Group of two channels whose gates are 3 and 4 (built from y' and z directly):
    mean of squares = 12.5, out = (3, 4) / sqrt(12.5 + eps) * w."""
    rng = np.random.default_rng(19)
    d, inp = rand_problem(rng, b=1, L=4, H=1, P=2, G=1, N=2, init=False)
    out = run(d, inp, stages=True)
    # choose z so that the gate y' * SiLU(z) equals (+-3, +-4) at token 0: take the sign
    # that makes SiLU(z) = gate / y' positive, then solve for z by bisection (SiLU is
    # increasing for z > 0 and SiLU(z) -> z)
    yp = out["y_pre"][0, 0]
    targets = np.array([3.0, 4.0]) * np.sign(yp)
    zsol = []
    for c in range(2):
        want = targets[c] / yp[c]
        lo, hi = 0.0, 2.0 * want + 10.0
        for _ in range(300):
            mid = 0.5 * (lo + hi)
            if mid / (1.0 + math.exp(-mid)) < want:
                lo = mid
            else:
                hi = mid
        zsol.append(0.5 * (lo + hi))
    inp["z"][0, 0] = zsol
    out = run(d, inp, stages=True)
    expect = targets / math.sqrt(12.5 + d.eps) * inp["norm_w"]
    np.testing.assert_allclose(out["y"][0, 0], expect, rtol=1e-9)


def test_constant_gate_gives_sign_times_weight():
    """Every channel of a group with the same gate c: out = c / sqrt(c^2 + eps) * w."""
    d = Dims(1, 2, 2, 2, 1, 1, 4, 1e-5)
    inp = dict(x=np.full((1, 2, 4), 0.7), z=np.full((1, 2, 4), 30.0), B=np.zeros((1, 2, 1)),
               C=np.zeros((1, 2, 1)), dt=np.zeros((1, 2, 2)), A=[-1.0, -2.0], D=[0.5, 0.5],
               conv_w=identity_conv(Dims(1, 2, 2, 2, 1, 1)), conv_b=np.zeros(6),
               dt_bias=[0.0, 0.0], norm_w=np.array([1.0, -2.0, 0.5, 3.0]))
    out = run(d, inp, stages=True)
    c = out["y_pre"][0, 0, 0] * 30.0 / (1.0 + math.exp(-30.0))
    np.testing.assert_allclose(out["y"][0, 0], c / math.sqrt(c * c + 1e-5) * inp["norm_w"], rtol=1e-13)


def test_head_to_group_map_is_contiguous():
    """Reading: head h reads B and C of group h // (H/G). With group 1's B at zero and a
    zero initial state, heads 2 and 3 (group 1) carry no state: y' = D x'."""
    rng = np.random.default_rng(23)
    d, inp = rand_problem(rng, b=1, L=20, H=4, P=2, G=2, N=3, init=False)
    inp["B"][:, :, 3:] = 0.0
    inp["conv_b"][d.d_inner + 3:d.d_inner + 6] = 0.0
    out = run(d, inp, stages=True)
    yp = out["y_pre"][0].reshape(20, 4, 2)
    xa = out["xbc_act"][0, :, :8].reshape(20, 4, 2)
    for h in (2, 3):
        np.testing.assert_allclose(yp[:, h], inp["D"][h] * xa[:, h], rtol=1e-14)
    for h in (0, 1):
        assert np.max(np.abs(yp[:, h] - inp["D"][h] * xa[:, h])) > 1e-3


def test_separable_by_group():
    """The full problem equals its per-group sub-problems (used for sampled checks at
    full size)."""
    rng = np.random.default_rng(29)
    d, inp = rand_problem(rng, b=2, L=21, H=6, P=2, G=3, N=4)
    full = run(d, inp)
    for g in range(d.ngroups):
        sd, sub, xs, hs, cidx = oracle.group_subproblem(d, g, inp)
        o = run(sd, sub)
        np.testing.assert_array_equal(o["y"], full["y"][:, :, xs])
        np.testing.assert_array_equal(o["final_ssm"], full["final_ssm"][:, hs])
        np.testing.assert_array_equal(o["final_conv"], full["final_conv"][:, cidx])


# ---------------------------------------------------------------- decode

def test_prefill_equals_prefill_then_decode_steps():
    rng = np.random.default_rng(31)
    d, inp = rand_problem(rng, b=3, L=25, H=4, P=4, G=2, N=8)
    full = run(d, inp)
    L0 = 20
    d0 = Dims(d.batch, L0, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    seq = ("x", "z", "B", "C", "dt")
    o = run(d0, {k: (v[:, :L0] if k in seq else v) for k, v in inp.items()})
    # slots in a permuted order: sequence i lives in slot perm[i]
    perm = np.array([2, 0, 1])
    ssm = np.zeros((3,) + o["final_ssm"].shape[1:])
    conv = np.zeros((3,) + o["final_conv"].shape[1:])
    ssm[perm], conv[perm] = o["final_ssm"], o["final_conv"]
    for t in range(L0, d.seqlen):
        y, ssm, conv = oracle.decode_step(
            d, inp["x"][:, t], inp["z"][:, t], inp["B"][:, t], inp["C"][:, t], inp["dt"][:, t],
            inp["A"], inp["D"], inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"],
            ssm, conv, slot_idx=perm)
        assert rel(y, full["y"][:, t]) <= 1e-12
    assert rel(ssm[perm], full["final_ssm"]) <= 1e-12
    np.testing.assert_array_equal(conv[perm], full["final_conv"])


def test_varlen_equal_lengths_equals_batched_prefill():
    """Packed sequences of one length on identity slots, all continuing from their slots,
    are the batched prefill row by row (bit for bit: the same per-row computation)."""
    rng = np.random.default_rng(41)
    d, inp = rand_problem(rng, b=3, L=17)
    ref = oracle.prefill_dict(d, inp)
    T = d.batch * d.seqlen
    pk = {k: inp[k].reshape(T, -1) for k in ("x", "z", "B", "C", "dt")}
    cu = np.arange(0, T + 1, d.seqlen)
    y, ssm, conv = oracle.prefill_varlen(d, cu, pk["x"], pk["z"], pk["B"], pk["C"], pk["dt"], inp["A"], inp["D"],
                                         inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"],
                                         inp["init_ssm"], inp["init_conv"])
    assert np.array_equal(y, ref["y"].reshape(T, -1))
    assert np.array_equal(ssm, ref["final_ssm"]) and np.array_equal(conv, ref["final_conv"])


def test_varlen_slots_fresh_starts_and_empty_sequences():
    """Slot mapping: a sequence with has_init = 0 equals a prefill from zero states; an empty
    sequence leaves its slot's states as they were; untouched slots are unchanged."""
    rng = np.random.default_rng(42)
    d, inp = rand_problem(rng, b=1, L=30, init=False)
    H, P, N, Cc = d.nheads, d.headdim, d.dstate, d.xbc_channels
    nslots = 5
    ssm0 = 0.1 * rng.standard_normal((nslots, H, P, N))
    conv0 = rng.standard_normal((nslots, Cc, 3))
    lens = [12, 0, 18]
    cu = np.concatenate([[0], np.cumsum(lens)])
    pk = {k: inp[k][0] for k in ("x", "z", "B", "C", "dt")}
    slots, has_init = [3, 1, 0], [0, 1, 1]
    y, ssm, conv = oracle.prefill_varlen(d, cu, pk["x"], pk["z"], pk["B"], pk["C"], pk["dt"], inp["A"], inp["D"],
                                         inp["conv_w"], inp["conv_b"], inp["dt_bias"], inp["norm_w"],
                                         ssm0, conv0, slot_idx=slots, has_init=has_init)
    par = {k: inp[k] for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
    fresh = oracle.prefill(Dims(1, 12, H, P, d.ngroups, N, 4, d.eps), *(inp[k][:, :12] for k in ("x", "z", "B", "C", "dt")),
                           *par.values())
    assert np.array_equal(y[:12], fresh["y"][0]) and np.array_equal(ssm[3], fresh["final_ssm"][0])
    cont = oracle.prefill(Dims(1, 18, H, P, d.ngroups, N, 4, d.eps), *(inp[k][:, 12:30] for k in ("x", "z", "B", "C", "dt")),
                          *par.values(), ssm0[0][None], conv0[0][None])
    assert np.array_equal(y[12:30], cont["y"][0]) and np.array_equal(conv[0], cont["final_conv"][0])
    for k in (1, 2, 4):     # the empty sequence's slot and the untouched slots
        assert np.array_equal(ssm[k], ssm0[k]) and np.array_equal(conv[k], conv0[k])


def test_final_state_is_linear_in_the_initial_state_with_the_decay_factor():
    """final(H0) = decay * H0 + final(0) for one piece (the recurrence is linear in the state,
    and the product of its per-token factors exp(delta_t A) is the decay); the basis of
    passing the state between the pieces of a split sequence."""
    rng = np.random.default_rng(43)
    d, inp = rand_problem(rng, b=2, L=37, init=True)
    with_init = oracle.prefill_dict(d, inp)
    zero = oracle.prefill_dict(d, dict(inp, init_ssm=None))
    a = oracle.decay(inp["dt"], inp["A"], inp["dt_bias"])
    pred = a[:, :, None, None] * inp["init_ssm"] + zero["final_ssm"]
    assert np.max(np.abs(pred - with_init["final_ssm"])) <= 1e-12 * np.max(np.abs(with_init["final_ssm"]))
    # and pieces chain: two pieces folded equal one prefill over both
    d1 = Dims(d.batch, 20, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    d2 = Dims(d.batch, 17, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
    cut = lambda v, s: v[:, s] if v is not None and v.ndim == 3 and v.shape[1] == d.seqlen else v
    p1 = {k: cut(v, slice(0, 20)) for k, v in inp.items()}
    p2 = {k: cut(v, slice(20, 37)) for k, v in inp.items()}
    r1 = oracle.prefill_dict(d1, p1)
    r2z = oracle.prefill_dict(d2, dict(p2, init_ssm=None, init_conv=r1["final_conv"]))
    a2 = oracle.decay(p2["dt"], inp["A"], inp["dt_bias"])
    chained = a2[:, :, None, None] * r1["final_ssm"] + r2z["final_ssm"]
    assert np.max(np.abs(chained - with_init["final_ssm"])) <= 1e-12 * np.max(np.abs(with_init["final_ssm"]))


def test_decay_equals_the_product_of_the_compiled_oracles_step_factors():
    """oracle.decay against exp(A * sum_t delta_t) with delta taken from the compiled C oracle's
    stage output (its own softplus), on steps whose argument dt + dt_bias spans (-40, 40): the
    large arguments (15 .. 40) are where a shortcut of softplus(u) ~ u would differ from the
    exact value log(1 + e^u). Small A keeps the product representable at those step sizes."""
    rng = np.random.default_rng(47)
    d, inp = rand_problem(rng, b=2, L=24, H=4, P=4, G=2, N=8, init=False)
    u = np.linspace(-40.0, 40.0, d.batch * d.seqlen * d.nheads).reshape(d.batch, d.seqlen, d.nheads)
    u[:, :6] = rng.uniform(15.0, 40.0, (d.batch, 6, d.nheads))
    inp["dt"] = u - inp["dt_bias"]
    inp["A"] = -np.array([1e-3, 2e-3, 5e-4, 1e-3])
    out = oracle.prefill_dict(d, inp, stages=True)
    want = np.exp(inp["A"][None, :] * out["delta"].sum(axis=1))
    got = oracle.decay(inp["dt"], inp["A"], inp["dt_bias"])
    assert rel(got, want) <= 1e-13
    # and the steps in (20, 30), where e^-u is still above half an fp64 ulp of u, carry the
    # correction log1p(e^-u) that a cutoff at 20 would drop
    big = (u > 20.0) & (u < 30.0)
    assert big.any() and np.all(out["delta"][big] > u[big])
    assert np.all(np.abs(got - want) <= 1e-13 * np.abs(want))
