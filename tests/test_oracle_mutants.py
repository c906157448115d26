"""The oracle's pins must catch plausible mistakes (CPU only).

Each case compiles a copy of oracle/ssd_oracle.c with one planted mistake (a dropped
term, a wrong sign or index, a transposed operand) into a temporary directory and runs
the pin tests against it: at least one pin must fail. Nothing here touches a GPU.
"""
import os

import numpy as np
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

MUTANTS = {
    "dropped D skip": ("yp[t * gw + (int64_t)i * P + p] = yv + Dh * xt[p];",
                       "yp[t * gw + (int64_t)i * P + p] = yv;"),
    "A sign flipped": ("const double decay = exp(dlt * Ah);", "const double decay = exp(-dlt * Ah);"),
    "B and C exchanged": ("hp[n] = decay * hp[n] + dlt * xt[p] * Bt[n];\n                    yv += hp[n] * Ct[n];",
                          "hp[n] = decay * hp[n] + dlt * xt[p] * Ct[n];\n                    yv += hp[n] * Bt[n];"),
    "readout before update": ("hp[n] = decay * hp[n] + dlt * xt[p] * Bt[n];\n                    yv += hp[n] * Ct[n];",
                              "yv += hp[n] * Ct[n];\n                    hp[n] = decay * hp[n] + dlt * xt[p] * Bt[n];"),
    "input not scaled by delta": ("dlt * xt[p] * Bt[n]", "xt[p] * Bt[n]"),
    "conv taps reversed": ("v += w[k] * s[t + k];", "v += w[K - 1 - k] * s[t + k];"),
    "conv bias dropped": ("double v = bias;", "double v = 0.0;"),
    "final conv state off by one": ("fin[k] = s[L + k];", "fin[k] = s[L + k - 1];"),
    "gate without SiLU": ("yp[t * gw + c] * silu(zt[c]);", "yp[t * gw + c] * zt[c];"),
    "norm by sum, not mean": ("sqrt(ss / (double)gw + d->eps)", "sqrt(ss + d->eps)"),
    "norm weight dropped": ("yt[c] = yt[c] * inv * j->norm_w[xc0 + c];", "yt[c] = yt[c] * inv;"),
    "softplus without log1p": ("log1p(exp(-fabs(u)))", "exp(-fabs(u))"),
    "dt bias dropped": ("softplus(j->dt[(b * L + t) * H + h] + j->dt_bias[h])",
                        "softplus(j->dt[(b * L + t) * H + h])"),
    "heads strided over groups": ("const int h = g * r + i;\n            dl[t * r + i]",
                                  "const int h = i * G + g;\n            dl[t * r + i]"),
    "initial state ignored": ("if (j->init_ssm) memcpy(hs", "if (0) memcpy(hs"),
}

PINS = [
    pins.test_softplus_closed_forms, pins.test_silu_closed_forms, pins.test_conv_hand_cases,
    pins.test_recurrence_closed_form_constant_inputs, pins.test_brute_force_by_hand_L3,
    lambda: pins.test_sequential_matches_chunked_form(8),
    pins.test_sequential_matches_quadratic_form, pins.test_zero_step_leaves_state_and_gives_readout,
    lambda: pins.test_split_and_chain_equals_one_call(2), pins.test_causality,
    pins.test_gated_norm_single_channel_groups, pins.test_gated_norm_two_channel_group_by_hand,
    pins.test_constant_gate_gives_sign_times_weight, pins.test_head_to_group_map_is_contiguous,
    pins.test_prefill_equals_prefill_then_decode_steps,
]


def test_unmutated_source_passes_every_pin():
    for pin in PINS:
        pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {name}"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(mutated),
                    "-lm", "-lpthread"], check=True)
    failures = 0
    with oracle.use_library(str(so)):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError, FloatingPointError, RuntimeError):
                failures += 1
    assert failures >= 1, f"no pin caught the planted mistake: {name}"


# The Python compositions of the oracle (decay, packed sequences on slots): plausible mistakes
# planted by swapping the function, each of which a pin must catch.

def _decay_without_bias(dt, A, dt_bias):
    u = np.asarray(dt, np.float64)
    return np.exp(np.asarray(A, np.float64) * np.log1p(np.exp(u)).sum(axis=1))


def _decay_sign_flipped(dt, A, dt_bias):
    return 1.0 / _real_decay(dt, A, dt_bias)


def _decay_last_token_only(dt, A, dt_bias):
    u = np.asarray(dt, np.float64) + np.asarray(dt_bias, np.float64)
    return np.exp(np.asarray(A, np.float64) * np.log1p(np.exp(u[:, -1])))


def _decay_softplus_cutoff(dt, A, dt_bias):
    # softplus(u) replaced by u above 20, a shortcut that drops log1p(e^-u)
    u = np.asarray(dt, np.float64) + np.asarray(dt_bias, np.float64)
    delta = np.where(u > 20.0, u, np.log1p(np.exp(np.minimum(u, 20.0))))
    return np.exp(np.asarray(A, np.float64) * delta.sum(axis=1))


_real_decay = oracle.decay


@pytest.mark.parametrize("mutant", [_decay_without_bias, _decay_sign_flipped, _decay_last_token_only,
                                    _decay_softplus_cutoff])
def test_decay_mutant_is_caught(mutant, monkeypatch):
    monkeypatch.setattr(oracle, "decay", mutant)
    caught = 0
    for pin in (pins.test_final_state_is_linear_in_the_initial_state_with_the_decay_factor,
                pins.test_decay_equals_the_product_of_the_compiled_oracles_step_factors):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, "no pin caught the planted mistake in decay()"


def _varlen_slots_ignored(d, cu, *args, slot_idx=None, has_init=None, **kw):
    return _real_varlen(d, cu, *args, slot_idx=None, has_init=has_init, **kw)


def _varlen_always_continues(d, cu, *args, slot_idx=None, has_init=None, **kw):
    return _real_varlen(d, cu, *args, slot_idx=slot_idx, has_init=None, **kw)


_real_varlen = oracle.prefill_varlen


@pytest.mark.parametrize("mutant", [_varlen_slots_ignored, _varlen_always_continues])
def test_varlen_mutant_is_caught(mutant, monkeypatch):
    monkeypatch.setattr(oracle, "prefill_varlen", mutant)
    with pytest.raises(AssertionError):
        pins.test_varlen_slots_fresh_starts_and_empty_sequences()
