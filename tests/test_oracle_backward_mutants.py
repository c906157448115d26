"""Mutation tests of the backward oracle (CPU only): each mutant is oracle/backward.py with
one plausible mistake (a dropped term, a wrong index or state, a wrong derivative), loaded
as a module of its own; the finite-difference pin must reject every one."""
import importlib.util
import os

import numpy as np
import pytest

from tests.test_oracle_backward import check_all_gradients, cotangents
from tests.test_oracle_pins import rand_problem

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "backward.py")

MUTANTS = {
    "SiLU derivative without its second term": ("return sg * (1.0 + u * (1.0 - sg))", "return sg"),
    "norm scale treated as a constant": ("- (r ** 3 / gs)[..., None] * g * dot[..., None]", ""),
    "norm weight missing from the gate gradient": ("wd = (dout * norm_w)", "wd = (dout * 1.0)"),
    "state gradient not decayed": ("Gt = a[:, :, None, None] * Gt", "Gt = Gt"),
    "delta gradient without the decay term": ("ddelta[:, t] = A * a * gh + gxb", "ddelta[:, t] = gxb"),
    "C' gradient from the previous state": ('np.einsum("bhpn,bhp->bhn", Hs[:, t + 1], dy[:, t])',
                                             'np.einsum("bhpn,bhp->bhn", Hs[:, t], dy[:, t])'),
    "D skip missing from the x' gradient": ("+ D[None, :, None] * dy[:, t]", ""),
    "dA without delta": ("dA += np.sum(delta[:, t] * a * gh, axis=0)", "dA += np.sum(a * gh, axis=0)"),
    "B' gradient of the first head only": ("dBs = dBh.reshape(b, L, G, r, N).sum(axis=3)",
                                           "dBs = dBh.reshape(b, L, G, r, N)[:, :, :, 0]"),
    "softplus derivative taken as exp": ("ddt = ddelta * sigmoid(", "ddt = ddelta * np.exp("),
    "taps reversed in the conv gradient": ("ds[:, k:k + L] += conv_w[:, k] * dv",
                                           "ds[:, k:k + L] += conv_w[:, K - 1 - k] * dv"),
    "final conv state gradient dropped": ("ds[:, L:L + K - 1] += _f64(dfinal_conv).transpose(0, 2, 1)", "pass"),
    "conv weight gradient against the wrong window": ("np.sum(dv * s[:, k:k + L], axis=(0, 1))",
                                                      "np.sum(dv * s[:, k + 1:k + 1 + L] if k < K - 1 else dv * s[:, k:k + L], axis=(0, 1))"),
}


def load_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    path = tmp_path / "backward_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("backward_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    mod = load_mutant(name, tmp_path)
    rng = np.random.default_rng(7)
    d, inp = rand_problem(rng, b=2, L=11, H=4, P=3, G=2, N=5, init=True)
    dout, dfs, dfc = cotangents(rng, d, True)
    with pytest.raises(AssertionError):
        check_all_gradients(d, inp, dout, dfs, dfc, rng, vjp=mod.prefill_vjp)


FORMS = os.path.join(os.path.dirname(SRC), "forms.py")

CHUNKED_MUTANTS = {
    "decay-gradient column sums dropped": ("T.sum(axis=1) - T.sum(axis=0)", "T.sum(axis=1)"),
    "state gradient not decayed across chunks": ("Gs[h] = e_end * Gc +", "Gs[h] = Gc +"),
    "B' gradient without the chunk-state term": ("dK.T @ Cc + e_rest[:, None] * (u @ Gc)", "dK.T @ Cc"),
}


@pytest.mark.parametrize("name", sorted(CHUNKED_MUTANTS))
def test_chunked_backward_mutant_is_caught(name, tmp_path, monkeypatch):
    import oracle.forms as forms
    from tests import test_oracle_backward as tob
    old, new = CHUNKED_MUTANTS[name]
    src = open(FORMS).read()
    assert src.count(old) == 1, f"mutation site not unique: {old!r}"
    path = tmp_path / "forms_mutant.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("forms_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(forms, "chunked_scan_vjp", mod.chunked_scan_vjp)
    with pytest.raises(AssertionError):
        tob.test_chunked_backward_form_matches_the_sequential_one(8)
