"""Pins of the whole-layer oracle (oracle/layer.py: in_proj, the mixer core, out_proj) on
CPU: identity projections reduce it to the core oracle exactly (which pins the
[z | x | B | C | dt] split of the in_proj output), and the output is linear in out_proj."""
import numpy as np
import pytest

import oracle
from oracle.layer import layer_prefill, split_in_proj
from tests.test_oracle_pins import rand_problem

PAR = ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")


def test_identity_projections_reduce_to_the_core():
    rng = np.random.default_rng(71)
    d, inp = rand_problem(rng, b=2, L=19, H=4, P=3, G=2, N=5)
    u = np.concatenate([inp["z"], inp["x"], inp["B"], inp["C"], inp["dt"]], axis=2)
    W_in = np.eye(u.shape[2])
    W_out = np.eye(d.nheads * d.headdim)
    out, fs, fc = layer_prefill(d, u, W_in, W_out, *(inp[k] for k in PAR), inp["init_ssm"], inp["init_conv"])
    ref = oracle.prefill_dict(d, inp)
    assert np.array_equal(out, ref["y"])
    assert np.array_equal(fs, ref["final_ssm"]) and np.array_equal(fc, ref["final_conv"])


def test_split_order_is_z_x_B_C_dt():
    d = oracle.Dims(1, 2, 2, 3, 1, 4)
    width = 2 * 6 + 2 * 4 + 2
    row = np.arange(width, dtype=np.float64)[None, None, :].repeat(2, axis=1)
    z, x, B, C, dt = split_in_proj(d, row)
    assert [a[0, 0, 0] for a in (z, x, B, C, dt)] == [0, 6, 12, 16, 20]
    assert [a.shape[-1] for a in (z, x, B, C, dt)] == [6, 6, 4, 4, 2]
    with pytest.raises(ValueError):
        split_in_proj(d, row[..., :-1])


def test_output_is_linear_in_out_proj():
    rng = np.random.default_rng(72)
    d, inp = rand_problem(rng, b=1, L=11, H=2, P=4, G=1, N=3)
    d_model = 7
    width = 2 * d.nheads * d.headdim + 2 * d.ngroups * d.dstate + d.nheads
    u = rng.standard_normal((1, 11, d_model))
    W_in = rng.standard_normal((d_model, width)) / np.sqrt(d_model)
    W1, W2 = rng.standard_normal((2, d.nheads * d.headdim, d_model))
    par = [inp[k] for k in PAR]
    o1, _, _ = layer_prefill(d, u, W_in, W1, *par)
    o2, _, _ = layer_prefill(d, u, W_in, W2, *par)
    o12, _, _ = layer_prefill(d, u, W_in, W1 + W2, *par)
    assert np.max(np.abs(o12 - (o1 + o2))) <= 1e-12 * np.max(np.abs(o12))
