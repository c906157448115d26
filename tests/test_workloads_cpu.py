"""The input recipe (hybrid_mamba_ssm_causal_b200/workloads.py) on CPU: the bf16 rounding is
round-to-nearest-even, as torch converts float32 to bfloat16; draws are deterministic per
seed; shapes and value ranges follow the recipe; bf16 workloads carry bf16 values only."""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_decode_inputs, make_prefill_inputs, round_bf16


def torch_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_round_bf16_is_round_to_nearest_even():
    rng = np.random.default_rng(5)
    mant = rng.uniform(1.0, 2.0, 200000) * rng.choice([-1.0, 1.0], 200000)
    vals = (mant * np.exp2(rng.integers(-126, 120, 200000))).astype(np.float32)
    # exact halfway cases: the 16 dropped bits are 0x8000, with the kept last bit even or odd
    hi = rng.integers(0x0080, 0x7F00, 4000, dtype=np.uint32) << 16
    ties = (hi | np.uint32(0x8000)).view(np.float32)
    special = np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, 1e-40, -1e-40, 3.0e38], dtype=np.float32)
    for a in (vals, ties, special):
        assert np.array_equal(round_bf16(a).view(np.uint32), torch_bf16(a).view(np.uint32))
    nans = np.array([0x7FC00000, 0x7F800001, 0xFF800001], dtype=np.uint32).view(np.float32)
    assert np.isnan(round_bf16(nans)).all()


def test_round_bf16_is_idempotent_and_nearest():
    rng = np.random.default_rng(6)
    a = rng.standard_normal(10000).astype(np.float32)
    r = round_bf16(a)
    assert np.array_equal(round_bf16(r), r)
    # within half a bf16 ulp (2^-8 relative) of the input
    assert np.all(np.abs(r - a) <= np.abs(a) * 2.0 ** -8)


@pytest.mark.parametrize("name", ["tiny_f32", "small_bf16", "mid_bf16", "long_bf16"])
def test_prefill_inputs_follow_the_recipe(name):
    w = WORKLOADS[name].with_(batch=2, seqlen=40)
    a, b = make_prefill_inputs(w), make_prefill_inputs(w)
    for k in a:
        assert (a[k] is None and b[k] is None) or np.array_equal(a[k], b[k]), k
    T, HP, GN, H, Cc = w.total_seqlen, w.d_inner, w.ngroups * w.dstate, w.nheads, w.xbc_channels
    shapes = {"x": (2, T, HP), "z": (2, T, HP), "B": (2, T, GN), "C": (2, T, GN), "dt": (2, T, H), "A": (H,),
              "D": (H,), "dt_bias": (H,), "conv_w": (Cc, 4), "conv_b": (Cc,), "norm_w": (HP,)}
    for k, s in shapes.items():
        assert a[k].shape == s and a[k].dtype == np.float32, k
    assert np.all(a["A"] <= -1.0) and np.all(a["A"] >= -16.0)
    assert np.all(a["D"] >= 0.0) and np.all(a["D"] <= 1.0)
    sp = np.log1p(np.exp(a["dt_bias"].astype(np.float64)))
    assert np.all(sp >= 1e-3 * (1 - 1e-5)) and np.all(sp <= 1e-1 * (1 + 1e-5))
    assert np.all(np.abs(a["conv_w"]) <= 0.5) and np.all(np.abs(a["conv_b"]) <= 0.1 * (1 + 2.0 ** -8))
    assert (a["init_ssm"] is None) == (w.init_ssm_std == 0.0)
    assert (a["init_conv"] is None) == (w.init_conv_std == 0.0)
    if w.act == "bf16":   # every activation, conv and norm weight is a bf16 value
        for k in ("x", "z", "B", "C", "dt", "conv_w", "conv_b", "norm_w", "init_conv"):
            if a[k] is not None:
                assert np.array_equal(round_bf16(a[k]), a[k]), k
    c = make_prefill_inputs(w, seed=w.seed + 100)
    assert not np.array_equal(c["x"], a["x"])


def test_decode_inputs_follow_the_recipe():
    w = WORKLOADS["decode_bf16"].with_(batch=3)
    a = make_decode_inputs(w, steps=5)
    assert a["x"].shape == (5, 3, w.d_inner) and a["dt"].shape == (5, 3, w.nheads)
    assert a["init_ssm"].shape == (3, w.nheads, w.headdim, w.dstate)
    assert a["init_conv"].shape == (3, w.xbc_channels, 3)
    assert np.array_equal(round_bf16(a["init_conv"]), a["init_conv"])
    assert np.array_equal(make_decode_inputs(w, steps=5)["x"], a["x"])
