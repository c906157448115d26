"""GPU parity of ssd_mixer_decode_step against the fp64 oracle (needs a B200).

A run of decode steps equals one prefill of the same tokens, so the oracle checks many
steps of a few sequences as one fp64 prefill; the full decode batch is checked step by
step for the first steps.
"""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_decode_inputs
from tests.gpu_util import TOL, assert_close, to_dev

pytestmark = pytest.mark.gpu


def ddims(w, batch=None):
    return sm.Dims(batch or w.batch, 1, w.nheads, w.headdim, w.ngroups, w.dstate, 1, w.dconv, w.eps, w.act)


def odims(w, batch, L):
    return oracle.Dims(batch, L, w.nheads, w.headdim, w.ngroups, w.dstate, w.dconv, w.eps)


def run_steps(w, inp, steps, batch, slot_idx=None, nslots=None):
    """Decode ``steps`` tokens; returns (y [steps, b, HP], ssm_state, conv_state)."""
    adt = torch.bfloat16 if w.act == "bf16" else torch.float32
    dv = to_dev({k: inp[k] for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}, w.act)
    nslots = nslots or batch
    ssm = torch.zeros(nslots, w.nheads, w.headdim, w.dstate, device="cuda")
    conv = torch.zeros(nslots, w.xbc_channels, 3, dtype=adt, device="cuda")
    slots = torch.arange(batch) if slot_idx is None else torch.as_tensor(slot_idx)
    ssm[slots] = torch.from_numpy(inp["init_ssm"][:batch]).cuda()
    conv[slots] = torch.from_numpy(inp["init_conv"][:batch]).to(adt).cuda()
    sidx = None if slot_idx is None else torch.as_tensor(slot_idx, dtype=torch.int32, device="cuda")
    seq = {k: torch.from_numpy(np.ascontiguousarray(inp[k][:steps, :batch])).to(adt).cuda()
           for k in ("x", "z", "B", "C", "dt")}
    d = ddims(w, batch)
    ys = torch.empty(steps, batch, w.d_inner, dtype=adt, device="cuda")
    for s in range(steps):
        sm.decode_step(d, seq["x"][s], seq["z"][s], seq["B"][s], seq["C"][s], seq["dt"][s],
                       dv["A"], dv["D"], dv["conv_w"], dv["conv_b"], dv["dt_bias"], dv["norm_w"],
                       ssm, conv, sidx, y=ys[s])
    torch.cuda.synchronize()
    return ys, ssm[slots], conv[slots]


def oracle_as_prefill(w, inp, steps, batch):
    seq = {k: np.swapaxes(inp[k][:steps, :batch], 0, 1) for k in ("x", "z", "B", "C", "dt")}
    params = {k: inp[k] for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
    return oracle.prefill_dict(odims(w, batch, steps), dict(seq, **params,
                               init_ssm=inp["init_ssm"][:batch], init_conv=inp["init_conv"][:batch]))


def test_decode_workload_first_steps_full_batch():
    w = WORKLOADS["decode_bf16"]
    inp = make_decode_inputs(w, steps=2)
    ys, ssm, conv = run_steps(w, inp, 2, w.batch)
    ref = oracle_as_prefill(w, inp, 2, w.batch)
    tol = TOL[w.act]
    assert_close("y", ys.permute(1, 0, 2), ref["y"], tol)
    assert_close("ssm_state", ssm, ref["final_ssm"], tol)
    assert_close("conv_state", conv, ref["final_conv"], tol)


def test_decode_workload_1000_steps_eight_sequences():
    w = WORKLOADS["decode_bf16"]
    inp = make_decode_inputs(w.with_(batch=8), steps=1000, seed=w.seed)
    ys, ssm, conv = run_steps(w, inp, 1000, 8)
    ref = oracle_as_prefill(w, inp, 1000, 8)
    tol = TOL[w.act]
    assert_close("y", ys.permute(1, 0, 2), ref["y"], tol)
    assert_close("ssm_state", ssm, ref["final_ssm"], tol)
    assert_close("conv_state", conv, ref["final_conv"], tol)


@pytest.mark.parametrize("act,H,P,G,N", [("f32", 4, 16, 1, 16), ("f32", 8, 32, 2, 64), ("bf16", 16, 64, 4, 32)])
def test_decode_small_shapes_with_permuted_slots(act, H, P, G, N):
    base = WORKLOADS["tiny_f32"] if act == "f32" else WORKLOADS["decode_bf16"]
    w = base.with_(batch=5, nheads=H, headdim=P, ngroups=G, dstate=N, init_ssm_std=0.1, init_conv_std=1.0)
    inp = make_decode_inputs(w, steps=40, seed=7)
    slots = [6, 0, 3, 2, 5]          # sequence i lives in slot slots[i]; slots 1 and 4 untouched
    ys, ssm, conv = run_steps(w, inp, 40, 5, slot_idx=slots, nslots=7)
    ref = oracle_as_prefill(w, inp, 40, 5)
    tol = TOL[act]
    assert_close("y", ys.permute(1, 0, 2), ref["y"], tol)
    assert_close("ssm_state", ssm, ref["final_ssm"], tol)
    assert_close("conv_state", conv, ref["final_conv"], tol)


@pytest.mark.parametrize("b,H,G", [(1, 256, 8), (3, 16, 2), (4, 4, 2)])
def test_decode_small_batches_split_groups_over_clusters(b, H, G):
    """Few sequences: each group's heads are split over a cluster of CTAs (8, 8 and 2 CTAs per
    group here) that exchange their partial sums of squares through distributed shared memory.
    The first case is the decode token of the long_bf16 step."""
    w = WORKLOADS["decode_bf16"].with_(batch=b, nheads=H, ngroups=G)
    inp = make_decode_inputs(w, steps=12, seed=9)
    slots = list(reversed(range(b))) if b > 1 else None
    ys, ssm, conv = run_steps(w, inp, 12, b, slot_idx=slots, nslots=b)
    ref = oracle_as_prefill(w, inp, 12, b)
    tol = TOL[w.act]
    assert_close("y", ys.permute(1, 0, 2), ref["y"], tol)
    assert_close("ssm_state", ssm, ref["final_ssm"], tol)
    assert_close("conv_state", conv, ref["final_conv"], tol)
