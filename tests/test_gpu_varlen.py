"""Parity of the packed variable-length prefill on state slots (ssd_mixer_prefill_varlen)
with the fp64 oracle, sequence by sequence: ragged lengths around the 128-token block (0, 1,
3, 127..129, 300), slots in any order, sequences that continue from their slot and ones that
start afresh, groups held by one cluster and groups wider than one; untouched slots stay bit
for bit. Also the in-place case of the plain prefill for groups wider than one cluster."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs, round_bf16
from tests.gpu_util import TOL, assert_close, dims_of, gpu_prefill, oracle_dims, to_dev

pytestmark = pytest.mark.gpu

PARAMS = ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")
SEQ = ("x", "z", "B", "C", "dt")


def run_varlen(H, G, lens, slots, has_init, nslots, seed):
    T = int(sum(lens))
    w = WORKLOADS["small_bf16"].with_(batch=1, seqlen=max(T, 1), nheads=H, headdim=64, ngroups=G, dstate=128,
                                      chunk=128, init_ssm_std=0.0, init_conv_std=0.0, seed=seed)
    inp = make_prefill_inputs(w)
    rng = np.random.default_rng(seed + 1000)
    ssm0 = (0.1 * rng.standard_normal((nslots, H, 64, 128))).astype(np.float32)
    conv0 = round_bf16(rng.standard_normal((nslots, w.xbc_channels, 3))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    pk = {k: inp[k][0, :T] for k in SEQ}
    y_ref, ssm_ref, conv_ref = oracle.prefill_varlen(
        oracle_dims(dims_of(w)), cu, *(pk[k] for k in SEQ), *(inp[k] for k in PARAMS), ssm0, conv0,
        slot_idx=slots, has_init=has_init)

    dv = to_dev({k: np.ascontiguousarray(pk[k]) for k in SEQ}, "bf16")
    par = to_dev({k: inp[k] for k in PARAMS}, "bf16")
    ssm = torch.from_numpy(ssm0).cuda()
    conv = torch.from_numpy(conv0).to(torch.bfloat16).cuda()
    y = torch.full((T, H * 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    d = sm.Dims(len(lens), T, H, 64, G, 128, 128, 4, w.eps, "bf16")
    ws = torch.empty(max(sm.ssd_mixer_prefill_varlen_workspace_size(d), 256), dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_prefill_varlen(
        d, torch.from_numpy(cu).cuda(),
        None if slots is None else torch.tensor(slots, dtype=torch.int32, device="cuda"),
        None if has_init is None else torch.tensor(has_init, dtype=torch.uint8, device="cuda"),
        *(dv[k] for k in SEQ), *(par[k] for k in PARAMS), ssm, conv, y, ws)
    torch.cuda.synchronize()
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    tol = TOL["bf16"]
    if T > 0:
        assert_close("y", y, y_ref, tol)
    used = sorted(set(slots if slots is not None else range(len(lens))))
    assert_close("ssm slots", ssm[used], ssm_ref[used], tol)
    assert_close("conv slots", conv[used], conv_ref[used], tol)
    for k in range(nslots):
        if k not in used:
            assert torch.equal(ssm[k].cpu(), torch.from_numpy(ssm0[k])), f"slot {k} changed"
            assert torch.equal(conv[k].float().cpu(), torch.from_numpy(conv0[k])), f"conv slot {k} changed"


def test_varlen_one_cluster_per_group():
    run_varlen(8, 2, lens=[5, 128, 0, 300, 1, 129, 3, 127], slots=[7, 0, 11, 3, 5, 9, 2, 10],
               has_init=[1, 0, 1, 1, 0, 1, 1, 0], nslots=12, seed=51)


def test_varlen_groups_wider_than_a_cluster():
    run_varlen(16, 2, lens=[200, 1, 130, 0, 256], slots=[4, 0, 2, 5, 1], has_init=[1, 1, 0, 1, 0],
               nslots=7, seed=52)


def test_varlen_identity_slots_and_defaults():
    run_varlen(8, 2, lens=[64, 192], slots=None, has_init=None, nslots=2, seed=53)


def test_varlen_all_sequences_empty():
    run_varlen(8, 2, lens=[0, 0, 0], slots=[2, 0, 1], has_init=[1, 0, 1], nslots=4, seed=54)


@pytest.mark.parametrize("b,L", [(2, 333), (1, 600)])
def test_wide_groups_final_states_may_alias_initial_states(b, L):
    """Plain prefill, bf16, 8 heads per group (two clusters of 4 per group), with the final
    states written over the initial ones: the first cluster of a group stages the B/C part
    of the final conv state, so no cluster overwrites an initial state another still reads."""
    base = WORKLOADS["small_bf16"]
    w = base.with_(batch=b, seqlen=L, nheads=16, headdim=64, ngroups=2, dstate=128, chunk=128,
                   init_ssm_std=0.1, init_conv_std=1.0, seed=55)
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    ssm, conv = dv["init_ssm"].clone(), dv["init_conv"].clone()
    y = torch.empty(w.batch, w.seqlen, w.d_inner, dtype=torch.bfloat16, device="cuda")
    gpu_prefill(d, dv, init_ssm=ssm, init_conv=conv, out=(y, ssm, conv))
    torch.cuda.synchronize()
    tol = TOL["bf16"]
    assert_close("y", y, ref["y"], tol)
    assert_close("final_ssm (aliased)", ssm, ref["final_ssm"], tol)
    assert_close("final_conv (aliased)", conv, ref["final_conv"], tol)


def test_one_token_sequences_match_the_decode_step():
    """Mixed prefill and decode in one packed call: one-token sequences give the same outputs
    and slot states as ssd_mixer_decode_step on the same slots (both run the recurrence once
    from the slot's states), next to a longer prefill on another slot."""
    H, G, nslots = 8, 2, 6
    lens = [1, 200, 1, 1]
    slots = [4, 1, 0, 5]
    T = sum(lens)
    w = WORKLOADS["small_bf16"].with_(batch=1, seqlen=T, nheads=H, headdim=64, ngroups=G, dstate=128,
                                      chunk=128, init_ssm_std=0.0, init_conv_std=0.0, seed=57)
    inp = make_prefill_inputs(w)
    rng = np.random.default_rng(58)
    ssm0 = torch.from_numpy((0.1 * rng.standard_normal((nslots, H, 64, 128))).astype(np.float32)).cuda()
    conv0 = torch.from_numpy(round_bf16(rng.standard_normal((nslots, w.xbc_channels, 3))).astype(np.float32))
    conv0 = conv0.to(torch.bfloat16).cuda()
    dv = to_dev({k: np.ascontiguousarray(inp[k][0]) for k in SEQ}, "bf16")
    par = to_dev({k: inp[k] for k in PARAMS}, "bf16")
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    # packed call
    ssm_a, conv_a = ssm0.clone(), conv0.clone()
    y_a = torch.empty(T, H * 64, dtype=torch.bfloat16, device="cuda")
    d = sm.Dims(len(lens), T, H, 64, G, 128, 128, 4, w.eps, "bf16")
    ws = torch.empty(sm.ssd_mixer_prefill_varlen_workspace_size(d), dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_prefill_varlen(d, cu, torch.tensor(slots, dtype=torch.int32, device="cuda"), None,
                                *(dv[k] for k in SEQ), *(par[k] for k in PARAMS), ssm_a, conv_a, y_a, ws)
    # decode steps for the one-token sequences
    ones = [i for i, n in enumerate(lens) if n == 1]
    rows = [int(cu[i]) for i in ones]
    ssm_b, conv_b = ssm0.clone(), conv0.clone()
    dd = sm.Dims(len(ones), 1, H, 64, G, 128, 1, 4, w.eps, "bf16")
    y_b = sm.decode_step(dd, *(dv[k][rows].contiguous() for k in SEQ), *(par[k] for k in PARAMS), ssm_b, conv_b,
                         torch.tensor([slots[i] for i in ones], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    for j, i in enumerate(ones):
        assert_close(f"y of one-token sequence {i}", y_a[rows[j]], y_b[j].float().cpu().numpy(), TOL["bf16"])
        k = slots[i]
        assert_close(f"ssm slot {k}", ssm_a[k], ssm_b[k].cpu().numpy(), TOL["bf16"])
        assert torch.equal(conv_a[k], conv_b[k]), f"conv slot {k}"
