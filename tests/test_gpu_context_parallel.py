"""The state-only prefill, the state pass, and a context-parallel prefill of one row in three
pieces (the ranks run phase by phase in one process on one GPU), against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import context_parallel as cp
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import TOL, assert_close, dims_of, oracle_dims, to_dev

pytestmark = pytest.mark.gpu

SEQ = ("x", "z", "B", "C", "dt")
PAR = ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")


def workload(b, L, H, G, seed):
    return WORKLOADS["small_bf16"].with_(batch=b, seqlen=L, nheads=H, headdim=64, ngroups=G, dstate=128, chunk=128,
                                         init_ssm_std=0.1, init_conv_std=1.0, seed=seed)


@pytest.mark.parametrize("b,L,H,G,alias", [(2, 300, 8, 2, False), (1, 200, 16, 2, True), (2, 2, 8, 2, False)])
def test_state_only_prefill_matches_oracle(b, L, H, G, alias):
    w = workload(b, L, H, G, seed=61)
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    dv = to_dev(inp, "bf16")
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    dec_ref = oracle.decay(inp["dt"], inp["A"], inp["dt_bias"])
    if alias:
        fs, fc = dv["init_ssm"].clone(), dv["init_conv"].clone()
        init_s, init_c = fs, fc
    else:
        fs = torch.empty(b, H, 64, 128, device="cuda")
        fc = torch.empty(b, w.xbc_channels, 3, dtype=torch.bfloat16, device="cuda")
        init_s, init_c = dv["init_ssm"], dv["init_conv"]
    a = torch.empty(b, H, device="cuda")
    ws = torch.empty(max(sm.ssd_mixer_prefill_state_workspace_size(d), 256), dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_prefill_state(d, dv["x"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["conv_w"], dv["conv_b"],
                               dv["dt_bias"], init_s, init_c, fs, fc, a, ws)
    torch.cuda.synchronize()
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    assert_close("final_ssm", fs, ref["final_ssm"], TOL["bf16"])
    assert_close("final_conv", fc, ref["final_conv"], TOL["bf16"])
    assert_close("decay", a, dec_ref, 1e-4)


def test_state_pass_folds_pieces():
    rng = np.random.default_rng(62)
    R, b, H, P, N = 4, 2, 3, 64, 128
    dec = rng.uniform(0.0, 1.0, (R, b, H)).astype(np.float32)
    st = rng.standard_normal((R, b, H, P, N)).astype(np.float32)
    h0 = rng.standard_normal((b, H, P, N)).astype(np.float32)
    for r in range(R + 1):
        ref = h0.astype(np.float64)
        for j in range(r):
            ref = dec[j][:, :, None, None] * ref + st[j]
        out = torch.empty(b, H, P, N, device="cuda")
        sm.ssd_mixer_state_pass(r, torch.from_numpy(dec).cuda(), torch.from_numpy(st).cuda(),
                                torch.from_numpy(h0).cuda(), out)
        torch.cuda.synchronize()
        assert_close(f"state entering piece {r}", out, ref, 1e-6)


@pytest.mark.parametrize("H,G,lens", [(8, 2, (300, 130, 260)), (16, 2, (129, 3, 256))])
def test_context_parallel_prefill_in_three_pieces(H, G, lens):
    b, L = 2, sum(lens)
    w = workload(b, L, H, G, seed=63)
    inp = make_prefill_inputs(w)
    ref = oracle.prefill_dict(oracle_dims(dims_of(w)), inp)
    dv = to_dev(inp, "bf16")
    params = {k: dv[k] for k in PAR}
    cuts = np.concatenate([[0], np.cumsum(lens)])
    pieces = [{k: dv[k][:, cuts[r]:cuts[r + 1]].contiguous() for k in SEQ} for r in range(len(lens))]
    dims = [dims_of(w, seqlen=n) for n in lens]
    cp.check_pieces(lens)
    # the ranks, one phase at a time; the all-gathers are plain lists here
    sts = [cp.phase1(dims[r], pieces[r], params) for r in range(len(lens))]
    tails = [s.conv_tail for s in sts]
    sts = [cp.phase2(r, sts[r], tails, dims[r], pieces[r], params, dv["init_ssm"], dv["init_conv"])
           for r in range(len(lens))]
    decays, states = [s.decay for s in sts], [s.zero_state for s in sts]
    outs = [cp.phase3(r, sts[r], decays, states, dims[r], pieces[r], params, dv["init_ssm"])
            for r in range(len(lens))]
    torch.cuda.synchronize()
    y = torch.cat([o[0] for o in outs], dim=1)
    tol = TOL["bf16"]
    assert_close("y", y, ref["y"], tol)
    assert_close("final_ssm", outs[-1][1], ref["final_ssm"], tol)
    assert_close("final_conv", outs[-1][2], ref["final_conv"], tol)
