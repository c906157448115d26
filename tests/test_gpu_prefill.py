"""GPU parity of ssd_mixer_prefill against the fp64 oracle (needs a B200).

Tolerance: max|err| / max|ref| <= 1e-4 for fp32 activations and <= 2e-2 for bf16
activations (fp32 accumulation and state), on y, the final SSM state and the final
conv state. Small cases span several chunks and tiles with a ragged tail; the full-size
workloads are checked on sampled (batch row, group) sub-problems, which the mixer core
computes independently of each other.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import (TOL, assert_close, dims_of, gpu_prefill, oracle_dims, slice_seq,
                            to_dev)

pytestmark = pytest.mark.gpu


def small(act, b, L, H, P, G, N, Q, init=True, seed=0):
    base = WORKLOADS["tiny_f32"] if act == "f32" else WORKLOADS["small_bf16"]
    return base.with_(batch=b, seqlen=L, nheads=H, headdim=P, ngroups=G, dstate=N, chunk=Q,
                      init_ssm_std=0.1 if init else 0.0, init_conv_std=1.0 if init else 0.0, seed=seed)


def check_full(w, inp, outs, d):
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    y, fs, fc = outs
    tol = TOL[w.act]
    return (assert_close("y", y, ref["y"], tol), assert_close("final_ssm", fs, ref["final_ssm"], tol),
            assert_close("final_conv", fc, ref["final_conv"], tol))


SMALL_CASES = [
    ("f32", 1, 256, 4, 16, 1, 16, 64, False),     # the tiny fp32 workload's shape
    ("f32", 2, 203, 4, 16, 2, 32, 64, True),      # ragged tail, two groups, initial states
    ("f32", 1, 77, 2, 32, 1, 64, 32, True),
    ("bf16", 2, 300, 8, 64, 2, 128, 128, True),    # ragged: 2 full chunks + 44 tokens
    ("bf16", 1, 700, 8, 64, 2, 128, 128, True),    # one row, 5 full blocks + 60 tokens
    ("bf16", 1, 1000, 16, 64, 2, 128, 128, True),  # groups wider than one cluster (8 heads)
    ("bf16", 1, 517, 4, 32, 1, 64, 256, True),     # Q = 256, ragged
    ("bf16", 3, 64, 8, 64, 4, 64, 64, False),      # exactly one chunk
    ("bf16", 1, 1, 4, 64, 2, 128, 128, True),      # one token
    ("bf16", 2, 2, 4, 64, 2, 128, 128, True),      # shorter than the conv window
    ("bf16", 1, 129, 2, 16, 1, 16, 16, True),      # smallest chunk
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: "-".join(map(str, c)))
def test_small_cases_match_oracle(case):
    act, b, L, H, P, G, N, Q, init = case
    w = small(act, b, L, H, P, G, N, Q, init, seed=sum(case[1:8]))
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    outs = gpu_prefill(d, to_dev(inp, act))
    torch.cuda.synchronize()
    check_full(w, inp, outs, d)


def test_tiny_f32_workload():
    w = WORKLOADS["tiny_f32"]
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    outs = gpu_prefill(d, to_dev(inp, w.act))
    torch.cuda.synchronize()
    errs = check_full(w, inp, outs, d)
    assert max(errs) <= 1e-4


def test_small_bf16_workload_full():
    w = WORKLOADS["small_bf16"]
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    outs = gpu_prefill(d, to_dev(inp, w.act))
    torch.cuda.synchronize()
    check_full(w, inp, outs, d)


def sampled_check(w, inp, d_full, y, fs, fc, rows, groups, total_inp=None):
    """Compare (row, group) sub-problems of a full-size run with the oracle, in parallel
    threads (the oracle call releases the GIL)."""
    src = total_inp if total_inp is not None else inp
    od = oracle.Dims(w.batch, src["x"].shape[1], w.nheads, w.headdim, w.ngroups, w.dstate, w.dconv, w.eps)
    jobs = []
    for g in groups:
        sd, sub, xs, hs, cidx = oracle.group_subproblem(od, g, src, batch_rows=rows)
        jobs.append((g, xs, hs, cidx, sd, sub))
    with ThreadPoolExecutor(len(jobs)) as ex:
        refs = list(ex.map(lambda j: oracle.prefill_dict(j[4], j[5], nthreads=2), jobs))
    tol = TOL[w.act]
    yn = y[rows]
    for (g, xs, hs, cidx, _, _), ref in zip(jobs, refs):
        assert_close(f"y group {g}", yn[:, :, xs], ref["y"], tol)
        assert_close(f"final_ssm group {g}", fs[rows][:, hs], ref["final_ssm"], tol)
        assert_close(f"final_conv group {g}", fc[rows][:, torch.as_tensor(cidx, device=fc.device)],
                     ref["final_conv"], tol)


def test_mid_bf16_workload_sampled():
    w = WORKLOADS["mid_bf16"]
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    y, fs, fc = gpu_prefill(d, to_dev(inp, w.act))
    torch.cuda.synchronize()
    sampled_check(w, inp, d, y, fs, fc, rows=[0, 5], groups=[0, 3, 7])


def test_long_bf16_workload_two_chained_calls():
    """32768 tokens as two 16384-token calls chained through the returned states, checked
    against one full-length oracle run on sampled groups."""
    w = WORKLOADS["long_bf16"]
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    T = w.total_seqlen
    y = torch.empty(w.batch, T, w.d_inner, dtype=torch.bfloat16, device="cuda")
    ws = sm.alloc_workspace(d)
    h1 = gpu_prefill(d, slice_seq(dv, 0, w.seqlen), workspace=ws,
                     out=(y[:, :w.seqlen], torch.empty(w.batch, w.nheads, w.headdim, w.dstate, device="cuda"),
                          torch.empty(w.batch, w.xbc_channels, 3, dtype=torch.bfloat16, device="cuda")))
    _, fs1, fc1 = h1
    _, fs, fc = gpu_prefill(d, slice_seq(dv, w.seqlen, T), init_ssm=fs1, init_conv=fc1, workspace=ws,
                            out=(y[:, w.seqlen:], fs1, fc1))     # final states written over the inits
    torch.cuda.synchronize()
    sampled_check(w, inp, d, y, fs, fc, rows=[0], groups=[2, 6])


def test_split_and_chain_matches_one_call():
    w = small("bf16", 2, 333, 8, 64, 2, 128, 128, True, seed=3)
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, w.act)
    ref = oracle.prefill_dict(oracle_dims(dims_of(w)), inp)
    for L1 in (1, 2, 3, 100, 128, 200):
        d1, d2 = dims_of(w, seqlen=L1), dims_of(w, seqlen=w.seqlen - L1)
        y1, fs1, fc1 = gpu_prefill(d1, slice_seq(dv, 0, L1))
        y2, fs2, fc2 = gpu_prefill(d2, slice_seq(dv, L1, w.seqlen), init_ssm=fs1, init_conv=fc1)
        torch.cuda.synchronize()
        assert_close(f"y split {L1}", torch.cat([y1, y2], 1), ref["y"], TOL["bf16"])
        assert_close(f"final_ssm split {L1}", fs2, ref["final_ssm"], TOL["bf16"])
        assert_close(f"final_conv split {L1}", fc2, ref["final_conv"], TOL["bf16"])


def test_final_states_may_alias_initial_states():
    w = small("f32", 2, 150, 4, 16, 2, 32, 64, True, seed=8)
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    ssm, conv = dv["init_ssm"].clone(), dv["init_conv"].clone()
    y = torch.empty(w.batch, w.seqlen, w.d_inner, device="cuda")
    gpu_prefill(d, dv, init_ssm=ssm, init_conv=conv, out=(y, ssm, conv))
    torch.cuda.synchronize()
    assert_close("y", y, ref["y"], TOL["f32"])
    assert_close("final_ssm (aliased)", ssm, ref["final_ssm"], TOL["f32"])
    assert_close("final_conv (aliased)", conv, ref["final_conv"], TOL["f32"])


def test_inputs_as_views_of_one_packed_projection():
    """x, z, B, C, dt given as column slices of one [b, L, z|x|B|C|dt] buffer, and y written
    into a wider buffer."""
    w = small("bf16", 2, 190, 8, 64, 2, 128, 64, True, seed=12)
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    width = 2 * HP + 2 * GN + H + 8      # padded so rows stay 16-byte aligned
    packed = torch.zeros(w.batch, w.seqlen, width, dtype=torch.bfloat16, device="cuda")
    packed[..., :HP] = dv["z"]
    packed[..., HP:2 * HP] = dv["x"]
    packed[..., 2 * HP:2 * HP + GN] = dv["B"]
    packed[..., 2 * HP + GN:2 * HP + 2 * GN] = dv["C"]
    packed[..., 2 * HP + 2 * GN:2 * HP + 2 * GN + H] = dv["dt"]
    views = dict(dv, z=packed[..., :HP], x=packed[..., HP:2 * HP], B=packed[..., 2 * HP:2 * HP + GN],
                 C=packed[..., 2 * HP + GN:2 * HP + 2 * GN], dt=packed[..., 2 * HP + 2 * GN:2 * HP + 2 * GN + H])
    ybig = torch.zeros(w.batch, w.seqlen, HP + 64, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty(w.batch, H, w.headdim, w.dstate, device="cuda")
    fc = torch.empty(w.batch, w.xbc_channels, 3, dtype=torch.bfloat16, device="cuda")
    gpu_prefill(d, views, out=(ybig[..., 32:32 + HP], fs, fc))
    torch.cuda.synchronize()
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y (strided)", ybig[..., 32:32 + HP], ref["y"], TOL["bf16"])
    assert torch.all(ybig[..., :32] == 0) and torch.all(ybig[..., 32 + HP:] == 0)
    assert_close("final_ssm", fs, ref["final_ssm"], TOL["bf16"])


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_chunk_size_invariance(act):
    """The chunk length Q is a schedule parameter: the CUDA-core path evaluates the chunked form
    with exactly Q-token chunks, and every Q gives the sequential recurrence's result. Both
    cases run that path (fp32, and bf16 with head dim 32, which the tensor-core kernel does not
    take); the tensor-core kernel always works in 128-token blocks, so Q has nothing to vary
    there."""
    w = small(act, 1, 640, 8, 32, 2, 64, 64, True, seed=21)
    assert not sm.prefill_uses_tensor_cores(dims_of(w))
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, act)
    ref = oracle.prefill_dict(oracle_dims(dims_of(w)), inp)
    outs = {}
    for Q in (64, 128, 256):
        outs[Q] = gpu_prefill(dims_of(w, chunk=Q), dv)
    torch.cuda.synchronize()
    for Q, (y, fs, fc) in outs.items():
        assert_close(f"y Q={Q}", y, ref["y"], TOL[act])
        assert_close(f"final_ssm Q={Q}", fs, ref["final_ssm"], TOL[act])


def test_causality():
    w = small("bf16", 1, 400, 8, 64, 2, 128, 128, True, seed=31)
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    y0, _, _ = gpu_prefill(d, to_dev(inp, w.act))
    tstar = 213
    rng = np.random.default_rng(5)
    pert = dict(inp)
    for k in ("x", "z", "B", "C", "dt"):
        v = inp[k].copy()
        v[:, tstar:] = rng.standard_normal(v[:, tstar:].shape).astype(np.float32)
        pert[k] = v
    y1, _, _ = gpu_prefill(d, to_dev(pert, w.act))
    torch.cuda.synchronize()
    assert torch.equal(y0[:, :tstar], y1[:, :tstar])
    assert not torch.equal(y0[:, tstar:], y1[:, tstar:])


def test_zero_step_keeps_state():
    """dt_raw = -1e4: delta underflows to exactly 0, so the SSM state passes through unchanged."""
    w = small("bf16", 2, 200, 8, 64, 2, 128, 64, True, seed=41)
    inp = make_prefill_inputs(w)
    inp["dt"] = np.full_like(inp["dt"], -1e4)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    y, fs, _ = gpu_prefill(d, dv)
    torch.cuda.synchronize()
    assert torch.equal(fs, dv["init_ssm"])
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y", y, ref["y"], TOL["bf16"])


def test_zero_tokens_passes_states_through():
    w = small("bf16", 2, 0, 4, 64, 2, 128, 64, True, seed=43)
    inp = make_prefill_inputs(w.with_(seqlen=4))
    inp = slice_seq(inp, 0, 0)
    d = dims_of(w)
    dv = to_dev(inp, w.act)
    _, fs, fc = gpu_prefill(d, dv)
    torch.cuda.synchronize()
    assert torch.equal(fs, dv["init_ssm"])
    assert torch.equal(fc, dv["init_conv"])


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_stages_of_the_cuda_core_path(act):
    """Per-stage parity: the CUDA-core path's intermediates in its workspace (SiLU(conv) of
    [x|B|C], delta = softplus(dt + dt_bias), and y before the gate and the norm) against the
    oracle's stage outputs, so a wrong stage is located by itself and not only through y and the
    final states. bf16 with head dim 32 runs this path too (the tensor-core kernel keeps its
    intermediates on chip)."""
    w = small(act, 2, 203, 4, 32, 2, 32, 64, True, seed=23)
    d = dims_of(w)
    assert sm.ssd_mixer_prefill_path(d) == sm.SSD_PATH_CUDA_CORES
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, act)
    ws = sm.alloc_workspace(d)
    gpu_prefill(d, dv, workspace=ws)
    torch.cuda.synchronize()
    off = sm.ssd_mixer_prefill_stage_offsets(d)
    b, L, H, HP, Cc = w.batch, w.seqlen, w.nheads, w.d_inner, w.xbc_channels
    adt = torch.bfloat16 if act == "bf16" else torch.float32
    es = 2 if act == "bf16" else 4

    def view(offset, n, dtype, esize):
        return ws[offset:offset + n * esize].view(dtype)

    xbc = view(off["xbc_act"], b * L * Cc, adt, es).view(b, L, Cc)
    delta = view(off["delta"], b * H * L, torch.float32, 4).view(b, H, L).transpose(1, 2)
    y_pre = view(off["y_pre"], b * L * HP, torch.float32, 4).view(b, L, HP)
    ref = oracle.prefill_dict(oracle_dims(d), inp, stages=True)
    assert_close("xbc_act", xbc, ref["xbc_act"], TOL[act])
    assert_close("delta", delta, ref["delta"], 1e-5)
    assert_close("y_pre", y_pre, ref["y_pre"], TOL[act])


def test_stage_offsets_refused_on_the_tensor_core_path():
    d = dims_of(WORKLOADS["small_bf16"])
    assert sm.ssd_mixer_prefill_path(d) == sm.SSD_PATH_TENSOR_CORES
    with pytest.raises(sm.SsdError):
        sm.ssd_mixer_prefill_stage_offsets(d)
