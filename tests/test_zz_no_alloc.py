"""GPU test of ssd_mixer_prefill_static, the prefill that allocates nothing (needs a B200).

Some callers cannot allocate device memory: a plugin slot that hands the library only
tensors and a stream, or a serving process whose memory is fully reserved by its own
pool. For them the library keeps a fixed device array as the prefill's scratch. This
test calls that entry point through the C ABI twice in a row on different inputs and
checks each result against the regular entry point (caller-supplied workspace). Both run
the same kernels on the same inputs, so the results must be bit for bit equal. The cases
cover the CUDA-core path (fp32), the tensor-core path whose group fits one cluster
(bf16, 4 heads per group: only the status word is scratch) and the tensor-core path with
wider groups (bf16, 8 heads per group: per-token partial sums and the staged B/C conv state
live in the array), so the array's reuse from one call to the next is exercised. The
array's status word is read back with ssd_mixer_prefill_static_status. An oversized
problem is refused. The file is named to be collected last, so a run that stops at the
first failure has already run every other test; it also passes when run alone in a fresh
process.
"""
import pytest
import torch

from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import dims_of, gpu_prefill, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    "f32": dict(base="tiny_f32", act="f32", shape={}),
    "bf16_cluster_group": dict(base="small_bf16", act="bf16", shape={}),
    "bf16_wide_group": dict(base="small_bf16", act="bf16", shape=dict(nheads=16, ngroups=2)),
}


def _static_call(d, dv, y, fs, fc):
    return sm.ssd_mixer_prefill_static(d, dv["x"], dv["z"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["D"],
                                       dv["conv_w"], dv["conv_b"], dv["dt_bias"], dv["norm_w"],
                                       dv["init_ssm"], dv["init_conv"], y, fs, fc)


@pytest.mark.parametrize("case", list(CASES))
def test_static_workspace_prefill_equals_regular_prefill_twice(case):
    c = CASES[case]
    act = c["act"]
    w = WORKLOADS[c["base"]].with_(batch=2, seqlen=333, init_ssm_std=0.1, init_conv_std=1.0, **c["shape"])
    d = dims_of(w)
    assert 0 < sm.ssd_mixer_prefill_workspace_size(d) <= sm.SSD_MIXER_STATIC_WORKSPACE_BYTES
    adt = torch.bfloat16 if act == "bf16" else torch.float32
    for seed in (101, 202):                       # two calls in a row, different inputs
        dv = to_dev(make_prefill_inputs(w, seed=seed), act)
        y = torch.empty(w.batch, w.seqlen, w.d_inner, dtype=adt, device="cuda")
        fs = torch.empty(w.batch, w.nheads, w.headdim, w.dstate, device="cuda")
        fc = torch.empty(w.batch, w.xbc_channels, 3, dtype=adt, device="cuda")
        st = _static_call(d, dv, y, fs, fc)
        assert st == sm.SSD_OK, st
        assert sm.ssd_mixer_prefill_static_status() == sm.SSD_OK
        y_ref, fs_ref, fc_ref = gpu_prefill(d, dv)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), "y differs from the regular entry point"
        assert torch.equal(fs, fs_ref), "final SSM state differs from the regular entry point"
        assert torch.equal(fc, fc_ref), "final conv state differs from the regular entry point"


def test_static_workspace_refuses_oversized_problem():
    # fp32 activations run the CUDA-core path, whose scratch grows with the token count:
    # 131072 tokens of this shape need more than the fixed array holds
    w = WORKLOADS["tiny_f32"].with_(batch=1, seqlen=131072)
    d = dims_of(w)
    assert sm.ssd_mixer_prefill_workspace_size(d) > sm.SSD_MIXER_STATIC_WORKSPACE_BYTES
    L, HP, GN = w.seqlen, w.d_inner, w.ngroups * w.dstate
    x = torch.zeros(1, L, HP, device="cuda")
    bc = torch.zeros(1, L, GN, device="cuda")
    dt = torch.zeros(1, L, w.nheads, device="cuda")
    prm = torch.zeros(w.xbc_channels * 4, device="cuda")
    fs = torch.zeros(1, w.nheads, w.headdim, w.dstate, device="cuda")
    fc = torch.zeros(1, w.xbc_channels, 3, device="cuda")
    y = torch.empty_like(x)
    st = sm.ssd_mixer_prefill_static(d, x, x, bc, bc, dt, prm, prm, prm, prm, prm, prm, None, None,
                                     y, fs, fc)
    assert st == sm.SSD_ERR_TOO_LARGE
