"""Failure detection on the GPU without a fault: a bounded device-side wait that nothing
satisfies gives up after its limit, the status word says so, ssd_mixer_workspace_status maps
it to SSD_ERR_TIMEOUT, and the CUDA context stays usable (a prefill afterwards still matches
the oracle)."""
import pytest
import torch

import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import TOL, assert_close, dims_of, gpu_prefill, oracle_dims, to_dev

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_satisfies_times_out_and_reports_it():
    ws = torch.full((256,), 0x5A, dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_selftest_wait(ws, 1_000_000, arrive=False)    # about half a millisecond
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_ERR_TIMEOUT
    sm.ssd_mixer_selftest_wait(ws, 1_000_000, arrive=True)
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    sm.ssd_mixer_selftest_wait(ws, 0, arrive=False)             # a limit of zero cycles
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_ERR_TIMEOUT
    # the context is still usable
    w = WORKLOADS["tiny_f32"]
    inp = make_prefill_inputs(w)
    d = dims_of(w)
    y, fs, fc = gpu_prefill(d, to_dev(inp, w.act))
    torch.cuda.synchronize()
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y after the timed-out wait", y, ref["y"], TOL[w.act])
