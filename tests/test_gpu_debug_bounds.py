"""The bounds-checked build (libssd_mixer_debug.so, compiled with -DSSD_DEBUG_BOUNDS): every
guarded index of the small parity cases stays inside its buffer, so the status word reads OK
and the results equal the oracle's. The cases run in a fresh process that opens the debug
library (the binding keeps one library per process)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import torch
import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import TOL, assert_close, dims_of, oracle_dims, to_dev
assert sm.load_library()._name.endswith("libssd_mixer_debug.so")
cases = [
    ("tiny_f32", {}),                                           # CUDA-core path
    ("small_bf16", dict(batch=2, seqlen=300)),                  # clusters of 4
    ("small_bf16", dict(batch=1, seqlen=333, nheads=16, ngroups=2, init_ssm_std=0.1, init_conv_std=1.0)),  # wide groups
]
for base, kw in cases:
    w = WORKLOADS[base].with_(**kw)
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, w.act)
    d = dims_of(w)
    ws = sm.alloc_workspace(d)
    y, fs, fc = sm.prefill(d, dv["x"], dv["z"], dv["B"], dv["C"], dv["dt"], dv["A"], dv["D"], dv["conv_w"],
                           dv["conv_b"], dv["dt_bias"], dv["norm_w"], dv["init_ssm"], dv["init_conv"], workspace=ws)
    torch.cuda.synchronize()
    st = sm.ssd_mixer_workspace_status(ws)
    assert st == sm.SSD_OK, (base, kw, st)
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y", y, ref["y"], TOL[w.act])
    assert_close("final_ssm", fs, ref["final_ssm"], TOL[w.act])
    assert_close("final_conv", fc, ref["final_conv"], TOL[w.act])
print("debug-bounds cases ok")
'''


@pytest.mark.gpu
def test_bounds_checked_build_reports_no_violation_on_the_parity_cases():
    from hybrid_mamba_ssm_causal_b200 import build
    lib = build.build(debug_bounds=True)
    env = dict(os.environ, SSD_MIXER_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "debug-bounds cases ok" in r.stdout


def test_bounds_checked_build_compiles_the_checks_in():
    """The flag reaches the kernels: the main prefill source compiled with and without it
    gives different objects (the checks are code), and both compile for sm_100a."""
    from hybrid_mamba_ssm_causal_b200 import build
    import tempfile
    src = os.path.join(build.CSRC, "ssd_prefill_ws.cu")
    outs = []
    with tempfile.TemporaryDirectory() as td:
        for i, extra in enumerate(([], ["-DSSD_DEBUG_BOUNDS"])):
            obj = os.path.join(td, f"o{i}.o")
            subprocess.run([build.nvcc(), *build.ARCH, *build.NVCC_FLAGS, *extra, "-c", src, "-o", obj],
                           check=True, capture_output=True, timeout=600)
            outs.append(os.path.getsize(obj))
    assert outs[0] != outs[1]
