"""Rows run as pieces over a series of launches (the tensor-core prefill of groups wider than a
cluster). A piece continues from the state its predecessor left in the final-state buffer,
and its conv halo is the row's own preceding tokens; each launch after the first may start
while the one before it finishes. The library picks the piece count itself (pieces only when
there are at least as many rows as SMs, as on long_bf16 and mid_bf16, which the prefill tests
cover); here SSD_MIXER_PREFILL_PIECES fixes it, so that small cases reach every edge: a last
piece of one or two tokens, single-block pieces, initial states, and states chained in place
across two calls. The variable is read once per process, so each count runs in a fresh one."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import os
import torch
import oracle
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
from tests.gpu_util import TOL, assert_close, dims_of, gpu_prefill, oracle_dims, slice_seq, to_dev

base = WORKLOADS["small_bf16"]
cases = [
    # 8 heads per group (no cluster); 513 tokens = 4 blocks and 1 token
    base.with_(batch=2, seqlen=513, nheads=16, ngroups=2, init_ssm_std=0.1, init_conv_std=1.0, seed=21),
    # 130 tokens: a second piece of 2 tokens, shorter than the conv window
    base.with_(batch=3, seqlen=130, nheads=8, ngroups=1, init_ssm_std=0.0, init_conv_std=0.0, seed=22),
    # 512 tokens = 4 whole blocks: 2 or 4 pieces of equal length
    base.with_(batch=2, seqlen=512, nheads=16, ngroups=2, init_ssm_std=0.1, init_conv_std=1.0, seed=25),
]
for w in cases:
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, w.act)
    d = dims_of(w)
    ws = sm.alloc_workspace(d)
    y, fs, fc = gpu_prefill(d, dv, workspace=ws)
    torch.cuda.synchronize()
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y", y, ref["y"], TOL["bf16"])
    assert_close("final_ssm", fs, ref["final_ssm"], TOL["bf16"])
    assert_close("final_conv", fc, ref["final_conv"], TOL["bf16"])

# two calls chained through states updated in place (the final states written over the inits)
w = cases[0]
inp = make_prefill_inputs(w)
dv = to_dev(inp, w.act)
ref = oracle.prefill_dict(oracle_dims(dims_of(w)), inp)
L1 = 300
ssm, conv = dv["init_ssm"].clone(), dv["init_conv"].clone()
y = torch.empty(w.batch, w.seqlen, w.d_inner, dtype=torch.bfloat16, device="cuda")
y1 = torch.empty(w.batch, L1, w.d_inner, dtype=torch.bfloat16, device="cuda")
y2 = torch.empty(w.batch, w.seqlen - L1, w.d_inner, dtype=torch.bfloat16, device="cuda")
gpu_prefill(dims_of(w, seqlen=L1), slice_seq(dv, 0, L1), init_ssm=ssm, init_conv=conv, out=(y1, ssm, conv))
gpu_prefill(dims_of(w, seqlen=w.seqlen - L1), slice_seq(dv, L1, w.seqlen), init_ssm=ssm, init_conv=conv,
            out=(y2, ssm, conv))
torch.cuda.synchronize()
assert_close("y chained", torch.cat([y1, y2], 1), ref["y"], TOL["bf16"])
assert_close("final_ssm chained", ssm, ref["final_ssm"], TOL["bf16"])
assert_close("final_conv chained", conv, ref["final_conv"], TOL["bf16"])
print("pieces ok", os.environ["SSD_MIXER_PREFILL_PIECES"])
'''


def run_with_pieces(n: int, library: str | None = None):
    env = dict(os.environ, SSD_MIXER_PREFILL_PIECES=str(n))
    if library:
        env["SSD_MIXER_LIBRARY"] = library
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert f"pieces ok {n}" in r.stdout


@pytest.mark.gpu
@pytest.mark.parametrize("n", [2, 3, 4, 5])
def test_rows_in_pieces_match_the_oracle(n):
    """On 513 tokens, n = 2: pieces of 3 and 2 blocks; 3: the last piece is the one-token block;
    5: every block its own piece. On 512 tokens, 2 and 4 pieces are equally long."""
    run_with_pieces(n)


@pytest.mark.gpu
def test_rows_in_pieces_stay_in_bounds():
    """The same cases in the bounds-checked build: every guarded index of a piece stays in its
    buffer (the status word reads OK)."""
    from hybrid_mamba_ssm_causal_b200 import build
    run_with_pieces(3, build.build(debug_bounds=True))


def _automatic_case(**kw):
    """The library's own plan, in this process: the whole outputs against the oracle."""
    import torch

    import oracle
    from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
    from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_prefill_inputs
    from tests.gpu_util import TOL, assert_close, dims_of, gpu_prefill, oracle_dims, to_dev
    w = WORKLOADS["small_bf16"].with_(**kw)
    inp = make_prefill_inputs(w)
    dv = to_dev(inp, w.act)
    d = dims_of(w)
    ws = sm.alloc_workspace(d)
    y, fs, fc = gpu_prefill(d, dv, workspace=ws)
    torch.cuda.synchronize()
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    ref = oracle.prefill_dict(oracle_dims(d), inp)
    assert_close("y", y, ref["y"], TOL["bf16"])
    assert_close("final_ssm", fs, ref["final_ssm"], TOL["bf16"])
    assert_close("final_conv", fc, ref["final_conv"], TOL["bf16"])


@pytest.mark.gpu
def test_many_short_rows_stay_whole_in_one_launch():
    """256 (sequence, head) rows of 3 blocks on 148 SMs: the plan keeps rows whole, so one
    launch must cover every row (not 148 per launch)."""
    if os.environ.get("SSD_MIXER_PREFILL_PIECES"):
        pytest.skip("piece count fixed by the environment")
    _automatic_case(batch=2, seqlen=300, nheads=128, ngroups=16, init_ssm_std=0.1, init_conv_std=1.0, seed=23)


@pytest.mark.gpu
def test_automatic_pieces_with_a_ragged_last_block():
    """192 rows of 8 blocks (the last 104 tokens): the plan splits each row in two."""
    if os.environ.get("SSD_MIXER_PREFILL_PIECES"):
        pytest.skip("piece count fixed by the environment")
    _automatic_case(batch=3, seqlen=1000, nheads=64, ngroups=8, init_ssm_std=0.1, init_conv_std=1.0, seed=24)
