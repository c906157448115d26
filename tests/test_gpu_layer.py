"""GPU parity of the mixer layer's projections and of the whole layer (needs a B200).

ssd_mixer_projection (C = A . W^T, bf16 in and out, fp32 accumulation on tcgen05) is compared
with an fp32 matmul of the same bf16 operands: max|err|/max|ref| <= 1e-2 (the output is rounded
to bf16, 2^-9 relative, and the sums run in a different order). The shapes span several
128 x 256 tiles with ragged edges in M, N and K.

ssd_mixer_layer_prefill (in_proj -> the core on column slices of the packed [z | x | B | C | dt]
row -> out_proj) is compared with the fp64 layer oracle (oracle/layer.py) within the bf16
tolerance 2e-2 on the layer output and both final states, for a norm group held by one cluster
(4 heads per group: the core normalises) and for a wider group (8 heads per group), with the
norm finished by the core's own pass or, on request, by out_proj applying the group scale and
norm weights to its input tiles.
"""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm
from hybrid_mamba_ssm_causal_b200.workloads import WORKLOADS, make_params, round_bf16
from oracle.layer import layer_prefill as oracle_layer
from tests.gpu_util import assert_close, dims_of, oracle_dims

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(300, 520, 264), (1000, 1304, 512), (128, 256, 64), (7, 40, 8), (513, 2688, 4096)])
def test_projection_matches_fp32_matmul(M, N, K):
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g, device="cuda") / np.sqrt(K)).to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_projection(A, W, C, ws)
    ref = A.float() @ W.float().T
    torch.cuda.synchronize()
    assert sm.ssd_mixer_workspace_status(ws) == sm.SSD_OK
    assert_close("C", C, ref.cpu().numpy(), 1e-2)


def test_projection_writes_strided_output_only_inside_its_columns():
    M, N, K = 200, 296, 128
    g = torch.Generator(device="cuda").manual_seed(5)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    W = torch.randn(N, K, generator=g, device="cuda").to(torch.bfloat16)
    big = torch.zeros(M, N + 64, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    sm.ssd_mixer_projection(A, W, big[:, 32:32 + N], ws)
    torch.cuda.synchronize()
    assert_close("C", big[:, 32:32 + N], (A.float() @ W.float().T).cpu().numpy(), 1e-2)
    assert torch.all(big[:, :32] == 0) and torch.all(big[:, 32 + N:] == 0)


def _layer_case(heads, groups, seqlen, d_model, seed):
    w = WORKLOADS["small_bf16"].with_(batch=2, seqlen=seqlen, nheads=heads, ngroups=groups, init_ssm_std=0.1,
                                      init_conv_std=1.0, seed=seed)
    rng = np.random.default_rng(seed)
    prm = make_params(w, rng)
    HP, GN, H = w.d_inner, w.ngroups * w.dstate, w.nheads
    width = 2 * HP + 2 * GN + H
    hidden = round_bf16(rng.standard_normal((w.batch, w.seqlen, d_model)).astype(np.float32))
    W_in = round_bf16((rng.standard_normal((width, d_model)) / np.sqrt(d_model)).astype(np.float32))
    W_out = round_bf16((rng.standard_normal((d_model, HP)) / np.sqrt(HP)).astype(np.float32))
    init_ssm = (0.1 * rng.standard_normal((w.batch, H, w.headdim, w.dstate))).astype(np.float32)
    init_conv = round_bf16(rng.standard_normal((w.batch, w.xbc_channels, 3)).astype(np.float32))
    return w, prm, hidden, W_in, W_out, init_ssm, init_conv


@pytest.mark.parametrize("heads,groups,in_out_proj", [(8, 2, False), (16, 2, False), (16, 2, True)])
def test_layer_matches_layer_oracle(heads, groups, in_out_proj):
    w, prm, hidden, W_in, W_out, init_ssm, init_conv = _layer_case(heads, groups, 333, 256, seed=61 + heads)
    d = dims_of(w)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float().cuda()
    P = {k: f32(prm[k]) for k in ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")}
    out, fs, fc = sm.layer_prefill(d, bf(hidden), bf(W_in), bf(W_out), P["A"], P["D"], P["conv_w"], P["conv_b"],
                                   P["dt_bias"], P["norm_w"], f32(init_ssm), bf(init_conv), norm_in_out_proj=in_out_proj)
    torch.cuda.synchronize()
    ref_out, ref_fs, ref_fc = oracle_layer(oracle_dims(d), hidden, W_in.T, W_out.T, prm["A"], prm["D"], prm["conv_w"],
                                           prm["conv_b"], prm["dt_bias"], prm["norm_w"], init_ssm, init_conv)
    assert_close("layer out", out, ref_out, 2e-2)
    assert_close("final_ssm", fs, ref_fs, 2e-2)
    assert_close("final_conv", fc, ref_fc, 2e-2)
