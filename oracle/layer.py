"""The whole Mamba-2 mixer layer in fp64: in_proj, the mixer core, out_proj (TEST
INFRASTRUCTURE ONLY; only tests/ may import this module).

The layer's input projection emits one packed row per token, split as [z | x | B | C | dt]
(gllm PR #86, section "2. feat(model): Nemotron-H on the CPU", "Supporting changes", on the
in_proj output [z | xBC | dt]; Modalities PR #459, commit notes on mamba2.py, on the packed
[z, x, B, C, dt] layout). The core (oracle.prefill) maps x, z, B, C, dt to y, and the output
projection maps y back to the model width. This is the computation that fusing the
projections with the core has to reproduce.
"""
from __future__ import annotations

import numpy as np

from . import prefill


def split_in_proj(d, zxbcdt):
    """[b, L, 2 HP + 2 GN + H] -> z, x, B, C, dt in that order."""
    HP, GN, H = d.nheads * d.headdim, d.ngroups * d.dstate, d.nheads
    edges = np.cumsum([0, HP, HP, GN, GN, H])
    if zxbcdt.shape[-1] != edges[-1]:
        raise ValueError(f"in_proj width {zxbcdt.shape[-1]} != {edges[-1]}")
    return tuple(zxbcdt[..., edges[k]:edges[k + 1]] for k in range(5))


def layer_prefill(d, u, W_in, W_out, A, D, conv_w, conv_b, dt_bias, norm_w, init_ssm=None, init_conv=None):
    """u [b, L, d_model] -> (out [b, L, d_model], final_ssm, final_conv).

    W_in [d_model, 2 HP + 2 GN + H] and W_out [HP, d_model]: out = core(split(u W_in)) W_out."""
    u = np.asarray(u, dtype=np.float64)
    zxbcdt = u @ np.asarray(W_in, dtype=np.float64)
    z, x, B, C, dt = split_in_proj(d, zxbcdt)
    core = prefill(d, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w, init_ssm, init_conv)
    out = core["y"] @ np.asarray(W_out, dtype=np.float64)
    return out, core["final_ssm"], core["final_conv"]
