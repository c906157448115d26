"""Context-parallel prefill: one long row split into pieces, one piece per rank.

The long-context phase needs the sequence split across GPUs, with the Mamba state handed
from piece to piece (Modalities PR #459, section "Next steps for production at scale", item
"MTP and long-context"). The same PR tests a state carried over between the parts of a
split sequence (section "Testing"). A
prefill's final state is linear in its initial state, so the pieces can run side by side:

  1. each rank runs a 3-token prefill of its piece's last raw tokens to get the conv state its
     successor starts from (the final conv state is the last K-1 raw inputs);
  2. the conv states are all-gathered; rank r starts from rank r-1's (rank 0 from the given
     initial conv state);
  3. each rank runs the state-only pass over its piece, from the row's initial SSM state on
     rank 0 and from a zero state elsewhere, getting its final state S_r and decay a_r
     (ssd_mixer_prefill_state);
  4. (a, S) are all-gathered, and rank r folds pieces 0..r-1 into the state entering its piece
     (ssd_mixer_state_pass: H_in(j+1) = a_j H_in(j) + S_j from H_in(0) = 0, S_0 carrying the
     initial state);
  5. each rank runs the full prefill of its piece from those states (ssd_mixer_prefill).

The last rank's final states are the row's final states. Every arithmetic step runs in the
library's kernels; this module slices views, calls the collectives and the C ABI. The
state-only pass runs on the tensor-core kernel, so the shapes are its own: bf16
activations, P = 64, N = 128, 2 or a multiple of 4 heads per group (other shapes raise
SsdError with SSD_ERR_UNSUPPORTED). The three
phases are separate functions, so a single process can also run the ranks one phase at a
time (the collectives are then plain lists).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

from . import ssd_mixer as sm

SEQ = ("x", "z", "B", "C", "dt")


@dataclass
class PieceState:
    conv_tail: torch.Tensor     # [b, Cc, K-1]: this piece's last raw inputs (successor's conv start)
    conv_in: torch.Tensor | None = None
    decay: torch.Tensor | None = None       # [b, H]
    zero_state: torch.Tensor | None = None  # [b, H, P, N]


class CudaOps:
    """The library's kernels through the C ABI (the default)."""

    def conv_tail(self, d: sm.Dims, piece: dict, params: dict) -> torch.Tensor:
        K1 = d.dconv - 1
        dt3 = replace(d, seqlen=K1)
        tail = {k: piece[k][:, -K1:] for k in SEQ}
        dev = piece["x"].device
        fs = torch.empty(d.batch, d.nheads, d.headdim, d.dstate, device=dev)
        fc = torch.empty(d.batch, d.xbc_channels, K1, dtype=d.torch_dtype, device=dev)
        ws = torch.empty(max(sm.ssd_mixer_prefill_state_workspace_size(dt3), 256), dtype=torch.uint8, device=dev)
        sm.ssd_mixer_prefill_state(dt3, *(tail[k].contiguous() for k in ("x", "B", "C", "dt")), params["A"],
                                   params["conv_w"], params["conv_b"], params["dt_bias"], None, None, fs, fc, None, ws)
        return fc

    def state(self, d: sm.Dims, piece: dict, params: dict, ssm_in, conv_in):
        dev = piece["x"].device
        fs = torch.empty(d.batch, d.nheads, d.headdim, d.dstate, device=dev)
        fc = torch.empty(d.batch, d.xbc_channels, d.dconv - 1, dtype=d.torch_dtype, device=dev)
        a = torch.empty(d.batch, d.nheads, device=dev)
        ws = torch.empty(max(sm.ssd_mixer_prefill_state_workspace_size(d), 256), dtype=torch.uint8, device=dev)
        sm.ssd_mixer_prefill_state(d, piece["x"], piece["B"], piece["C"], piece["dt"], params["A"], params["conv_w"],
                                   params["conv_b"], params["dt_bias"], ssm_in, conv_in, fs, fc, a, ws)
        return a, fs

    def state_in(self, r: int, decays: torch.Tensor, states: torch.Tensor, init):
        out = torch.empty_like(states[0])
        sm.ssd_mixer_state_pass(r, decays, states, init, out)
        return out

    def prefill(self, d: sm.Dims, piece: dict, params: dict, ssm_in, conv_in):
        return sm.prefill(d, *(piece[k] for k in SEQ), *(params[k] for k in
                          ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")), ssm_in, conv_in)


def check_pieces(lengths) -> None:
    """Every piece must hold at least K-1 = 3 tokens: a piece's final conv state is then its
    own last raw inputs, whatever it started from."""
    if any(n < 3 for n in lengths):
        raise ValueError("context-parallel pieces need at least 3 tokens each")


def phase1(d: sm.Dims, piece: dict, params: dict, ops=None) -> PieceState:
    """Step 1: the conv state this piece hands to its successor."""
    ops = ops or CudaOps()
    return PieceState(conv_tail=ops.conv_tail(d, piece, params))


def phase2(r: int, st: PieceState, tails: list, d: sm.Dims, piece: dict, params: dict, init_ssm, init_conv,
           ops=None) -> PieceState:
    """Steps 2-3: this piece's initial conv state, its final state from the row's initial
    state (rank 0) or from zero (other ranks), and its decay."""
    ops = ops or CudaOps()
    st.conv_in = init_conv if r == 0 else tails[r - 1]
    st.decay, st.zero_state = ops.state(d, piece, params, init_ssm if r == 0 else None, st.conv_in)
    return st


def phase3(r: int, st: PieceState, decays: list, states: list, d: sm.Dims, piece: dict, params: dict,
           init_ssm, ops=None):
    """Steps 4-5: the state entering this piece, then its full prefill.
    Returns (y, final_ssm, final_conv) of this piece."""
    ops = ops or CudaOps()
    ssm_in = ops.state_in(r, torch.stack(decays), torch.stack(states), None) if r > 0 else init_ssm
    return ops.prefill(d, piece, params, ssm_in, st.conv_in)


def context_parallel_prefill(d: sm.Dims, piece: dict, params: dict, init_ssm=None, init_conv=None,
                             group=None, ops=None):
    """Run this rank's piece of a context-parallel prefill (torch.distributed must be
    initialised; rank r holds piece r, d.seqlen is this piece's length). init_ssm and
    init_conv are the row's initial states (read on rank 0 only). Returns this piece's
    (y, final_ssm, final_conv); the last rank's final states are the row's."""
    import torch.distributed as dist
    r, world = dist.get_rank(group), dist.get_world_size(group)
    check_pieces([d.seqlen])

    def gather(t):
        out = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(out, t.contiguous(), group=group)
        return out

    st = phase1(d, piece, params, ops)
    st = phase2(r, st, gather(st.conv_tail), d, piece, params, init_ssm if r == 0 else None,
                init_conv if r == 0 else None, ops)
    decays, states = gather(st.decay), gather(st.zero_state)
    return phase3(r, st, decays, states, d, piece, params, init_ssm, ops)
