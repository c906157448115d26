"""The context-parallel driver's multi-rank logic on CPU: two or three gloo ranks, each
holding one piece of a row, run hybrid_mamba_ssm_causal_b200.context_parallel with the
kernels replaced by the fp64 oracle; the pieces' outputs and the last rank's final states
must equal one oracle prefill over the whole row."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from hybrid_mamba_ssm_causal_b200 import context_parallel as cp
from hybrid_mamba_ssm_causal_b200 import ssd_mixer as sm

SEQ = ("x", "z", "B", "C", "dt")
PAR = ("A", "D", "conv_w", "conv_b", "dt_bias", "norm_w")


def odims(d):
    return oracle.Dims(d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)


def npy(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float64)


class OracleOps:
    """Stand-ins for the library's kernels (test infrastructure): the same four steps in fp64."""

    def conv_tail(self, d, piece, params):
        d3 = oracle.Dims(d.batch, 3, d.nheads, d.headdim, d.ngroups, d.dstate, d.dconv, d.eps)
        out = oracle.prefill(d3, *(npy(piece[k][:, -3:]) for k in SEQ), *(npy(params[k]) for k in PAR))
        return torch.from_numpy(out["final_conv"])

    def state(self, d, piece, params, ssm_in, conv_in):
        out = oracle.prefill(odims(d), *(npy(piece[k]) for k in SEQ), *(npy(params[k]) for k in PAR),
                             npy(ssm_in), npy(conv_in))
        a = oracle.decay(npy(piece["dt"]), npy(params["A"]), npy(params["dt_bias"]))
        return torch.from_numpy(a), torch.from_numpy(out["final_ssm"])

    def state_in(self, r, decays, states, init):
        h = np.zeros_like(npy(states[0])) if init is None else npy(init)
        for j in range(r):
            h = npy(decays[j])[:, :, None, None] * h + npy(states[j])
        return torch.from_numpy(h)

    def prefill(self, d, piece, params, ssm_in, conv_in):
        out = oracle.prefill(odims(d), *(npy(piece[k]) for k in SEQ), *(npy(params[k]) for k in PAR),
                             npy(ssm_in), npy(conv_in))
        return tuple(torch.from_numpy(out[k]) for k in ("y", "final_ssm", "final_conv"))


def problem(seed=7, b=2, lens=(23, 19), H=4, P=4, G=2, N=8):
    rng = np.random.default_rng(seed)
    L = sum(lens)
    Cc = H * P + 2 * G * N
    full = dict(x=rng.standard_normal((b, L, H * P)), z=rng.standard_normal((b, L, H * P)),
                B=rng.standard_normal((b, L, G * N)), C=rng.standard_normal((b, L, G * N)),
                dt=rng.standard_normal((b, L, H)))
    params = dict(A=-np.exp(rng.uniform(0, np.log(16), H)), D=rng.uniform(0, 1, H),
                  conv_w=rng.uniform(-0.5, 0.5, (Cc, 4)), conv_b=rng.uniform(-0.1, 0.1, Cc),
                  dt_bias=np.log(np.expm1(np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), H)))),
                  norm_w=1 + 0.1 * rng.standard_normal(H * P))
    init_ssm = 0.1 * rng.standard_normal((b, H, P, N))
    init_conv = rng.standard_normal((b, Cc, 3))
    return full, params, init_ssm, init_conv, (b, H, P, G, N)


def worker(rank, world, port, lens, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full, params, init_ssm, init_conv, (b, H, P, G, N) = problem(lens=lens)
        s0 = sum(lens[:rank])
        piece = {k: torch.from_numpy(full[k][:, s0:s0 + lens[rank]].copy()) for k in SEQ}
        par = {k: torch.from_numpy(v) for k, v in params.items()}
        d = sm.Dims(b, lens[rank], H, P, G, N, 64, 4, 1e-5, "f32")
        y, fs, fc = cp.context_parallel_prefill(d, piece, par, torch.from_numpy(init_ssm) if rank == 0 else None,
                                                torch.from_numpy(init_conv) if rank == 0 else None, ops=OracleOps())
        q.put((rank, y.numpy(), fs.numpy(), fc.numpy()))
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("lens", [(23, 19), (3, 40), (11, 7, 9)])
def test_gloo_ranks_match_one_prefill(lens):
    world = len(lens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, lens, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict()
    for _ in range(world):
        r, y, fs, fc = q.get(timeout=120)
        res[r] = (y, fs, fc)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full, params, init_ssm, init_conv, (b, H, P, G, N) = problem(lens=lens)
    ref = oracle.prefill(oracle.Dims(b, sum(lens), H, P, G, N, 4, 1e-5), *(full[k] for k in SEQ),
                         *(params[k] for k in PAR), init_ssm, init_conv)
    y = np.concatenate([res[r][0] for r in range(world)], axis=1)
    scale = np.max(np.abs(ref["y"]))
    assert np.max(np.abs(y - ref["y"])) <= 1e-10 * scale
    last = res[world - 1]
    assert np.max(np.abs(last[1] - ref["final_ssm"])) <= 1e-10 * np.max(np.abs(ref["final_ssm"]))
    assert np.array_equal(last[2], ref["final_conv"])


def test_pieces_need_three_tokens():
    with pytest.raises(ValueError):
        cp.check_pieces([5, 2])
