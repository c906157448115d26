"""Backward pass of the mixer core in fp64 (TEST INFRASTRUCTURE ONLY).

Only tests/ may import this module. It shares no code with the CUDA library.

The mixer is trained through its scan, and gradient flow through it is one of the checks
that the pages run on it (Modalities PR #459, sections "Testing" and "Caveats"). This module
gives the vector-Jacobian product of the mixer core: given the forward's inputs and the
gradients of a scalar loss with respect to its outputs (``dout`` for y, optionally
``dfinal_ssm`` and ``dfinal_conv`` for the final states), it returns the gradients with
respect to every input, parameter and initial state. Each step is the chain rule applied
to one step of the forward's definition, taken in reverse order:

  forward step                                          its vector-Jacobian product
  s = [init_conv ; x|B|C], v_t = conv_b + sum_k w_k s_{t+k}, xBC' = SiLU(v)   conv_silu_vjp
  delta = softplus(dt + dt_bias)                                               softplus_vjp
  H_t = exp(delta_t A) H_{t-1} + delta_t x'_t (x) B'_t,  y_t = H_t C'_t + D x'_t   scan_vjp
  g = y SiLU(z), out = g / sqrt(mean over the group of g^2 + eps) * norm_w     gated_norm_vjp

The forward here (:func:`forward_saved`) is a plain numpy restatement of the same
definition that keeps every intermediate (all states H_t); the tests check it against the
compiled oracle, and check every gradient against central finite differences of the
compiled oracle along random directions.
"""
from __future__ import annotations

import numpy as np

K = 4  # conv width


def sigmoid(u):
    return 0.5 * (1.0 + np.tanh(0.5 * u))


def silu(u):
    return u * sigmoid(u)


def dsilu(u):
    """d/du [u sigmoid(u)] = sigmoid(u) (1 + u (1 - sigmoid(u)))."""
    sg = sigmoid(u)
    return sg * (1.0 + u * (1.0 - sg))


def softplus(u):
    return np.maximum(u, 0.0) + np.log1p(np.exp(-np.abs(u)))


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def forward_saved(d, x, z, B, C, dt, A, D, conv_w, conv_b, dt_bias, norm_w, init_ssm=None, init_conv=None):
    """The forward of the mixer core, keeping what the backward needs.

    Shapes as in oracle.prefill: x, z [b, L, H*P]; B, C [b, L, G*N]; dt [b, L, H]; A, D,
    dt_bias [H]; conv_w [Cc, 4]; conv_b [Cc]; norm_w [H*P]; init_ssm [b, H, P, N];
    init_conv [b, Cc, 3] (oldest first). Head h reads group h // (H/G).
    """
    x, z, B, C, dt = (_f64(a) for a in (x, z, B, C, dt))
    A, D, conv_w, conv_b, dt_bias, norm_w = (_f64(a) for a in (A, D, conv_w, conv_b, dt_bias, norm_w))
    b, L, H, P, G, N = d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate
    HP, GN = H * P, G * N
    Cc = HP + 2 * GN
    grp = np.arange(H) // (H // G)
    # conv over s = [initial conv state ; raw inputs], tap K-1 on the current token
    u = np.concatenate([x, B, C], axis=2)
    s0 = np.zeros((b, K - 1, Cc)) if init_conv is None else _f64(init_conv).transpose(0, 2, 1)
    s = np.concatenate([s0, u], axis=1)
    v = conv_b + sum(conv_w[:, k] * s[:, k:k + L] for k in range(K))
    xbc = silu(v)
    xs = xbc[..., :HP].reshape(b, L, H, P)
    Bh = xbc[..., HP:HP + GN].reshape(b, L, G, N)[:, :, grp]
    Ch = xbc[..., HP + GN:].reshape(b, L, G, N)[:, :, grp]
    delta = softplus(dt + dt_bias)
    # the recurrence, every state kept: Hs[:, t] is the state after t tokens
    Hs = np.zeros((b, L + 1, H, P, N))
    if init_ssm is not None:
        Hs[:, 0] = _f64(init_ssm)
    for t in range(L):
        a = np.exp(delta[:, t] * A)
        Hs[:, t + 1] = (a[:, :, None, None] * Hs[:, t]
                        + delta[:, t, :, None, None] * xs[:, t, :, :, None] * Bh[:, t, :, None, :])
    y = np.einsum("blhpn,blhn->blhp", Hs[:, 1:], Ch) + D[None, None, :, None] * xs
    y = y.reshape(b, L, HP)
    gate = y * silu(z)
    gs = HP // G
    rr = 1.0 / np.sqrt(np.mean(gate.reshape(b, L, G, gs) ** 2, axis=-1) + d.eps)
    out = (gate.reshape(b, L, G, gs) * rr[..., None]).reshape(b, L, HP) * norm_w
    return {"out": out, "final_ssm": Hs[:, L].copy(), "final_conv": s[:, L:L + K - 1].transpose(0, 2, 1).copy(),
            "s": s, "v": v, "xs": xs, "Bh": Bh, "Ch": Ch, "delta": delta, "Hs": Hs, "y": y, "grp": grp}


def gated_norm_vjp(y, z, norm_w, G, eps, dout):
    """out = g r norm_w with g = y SiLU(z) and r = (mean over the group of g^2 + eps)^(-1/2).
    d out_i / d g_j = norm_w_i (r [i = j] - r^3 g_i g_j / gs), so
    dg_j = r norm_w_j dout_j - (r^3 / gs) g_j sum_i norm_w_i dout_i g_i.
    Returns (dy, dz, dnorm_w)."""
    b, L, HP = y.shape
    gs = HP // G
    sil = silu(z)
    g = (y * sil).reshape(b, L, G, gs)
    r = 1.0 / np.sqrt(np.mean(g * g, axis=-1) + eps)
    wd = (dout * norm_w).reshape(b, L, G, gs)
    dot = np.sum(wd * g, axis=-1)
    dg = r[..., None] * wd - (r ** 3 / gs)[..., None] * g * dot[..., None]
    dg = dg.reshape(b, L, HP)
    dnorm_w = np.sum(dout * (g * r[..., None]).reshape(b, L, HP), axis=(0, 1))
    return dg * sil, dg * y * dsilu(z), dnorm_w


def scan_vjp(Hs, xs, Bh, Ch, delta, A, D, dy, dfinal_ssm=None):
    """The recurrence run backwards. With Gt the gradient with respect to H_t (the state
    after token t), starting from dfinal_ssm:
      Gt += dy_t (x) C'_t                           (y_t = H_t C'_t + D x'_t)
      dC'_t = H_t^T dy_t,  dx'_t = delta_t Gt B'_t + D dy_t,  dB'_t = delta_t Gt^T x'_t
      ddelta_t = A a_t <Gt, H_{t-1}> + <Gt, x'_t (x) B'_t>,  dA += delta_t a_t <Gt, H_{t-1}>
      G_{t-1} = a_t Gt                              (a_t = exp(delta_t A))
    B' and C' are per head here (Bh, Ch); the caller sums them over a group's heads.
    Returns (dxs, dBh, dCh, ddelta, dA, dD, dinit_ssm)."""
    b, L1, H, P, N = Hs.shape
    L = L1 - 1
    Gt = np.zeros((b, H, P, N)) if dfinal_ssm is None else np.array(dfinal_ssm, dtype=np.float64)
    dxs = np.zeros((b, L, H, P))
    dBh = np.zeros((b, L, H, N))
    dCh = np.zeros((b, L, H, N))
    ddelta = np.zeros((b, L, H))
    dA = np.zeros(H)
    dD = np.sum(dy * xs, axis=(0, 1, 3))
    for t in range(L - 1, -1, -1):
        Gt = Gt + dy[:, t, :, :, None] * Ch[:, t, :, None, :]
        dCh[:, t] = np.einsum("bhpn,bhp->bhn", Hs[:, t + 1], dy[:, t])
        a = np.exp(delta[:, t] * A)
        gh = np.einsum("bhpn,bhpn->bh", Gt, Hs[:, t])
        gxb = np.einsum("bhpn,bhp,bhn->bh", Gt, xs[:, t], Bh[:, t])
        ddelta[:, t] = A * a * gh + gxb
        dA += np.sum(delta[:, t] * a * gh, axis=0)
        dxs[:, t] = delta[:, t, :, None] * np.einsum("bhpn,bhn->bhp", Gt, Bh[:, t]) + D[None, :, None] * dy[:, t]
        dBh[:, t] = delta[:, t, :, None] * np.einsum("bhpn,bhp->bhn", Gt, xs[:, t])
        Gt = a[:, :, None, None] * Gt
    return dxs, dBh, dCh, ddelta, dA, dD, Gt


def softplus_vjp(dt, dt_bias, ddelta):
    """delta = softplus(dt + dt_bias): d delta / d dt = sigmoid(dt + dt_bias).
    Returns (ddt, ddt_bias)."""
    ddt = ddelta * sigmoid(_f64(dt) + _f64(dt_bias))
    return ddt, np.sum(ddt, axis=(0, 1))


def conv_silu_vjp(s, v, conv_w, dxbc, dfinal_conv=None):
    """xBC' = SiLU(v), v_t = conv_b + sum_k w_k s_{t+k}, final_conv = s_{L..L+2}.
    ds_j = sum_k w_k dv_{j-k} (+ dfinal_conv on the last three positions); the raw inputs'
    gradient is ds_{3..L+2}, the initial conv state's ds_{0..2}.
    Returns (du, dconv_w, dconv_b, dinit_conv)."""
    b, L, Cc = v.shape
    dv = dxbc * dsilu(v)
    ds = np.zeros((b, L + K - 1, Cc))
    for k in range(K):
        ds[:, k:k + L] += conv_w[:, k] * dv
    if dfinal_conv is not None:
        ds[:, L:L + K - 1] += _f64(dfinal_conv).transpose(0, 2, 1)
    dconv_w = np.stack([np.sum(dv * s[:, k:k + L], axis=(0, 1)) for k in range(K)], axis=1)
    dconv_b = np.sum(dv, axis=(0, 1))
    return ds[:, K - 1:], dconv_w, dconv_b, ds[:, :K - 1].transpose(0, 2, 1).copy()


def prefill_vjp(d, inp: dict, dout, dfinal_ssm=None, dfinal_conv=None) -> dict:
    """Gradients of sum(dout * y) + sum(dfinal_ssm * final_ssm) + sum(dfinal_conv * final_conv)
    with respect to every entry of ``inp`` (keys as in oracle.prefill_dict). The gradients
    of the initial states are returned whether or not the states were given (zeros stand in
    for missing ones)."""
    b, L, H, P, G, N = d.batch, d.seqlen, d.nheads, d.headdim, d.ngroups, d.dstate
    HP, GN = H * P, G * N
    A, D, conv_w = _f64(inp["A"]), _f64(inp["D"]), _f64(inp["conv_w"])
    f = forward_saved(d, inp["x"], inp["z"], inp["B"], inp["C"], inp["dt"], A, D, conv_w, inp["conv_b"],
                      inp["dt_bias"], inp["norm_w"], inp.get("init_ssm"), inp.get("init_conv"))
    dy, dz, dnorm_w = gated_norm_vjp(f["y"], _f64(inp["z"]), _f64(inp["norm_w"]), G, d.eps, _f64(dout))
    dxs, dBh, dCh, ddelta, dA, dD, dinit_ssm = scan_vjp(f["Hs"], f["xs"], f["Bh"], f["Ch"], f["delta"], A, D,
                                                        dy.reshape(b, L, H, P), dfinal_ssm)
    r = H // G
    dBs = dBh.reshape(b, L, G, r, N).sum(axis=3)
    dCs = dCh.reshape(b, L, G, r, N).sum(axis=3)
    ddt, ddt_bias = softplus_vjp(inp["dt"], inp["dt_bias"], ddelta)
    dxbc = np.concatenate([dxs.reshape(b, L, HP), dBs.reshape(b, L, GN), dCs.reshape(b, L, GN)], axis=2)
    du, dconv_w, dconv_b, dinit_conv = conv_silu_vjp(f["s"], f["v"], conv_w, dxbc, dfinal_conv)
    return {"x": du[..., :HP], "z": dz, "B": du[..., HP:HP + GN], "C": du[..., HP + GN:], "dt": ddt,
            "A": dA, "D": dD, "conv_w": dconv_w, "conv_b": dconv_b, "dt_bias": ddt_bias, "norm_w": dnorm_w,
            "init_ssm": dinit_ssm, "init_conv": dinit_conv}
