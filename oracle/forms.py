"""Two further fp64 forms of the SSD scan, written separately from ssd_oracle.c.

TEST INFRASTRUCTURE ONLY (used to pin the oracle; see oracle/__init__.py).

Both take the scan's own inputs for ONE batch row, after the conv and softplus:
  xa [L, H, P]   activated x          Ba, Ca [L, G, N]   activated B and C
  delta [L, H]   softplus(dt + bias)  A, D [H]           H0 [H, P, N] (state in)
and return (y_pre [L, H, P], H_final [H, P, N]), where y_pre includes the D skip.
Head h reads group h // (H // G).

* :func:`chunked_scan` is the chunk-parallel "structured state-space duality"
  block decomposition that the Modalities PR #459 ("feat(model): add Nemotron-3 Nano
  hybrid Mamba-Transformer MoE architecture", commit notes on ssd.py) names: a
  within-chunk cumulative sum of the log-decays, an intra-chunk causal product, a
  per-chunk state, a sequential pass over chunk states, and the state's contribution
  to each chunk's outputs. The gllm PR #86 "Reference quirk" paragraph reports a
  pure-torch version of this form whose error appears where each chunk after the first
  begins; the form here must match the sequential recurrence at every position, which
  the oracle tests check at positions k*Q.
* :func:`quadratic_scan` materialises the whole causal L x L mixing matrix
  M[i, j] = (C_i . B_j) * exp(sum_{k=j+1..i} delta_k A) * delta_j (the "dual",
  attention-like side of the duality) with every segment sum taken by a direct loop.
  It is O(L^3) and meant for tiny L only.
* :func:`chunked_scan_vjp` is the backward pass of :func:`chunked_scan` written in the
  same block form (per chunk: products of the chunk's matrices with the decay mask, and
  a reverse pass over the states entering the chunks), for the tests to hold against the
  sequential backward in oracle/backward.py. The mixer is trained through this scan
  (Modalities PR #459, sections "Testing" and "Caveats").
"""
from __future__ import annotations

import numpy as np


def _group_of(H: int, G: int) -> np.ndarray:
    return np.arange(H) // (H // G)


def chunked_scan(xa, Ba, Ca, delta, A, D, H0, Q: int):
    xa, Ba, Ca, delta = (np.asarray(a, dtype=np.float64) for a in (xa, Ba, Ca, delta))
    A, D = np.asarray(A, np.float64), np.asarray(D, np.float64)
    L, H, P = xa.shape
    G, N = Ba.shape[1], Ba.shape[2]
    grp = _group_of(H, G)
    y = np.zeros((L, H, P))
    Hst = np.array(H0, dtype=np.float64, copy=True)  # state entering the current chunk
    for c0 in range(0, L, Q):
        c1 = min(c0 + Q, L)
        for h in range(H):
            g = grp[h]
            a = delta[c0:c1, h] * A[h]                     # log-decays of the chunk
            lam = np.cumsum(a)                              # inclusive in-chunk prefix sums
            Xc, Bc, Cc = xa[c0:c1, h, :], Ba[c0:c1, g, :], Ca[c0:c1, g, :]
            dl = delta[c0:c1, h]
            # intra-chunk: (C B^T) masked by exp(lam_i - lam_j) for j <= i, times delta_j
            seg = lam[:, None] - lam[None, :]
            mask = np.tril(np.ones((c1 - c0, c1 - c0), dtype=bool))
            decay = np.where(mask, np.exp(np.where(mask, seg, 0.0)), 0.0)
            M = (Cc @ Bc.T) * decay * dl[None, :]
            y[c0:c1, h, :] += M @ Xc
            # state entering the chunk, decayed to each position (includes a_i itself)
            y[c0:c1, h, :] += np.exp(lam)[:, None] * (Cc @ Hst[h].T)
            # chunk state and hand-off to the next chunk
            w = np.exp(lam[-1] - lam) * dl                  # weight of token j at chunk end
            S = (Xc * w[:, None]).T @ Bc                    # [P, N]
            Hst[h] = np.exp(lam[-1]) * Hst[h] + S
    y += D[None, :, None] * xa
    return y, Hst


def quadratic_scan(xa, Ba, Ca, delta, A, D, H0):
    xa, Ba, Ca, delta = (np.asarray(a, dtype=np.float64) for a in (xa, Ba, Ca, delta))
    A, D = np.asarray(A, np.float64), np.asarray(D, np.float64)
    L, H, P = xa.shape
    G, N = Ba.shape[1], Ba.shape[2]
    grp = _group_of(H, G)
    H0 = np.asarray(H0, dtype=np.float64)
    y = np.zeros((L, H, P))
    Hf = np.zeros((H, P, N))
    for h in range(H):
        g = grp[h]
        a = delta[:, h] * A[h]

        def segsum(j0: int, i: int) -> float:       # sum of a[k] for j0 <= k <= i, by loop
            s = 0.0
            for k in range(j0, i + 1):
                s += a[k]
            return s

        M = np.zeros((L, L))
        for i in range(L):
            for j in range(i + 1):
                M[i, j] = float(Ca[i, g] @ Ba[j, g]) * np.exp(segsum(j + 1, i)) * delta[j, h]
        y[:, h, :] = M @ xa[:, h, :]
        for i in range(L):
            y[i, h, :] += np.exp(segsum(0, i)) * (H0[h] @ Ca[i, g])
        acc = np.exp(segsum(0, L - 1)) * H0[h]
        for j in range(L):
            acc = acc + np.exp(segsum(j + 1, L - 1)) * delta[j, h] * np.outer(xa[j, h], Ba[j, g])
        Hf[h] = acc
    y += D[None, :, None] * xa
    return y, Hf


def chunked_scan_vjp(xa, Ba, Ca, delta, A, D, H0, dy, dH_final, Q: int):
    """Gradients of sum(dy * y_pre) + sum(dH_final * H_final) through :func:`chunked_scan`.

    Per chunk (local tokens i, j; lam the inclusive cumsum of a = delta A; u_j = delta_j x_j;
    W_ij = exp(lam_i - lam_j) for j <= i; K_ij = C_i . B_j; G the gradient of the state
    leaving the chunk, H the state entering it):
      y_i      = sum_j K_ij W_ij u_j + exp(lam_i) H C_i + D x_i
      H_next   = exp(lam_end) H + sum_j exp(lam_end - lam_j) u_j B_j^T
    so  du_j   = sum_i K_ij W_ij dy_i + exp(lam_end - lam_j) G B_j
        dC_i   = sum_j W_ij (dy_i . u_j) B_j + exp(lam_i) H^T dy_i
        dB_j   = sum_i W_ij (dy_i . u_j) C_i + exp(lam_end - lam_j) G^T u_j
        dlam_i = sum_j K_ij W_ij (dy_i . u_j) - sum_k K_ki W_ki (dy_k . u_i)
                 + exp(lam_i) dy_i . (H C_i) - exp(lam_end - lam_i) u_i^T G B_i
                 + [i = end] (exp(lam_end) <G, H> + sum_j exp(lam_end - lam_j) u_j^T G B_j)
        da_k   = sum_{i >= k} dlam_i,  ddelta = du . x + A da,  dA = sum delta da,
        dH     = exp(lam_end) G + sum_i exp(lam_i) dy_i C_i^T   (the previous chunk's G).
    Shapes as :func:`chunked_scan`; dy [L, H, P]; dH_final [H, P, N] or None.
    Returns (dxa [L, H, P], dBa [L, G, N], dCa [L, G, N], ddelta [L, H], dA [H], dD [H],
    dH0 [H, P, N])."""
    xa, Ba, Ca, delta, dy = (np.asarray(a, dtype=np.float64) for a in (xa, Ba, Ca, delta, dy))
    A, D = np.asarray(A, np.float64), np.asarray(D, np.float64)
    L, H, P = xa.shape
    G, N = Ba.shape[1], Ba.shape[2]
    grp = _group_of(H, G)
    starts = list(range(0, L, Q))
    # the state entering every chunk, per head
    Hin = np.zeros((len(starts) + 1, H, P, N))
    Hin[0] = np.asarray(H0, dtype=np.float64)
    for c, c0 in enumerate(starts):
        c1 = min(c0 + Q, L)
        for h in range(H):
            g = grp[h]
            lam = np.cumsum(delta[c0:c1, h] * A[h])
            u = delta[c0:c1, h][:, None] * xa[c0:c1, h, :]
            S = (u * np.exp(lam[-1] - lam)[:, None]).T @ Ba[c0:c1, g, :]
            Hin[c + 1, h] = np.exp(lam[-1]) * Hin[c, h] + S
    dxa, ddelta = np.zeros((L, H, P)), np.zeros((L, H))
    dBa, dCa = np.zeros((L, G, N)), np.zeros((L, G, N))
    dA, dD = np.zeros(H), np.sum(dy * xa, axis=(0, 2))
    Gs = np.zeros((H, P, N)) if dH_final is None else np.array(dH_final, dtype=np.float64)
    for c in range(len(starts) - 1, -1, -1):
        c0 = starts[c]
        c1 = min(c0 + Q, L)
        q = c1 - c0
        mask = np.tril(np.ones((q, q), dtype=bool))
        for h in range(H):
            g = grp[h]
            Xc, Bc, Cc, dYc = xa[c0:c1, h, :], Ba[c0:c1, g, :], Ca[c0:c1, g, :], dy[c0:c1, h, :]
            dl = delta[c0:c1, h]
            lam = np.cumsum(dl * A[h])
            u = dl[:, None] * Xc
            Hc, Gc = Hin[c, h], Gs[h]
            W = np.where(mask, np.exp(np.where(mask, lam[:, None] - lam[None, :], 0.0)), 0.0)
            K = Cc @ Bc.T
            dyu = dYc @ u.T                                   # [i, j] = dy_i . u_j
            e_i, e_end, e_rest = np.exp(lam), np.exp(lam[-1]), np.exp(lam[-1] - lam)
            GB = Bc @ Gc.T                                    # [j] = G B_j
            du = (K * W).T @ dYc + e_rest[:, None] * GB
            dxa[c0:c1, h, :] = dl[:, None] * du + D[h] * dYc
            dK = W * dyu
            dCa[c0:c1, g, :] += dK @ Bc + e_i[:, None] * (dYc @ Hc)
            dBa[c0:c1, g, :] += dK.T @ Cc + e_rest[:, None] * (u @ Gc)
            T = K * W * dyu
            uGB = np.sum(u * GB, axis=1)                      # [j] = u_j^T G B_j
            dlam = T.sum(axis=1) - T.sum(axis=0) + e_i * np.sum(dYc * (Cc @ Hc.T), axis=1) - e_rest * uGB
            dlam[-1] += e_end * np.sum(Gc * Hc) + np.sum(e_rest * uGB)
            da = np.cumsum(dlam[::-1])[::-1]
            ddelta[c0:c1, h] = np.sum(du * Xc, axis=1) + A[h] * da
            dA[h] += np.sum(dl * da)
            Gs[h] = e_end * Gc + (dYc * e_i[:, None]).T @ Cc
    return dxa, dBa, dCa, ddelta, dA, dD, Gs
