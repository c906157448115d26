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
  to each chunk's outputs. The gllm PR #86 "Reference quirk" paragraph reports that
  one widely used pure-torch version of this form is off at the first token of every
  later chunk; the form here must match the sequential recurrence at every position,
  which the oracle tests check at positions k*Q.
* :func:`quadratic_scan` materialises the whole causal L x L mixing matrix
  M[i, j] = (C_i . B_j) * exp(sum_{k=j+1..i} delta_k A) * delta_j (the "dual",
  attention-like side of the duality) with every segment sum taken by a direct loop.
  It is O(L^3) and meant for tiny L only.
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
