"""Test-only chunked backward pass in numpy: the reverse-time counterpart of
tests/chunked_ref.py, in the three-phase shape of the Flash PD-SSM page (Technical
Summary, Methodology 3) with the time direction reversed.

The adjoint Lam_t = dLoss/dH_t obeys Lam_t = Lam'_t + C_t dy_t^T and
Lam'_{t-1} = A_t^H Lam_t, a linear recurrence backwards in time whose transition
is the (conjugate) transpose of a column-one-hot matrix:
(A^H Lam)[j] = conj(val[j]) Lam[idx[j]], a gather. So it splits like the forward
scan (below, ^T stands for ^H when the state is complex):

  phase A'  per chunk [t0, t1), from a zero adjoint at the chunk end: the local
            adjoints Lam^loc_t and the chunk's outgoing local adjoint
            G_c = (A_{t0}^T ... ) part that reaches H_{t0-1};
  phase B'  a scan over the chunks in reverse: the adjoint entering chunk c from
            the future, In_c = dLoss/dH_{t1-1} from steps >= t1:
                In_{nC-1} = dh_final,  In_{c-1} = G_c + M_c^T In_c,
            with M_c = A_{t1-1} ... A_{t0} the chunk's pair;
  phase C'  Lam_t = Lam^loc_t + S_t^T In_c, S_t = A_{t1-1} ... A_{t+1} the
            suffix pair of the chunk after t.

The forward states H_{t-1} that the gradients need come from chunk-start states
(phase B of the forward scan) and a local recomputation inside each chunk. The
gradients are then those of the backward oracle (oracle/backward.py), which this
module does not import: it shares nothing with it (sparse index arithmetic here,
dense matrices there) and nothing with the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np

from tests.chunked_ref import apply_pair, compose, identity_pair


def apply_pair_T(pair, Lam):
    """Conjugate transpose of a column-one-hot matrix on rows: (M^H Lam)[j] = conj(val[j]) * Lam[idx[j]]
    (a gather; the plain transpose for real values)."""
    idx, val = pair
    return np.conj(val)[:, None] * Lam[idx]


def chunked_backward(logits, idx, d, B, C, x, dy, dh_final=None, h0=None, T=16, tau=1.0):
    """One slice; returns the gradients of Re[sum_t <dy_t, y_t> + <dh_final, H_{L-1}>]
    (gradient du + i dv for a complex z = u + i v, as oracle/backward.py)."""
    logits = np.asarray(logits, np.float64)
    L, K = logits.shape
    N, P = B.shape[1], x.shape[1]
    cplx = any(np.iscomplexobj(a) for a in (d, dy, dh_final, h0) if a is not None)
    cdt = np.complex128 if cplx else np.float64
    d, dy = np.asarray(d, cdt), np.asarray(dy, cdt)
    s = np.argmax(logits, axis=1)
    steps = [(idx[s[t]], d[t]) for t in range(L)]
    nC = max(1, math.ceil(L / T))
    bounds = [(c * T, min(L, (c + 1) * T)) for c in range(nC)]

    # forward: chunk-start states by the three-phase forward route (local states + carries)
    H_loc, pairs = [], []
    for t0, t1 in bounds:
        H = np.zeros((N, P), cdt)
        pair = identity_pair(N, cdt)
        for t in range(t0, t1):
            H = apply_pair(steps[t], H) + np.outer(B[t], x[t])
            pair = compose(steps[t], pair)
        H_loc.append(H)
        pairs.append(pair)
    H_start, car = [], (np.zeros((N, P), cdt) if h0 is None else np.asarray(h0, cdt))
    for c in range(nC):
        H_start.append(car)
        car = apply_pair(pairs[c], car) + H_loc[c]

    # phase A': local adjoints from a zero adjoint at each chunk end
    lam_loc, G = [], []
    for t0, t1 in bounds:
        lam = np.zeros((N, P), cdt)
        local = {}
        for t in range(t1 - 1, t0 - 1, -1):
            lam = lam + np.outer(C[t], dy[t])
            local[t] = lam
            lam = apply_pair_T(steps[t], lam)
        lam_loc.append(local)
        G.append(lam)
    # phase B': the adjoint entering each chunk from the future, in reverse chunk order
    In = [None] * nC
    cur = np.zeros((N, P), cdt) if dh_final is None else np.asarray(dh_final, cdt)
    for c in range(nC - 1, -1, -1):
        In[c] = cur
        cur = G[c] + apply_pair_T(pairs[c], cur)
    dh0 = cur

    out = {"dd": np.zeros((L, N), cdt), "dB": np.zeros((L, N)), "dC": np.zeros((L, N)), "dx": np.zeros((L, P)),
           "dlogits": np.zeros((L, K))}
    for c, (t0, t1) in enumerate(bounds):
        # forward states of the chunk, from its start state
        Hs = [H_start[c]]
        for t in range(t0, t1):
            Hs.append(apply_pair(steps[t], Hs[-1]) + np.outer(B[t], x[t]))
        # phase C': suffix pairs after t, applied transposed to the incoming adjoint
        suf = identity_pair(N, cdt)
        for t in range(t1 - 1, t0 - 1, -1):
            lam = lam_loc[c][t] + apply_pair_T(suf, In[c])
            Ht, Hp = Hs[t - t0 + 1], Hs[t - t0]
            out["dC"][t] = np.real(Ht @ np.conj(dy[t]))
            out["dB"][t] = np.real(lam @ x[t])
            out["dx"][t] = np.real(lam.T @ B[t])
            # sum_p Lam_t[idx_k[j]][p] conj(H_{t-1}[j][p]) for every entry k
            q = np.stack([np.einsum("jp,jp->j", lam[idx[k]], np.conj(Hp)) for k in range(K)])
            out["dd"][t] = q[s[t]]
            dpi = np.real(np.conj(q) @ d[t])
            z = logits[t] / tau
            e = np.exp(z - z.max())
            pit = e / e.sum()
            out["dlogits"][t] = pit * (dpi - pit @ dpi) / tau
            suf = compose(suf, steps[t])  # S_{t-1} = S_t A_t
    out["dh0"] = dh0
    out["s"] = s.astype(np.int32)
    return out
