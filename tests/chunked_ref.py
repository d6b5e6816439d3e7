"""Test-only chunked scan in numpy, used to pin the oracle's sequential result.

It takes the three-phase route the Flash PD-SSM page describes (Technical
Summary, Methodology 3: phase A = independent sequential recurrences inside
chunks, phase B = prefix scan over chunk dependencies for the carry states,
phase C = carry corrections) and combines chunks with the associative
composition of (index, value) pairs that the prefix-scan framing of the
Prefix-Scannable Models abstract calls for (state updates computed by a
parallel prefix scan with a custom associative operator).

It shares nothing with the oracle (sparse index arithmetic here, dense matrix
products there) and nothing with the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np


def compose(a, b):
    """(idx, val) o (idx', val') = (idx[idx'], val[idx'] * val'): the pair of A.A' (A' applied first)."""
    ia, va = a
    ib, vb = b
    return ia[ib], va[ib] * vb


def identity_pair(N, dtype=np.float64):
    return np.arange(N), np.ones(N, dtype=dtype)


def apply_pair(pair, H):
    """Rows of H moved by a column-one-hot matrix: H'[idx[j]] += val[j] * H[j]."""
    idx, val = pair
    out = np.zeros_like(H)
    np.add.at(out, idx, val[:, None] * H)
    return out


def chunked_scan(s, idx, d, B, C, x, h0, T):
    """One slice: s [L], idx [K,N], d/B/C [L,N], x [L,P], h0 [N,P] or None; chunk length T."""
    L, N = B.shape
    P = x.shape[1]
    cdt = np.result_type(d.dtype, np.float64)
    nC = max(1, math.ceil(L / T))
    y_loc = np.zeros((L, P), dtype=cdt)
    H_loc, pairs = [], []
    # phase A: local recurrence from zero in each chunk, plus the chunk's pair
    for c in range(nC):
        H = np.zeros((N, P), dtype=cdt)
        pair = identity_pair(N, cdt)
        for t in range(c * T, min(L, (c + 1) * T)):
            step = (idx[s[t]], d[t].astype(cdt))
            H = apply_pair(step, H) + np.outer(B[t], x[t])
            y_loc[t] = H.T @ C[t]
            pair = compose(step, pair)
        H_loc.append(H)
        pairs.append(pair)
    # phase B: carries
    H_in = []
    car = np.zeros((N, P), dtype=cdt) if h0 is None else h0.astype(cdt)
    total = identity_pair(N, cdt)
    for c in range(nC):
        H_in.append(car)
        car = apply_pair(pairs[c], car) + H_loc[c]
        total = compose(pairs[c], total)
    # phase C: y_t += H_in^T (Phi_t^T C_t), Phi_t = prefix pair from the chunk start
    y = y_loc.copy()
    for c in range(nC):
        pre = identity_pair(N, cdt)
        for t in range(c * T, min(L, (c + 1) * T)):
            pre = compose((idx[s[t]], d[t].astype(cdt)), pre)
            ct = pre[1] * C[t][pre[0]]
            y[t] += H_in[c].T @ ct
    return {"y": y, "h_final": car, "prod_idx": total[0], "prod_val": total[1]}
