"""Backward pass of the Flash PD-SSM forward pass -- dense CPU oracle.

TEST INFRASTRUCTURE ONLY: the tests are the only callers. It shares no code
with the CUDA path and never stands in for it.

What it computes (plain, slow and literal, in fp64 / complex128; per slice):

  Forward, as the forward oracle (Flash PD-SSM page, Technical Summary,
  Methodology 1 and 2): s_t = argmax_k logits_t[k] (lowest k on ties),
  A_t = P_{s_t} diag(d_t) with P_k[idx[k][j]][j] = 1, H_t = A_t H_{t-1} + B_t x_t^T
  (H_{-1} = h0 or 0), y_t = H_t^T C_t. Every H_t is kept.

  Loss: the caller's upstream gradients dy_t (of y_t) and dh_final (of H_{L-1}),
  i.e. the gradients are those of  Re[ sum_t <dy_t, y_t> + <dh_final, H_{L-1}> ]
  with <a, b> = sum conj(a) b. For a complex quantity z = u + i v the gradient is
  dLoss/du + i dLoss/dv (the convention of PyTorch's complex autograd); for real
  states every conjugate and real part below is the identity.

  Gradients of d, B, C, x and h0 are the exact derivatives of the forward (the
  hard selection does not depend on them). With Lam_t = dLoss/dH_t, taken from
  t = L-1 down to 0:
      Lam_t    = Lam'_t + C_t dy_t^T          Lam'_{L-1} = dh_final
      dC_t     = Re(H_t conj(dy_t))
      dB_t     = Re(Lam_t x_t),  dx_t = Re(Lam_t^T B_t)
      dA_t     = Lam_t H_{t-1}^H                    (dense N x N)
      dd_t[j]  = dA_t[idx_{s_t}[j]][j]
      Lam'_{t-1} = A_t^H Lam_t,  dh0 = Lam'_{-1}

  Logits (Methodology 2, "Gradient Propagation": straight-through estimator
  with a tempered softmax). Reading: the step's transition is the mixture
  A_t = sum_k pi_k(t) P_k diag(d_t) whose weights are the one-hot pi(t) of s_t
  in the forward pass; the backward pass takes the gradient with respect to
  the weights at that point,
      dpi_t[k] = Re <dA_t, P_k diag(d_t)> = Re sum_j conj(dA_t[idx_k[j]][j]) d_t[j],
  and passes it through the Jacobian of the tempered softmax
  pit_t = softmax(logits_t / tau) in place of the argmax:
      dlogits_t = (diag(pit_t) - pit_t pit_t^T) dpi_t / tau.
  The temperature tau (annealed by the caller, "slope annealing") is an
  argument. The pages print no formula for this surrogate (their Proposition 2
  is not reproduced); this is the plainest reading of their words.

Arrays are slice-major like the forward oracle's: logits [S][L][K],
d/B/C [S][L][N], x/dy [S][L][P], h0/dh_final [S][N][P].
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _dense_P(idx_k: np.ndarray) -> np.ndarray:
    """P_k[idx[k][j]][j] = 1: one nonzero per column (the one-hot column selector)."""
    N = idx_k.shape[0]
    P = np.zeros((N, N))
    P[idx_k, np.arange(N)] = 1.0
    return P


def _select(row: np.ndarray) -> int:
    """Hard argmax, lowest index on ties (no NaN handling needed for the backward's inputs)."""
    return int(np.argmax(row))


def _softmax(v: np.ndarray) -> np.ndarray:
    e = np.exp(v - v.max())
    return e / e.sum()


def slice_backward(logits, idx, d, B, C, x, dy, dh_final=None, h0=None, tau: float = 1.0) -> Dict[str, np.ndarray]:
    """Gradients of one (batch, head) slice; arrays [L][*] (fp64), idx [K][N]."""
    logits = np.asarray(logits, np.float64)
    idx = np.asarray(idx, np.int64)
    cplx = any(np.iscomplexobj(a) for a in (d, dy, dh_final, h0) if a is not None)
    cdt = np.complex128 if cplx else np.float64
    d, dy = np.asarray(d, cdt), np.asarray(dy, cdt)
    B, C, x = (np.asarray(a, np.float64) for a in (B, C, x))
    L, K = logits.shape
    N = B.shape[1]
    P = x.shape[1]
    Pk = [_dense_P(idx[k]) for k in range(K)]
    s = [_select(logits[t]) for t in range(L)]
    A = [Pk[s[t]] @ np.diag(d[t]) for t in range(L)]

    # forward, keeping every state (H[t + 1] is H_t; H[0] is H_{-1})
    H = [np.zeros((N, P), cdt) if h0 is None else np.asarray(h0, cdt).copy()]
    for t in range(L):
        H.append(A[t] @ H[-1] + np.outer(B[t], x[t]))

    out = {k: np.zeros_like(v) for k, v in (("dd", d), ("dB", B), ("dC", C), ("dx", x))}
    out["dlogits"] = np.zeros_like(logits)
    lam = np.zeros((N, P), cdt) if dh_final is None else np.asarray(dh_final, cdt).copy()
    for t in range(L - 1, -1, -1):
        Ht, Hprev = H[t + 1], H[t]
        lam = lam + np.outer(C[t], dy[t])
        out["dC"][t] = np.real(Ht @ np.conj(dy[t]))
        out["dB"][t] = np.real(lam @ x[t])
        out["dx"][t] = np.real(lam.T @ B[t])
        dA = lam @ np.conj(Hprev).T
        out["dd"][t] = dA[idx[s[t]], np.arange(N)]
        dpi = np.array([np.real(np.sum(np.conj(dA[idx[k], np.arange(N)]) * d[t])) for k in range(K)])
        pit = _softmax(logits[t] / tau)
        out["dlogits"][t] = (np.diag(pit) - np.outer(pit, pit)) @ dpi / tau
        lam = np.conj(A[t]).T @ lam
    out["dh0"] = lam
    out["s"] = np.array(s, dtype=np.int32)
    return out


def scan_backward(logits, idx, d, B, C, x, dy, dh_final=None, h0=None, tau: float = 1.0) -> Dict[str, np.ndarray]:
    """Gradients of S slices given slice-major arrays; returns slice-major arrays. ``idx`` is
    one dictionary [K, N] for every slice, or one per slice [S, K, N]."""
    S = np.asarray(logits).shape[0]
    idx = np.asarray(idx)
    res = [slice_backward(logits[i], idx[i] if idx.ndim == 3 else idx, d[i], B[i], C[i], x[i], dy[i],
                          None if dh_final is None else dh_final[i], None if h0 is None else h0[i], tau)
           for i in range(S)]
    return {k: np.stack([r[k] for r in res]) for k in res[0]}
