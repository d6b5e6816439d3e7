"""Oracle for the selection inputs built from dense matrices (test infrastructure only).

TEST INFRASTRUCTURE ONLY: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU legs call this module; the product path never imports it.

Flash PD-SSM page, Technical Summary, Methodology 1:
  * dictionary construction: the dictionary's sparse matrices come from dense
    trainable matrices by a column-wise hardmax, idx[k][j] = argmax_i M_k[i][j];
  * fused projection: the input u_t gives each head's K scores by a linear map,
    logits = u W, and the highest score selects (Methodology 2: hard argmax);
  * the original PD-SSM's soft selection: a convex (softmax) combination of the
    K dense dictionary matrices, made sparse by the same column-wise hardmax.
Every argmax is the pinned ``oracle.select`` (lowest index on ties, the first NaN
wins); the contractions are plain fp64 library products.
"""
from __future__ import annotations

import numpy as np

from . import select


def dict_hardmax(M) -> np.ndarray:
    """M [..., N, N] -> idx [..., N]: idx[..., j] = argmax over rows i of M[..., i, j]."""
    M = np.asarray(M, dtype=np.float64)
    return select(np.ascontiguousarray(np.swapaxes(M, -1, -2)))


def proj_logits(u, W, heads: int, K: int) -> np.ndarray:
    """u [..., D], W [D, heads * K] -> logits [..., heads, K] = u W in fp64."""
    u = np.asarray(u, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    lg = u @ W
    return lg.reshape(lg.shape[:-1] + (heads, K))


def select_proj(u, W, heads: int, K: int):
    """Fused projection and selection: (s [..., heads], logits [..., heads, K])."""
    lg = proj_logits(u, W, heads, K)
    return select(lg), lg


def softmax(v, tau: float = 1.0) -> np.ndarray:
    """softmax(v / tau) over the last axis, fp64."""
    v = np.asarray(v, dtype=np.float64) / tau
    e = np.exp(v - v.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def soft_mixture(logits, M, tau: float = 1.0) -> np.ndarray:
    """The original PD-SSM's dense transition before sparsification: sum_k softmax(logits/tau)_k M_k.
    logits [..., K], M [K, N, N] -> [..., N, N]."""
    pi = softmax(logits, tau)
    return np.einsum("...k,kij->...ij", pi, np.asarray(M, dtype=np.float64))


def soft_select(logits, M, tau: float = 1.0) -> np.ndarray:
    """Per-step transitions of the original PD-SSM: the column-wise hardmax of the soft mixture.
    logits [..., K], M [K, N, N] -> idx_steps [..., N]."""
    return dict_hardmax(soft_mixture(logits, M, tau))
