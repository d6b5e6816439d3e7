"""Dense CPU oracle for the Flash PD-SSM forward pass (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The product path never
imports this package and has no CPU fallback.

Every input is upcast exactly to fp64 (complex128 for complex d) before the C
routine sees it, so the oracle reads the same rounded values the GPU reads.
See ``pdssm_oracle.c`` for what is computed and which passage each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pdssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpdssm_oracle.so")
_lib = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle (plain C, OpenMP) in place; returns the library path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.pdssm_oracle_threads.restype = ctypes.c_int
        lib.pdssm_oracle_select.argtypes = [_ptr, _i64, _i64, _ptr]
        lib.pdssm_oracle_select.restype = None
        for name in ("pdssm_oracle_scan_real", "pdssm_oracle_scan_complex"):
            fn = getattr(lib, name)
            fn.argtypes = [_i64] * 5 + [_ptr] * 12
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses (the core count of a CPU-baseline figure)."""
    return int(_load().pdssm_oracle_threads())


def _np(t, dtype) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.to(torch.float32)  # exact
        t = t.numpy()
    return np.ascontiguousarray(np.asarray(t).astype(dtype, copy=False))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def select(logits) -> np.ndarray:
    """s = argmax over the last axis, lowest index on ties, first NaN wins."""
    lg = _np(logits, np.float64)
    K = lg.shape[-1]
    rows = lg.size // K if K else 0
    s = np.empty(lg.shape[:-1], dtype=np.int32)
    _load().pdssm_oracle_select(_p(lg), rows, K, _p(s))
    return s


def scan_slices(logits, idx, d, B, C, x, h0=None, want_prod: bool = True) -> Dict[str, np.ndarray]:
    """Dense recurrence over S independent slices given slice-major arrays.

    logits [S,L,K], d [S,L,N] (real or complex), B/C [S,L,N], x [S,L,P],
    h0 [S,N,P] or None. Returns y [S,L,P], h_final [S,N,P], s [S,L] and, if
    ``want_prod``, prod_idx [S,N] and prod_val [S,N].
    """
    is_complex = (isinstance(d, torch.Tensor) and d.is_complex()) or (
        isinstance(d, np.ndarray) and np.iscomplexobj(d))
    cdt = np.complex128 if is_complex else np.float64
    lg = _np(logits, np.float64)
    ix = _np(idx, np.int32)
    dd = _np(d, cdt)
    Bb = _np(B, np.float64)
    Cc = _np(C, np.float64)
    xx = _np(x, np.float64)
    S, L, K = lg.shape
    N = Bb.shape[-1]
    P = xx.shape[-1]
    hh = None if h0 is None else _np(h0, cdt)
    y = np.zeros((S, L, P), dtype=cdt)
    hf = np.zeros((S, N, P), dtype=cdt)
    s = np.zeros((S, L), dtype=np.int32)
    pi = np.zeros((S, N), dtype=np.int32) if want_prod else None
    pv = np.zeros((S, N), dtype=cdt) if want_prod else None
    lib = _load()
    fn = lib.pdssm_oracle_scan_complex if is_complex else lib.pdssm_oracle_scan_real
    rc = fn(S, L, N, P, K, _p(lg), _p(ix), _p(dd), _p(Bb), _p(Cc), _p(xx), _p(hh), _p(y), _p(hf),
            _p(pi), _p(pv), _p(s))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    out = {"y": y, "h_final": hf, "s": s}
    if want_prod:
        out["prod_idx"] = pi
        out["prod_val"] = pv
    return out


def _to_slices(t: torch.Tensor) -> torch.Tensor:
    """[Bt, L, H, X] -> [Bt*H, L, X]"""
    Bt, L, H, X = t.shape
    return t.permute(0, 2, 1, 3).reshape(Bt * H, L, X)


def scan(logits, idx, d, B, C, x, h0=None, want_prod: bool = True) -> Dict[str, np.ndarray]:
    """Dense recurrence on full [Bt, L, H, *] arrays; outputs in the same layout.
    ``idx`` is the shared dictionary [K, N] or per-head dictionaries [H, K, N].

    Returns y [Bt,L,H,P], h_final [Bt,H,N,P], s [Bt,L,H] and optionally
    prod_idx [Bt,H,N], prod_val [Bt,H,N].
    """
    Bt, L, H, K = logits.shape
    N = B.shape[-1]
    P = x.shape[-1]
    h0s = None if h0 is None else h0.reshape(Bt * H, N, P)
    if getattr(idx, "ndim", 2) == 3:
        # per-head dictionaries idx[H][K][N]: the slices of head h use idx[h]
        sl = {k: _to_slices(v) for k, v in (("logits", logits), ("d", d), ("B", B), ("C", C), ("x", x))}
        parts = []
        for hh in range(H):
            rows = list(range(hh, Bt * H, H))
            parts.append((rows, scan_slices(sl["logits"][rows], idx[hh], sl["d"][rows], sl["B"][rows],
                                            sl["C"][rows], sl["x"][rows],
                                            None if h0s is None else h0s[rows], want_prod)))
        r = {k: np.empty((Bt * H,) + v.shape[1:], dtype=v.dtype) for k, v in parts[0][1].items()}
        for rows, part in parts:
            for k, v in part.items():
                r[k][rows] = v
    else:
        r = scan_slices(_to_slices(logits), idx, _to_slices(d), _to_slices(B), _to_slices(C),
                        _to_slices(x), h0s, want_prod)
    out = {
        "y": r["y"].reshape(Bt, H, L, P).transpose(0, 2, 1, 3),
        "h_final": r["h_final"].reshape(Bt, H, N, P),
        "s": r["s"].reshape(Bt, H, L).transpose(0, 2, 1),
    }
    if want_prod:
        out["prod_idx"] = r["prod_idx"].reshape(Bt, H, N)
        out["prod_val"] = r["prod_val"].reshape(Bt, H, N)
    return out


def scan_steps(idx_steps, d, B, C, x, h0=None, want_prod: bool = True) -> Dict[str, np.ndarray]:
    """The recurrence with a transition given per step (the original PD-SSM's per-step
    matrices): step t of slice (b, h) applies P_t with P_t[idx_steps[b, t, h, j]][j] = 1.
    Each slice is the dense loop above with its L step rows as the dictionary and step t
    selecting row t. idx_steps [Bt, L, H, N]; other arrays as in scan()."""
    st = np.asarray(idx_steps.cpu() if isinstance(idx_steps, torch.Tensor) else idx_steps).astype(np.int32)
    Bt, L, H, N = st.shape
    P = x.shape[-1]
    pick = np.eye(L)  # logits: step t selects dictionary row t
    out = {"y": None}
    ys, hfs, pis, pvs = [], [], [], []
    for b in range(Bt):
        for h in range(H):
            r = scan_slices(pick[None], st[b, :, h], d[b:b + 1, :, h], B[b:b + 1, :, h], C[b:b + 1, :, h],
                            x[b:b + 1, :, h], None if h0 is None else h0[b:b + 1, h], want_prod)
            ys.append(r["y"][0]); hfs.append(r["h_final"][0])
            if want_prod:
                pis.append(r["prod_idx"][0]); pvs.append(r["prod_val"][0])
    out["y"] = np.stack(ys).reshape(Bt, H, L, P).transpose(0, 2, 1, 3)
    out["h_final"] = np.stack(hfs).reshape(Bt, H, N, P)
    if want_prod:
        out["prod_idx"] = np.stack(pis).reshape(Bt, H, N)
        out["prod_val"] = np.stack(pvs).reshape(Bt, H, N)
    return out
