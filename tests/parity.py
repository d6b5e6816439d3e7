"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the oracle slice by slice.

Tolerance (per (batch, head) slice): max|gpu - oracle| / max(max|oracle|, 1e-30)
must stay within 1e-4 for fp32 / complex64 outputs and 2e-2 for bf16 outputs.
Selections and composed index arrays must be bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import structured_sparse_selective_b200 as pd
import workloads

TOL = {torch.float32: 1e-4, torch.complex64: 1e-4, torch.bfloat16: 2e-2}

# Largest errors seen in this test session, by output dtype and measure; printed in the
# terminal summary (tests/conftest.py) beside the pass/fail result.
REPORT: dict = {}


def _note(dtype, name: str, value: float) -> None:
    key = (str(dtype).replace("torch.", ""), name)
    REPORT[key] = max(REPORT.get(key, 0.0), float(value))


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def slice_rel_err(g: np.ndarray, r: np.ndarray) -> float:
    """Largest per-slice error; arrays are [S, ...] with the slice axis first."""
    g = g.reshape(g.shape[0], -1).astype(np.complex128)
    r = r.reshape(r.shape[0], -1).astype(np.complex128)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((np.abs(g - r).max(axis=1) / den).max()) if g.size else 0.0


def elementwise_rel_err(g: np.ndarray, r: np.ndarray, floor: float = 1e-3) -> float:
    """Largest |g - r| / |r| over the entries with |r| > floor * max|r| of their slice
    (reported beside the per-slice max-norm error; arrays are [S, ...])."""
    g = g.reshape(g.shape[0], -1).astype(np.complex128)
    r = r.reshape(r.shape[0], -1).astype(np.complex128)
    if not g.size:
        return 0.0
    mag = np.abs(r)
    keep = mag > floor * mag.max(axis=1, keepdims=True)
    if not keep.any():
        return 0.0
    return float((np.abs(g - r)[keep] / mag[keep]).max())


def bhl_to_slices(a: np.ndarray) -> np.ndarray:
    """[Bt, L, H, X] -> [Bt*H, L, X]"""
    Bt, L, H = a.shape[:3]
    return a.transpose(0, 2, 1, 3).reshape(Bt * H, L, -1)


def run_gpu(inp, device, chunk=0, h0=None, via_scan=False, flags=0, want_s=True):
    """Runs pdssm_forward (or pdssm_select + pdssm_scan_fwd) on device copies of ``inp``."""
    dev = torch.device(device)
    g = {k: v.to(dev) for k, v in inp.items()}
    h0d = None if h0 is None else h0.to(dev)
    if not via_scan:
        out = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], h0=h0d, chunk=chunk,
                         flags=flags, want_s=want_s)
    else:
        if g["idx"].dim() == 3:  # per-head dictionaries
            flags |= pd.FLAG_HEAD_DICTS
        pb = pd.make_problem(g["logits"], g["d"], g["B"], g["x"], chunk=chunk, flags=flags)
        Bt, L, H, N = g["B"].shape
        P = g["x"].shape[-1]
        s = torch.empty(Bt, L, H, dtype=torch.int32, device=dev)
        pd.pdssm_select(pb, g["logits"], s)
        sdt = torch.complex64 if pb.state_t == pd.C64 else torch.float32
        ydt = {pd.F32: torch.float32, pd.BF16: torch.bfloat16, pd.C64: torch.complex64}[pb.out_t]
        out = {"y": torch.empty(Bt, L, H, P, dtype=ydt, device=dev),
               "h_final": torch.empty(Bt, H, N, P, dtype=sdt, device=dev),
               "prod_idx": torch.empty(Bt, H, N, dtype=torch.int32, device=dev),
               "prod_val": torch.empty(Bt, H, N, dtype=sdt, device=dev), "s": s}
        ws = pd.alloc_workspace(pb, dev)
        pd.pdssm_scan_fwd(pb, s, g["idx"], g["d"], g["B"], g["C"], g["x"], h0d, out["y"], out["h_final"],
                          out["prod_idx"], out["prod_val"], ws)
    torch.cuda.synchronize(dev)
    return out


def compare_full(inp, out, h0=None, y_tol=None):
    """Oracle on every slice; returns dict of errors (asserts on exact parts)."""
    r = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], h0=h0)
    y_tol = y_tol or TOL[out["y"].dtype]
    errs = {}
    errs["y"] = slice_rel_err(bhl_to_slices(to_np(out["y"])), bhl_to_slices(r["y"]))
    errs["y_elementwise"] = elementwise_rel_err(bhl_to_slices(to_np(out["y"])), bhl_to_slices(r["y"]))
    Bt, H = r["h_final"].shape[:2]
    errs["h_final"] = slice_rel_err(to_np(out["h_final"]).reshape(Bt * H, -1), r["h_final"].reshape(Bt * H, -1))
    errs["h_final_elementwise"] = elementwise_rel_err(to_np(out["h_final"]).reshape(Bt * H, -1),
                                                      r["h_final"].reshape(Bt * H, -1))
    if "prod_idx" in out:
        assert np.array_equal(to_np(out["prod_idx"]), r["prod_idx"]), "composed index arrays differ"
        errs["prod_val"] = slice_rel_err(to_np(out["prod_val"]).reshape(Bt * H, -1),
                                         r["prod_val"].reshape(Bt * H, -1))
    if "s" in out:
        assert np.array_equal(to_np(out["s"]), r["s"]), "selections differ"
    for name, v in errs.items():
        _note(out["y"].dtype if name.startswith("y") else out["h_final"].dtype, name, v)
    assert errs["y"] <= y_tol, errs
    assert errs["h_final"] <= 1e-4, errs
    if "prod_val" in errs:
        assert errs["prod_val"] <= 1e-4, errs
    return errs


def sparse_prod_all_slices(s: np.ndarray, idx: np.ndarray, N: int) -> np.ndarray:
    """Composed index arrays of every slice by the (idx, val) composition (indices only).
    s [Bt, L, H] -> [Bt, H, N]."""
    Bt, L, H = s.shape
    cur = np.broadcast_to(np.arange(N), (Bt, H, N)).copy()
    for t in range(L):
        sel = idx[s[:, t, :]]                      # [Bt, H, N] = idx_{s_t}
        cur = np.take_along_axis(sel, cur, axis=-1)
    return cur


def sampled_slices(sp: workloads.Spec, n: int, seed: int = 0):
    rng = np.random.default_rng(seed + sp.batch * 7 + sp.heads)
    total = sp.batch * sp.heads
    picks = sorted(set(int(v) for v in rng.choice(total, size=min(n, total), replace=False)))
    picks = sorted(set(picks) | {0, total - 1})
    return [(p // sp.heads, p % sp.heads) for p in picks]
