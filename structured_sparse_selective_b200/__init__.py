"""Python binding of libpdssm.so, the B200 forward pass of Flash PD-SSM.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels behind the C ABI declared in ``include/pdssm.h``. PyTorch supplies
device memory and the current stream. There is no CPU fallback: if the
library is missing, importing this package raises.

The functions keep the C names:

    pdssm_workspace_size(problem) -> int
    pdssm_select(problem, logits, s, stream=None)
    pdssm_scan_fwd(problem, s, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, workspace, stream=None)
    pdssm_forward(problem, logits, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, s_out, workspace, stream=None)
    pdssm_read_device_check(workspace, stream=None)
    pdssm_bwd_workspace_size(problem) -> int
    pdssm_scan_bwd(problem, logits, s, idx, d, B, C, x, h0, dy, dh_final, tau, dlogits, dd, dB, dC, dx, dh0,
                   workspace, stream=None)

``forward(...)`` is a convenience wrapper that allocates the outputs and the
workspace with torch and calls ``pdssm_forward``; ``backward(...)`` does the
same for ``pdssm_scan_bwd``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

__all__ = [
    "PdssmError", "Problem", "F32", "BF16", "C64", "FLAG_DEVICE_CHECK", "FLAG_REFERENCE_PATH", "FLAG_SHORT_WAITS",
    "FLAG_HEAD_DICTS",
    "library_path", "make_problem", "pdssm_workspace_size", "pdssm_select", "pdssm_scan_fwd",
    "pdssm_forward", "pdssm_read_device_check", "pdssm_status_string", "forward", "EXPORTED_SYMBOLS",
    "KernelTrace", "alloc_workspace", "pdssm_forward_noalloc", "pdssm_bwd_workspace_size", "pdssm_scan_bwd",
    "backward", "pdssm_dict_hardmax", "pdssm_select_proj", "dict_hardmax", "select_proj",
    "pdssm_soft_select_workspace_size", "pdssm_soft_select", "pdssm_scan_fwd_steps", "soft_select",
    "forward_steps",
]

F32, BF16, C64 = 0, 1, 2
FLAG_DEVICE_CHECK = 1
FLAG_REFERENCE_PATH = 2
FLAG_SHORT_WAITS = 4
FLAG_HEAD_DICTS = 8
MAX_N, MAX_P, MAX_K = 128, 128, 64

EXPORTED_SYMBOLS = (
    "pdssm_status_string", "pdssm_version", "pdssm_workspace_size", "pdssm_select",
    "pdssm_scan_fwd", "pdssm_forward", "pdssm_read_device_check", "pdssm_trace_begin",
    "pdssm_trace_end", "pdssm_trace_kernel_name", "pdssm_forward_noalloc", "pdssm_bwd_workspace_size",
    "pdssm_scan_bwd", "pdssm_dict_hardmax", "pdssm_select_proj", "pdssm_soft_select_workspace_size",
    "pdssm_soft_select", "pdssm_scan_fwd_steps",
)

_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_DIR, "libpdssm.so")


def library_path() -> str:
    return _LIB_PATH


class Problem(ctypes.Structure):
    """Mirror of ``pdssm_problem``."""

    _fields_ = [
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
        ("N", ctypes.c_int64), ("P", ctypes.c_int64), ("K", ctypes.c_int64),
        ("chunk", ctypes.c_int32), ("logits_t", ctypes.c_int32), ("in_t", ctypes.c_int32),
        ("d_t", ctypes.c_int32), ("state_t", ctypes.c_int32), ("out_t", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
    ]


class PdssmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pdssm_status_string(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing; build it with `python structured_sparse_selective_b200/build.py`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32p, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    pb = ctypes.POINTER(Problem)
    lib.pdssm_status_string.argtypes = [ctypes.c_int32]
    lib.pdssm_status_string.restype = ctypes.c_char_p
    lib.pdssm_version.restype = ctypes.c_char_p
    lib.pdssm_workspace_size.argtypes = [pb, ctypes.POINTER(sz)]
    lib.pdssm_workspace_size.restype = ctypes.c_int
    lib.pdssm_select.argtypes = [pb, vp, i32p, vp]
    lib.pdssm_select.restype = ctypes.c_int
    lib.pdssm_scan_fwd.argtypes = [pb, i32p, i32p, vp, vp, vp, vp, vp, vp, vp, i32p, vp, vp, sz, vp]
    lib.pdssm_scan_fwd.restype = ctypes.c_int
    lib.pdssm_forward.argtypes = [pb, vp, i32p, vp, vp, vp, vp, vp, vp, vp, i32p, vp, i32p, vp, sz, vp]
    lib.pdssm_forward.restype = ctypes.c_int
    lib.pdssm_forward_noalloc.argtypes = [pb, vp, i32p, vp, vp, vp, vp, vp, vp, vp, i32p, vp, i32p, vp]
    lib.pdssm_forward_noalloc.restype = ctypes.c_int
    lib.pdssm_bwd_workspace_size.argtypes = [pb, ctypes.POINTER(sz)]
    lib.pdssm_bwd_workspace_size.restype = ctypes.c_int
    lib.pdssm_scan_bwd.argtypes = [pb, vp, i32p, i32p, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float,
                                   vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.pdssm_scan_bwd.restype = ctypes.c_int
    lib.pdssm_dict_hardmax.argtypes = [ctypes.c_int64, ctypes.c_int64, vp, vp, vp]
    lib.pdssm_dict_hardmax.restype = ctypes.c_int
    lib.pdssm_select_proj.argtypes = [pb, ctypes.c_int64, vp, vp, vp, vp, vp, sz, vp]
    lib.pdssm_select_proj.restype = ctypes.c_int
    lib.pdssm_soft_select_workspace_size.argtypes = [pb, ctypes.POINTER(sz)]
    lib.pdssm_soft_select_workspace_size.restype = ctypes.c_int
    lib.pdssm_soft_select.argtypes = [pb, vp, vp, ctypes.c_float, vp, vp, sz, vp]
    lib.pdssm_soft_select.restype = ctypes.c_int
    lib.pdssm_scan_fwd_steps.argtypes = [pb, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.pdssm_scan_fwd_steps.restype = ctypes.c_int
    lib.pdssm_read_device_check.argtypes = [vp, vp]
    lib.pdssm_read_device_check.restype = ctypes.c_int
    lib.pdssm_trace_begin.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
    lib.pdssm_trace_begin.restype = ctypes.c_int
    lib.pdssm_trace_end.argtypes = []
    lib.pdssm_trace_end.restype = ctypes.c_int32
    lib.pdssm_trace_kernel_name.argtypes = [ctypes.c_int32]
    lib.pdssm_trace_kernel_name.restype = ctypes.c_char_p
    return lib


_lib = _load()

_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.complex64: C64}


def pdssm_status_string(status: int) -> str:
    return _lib.pdssm_status_string(int(status)).decode()


def version() -> str:
    return _lib.pdssm_version().decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PdssmError(status, where)


def _ptr(t: Optional[torch.Tensor], device: Optional[torch.device] = None):
    """Device address of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("libpdssm takes device memory only; got a CPU tensor")
    if device is not None and t.device != device:
        raise ValueError(f"tensor on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else ctypes.c_void_p(t.data_ptr() or 0)


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(handle)


def make_problem(logits: torch.Tensor, d: torch.Tensor, B: torch.Tensor, x: torch.Tensor,
                 out_dtype: Optional[torch.dtype] = None, chunk: int = 0, flags: int = 0,
                 K: Optional[int] = None) -> Problem:
    """Problem description from tensor shapes and dtypes (logits may be None if K is given)."""
    Bt, L, H, N = B.shape
    P = x.shape[-1]
    cplx = d.dtype == torch.complex64
    if out_dtype is None:
        out_dtype = torch.complex64 if cplx else B.dtype
    return Problem(
        batch=Bt, seqlen=L, heads=H, N=N, P=P, K=(logits.shape[-1] if logits is not None else K),
        chunk=chunk, logits_t=_DT[logits.dtype] if logits is not None else F32, in_t=_DT[B.dtype],
        d_t=_DT[d.dtype], state_t=C64 if cplx else F32, out_t=_DT[out_dtype], flags=flags)


def pdssm_workspace_size(pb: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.pdssm_workspace_size(ctypes.byref(pb), ctypes.byref(n)), "pdssm_workspace_size")
    return int(n.value)


def pdssm_select(pb: Problem, logits: torch.Tensor, s: torch.Tensor, stream=None) -> None:
    dev = logits.device
    _check(_lib.pdssm_select(ctypes.byref(pb), _ptr(logits, dev), _ptr(s, dev), _stream(stream, dev)),
           "pdssm_select")


def pdssm_scan_fwd(pb: Problem, s, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, workspace,
                   stream=None) -> None:
    dev = idx.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_scan_fwd(
        ctypes.byref(pb), _ptr(s, dev), _ptr(idx, dev), _ptr(d, dev), _ptr(B, dev), _ptr(C, dev),
        _ptr(x, dev), _ptr(h0, dev), _ptr(y, dev), _ptr(h_final, dev), _ptr(prod_idx, dev),
        _ptr(prod_val, dev), _ptr(workspace, dev), ws_bytes, _stream(stream, dev)), "pdssm_scan_fwd")


def pdssm_forward(pb: Problem, logits, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val, s_out,
                  workspace, stream=None) -> None:
    dev = idx.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_forward(
        ctypes.byref(pb), _ptr(logits, dev), _ptr(idx, dev), _ptr(d, dev), _ptr(B, dev), _ptr(C, dev),
        _ptr(x, dev), _ptr(h0, dev), _ptr(y, dev), _ptr(h_final, dev), _ptr(prod_idx, dev),
        _ptr(prod_val, dev), _ptr(s_out, dev), _ptr(workspace, dev), ws_bytes, _stream(stream, dev)),
        "pdssm_forward")


def pdssm_forward_noalloc(pb: Problem, logits, idx, d, B, C, x, h0, y, h_final, prod_idx, prod_val,
                          s_out, stream=None) -> None:
    """pdssm_forward with the library's built-in 32 MiB device workspace (no caller workspace)."""
    dev = idx.device
    _check(_lib.pdssm_forward_noalloc(
        ctypes.byref(pb), _ptr(logits, dev), _ptr(idx, dev), _ptr(d, dev), _ptr(B, dev), _ptr(C, dev),
        _ptr(x, dev), _ptr(h0, dev), _ptr(y, dev), _ptr(h_final, dev), _ptr(prod_idx, dev),
        _ptr(prod_val, dev), _ptr(s_out, dev), _stream(stream, dev)), "pdssm_forward_noalloc")


def pdssm_bwd_workspace_size(pb: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.pdssm_bwd_workspace_size(ctypes.byref(pb), ctypes.byref(n)), "pdssm_bwd_workspace_size")
    return int(n.value)


def pdssm_scan_bwd(pb: Problem, logits, s, idx, d, B, C, x, h0, dy, dh_final, tau: float, dlogits, dd, dB, dC,
                   dx, dh0, workspace, stream=None) -> None:
    dev = idx.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_scan_bwd(
        ctypes.byref(pb), _ptr(logits, dev), _ptr(s, dev), _ptr(idx, dev), _ptr(d, dev), _ptr(B, dev),
        _ptr(C, dev), _ptr(x, dev), _ptr(h0, dev), _ptr(dy, dev), _ptr(dh_final, dev), float(tau),
        _ptr(dlogits, dev), _ptr(dd, dev), _ptr(dB, dev), _ptr(dC, dev), _ptr(dx, dev), _ptr(dh0, dev),
        _ptr(workspace, dev), ws_bytes, _stream(stream, dev)), "pdssm_scan_bwd")


def pdssm_dict_hardmax(K: int, N: int, M: torch.Tensor, idx: torch.Tensor, stream=None) -> None:
    dev = M.device
    _check(_lib.pdssm_dict_hardmax(int(K), int(N), _ptr(M, dev), _ptr(idx, dev), _stream(stream, dev)),
           "pdssm_dict_hardmax")


def pdssm_select_proj(pb: Problem, D: int, u, W, s, logits, workspace, stream=None) -> None:
    dev = u.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_select_proj(ctypes.byref(pb), int(D), _ptr(u, dev), _ptr(W, dev), _ptr(s, dev),
                                  _ptr(logits, dev), _ptr(workspace, dev), ws_bytes, _stream(stream, dev)),
           "pdssm_select_proj")


def dict_hardmax(M: torch.Tensor, stream=None) -> torch.Tensor:
    """Column-wise hardmax of dense matrices M [..., N, N] (float32): idx [..., N] int32."""
    N = M.shape[-1]
    K = M.numel() // (N * N)
    idx = torch.empty(M.shape[:-2] + (N,), dtype=torch.int32, device=M.device)
    pdssm_dict_hardmax(K, N, M.contiguous(), idx, stream)
    return idx


def select_proj(u: torch.Tensor, W: torch.Tensor, heads: int, K: int, want_logits: bool = False,
                stream=None) -> Dict[str, torch.Tensor]:
    """u [Bt, L, D] bf16, W [D, heads * K] bf16 -> s [Bt, L, heads] int32 (and logits [Bt, L, heads, K])."""
    Bt, L, D = u.shape
    pb = Problem(batch=Bt, seqlen=L, heads=heads, N=1, P=1, K=K, chunk=0, logits_t=BF16, in_t=BF16, d_t=BF16,
                 state_t=F32, out_t=BF16, flags=0)
    out = {"s": torch.empty(Bt, L, heads, dtype=torch.int32, device=u.device)}
    if want_logits:
        out["logits"] = torch.empty(Bt, L, heads, K, dtype=torch.float32, device=u.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=u.device)
    pdssm_select_proj(pb, D, u.contiguous(), W.contiguous(), out["s"], out.get("logits"), ws, stream)
    out["workspace"] = ws
    return out


def pdssm_soft_select_workspace_size(pb: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.pdssm_soft_select_workspace_size(ctypes.byref(pb), ctypes.byref(n)),
           "pdssm_soft_select_workspace_size")
    return int(n.value)


def pdssm_soft_select(pb: Problem, logits, M, tau: float, idx_steps, workspace, stream=None) -> None:
    dev = logits.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_soft_select(ctypes.byref(pb), _ptr(logits, dev), _ptr(M, dev), float(tau), _ptr(idx_steps, dev),
                                  _ptr(workspace, dev), ws_bytes, _stream(stream, dev)), "pdssm_soft_select")


def pdssm_scan_fwd_steps(pb: Problem, idx_steps, d, B, C, x, h0, y, h_final, prod_idx, prod_val, workspace,
                         stream=None) -> None:
    dev = d.device
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pdssm_scan_fwd_steps(
        ctypes.byref(pb), _ptr(idx_steps, dev), _ptr(d, dev), _ptr(B, dev), _ptr(C, dev), _ptr(x, dev),
        _ptr(h0, dev), _ptr(y, dev), _ptr(h_final, dev), _ptr(prod_idx, dev), _ptr(prod_val, dev),
        _ptr(workspace, dev), ws_bytes, _stream(stream, dev)), "pdssm_scan_fwd_steps")


def soft_select(logits: torch.Tensor, M: torch.Tensor, tau: float = 1.0, N: Optional[int] = None,
                stream=None) -> Dict[str, torch.Tensor]:
    """The original PD-SSM's per-step transitions: idx_steps [Bt, L, H, N] uint8 from logits
    [Bt, L, H, K] and dense dictionary matrices M [K, N, N] (or per head [H, K, N, N])."""
    Bt, L, H, K = logits.shape
    N = M.shape[-1]
    flags = FLAG_HEAD_DICTS if M.dim() == 4 else 0
    pb = Problem(batch=Bt, seqlen=L, heads=H, N=N, P=1, K=K, chunk=0, logits_t=_DT[logits.dtype], in_t=F32,
                 d_t=F32, state_t=F32, out_t=F32, flags=flags)
    ws = torch.empty(pdssm_soft_select_workspace_size(pb), dtype=torch.uint8, device=logits.device)
    steps = torch.empty(Bt, L, H, N, dtype=torch.uint8, device=logits.device)
    pdssm_soft_select(pb, logits.contiguous(), M.contiguous(), tau, steps, ws, stream)
    return {"idx_steps": steps, "workspace": ws}


def forward_steps(idx_steps: torch.Tensor, d: torch.Tensor, B: torch.Tensor, C: torch.Tensor, x: torch.Tensor,
                  h0: Optional[torch.Tensor] = None, out_dtype: Optional[torch.dtype] = None, flags: int = 0,
                  stream=None) -> Dict[str, torch.Tensor]:
    """The scan with a transition per step (idx_steps [Bt, L, H, N] uint8), e.g. from soft_select."""
    Bt, L, H, N = B.shape
    P = x.shape[-1]
    if out_dtype is None:
        out_dtype = B.dtype
    pb = Problem(batch=Bt, seqlen=L, heads=H, N=N, P=P, K=1, chunk=0, logits_t=BF16, in_t=_DT[B.dtype],
                 d_t=_DT[d.dtype], state_t=F32, out_t=_DT[out_dtype], flags=flags)
    dev = B.device
    out = {"y": torch.empty(Bt, L, H, P, dtype=out_dtype, device=dev),
           "h_final": torch.empty(Bt, H, N, P, dtype=torch.float32, device=dev),
           "prod_idx": torch.empty(Bt, H, N, dtype=torch.int32, device=dev),
           "prod_val": torch.empty(Bt, H, N, dtype=torch.float32, device=dev)}
    ws = alloc_workspace(pb, dev)
    pdssm_scan_fwd_steps(pb, idx_steps, d, B, C, x, h0, out["y"], out["h_final"], out["prod_idx"], out["prod_val"],
                         ws, stream)
    out["workspace"] = ws
    return out


def pdssm_read_device_check(workspace: torch.Tensor, stream=None) -> int:
    """Status left in the workspace's error word by the last scan (synchronises)."""
    return int(_lib.pdssm_read_device_check(_ptr(workspace), _stream(stream, workspace.device)))


class KernelTrace:
    """Times each kernel the library launches inside a ``with`` block (CUDA events).

        with KernelTrace(max_launches=16) as tr:
            pdssm_forward(...)
        torch.cuda.synchronize(); tr.timings() -> [(kernel_name, ms), ...]
    """

    def __init__(self, max_launches: int = 16):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * max_launches)]
        for e in self.events:  # torch creates the CUDA event on first record
            e.record()
        self._arr = (ctypes.c_void_p * len(self.events))(*[ctypes.c_void_p(e.cuda_event) for e in self.events])
        self.names = []

    def __enter__(self):
        _check(_lib.pdssm_trace_begin(self._arr, len(self.events)), "pdssm_trace_begin")
        return self

    def __exit__(self, *exc):
        n = int(_lib.pdssm_trace_end())
        self.names = [_lib.pdssm_trace_kernel_name(i).decode() for i in range(n)]
        return False

    def timings(self):
        return [(nm, self.events[2 * i].elapsed_time(self.events[2 * i + 1])) for i, nm in enumerate(self.names)]


def _dict_flags(idx: torch.Tensor, heads: int, K: int, N: int) -> int:
    """FLAG_HEAD_DICTS for a per-head dictionary [heads, K, N]; 0 for a shared [K, N] one."""
    if idx.dim() == 3:
        if tuple(idx.shape) != (heads, K, N):
            raise ValueError(f"per-head dictionary must be [{heads}, {K}, {N}], got {tuple(idx.shape)}")
        return FLAG_HEAD_DICTS
    if tuple(idx.shape) != (K, N):
        raise ValueError(f"dictionary must be [{K}, {N}], got {tuple(idx.shape)}")
    return 0


def alloc_workspace(pb: Problem, device) -> torch.Tensor:
    return torch.empty(max(1, pdssm_workspace_size(pb)), dtype=torch.uint8, device=device)


def forward(logits: torch.Tensor, idx: torch.Tensor, d: torch.Tensor, B: torch.Tensor,
            C: torch.Tensor, x: torch.Tensor, h0: Optional[torch.Tensor] = None,
            out_dtype: Optional[torch.dtype] = None, chunk: int = 0, flags: int = 0,
            want_prod: bool = True, want_s: bool = False, workspace: Optional[torch.Tensor] = None,
            stream=None) -> Dict[str, torch.Tensor]:
    """Allocates the outputs (torch) and runs ``pdssm_forward`` on the inputs' device.
    A 3-D ``idx`` [heads, K, N] is a per-head dictionary (PDSSM_FLAG_HEAD_DICTS)."""
    flags |= _dict_flags(idx, B.shape[2], logits.shape[-1], B.shape[-1])
    pb = make_problem(logits, d, B, x, out_dtype=out_dtype, chunk=chunk, flags=flags)
    dev = B.device
    Bt, L, H, N = B.shape
    P = x.shape[-1]
    sdt = torch.complex64 if pb.state_t == C64 else torch.float32
    ydt = {F32: torch.float32, BF16: torch.bfloat16, C64: torch.complex64}[pb.out_t]
    out = {
        "y": torch.empty(Bt, L, H, P, dtype=ydt, device=dev),
        "h_final": torch.empty(Bt, H, N, P, dtype=sdt, device=dev),
    }
    if want_prod:
        out["prod_idx"] = torch.empty(Bt, H, N, dtype=torch.int32, device=dev)
        out["prod_val"] = torch.empty(Bt, H, N, dtype=sdt, device=dev)
    if want_s:
        out["s"] = torch.empty(Bt, L, H, dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else alloc_workspace(pb, dev)
    pdssm_forward(pb, logits, idx, d, B, C, x, h0, out["y"], out["h_final"], out.get("prod_idx"),
                  out.get("prod_val"), out.get("s"), ws, stream)
    return out


def backward(logits: Optional[torch.Tensor], s: torch.Tensor, idx: torch.Tensor, d: torch.Tensor,
             B: torch.Tensor, C: torch.Tensor, x: torch.Tensor, dy: torch.Tensor,
             h0: Optional[torch.Tensor] = None, dh_final: Optional[torch.Tensor] = None, tau: float = 1.0,
             want_dh0: bool = True, workspace: Optional[torch.Tensor] = None, stream=None) -> Dict[str, torch.Tensor]:
    """Allocates the gradients and runs ``pdssm_scan_bwd``; ``s`` are the forward's selections,
    ``dy`` has the forward output's dtype. dd and dh0 have the state's dtype (float32, or
    complex64 for a complex ``d``), the others are float32. No logits -> no ``dlogits``."""
    K = logits.shape[-1] if logits is not None else int(idx.shape[-2])
    pb = make_problem(logits, d, B, x, out_dtype=dy.dtype, K=K,
                      flags=_dict_flags(idx, B.shape[2], K, B.shape[-1]))
    dev = B.device
    Bt, L, H, N = B.shape
    P = x.shape[-1]
    f = dict(dtype=torch.float32, device=dev)
    fs = dict(dtype=torch.complex64 if d.is_complex() else torch.float32, device=dev)
    out = {"dd": torch.empty(Bt, L, H, N, **fs), "dB": torch.empty(Bt, L, H, N, **f),
           "dC": torch.empty(Bt, L, H, N, **f), "dx": torch.empty(Bt, L, H, P, **f)}
    if logits is not None:
        out["dlogits"] = torch.empty(Bt, L, H, K, **f)
    if want_dh0:
        out["dh0"] = torch.empty(Bt, H, N, P, **fs)
    ws = workspace if workspace is not None else torch.empty(max(1, pdssm_bwd_workspace_size(pb)),
                                                              dtype=torch.uint8, device=dev)
    pdssm_scan_bwd(pb, logits, s, idx, d, B, C, x, h0, dy, dh_final, tau, out.get("dlogits"), out["dd"], out["dB"],
                   out["dC"], out["dx"], out.get("dh0"), ws, stream)
    return out
