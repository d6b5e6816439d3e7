"""Seeded synthetic inputs for the Flash PD-SSM forward scan.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no selection, no recurrence, no composition). Both the CPU
oracle (``oracle/``) and the CUDA path are fed from it, so the two always see
the same already-rounded values.

Recipes follow the five workloads the build is measured on (the shapes of the
Flash PD-SSM explainer's workloads: an FSA state-tracking task, a language-model
layer, a long time series and a large complex-diagonal layer; see the
"Experimental Results" section of the Flash PD-SSM page). None of the pages'
datasets is used; these inputs stand in for their shapes only.

Layout (all row-major, contiguous):
    idx     [K, N]          int32   idx[k][j] = row of the nonzero in column j of P_k
    logits  [Bt, L, H, K]   f32 | bf16
    d       [Bt, L, H, N]   f32 | bf16 | complex64
    B, C    [Bt, L, H, N]   f32 | bf16
    x       [Bt, L, H, P]   f32 | bf16

Determinism: ``idx`` comes from a generator seeded with ``seed``; every
(batch, head) slice has its own generator seeded from (seed, recipe, b, h) and
draws, in order, logits, d, B, C, x for all L steps of that slice. A slice can
therefore be regenerated on its own (the oracle checks sampled slices of the
large workloads without building the whole tensor).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Tuple

import torch

__all__ = ["Spec", "RECIPES", "spec", "generate", "generate_slice", "CONFIG_ORDER"]


@dataclasses.dataclass(frozen=True)
class Spec:
    """Shape, dtypes and value recipe of one synthetic workload."""

    recipe: str
    batch: int
    seqlen: int
    heads: int
    N: int
    P: int
    K: int
    logits_dtype: torch.dtype
    in_dtype: torch.dtype        # B, C, x
    d_dtype: torch.dtype         # float32, bfloat16 or complex64
    state_complex: bool
    out_dtype: torch.dtype       # y

    @property
    def token_heads(self) -> int:
        return self.batch * self.seqlen * self.heads

    def algorithmic_bytes_per_token_head(self, with_logits: bool = True) -> int:
        """Bytes that must cross HBM per (b, t, h): inputs read once, y written once."""
        def sz(dt):
            return torch.empty((), dtype=dt).element_size()
        b = self.N * sz(self.d_dtype) + 2 * self.N * sz(self.in_dtype) + self.P * sz(self.in_dtype)
        b += self.P * sz(self.out_dtype)
        b += self.K * sz(self.logits_dtype) if with_logits else 4
        return b


_F32, _BF16, _C64 = torch.float32, torch.bfloat16, torch.complex64

# name -> (shape, dtypes); shapes are the full-size workloads.
RECIPES: Dict[str, Spec] = {
    # tiny fp32: batch 1, heads 1, L=256, N=8, P=4, K=4
    "tiny": Spec("tiny", 1, 256, 1, 8, 4, 4, _F32, _F32, _F32, False, _F32),
    # FSA state tracking on Z_5: batch 64, L=512, N=5, P=1, K=5
    "z5": Spec("z5", 64, 512, 1, 5, 1, 5, _F32, _F32, _F32, False, _F32),
    # LM layer, bf16 in / fp32 state / bf16 y: batch 8, L=2048, heads 32, N=P=64, K=16
    "lm": Spec("lm", 8, 2048, 32, 64, 64, 16, _BF16, _BF16, _BF16, False, _BF16),
    # long fp32 time series with permutation dictionary: batch 4, L=18000, heads 8, N=P=32, K=8
    "long": Spec("long", 4, 18000, 8, 32, 32, 8, _F32, _F32, _F32, False, _F32),
    # large complex-diagonal: batch 16, L=8192, heads 64, N=128, P=64, K=64
    "complex": Spec("complex", 16, 8192, 64, 128, 64, 64, _BF16, _BF16, _C64, True, _C64),
}

CONFIG_ORDER = ("tiny", "z5", "lm", "long", "complex")

_SALT = {"tiny": 11, "z5": 23, "lm": 37, "long": 41, "complex": 53}


def spec(recipe: str, **overrides) -> Spec:
    """The full-size workload ``recipe``, optionally with shape fields replaced."""
    return dataclasses.replace(RECIPES[recipe], **overrides)


def _mix(*parts: int) -> int:
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h ^= (int(p) + 0x632BE59BD9B4E019 + ((h << 6) & (2**64 - 1)) + (h >> 2)) & (2**64 - 1)
        h = (h * 0xBF58476D1CE4E5B9) & (2**64 - 1)
    return h & (2**63 - 1)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def generate_idx(sp: Spec, seed: int = 0) -> torch.Tensor:
    """Dictionary index arrays idx[K][N] (int32)."""
    g = _gen(_mix(seed, _SALT[sp.recipe], 0xD1C7))
    if sp.recipe == "z5":
        # cyclic shifts by 0..K-1: idx_k[j] = (j + k) mod N
        j = torch.arange(sp.N)
        return torch.stack([(j + k) % sp.N for k in range(sp.K)]).to(torch.int32)
    if sp.recipe == "long":
        return torch.stack([torch.randperm(sp.N, generator=g) for _ in range(sp.K)]).to(torch.int32)
    return torch.randint(0, sp.N, (sp.K, sp.N), generator=g).to(torch.int32)


def generate_slice(sp: Spec, b: int, h: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Inputs of one (batch b, head h) slice: logits [L,K], d [L,N], B [L,N], C [L,N], x [L,P]."""
    L, N, P, K = sp.seqlen, sp.N, sp.P, sp.K
    g = _gen(_mix(seed, _SALT[sp.recipe], b, h))
    if sp.recipe == "z5":
        tokens = torch.randint(0, K, (L,), generator=g)
        logits = torch.nn.functional.one_hot(tokens, K).to(torch.float32)
        d = torch.ones(L, N)
        B = torch.zeros(L, N)
        B[0, 0] = 1.0
        C = torch.nn.functional.one_hot(torch.arange(L) % N, N).to(torch.float32)
        x = torch.ones(L, P)
    else:
        logits = torch.randn(L, K, generator=g)
        if sp.recipe == "tiny":
            d = 0.5 + 0.5 * torch.rand(L, N, generator=g)
        elif sp.recipe == "complex":
            r = torch.exp(-torch.nn.functional.softplus(torch.randn(L, N, generator=g)))
            theta = 2.0 * math.pi * torch.rand(L, N, generator=g)
            d = torch.polar(r, theta)
        else:
            d = torch.exp(-torch.nn.functional.softplus(torch.randn(L, N, generator=g)))
        if sp.recipe == "lm":
            std = 1.0 / math.sqrt(N)
            B = std * torch.randn(L, N, generator=g)
            C = std * torch.randn(L, N, generator=g)
        else:
            B = torch.randn(L, N, generator=g)
            C = torch.randn(L, N, generator=g)
        x = torch.randn(L, P, generator=g)
    return {
        "logits": logits.to(sp.logits_dtype),
        "d": d.to(sp.d_dtype),
        "B": B.to(sp.in_dtype),
        "C": C.to(sp.in_dtype),
        "x": x.to(sp.in_dtype),
    }


def _slices(sp: Spec) -> Iterable[Tuple[int, int]]:
    for b in range(sp.batch):
        for h in range(sp.heads):
            yield b, h


def generate(sp: Spec, seed: int = 0, device: Optional[torch.device] = None) -> Dict[str, torch.Tensor]:
    """All inputs of a workload, in the [Bt, L, H, *] layout, on ``device`` (CPU by default).

    Slices are generated one at a time on the CPU and copied into place, so the
    host never holds more than one slice of temporaries.
    """
    dev = torch.device("cpu") if device is None else torch.device(device)
    Bt, L, H, N, P, K = sp.batch, sp.seqlen, sp.heads, sp.N, sp.P, sp.K
    out = {
        "idx": generate_idx(sp, seed).to(dev),
        "logits": torch.empty(Bt, L, H, K, dtype=sp.logits_dtype, device=dev),
        "d": torch.empty(Bt, L, H, N, dtype=sp.d_dtype, device=dev),
        "B": torch.empty(Bt, L, H, N, dtype=sp.in_dtype, device=dev),
        "C": torch.empty(Bt, L, H, N, dtype=sp.in_dtype, device=dev),
        "x": torch.empty(Bt, L, H, P, dtype=sp.in_dtype, device=dev),
    }
    for b, h in _slices(sp):
        sl = generate_slice(sp, b, h, seed)
        for k, v in sl.items():
            out[k][b, :, h].copy_(v, non_blocking=False)
    return out


def generate_on_device(sp: Spec, seed: int = 0, device: Optional[torch.device] = None) -> Dict[str, torch.Tensor]:
    """The workload's recipe drawn directly on ``device`` (one generator there, whole
    tensors at once): the same shapes, dtypes, structure and distributions as
    ``generate`` but not the same numbers. For timing the largest workloads without
    building them on the host; parity tests use ``generate``."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    Bt, L, H, N, P, K = sp.batch, sp.seqlen, sp.heads, sp.N, sp.P, sp.K
    g = torch.Generator(device=dev)
    g.manual_seed(_mix(seed, _SALT[sp.recipe], 0xDE71CE))
    out = {"idx": generate_idx(sp, seed).to(dev)}
    if sp.recipe == "z5":
        tokens = torch.randint(0, K, (Bt, L, H), generator=g, device=dev)
        out["logits"] = torch.nn.functional.one_hot(tokens, K).to(sp.logits_dtype)
        out["d"] = torch.ones(Bt, L, H, N, device=dev).to(sp.d_dtype)
        Bv = torch.zeros(Bt, L, H, N, device=dev)
        Bv[:, 0, :, 0] = 1.0
        out["B"] = Bv.to(sp.in_dtype)
        out["C"] = torch.nn.functional.one_hot(torch.arange(L, device=dev) % N, N).to(sp.in_dtype)[None, :, None, :] \
            .expand(Bt, L, H, N).contiguous()
        out["x"] = torch.ones(Bt, L, H, P, device=dev).to(sp.in_dtype)
        return out
    out["logits"] = torch.randn(Bt, L, H, K, generator=g, device=dev).to(sp.logits_dtype)
    z = torch.randn(Bt, L, H, N, generator=g, device=dev)
    if sp.recipe == "tiny":
        d = 0.5 + 0.5 * torch.rand(Bt, L, H, N, generator=g, device=dev)
    elif sp.recipe == "complex":
        r = torch.exp(-torch.nn.functional.softplus(z))
        d = torch.polar(r, 2.0 * math.pi * torch.rand(Bt, L, H, N, generator=g, device=dev))
    else:
        d = torch.exp(-torch.nn.functional.softplus(z))
    out["d"] = d.to(sp.d_dtype)
    del z, d
    std = 1.0 / math.sqrt(N) if sp.recipe == "lm" else 1.0
    for k, X in (("B", N), ("C", N), ("x", P)):
        v = torch.randn(Bt, L, H, X, generator=g, device=dev)
        if k != "x":
            v.mul_(std)
        out[k] = v.to(sp.in_dtype)
    return out
