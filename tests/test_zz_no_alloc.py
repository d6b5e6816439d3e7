"""The allocation-free forward entry point, through the C ABI.

pdssm_forward_noalloc serves callers that cannot allocate device memory on
their call path: it uses a workspace array built into the library's device
image instead of a caller buffer. Its results must match pdssm_forward's, call
after call, because every call reuses the same array.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_selective_b200 as pd
import workloads
from tests.parity import TOL, bhl_to_slices, slice_rel_err, to_np

pytestmark = pytest.mark.gpu


def _outputs(sp, dev):
    sdt = torch.complex64 if sp.state_complex else torch.float32
    return {
        "y": torch.empty(sp.batch, sp.seqlen, sp.heads, sp.P, dtype=sp.out_dtype, device=dev),
        "h_final": torch.empty(sp.batch, sp.heads, sp.N, sp.P, dtype=sdt, device=dev),
        "prod_idx": torch.empty(sp.batch, sp.heads, sp.N, dtype=torch.int32, device=dev),
        "prod_val": torch.empty(sp.batch, sp.heads, sp.N, dtype=sdt, device=dev),
        "s": torch.empty(sp.batch, sp.seqlen, sp.heads, dtype=torch.int32, device=dev),
    }


@pytest.mark.parametrize("recipe,kw", [
    ("lm", dict(batch=2, seqlen=300, heads=2)),      # the fused single-kernel path
    ("tiny", dict(batch=2, seqlen=200, heads=3)),    # the three-kernel path (uses the workspace)
    ("complex", dict(batch=1, seqlen=90, heads=2, N=32, P=16, K=8)),
])
def test_noalloc_matches_forward_on_consecutive_calls(cuda_device, recipe, kw):
    sp = workloads.spec(recipe, **kw)
    host = workloads.generate(sp, seed=21)
    inp = {k: v.to(cuda_device) for k, v in host.items()}
    r = oracle.scan(host["logits"], host["idx"], host["d"], host["B"], host["C"], host["x"])
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"])
    ref = _outputs(sp, cuda_device)
    ws = pd.alloc_workspace(pb, cuda_device)
    pd.pdssm_forward(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None, ref["y"],
                     ref["h_final"], ref["prod_idx"], ref["prod_val"], ref["s"], ws)
    torch.cuda.synchronize()
    S = sp.batch * sp.heads
    for call in range(2):
        out = _outputs(sp, cuda_device)
        pd.pdssm_forward_noalloc(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None,
                                 out["y"], out["h_final"], out["prod_idx"], out["prod_val"], out["s"])
        torch.cuda.synchronize()
        assert torch.equal(out["s"], ref["s"]), call
        assert torch.equal(out["prod_idx"], ref["prod_idx"]), call
        assert slice_rel_err(bhl_to_slices(to_np(out["y"])), bhl_to_slices(to_np(ref["y"]))) <= TOL[sp.out_dtype]
        for k in ("h_final", "prod_val"):
            assert slice_rel_err(to_np(out[k]).reshape(S, -1), to_np(ref[k]).reshape(S, -1)) <= 1e-4, (call, k)
        # and against the oracle itself
        assert np.array_equal(to_np(out["s"]), r["s"]), call
        assert np.array_equal(to_np(out["prod_idx"]), r["prod_idx"]), call
        assert slice_rel_err(bhl_to_slices(to_np(out["y"])), bhl_to_slices(r["y"])) <= TOL[sp.out_dtype], call
        for k in ("h_final", "prod_val"):
            assert slice_rel_err(to_np(out[k]).reshape(S, -1), r[k].reshape(S, -1)) <= 1e-4, (call, k)


def test_noalloc_rejects_problems_beyond_its_workspace(cuda_device):
    """A three-kernel problem whose workspace exceeds the built-in array is refused before launch."""
    # real, full-size buffers: nothing here can make a kernel touch memory it does not own
    sp = workloads.spec("lm", batch=8, seqlen=2048, heads=8)
    g = torch.Generator(device=cuda_device).manual_seed(0)
    inp = {
        "logits": torch.randn(sp.batch, sp.seqlen, sp.heads, sp.K, device=cuda_device, generator=g).to(torch.bfloat16),
        "idx": torch.zeros(sp.K, sp.N, dtype=torch.int32, device=cuda_device),
        "d": torch.full((sp.batch, sp.seqlen, sp.heads, sp.N), 0.5, dtype=torch.bfloat16, device=cuda_device),
        "B": torch.zeros(sp.batch, sp.seqlen, sp.heads, sp.N, dtype=torch.bfloat16, device=cuda_device),
        "C": torch.zeros(sp.batch, sp.seqlen, sp.heads, sp.N, dtype=torch.bfloat16, device=cuda_device),
        "x": torch.zeros(sp.batch, sp.seqlen, sp.heads, sp.P, dtype=torch.bfloat16, device=cuda_device),
    }
    # the three-kernel path needs far more than the built-in 32 MiB at this size
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"], flags=pd.FLAG_REFERENCE_PATH)
    assert pd.pdssm_workspace_size(pb) > 32 << 20
    out = _outputs(sp, cuda_device)
    with pytest.raises(pd.PdssmError) as e:
        pd.pdssm_forward_noalloc(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None,
                                 out["y"], out["h_final"], out["prod_idx"], out["prod_val"], out["s"])
    assert e.value.status == 3  # PDSSM_ERR_WORKSPACE, before anything is enqueued


def test_noalloc_serves_full_size_fused_problems(cuda_device):
    """The fused kernel needs only the error word, so the full LM-layer problem (batch 8, L 2048,
    heads 32) runs allocation-free; its outputs equal pdssm_forward's bit for bit (the fused
    kernel is deterministic), call after call."""
    sp = workloads.spec("lm")
    inp = {k: v.to(cuda_device) for k, v in workloads.generate(sp, seed=5).items()}
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"])
    assert pd.pdssm_workspace_size(pb) <= 256
    ref = _outputs(sp, cuda_device)
    ws = pd.alloc_workspace(pb, cuda_device)
    pd.pdssm_forward(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None, ref["y"],
                     ref["h_final"], ref["prod_idx"], ref["prod_val"], ref["s"], ws)
    torch.cuda.synchronize()
    for call in range(2):
        out = _outputs(sp, cuda_device)
        pd.pdssm_forward_noalloc(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None,
                                 out["y"], out["h_final"], out["prod_idx"], out["prod_val"], out["s"])
        torch.cuda.synchronize()
        for k in ref:
            assert torch.equal(out[k], ref[k]), (call, k)
