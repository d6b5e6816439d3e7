"""Failure detection on the GPU without a fault: the fused kernel's bounded waits.

Every wait of one role of the fused kernel on another is bounded. With
PDSSM_FLAG_SHORT_WAITS the bound is about a microsecond, far shorter than the
time the first sub-chunk's preparation takes, so a wait runs out on purpose:
the kernel must record PDSSM_ERR_TIMEOUT in the workspace's error word, return
(no trap, no hang, tensor memory freed), and leave the device usable, so that
the very next normal call reproduces a clean run bit for bit.
"""
import pytest
import torch

import structured_sparse_selective_b200 as pd
import workloads

pytestmark = pytest.mark.gpu

PDSSM_OK, PDSSM_ERR_TIMEOUT = 0, 6


def _call(inp, pb, ws, out):
    pd.pdssm_forward(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None, out["y"],
                     out["h_final"], out["prod_idx"], out["prod_val"], out["s"], ws)


def _outputs(sp, dev):
    return {"y": torch.empty(sp.batch, sp.seqlen, sp.heads, sp.P, dtype=sp.out_dtype, device=dev),
            "h_final": torch.empty(sp.batch, sp.heads, sp.N, sp.P, dtype=torch.float32, device=dev),
            "prod_idx": torch.empty(sp.batch, sp.heads, sp.N, dtype=torch.int32, device=dev),
            "prod_val": torch.empty(sp.batch, sp.heads, sp.N, dtype=torch.float32, device=dev),
            "s": torch.empty(sp.batch, sp.seqlen, sp.heads, dtype=torch.int32, device=dev)}


def test_short_waits_report_a_timeout_and_the_next_call_is_clean(cuda_device):
    sp = workloads.spec("lm", batch=2, seqlen=512, heads=4)
    inp = {k: v.to(cuda_device) for k, v in workloads.generate(sp, seed=12).items()}
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"])
    ws = pd.alloc_workspace(pb, cuda_device)
    clean = _outputs(sp, cuda_device)
    _call(inp, pb, ws, clean)
    assert pd.pdssm_read_device_check(ws) == PDSSM_OK

    short = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"], flags=pd.FLAG_SHORT_WAITS)
    for _ in range(2):
        _call(inp, short, ws, _outputs(sp, cuda_device))
        assert pd.pdssm_read_device_check(ws) == PDSSM_ERR_TIMEOUT
    torch.cuda.synchronize()  # the context is still usable

    again = _outputs(sp, cuda_device)
    _call(inp, pb, ws, again)
    assert pd.pdssm_read_device_check(ws) == PDSSM_OK
    for k in clean:
        assert torch.equal(again[k], clean[k]), k


def test_short_waits_flag_is_accepted_by_the_three_kernel_path(cuda_device):
    """The three-kernel path has no inter-role waits: the flag changes nothing there."""
    sp = workloads.spec("tiny", batch=1, seqlen=100)
    inp = {k: v.to(cuda_device) for k, v in workloads.generate(sp, seed=2).items()}
    a = pd.forward(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    b = pd.forward(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], flags=pd.FLAG_SHORT_WAITS)
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), k
