"""Parity of the backward pass (pdssm_scan_bwd through the C ABI) with the backward
oracle (oracle/backward.py) on seeded workloads, real and complex states: every
gradient, per (batch, head) slice, within 1e-4 of the slice's largest value."""
import numpy as np
import pytest
import torch

import structured_sparse_selective_b200 as pd
import workloads
from oracle import backward as bwd

TOL = 1e-4


def _np64(t):
    """fp64 (or complex128) numpy copy of a tensor"""
    t = t.detach().cpu()
    return (t.to(torch.complex128) if t.is_complex() else t.double()).numpy()


def _slices(t):
    """[Bt, L, H, X] -> [Bt*H, L, X] fp64 / complex128 numpy"""
    Bt, L, H, X = t.shape
    return _np64(t.permute(0, 2, 1, 3).reshape(Bt * H, L, X))


def _rel(got, ref):
    scale = np.abs(ref).max(axis=tuple(range(1, ref.ndim)), keepdims=True)
    return float((np.abs(got - ref) / np.maximum(scale, 1e-30)).max()) if ref.size else 0.0


def _run(recipe, kw, dev, seed=0, with_h0=True, with_dh=True, with_logits=True, tau=0.7, head_dicts=False):
    sp = workloads.spec(recipe, **kw)
    inp = workloads.generate(sp, seed=seed)
    if head_dicts:  # a dictionary per head [H, K, N]
        g = torch.Generator().manual_seed(40 + seed)
        inp["idx"] = torch.randint(0, sp.N, (sp.heads, sp.K, sp.N), generator=g).to(torch.int32)
    g = {k: v.to(dev) for k, v in inp.items()}
    # the forward pass gives the selections (they do not depend on h0)
    fwd = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], want_s=True, want_prod=False)
    Bt, L, H, N = inp["B"].shape
    P = inp["x"].shape[-1]
    gen = torch.Generator().manual_seed(100 + seed)
    sdt = torch.complex64 if sp.state_complex else torch.float32  # complex draws have both parts
    dy = torch.randn(Bt, L, H, P, generator=gen, dtype=sdt).to(fwd["y"].dtype)
    h0 = torch.randn(Bt, H, N, P, generator=gen, dtype=sdt) if with_h0 else None
    dh = torch.randn(Bt, H, N, P, generator=gen, dtype=sdt) if with_dh else None
    out = pd.backward(g["logits"] if with_logits else None, fwd["s"], g["idx"], g["d"], g["B"], g["C"], g["x"],
                      dy.to(dev), h0=None if h0 is None else h0.to(dev), dh_final=None if dh is None else dh.to(dev),
                      tau=tau)
    torch.cuda.synchronize(dev)
    S = Bt * H
    idx_ref = inp["idx"].numpy()
    if idx_ref.ndim == 3:  # slice b * H + h uses head h's dictionary
        idx_ref = np.stack([idx_ref[i % H] for i in range(Bt * H)])
    ref = bwd.scan_backward(_slices(inp["logits"]), idx_ref, _slices(inp["d"]), _slices(inp["B"]),
                            _slices(inp["C"]), _slices(inp["x"]), _slices(dy),
                            None if dh is None else _np64(dh.reshape(S, N, P)),
                            None if h0 is None else _np64(h0.reshape(S, N, P)), tau=tau)
    s_slices = fwd["s"].cpu().permute(0, 2, 1).reshape(S, L).numpy()
    assert np.array_equal(s_slices, ref["s"])
    errs = {}
    for k in ("dd", "dB", "dC", "dx") + (("dlogits",) if with_logits else ()):
        errs[k] = _rel(_slices(out[k]), ref[k])
    errs["dh0"] = _rel(_np64(out["dh0"].reshape(S, N, P)), ref["dh0"])
    if sp.state_complex:  # the complex gradients carry imaginary parts, the rest are real
        assert out["dd"].dtype == torch.complex64 and out["dh0"].dtype == torch.complex64
        assert np.abs(ref["dd"].imag).max() > 1e-3 * np.abs(ref["dd"]).max()
        assert np.abs(ref["dh0"].imag).max() > 1e-3 * np.abs(ref["dh0"]).max()
        assert all(out[k].dtype == torch.float32 for k in ("dB", "dC", "dx"))
    return errs


@pytest.mark.gpu
@pytest.mark.parametrize("recipe,kw", [
    ("tiny", dict()),
    ("tiny", dict(seqlen=1)),
    ("tiny", dict(seqlen=15)),
    ("z5", dict(batch=3, seqlen=37)),
    ("lm", dict(batch=1, seqlen=70, heads=2)),
    ("long", dict(batch=1, seqlen=53, heads=2)),
    ("complex", dict(batch=1, seqlen=45, heads=2, N=16, P=8, K=8)),
    ("complex", dict(batch=2, seqlen=17, heads=1, N=40, P=24, K=12)),
])
def test_backward_matches_oracle(cuda_device, recipe, kw):
    errs = _run(recipe, kw, cuda_device)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_without_initial_state_final_gradient_or_logits(cuda_device):
    errs = _run("lm", dict(batch=1, seqlen=33, heads=2), cuda_device, seed=3, with_h0=False, with_dh=False,
                with_logits=False)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_maximum_sizes(cuda_device):
    """N = P = 128, K = 64: the largest shared-memory footprint of the backward block."""
    sp = dict(batch=1, seqlen=20, heads=1, N=128, P=128, K=64)
    errs = _run("tiny", sp, cuda_device, seed=4)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_complex_maximum_sizes(cuda_device):
    """Complex state at N = 128, P = 64, K = 64 (the complex-diagonal layer's head shape): the
    largest complex footprint the backward block holds (three 128 x 65 complex buffers)."""
    errs = _run("complex", dict(batch=1, seqlen=20, heads=1), cuda_device, seed=8)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
@pytest.mark.parametrize("recipe,kw", [
    ("lm", dict(batch=150, seqlen=10, heads=2)),                        # 300 sequences: whole rows
    ("complex", dict(batch=300, seqlen=12, heads=1, N=16, P=8, K=4)),   # 300 sequences: whole rows
    ("complex", dict(batch=1, seqlen=10, heads=1, N=128, P=128, K=64)),  # rows split to fit
])
def test_backward_whole_and_split_column_blocks(cuda_device, recipe, kw):
    """With about two sequences per SM or more a block owns whole state rows; with fewer,
    or when a whole row does not fit in shared memory, a sequence's columns are split over
    blocks whose shares of the column sums a second kernel adds. Both match the oracle."""
    errs = _run(recipe, kw, cuda_device, seed=10)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_complex_without_initial_state_or_logits(cuda_device):
    errs = _run("complex", dict(batch=1, seqlen=33, heads=2, N=32, P=16, K=8), cuda_device, seed=9,
                with_h0=False, with_dh=False, with_logits=False)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_empty_sequence_passes_the_final_gradient_through(cuda_device):
    dev = cuda_device
    Bt, H, N, P, K = 2, 3, 8, 4, 4
    z = lambda *s: torch.zeros(*s, device=dev)
    dh = torch.randn(Bt, H, N, P, device=dev)
    out = pd.backward(z(Bt, 0, H, K), torch.zeros(Bt, 0, H, dtype=torch.int32, device=dev),
                      torch.zeros(K, N, dtype=torch.int32, device=dev), z(Bt, 0, H, N), z(Bt, 0, H, N),
                      z(Bt, 0, H, N), z(Bt, 0, H, P), z(Bt, 0, H, P), dh_final=dh)
    torch.cuda.synchronize(dev)
    assert torch.equal(out["dh0"], dh)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["fsa_advance_merge_weighted"])
def test_backward_reproduces_the_hand_worked_gradients(cuda_device, name):
    """pdssm_scan_bwd on the weighted automaton fixture (loss sum_t y_t: dy = 1, no final-state
    gradient, no logits): every gradient is a small integer worked by hand in the fixture header
    and exact in fp32, so the C ABI must return it exactly."""
    from tests import golden
    inp, exp = golden.load(name)
    g = {k: v.to(cuda_device) for k, v in inp.items()}
    fwd = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], want_s=True, want_prod=False)
    assert fwd["s"][0, :, 0].tolist() == exp["s"]
    dy = torch.ones_like(fwd["y"])
    out = pd.backward(None, fwd["s"], g["idx"], g["d"], g["B"], g["C"], g["x"], dy)
    torch.cuda.synchronize()
    assert out["dC"][0, :, 0].tolist() == exp["bwd_dC"]
    assert out["dB"][0, :, 0].tolist() == exp["bwd_dB"]
    assert out["dd"][0, :, 0].tolist() == exp["bwd_dd"]
    assert out["dx"][0, :, 0, 0].tolist() == exp["bwd_dx"]
    assert out["dh0"][0, 0, :, 0].tolist() == exp["bwd_dh0"]


@pytest.mark.gpu
@pytest.mark.parametrize("recipe,kw", [("lm", dict(batch=2, seqlen=40, heads=3)), ("tiny", dict(heads=2, seqlen=50)),
                                       ("complex", dict(batch=1, seqlen=30, heads=3, N=16, P=8, K=8))])
def test_backward_with_per_head_dictionaries(cuda_device, recipe, kw):
    errs = _run(recipe, kw, cuda_device, seed=6, head_dicts=True)
    assert all(v <= TOL for v in errs.values()), errs


@pytest.mark.gpu
def test_backward_full_size_lm_sampled_slices(cuda_device):
    """The backward pass on the whole LM-layer workload (batch 8, L 2048, heads 32), in the
    launch configuration the bench times; three sampled (batch, head) slices, the first and
    the last among them, against the backward oracle (each slice depends on its own inputs
    only)."""
    sp = workloads.spec("lm")
    inp = workloads.generate(sp, seed=12)
    g = {k: v.to(cuda_device) for k, v in inp.items()}
    fwd = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], want_s=True, want_prod=False)
    gen = torch.Generator().manual_seed(112)
    dy = torch.randn(sp.batch, sp.seqlen, sp.heads, sp.P, generator=gen).to(torch.bfloat16)
    out = pd.backward(g["logits"], fwd["s"], g["idx"], g["d"], g["B"], g["C"], g["x"], dy.to(cuda_device), tau=0.8)
    torch.cuda.synchronize(cuda_device)
    idx = inp["idx"].numpy()
    for b, h in [(0, 0), (3, 17), (sp.batch - 1, sp.heads - 1)]:
        sl = {k: _np64(inp[k][b, :, h]) for k in ("logits", "d", "B", "C", "x")}
        ref = bwd.slice_backward(sl["logits"], idx, sl["d"], sl["B"], sl["C"], sl["x"], _np64(dy[b, :, h]), tau=0.8)
        assert np.array_equal(fwd["s"][b, :, h].cpu().numpy(), ref["s"])
        for k in ("dd", "dB", "dC", "dx", "dlogits"):
            got = _np64(out[k][b, :, h])
            err = float(np.abs(got - ref[k]).max() / max(np.abs(ref[k]).max(), 1e-30))
            assert err <= TOL, (b, h, k, err)
        err = float(np.abs(_np64(out["dh0"][b, h]) - ref["dh0"]).max() / max(np.abs(ref["dh0"]).max(), 1e-30))
        assert err <= TOL, (b, h, "dh0", err)
