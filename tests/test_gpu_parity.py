"""GPU parity: the CUDA path, called through the C ABI, against the oracle.

Small cases compare every output element; the full-size workloads compare
sampled (batch, head) slices (whole sequences) plus properties that hold on
every slice (bit-exact selections, composed index arrays).
"""
import numpy as np
import pytest
import torch

import oracle
import structured_sparse_selective_b200 as pd
import workloads
from tests.parity import (TOL, bhl_to_slices, compare_full, run_gpu, sampled_slices, slice_rel_err,
                          sparse_prod_all_slices, to_np)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------- select

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("K", [1, 2, 5, 16, 33, 64])
def test_select_bit_exact(cuda_device, dtype, K):
    g = torch.Generator().manual_seed(K)
    lg = torch.randn(3, 1001, 2, K, generator=g).to(dtype)
    if K > 1:  # plant ties, signed zeros and NaNs
        lg[0, :50, 0, :] = 0.5
        lg[0, 50:100, 0, : K // 2] = -0.0
        lg[0, 50:100, 0, K // 2:] = 0.0
        lg[1, :20, 1, K // 2] = float("nan")
        lg[1, 20:40, 1, :] = float("nan")
        lg[2, :30, 0, -1] = float("inf")
    pb = pd.Problem(batch=3, seqlen=1001, heads=2, N=4, P=4, K=K, chunk=0,
                    logits_t=pd.BF16 if dtype == torch.bfloat16 else pd.F32, in_t=pd.F32,
                    d_t=pd.F32, state_t=pd.F32, out_t=pd.F32, flags=0)
    s = torch.full((3, 1001, 2), -7, dtype=torch.int32, device=cuda_device)
    pd.pdssm_select(pb, lg.to(cuda_device), s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), oracle.select(lg))


# --------------------------------------------------------- small, element-wise

SMALL = [
    ("tiny", dict()),
    ("tiny", dict(seqlen=37, batch=2, heads=3)),
    ("z5", dict(batch=8, seqlen=133)),
    ("lm", dict(batch=2, seqlen=300, heads=3)),
    ("long", dict(batch=2, seqlen=517, heads=2)),
    ("complex", dict(batch=1, seqlen=150, heads=2)),
    ("complex", dict(batch=2, seqlen=70, heads=1, N=16, P=8, K=5)),
]


@pytest.mark.parametrize("recipe,kw", SMALL)
@pytest.mark.parametrize("chunk", [0, 1, 7, 64, 1000])
def test_small_workloads_match_oracle(cuda_device, recipe, kw, chunk):
    sp = workloads.spec(recipe, **kw)
    inp = workloads.generate(sp, seed=3)
    out = run_gpu(inp, cuda_device, chunk=chunk)
    compare_full(inp, out)


@pytest.mark.parametrize("recipe,kw", [("lm", dict(batch=2, seqlen=129, heads=2)),
                                       ("complex", dict(batch=1, seqlen=77, heads=2, N=32, P=16, K=8)),
                                       ("long", dict(batch=1, seqlen=100, heads=2))])
def test_initial_state(cuda_device, recipe, kw):
    sp = workloads.spec(recipe, **kw)
    inp = workloads.generate(sp, seed=4)
    g = torch.Generator().manual_seed(9)
    shape = (sp.batch, sp.heads, sp.N, sp.P)
    h0 = torch.randn(*shape, generator=g)
    if sp.state_complex:
        h0 = torch.complex(h0, torch.randn(*shape, generator=g))
    for chunk in (0, 13):
        out = run_gpu(inp, cuda_device, chunk=chunk, h0=h0)
        compare_full(inp, out, h0=h0)


def test_scan_entry_equals_forward_entry(cuda_device):
    sp = workloads.spec("lm", batch=2, seqlen=200, heads=2)
    inp = workloads.generate(sp, seed=5)
    a = run_gpu(inp, cuda_device, chunk=64)
    b = run_gpu(inp, cuda_device, chunk=64, via_scan=True)
    for k in ("y", "h_final", "prod_idx", "prod_val", "s"):
        assert torch.equal(a[k], b[k]), k


def test_segmented_run_equals_whole_run(cuda_device):
    sp = workloads.spec("long", batch=1, seqlen=300, heads=2)
    inp = workloads.generate(sp, seed=6)
    whole = run_gpu(inp, cuda_device)
    first = {k: (v[:, :123] if v.dim() == 4 else v) for k, v in inp.items()}
    second = {k: (v[:, 123:].contiguous() if v.dim() == 4 else v) for k, v in inp.items()}
    a = run_gpu(first, cuda_device)
    b = run_gpu(second, cuda_device, h0=a["h_final"].cpu())
    y = torch.cat([a["y"], b["y"]], dim=1)
    assert slice_rel_err(bhl_to_slices(to_np(y)), bhl_to_slices(to_np(whole["y"]))) < 1e-5
    assert slice_rel_err(to_np(b["h_final"]).reshape(2, -1), to_np(whole["h_final"]).reshape(2, -1)) < 1e-5


# --------------------------------------------------------------- edge cases

@pytest.mark.parametrize("kw", [dict(seqlen=0), dict(batch=0), dict(heads=0)])
def test_empty_problems(cuda_device, kw):
    sp = workloads.spec("tiny", **kw)
    inp = workloads.generate(sp)
    h0 = torch.randn(sp.batch, sp.heads, sp.N, sp.P)
    out = run_gpu(inp, cuda_device, h0=h0 if sp.batch * sp.heads else None)
    if sp.seqlen == 0:
        assert torch.equal(out["h_final"].cpu(), h0)
        assert torch.equal(out["prod_idx"].cpu(), torch.arange(sp.N, dtype=torch.int32).expand(1, 1, -1))
        assert torch.equal(out["prod_val"].cpu(), torch.ones(1, 1, sp.N))


@pytest.mark.parametrize("kw", [
    dict(N=1, P=1, K=1, seqlen=40),
    dict(N=1, P=7, K=3, seqlen=40),
    dict(N=9, P=1, K=1, seqlen=40),
    dict(seqlen=1),
    dict(N=128, P=128, K=64, seqlen=70),
    dict(N=128, P=128, K=64, seqlen=70, batch=2),
])
def test_degenerate_and_maximum_sizes(cuda_device, kw):
    sp = workloads.spec("tiny", **kw)
    inp = workloads.generate(sp, seed=7)
    for chunk in (0, 5):
        compare_full(inp, run_gpu(inp, cuda_device, chunk=chunk))


def test_maximum_sizes_complex(cuda_device):
    sp = workloads.spec("complex", batch=1, heads=1, seqlen=40, N=128, P=128, K=64)
    inp = workloads.generate(sp, seed=8)
    compare_full(inp, run_gpu(inp, cuda_device, chunk=16))


def test_out_of_range_indices_are_flagged_not_faulted(cuda_device):
    sp = workloads.spec("tiny", seqlen=50)
    inp = workloads.generate(sp)
    ok = run_gpu(inp, cuda_device, flags=pd.FLAG_DEVICE_CHECK)  # clean input: no error
    assert torch.isfinite(ok["y"]).all()
    bad = dict(inp)
    bad["idx"] = inp["idx"].clone()
    bad["idx"][1, 3] = sp.N + 5
    bad["idx"][2, 0] = -1
    with pytest.raises(pd.PdssmError) as e:
        run_gpu(bad, cuda_device, flags=pd.FLAG_DEVICE_CHECK)
    assert e.value.status == 5
    # out-of-range selections through the scan entry
    dev = cuda_device
    g = {k: v.to(dev) for k, v in inp.items()}
    pb = pd.make_problem(g["logits"], g["d"], g["B"], g["x"])
    s = torch.full((1, 50, 1), sp.K + 3, dtype=torch.int32, device=dev)
    y = torch.empty(1, 50, 1, sp.P, device=dev)
    ws = pd.alloc_workspace(pb, dev)
    pd.pdssm_scan_fwd(pb, s, g["idx"], g["d"], g["B"], g["C"], g["x"], None, y, None, None, None, ws)
    assert pd.pdssm_read_device_check(ws) == 5
    assert torch.isfinite(y).all()


def test_bf16_and_mixed_dtypes(cuda_device):
    sp = workloads.spec("tiny", batch=2, seqlen=90, heads=2, N=16, P=8, K=6)
    base = workloads.generate(sp, seed=10)
    for ddt in (torch.float32, torch.bfloat16):
        for idt in (torch.float32, torch.bfloat16):
            for ldt in (torch.float32, torch.bfloat16):
                inp = dict(base)
                inp["d"] = base["d"].to(ddt)
                for k in ("B", "C", "x"):
                    inp[k] = base[k].to(idt)
                inp["logits"] = base["logits"].to(ldt)
                for odt in (torch.float32, torch.bfloat16):
                    g = {k: v.to(cuda_device) for k, v in inp.items()}
                    out = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], out_dtype=odt,
                                     want_s=True)
                    torch.cuda.synchronize()
                    compare_full(inp, out)


# --------------------------------------------------- full-size workloads

FULL = {  # recipe -> (slices checked against the oracle at full length)
    "tiny": None, "z5": None, "lm": 6, "long": 6, "complex": 2,
}


@pytest.mark.parametrize("recipe", workloads.CONFIG_ORDER)
def test_full_size_workload(cuda_device, recipe):
    sp = workloads.spec(recipe)
    inp = workloads.generate(sp, device=cuda_device)
    out = pd.forward(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], want_s=True)
    torch.cuda.synchronize()
    idx = inp["idx"].cpu().numpy()
    # selections: bit-exact on every row (oracle in batch-sized pieces)
    s_ref = np.concatenate([oracle.select(inp["logits"][b:b + 1].cpu()) for b in range(sp.batch)])
    s_gpu = to_np(out["s"])
    assert np.array_equal(s_gpu, s_ref)
    # composed index arrays: bit-exact on every slice
    assert np.array_equal(to_np(out["prod_idx"]), sparse_prod_all_slices(s_ref, idx, sp.N))
    n = FULL[recipe]
    if n is None:
        host = {k: v.cpu() for k, v in inp.items()}
        del inp
        compare_full(host, {k: v for k, v in out.items()})
        return
    picks = sampled_slices(sp, n)
    tol = TOL[out["y"].dtype]
    sls = [workloads.generate_slice(sp, b, h) for b, h in picks]
    for (b, h), sl in zip(picks, sls):
        # the sample regenerated on the host equals what the device holds
        assert torch.equal(sl["x"], inp["x"][b, :, h].cpu())
    stack = {k: torch.stack([sl[k] for sl in sls]) for k in sls[0]}
    r = oracle.scan_slices(stack["logits"], idx, stack["d"], stack["B"], stack["C"], stack["x"])
    for i, (b, h) in enumerate(picks):
        ey = slice_rel_err(to_np(out["y"][b, :, h])[None], r["y"][i:i + 1])
        eh = slice_rel_err(to_np(out["h_final"][b, h])[None], r["h_final"][i:i + 1])
        ep = slice_rel_err(to_np(out["prod_val"][b, h])[None], r["prod_val"][i:i + 1])
        assert np.array_equal(to_np(out["prod_idx"][b, h]), r["prod_idx"][i])
        assert ey <= tol and eh <= 1e-4 and ep <= 1e-4, (b, h, ey, eh, ep)


# ------------------------------------------- fused single-kernel path (N = P = 64, bf16)

FUSED = [
    dict(batch=1, seqlen=1, heads=1),
    dict(batch=1, seqlen=15, heads=2),
    dict(batch=1, seqlen=16, heads=1),
    dict(batch=2, seqlen=17, heads=1),
    dict(batch=1, seqlen=100, heads=3),
    dict(batch=3, seqlen=257, heads=2),
]


@pytest.mark.parametrize("kw", FUSED)
def test_fused_path_matches_oracle(cuda_device, kw):
    sp = workloads.spec("lm", **kw)
    inp = workloads.generate(sp, seed=11)
    compare_full(inp, run_gpu(inp, cuda_device, chunk=0))


def test_fused_path_with_initial_state_and_selection_entry(cuda_device):
    sp = workloads.spec("lm", batch=2, seqlen=99, heads=2)
    inp = workloads.generate(sp, seed=12)
    h0 = torch.randn(sp.batch, sp.heads, sp.N, sp.P, generator=torch.Generator().manual_seed(3))
    a = run_gpu(inp, cuda_device, chunk=0, h0=h0)
    compare_full(inp, a, h0=h0)
    b = run_gpu(inp, cuda_device, chunk=0, h0=h0, via_scan=True)  # selections given
    for k in ("y", "h_final", "prod_idx", "prod_val", "s"):
        assert torch.equal(a[k], b[k]), k


def test_fused_path_is_deterministic_and_agrees_with_reference_path(cuda_device):
    sp = workloads.spec("lm", batch=2, seqlen=200, heads=2)
    inp = workloads.generate(sp, seed=13)
    a = run_gpu(inp, cuda_device, chunk=0)
    b = run_gpu(inp, cuda_device, chunk=0)
    for k in ("y", "h_final", "prod_idx", "prod_val", "s"):
        assert torch.equal(a[k], b[k]), k
    r = run_gpu(inp, cuda_device, chunk=0, flags=pd.FLAG_REFERENCE_PATH)
    assert torch.equal(a["s"], r["s"]) and torch.equal(a["prod_idx"], r["prod_idx"])
    assert slice_rel_err(to_np(a["h_final"]).reshape(4, -1), to_np(r["h_final"]).reshape(4, -1)) < 1e-5


@pytest.mark.parametrize("dictionary", ["permutation", "identity", "constant"])
def test_fused_path_dictionary_shapes(cuda_device, dictionary):
    sp = workloads.spec("lm", batch=1, seqlen=150, heads=2)
    inp = workloads.generate(sp, seed=14)
    g = torch.Generator().manual_seed(5)
    if dictionary == "permutation":
        inp["idx"] = torch.stack([torch.randperm(64, generator=g) for _ in range(sp.K)]).to(torch.int32)
    elif dictionary == "identity":
        inp["idx"] = torch.arange(64, dtype=torch.int32).repeat(sp.K, 1)
    else:  # every column into one row: maximal collisions
        inp["idx"] = torch.full((sp.K, 64), 7, dtype=torch.int32)
    compare_full(inp, run_gpu(inp, cuda_device, chunk=0))


@pytest.mark.parametrize("ldt,odt", [(torch.float32, torch.bfloat16), (torch.bfloat16, torch.float32),
                                     (torch.float32, torch.float32)])
def test_fused_path_logit_and_output_dtypes(cuda_device, ldt, odt):
    sp = workloads.spec("lm", batch=1, seqlen=70, heads=2)
    inp = workloads.generate(sp, seed=15)
    inp["logits"] = inp["logits"].to(ldt)
    g = {k: v.to(cuda_device) for k, v in inp.items()}
    out = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], out_dtype=odt, want_s=True)
    torch.cuda.synchronize()
    compare_full(inp, out)


# ------------------------------------------- recurrent decode: one token per call

@pytest.mark.parametrize("recipe,kw", [("lm", dict(batch=2, seqlen=40, heads=2)),
                                       ("tiny", dict(batch=1, seqlen=33, heads=2))])
def test_token_by_token_decode_matches_the_whole_sequence(cuda_device, recipe, kw):
    """Decoding one step at a time (L = 1, the state carried through h0 -> h_final)
    gives the outputs and final state of the whole-sequence forward pass, which is the
    oracle's recurrence read one step at a time."""
    sp = workloads.spec(recipe, **kw)
    inp = workloads.generate(sp, seed=16)
    g = {k: v.to(cuda_device) for k, v in inp.items()}
    whole = pd.forward(g["logits"], g["idx"], g["d"], g["B"], g["C"], g["x"], out_dtype=torch.float32,
                       want_s=True)
    h = torch.zeros(sp.batch, sp.heads, sp.N, sp.P, dtype=torch.float32, device=cuda_device)
    ys, ss = [], []
    for t in range(sp.seqlen):
        step = {k: g[k][:, t:t + 1].contiguous() for k in ("logits", "d", "B", "C", "x")}
        o = pd.forward(step["logits"], g["idx"], step["d"], step["B"], step["C"], step["x"], h0=h,
                       out_dtype=torch.float32, want_s=True)
        ys.append(o["y"])
        ss.append(o["s"])
        h = o["h_final"]
    torch.cuda.synchronize(cuda_device)
    y = torch.cat(ys, dim=1)
    assert torch.equal(torch.cat(ss, dim=1), whole["s"])
    scale = whole["y"].abs().amax().item()
    assert (y - whole["y"]).abs().amax().item() <= 1e-4 * scale
    hs = whole["h_final"].abs().amax().item()
    assert (h - whole["h_final"]).abs().amax().item() <= 1e-4 * hs
    compare_full(inp, {"y": y.cpu(), "h_final": h.cpu()})


def test_fused_path_reports_no_device_error_across_repeated_launches(cuda_device):
    """The fused kernel's bounded waits never give up on the LM workload: the device
    check word stays clear over repeated full-size launches (a stall that the bounded
    waits caught would set its timeout bit)."""
    sp = workloads.spec("lm")
    inp = workloads.generate(sp, seed=17, device=cuda_device)
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"])
    ws = pd.alloc_workspace(pb, cuda_device)
    for _ in range(8):
        out = pd.forward(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], workspace=ws)
        assert pd.pdssm_read_device_check(ws) == 0  # PDSSM_OK
    assert torch.isfinite(out["y"].float()).all()


@pytest.mark.gpu
@pytest.mark.parametrize("chunk", [0, 1, 3])
@pytest.mark.parametrize("via_scan", [False, True])
def test_hand_worked_automaton_runs(cuda_device, chunk, via_scan):
    """The C-ABI reproduces the hand-worked automaton runs of tests/golden exactly
    (Proposition 1 of the Flash PD-SSM summary page): selections, every output,
    the final state and the composed product."""
    from tests import golden
    for name in golden.names():
        inp, exp = golden.load(name)
        out = run_gpu(inp, cuda_device, chunk=chunk, via_scan=via_scan)
        assert out["s"][0, :, 0].tolist() == exp["s"], name
        assert out["y"][0, :, 0, 0].tolist() == exp["y"], name
        assert out["h_final"][0, 0, :, 0].tolist() == exp["h_final"], name
        assert out["prod_idx"][0, 0].tolist() == exp["prod_idx"], name
        assert out["prod_val"][0, 0].tolist() == exp["prod_val"], name


# ------------------------------------------------------- per-head dictionaries

@pytest.mark.parametrize("recipe,kw,chunk", [
    ("lm", dict(batch=2, seqlen=300, heads=3), 0),            # the fused kernel
    ("lm", dict(batch=1, seqlen=100, heads=2), 7),            # the three-kernel path
    ("tiny", dict(batch=2, seqlen=90, heads=3), 0),
    ("long", dict(batch=1, seqlen=130, heads=3), 16),
    ("complex", dict(batch=1, seqlen=60, heads=2, N=16, P=8, K=5), 0),
])
def test_per_head_dictionaries_match_oracle(cuda_device, recipe, kw, chunk):
    """Methodology 4 (multi-head layers): a dictionary per head, idx [H, K, N]."""
    sp = workloads.spec(recipe, **kw)
    inp = workloads.generate(sp, seed=9)
    g = torch.Generator().manual_seed(5)
    inp["idx"] = torch.randint(0, sp.N, (sp.heads, sp.K, sp.N), generator=g).to(torch.int32)
    out = run_gpu(inp, cuda_device, chunk=chunk)
    compare_full(inp, out)
    # the selection-given entry point too
    compare_full(inp, run_gpu(inp, cuda_device, chunk=chunk, via_scan=True))
