"""The dense-selection kernels through the C ABI against oracle/dense_select.py:
dictionary construction (column-wise hardmax, bit-exact) and the fused
projection + selection on the tensor cores (logits within the fp32 accumulation
bound; selections equal wherever the fp64 winner is ahead by more than that
bound, and among the near-tied winners otherwise)."""
import numpy as np
import pytest
import torch

import structured_sparse_selective_b200 as pd
from oracle import dense_select as ds

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K,N", [(1, 1), (4, 8), (16, 64), (5, 100), (64, 128)])
def test_dict_hardmax_is_bit_exact(cuda_device, K, N):
    g = torch.Generator().manual_seed(K * 1000 + N)
    M = torch.randn(K, N, N, generator=g)
    if N > 2:
        M[0] = 0.5                           # all tied: row 0
        M[-1, :, 1] = torch.round(M[-1, :, 1])  # integer ties
        M[-1, 2, 0] = float("nan")
    idx = pd.dict_hardmax(M.to(cuda_device))
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ds.dict_hardmax(M.numpy()))


def test_dict_hardmax_builds_per_head_dictionaries(cuda_device):
    H, K, N = 3, 4, 16
    M = torch.randn(H, K, N, N, generator=torch.Generator().manual_seed(3))
    idx = pd.dict_hardmax(M.to(cuda_device))
    torch.cuda.synchronize()
    assert idx.shape == (H, K, N)
    assert np.array_equal(idx.cpu().numpy(), ds.dict_hardmax(M.numpy()))


def _check_selection(s, lg_ref, bound):
    """s [..., H] from the GPU; lg_ref [..., H, K] fp64; bound [..., H] on the logits' error."""
    srt = np.sort(lg_ref, axis=-1)
    gap = srt[..., -1] - srt[..., -2] if lg_ref.shape[-1] > 1 else np.full(lg_ref.shape[:-1], np.inf)
    ref = np.argmax(lg_ref, axis=-1)
    clear = gap > 2 * bound
    assert np.array_equal(s[clear], ref[clear])
    # near ties: the GPU's pick is within the bound of the best
    picked = np.take_along_axis(lg_ref, s[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(picked >= srt[..., -1] - 2 * bound - 1e-300)
    return int((~clear).sum())


@pytest.mark.parametrize("Bt,L,D,H,K", [
    (1, 128, 64, 2, 16),      # one tile, H K = 32
    (2, 300, 128, 4, 16),     # ragged last row tile
    (1, 257, 256, 16, 16),    # H K = 256, one column tile
    (2, 640, 512, 32, 16),    # the LM layer's 32 heads x 16 entries: two column tiles
    (1, 130, 192, 2, 64),
])
def test_projection_selection_matches_oracle(cuda_device, Bt, L, D, H, K):
    g = torch.Generator().manual_seed(D + H * K)
    u = torch.randn(Bt, L, D, generator=g).to(torch.bfloat16)
    W = (torch.randn(D, H * K, generator=g) / D ** 0.5).to(torch.bfloat16)
    out = pd.select_proj(u.to(cuda_device), W.to(cuda_device), H, K, want_logits=True)
    torch.cuda.synchronize()
    assert pd.pdssm_read_device_check(out["workspace"]) == 0
    lg_ref = ds.proj_logits(u.float().numpy(), W.float().numpy(), H, K)
    absum = ds.proj_logits(np.abs(u.float().numpy()), np.abs(W.float().numpy()), H, K)
    tol = absum * (D * 2.0 ** -23)
    got = out["logits"].cpu().double().numpy()
    assert np.all(np.abs(got - lg_ref) <= tol + 1e-30)
    _check_selection(out["s"].cpu().numpy(), lg_ref, tol.max(axis=-1))


def test_projection_selection_feeds_the_scan(cuda_device):
    """s from the fused projection is the s pdssm_scan_fwd reads: with the logits it returns,
    pdssm_forward selects the same dictionary entries."""
    import workloads
    sp = workloads.spec("lm", batch=1, seqlen=200, heads=2)
    inp = {k: v.to(cuda_device) for k, v in workloads.generate(sp, seed=3).items()}
    D = 128
    g = torch.Generator().manual_seed(8)
    u = torch.randn(1, 200, D, generator=g).to(torch.bfloat16).to(cuda_device)
    W = (torch.randn(D, 2 * sp.K, generator=g) / D ** 0.5).to(torch.bfloat16).to(cuda_device)
    pr = pd.select_proj(u, W, 2, sp.K, want_logits=True)
    fw = pd.forward(pr["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], want_s=True)
    torch.cuda.synchronize()
    assert torch.equal(fw["s"], pr["s"])


# ------------------------------------------------ the original PD-SSM's soft selection

def _soft_bound(logits, M, tau):
    """Bound on the error of a mixture value computed with bf16 hi + lo parts of pi and M
    (three products, fp32 accumulation): 2^-15 of sum_k pi_k |M_k[i][j]| per entry."""
    pi = ds.softmax(logits, tau)
    return np.einsum("...k,kij->...ij", pi, np.abs(M)) * 2.0 ** -15


@pytest.mark.parametrize("Bt,L,H,N,K,tau", [(1, 128, 1, 64, 16, 1.0), (2, 200, 3, 64, 16, 0.5),
                                           (1, 130, 2, 32, 5, 1.0), (1, 64, 1, 128, 64, 2.0),
                                           (1, 100, 2, 16, 3, 1.0)])
def test_soft_selection_matches_oracle(cuda_device, Bt, L, H, N, K, tau):
    g = torch.Generator().manual_seed(N + K)
    logits = torch.randn(Bt, L, H, K, generator=g).to(torch.bfloat16)
    M = torch.randn(K, N, N, generator=g)
    out = pd.soft_select(logits.to(cuda_device), M.to(cuda_device), tau)
    torch.cuda.synchronize()
    assert pd.pdssm_read_device_check(out["workspace"]) == 0
    got = out["idx_steps"].cpu().numpy().astype(np.int64)
    lg = logits.float().numpy()
    mix = ds.soft_mixture(lg, M.numpy(), tau)                 # [Bt, L, H, N(i), N(j)]
    bound = _soft_bound(lg, M.numpy(), tau).max(axis=-2)      # per column j
    col = np.swapaxes(mix, -1, -2)                            # [..., j, i]
    srt = np.sort(col, axis=-1)
    ref = ds.soft_select(lg, M.numpy(), tau)
    clear = (srt[..., -1] - srt[..., -2]) > 2 * bound
    assert np.array_equal(got[clear], ref[clear])
    picked = np.take_along_axis(col, got[..., None], axis=-1)[..., 0]
    assert np.all(picked >= srt[..., -1] - 2 * bound)
    assert clear.mean() > 0.99


def test_soft_selection_with_per_head_dictionaries(cuda_device):
    g = torch.Generator().manual_seed(2)
    Bt, L, H, N, K = 1, 150, 2, 32, 4
    logits = torch.randn(Bt, L, H, K, generator=g)
    M = torch.randn(H, K, N, N, generator=g)
    out = pd.soft_select(logits.to(cuda_device), M.to(cuda_device))
    torch.cuda.synchronize()
    got = out["idx_steps"].cpu().numpy()
    for h in range(H):
        ref = ds.soft_select(logits[:, :, h].numpy(), M[h].numpy())
        agree = (got[:, :, h] == ref).mean()
        assert agree > 0.999, (h, agree)


def test_dominant_score_selects_that_entrys_hardmax(cuda_device):
    """With one score far above the others the mixture is that dictionary matrix, so the soft
    selection equals the column-wise hardmax of the entry (the dictionary construction)."""
    K, N = 8, 64
    M = torch.randn(K, N, N, generator=torch.Generator().manual_seed(4))
    logits = torch.full((1, 128, 1, K), -30.0)
    for t in range(128):
        logits[0, t, 0, t % K] = 30.0
    out = pd.soft_select(logits.to(cuda_device), M.to(cuda_device))
    hard = pd.dict_hardmax(M.to(cuda_device))
    torch.cuda.synchronize()
    for t in range(128):
        assert torch.equal(out["idx_steps"][0, t, 0].long(), hard[t % K].long()), t


@pytest.mark.parametrize("seqlen", [1, 16, 250])
def test_scan_with_soft_selected_transitions_matches_oracle(cuda_device, seqlen):
    """The original PD-SSM end to end: soft selection, then the scan with per-step transitions
    (the fused kernel), against the oracle's scan of the same transitions."""
    import oracle
    import workloads
    from tests.parity import TOL, bhl_to_slices, slice_rel_err, to_np
    sp = workloads.spec("lm", batch=2, seqlen=seqlen, heads=2)
    inp = workloads.generate(sp, seed=14)
    M = torch.randn(sp.K, sp.N, sp.N, generator=torch.Generator().manual_seed(15))
    g = {k: v.to(cuda_device) for k, v in inp.items()}
    steps = pd.soft_select(g["logits"], M.to(cuda_device))["idx_steps"]
    out = pd.forward_steps(steps, g["d"], g["B"], g["C"], g["x"])
    torch.cuda.synchronize()
    assert pd.pdssm_read_device_check(out["workspace"]) == 0
    r = oracle.scan_steps(steps.cpu().numpy(), inp["d"], inp["B"], inp["C"], inp["x"])
    S = sp.batch * sp.heads
    assert np.array_equal(to_np(out["prod_idx"]), r["prod_idx"])
    assert slice_rel_err(bhl_to_slices(to_np(out["y"])), bhl_to_slices(r["y"])) <= TOL[torch.bfloat16]
    assert slice_rel_err(to_np(out["h_final"]).reshape(S, -1), r["h_final"].reshape(S, -1)) <= 1e-4
    assert slice_rel_err(to_np(out["prod_val"]).reshape(S, -1), r["prod_val"].reshape(S, -1)) <= 1e-4


def test_scan_with_per_step_transitions_flags_out_of_range_rows(cuda_device):
    import workloads
    sp = workloads.spec("lm", batch=1, seqlen=40, heads=1)
    g = {k: v.to(cuda_device) for k, v in workloads.generate(sp, seed=2).items()}
    steps = torch.randint(0, sp.N, (1, 40, 1, sp.N), dtype=torch.uint8, device=cuda_device)
    steps[0, 5, 0, 3] = 200
    out = pd.forward_steps(steps, g["d"], g["B"], g["C"], g["x"])
    torch.cuda.synchronize()
    assert pd.pdssm_read_device_check(out["workspace"]) == 5  # PDSSM_ERR_DEVICE_CHECK
