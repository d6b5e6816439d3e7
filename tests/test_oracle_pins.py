"""Pins of the dense CPU oracle to facts that do not come from the oracle itself.

Each test states which passage or mathematical fact fixes the expected value:
library argmax, closed forms built from explicit dense products, the
cyclic-group state tracking of Proposition 1, the diagonal-SSM and causal
linear-attention special cases, and the three-phase chunked route.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.chunked_ref import apply_pair, chunked_scan, compose

RNG = np.random.default_rng(1234)


def _rand_problem(L, N, P, K, complex_d=False, perm=False, seed=0, h0=False):
    g = np.random.default_rng(seed)
    if perm:
        idx = np.stack([g.permutation(N) for _ in range(K)]).astype(np.int32)
    else:
        idx = g.integers(0, N, size=(K, N)).astype(np.int32)
    logits = g.standard_normal((L, K))
    if complex_d:
        d = g.uniform(0.5, 1.0, (L, N)) * np.exp(1j * g.uniform(0, 2 * np.pi, (L, N)))
    else:
        d = g.uniform(0.5, 1.0, (L, N)) * g.choice([-1.0, 1.0], (L, N))
    B = g.standard_normal((L, N))
    C = g.standard_normal((L, N))
    x = g.standard_normal((L, P))
    hh = None
    if h0:
        hh = g.standard_normal((N, P))
        if complex_d:
            hh = hh + 1j * g.standard_normal((N, P))
    return idx, logits, d, B, C, x, hh


def _run(idx, logits, d, B, C, x, h0=None):
    h0s = None if h0 is None else h0[None]
    return {k: v[0] for k, v in oracle.scan_slices(logits[None], idx, d[None], B[None], C[None], x[None],
                                                    h0s).items()}


def _dense_A(idx_s, d_t):
    """P_s diag(d_t): column j holds d_t[j] at row idx_s[j] (one-hot column selector)."""
    N = idx_s.shape[0]
    A = np.zeros((N, N), dtype=np.result_type(d_t.dtype, np.float64))
    A[idx_s, np.arange(N)] = d_t
    return A


# ------------------------------------------------------------------ selection

def test_select_matches_library_argmax_on_random_rows():
    # np.argmax returns the first occurrence of the maximum (lowest k on ties)
    lg = RNG.standard_normal((1000, 17))
    assert np.array_equal(oracle.select(lg), np.argmax(lg, axis=-1))


def test_select_ties_signed_zero_and_nan():
    rows = np.array([
        [1.0, 1.0, 1.0, 1.0],             # all equal -> 0
        [0.0, 3.0, 1.0, 3.0],             # tie at the max -> lowest, 1
        [-0.0, 0.0, -1.0, -2.0],          # -0 == +0 -> 0
        [0.0, -0.0, -1.0, -2.0],          # +0 == -0 -> 0
        [1.0, np.nan, 5.0, np.nan],       # first NaN wins -> 1
        [np.nan, 2.0, np.nan, 0.0],       # -> 0
        [-np.inf, -np.inf, -np.inf, -5.0],
    ])
    expect = np.array([0, 1, 0, 0, 1, 0, 3])
    assert np.array_equal(oracle.select(rows), expect)
    assert np.array_equal(expect, np.argmax(rows, axis=-1))


def test_select_bf16_quantised_rows_with_real_ties():
    # bf16 rounding of N(0,1) at K=16 produces genuine ties
    lg = torch.randn(20000, 16, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    s = oracle.select(lg)
    ref = np.argmax(lg.float().numpy(), axis=-1)
    assert np.array_equal(s, ref)
    srt = np.sort(lg.float().numpy(), axis=-1)
    assert (srt[:, -1] == srt[:, -2]).any(), "expected at least one tie in the sample"


# ------------------------------------------------------- dense recurrence pins

@pytest.mark.parametrize("complex_d", [False, True])
@pytest.mark.parametrize("with_h0", [False, True])
@pytest.mark.parametrize("N,P,K,L", [(1, 1, 1, 5), (3, 2, 2, 17), (8, 4, 4, 64), (5, 3, 7, 40)])
def test_recurrence_matches_closed_form(N, P, K, L, complex_d, with_h0):
    """H_t = A_t..A_0 h0 + sum_{s<=t} (A_t..A_{s+1}) B_s x_s^T, y_t = H_t^T C_t, by explicit products."""
    idx, logits, d, B, C, x, h0 = _rand_problem(L, N, P, K, complex_d, seed=N * 100 + L, h0=with_h0)
    r = _run(idx, logits, d, B, C, x, h0)
    s = np.argmax(logits, axis=-1)
    A = [_dense_A(idx[s[t]], d[t]) for t in range(L)]
    cdt = np.complex128 if complex_d else np.float64
    for t in range(L):
        H = np.zeros((N, P), dtype=cdt)
        if h0 is not None:
            M = np.eye(N, dtype=cdt)
            for r_ in range(t + 1):
                M = A[r_] @ M
            H += M @ h0
        for s_ in range(t + 1):
            M = np.eye(N, dtype=cdt)
            for r_ in range(s_ + 1, t + 1):
                M = A[r_] @ M
            H += M @ np.outer(B[s_], x[s_])
        np.testing.assert_allclose(r["y"][t], H.T @ C[t], rtol=1e-11, atol=1e-11)
        if t == L - 1:
            np.testing.assert_allclose(r["h_final"], H, rtol=1e-11, atol=1e-11)
    assert np.array_equal(r["s"], s)


@pytest.mark.parametrize("perm", [False, True])
@pytest.mark.parametrize("N,K,L", [(2, 2, 9), (5, 3, 30), (8, 4, 64)])
def test_prod_matches_dense_product_and_pair_composition(N, K, L, perm):
    idx, logits, d, B, C, x, _ = _rand_problem(L, N, 1, K, perm=perm, seed=7 * N + L)
    r = _run(idx, logits, d, B, C, x)
    s = np.argmax(logits, axis=-1)
    M = np.eye(N)
    pair = (np.arange(N), np.ones(N))
    for t in range(L):
        M = _dense_A(idx[s[t]], d[t]) @ M
        pair = compose((idx[s[t]], d[t]), pair)
    # one nonzero per column of the product of column-one-hot matrices
    assert ((M != 0).sum(axis=0) == 1).all()
    rows = np.argmax(M != 0, axis=0)
    assert np.array_equal(r["prod_idx"], rows)
    assert np.array_equal(r["prod_idx"], pair[0])
    np.testing.assert_allclose(r["prod_val"], M[rows, np.arange(N)], rtol=1e-12)
    np.testing.assert_allclose(r["prod_val"], pair[1], rtol=1e-12)


def test_prod_exact_for_power_of_two_values():
    N, K, L = 6, 3, 25
    g = np.random.default_rng(3)
    idx = g.integers(0, N, (K, N)).astype(np.int32)
    logits = g.standard_normal((L, K))
    d = g.choice([-1.0, 1.0, 0.5, 2.0, -0.25], (L, N))
    r = _run(idx, logits, d, np.zeros((L, N)), np.zeros((L, N)), np.zeros((L, 1)))
    s = np.argmax(logits, axis=-1)
    pair = (np.arange(N), np.ones(N))
    for t in range(L):
        pair = compose((idx[s[t]], d[t]), pair)
    assert np.array_equal(r["prod_idx"], pair[0])
    assert np.array_equal(r["prod_val"], pair[1])  # exact: powers of two


def test_pair_composition_is_associative():
    g = np.random.default_rng(9)
    for _ in range(200):
        N = int(g.integers(1, 12))
        a, b, c = [(g.integers(0, N, N), g.choice([-2.0, -1.0, 0.5, 1.0, 4.0], N)) for _ in range(3)]
        l = compose(compose(a, b), c)
        r = compose(a, compose(b, c))
        assert np.array_equal(l[0], r[0]) and np.array_equal(l[1], r[1])


def test_pair_composition_is_the_matrix_product():
    g = np.random.default_rng(10)
    for _ in range(100):
        N = int(g.integers(1, 9))
        a = (g.integers(0, N, N), g.standard_normal(N))
        b = (g.integers(0, N, N), g.standard_normal(N))
        ab = compose(a, b)
        np.testing.assert_allclose(_dense_A(*ab), _dense_A(*a) @ _dense_A(*b), rtol=1e-13, atol=1e-15)
        H = g.standard_normal((N, 3))
        np.testing.assert_allclose(apply_pair(a, H), _dense_A(*a) @ H, rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------ special cases

@pytest.mark.parametrize("complex_d", [False, True])
def test_identity_dictionary_is_a_diagonal_ssm(complex_d):
    """K=1, idx = identity: H_t[i] = sum_s (prod_{r=s+1..t} d_r[i]) B_s[i] x_s."""
    N, P, L = 6, 3, 50
    idx, logits, d, B, C, x, _ = _rand_problem(L, N, P, 1, complex_d, seed=77)
    idx = np.arange(N, dtype=np.int32)[None]
    r = _run(idx, logits, d, B, C, x)
    cdt = np.complex128 if complex_d else np.float64
    # cumulative products of the diagonal, written as ratios of prefix products
    cp = np.ones((L + 1, N), dtype=cdt)
    for t in range(L):
        cp[t + 1] = cp[t] * d[t]
    for t in (0, 1, 17, L - 1):
        H = np.zeros((N, P), dtype=cdt)
        for s_ in range(t + 1):
            decay = cp[t + 1] / cp[s_ + 1]
            H += (decay * B[s_])[:, None] * x[s_][None, :]
        np.testing.assert_allclose(r["y"][t], H.T @ C[t], rtol=1e-9, atol=1e-10)


def test_identity_dictionary_unit_decay_is_causal_linear_attention():
    """K=1, identity idx, d=1: y = tril(C B^T) X."""
    N, P, L = 7, 5, 60
    g = np.random.default_rng(4)
    idx = np.arange(N, dtype=np.int32)[None]
    logits = g.standard_normal((L, 1))
    d = np.ones((L, N))
    B, C, x = g.standard_normal((L, N)), g.standard_normal((L, N)), g.standard_normal((L, P))
    r = _run(idx, logits, d, B, C, x)
    np.testing.assert_allclose(r["y"], np.tril(C @ B.T) @ x, rtol=1e-10, atol=1e-10)


def test_cyclic_group_state_tracking_is_exact():
    """Proposition 1 (Flash PD-SSM page, Key Contributions): an N-state deterministic FSA is
    represented exactly by one layer of size N. With the Z_5 cyclic shifts, d=1, B=e_0 at t=0 and
    C_t = e_{t mod 5}: H_t = e_{(s_1+..+s_t) mod 5}, y_t = [state == t mod 5] and
    M = shift by (s_0+..+s_{L-1}) mod 5, all exactly."""
    sp = workloads.spec("z5")
    inp = workloads.generate(sp)
    r = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    s = np.argmax(inp["logits"].numpy(), axis=-1)[:, :, 0]  # [Bt, L]
    L = sp.seqlen
    state = np.cumsum(np.concatenate([np.zeros_like(s[:, :1]), s[:, 1:]], axis=1), axis=1) % 5
    y = r["y"][:, :, 0, 0]
    assert np.array_equal(y, (state == (np.arange(L) % 5)[None]).astype(np.float64))
    hf = r["h_final"][:, 0, :, 0]
    assert np.array_equal(hf, np.eye(5)[state[:, -1]])
    total = s.sum(axis=1) % 5
    assert np.array_equal(r["prod_idx"][:, 0], (np.arange(5)[None] + total[:, None]) % 5)
    assert np.array_equal(r["prod_val"][:, 0], np.ones((sp.batch, 5)))


def test_conjugate_decay_conjugates_outputs():
    """Real B, C, x: replacing every d by its conjugate conjugates y and H exactly."""
    N, P, K, L = 5, 3, 3, 40
    idx, logits, d, B, C, x, _ = _rand_problem(L, N, P, K, complex_d=True, seed=21)
    r1 = _run(idx, logits, d, B, C, x)
    r2 = _run(idx, logits, np.conj(d), B, C, x)
    assert np.array_equal(r2["y"], np.conj(r1["y"]))
    assert np.array_equal(r2["h_final"], np.conj(r1["h_final"]))


def test_linearity_in_x_and_sign_of_B():
    N, P, K, L = 6, 4, 3, 33
    idx, logits, d, B, C, x, _ = _rand_problem(L, N, P, K, seed=5)
    r1 = _run(idx, logits, d, B, C, x)
    r2 = _run(idx, logits, d, B, C, 2.0 * x)
    r3 = _run(idx, logits, d, -B, C, x)
    assert np.array_equal(r2["y"], 2.0 * r1["y"])
    assert np.array_equal(r3["y"], -r1["y"])


def test_single_step():
    N, P, K = 4, 2, 2
    idx, logits, d, B, C, x, h0 = _rand_problem(1, N, P, K, seed=8, h0=True)
    r = _run(idx, logits, d, B, C, x, h0)
    s = int(np.argmax(logits[0]))
    H = np.zeros((N, P))
    for j in range(N):  # column j of P_s diag(d) moves row j of h0 to row idx[s][j]
        H[idx[s][j]] += d[0][j] * h0[j]
    H += np.outer(B[0], x[0])
    np.testing.assert_allclose(r["h_final"], H, rtol=1e-14)
    np.testing.assert_allclose(r["y"][0], H.T @ C[0], rtol=1e-13)


# ------------------------------------------- three-phase decomposition pin

@pytest.mark.parametrize("complex_d", [False, True])
@pytest.mark.parametrize("T", [1, 3, 16, 64, 100, 200])
def test_chunked_three_phase_scan_equals_sequential(T, complex_d):
    N, P, K, L = 8, 4, 5, 100
    idx, logits, d, B, C, x, h0 = _rand_problem(L, N, P, K, complex_d, seed=T, h0=True)
    r = _run(idx, logits, d, B, C, x, h0)
    s = np.argmax(logits, axis=-1)
    c = chunked_scan(s, idx, d, B, C, x, h0, T)
    np.testing.assert_allclose(c["y"], r["y"], rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(c["h_final"], r["h_final"], rtol=1e-9, atol=1e-9)
    assert np.array_equal(c["prod_idx"], r["prod_idx"])
    np.testing.assert_allclose(c["prod_val"], r["prod_val"], rtol=1e-12)


def test_segmented_run_equals_whole_run():
    """forward(L1 + L2) == forward(L1) then forward(L2, h0 = h_final)."""
    N, P, K, L = 6, 3, 4, 70
    idx, logits, d, B, C, x, _ = _rand_problem(L, N, P, K, seed=31)
    whole = _run(idx, logits, d, B, C, x)
    a = _run(idx, logits[:29], d[:29], B[:29], C[:29], x[:29])
    b = _run(idx, logits[29:], d[29:], B[29:], C[29:], x[29:], a["h_final"])
    np.testing.assert_allclose(np.concatenate([a["y"], b["y"]]), whole["y"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(b["h_final"], whole["h_final"], rtol=1e-11, atol=1e-12)
    pair = compose((b["prod_idx"], b["prod_val"]), (a["prod_idx"], a["prod_val"]))
    assert np.array_equal(pair[0], whole["prod_idx"])


def test_full_array_layout_matches_slices():
    sp = workloads.spec("lm", batch=2, seqlen=20, heads=3)
    inp = workloads.generate(sp)
    full = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    for b in range(2):
        for h in range(3):
            sl = workloads.generate_slice(sp, b, h)
            r = _run(inp["idx"].numpy(), sl["logits"].float().numpy(), sl["d"].float().numpy(),
                     sl["B"].float().numpy(), sl["C"].float().numpy(), sl["x"].float().numpy())
            assert np.array_equal(full["y"][b, :, h], r["y"])
            assert np.array_equal(full["h_final"][b, h], r["h_final"])


def test_per_head_dictionaries_use_each_heads_own_matrices():
    """Multi-head layers with a dictionary per head (Flash PD-SSM page, Methodology 4): head h's
    step t applies P_{s_t} of idx[h]. Pinned by the closed form of explicit dense products per head;
    a per-head dictionary whose heads are all equal reproduces the shared dictionary exactly, and a
    head's outputs do not depend on the other heads' dictionaries."""
    sp = workloads.spec("tiny", batch=2, seqlen=12, heads=3)
    inp = workloads.generate(sp, seed=4)
    g = torch.Generator().manual_seed(11)
    idx_h = torch.randint(0, sp.N, (sp.heads, sp.K, sp.N), generator=g).to(torch.int32)
    r = oracle.scan(inp["logits"], idx_h.numpy(), inp["d"], inp["B"], inp["C"], inp["x"])
    for b in range(sp.batch):
        for h in range(sp.heads):
            lg, d, B, C, x = (inp[k][b, :, h].double().numpy() for k in ("logits", "d", "B", "C", "x"))
            s = np.argmax(lg, axis=-1)
            A = [_dense_A(idx_h[h].numpy()[s[t]], d[t]) for t in range(sp.seqlen)]
            for t in range(sp.seqlen):
                H = np.zeros((sp.N, sp.P))
                for s_ in range(t + 1):
                    M = np.eye(sp.N)
                    for r_ in range(s_ + 1, t + 1):
                        M = A[r_] @ M
                    H += M @ np.outer(B[s_], x[s_])
                np.testing.assert_allclose(r["y"][b, t, h], H.T @ C[t], rtol=1e-11, atol=1e-11)
    same = np.broadcast_to(inp["idx"].numpy(), (sp.heads, sp.K, sp.N)).copy()
    a = oracle.scan(inp["logits"], same, inp["d"], inp["B"], inp["C"], inp["x"])
    s_ = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    for k in a:
        assert np.array_equal(a[k], s_[k]), k
    other = idx_h.clone()
    other[1] = torch.randint(0, sp.N, (sp.K, sp.N), generator=g).to(torch.int32)
    o = oracle.scan(inp["logits"], other.numpy(), inp["d"], inp["B"], inp["C"], inp["x"])
    for h in (0, 2):
        assert np.array_equal(o["y"][:, :, h], r["y"][:, :, h])
        assert np.array_equal(o["h_final"][:, h], r["h_final"][:, h])
