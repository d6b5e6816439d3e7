"""Pins of the dense-selection oracle (oracle/dense_select.py): brute force on small
sizes, the one-hot-column round trip of the dictionary's definition, ties and NaN."""
import numpy as np
import pytest

from oracle import dense_select as ds


def _brute_column_argmax(M):
    K, N, _ = M.shape
    out = np.zeros((K, N), dtype=np.int64)
    for k in range(K):
        for j in range(N):
            best, bi = None, None
            for i in range(N):
                v = M[k, i, j]
                if bi is None:
                    best, bi = v, i
                elif np.isnan(v):
                    if not np.isnan(best):
                        best, bi = v, i
                elif not np.isnan(best) and v > best:
                    best, bi = v, i
            out[k, j] = bi
    return out


def test_dict_hardmax_matches_brute_force_with_ties_and_nan():
    rng = np.random.default_rng(0)
    M = rng.standard_normal((5, 7, 7))
    M[0] = 0.25                      # all equal: row 0 everywhere
    M[1, :, 2] = [-0.0, 0.0, -1, -2, -3, -4, -5]  # signed zeros tie: row 0
    M[2, 3, 4] = np.nan              # a NaN wins its column
    M[2, 5, 4] = np.nan              # ... the first one
    M[3, :, :] = np.round(M[3])      # integer ties
    assert np.array_equal(ds.dict_hardmax(M), _brute_column_argmax(M))


def test_dict_hardmax_inverts_the_one_hot_column_dictionary():
    """Methodology 1: P_k[idx[k][j]][j] = 1 is the only nonzero of column j; the
    column-wise hardmax of P_k diag(v) with v > 0 gives back idx exactly."""
    rng = np.random.default_rng(1)
    K, N = 6, 9
    idx = rng.integers(0, N, (K, N))
    P = np.zeros((K, N, N))
    for k in range(K):
        P[k, idx[k], np.arange(N)] = rng.uniform(0.5, 2.0, N)
    assert np.array_equal(ds.dict_hardmax(P), idx)


def test_projection_matches_explicit_sums():
    rng = np.random.default_rng(2)
    Bt, L, D, H, K = 2, 3, 5, 2, 4
    u = rng.standard_normal((Bt, L, D))
    W = rng.standard_normal((D, H * K))
    s, lg = ds.select_proj(u, W, H, K)
    for b in range(Bt):
        for t in range(L):
            for h in range(H):
                ref = [sum(u[b, t, d] * W[d, h * K + k] for d in range(D)) for k in range(K)]
                np.testing.assert_allclose(lg[b, t, h], ref, rtol=1e-13, atol=1e-13)
                assert s[b, t, h] == int(np.argmax(ref))


def test_projection_of_one_hot_inputs_reads_rows_of_W():
    D, H, K = 6, 3, 2
    W = np.arange(D * H * K, dtype=np.float64).reshape(D, H * K) % 5 - 2
    u = np.eye(D)
    s, lg = ds.select_proj(u, W, H, K)
    assert np.array_equal(lg.reshape(D, H * K), W)
    assert np.array_equal(s, np.argmax(W.reshape(D, H, K), axis=-1))


def test_soft_selection_with_a_dominant_score_is_the_entrys_hardmax():
    """A score far above the others puts all of the convex combination on its matrix: the
    soft selection then equals the column-wise hardmax of that dictionary matrix."""
    rng = np.random.default_rng(3)
    K, N = 4, 8
    M = rng.standard_normal((K, N, N))
    for k in range(K):
        lg = np.zeros(K)
        lg[k] = 80.0
        assert np.array_equal(ds.soft_select(lg, M), ds.dict_hardmax(M[k]))


def test_soft_selection_matches_brute_force_mixture():
    rng = np.random.default_rng(4)
    K, N, tau = 3, 5, 0.7
    M = rng.standard_normal((K, N, N))
    lg = rng.standard_normal((6, K))
    got = ds.soft_select(lg, M, tau)
    for r in range(6):
        e = [np.exp(lg[r, k] / tau) for k in range(K)]
        pi = [x / sum(e) for x in e]
        mix = sum(pi[k] * M[k] for k in range(K))
        assert np.array_equal(got[r], _brute_column_argmax(mix[None])[0])
    # one entry: the scores do not matter
    assert np.array_equal(ds.soft_select(lg, M[:1]), np.broadcast_to(ds.dict_hardmax(M[0]), (6, N)))


def test_softmax_is_a_convex_combination():
    rng = np.random.default_rng(5)
    p = ds.softmax(rng.standard_normal((10, 7)), tau=0.3)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=1e-15)


def test_scan_with_per_step_transitions_reproduces_the_dictionary_scan():
    """Per-step transitions idx_t = idx[s_t] are exactly the Flash PD-SSM scan of the
    selections s_t; and each slice matches the closed form of explicit dense products."""
    import torch
    import oracle
    import workloads
    sp = workloads.spec("tiny", batch=2, seqlen=20, heads=2)
    inp = workloads.generate(sp, seed=6)
    ref = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    steps = inp["idx"].numpy()[ref["s"]]                      # [Bt, L, H, N]
    got = oracle.scan_steps(steps, inp["d"], inp["B"], inp["C"], inp["x"])
    for k in ("y", "h_final", "prod_idx", "prod_val"):
        assert np.array_equal(got[k], ref[k]), k
    rng = np.random.default_rng(7)
    steps = rng.integers(0, sp.N, (sp.batch, sp.seqlen, sp.heads, sp.N))
    got = oracle.scan_steps(steps, inp["d"], inp["B"], inp["C"], inp["x"])
    for b in range(sp.batch):
        for h in range(sp.heads):
            d, B, C, x = (inp[k][b, :, h].double().numpy() for k in ("d", "B", "C", "x"))
            A = []
            for t in range(sp.seqlen):
                M = np.zeros((sp.N, sp.N))
                M[steps[b, t, h], np.arange(sp.N)] = d[t]
                A.append(M)
            for t in (0, 7, sp.seqlen - 1):  # closed form: H_t = sum_s A_t..A_{s+1} B_s x_s^T
                H = np.zeros((sp.N, sp.P))
                for s_ in range(t + 1):
                    M = np.eye(sp.N)
                    for r_ in range(s_ + 1, t + 1):
                        M = A[r_] @ M
                    H += M @ np.outer(B[s_], x[s_])
                np.testing.assert_allclose(got["y"][b, t, h], H.T @ C[t], rtol=1e-12, atol=1e-12)
