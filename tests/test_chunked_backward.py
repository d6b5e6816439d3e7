"""The chunk-parallel shape of the backward pass (tests/chunked_bwd_ref.py: local
adjoints per chunk, a reverse scan of the chunks' transposed pairs, suffix
corrections) equals the sequential adjoint of the backward oracle, for chunk lengths
that divide L, do not divide it, exceed it, and for a single step per chunk."""
import numpy as np
import pytest

from oracle import backward as bwd
from tests.chunked_bwd_ref import chunked_backward


def _problem(L, N, P, K, seed, perm=False):
    g = np.random.default_rng(seed)
    idx = (np.stack([g.permutation(N) for _ in range(K)]) if perm else g.integers(0, N, size=(K, N))).astype(np.int64)
    return dict(logits=g.standard_normal((L, K)), idx=idx,
                d=g.uniform(0.5, 1.0, (L, N)) * g.choice([-1.0, 1.0], (L, N)),
                B=g.standard_normal((L, N)), C=g.standard_normal((L, N)), x=g.standard_normal((L, P)),
                dy=g.standard_normal((L, P)), dh_final=g.standard_normal((N, P)), h0=g.standard_normal((N, P)))


@pytest.mark.parametrize("T", [1, 3, 16, 40, 64])
@pytest.mark.parametrize("perm", [False, True])
def test_chunked_adjoint_equals_sequential(T, perm):
    pr = _problem(40, 7, 3, 5, seed=T + 100 * perm, perm=perm)
    ref = bwd.slice_backward(**pr, tau=0.8)
    got = chunked_backward(**pr, T=T, tau=0.8)
    assert np.array_equal(got["s"], ref["s"])
    for k in ("dd", "dB", "dC", "dx", "dlogits", "dh0"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-10, atol=1e-11, err_msg=k)


def test_chunked_adjoint_without_initial_state_or_final_gradient():
    pr = _problem(23, 5, 2, 3, seed=7)
    pr["h0"] = None
    pr["dh_final"] = None
    ref = bwd.slice_backward(**pr)
    got = chunked_backward(**pr, T=6)
    for k in ("dd", "dB", "dC", "dx", "dlogits", "dh0"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-10, atol=1e-11, err_msg=k)


@pytest.mark.parametrize("T", [1, 4, 16, 50])
def test_chunked_adjoint_equals_sequential_for_complex_states(T):
    g = np.random.default_rng(T)
    pr = _problem(33, 6, 3, 4, seed=T)
    pr["d"] = g.uniform(0.5, 1.0, (33, 6)) * np.exp(1j * g.uniform(0, 2 * np.pi, (33, 6)))
    pr["dy"] = g.standard_normal((33, 3)) + 1j * g.standard_normal((33, 3))
    pr["dh_final"] = g.standard_normal((6, 3)) + 1j * g.standard_normal((6, 3))
    pr["h0"] = g.standard_normal((6, 3)) + 1j * g.standard_normal((6, 3))
    ref = bwd.slice_backward(**pr, tau=0.9)
    got = chunked_backward(**pr, T=T, tau=0.9)
    for k in ("dd", "dB", "dC", "dx", "dlogits", "dh0"):
        np.testing.assert_allclose(got[k], ref[k], rtol=1e-10, atol=1e-11, err_msg=k)
