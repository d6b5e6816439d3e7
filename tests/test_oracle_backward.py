"""Pins of the backward oracle (oracle/backward.py) to routes that do not share its
derivation: automatic differentiation of the dense forward with straight-through
weights, central finite differences of the C forward oracle, a closed form for the
identity dictionary with unit decay, and properties of the tempered softmax. A
planted mistake in a copy of the oracle must fail the automatic-differentiation pin.
"""
import inspect

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bwd


def _problem(L, N, P, K, seed, h0=True, perm=False):
    g = np.random.default_rng(seed)
    idx = (np.stack([g.permutation(N) for _ in range(K)]) if perm else g.integers(0, N, size=(K, N))).astype(np.int64)
    logits = g.standard_normal((L, K))
    d = g.uniform(0.5, 1.0, (L, N)) * g.choice([-1.0, 1.0], (L, N))
    B, C = g.standard_normal((L, N)), g.standard_normal((L, N))
    x, dy = g.standard_normal((L, P)), g.standard_normal((L, P))
    dh = g.standard_normal((N, P))
    hh = g.standard_normal((N, P)) if h0 else None
    return dict(logits=logits, idx=idx, d=d, B=B, C=C, x=x, dy=dy, dh_final=dh, h0=hh)


def _autograd(pr, tau):
    """Gradients by automatic differentiation of the dense forward, the selection
    weights being one-hot in value and tempered-softmax in gradient."""
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=k not in ("idx", "dy", "dh_final"))
         for k, v in pr.items() if v is not None}
    L, K = t["logits"].shape
    N = t["B"].shape[1]
    Pk = torch.zeros(K, N, N, dtype=torch.float64)
    for k in range(K):
        Pk[k, torch.as_tensor(pr["idx"][k]), torch.arange(N)] = 1.0
    soft = torch.softmax(t["logits"] / tau, dim=-1)
    hard = torch.nn.functional.one_hot(t["logits"].argmax(dim=-1), K).to(torch.float64)
    pi = hard + soft - soft.detach()
    H = t["h0"] if "h0" in t else torch.zeros(N, t["x"].shape[1], dtype=torch.float64)
    loss = torch.zeros((), dtype=torch.float64)
    for s in range(L):
        A = torch.einsum("k,kij->ij", pi[s], Pk) * t["d"][s][None, :]
        H = A @ H + torch.outer(t["B"][s], t["x"][s])
        loss = loss + (H.T @ t["C"][s] * t["dy"][s]).sum()
    loss = loss + (H * t["dh_final"]).sum()
    names = [k for k in ("logits", "d", "B", "C", "x", "h0") if k in t]
    grads = torch.autograd.grad(loss, [t[k] for k in names])
    return {"d" + k: g.numpy() for k, g in zip(names, grads)}


@pytest.mark.parametrize("L,N,P,K,perm", [(1, 3, 2, 2, False), (9, 5, 3, 4, False), (24, 8, 4, 6, False),
                                          (17, 6, 2, 3, True)])
@pytest.mark.parametrize("tau", [1.0, 0.3])
def test_matches_automatic_differentiation(L, N, P, K, perm, tau):
    pr = _problem(L, N, P, K, seed=L * 7 + N, perm=perm)
    got = bwd.slice_backward(**pr, tau=tau)
    ref = _autograd(pr, tau)
    for k, v in ref.items():
        np.testing.assert_allclose(got[k], v, rtol=1e-10, atol=1e-11, err_msg=k)


def _loss_forward(pr):
    """Loss sum_t <dy_t, y_t> + <dh_final, H_{L-1}> through the C forward oracle."""
    S = lambda a: None if a is None else a[None]
    r = oracle.scan_slices(S(pr["logits"]), pr["idx"].astype(np.int32), S(pr["d"]), S(pr["B"]), S(pr["C"]),
                           S(pr["x"]), S(pr["h0"]), want_prod=False)
    return float((r["y"][0] * pr["dy"]).sum() + (r["h_final"][0] * pr["dh_final"]).sum())


@pytest.mark.parametrize("name", ["d", "B", "C", "x", "h0"])
def test_matches_central_differences_of_the_forward_oracle(name):
    pr = _problem(12, 5, 3, 4, seed=3)
    got = bwd.slice_backward(**pr)["d" + name]
    base = pr[name]
    fd = np.zeros_like(base)
    eps = 1e-6
    for i in np.ndindex(base.shape):
        hi, lo = dict(pr), dict(pr)
        hi[name], lo[name] = base.copy(), base.copy()
        hi[name][i] += eps
        lo[name][i] -= eps
        fd[i] = (_loss_forward(hi) - _loss_forward(lo)) / (2 * eps)
    np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7)


def test_selection_weight_gradient_matches_differences_of_the_mixture():
    """dlogits = J_softmax(logits / tau) dpi / tau, with dpi the derivative of the loss
    in the mixture weights pi of A_t = sum_k pi_k P_k diag(d_t) at the one-hot point:
    dpi from central differences of the mixture forward, J from differences of softmax."""
    pr = _problem(6, 4, 2, 3, seed=11)
    tau = 0.7
    got = bwd.slice_backward(**pr, tau=tau)["dlogits"]
    L, K = pr["logits"].shape
    N = pr["B"].shape[1]
    Pk = []
    for k in range(K):
        m = np.zeros((N, N))
        m[pr["idx"][k], np.arange(N)] = 1.0
        Pk.append(m)
    onehot = np.eye(K)[np.argmax(pr["logits"], axis=1)]

    def mixture_loss(pi):
        H = pr["h0"].copy()
        loss = 0.0
        for t in range(L):
            A = sum(pi[t, k] * Pk[k] for k in range(K)) * pr["d"][t][None, :]
            H = A @ H + np.outer(pr["B"][t], pr["x"][t])
            loss += (H.T @ pr["C"][t] * pr["dy"][t]).sum()
        return loss + (H * pr["dh_final"]).sum()

    def sm(v):
        e = np.exp(v / tau - (v / tau).max())
        return e / e.sum()

    eps = 1e-6
    for t in range(L):
        dpi = np.zeros(K)
        for k in range(K):
            hi, lo = onehot.copy(), onehot.copy()
            hi[t, k] += eps
            lo[t, k] -= eps
            dpi[k] = (mixture_loss(hi) - mixture_loss(lo)) / (2 * eps)
        J = np.zeros((K, K))  # J[k, m] = d softmax_k / d logit_m
        for m in range(K):
            hi, lo = pr["logits"][t].copy(), pr["logits"][t].copy()
            hi[m] += eps
            lo[m] -= eps
            J[:, m] = (sm(hi) - sm(lo)) / (2 * eps)
        np.testing.assert_allclose(got[t], J.T @ dpi, rtol=1e-5, atol=1e-6)


def test_identity_dictionary_unit_decay_closed_form():
    """K = 1, identity idx, d = 1, no initial state: y = tril(C B^T) X (causal linear
    attention), so dX = tril(C B^T)^T dY, dC = (tril o dY X^T) B, dB = (tril o dY X^T)^T C
    and the single logit gets no gradient."""
    L, N, P = 20, 6, 3
    g = np.random.default_rng(5)
    pr = dict(logits=g.standard_normal((L, 1)), idx=np.arange(N)[None], d=np.ones((L, N)),
              B=g.standard_normal((L, N)), C=g.standard_normal((L, N)), x=g.standard_normal((L, P)),
              dy=g.standard_normal((L, P)), dh_final=np.zeros((N, P)), h0=None)
    got = bwd.slice_backward(**pr)
    T = np.tril(np.ones((L, L)))
    M = T * (pr["dy"] @ pr["x"].T)
    np.testing.assert_allclose(got["dx"], (T * (pr["C"] @ pr["B"].T)).T @ pr["dy"], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(got["dC"], M @ pr["B"], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(got["dB"], M.T @ pr["C"], rtol=1e-11, atol=1e-11)
    assert np.all(got["dlogits"] == 0.0)


def test_logit_gradients_sum_to_zero_and_scale_with_temperature():
    """Each row of a softmax Jacobian sums to zero; at equal logits the Jacobian is
    (I - 1/K) / K, so the gradient scales as 1 / tau."""
    pr = _problem(10, 5, 2, 4, seed=9)
    g1 = bwd.slice_backward(**pr, tau=1.0)["dlogits"]
    np.testing.assert_allclose(g1.sum(axis=1), 0.0, atol=1e-12)
    pr["logits"] = np.zeros_like(pr["logits"])  # ties: k = 0 selected everywhere
    a = bwd.slice_backward(**pr, tau=1.0)["dlogits"]
    b = bwd.slice_backward(**pr, tau=0.25)["dlogits"]
    np.testing.assert_allclose(b, 4.0 * a, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("mutation", [
    ("lam = np.conj(A[t]).T @ lam", "lam = np.conj(A[t]) @ lam"),                # adjoint not transposed
    ("lam = lam + np.outer(C[t], dy[t])", "lam = lam + 0 * np.outer(C[t], dy[t])"),  # output term dropped
    ("dA = lam @ np.conj(Hprev).T", "dA = lam @ np.conj(Ht).T"),                 # state one step late
    ('out["dd"][t] = dA[idx[s[t]], np.arange(N)]', 'out["dd"][t] = dA[np.arange(N), idx[s[t]]]'),  # transposed pick
    ("(np.diag(pit) - np.outer(pit, pit)) @ dpi / tau", "(np.diag(pit) - np.outer(pit, pit)) @ dpi"),  # no 1/tau
])
def test_a_planted_mistake_fails_the_automatic_differentiation_pin(mutation):
    src = inspect.getsource(bwd.slice_backward)
    assert src.count(mutation[0]) == 1
    ns = dict(vars(bwd))
    exec(src.replace(mutation[0], mutation[1]), ns)
    pr = _problem(9, 5, 3, 4, seed=2)
    got = ns["slice_backward"](**pr, tau=0.5)
    ref = _autograd(pr, 0.5)
    assert any(not np.allclose(got[k], v, rtol=1e-8, atol=1e-9) for k, v in ref.items())


# ---------------------------------------------------------------- complex states

def _cproblem(L, N, P, K, seed):
    g = np.random.default_rng(seed)
    pr = _problem(L, N, P, K, seed)
    r = g.uniform(0.5, 1.0, (L, N))
    pr["d"] = r * np.exp(1j * g.uniform(0, 2 * np.pi, (L, N)))
    pr["dy"] = g.standard_normal((L, P)) + 1j * g.standard_normal((L, P))
    pr["dh_final"] = g.standard_normal((N, P)) + 1j * g.standard_normal((N, P))
    pr["h0"] = g.standard_normal((N, P)) + 1j * g.standard_normal((N, P))
    return pr


def _autograd_complex(pr, tau):
    """Complex autograd (PyTorch's gradient dL/du + i dL/dv of a real loss) of the dense
    forward with straight-through selection weights."""
    real = ("logits", "B", "C", "x")
    t = {k: torch.tensor(v, dtype=torch.float64 if k in real else torch.complex128,
                         requires_grad=k in real + ("d", "h0")) for k, v in pr.items() if k != "idx"}
    L, K = t["logits"].shape
    N = t["B"].shape[1]
    Pk = torch.zeros(K, N, N, dtype=torch.complex128)
    for k in range(K):
        Pk[k, torch.as_tensor(pr["idx"][k]), torch.arange(N)] = 1.0
    soft = torch.softmax(t["logits"] / tau, dim=-1)
    hard = torch.nn.functional.one_hot(t["logits"].argmax(dim=-1), K).to(torch.float64)
    pi = (hard + soft - soft.detach()).to(torch.complex128)
    H = t["h0"]
    loss = torch.zeros((), dtype=torch.float64)
    for s in range(L):
        A = torch.einsum("k,kij->ij", pi[s], Pk) * t["d"][s][None, :]
        H = A @ H + torch.outer(t["B"][s], t["x"][s]).to(torch.complex128)
        y = H.T @ t["C"][s].to(torch.complex128)
        loss = loss + (t["dy"][s].conj() * y).sum().real
    loss = loss + (t["dh_final"].conj() * H).sum().real
    names = ["logits", "d", "B", "C", "x", "h0"]
    grads = torch.autograd.grad(loss, [t[k] for k in names])
    return {"d" + k: g.numpy() for k, g in zip(names, grads)}


@pytest.mark.parametrize("L,N,P,K", [(1, 3, 2, 2), (11, 5, 3, 4), (20, 8, 4, 6)])
def test_complex_matches_automatic_differentiation(L, N, P, K):
    pr = _cproblem(L, N, P, K, seed=L + N)
    got = bwd.slice_backward(**pr, tau=0.6)
    for k, v in _autograd_complex(pr, 0.6).items():
        np.testing.assert_allclose(got[k], v, rtol=1e-10, atol=1e-11, err_msg=k)


@pytest.mark.parametrize("name", ["d", "h0"])
def test_complex_matches_differences_of_real_and_imaginary_parts(name):
    """dL/du + i dL/dv by central differences of the C forward oracle (complex mode)."""
    pr = _cproblem(8, 4, 2, 3, seed=21)

    def loss(q):
        S = lambda a: a[None]
        r = oracle.scan_slices(S(q["logits"]), q["idx"].astype(np.int32), S(q["d"]), S(q["B"]), S(q["C"]),
                               S(q["x"]), S(q["h0"]), want_prod=False)
        return float(np.real(np.sum(np.conj(q["dy"]) * r["y"][0]) + np.sum(np.conj(q["dh_final"]) * r["h_final"][0])))

    got = bwd.slice_backward(**pr)["d" + name]
    base = pr[name]
    fd = np.zeros_like(base)
    eps = 1e-6
    for i in np.ndindex(base.shape):
        parts = []
        for step in (eps, 1j * eps):
            hi, lo = dict(pr), dict(pr)
            hi[name], lo[name] = base.copy(), base.copy()
            hi[name][i] += step
            lo[name][i] -= step
            parts.append((loss(hi) - loss(lo)) / (2 * eps))
        fd[i] = parts[0] + 1j * parts[1]
    np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7)


def test_conjugating_every_complex_input_conjugates_the_complex_gradients():
    """With B, C, x real, conj(d, h0, dy, dh_final) leaves the loss unchanged and
    conjugates y and H, so dd and dh0 conjugate and the real gradients stay."""
    pr = _cproblem(15, 5, 3, 4, seed=8)
    a = bwd.slice_backward(**pr)
    pc = dict(pr)
    for k in ("d", "h0", "dy", "dh_final"):
        pc[k] = np.conj(pr[k])
    b = bwd.slice_backward(**pc)
    np.testing.assert_allclose(b["dd"], np.conj(a["dd"]), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b["dh0"], np.conj(a["dh0"]), rtol=1e-12, atol=1e-13)
    for k in ("dB", "dC", "dx", "dlogits"):
        np.testing.assert_allclose(b[k], a[k], rtol=1e-12, atol=1e-13, err_msg=k)
