"""The oracle against hand-worked automaton runs (tests/golden/*.txt): exact
state tracking through non-invertible transitions (Proposition 1 of the Flash
PD-SSM summary page) and exact composed products with non-unit decays."""
import numpy as np
import pytest

import oracle
from tests import golden


@pytest.mark.parametrize("name", golden.names())
def test_oracle_reproduces_the_hand_worked_run(name):
    inp, exp = golden.load(name)
    r = oracle.scan(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"])
    assert r["s"][0, :, 0].tolist() == exp["s"]
    assert r["y"][0, :, 0, 0].tolist() == exp["y"]
    assert r["h_final"][0, 0, :, 0].tolist() == exp["h_final"]
    assert r["prod_idx"][0, 0].tolist() == exp["prod_idx"]
    assert r["prod_val"][0, 0].tolist() == exp["prod_val"]


def test_fixtures_are_present():
    assert len(golden.names()) >= 2


def test_a_planted_transposition_is_caught():
    """Reading idx as row one-hot (the transposed reading the pages rule out) must
    break the hand-worked run: the fixtures distinguish the two orientations."""
    inp, exp = golden.load("fsa_advance_merge_weighted")
    idx = inp["idx"].numpy()
    L, N = inp["B"].shape[1], inp["B"].shape[-1]
    H = np.zeros(N)
    s = exp["s"]
    d = inp["d"][0, :, 0].numpy()
    for t in range(L):
        Pk = np.zeros((N, N))
        Pk[idx[s[t]], np.arange(N)] = 1.0       # column one-hot, as in the pages
        A = Pk.T @ np.diag(d[t])                # the transposed operand
        H = A @ H + inp["B"][0, t, 0].numpy()
    assert H.tolist() != exp["h_final"]


@pytest.mark.parametrize("name", [n for n in golden.names() if "bwd_dB" in golden.load(n)[1]])
def test_backward_oracle_reproduces_the_hand_worked_gradients(name):
    """The loss sum_t y_t (dy = 1, no final-state gradient) on the weighted automaton:
    every gradient worked by hand in the fixture header."""
    import numpy as np
    from oracle import backward as bwd
    inp, exp = golden.load(name)
    sl = lambda t: t[0, :, 0].double().numpy()
    L, P = inp["x"].shape[1], inp["x"].shape[-1]
    r = bwd.slice_backward(sl(inp["logits"]), inp["idx"].numpy(), sl(inp["d"]), sl(inp["B"]), sl(inp["C"]),
                           sl(inp["x"]), np.ones((L, P)))
    assert r["dC"].tolist() == exp["bwd_dC"]
    assert r["dB"].tolist() == exp["bwd_dB"]
    assert r["dd"].tolist() == exp["bwd_dd"]
    assert r["dx"][:, 0].tolist() == exp["bwd_dx"]
    assert r["dh0"][:, 0].tolist() == exp["bwd_dh0"]
