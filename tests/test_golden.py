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
