"""Hand-worked fixtures (text) and their reader; the expected values in each file are
derived by hand in its header and come from no program."""
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def names():
    return sorted(f[:-4] for f in os.listdir(HERE) if f.endswith(".txt"))


def load(name):
    """Returns (inputs as [1, L, 1, *] tensors in the given dtypes, expected values)."""
    fields = {}
    with open(os.path.join(HERE, name + ".txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, _, v = line.partition(":")
                fields[k.strip()] = v.strip()
    N, P, K = int(fields["N"]), int(fields["P"]), int(fields["K"])
    idx = [[int(v) for v in row.split()] for row in fields["idx"].split("|")]
    letters = [int(v) for v in fields["letters"].split()]
    L = len(letters)
    d = [float(v) for v in fields["d"].split()]
    d = d * N if len(d) == 1 else d
    C = [float(v) for v in fields["C"].split()]
    logits = torch.zeros(1, L, 1, K)
    for t, k in enumerate(letters):
        logits[0, t, 0, k] = 1.0
    B = torch.zeros(1, L, 1, N)
    B[0, 0, 0, 0] = 1.0
    inp = {
        "logits": logits,
        "idx": torch.tensor(idx, dtype=torch.int32),
        "d": torch.tensor(d).expand(1, L, 1, N).contiguous(),
        "B": B,
        "C": torch.tensor(C).expand(1, L, 1, N).contiguous(),
        "x": torch.ones(1, L, 1, P),
    }
    exp = {
        "y": [float(v) for v in fields["y"].split()],
        "h_final": [float(v) for v in fields["h_final"].split()],
        "prod_idx": [int(v) for v in fields["prod_idx"].split()],
        "prod_val": [float(v) for v in fields["prod_val"].split()],
        "s": letters,
    }
    for k in ("bwd_dC", "bwd_dB", "bwd_dd"):  # [L][N], rows separated by |
        if k in fields:
            exp[k] = [[float(v) for v in row.split()] for row in fields[k].split("|")]
    for k in ("bwd_dx", "bwd_dh0"):
        if k in fields:
            exp[k] = [float(v) for v in fields[k].split()]
    assert len(idx) == K and all(len(r) == N for r in idx) and len(exp["y"]) == L
    return inp, exp
