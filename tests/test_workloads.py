"""The seeded synthetic inputs follow the recipes of the five workloads (shapes, dtypes,
value distributions and structure) and are reproducible."""
import math

import pytest
import torch

import workloads


def test_generation_is_reproducible_and_seed_dependent():
    sp = workloads.spec("lm", batch=2, seqlen=40, heads=3)
    a, b = workloads.generate(sp, seed=5), workloads.generate(sp, seed=5)
    c = workloads.generate(sp, seed=6)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert not torch.equal(a["B"], c["B"]) and not torch.equal(a["idx"], c["idx"])


@pytest.mark.parametrize("recipe", workloads.CONFIG_ORDER)
def test_shapes_and_dtypes(recipe):
    full = workloads.spec(recipe)
    sp = workloads.spec(recipe, batch=1, seqlen=min(full.seqlen, 64), heads=min(full.heads, 2))
    g = workloads.generate(sp)
    Bt, L, H, N, P, K = sp.batch, sp.seqlen, sp.heads, sp.N, sp.P, sp.K
    assert g["idx"].shape == (K, N) and g["idx"].dtype == torch.int32
    assert g["logits"].shape == (Bt, L, H, K) and g["logits"].dtype == sp.logits_dtype
    assert g["d"].shape == (Bt, L, H, N) and g["d"].dtype == sp.d_dtype
    for k in ("B", "C"):
        assert g[k].shape == (Bt, L, H, N) and g[k].dtype == sp.in_dtype
    assert g["x"].shape == (Bt, L, H, P) and g["x"].dtype == sp.in_dtype
    assert int(g["idx"].min()) >= 0 and int(g["idx"].max()) < N


def test_full_size_shapes_of_the_five_workloads():
    shapes = {r: (s.batch, s.seqlen, s.heads, s.N, s.P, s.K) for r, s in workloads.RECIPES.items()}
    assert shapes == {"tiny": (1, 256, 1, 8, 4, 4), "z5": (64, 512, 1, 5, 1, 5), "lm": (8, 2048, 32, 64, 64, 16),
                      "long": (4, 18000, 8, 32, 32, 8), "complex": (16, 8192, 64, 128, 64, 64)}
    assert workloads.RECIPES["long"].seqlen % 64 != 0  # the long series is not a chunk multiple


def test_z5_is_the_cyclic_automaton():
    sp = workloads.spec("z5", batch=2, seqlen=30)
    g = workloads.generate(sp)
    j = torch.arange(5)
    for k in range(5):
        assert torch.equal(g["idx"][k], ((j + k) % 5).to(torch.int32))
    assert torch.all(g["d"] == 1) and torch.all(g["x"] == 1)
    assert torch.all(g["logits"].sum(-1) == 1) and torch.all((g["logits"] == 0) | (g["logits"] == 1))
    assert torch.all(g["B"][:, 0, :, 0] == 1) and g["B"].sum() == sp.batch * sp.heads
    t = torch.arange(sp.seqlen)
    assert torch.equal(g["C"][0, :, 0].argmax(-1), t % 5) and torch.all(g["C"].sum(-1) == 1)


def test_long_dictionary_is_permutations():
    idx = workloads.generate_idx(workloads.spec("long"))
    for row in idx:
        assert torch.equal(torch.sort(row).values, torch.arange(row.numel(), dtype=torch.int32))


def test_value_distributions():
    # tiny: d ~ U(0.5, 1); logits, B, C, x ~ N(0, 1)
    g = workloads.generate_slice(workloads.spec("tiny", seqlen=4000), 0, 0)
    assert float(g["d"].min()) >= 0.5 and float(g["d"].max()) < 1.0
    for k in ("logits", "B", "C", "x"):
        assert abs(float(g[k].mean())) < 0.05 and abs(float(g[k].std()) - 1.0) < 0.05, k
    # lm: d = exp(-softplus(z)) in (0, 1); B, C ~ N(0, 1/N); bf16 storage
    sp = workloads.spec("lm", seqlen=512)
    g = workloads.generate_slice(sp, 0, 0)
    d = g["d"].float()
    assert float(d.min()) > 0 and float(d.max()) < 1
    z = torch.log(torch.expm1(-torch.log(d.double())))  # softplus^-1(-log d), inverted in fp64
    assert abs(float(z.mean())) < 0.05 and abs(float(z.std()) - 1.0) < 0.1
    for k in ("B", "C"):
        assert abs(float(g[k].float().std()) - 1 / math.sqrt(sp.N)) < 0.01, k
    # complex: |d| = exp(-softplus(z)), angle uniform on (0, 2 pi)
    g = workloads.generate_slice(workloads.spec("complex", seqlen=256), 0, 0)
    r, th = g["d"].abs(), torch.angle(g["d"]) % (2 * math.pi)
    assert float(r.min()) > 0 and float(r.max()) < 1
    assert abs(float(th.mean()) - math.pi) < 0.05 and abs(float(th.std()) - math.pi / math.sqrt(3)) < 0.05
