"""The synthetic input recipe: seeded and reproducible, with the shapes, value
distributions and outlier structure the benchmark and the parity tests state."""
import numpy as np
import torch

import workloads


def test_inputs_are_reproducible_and_shaped():
    w = workloads.WORKLOADS["single_1024"]
    a, b = workloads.make_inputs(w), workloads.make_inputs(w)
    for k in ("W0", "A", "B", "x", "dY"):
        assert torch.equal(a[k], b[k]), k
    assert a["W0"].shape == (w.N, w.K) and a["W0"].dtype == torch.float32
    assert a["x"].shape == (w.M, w.K) and a["x"].dtype == torch.bfloat16
    assert a["A"].shape == (w.r, w.K) and a["B"].shape == (w.N, w.r) and a["dY"].shape == (w.M, w.N)
    # another seed gives other tensors; fewer tokens keep the same weights
    c = workloads.make_inputs(w, seed=w.seed + 1)
    assert not torch.equal(a["W0"], c["W0"])
    d = workloads.make_inputs(w, M=4)
    assert torch.equal(a["W0"], d["W0"]) and d["x"].shape == (4, w.K)


def test_value_distributions():
    w = workloads.WORKLOADS["single_1024"]
    a = workloads.make_inputs(w)
    W0 = a["W0"].double()
    assert abs(W0.std().item() - w.sigma) < 0.02 * w.sigma and abs(W0.mean().item()) < 1e-3 * 5
    bound = 1.0 / w.K ** 0.5
    A = a["A"].double()
    assert A.abs().max().item() <= bound * (1 + 2 ** -8) and A.abs().max().item() > 0.9 * bound
    assert abs(a["B"].double().std().item() - 0.01) < 0.001
    assert abs(a["x"].double().std().item() - 1.0) < 0.02


def test_decode_weight_outliers():
    """round(0.001 N K) distinct positions of the 13824x5120 weight scaled by 20."""
    w = workloads.WORKLOADS["decode_mlp_up_13824x5120"]
    W = workloads.make_weight(w)
    plain = workloads.make_weight(w.with_(outlier_frac=0.0))
    ratio = (W / torch.where(plain == 0, torch.ones_like(plain), plain)).reshape(-1)
    scaled = torch.isclose(ratio, torch.tensor(20.0)).sum().item()
    assert scaled == int(round(0.001 * w.N * w.K))
    assert torch.equal(W[plain == 0], plain[plain == 0])


def test_stack_seeds_are_distinct():
    seeds = {workloads.stack_seed(l, p) for l in range(40) for p in range(4)}
    assert len(seeds) == 160
