"""The seeded input recipe: shapes, dtypes, reproducibility and the value
distributions each configuration states (weights ~N(0, 0.02) with 1 % of the
decode weight at +-6 sigma, A ~U(+-1/sqrt(K)), B ~N(0, 0.01), X and dY ~N(0, 1))."""
import math

import numpy as np
import pytest
import torch

from bit_nf4_quantized_24_b200 import workloads as wl

SHAPES = {
    "fwd_2048": (128, [(2048, 2048)], 8, 16.0, False),
    "qproj_7b": (4096, [(4096, 4096)], 16, 32.0, True),
    "mlp_7b": (8192, [(11008, 4096), (11008, 4096), (4096, 11008)], 64, 128.0, True),
    "decode_70b_up": (16, [(28672, 8192)], 16, 32.0, False),
    "layer_70b": (4096, [(8192, 8192), (1024, 8192), (1024, 8192), (8192, 8192), (28672, 8192), (28672, 8192),
                         (8192, 28672)], 64, 16.0, True),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_workload_shapes(name):
    M, projs, r, alpha, bwd = SHAPES[name]
    w = wl.WORKLOADS[name]
    assert w.M == M and w.r == r and w.alpha == alpha and w.backward == bwd
    assert [(p.N, p.K) for p in w.projections] == projs
    assert w.scale == alpha / r


def test_draw_is_seeded_and_typed():
    w = wl.WORKLOADS["fwd_2048"]
    a, b = wl.draw_linear(w), wl.draw_linear(w)
    for k in ("X", "W", "A", "B"):
        assert torch.equal(a[k], b[k]), k
    assert a["X"].dtype == a["A"].dtype == a["B"].dtype == torch.bfloat16 and a["W"].dtype == torch.float32
    assert a["X"].shape == (128, 2048) and a["A"].shape == (8, 2048) and a["B"].shape == (2048, 8)
    # the weight and adapters do not depend on the token count; the activations do
    c = wl.draw_linear(w, M=64)
    assert torch.equal(c["W"], a["W"]) and torch.equal(c["A"], a["A"]) and c["X"].shape == (64, 2048)


def test_value_distributions():
    w = wl.WORKLOADS["qproj_7b"]
    p = wl.draw_linear(w)
    W, A, B = p["W"].numpy(), p["A"].float().numpy(), p["B"].float().numpy()
    X, dY = p["X"].float().numpy(), p["dY"].float().numpy()
    assert abs(W.std() - 0.02) < 2e-4 and abs(W.mean()) < 1e-4
    bound = 1 / math.sqrt(4096)
    assert np.abs(A).max() <= bound * (1 + 2 ** -8) and abs(A.std() - bound / math.sqrt(3)) < 2e-3 * bound * 10
    assert abs(B.std() - 0.01) < 3e-4
    assert abs(X.std() - 1) < 5e-3 and abs(dY.std() - 1) < 5e-3


def test_decode_weight_outliers():
    g = wl.generator(3)
    W = wl.draw_weight(g, 1024, 2048, 0.02, outlier_frac=0.01, outlier_sigmas=6.0).numpy()
    big = np.isclose(np.abs(W), 0.12, rtol=0, atol=1e-7)
    frac = big.mean()
    assert 0.009 < frac < 0.011
    assert abs((W[big] > 0).mean() - 0.5) < 0.03   # random sign
    w = wl.WORKLOADS["decode_70b_up"]
    assert w.outlier_frac == 0.01 and w.outlier_sigmas == 6.0 and w.w_std == 0.02
