"""The CPU oracle against its pins (see ``pins.py`` for what pins what)."""
import pytest

import pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(oracle, check):
    check(oracle)


def test_oracle_layer_is_composition(oracle):
    """orc_bitlinear is exactly its four steps run one after another."""
    import numpy as np
    rng = np.random.default_rng(3)
    M, K, N = 5, 128, 24
    x = pins._rand_bf16_x(rng, M, K)
    g = (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    y, beta = oracle.bitlinear(x, g, 1e-6, W, 1e-5)
    wt, b2 = oracle.absmean_ternary(W, 1e-5)
    q, a = oracle.rmsnorm_quant(x, g, 1e-6)
    y2 = oracle.rescale(oracle.ternary_acc(q, wt), a, b2)
    assert beta == b2 and (y == y2).all()


def test_oracle_thread_count_independent(oracle, monkeypatch):
    """The OpenMP split of orc_ternary_acc over tokens does not change results."""
    import numpy as np
    rng = np.random.default_rng(4)
    q = rng.integers(-127, 128, size=(33, 256)).astype(np.int8)
    wt = rng.integers(-1, 2, size=(17, 256)).astype(np.int8)
    ref = q.astype(np.int64) @ wt.astype(np.int64).T
    assert (oracle.ternary_acc(q, wt) == ref).all()
