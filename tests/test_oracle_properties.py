"""Property checks of the oracle over random shapes (CPU, hypothesis).

Each property is fixed by the definitions, not by the oracle's own formulas: a layout round
trip is the identity, the two layouts agree, and the gradients are the adjoint and the
directional derivative of the (separately pinned) forward product.
"""
import numpy as np
import pytest

import oracle

hyp = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

F16, F64 = np.float16, np.float64
SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


def _weak(rng, K, k):
    return np.sort(rng.choice(K, size=k, replace=False)).astype(np.int32)


@SETTINGS
@given(bits=st.sampled_from([3, 4]), N=st.integers(1, 9), kb=st.integers(1, 3), k=st.integers(0, 20),
       seed=st.integers(0, 2 ** 31 - 1))
def test_both_layouts_round_trip_to_the_same_codes(bits, N, kb, k, seed):
    rng = np.random.default_rng(seed)
    K = 128 * kb
    codes = rng.integers(0, 1 << bits, size=(N, K)).astype(np.uint8)
    idx = _weak(rng, K, k)
    zeros = rng.integers(0, 1 << bits, size=(N, 1)).astype(F16)
    for t in idx:
        codes[:, t] = zeros[:, 0].astype(np.uint8)
    assert np.array_equal(oracle.unpack(oracle.pack(codes, bits), K, bits), codes)
    back = oracle.unpack_storage(oracle.pack_storage(codes, idx, bits), K, idx, bits, zeros, K)
    assert np.array_equal(back, codes)


@SETTINGS
@given(N=st.integers(1, 8), K=st.integers(1, 40), k=st.integers(0, 6), M=st.integers(1, 4),
       seed=st.integers(0, 2 ** 31 - 1))
def test_gradients_are_adjoint_and_derivative_of_forward(N, K, k, M, seed):
    rng = np.random.default_rng(seed)
    k = min(k, K)
    idx = _weak(rng, K, k)
    W_hat = (rng.standard_normal((N, K)) * 0.1).astype(F16)
    W_hat[:, idx] = 0
    w_weak = (rng.standard_normal((N, k)) * 0.1).astype(F16)
    x = rng.standard_normal((M, K)).astype(F16)
    dy = rng.standard_normal((M, N)).astype(F16)
    y = oracle.matmul(W_hat, w_weak, idx, x)
    dx = oracle.input_grad(W_hat, w_weak, idx, dy)
    lhs = float((dy.astype(F64) * y).sum())
    assert float((dx * x.astype(F64)).sum()) == pytest.approx(lhs, rel=1e-10, abs=1e-10)
    if k:
        V = rng.standard_normal((N, k)).astype(F16)
        g = oracle.weak_grad(x, dy, idx)
        yv = oracle.matmul(np.zeros_like(W_hat), V, idx, x)
        assert float((g * V.astype(F64)).sum()) == pytest.approx(float((dy.astype(F64) * yv).sum()),
                                                                 rel=1e-10, abs=1e-10)
