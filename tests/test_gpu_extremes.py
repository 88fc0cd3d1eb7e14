"""Parity at the extremes of the documented ranges: the longest rows (K = 65536) with the most
weak columns (k = 1024), the shortest rows (K = 128, one block per row) on a tall layer, a
single output row, and the largest prefill token count (M = 65536).

Each case is quantised by the oracle and by the GPU (bit-exact), packed, dequantised
(bit-exact) and multiplied (owq_gemv at 1 and 16 tokens, owq_gemm) against the oracle's fp64
product within the tolerance of tests/owq_checks.py.
"""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output, check_output_short

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"

# (name, N, K, bits, group, k, T, gemm token counts)
CASES = [
    ("longest-rows-most-weak", 48, 65536, 3, 65536, 1024, 32, (64, 300)),
    ("longest-rows-g128", 40, 65536, 4, 128, 512, 32, (129,)),
    ("tall-one-block", 131072, 128, 4, 128, 1, 16, (100,)),
    ("single-row", 1, 128, 3, 128, 1, 16, (1, 64)),
]


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _bits16(a):
    return np.asarray(a).view(np.uint16)


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_extreme_shapes(owq, case):
    name, N, K, bits, group, k, T, gemm_Ms = case
    d = owq_synth.draw_small(N, K, max(16, max(gemm_Ms)), T, seed=4000 + K + N, n_outliers=min(3, k))
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    q = owq.quantize(_gpu(d["W"]), _gpu(d["X"]), bits, group, k)
    torch.cuda.synchronize()
    assert q["idx"].cpu().numpy().tolist() == ref["idx"].tolist()
    assert np.array_equal(q["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(_bits16(q["scales"].cpu().numpy()), _bits16(ref["scales"]))
    assert np.array_equal(_bits16(q["zeros"].cpu().numpy()), _bits16(ref["zeros"]))
    assert np.array_equal(_bits16(q["w_weak"].cpu().numpy()), _bits16(ref["w_weak"]))
    layer = owq.OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"], q["w_weak"], bits, group)
    w_hat = layer.dequant()
    torch.cuda.synchronize()
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    assert np.array_equal(_bits16(w_hat.cpu().numpy()), _bits16(W_hat))
    del w_hat
    for M in (1, 16):
        x = d["x"][:M]
        y = layer.gemv(_gpu(x))
        torch.cuda.synchronize()
        y64 = oracle.matmul(W_hat, ref["w_weak"], ref["idx"], x)
        if N * M == 1:   # one output: rel-L2 is the relative error of one dot product
            check_output_short(y.cpu().numpy(), W_hat, ref["w_weak"], ref["idx"], x, y64, f"{name} gemv M={M}")
        else:
            check_output(y.cpu().numpy(), y64, f"{name} gemv M={M}")
    for M in gemm_Ms:
        x = d["x"][:M]
        y = layer.gemm(_gpu(x))
        torch.cuda.synchronize()
        assert owq.owq_device_status() == 0
        check_output(y.cpu().numpy(), oracle.matmul(W_hat, ref["w_weak"], ref["idx"], x), f"{name} gemm M={M}")
    layer.close()


def test_gemm_largest_token_count(owq):
    """M = 65536 (the documented maximum) on a small layer: every output checked."""
    N, K, bits, group, k, M = 128, 256, 3, 128, 2, 65536
    d = owq_synth.draw_small(N, K, 16, 64, seed=4242, n_outliers=2)
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    layer = owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]), _gpu(ref["idx"]),
                         _gpu(ref["w_weak"]), bits, group)
    g = owq_synth.rng(4243)
    gain = np.ones(K, np.float32)
    gain[ref["idx"]] = 20.0
    x = owq_synth.draw_activations(g, M, gain)
    y = layer.gemm(_gpu(x))
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    check_output(y.cpu().numpy(), oracle.matmul(W_hat, ref["w_weak"], ref["idx"], x), "gemm M=65536")
    layer.close()
