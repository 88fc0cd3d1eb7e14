"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: quantiser outputs (codes, scales, zeros, weak indices, weak block), unpacked
codes and dequantised fp16 weights.  Within tolerance (tests/owq_checks.py): the GEMV and
GEMM outputs against the oracle's fp64 product.
"""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _bits16(a):
    return np.asarray(a).view(np.uint16)


# (name, N, K, bits, group, k, T, edges) -- edges: channels whose calibration and activations
# get a x50 outlier so they are selected (weak columns at 0, K-1 and an adjacent pair).
SMALL_CASES = [
    ("w0-512", 512, 512, 3, 512, 4, 256, None),
    ("ragged-n37-g128-b4", 37, 256, 4, 128, 5, 64, None),
    ("k0", 64, 384, 3, 128, 0, 32, None),
    ("k1-perchannel", 64, 384, 3, 384, 1, 32, None),
    ("edges", 130, 1024, 4, 1024, 6, 48, (0, 1023, 127, 128, 511, 512)),
    ("edges-g128", 96, 640, 3, 128, 4, 48, (0, 639, 255, 256)),
    ("kb-odd", 48, 11 * 128, 3, 128, 11, 40, None),
    ("k-all-in-one-group", 40, 512, 4, 128, 7, 40, (130, 131, 132, 133, 134, 135, 136)),
]

_CACHE = {}


def _case_data(case):
    name, N, K, bits, group, k, T, edges = case
    if name in _CACHE:
        return _CACHE[name]
    if name == "w0-512":
        spec = owq_synth.WORKLOADS[0]
        d = owq_synth.draw_layer(spec.layers[0], spec, 16, owq_synth.seed_for(0, 0))
    else:
        d = owq_synth.draw_small(N, K, 16, T, seed=1000 + N + K + k, n_outliers=0 if edges else min(3, k))
        if edges:
            ch = np.array(edges)
            d["X"][:, ch] = (d["X"][:, ch].astype(np.float32) * 50).astype(np.float16)
            d["x"][:, ch] = (d["x"][:, ch].astype(np.float32) * 20).astype(np.float16)
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    ref["W_hat"] = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    _CACHE[name] = (d, ref)
    return d, ref


def _quantize(owq, d, bits, group, k):
    q = owq.quantize(_gpu(d["W"]), _gpu(d["X"]), bits, group, k)
    torch.cuda.synchronize()
    return q


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_quantize_bit_exact(owq, case):
    name, N, K, bits, group, k, T, edges = case
    d, ref = _case_data(case)
    q = _quantize(owq, d, bits, group, k)
    assert q["idx"].cpu().numpy().tolist() == ref["idx"].tolist()
    if edges:
        assert set(edges) <= set(ref["idx"].tolist())
    assert np.array_equal(q["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(_bits16(q["scales"].cpu().numpy()), _bits16(ref["scales"]))
    assert np.array_equal(_bits16(q["zeros"].cpu().numpy()), _bits16(ref["zeros"]))
    assert np.array_equal(_bits16(q["w_weak"].cpu().numpy()), _bits16(ref["w_weak"]))


@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_pack_dequant_bit_exact(owq, case):
    name, N, K, bits, group, k, T, edges = case
    d, ref = _case_data(case)
    layer = owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]),
                         _gpu(ref["idx"]) if k else None, _gpu(ref["w_weak"]) if k else None, bits, group)
    w_hat, codes = layer.dequant(with_codes=True)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(_bits16(w_hat.cpu().numpy()), _bits16(ref["W_hat"]))
    b = layer.nbytes()
    assert b == oracle.layer_bytes(N, K, bits, group, k)
    layer.close()


@pytest.mark.parametrize("bits", [3, 4])
def test_pack_rewrites_weak_codes_to_zero_point(owq, bits):
    g = owq_synth.rng(77 + bits)
    N, K, group = 33, 512, 128
    codes = owq_synth.draw_codes(g, N, K, bits)
    zeros = g.integers(0, 1 << bits, size=(N, K // group)).astype(np.float16)
    scales = (g.uniform(0.001, 0.01, size=(N, K // group))).astype(np.float16)
    idx = np.array([0, 31, 32, 200, 511], dtype=np.int32)
    w_weak = owq_synth.draw_weight(g, N, idx.size)
    layer = owq.OwqLayer(_gpu(codes), _gpu(scales), _gpu(zeros), _gpu(idx), _gpu(w_weak), bits, group)
    w_hat, got = layer.dequant(with_codes=True)
    torch.cuda.synchronize()
    expect = codes.copy()
    expect[:, idx] = np.repeat(zeros.astype(np.uint8), group, axis=1)[:, idx]
    assert np.array_equal(got.cpu().numpy(), expect)
    assert np.array_equal(_bits16(w_hat.cpu().numpy()), _bits16(oracle.dequant(expect, scales, zeros)))
    assert np.all(w_hat.cpu().numpy()[:, idx] == 0)


def _layer_from_ref(owq, ref, bits, group, k):
    return owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]),
                        _gpu(ref["idx"]) if k else None, _gpu(ref["w_weak"]) if k else None, bits, group)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_gemv_parity(owq, case, M):
    name, N, K, bits, group, k, T, edges = case
    d, ref = _case_data(case)
    layer = _layer_from_ref(owq, ref, bits, group, k)
    x = d["x"][:M]
    y = layer.gemv(_gpu(x))
    torch.cuda.synchronize()
    y64 = oracle.matmul(ref["W_hat"], ref["w_weak"], ref["idx"], x)
    check_output(y.cpu().numpy(), y64, f"{name} M={M}")
    layer.close()


@pytest.mark.parametrize("M", [1, 7, 16, 64, 65, 100, 128, 129, 300])
@pytest.mark.parametrize("case", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_gemm_parity(owq, case, M):
    name, N, K, bits, group, k, T, edges = case
    d, ref = _case_data(case)
    layer = _layer_from_ref(owq, ref, bits, group, k)
    g = owq_synth.rng(5000 + M)
    gain = np.ones(K, np.float32)
    if edges:
        gain[list(edges)] = 20.0
    x = owq_synth.draw_activations(g, M, gain)
    y = layer.gemm(_gpu(x))
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    y64 = oracle.matmul(ref["W_hat"], ref["w_weak"], ref["idx"], x)
    check_output(y.cpu().numpy(), y64, f"{name} M={M}")
    layer.close()


def test_gemv_multi_matches_single(owq):
    layers, xs, ys_single = [], [], []
    for j, case in enumerate(SMALL_CASES[:3]):
        name, N, K, bits, group, k, T, edges = case
        if bits != 3:
            continue
        d, ref = _case_data(case)
        layers.append(_layer_from_ref(owq, ref, bits, group, k))
        xs.append(_gpu(d["x"][:2]))
        ys_single.append(layers[-1].gemv(xs[-1]))
    ys = [torch.empty_like(y) for y in ys_single]
    assert owq.owq_gemv_multi([L.handle for L in layers], xs, ys, 2) == 0
    torch.cuda.synchronize()
    for a, b in zip(ys, ys_single):
        # the multi launch may split K differently (fp32 sums in another order)
        assert float(torch.abs(a.float() - b.float()).max()) <= 1e-2
    for L in layers:
        L.close()


def test_gpu_error_paths(owq):
    N, K = 16, 256
    codes = torch.zeros((N, K), dtype=torch.uint8, device=DEV)
    sz = torch.ones((N, 2), dtype=torch.float16, device=DEV)
    w_weak = torch.zeros((N, 8), dtype=torch.float16, device=DEV)
    for bad in ([3, 3], [5, 2], [-1, 4], [4, 256]):
        idx = torch.tensor(bad + [0] * 2, dtype=torch.int32, device=DEV)
        st, h = owq.owq_pack(codes, N, K, 3, 128, sz, sz, idx, 2, w_weak)
        assert st == 5 and h is None, bad
    layer = owq.OwqLayer(codes, sz, sz, None, None, 3, 128)
    x = torch.zeros((32, K), dtype=torch.float16, device=DEV)
    y = torch.zeros((32, N), dtype=torch.float16, device=DEV)
    assert owq.owq_gemv(layer.handle, x, y, 0) == 2
    assert owq.owq_gemv(layer.handle, x, y, 17) == 2
    assert owq.owq_gemm(layer.handle, x, y, 0) == 2
    assert owq.owq_gemv(layer.handle, x[:, 1:], y, 1) == 6
    layer.close()
    assert owq.owq_gemv(layer.handle or 0, x, y, 1) == 10


# Shapes whose row tiles are split inside CTAs and across CTAs in the decode launch (N x K,
# bits, group, k): every partial sum is added in a fixed order, so repeated calls agree bit
# for bit.
DETERMINISM_SHAPES = [(4096, 11008, 4, 128, 86), (16384, 4096, 3, 4096, 32), (4096, 4096, 3, 4096, 32)]


@pytest.mark.parametrize("shape", DETERMINISM_SHAPES, ids=[f"{s[0]}x{s[1]}" for s in DETERMINISM_SHAPES])
def test_repeated_calls_are_bit_identical(owq, shape):
    N, K, bits, group, k = shape
    d = owq_synth.draw_small(N, K, 64, 64, seed=300 + bits)
    layer, _ = owq.quantize_pack(_gpu(d["W"]), _gpu(d["X"]), bits, group, k)
    x = _gpu(d["x"])
    for M in (1, 5, 9, 16):
        xm = x[:M].contiguous()
        y0 = layer.gemv(xm)
        for _ in range(3):
            assert torch.equal(layer.gemv(xm).view(torch.int16), y0.view(torch.int16)), M
    y0 = layer.gemm(x)
    assert torch.equal(layer.gemm(x).view(torch.int16), y0.view(torch.int16))
    assert owq.owq_device_status() == 0
    layer.close()
