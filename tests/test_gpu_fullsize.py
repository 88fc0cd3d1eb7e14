"""Parity at the full layer sizes of the OPT / LLaMA-shaped workloads, in the launch
configurations bench.py times.

The quantiser is compared bit for bit on the whole layer; the products on seeded samples of
output rows (the oracle's fp64 product of those rows), with the tolerance of
tests/owq_checks.py.
"""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"
_CACHE = {}

# (workload id, layer index, token counts for the decode product, token counts for the prefill product)
CASES = [
    (1, 5, (1, 3), ()),            # OPT-6.7B fc2 4096 x 16384, 3-bit per channel, k = 128
    (1, 4, (1,), ()),              # OPT-6.7B fc1 16384 x 4096
    (2, 6, (1, 2, 4, 8, 16), ()),  # LLaMA-7B down 4096 x 11008, 4-bit g128, k = 86
    (3, 5, (1,), ()),              # OPT-66B fc2 9216 x 36864, 3-bit per channel, k = 288
    (4, 0, (), (64, 2048)),        # LLaMA-13B up 13824 x 5120, 3-bit g128, k = 40
    (4, 1, (), (128,)),            # LLaMA-13B down 5120 x 13824, k = 108
]


def _layer(wid, li):
    key = (wid, li)
    if key not in _CACHE:
        spec = owq_synth.WORKLOADS[wid]
        L = spec.layers[li]
        d = owq_synth.draw_layer(L, spec, max(spec.Ms), owq_synth.seed_for(wid, li))
        ref = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
        _CACHE.clear()
        _CACHE[key] = (L, d, ref)
    return _CACHE[key]


def _rows(N, seed, n=256):
    g = owq_synth.rng(seed)
    return np.unique(np.concatenate([[0, N - 1], g.choice(N, size=min(n, N), replace=False)]))


@pytest.mark.parametrize("case", CASES, ids=[f"w{c[0]}l{c[1]}" for c in CASES])
def test_fullsize_quantize_and_products(case):
    import weight_only_mixed_owq_b200 as owq
    wid, li, Ms_dec, Ms_pre = case
    L, d, ref = _layer(wid, li)
    W = torch.from_numpy(d["W"]).to(DEV)
    X = torch.from_numpy(d["X"]).to(DEV)
    layer, q = owq.quantize_pack(W, X, L.bits, L.group, L.k)
    torch.cuda.synchronize()
    del W, X
    assert q["idx"].cpu().numpy().tolist() == ref["idx"].tolist()
    assert np.array_equal(q["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(q["scales"].cpu().numpy().view(np.uint16), ref["scales"].view(np.uint16))
    assert np.array_equal(q["zeros"].cpu().numpy().view(np.uint16), ref["zeros"].view(np.uint16))
    rows = _rows(L.N, 17 + li)
    for M in Ms_dec:
        x = d["x"][:M]
        y = layer.gemv(torch.from_numpy(x).to(DEV))
        torch.cuda.synchronize()
        y64 = oracle.matmul_rows(ref["codes"], ref["scales"], ref["zeros"], ref["w_weak"], ref["idx"], x, rows)
        check_output(y.cpu().numpy()[:, rows], y64, f"{L.name} gemv M={M}")
    for M in Ms_pre:
        x = d["x"][:M]
        y = layer.gemm(torch.from_numpy(x).to(DEV))
        torch.cuda.synchronize()
        assert owq.owq_device_status() == 0
        y64 = oracle.matmul_rows(ref["codes"], ref["scales"], ref["zeros"], ref["w_weak"], ref["idx"], x, rows)
        check_output(y.cpu().numpy()[:, rows], y64, f"{L.name} gemm M={M}")
    layer.close()


def test_fullsize_qkv_multi_launch_matches_oracle():
    """q, k, v of the OPT-6.7B set in one owq_gemv_multi launch (as bench.py runs them).

    A multi launch may split K differently from three single launches (it has three times the
    row tiles), so the two agree to fp32 rounding, not bit for bit; both must meet the
    tolerance against the oracle."""
    import weight_only_mixed_owq_b200 as owq
    spec = owq_synth.WORKLOADS[1]
    layers, xs, single, refs, xs_np = [], [], [], [], []
    for li in range(3):
        L = spec.layers[li]
        d = owq_synth.draw_layer(L, spec, 1, owq_synth.seed_for(1, li))
        ref = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
        lay, _ = owq.quantize_pack(torch.from_numpy(d["W"]).to(DEV), torch.from_numpy(d["X"]).to(DEV),
                                   L.bits, L.group, L.k)
        layers.append(lay)
        xs.append(torch.from_numpy(d["x"]).to(DEV))
        xs_np.append(d["x"])
        refs.append(ref)
        single.append(lay.gemv(xs[-1]))
    ys = [torch.empty_like(y) for y in single]
    assert owq.owq_gemv_multi([l.handle for l in layers], xs, ys, 1) == 0
    torch.cuda.synchronize()
    rows = _rows(4096, 99)
    for a, b, ref, x in zip(ys, single, refs, xs_np):
        assert float(torch.abs(a.float() - b.float()).max()) <= 1e-2
        y64 = oracle.matmul_rows(ref["codes"], ref["scales"], ref["zeros"], ref["w_weak"], ref["idx"], x, rows)
        check_output(a.cpu().numpy()[:, rows], y64, "qkv multi")
        check_output(b.cpu().numpy()[:, rows], y64, "qkv single")
    for l in layers:
        l.close()
