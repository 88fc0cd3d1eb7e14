"""Parity at the full layer sizes of the OPT / LLaMA-shaped workloads, in the launch
configurations bench.py times.

The quantiser is compared bit for bit on the whole layer; the products on every output row
(the oracle's fp64 product, computed in row slabs), with the tolerance of tests/owq_checks.py.
The layer sets bench.py launches together (q/k/v, gate/up) are also run as one
owq_gemv_multi launch and compared with the oracle.
"""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output, oracle_rows_all

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
    (4, 1, (), (128, 2048)),       # LLaMA-13B down 5120 x 13824, k = 108 (2048: split tail)
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
    for M in Ms_dec:
        x = d["x"][:M]
        y = layer.gemv(torch.from_numpy(x).to(DEV))
        torch.cuda.synchronize()
        check_output(y.cpu().numpy(), oracle_rows_all(ref, x), f"{L.name} gemv M={M}")
    for M in Ms_pre:
        x = d["x"][:M]
        y = layer.gemm(torch.from_numpy(x).to(DEV))
        torch.cuda.synchronize()
        assert owq.owq_device_status() == 0
        check_output(y.cpu().numpy(), oracle_rows_all(ref, x), f"{L.name} gemm M={M}")
    layer.close()


# layer sets bench.py issues as one owq_gemv_multi launch: (workload id, layer indices, token counts)
MULTI = [
    (1, (0, 1, 2), (1,)),          # OPT-6.7B q, k, v: 3 x 4096 x 4096, 3-bit per channel, k = 32
    (2, (4, 5), (1, 4, 16)),       # LLaMA-7B gate, up: 2 x 11008 x 4096, 4-bit g128, k = 32
    (3, (0, 1, 2), (1,)),          # OPT-66B q, k, v: 3 x 9216 x 9216, 3-bit per channel, k = 72
]


@pytest.mark.parametrize("case", MULTI, ids=[f"w{c[0]}-{'-'.join(map(str, c[1]))}" for c in MULTI])
def test_fullsize_multi_launch_matches_oracle(case):
    """The layers that share an input in one owq_gemv_multi launch, exactly as bench.py issues
    them, against the oracle on every output row.  A multi launch apportions the SMs
    differently from single launches (so its fp32 sums may round differently from theirs);
    each must meet the tolerance against the oracle on its own."""
    import weight_only_mixed_owq_b200 as owq
    wid, lis, Ms = case
    spec = owq_synth.WORKLOADS[wid]
    layers, xs, refs, xs_np = [], [], [], []
    for li in lis:
        L = spec.layers[li]
        d = owq_synth.draw_layer(L, spec, max(Ms), owq_synth.seed_for(wid, li))
        ref = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
        layers.append(owq.OwqLayer(torch.from_numpy(ref["codes"]).to(DEV), torch.from_numpy(ref["scales"]).to(DEV),
                                   torch.from_numpy(ref["zeros"]).to(DEV), torch.from_numpy(ref["idx"]).to(DEV),
                                   torch.from_numpy(ref["w_weak"]).to(DEV), L.bits, L.group))
        xs_np.append(d["x"])
        refs.append(ref)
    for M in Ms:
        xs = [torch.from_numpy(np.ascontiguousarray(x[:M])).to(DEV) for x in xs_np]
        ys = [torch.empty((M, l.N), dtype=torch.float16, device=DEV) for l in layers]
        assert owq.owq_gemv_multi([l.handle for l in layers], xs, ys, M) == 0
        single = [l.gemv(x) for l, x in zip(layers, xs)]
        torch.cuda.synchronize()
        for j, (a, b, ref, x) in enumerate(zip(ys, single, refs, xs_np)):
            y64 = oracle_rows_all(ref, x[:M])
            check_output(a.cpu().numpy(), y64, f"w{wid} layer {lis[j]} multi M={M}")
            check_output(b.cpu().numpy(), y64, f"w{wid} layer {lis[j]} single M={M}")
    for l in layers:
        l.close()
