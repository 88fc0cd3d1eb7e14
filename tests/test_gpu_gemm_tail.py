"""Prefill products with a split tail: the last wave of whole tiles is short, so the row tiles
of the last one or two token tiles are split over K (owq_gemm_plan), their fp32 partials kept
in the handle's workspace and added in split order by the reduction.  Each case first asserts
that this device's plan takes the tail, then compares every output with the oracle's fp64
product (tolerance of tests/owq_checks.py) and checks that repeated calls give identical bits.
Cases: ragged token tiles, ragged row tiles, per-channel and per-group scales, 3 and 4 bits,
no weak columns, a two-token-tile tail."""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"

# (name, N, K, bits, group, k, token counts, tail token tiles expected)
CASES = [
    ("per-channel-3b", 5120, 4096, 3, 4096, 32, (1000, 2048), 1),
    ("g128-4b-no-weak", 5120, 4096, 4, 128, 0, (1024,), 1),
    ("ragged-rows-g128", 5100, 4096, 3, 128, 5, (1024,), 1),
    ("two-token-tiles", 2816, 4096, 3, 128, 16, (2048,), 2),
]


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gemm_tail_parity(case):
    import weight_only_mixed_owq_b200 as owq
    name, N, K, bits, group, k, Ms, tail_tiles = case
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for M in Ms:
        st, p = owq.owq_gemm_plan(N, K, M, sms)
        assert st == 0 and p["tail_tiles"] == tail_tiles and p["tail_splits"] > 1, (name, M, p)
    d = owq_synth.draw_small(N, K, max(Ms), 64, seed=5000 + N + bits, n_outliers=min(3, k))
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    layer = owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]), _gpu(ref["idx"]),
                         _gpu(ref["w_weak"]), bits, group)
    for M in Ms:
        x = d["x"][:M]
        xg = _gpu(x)
        y = layer.gemm(xg)
        y2 = layer.gemm(xg)
        torch.cuda.synchronize()
        assert owq.owq_device_status() == 0
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"{name} M={M}: repeated calls differ"
        check_output(y.cpu().numpy(), oracle.matmul(W_hat, ref["w_weak"], ref["idx"], x), f"{name} gemm M={M}")
    layer.close()
