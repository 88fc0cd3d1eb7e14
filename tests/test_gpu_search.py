"""The truncation-aware (step, zero) grid search on the GPU ("Low-precision quantization",
paper "Quantization Configuration Search", pp.4-5, as summarised on paperlayer.ai), against
oracle.search_params bit for bit: the chosen fp16 scale and zero point of every (row, group).

Cases cover per-channel and g = 128 groups, 3 and 4 bits, weak columns left out of the search
(a whole group of them too), an all-zero row (the [-1, 1] range), a row below fp16 resolution
(every candidate step rounds to 0: the fallback), planted outliers that the search truncates,
and sampled rows of full-size layers (the search is independent per row).
"""
import numpy as np
import pytest

import oracle
import owq_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _search_gpu(owq, W, bits, group, idx):
    N, K = W.shape
    k = len(idx)
    s = torch.empty((N, K // group), dtype=torch.float16, device=DEV)
    z = torch.empty((N, K // group), dtype=torch.float16, device=DEV)
    st = owq.owq_search_params(_gpu(W), N, K, bits, group, _gpu(np.asarray(idx, np.int32)) if k else None, k, s, z)
    assert st == 0
    torch.cuda.synchronize()
    return s.cpu().numpy(), z.cpu().numpy()


def _weights(N, K, seed, outliers=True):
    g = owq_synth.rng(seed)
    W = owq_synth.draw_weight(g, N, K)
    if outliers:   # a few large weights per row: the search should truncate them
        r = g.integers(0, K, size=(N, 2))
        W[np.arange(N)[:, None], r] = (W[np.arange(N)[:, None], r].astype(np.float32) * 12).astype(np.float16)
    return W


SMALL = [
    ("b3-g128", 8, 256, 3, 128, [5, 77, 200]),
    ("b3-perchannel", 16, 512, 3, 512, [0, 1, 300, 511]),
    ("b4-g128", 12, 384, 4, 128, [127, 128, 129]),
    ("b4-perchannel-k0", 6, 256, 4, 256, []),
    ("b3-g128-weak-group", 4, 256, 3, 128, list(range(128, 256))),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_search_params_bit_exact(owq, case):
    name, N, K, bits, group, idx = case
    W = _weights(N, K, 600 + N + K)
    W[0, :] = 0                                        # an all-zero row: range [-1, 1]
    W[1, :] = np.float16(6e-8)                         # below fp16 resolution: fallback
    s, z = _search_gpu(owq, W, bits, group, idx)
    s_ref, z_ref = oracle.search_params(W, bits, group, np.asarray(idx, np.int64) if idx else None)
    assert np.array_equal(s.view(np.uint16), s_ref.view(np.uint16)), name
    assert np.array_equal(z.view(np.uint16), z_ref.view(np.uint16)), name


@pytest.mark.parametrize("wid,li,rows", [(1, 0, 12), (2, 4, 2), (4, 1, 2)], ids=["opt6.7b-q", "llama7b-gate", "llama13b-down"])
def test_search_params_fullsize_sampled_rows(owq, wid, li, rows):
    spec = owq_synth.WORKLOADS[wid]
    L = spec.layers[li]
    g = owq_synth.rng(700 + li)
    W = owq_synth.draw_weight(g, L.N, L.K)
    idx = np.sort(g.choice(L.K, size=L.k, replace=False)).astype(np.int32)
    s, z = _search_gpu(owq, W, L.bits, L.group, idx)
    sel = np.unique(np.r_[0:rows // 2, L.N - rows // 2:L.N])
    s_ref, z_ref = oracle.search_params(W[sel], L.bits, L.group, idx.astype(np.int64))
    assert np.array_equal(s[sel].view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(z[sel].view(np.uint16), z_ref.view(np.uint16))


def test_search_params_rejects_bad_indices(owq):
    W = torch.zeros((4, 256), dtype=torch.float16, device=DEV)
    s = torch.empty((4, 2), dtype=torch.float16, device=DEV)
    for bad in ([3, 3], [5, 2], [-1, 4], [4, 256]):
        assert owq.owq_search_params(W, 4, 256, 3, 128, _gpu(np.array(bad, np.int32)), 2, s, s) == 5
