"""OPTQ with the weak columns last on the GPU ("Low-precision quantization", paper p.4, as
summarised on paperlayer.ai), against oracle.optq_quantize.

The oracle recomputes the inverse of H over the columns not yet quantised at every step; the
kernels keep that inverse by the exact Schur-complement downdate.  The two are the same
arithmetic up to fp64 rounding order, so a code decision can differ only where a compensated
weight sits within fp64 noise of a rounding boundary: the codes must agree (all but a
vanishing fraction), and the compensated weak block to one fp16 spacing.  At a size the
oracle cannot reach in seconds, the result is checked against the property that defines it:
the weak columns end at the least-squares optimum of the row's calibration error given its
quantised dense columns.
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


def _optq_gpu(owq, W, X, bits, group, idx, scales, zeros, damp):
    N, K = W.shape
    k = len(idx)
    codes = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    w_weak = torch.empty((N, max(k, 1)), dtype=torch.float16, device=DEV)
    st = owq.owq_optq(_gpu(W), _gpu(X), N, K, X.shape[0], bits, group, _gpu(idx) if k else None, k,
                      _gpu(scales), _gpu(zeros), damp, codes, w_weak if k else None)
    assert st == 0
    torch.cuda.synchronize()
    return codes.cpu().numpy(), w_weak.cpu().numpy()[:, :k]


def _ulps(a, b):
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    sp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float16)).astype(np.float64)
    return np.abs(a64 - b64) / sp


# (name, N, K, T, bits, group, k, damp)
CASES = [
    ("b3-g128", 32, 256, 64, 3, 128, 4, 0.01),
    ("b4-perchannel", 24, 384, 48, 4, 384, 6, 0.01),
    ("b3-perchannel-k0", 16, 128, 32, 3, 128, 0, 0.01),
    ("b4-g128-nodamp", 16, 128, 512, 4, 128, 3, 0.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_optq_matches_oracle(owq, case):
    name, N, K, T, bits, group, k, damp = case
    d = owq_synth.draw_small(N, K, 1, T, seed=800 + K + k, n_outliers=min(3, k))
    W, X = d["W"], d["X"]
    sel = oracle.owq_quantize(W, X, bits, group, k)
    idx = sel["idx"]
    scales, zeros = oracle.search_params(W, bits, group, idx if k else None)
    ref = oracle.optq_quantize(W, X, bits, group, idx, scales, zeros, damp)
    codes, w_weak = _optq_gpu(owq, W, X, bits, group, idx, scales, zeros, damp)
    mism = codes != ref["codes"]
    assert mism.mean() <= 1e-3, f"{name}: {int(mism.sum())} codes differ"
    ok_rows = ~mism.any(axis=1)
    assert ok_rows.mean() >= 0.9, name
    if k:
        assert np.all(_ulps(w_weak[ok_rows], ref["w_weak"][ok_rows]) <= 1.0), name
        # the weak columns keep the group's zero point in the code matrix
        zc = np.repeat(zeros.astype(np.uint8), group, axis=1)[:, idx]
        assert np.array_equal(codes[:, idx], zc)


def test_quantize_optq_pipeline_matches_oracle(owq):
    """Selection (owq_quantize), search (owq_search_params), OPTQ (owq_optq) composed as the
    paper's quantiser, against oracle.owq_quantize_optq."""
    N, K, T, bits, group, k = 40, 256, 64, 3, 128, 5
    d = owq_synth.draw_small(N, K, 1, T, seed=901, n_outliers=3)
    ref = oracle.owq_quantize_optq(d["W"], d["X"], bits, group, k)
    got = owq.quantize_optq(_gpu(d["W"]), _gpu(d["X"]), bits, group, k)
    torch.cuda.synchronize()
    assert got["idx"].cpu().numpy().tolist() == ref["idx"].tolist()
    assert np.array_equal(got["scales"].cpu().numpy().view(np.uint16), ref["scales"].view(np.uint16))
    assert np.array_equal(got["zeros"].cpu().numpy().view(np.uint16), ref["zeros"].view(np.uint16))
    codes = got["codes"].cpu().numpy()
    assert (codes != ref["codes"]).mean() <= 1e-3
    assert np.all(_ulps(got["w_weak"].cpu().numpy(), ref["w_weak"]) <= 1.0)


def test_optq_weak_columns_are_the_least_squares_optimum(owq):
    """A 2048-column layer (beyond the oracle's reach in seconds): given the quantised dense
    columns, the compensated weak columns minimise the row's damped calibration error
    (w - w_final) H (w - w_final)^T, i.e. H_ww (v - w_w) = -H_wd (w_hat_d - w_d)."""
    N, K, T, bits, group, k, damp = 64, 2048, 256, 3, 128, 16, 0.01
    d = owq_synth.draw_small(N, K, 1, T, seed=905, n_outliers=4)
    W, X = d["W"], d["X"]
    g = owq_synth.rng(906)
    idx = np.sort(g.choice(K, size=k, replace=False)).astype(np.int32)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=DEV)
    zeros = torch.empty_like(scales)
    assert owq.owq_search_params(_gpu(W), N, K, bits, group, _gpu(idx), k, scales, zeros) == 0
    s_np, z_np = scales.cpu().numpy(), zeros.cpu().numpy()
    codes, w_weak = _optq_gpu(owq, W, X, bits, group, idx, s_np, z_np, damp)
    W_hat = oracle.dequant(codes, s_np, z_np).astype(np.float64)
    X64 = X.astype(np.float64)
    H = X64.T @ X64
    H += damp * np.mean(np.diag(H)) * np.eye(K)
    dense = np.setdiff1d(np.arange(K), idx)
    Hww = H[np.ix_(idx, idx)]
    Hwd = H[np.ix_(idx, dense)]
    W64 = W.astype(np.float64)
    for r in range(0, N, 8):
        v = W64[r, idx] - np.linalg.solve(Hww, Hwd @ (W_hat[r, dense] - W64[r, dense]))
        assert np.all(_ulps(w_weak[r], v.astype(np.float16)) <= 1.0), r
