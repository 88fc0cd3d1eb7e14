"""owq_quantize_noalloc: the quantiser for callers that cannot let a library allocate GPU
memory (serving processes that reserve the device's memory for their own pool up front, or
that forbid allocation after start-up).  Its scratch is a static device array, so two calls
in a row reuse the same memory; both must give exactly what owq_quantize gives (the
quantiser's outputs are compared bit for bit everywhere in these tests).

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.  It also passes alone in a fresh process.
"""
import numpy as np
import pytest

import owq_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"


def _alloc(N, K, group, k):
    return {
        "codes": torch.empty((N, K), dtype=torch.uint8, device=DEV),
        "scales": torch.empty((N, K // group), dtype=torch.float16, device=DEV),
        "zeros": torch.empty((N, K // group), dtype=torch.float16, device=DEV),
        "idx": torch.empty((k,), dtype=torch.int32, device=DEV),
        "w_weak": torch.empty((N, k), dtype=torch.float16, device=DEV),
    }


def _run(fn, W, X, bits, group, k):
    N, K = W.shape
    out = _alloc(N, K, group, k)
    st = fn(W, X, N, K, X.shape[0], bits, group, k, out["codes"], out["scales"], out["zeros"],
            out["idx"], out["w_weak"])
    assert st == 0, st
    return out


def _same(a, b):
    for key in ("codes", "scales", "zeros", "idx", "w_weak"):
        x, y = a[key], b[key]
        if x.dtype == torch.float16:
            x, y = x.view(torch.int16), y.view(torch.int16)
        assert torch.equal(x, y), key


def test_noalloc_matches_allocating_quantiser_on_two_calls_in_a_row():
    import weight_only_mixed_owq_b200 as owq
    cases = [(256, 1024, 3, 1024, 8, 64, 11), (96, 640, 4, 128, 5, 48, 12)]
    inputs = []
    for N, K, bits, group, k, T, seed in cases:
        d = owq_synth.draw_small(N, K, 1, T, seed=seed, n_outliers=3)
        inputs.append((torch.from_numpy(d["W"]).to(DEV), torch.from_numpy(d["X"]).to(DEV), bits, group, k))
    # two back-to-back no-alloc calls (the second reuses the scratch the first left behind)
    got = [_run(owq.owq_quantize_noalloc, W, X, b, g, k) for W, X, b, g, k in inputs]
    # and the first problem again, after the second one changed the scratch
    again = _run(owq.owq_quantize_noalloc, *inputs[0])
    torch.cuda.synchronize()
    ref = [_run(owq.owq_quantize, W, X, b, g, k) for W, X, b, g, k in inputs]
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        _same(a, b)
    _same(again, ref[0])


def test_noalloc_rejects_k_beyond_static_scratch():
    import weight_only_mixed_owq_b200 as owq
    A = torch.empty(16, dtype=torch.uint8, device=DEV)
    K = 40960 + 128
    st = owq.owq_quantize_noalloc(A, A, 8, K, 4, 3, K, 1, A, A, A, A, A)
    assert st == 2  # OWQ_ERR_SHAPE, nothing launched
