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


def _pool_counters():
    """(high-water mark of the default memory pool since its last reset, its reserved bytes,
    free device memory) of the current device."""
    from cuda.bindings import runtime as rt
    dev = torch.cuda.current_device()
    err, pool = rt.cudaDeviceGetDefaultMemPool(dev)
    assert err == rt.cudaError_t.cudaSuccess
    err, high = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh)
    assert err == rt.cudaError_t.cudaSuccess
    err, reserved = rt.cudaMemPoolGetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrReservedMemCurrent)
    assert err == rt.cudaError_t.cudaSuccess
    err, free, _ = rt.cudaMemGetInfo()
    assert err == rt.cudaError_t.cudaSuccess
    return int(high), int(reserved), int(free)


def _reset_pool_high():
    from cuda.bindings import driver
    from cuda.bindings import runtime as rt
    err, pool = rt.cudaDeviceGetDefaultMemPool(torch.cuda.current_device())
    assert err == rt.cudaError_t.cudaSuccess
    err, = rt.cudaMemPoolSetAttribute(pool, rt.cudaMemPoolAttr.cudaMemPoolAttrUsedMemHigh, driver.cuuint64_t(0))
    assert err == rt.cudaError_t.cudaSuccess


def test_noalloc_allocates_no_device_memory():
    """The point of the entry point: no device allocation, neither stream-ordered (the default
    memory pool's high-water mark stays put) nor plain (free device memory does not drop).
    The same probe around the allocating owq_quantize sees its scratch, so it can tell."""
    import weight_only_mixed_owq_b200 as owq
    N, K, bits, group, k, T = 512, 4096, 3, 4096, 32, 64
    d = owq_synth.draw_small(N, K, 1, T, seed=21, n_outliers=3)
    W, X = torch.from_numpy(d["W"]).to(DEV), torch.from_numpy(d["X"]).to(DEV)
    outs = [_alloc(N, K, group, k) for _ in range(2)]
    # the first call on the device is its set-up (in a fresh process it also loads the code,
    # which takes device memory): the counters start after it
    out = outs[1]
    assert owq.owq_quantize_noalloc(W, X, N, K, T, bits, group, k, out["codes"], out["scales"], out["zeros"],
                                    out["idx"], out["w_weak"]) == 0
    torch.cuda.synchronize()
    _reset_pool_high()
    high0, reserved0, free0 = _pool_counters()
    for out in outs:
        assert owq.owq_quantize_noalloc(W, X, N, K, T, bits, group, k, out["codes"], out["scales"], out["zeros"],
                                        out["idx"], out["w_weak"]) == 0
    torch.cuda.synchronize()
    high1, reserved1, free1 = _pool_counters()
    assert high1 == high0, (high0, high1)
    assert reserved1 <= reserved0, (reserved0, reserved1)
    assert free1 >= free0, (free0, free1)
    # control: the allocating quantiser's stream-ordered scratch shows in the same counters
    _reset_pool_high()
    high2, _, _ = _pool_counters()
    out = outs[0]
    assert owq.owq_quantize(W, X, N, K, T, bits, group, k, out["codes"], out["scales"], out["zeros"],
                            out["idx"], out["w_weak"]) == 0
    torch.cuda.synchronize()
    high3, _, _ = _pool_counters()
    assert high3 > high2, (high2, high3)
