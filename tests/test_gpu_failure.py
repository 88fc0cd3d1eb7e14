"""Failure detection on the GPU without a fault: a hand-off that never comes makes the
kernel's bounded waits run out.

owq_debug_inject arms one lost hand-off for the next call (split-tile partial sums published
under a tag no reader accepts for the decode kernel; one skipped mbarrier arrival for the
prefill kernel) and shortens that call's wait bound to about a millisecond.  The call must
end by itself, the device status word must read OWQ_ERR_TIMEOUT, and the next call on the
same handle must reproduce the earlier output bit for bit (the context stays usable and the
injection is one-shot).
"""
import numpy as np
import pytest

import owq_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"
WAIT_CYCLES = 2_000_000   # about 1 ms at the B200's clock
OWQ_ERR_TIMEOUT = 8

# N x K layers whose row tiles cross CTA boundaries in the decode split (K / 128 = 86 blocks
# per tile does not divide a CTA's share of the units)
LAYERS = [
    (4096, 11008, 3, 11008, 86),
    (4096, 11008, 4, 128, 86),
]


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


def _layer(owq, N, K, bits, group, k, seed):
    d = owq_synth.draw_small(N, K, 16, 64, seed=seed)
    W = torch.from_numpy(d["W"]).to(DEV)
    X = torch.from_numpy(d["X"]).to(DEV)
    layer, _ = owq.quantize_pack(W, X, bits, group, k)
    x = torch.from_numpy(d["x"]).to(DEV)
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    return layer, x


@pytest.mark.parametrize("spec", LAYERS, ids=[f"b{s[2]}g{s[3]}" for s in LAYERS])
@pytest.mark.parametrize("M", [1, 16])
def test_gemv_lost_handoff_times_out_then_recovers(owq, spec, M):
    N, K, bits, group, k = spec
    layer, x = _layer(owq, N, K, bits, group, k, seed=71 + bits)
    xm = x[:M].contiguous()
    y0 = layer.gemv(xm)
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    assert owq.owq_debug_inject(owq.OWQ_INJECT_GEMV_TAG, WAIT_CYCLES) == 0
    y_bad = torch.zeros_like(y0)
    layer.gemv(xm, y_bad)
    assert owq.owq_device_status() == OWQ_ERR_TIMEOUT
    y1 = layer.gemv(xm)
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    layer.close()


@pytest.mark.parametrize("M", [64, 128, 1024])   # split-K (64, 128) and one split (1024)
def test_gemm_lost_arrival_times_out_then_recovers(owq, M):
    N, K, bits, group, k = 4096, 4096, 3, 128, 32
    d = owq_synth.draw_small(N, K, M, 64, seed=5 + M)
    layer, _ = owq.quantize_pack(torch.from_numpy(d["W"]).to(DEV), torch.from_numpy(d["X"]).to(DEV), bits, group, k)
    x = torch.from_numpy(d["x"]).to(DEV)
    y0 = layer.gemm(x)
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    assert owq.owq_debug_inject(owq.OWQ_INJECT_GEMM_ARRIVE, WAIT_CYCLES) == 0
    layer.gemm(x, torch.empty_like(y0))
    assert owq.owq_device_status() == OWQ_ERR_TIMEOUT
    y1 = layer.gemm(x)
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    layer.close()


def test_injection_of_one_kind_leaves_the_other_untouched(owq):
    N, K, bits, group, k = 4096, 11008, 3, 11008, 86
    layer, x = _layer(owq, N, K, bits, group, k, seed=90)
    y0 = layer.gemv(x[:1].contiguous())
    assert owq.owq_debug_inject(owq.OWQ_INJECT_GEMM_ARRIVE, WAIT_CYCLES) == 0
    y1 = layer.gemv(x[:1].contiguous())          # a decode call does not take a prefill failure
    assert owq.owq_device_status() == 0
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert owq.owq_debug_inject(owq.OWQ_INJECT_NONE, 0) == 0   # disarm
    layer.gemm(x[:64].contiguous())
    assert owq.owq_device_status() == 0
    layer.close()
