"""Parity of the weak column tuning kernels with the CPU oracle, through the C ABI.

owq_input_grad (fp16 dX = dY W_eff, read from the packed layout) is held to the output
tolerance of tests/owq_checks.py against the oracle's fp64 input_grad.  owq_weak_grad (fp32
dW_weak = dY^T x[:, idx]) is held to the fp32 accumulation bound: the fp16 x fp16 products
are exact in fp32, so each of the M additions adds at most 2^-24 of the running sum.
Layers are quantised by the oracle and packed by owq_pack; no expected value comes from the
GPU.
"""
import numpy as np
import pytest

import oracle
import owq_synth
from tests.owq_checks import check_output

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"
F64 = np.float64

# (name, N, K, bits, group, k, token counts, channels forced weak)
CASES = [
    ("one-slice", 48, 256, 3, 256, 3, (1, 2), None),
    ("ragged-n200", 200, 640, 3, 640, 7, (1, 5, 16), None),
    ("g128-b4-two-passes", 200, 640, 4, 128, 7, (3, 37), None),
    ("k0", 96, 384, 3, 128, 0, (4,), None),
    ("many-slices", 1000, 1280, 3, 128, 13, (16,), None),
    ("edges-pair-weak", 130, 1024, 4, 1024, 6, (8,), (0, 1023, 2, 3, 511, 512)),
    ("token-splits", 256, 512, 3, 128, 40, (1000,), None),
    ("cluster-of-3", 300, 384, 3, 384, 5, (1, 9), None),
    # 40 weak columns in one block over 512-row slices: too many to stage in shared memory
    ("weak-heavy-block", 4096, 256, 4, 128, 40, (2, 16), tuple(range(0, 80, 2))),
    # from 17 tokens (N % 8 == 0): the tensor-memory pipeline, token tiles of 64 / 128 / 256,
    # ragged 128-row steps, then the weak-column pass
    ("many-tokens-3b", 520, 640, 3, 640, 7, (17, 33, 100, 300), None),
    ("many-tokens-4b-g128", 384, 512, 4, 128, 13, (64, 257), None),
    ("many-tokens-k0", 256, 384, 4, 128, 0, (40,), None),
    ("many-tokens-weak-heavy", 1024, 256, 3, 128, 40, (48,), tuple(range(0, 80, 2))),
    # N % 8 != 0: many tokens run through the 16-token kernel
    ("many-tokens-n-odd", 130, 512, 3, 128, 6, (40,), None),
]


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _layer(owq, ref, bits, group):
    k = len(ref["idx"])
    return owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]),
                        _gpu(ref["idx"]) if k else None, _gpu(ref["w_weak"]) if k else None, bits, group)


def _dy(M, N, seed):
    return owq_synth.rng(seed).standard_normal((M, N), dtype=np.float32).astype(np.float16)


def _check_weak_grad(got, x, dy, idx, where):
    want = oracle.weak_grad(x, dy, idx)
    got = np.asarray(got, dtype=F64)
    assert got.shape == want.shape
    terms = np.abs(dy.astype(F64)).T @ np.abs(x.astype(F64)[:, idx])
    bound = dy.shape[0] * 2.0 ** -24 * terms + 1e-30
    err = np.abs(got - want)
    assert np.all(err <= bound), f"{where}: weak grad error {float(err.max()):.3g}"


def _check_input_grad_bound(got, W_hat, w_weak, idx, dy, where):
    """Per output: the kernel multiplies dY by the unrounded s (q - z) (dY s carried as an fp16
    pair to 2^-22), the oracle by W_hat = fp16_rn(s (q - z)); each weight differs by at most half
    an fp16 spacing, 2^-11 of its magnitude (2^-25 absolute below the normal range).  So
    |dx - dx64| <= 2^-11 sum_i |dY_i W_eff_ij| + 2^-25 sum_i |dY_i| + half an fp16 spacing of
    dx64 + 2^-20 sum_i |dY_i W_eff_ij| (fp32 accumulation)."""
    want = oracle.input_grad(W_hat, w_weak, idx, dy)
    w_eff = np.abs(W_hat.astype(F64))
    if len(idx):
        w_eff[:, idx] = np.abs(w_weak.astype(F64))
    ady = np.abs(dy.astype(F64))
    terms = ady @ w_eff
    bound = ((2.0 ** -11 + 2.0 ** -20) * terms + 2.0 ** -25 * ady.sum(axis=1, keepdims=True)
             + 0.5 * np.spacing(np.abs(want).astype(np.float16)).astype(F64))
    err = np.abs(np.asarray(got, dtype=np.float16).astype(F64) - want)
    assert np.all(err <= bound), f"{where}: input grad error {float((err - bound).max()):.3g} over the bound"


def _case(case):
    name, N, K, bits, group, k, Ms, forced = case
    d = owq_synth.draw_small(N, K, max(Ms), 48, seed=2000 + N + K + k, n_outliers=0 if forced else min(3, k))
    if forced:
        ch = np.array(forced)
        d["X"][:, ch] = (d["X"][:, ch].astype(np.float32) * 50).astype(np.float16)
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    if forced:
        assert set(forced) <= set(ref["idx"].tolist())
    return d, ref


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_wct_gradients_match_oracle(case):
    import weight_only_mixed_owq_b200 as owq
    name, N, K, bits, group, k, Ms, forced = case
    d, ref = _case(case)
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    layer = _layer(owq, ref, bits, group)
    for M in Ms:
        dy = _dy(M, N, 31 + M)
        x = d["x"][:M]
        dy_g, x_g = _gpu(dy), _gpu(x)
        dx = layer.input_grad(dy_g)
        dx2 = layer.input_grad(dy_g)
        dw = layer.weak_grad(x_g, dy_g)
        torch.cuda.synchronize()
        check_output(dx.cpu().numpy(), oracle.input_grad(W_hat, ref["w_weak"], ref["idx"], dy),
                     f"{name} input_grad M={M}")
        _check_input_grad_bound(dx.cpu().numpy(), W_hat, ref["w_weak"], ref["idx"], dy, f"{name} M={M}")
        assert torch.equal(dx.view(torch.int16), dx2.view(torch.int16)), "repeat differs"
        if k:
            _check_weak_grad(dw.cpu().numpy(), x, dy, ref["idx"], f"{name} M={M}")
    layer.close()


def test_wct_gradients_fullsize_opt67b_attention_layer():
    """4096 x 4096, 3-bit per channel, k = 32 (the OPT-6.7B q/k/v/out shape), in the launch
    configuration bench.py times; every output compared."""
    import weight_only_mixed_owq_b200 as owq
    spec = owq_synth.WORKLOADS[1]
    L = spec.layers[0]
    d = owq_synth.draw_layer(L, spec, 2048, owq_synth.seed_for(1, 0))
    ref = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    layer = _layer(owq, ref, L.bits, L.group)
    for M in (1, 16, 256, 2048):   # the 16-token kernel, then the tcgen05 path (128- / 256-token tiles)
        dy = _dy(M, L.N, 77 + M)
        x = d["x"][:M]
        dx = layer.input_grad(_gpu(dy))
        dw = layer.weak_grad(_gpu(x), _gpu(dy))
        torch.cuda.synchronize()
        check_output(dx.cpu().numpy(), oracle.input_grad(W_hat, ref["w_weak"], ref["idx"], dy),
                     f"{L.name} input_grad M={M}")
        _check_input_grad_bound(dx.cpu().numpy(), W_hat, ref["w_weak"], ref["idx"], dy, f"{L.name} M={M}")
        _check_weak_grad(dw.cpu().numpy(), x, dy, ref["idx"], f"{L.name} M={M}")
    layer.close()


ONE_HOT = [CASES[1], CASES[2], CASES[5], CASES[7], CASES[8], CASES[9], CASES[10], CASES[12]]


@pytest.mark.parametrize("case", ONE_HOT, ids=lambda c: c[0])
def test_input_grad_one_hot_rows_are_w_eff(case):
    """One nonzero dY (1.0) per token: dX's row is row i of W_eff (W_hat with the weak columns'
    fp16 values) bit for bit, since the kernel's only rounding is then the final fp16 one
    (-0 weak values give +0: +0 (dense) + (-0) (weak) = +0)."""
    import weight_only_mixed_owq_b200 as owq
    name, N, K, bits, group, k, Ms, forced = case
    d, ref = _case(case)
    w = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"]).copy()
    if k:
        assert np.all(w[:, ref["idx"]] == 0)
        w[:, ref["idx"]] = ref["w_weak"]
    want = w.view(np.uint16).copy()
    want[want == 0x8000] = 0
    layer = _layer(owq, ref, bits, group)
    rows = np.unique(np.concatenate([[0, N - 1, N // 2], np.arange(0, N, max(1, N // 29))]))
    # 16 tokens per call (the 16-token kernel); with M >= 17 in a case, all rows in one call too
    # (the tensor-memory pipeline when N % 8 == 0; rows repeated up to 40 tokens)
    groups = [rows[r0:r0 + 16] for r0 in range(0, len(rows), 16)]
    if max(Ms) >= 17:
        groups.append(np.resize(rows, max(40, len(rows))))
    for rr in groups:
        dy = np.zeros((len(rr), N), dtype=np.float16)
        dy[np.arange(len(rr)), rr] = 1.0
        got = layer.input_grad(_gpu(dy)).cpu().numpy().view(np.uint16)
        bad = np.argwhere(got != want[rr])
        assert bad.size == 0, f"{name}: row {rr[bad[0][0]]} column {bad[0][1]}: {got[tuple(bad[0])]:#06x} != {want[rr][tuple(bad[0])]:#06x}"
    layer.close()


def test_wct_error_paths():
    import weight_only_mixed_owq_b200 as owq
    d, ref = _case(CASES[0])
    layer = _layer(owq, ref, 3, 256)
    buf = torch.zeros(4096, dtype=torch.float16, device=DEV)
    f32 = torch.zeros(4096, dtype=torch.float32, device=DEV)
    h = layer.handle
    assert owq.owq_input_grad(h, buf, buf, 0) == 2            # OWQ_ERR_SHAPE
    assert owq.owq_input_grad(h, buf, buf, 65537) == 2
    assert owq.owq_input_grad(h, None, buf, 1) == 1           # OWQ_ERR_NULL
    assert owq.owq_input_grad(h, buf.data_ptr() + 2, buf, 1) == 6   # OWQ_ERR_ALIGN
    assert owq.owq_weak_grad(h, buf, buf, None, 1) == 1       # k > 0 needs an output
    assert owq.owq_weak_grad(h, buf, buf, f32.data_ptr() + 4, 1) == 6
    assert owq.owq_weak_grad(h, buf, buf, f32, 0) == 2
    assert owq.owq_weak_grad(None, buf, buf, f32, 1) == owq.owq_input_grad(None, buf, buf, 1)
    layer.close()


@pytest.mark.parametrize("M", [8, 300])
def test_wct_products_captured_in_a_graph_on_a_fresh_handle(M):
    """Both products inside a CUDA graph capture on a handle that has never run them, so no
    scratch can be grown: the input gradient (16-token kernel at M = 8, tcgen05 path with the
    weak-column pass at M = 300) and the weak-block gradient take their one-split forms; the
    replayed results meet the same bounds as uncaptured calls."""
    import weight_only_mixed_owq_b200 as owq
    case = CASES[9]   # 520 x 640, 3-bit, 7 weak columns
    name, N, K, bits, group, k, Ms, forced = case
    d, ref = _case(case)
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    layer = _layer(owq, ref, bits, group)
    dy = _dy(M, N, 123)
    x = d["x"][:M] if d["x"].shape[0] >= M else np.resize(d["x"], (M, K)).astype(np.float16)
    dy_g, x_g = _gpu(dy), _gpu(x)
    dx = torch.empty((M, K), dtype=torch.float16, device=DEV)
    dw = torch.empty((N, k), dtype=torch.float32, device=DEV)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.input_grad(dy_g, dx)
        layer.weak_grad(x_g, dy_g, dw)
    dx.zero_()
    dw.zero_()
    g.replay()
    torch.cuda.synchronize()
    want = oracle.input_grad(W_hat, ref["w_weak"], ref["idx"], dy)
    check_output(dx.cpu().numpy(), want, f"captured input_grad M={M}")
    _check_input_grad_bound(dx.cpu().numpy(), W_hat, ref["w_weak"], ref["idx"], dy, f"captured M={M}")
    _check_weak_grad(dw.cpu().numpy(), x, dy, ref["idx"], f"captured weak_grad M={M}")
    assert owq.owq_device_status() == owq.OWQ_OK
    del g
    layer.close()
