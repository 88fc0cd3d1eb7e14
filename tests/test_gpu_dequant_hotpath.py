"""Bit-exact check of the dequantisation inside the product kernels themselves.

With one-hot activations every fp32 sum of a product has exactly one non-zero term, so each
output of owq_gemv / owq_gemm must equal one dequantised weight of the effective matrix bit
for bit: W_hat[i, j] = fp16_rn(s (q - z)) ("Storage Methods", appendix §2 of the OWQ paper as
summarised on paperlayer.ai: the zero-filled low-precision matrix) at a dense column, and the
fp16 weak value W[i, j] at a weak column (its zero-filled code contributes exactly 0).

This reaches every dequantisation form the product kernels use:
  * decode, 1-8 tokens, per-channel scales: codes as exact q 2^(o - 24) into offset-class
    accumulators, y = s (sum q x - z sum x) per row segment (one rounding to fp16);
  * decode, 1-3 tokens, per-group scales: the same, folded per 128-code block;
  * decode, 9-16 tokens (and per-group layers from 4 tokens): each code pair dequantised in
    registers to fp16_rn(s (q - z)) before the tensor-core product;
  * decode with the activations read from global memory in fragment order (wide layers);
  * prefill (tcgen05): the A operand dequantised into tensor memory;
and the fused weak-column term of each.  The expected values come only from the oracle.

One IEEE-754 detail: an output is the sum of its dense term and its weak term.  At a weak
column the dense term is the zero-filled code's +0, so a weak value of -0 gives +0 + (-0) = +0
(the oracle's fp64 product gives +0 as well); the expected bit pattern of such an entry is +0.
"""
import numpy as np
import pytest

import oracle
import owq_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"
_CACHE = {}

# (name, N, K, bits, group, k, T, planted weak channels)
SMALL = [
    ("b3-perchannel", 512, 512, 3, 512, 4, 256, None),
    ("b4-g128-ragged-n", 37, 256, 4, 128, 5, 64, None),
    ("b3-g128-edges", 96, 640, 3, 128, 4, 48, (0, 639, 255, 256)),
    ("b4-perchannel-edges", 130, 1024, 4, 1024, 6, 48, (0, 1023, 127, 128, 511, 512)),
    ("b3-g128-k0", 64, 384, 3, 128, 0, 32, None),
    ("b4-g128-kb-odd", 48, 11 * 128, 4, 128, 11, 40, None),
]

# full-size layers of the decode / prefill workloads: (workload id, layer index)
FULL = [(1, 0), (1, 5), (2, 4), (4, 0)]


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _small(case):
    name, N, K, bits, group, k, T, edges = case
    if name not in _CACHE:
        d = owq_synth.draw_small(N, K, 1, T, seed=4000 + N + K + k, n_outliers=0 if edges else min(3, k))
        if edges:
            ch = np.array(edges)
            d["X"][:, ch] = (d["X"][:, ch].astype(np.float32) * 50).astype(np.float16)
        _CACHE[name] = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    return _CACHE[name]


def _full(wid, li):
    key = ("full", wid, li)
    if key not in _CACHE:
        for kk in [c for c in _CACHE if c[0] == "full"]:
            del _CACHE[kk]
        spec = owq_synth.WORKLOADS[wid]
        L = spec.layers[li]
        d = owq_synth.draw_layer(L, spec, 1, owq_synth.seed_for(wid, li))
        _CACHE[key] = (L, oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k))
    return _CACHE[key]


def _w_eff_bits(ref):
    """The effective matrix as fp16 bit patterns: W_hat, with the weak columns' fp16 values."""
    w = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"]).copy()
    if ref["idx"].size:
        assert np.all(w[:, ref["idx"]] == 0)
        w[:, ref["idx"]] = ref["w_weak"]
    bits = w.view(np.uint16).copy()
    bits[bits == 0x8000] = 0   # +0 (dense) + (-0) (weak) = +0
    return bits


def _layer(owq, ref, bits, group):
    k = ref["idx"].size
    return owq.OwqLayer(_gpu(ref["codes"]), _gpu(ref["scales"]), _gpu(ref["zeros"]),
                        _gpu(ref["idx"]) if k else None, _gpu(ref["w_weak"]) if k else None, bits, group)


def _one_hot(cols, K):
    x = np.zeros((len(cols), K), np.float16)
    x[np.arange(len(cols)), cols] = 1.0
    return x


def _gemv_columns(layer, cols, K, M):
    """y[:, c] for every column c of `cols`, M one-hot tokens per call (as N x len(cols))."""
    out = []
    for c0 in range(0, len(cols), M):
        cs = list(cols[c0:c0 + M])
        pad = M - len(cs)
        x = _one_hot(cs + [cs[-1]] * pad, K)
        y = layer.gemv(_gpu(x))
        out.append(y[:len(cs)].cpu().numpy())
    torch.cuda.synchronize()
    return np.concatenate(out, axis=0).T


def _sample_cols(K, idx, n, seed):
    """Block edges, every weak column and its neighbours, and a seeded sample."""
    g = owq_synth.rng(seed)
    cols = {0, K - 1}
    for b in range(0, K, 128):
        cols |= {b, b + 1, min(K - 1, b + 127)}
    for j in np.asarray(idx).tolist():
        cols |= {j, max(0, j - 1), min(K - 1, j + 1)}
    cols |= set(g.choice(K, size=min(n, K), replace=False).tolist())
    return np.array(sorted(cols))


def _assert_bits(got_fp16, expect_bits, where):
    got = np.asarray(got_fp16, dtype=np.float16).view(np.uint16)
    bad = got != expect_bits
    assert not bad.any(), (f"{where}: {int(bad.sum())} of {bad.size} outputs differ from W_eff, first at "
                           f"{np.argwhere(bad)[0].tolist()}")


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


@pytest.mark.parametrize("M", [1, 3, 8, 16])
@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_gemv_one_hot_reproduces_w_eff(owq, case, M):
    name, N, K, bits, group, k, T, edges = case
    ref = _small(case)
    want = _w_eff_bits(ref)
    layer = _layer(owq, ref, bits, group)
    cols = np.arange(K) if M > 1 else _sample_cols(K, ref["idx"], 48, 11)
    y = _gemv_columns(layer, cols, K, M)
    _assert_bits(y, want[:, cols], f"{name} gemv M={M}")
    layer.close()


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_gemm_identity_reproduces_w_eff_transposed(owq, case):
    """x = I_K (K one-hot tokens): y = W_eff^T, every entry bit for bit."""
    name, N, K, bits, group, k, T, edges = case
    ref = _small(case)
    layer = _layer(owq, ref, bits, group)
    y = layer.gemm(_gpu(np.eye(K, dtype=np.float16)))
    torch.cuda.synchronize()
    assert owq.owq_device_status() == 0
    _assert_bits(y.cpu().numpy().T, _w_eff_bits(ref), f"{name} gemm x=I")
    layer.close()


@pytest.mark.parametrize("wid,li", FULL, ids=[f"w{w}l{l}" for w, l in FULL])
def test_fullsize_one_hot_products_reproduce_w_eff(owq, wid, li):
    """Full-size layers: every column through the tcgen05 GEMM (x = I_K, in slabs of 2048
    tokens), and sampled columns through the decode GEMV at 1, 8 and 16 tokens."""
    L, ref = _full(wid, li)
    want = _w_eff_bits(ref)
    layer = _layer(owq, ref, L.bits, L.group)
    slab = 2048
    for c0 in range(0, L.K, slab):
        cs = np.arange(c0, min(L.K, c0 + slab))
        y = layer.gemm(_gpu(_one_hot(cs, L.K)))
        torch.cuda.synchronize()
        _assert_bits(y.cpu().numpy().T, want[:, cs], f"{L.name} gemm cols {c0}..")
    assert owq.owq_device_status() == 0
    cols = _sample_cols(L.K, ref["idx"], 64, 100 + li)
    for M in (1, 8, 16):
        sel = cols if M > 1 else cols[:: max(1, len(cols) // 64)]
        _assert_bits(_gemv_columns(layer, sel, L.K, M), want[:, sel], f"{L.name} gemv M={M}")
    layer.close()


@pytest.mark.parametrize("kind", ["b4-g128", "b3-perchannel"])
def test_gemv_multi_one_hot_reproduces_w_eff(owq, kind):
    """Several layers of one kind in one owq_gemv_multi launch, as gate/up (4-bit, g = 128)
    and q/k/v (3-bit, per channel) run: every column of each layer."""
    if kind == "b4-g128":
        cases = [c for c in SMALL if c[4] == 128 and c[3] == 4]
    else:
        cases = [("mq", 64, 512, 3, 512, 4, 32, None), ("mk", 80, 512, 3, 512, 3, 32, None),
                 ("mv", 48, 512, 3, 512, 0, 32, None)]
    refs = [_small(c) for c in cases]
    layers = [_layer(owq, r, c[3], c[4]) for r, c in zip(refs, cases)]
    Kmax = max(c[2] for c in cases)
    for M in (1, 3, 8, 16):
        for c0 in range(0, Kmax, M):
            xs, cols_all = [], []
            for c, r in zip(cases, refs):
                K = c[2]
                cols = [(c0 + m) % K for m in range(M)]
                cols_all.append(cols)
                xs.append(_gpu(_one_hot(cols, K)))
            ys = [torch.empty((M, c[1]), dtype=torch.float16, device=DEV) for c in cases]
            assert owq.owq_gemv_multi([l.handle for l in layers], xs, ys, M) == 0
            torch.cuda.synchronize()
            for c, r, y, cols in zip(cases, refs, ys, cols_all):
                _assert_bits(y.cpu().numpy().T, _w_eff_bits(r)[:, cols], f"{c[0]} multi M={M} c0={c0}")
    for l in layers:
        l.close()
