"""Pins of the CPU oracle against what the OWQ pages and plain mathematics fix.

None of these tests re-types the oracle's formula: each one checks it against a hand-worked
value, a brute-force computation of a different quantity, a special case that reduces to a
library routine, or a bound.
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import owq_synth

F16, F64 = np.float16, np.float64


# ------------------------------------------------------------------ golden fixtures
def _read_rows(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([p.strip() for p in line.split("|")])
    return rows


def test_rtn_hand_worked_rows(golden_dir):
    for bits, weak, w, s, z, codes, w_hat in _read_rows(os.path.join(golden_dir, "rtn_rows.txt")):
        bits = int(bits)
        weak = [] if weak == "-" else [int(v) for v in weak.split(",")]
        W = np.array([[float(v) for v in w.split()]], dtype=F16)
        c, sc, zz = oracle.quantize_rtn(W, bits, W.shape[1], weak)
        assert float(sc[0, 0]) == float(s)
        assert float(zz[0, 0]) == float(z)
        assert c[0].tolist() == [int(v) for v in codes.split()]
        got = oracle.dequant(c, sc, zz)[0].astype(np.float64)
        assert got.tolist() == [float(v) for v in w_hat.split()]


def test_pack_hand_derived_words(golden_dir):
    for bits, rule, words in _read_rows(os.path.join(golden_dir, "pack_words.txt")):
        bits = int(bits)
        k = np.arange(128)
        if rule.startswith("pair"):   # pair p = (p mod 8, p // 8)
            codes = np.where(k % 2 == 0, (k // 2) % 8, (k // 16) % 8).astype(np.uint8)[None, :]
        else:
            mod = int(rule.split()[-1])
            codes = ((k // 8 if "//" in rule else k) % mod).astype(np.uint8)[None, :]
        got = oracle.pack(codes, bits)[0]
        assert [f"{int(v):08x}" for v in got] == words.split()
        assert oracle.unpack(got[None, :], 128, bits).tolist() == codes.tolist()


# ------------------------------------------------------------------ quantiser invariants
@pytest.mark.parametrize("bits,group", [(3, 64), (3, 256), (4, 128), (4, 256)])
def test_rtn_invariants_and_error_bound(bits, group):
    g = owq_synth.rng(7)
    N, K = 24, 256
    W = owq_synth.draw_weight(g, N, K)
    weak = np.sort(g.choice(K, size=5, replace=False))
    codes, s, z = oracle.quantize_rtn(W, bits, group, weak)
    qmax = (1 << bits) - 1
    assert codes.max() <= qmax
    zf = z.astype(np.float64)
    assert np.all(zf == np.round(zf)) and zf.min() >= 0 and zf.max() <= qmax
    W_hat = oracle.dequant(codes, s, z)
    # weak columns dequantise to exactly 0 (zero-filled latency layout)
    assert np.all(W_hat[:, weak] == 0)
    G = K // group
    s_full = np.repeat(s.astype(np.float64), group, axis=1)
    dense = np.ones(K, bool)
    dense[weak] = False
    err = np.abs(W.astype(F64) - W_hat.astype(F64))[:, dense]
    # RTN: at most s/2 from the grid, plus the final fp16 rounding of w_hat (2^-11 relative),
    # plus at most one step where a rounded-down fp16 scale forces a clamp at 2^b - 1.
    bound = s_full[:, dense] * 0.5 + np.abs(W_hat.astype(F64)[:, dense]) * 2.0 ** -11
    clamped = codes[:, dense] == qmax
    assert np.all((err <= bound * (1 + 1e-12)) | (clamped & (err <= s_full[:, dense] * 1.0001)))
    # the grid covers the dense range: max |w| within one step of the representable extremes
    assert np.all(s.astype(np.float64) > 0)
    assert G == s.shape[1]


def test_rtn_zero_point_is_canonical_integer():
    # a row with no negative entry has mn = 0, so z = 0: stored as +0 (bits 0x0000)
    W = np.array([[0.0, 0.25, 0.5, 1.0, -0.0, 0.125, 0.75, 0.0]], dtype=F16)
    c, s, z = oracle.quantize_rtn(W, 3, 8)
    assert z.view(np.uint16)[0, 0] == 0
    assert c[0].tolist() == [0, 2, 4, 7, 0, 1, 5, 0]


def test_rtn_k_equal_bits_reaches_extremes():
    # a row whose min and max are both non-zero uses code 0 and code 2^b - 1 exactly
    W = np.array([[-0.5, 0.25, 0.1, 1.25, 0.0, -0.3, 0.7, 0.9]], dtype=F16)
    for bits in (3, 4):
        c, s, z = oracle.quantize_rtn(W, bits, 8)
        assert c.min() == 0 and c.max() == (1 << bits) - 1


# ------------------------------------------------------------------ sensitivity (Eq. (10))
def test_sensitivity_is_output_error_of_one_column():
    """sens_j equals || W X^T - W'_j X^T ||_F^2, W'_j = W with only column j quantised.

    The pages define the layer objective as the output difference before/after quantisation
    and derive the per-column score from it; this computes that output error by brute force
    with full matmuls, column by column.
    """
    g = owq_synth.rng(11)
    N, K, T = 7, 12, 9
    W = owq_synth.draw_weight(g, N, K)
    X = owq_synth.draw_activations(g, T, np.linspace(1, 4, K).astype(np.float32))
    c0, s0, z0 = oracle.quantize_rtn(W, 3, K)
    W_hat0 = oracle.dequant(c0, s0, z0)
    sens = oracle.sensitivity(W, W_hat0, oracle.hessian_diag(X))
    W64, X64 = W.astype(F64), X.astype(F64)
    ref = W64 @ X64.T
    for j in range(K):
        Wj = W64.copy()
        Wj[:, j] = W_hat0[:, j].astype(F64)
        e = np.sum((ref - Wj @ X64.T) ** 2)
        assert sens[j] == pytest.approx(e, rel=1e-12, abs=1e-300)


def test_hessian_diag_matches_gram_diagonal():
    g = owq_synth.rng(3)
    X = owq_synth.draw_activations(g, 33, np.ones(20, np.float32))
    X64 = X.astype(F64)
    assert np.array_equal(oracle.hessian_diag(X), np.einsum("tj,tj->j", X64, X64)) or \
        np.allclose(oracle.hessian_diag(X), np.diag(X64.T @ X64), rtol=1e-15)


# ------------------------------------------------------------------ selection
def test_select_weak_exhaustive_subset_search():
    g = owq_synth.rng(5)
    for trial in range(5):
        sens = g.exponential(size=10)
        k = 3
        got = oracle.select_weak(sens, k)
        best = max(itertools.combinations(range(10), k), key=lambda S: sum(sens[list(S)]))
        assert got.tolist() == sorted(best)
        assert got.dtype == np.int32


def test_select_weak_ties_go_to_lower_index():
    sens = np.array([1.0, 3.0, 2.0, 3.0, 2.0, 2.0])
    assert oracle.select_weak(sens, 3).tolist() == [1, 2, 3]
    assert oracle.select_weak(sens, 0).tolist() == []
    assert oracle.select_weak(sens, 6).tolist() == list(range(6))


def test_planted_outlier_channels_are_selected():
    """Workload 0 plants 4 calibration channels x50: those columns must be the weak ones
    (activation outliers make the matching weight columns sensitive, OWQ p.3-4)."""
    spec = owq_synth.WORKLOADS[0]
    L = spec.layers[0]
    d = owq_synth.draw_layer(L, spec, 1, owq_synth.seed_for(0, 0))
    r = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, L.k)
    assert r["idx"].tolist() == sorted(d["outliers"].tolist())


def test_weak_block_is_bit_exact_copy():
    d = owq_synth.draw_small(16, 64, 1, 32, seed=9)
    r = oracle.owq_quantize(d["W"], d["X"], 3, 64, 3)
    assert r["w_weak"].view(np.uint16).tolist() == d["W"][:, r["idx"]].view(np.uint16).tolist()
    assert np.all(r["codes"][:, r["idx"]] == np.repeat(r["zeros"].astype(np.uint8), 64, axis=1)[:, r["idx"]])


# ------------------------------------------------------------------ product
def test_all_columns_weak_is_exact_full_precision_product():
    """k = K: nothing is quantised, so y must be W x exactly (fp64 of fp16 inputs)."""
    d = owq_synth.draw_small(9, 32, 3, 16, seed=21)
    r = oracle.owq_quantize(d["W"], d["X"], 3, 32, 32)
    W_hat = oracle.dequant(r["codes"], r["scales"], r["zeros"])
    assert np.all(W_hat == 0)
    y = oracle.matmul(W_hat, r["w_weak"], r["idx"], d["x"])
    W64, x64 = d["W"].astype(F64), d["x"].astype(F64)
    brute = np.array([[sum(W64[i, j] * x64[m, j] for j in range(32)) for i in range(9)] for m in range(3)])
    assert np.allclose(y, brute, rtol=1e-14, atol=1e-300)


def test_no_weak_columns_is_plain_quantised_product():
    d = owq_synth.draw_small(8, 64, 2, 16, seed=22)
    r = oracle.owq_quantize(d["W"], d["X"], 4, 32, 0)
    c, s, z = oracle.quantize_rtn(d["W"], 4, 32)
    assert np.array_equal(r["codes"], c)
    y = oracle.matmul(oracle.dequant(c, s, z), r["w_weak"], r["idx"], d["x"])
    W_hat64, x64 = oracle.dequant(c, s, z).astype(F64), d["x"].astype(F64)
    brute = np.array([[sum(W_hat64[i, j] * x64[m, j] for j in range(64)) for i in range(8)] for m in range(2)])
    assert np.allclose(y, brute, rtol=1e-14)


@pytest.mark.parametrize("bits,group,k", [(3, 16, 2), (4, 8, 3), (3, 16, 0)])
def test_split_product_equals_patched_matrix_brute_force(bits, group, k):
    """y = (W_hat with the weak columns replaced by W[:, idx]) x, by pure-Python loops."""
    d = owq_synth.draw_small(6, 16, 3, 12, seed=30 + k)
    r = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    W_hat = oracle.dequant(r["codes"], r["scales"], r["zeros"])
    y = oracle.matmul(W_hat, r["w_weak"], r["idx"], d["x"])
    patched = [[float(W_hat[i, j]) for j in range(16)] for i in range(6)]
    for t, j in enumerate(r["idx"].tolist()):
        for i in range(6):
            patched[i][j] = float(d["W"][i, j])
    xs = [[float(v) for v in row] for row in d["x"]]
    for m in range(3):
        for i in range(6):
            acc = 0.0
            for j in range(16):
                acc += patched[i][j] * xs[m][j]
            assert y[m, i] == pytest.approx(acc, rel=1e-13, abs=1e-12)


def test_product_within_rtn_error_bound_of_full_precision():
    d = owq_synth.draw_small(32, 256, 2, 64, seed=40)
    r = oracle.owq_quantize(d["W"], d["X"], 3, 256, 4)
    W_hat = oracle.dequant(r["codes"], r["scales"], r["zeros"])
    y = oracle.matmul(W_hat, r["w_weak"], r["idx"], d["x"])
    exact = d["x"].astype(F64) @ d["W"].astype(F64).T
    dense = np.ones(256, bool)
    dense[r["idx"]] = False
    s = r["scales"].astype(F64)[:, 0]
    bound = (np.abs(d["x"].astype(F64))[:, dense].sum(axis=1)[:, None]) * s[None, :]
    assert np.all(np.abs(y - exact) <= bound)
    # and the bound is not vacuous: the quantised product differs from the exact one
    assert np.abs(y - exact).max() > 0


def test_weak_columns_reduce_output_error_on_planted_outliers():
    """The point of OWQ: keeping the outlier-aligned columns in fp16 lowers the output error
    against the full-precision product compared with keeping no column."""
    spec = owq_synth.WORKLOADS[0]
    L = spec.layers[0]
    d = owq_synth.draw_layer(L, spec, 4, owq_synth.seed_for(0, 0))
    exact = d["x"].astype(F64) @ d["W"].astype(F64).T
    errs = {}
    for k in (0, L.k):
        r = oracle.owq_quantize(d["W"], d["X"], L.bits, L.group, k)
        y = oracle.matmul(oracle.dequant(r["codes"], r["scales"], r["zeros"]), r["w_weak"], r["idx"], d["x"])
        errs[k] = np.linalg.norm(y - exact)
    assert errs[L.k] < 0.5 * errs[0]


# ------------------------------------------------------------------ pack
@pytest.mark.parametrize("bits", [3, 4])
def test_pack_roundtrip_and_size(bits):
    g = owq_synth.rng(50 + bits)
    codes = owq_synth.draw_codes(g, 5, 384, bits)
    words = oracle.pack(codes, bits)
    assert words.shape == (5, 384 * bits // 32)
    assert np.array_equal(oracle.unpack(words, 384, bits), codes)


@pytest.mark.parametrize("bits", [3, 4])
def test_pack_single_code_moves_single_bits(bits):
    """Each code occupies exactly `bits` bits of its block and no two codes share a bit."""
    seen = np.zeros(bits * 128, dtype=int)
    for k in range(128):
        codes = np.zeros((1, 128), np.uint8)
        codes[0, k] = (1 << bits) - 1
        w = oracle.pack(codes, bits)[0]
        bitsset = [wi * 32 + b for wi in range(4 * bits) for b in range(32) if (int(w[wi]) >> b) & 1]
        assert len(bitsset) == bits
        seen[bitsset] += 1
    assert np.all(seen == 1)


def test_pack_blocks_are_independent():
    """A code only moves bits of its own 128-code block (block b at words b * 4 * bits)."""
    codes = np.zeros((1, 384), np.uint8)
    codes[0, 200] = 5
    w = oracle.pack(codes, 3)[0]
    nz = np.nonzero(w)[0]
    assert nz.min() >= 12 and nz.max() < 24


# ------------------------------------------------------------------ storage accounting
def test_bits_per_weight_reproduces_page_numbers():
    # "Storage Methods" (appendix §2 p.11): 3.01 effective bits -> 3.012 with the zero-filled matrix
    k_over_K = 0.01 / 13.0
    K = 13000
    k = k_over_K * K
    assert oracle.bits_per_weight(K, 3, k, "storage") == pytest.approx(3.01)
    assert round(oracle.bits_per_weight(K, 3, k, "latency"), 3) == 3.012
    # "Key points": 3.005 bits costs about 0.21% memory over 3-bit
    k = 0.005 / 13.0 * K
    over = (oracle.bits_per_weight(K, 3, k, "latency") - 3.0) / 3.0
    assert round(100 * over, 2) == 0.21
    # k = K/128 at 3 bits is the pages' "about 3.1 bits" setting
    assert round(oracle.bits_per_weight(4096, 3, 32, "storage"), 1) == 3.1
    b = oracle.layer_bytes(4096, 4096, 3, 4096, 32)
    tot = 8.0 * sum(b.values()) / (4096 * 4096)
    assert tot == pytest.approx(oracle.bits_per_weight(4096, 3, 32, "latency", group=4096, N=4096))


def test_single_output_bound_accepts_unrounded_weights_and_rejects_mistakes():
    """The analytic check used for one-element decode outputs (tests/owq_checks.py) holds for the
    product of the unrounded dequantised weights s (q - z) and fails for a dropped weak term, a
    zero point off by one or a 10% scale error."""
    from tests.owq_checks import check_output_short
    N, K, bits, group, k = 1, 128, 3, 128, 1
    d = owq_synth.draw_small(N, K, 8, 16, seed=4129, n_outliers=1)
    ref = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    W_hat = oracle.dequant(ref["codes"], ref["scales"], ref["zeros"])
    x = d["x"][:1]
    y64 = oracle.matmul(W_hat, ref["w_weak"], ref["idx"], x)
    s = ref["scales"].astype(np.float64)[:, :1]
    z = ref["zeros"].astype(np.float64)[:, :1]
    xw = x[:, ref["idx"]].astype(np.float64) @ ref["w_weak"].astype(np.float64).T

    def product(scale, zero, weak):
        w = scale * (ref["codes"].astype(np.float64) - zero)
        w[:, ref["idx"]] = 0.0
        return (x.astype(np.float64) @ w.T + weak).astype(np.float16)

    check_output_short(product(s, z, xw), W_hat, ref["w_weak"], ref["idx"], x, y64, "unrounded")
    # (at this near-cancelled output the bound is ~5% of |y|: a 10% scale error must fail)
    for bad in (product(s, z, 0.0 * xw), product(s, z + 1, xw), product(s * 1.1, z, xw)):
        with pytest.raises(AssertionError):
            check_output_short(bad, W_hat, ref["w_weak"], ref["idx"], x, y64, "planted")


# ------------------------------------------------------------------ weak column tuning gradients
def _wct_case(bits, group, k, M, seed):
    d = owq_synth.draw_small(12, 256, M, 32, seed=seed)
    r = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    W_hat = oracle.dequant(r["codes"], r["scales"], r["zeros"])
    rng = np.random.default_rng(seed + 1)
    dy = rng.standard_normal((M, 12)).astype(F16)
    return d, r, W_hat, dy


@pytest.mark.parametrize("bits,group,k,M", [(3, 256, 5, 3), (4, 128, 9, 1), (3, 128, 0, 2)])
def test_input_grad_is_adjoint_of_forward_product(bits, group, k, M):
    """<dy, y(x)> = <dX(dy), x> for every x: the forward product (pinned above) is linear in
    x, so its adjoint is fixed by it; checked on several random x."""
    d, r, W_hat, dy = _wct_case(bits, group, k, M, seed=70 + k)
    dx = oracle.input_grad(W_hat, r["w_weak"], r["idx"], dy)
    rng = np.random.default_rng(5)
    for _ in range(3):
        x = rng.standard_normal((M, 256)).astype(F16)
        y = oracle.matmul(W_hat, r["w_weak"], r["idx"], x)
        lhs = float((dy.astype(F64) * y).sum())
        rhs = float((dx * x.astype(F64)).sum())
        assert rhs == pytest.approx(lhs, rel=1e-12, abs=1e-12)
    # one-hot x reads single entries: dX[m, j] = <dy[m], y(e_j)[m]>
    for j in [0, 17, 255] + [int(v) for v in r["idx"][:2]]:
        x = np.zeros((M, 256), dtype=F16)
        x[:, j] = 1
        y = oracle.matmul(W_hat, r["w_weak"], r["idx"], x)
        for m in range(M):
            assert dx[m, j] == pytest.approx(float((dy[m].astype(F64) * y[m]).sum()), rel=1e-12, abs=1e-14)


@pytest.mark.parametrize("k,M", [(5, 3), (1, 7)])
def test_weak_grad_is_directional_derivative_of_forward_product(k, M):
    """The loss <dy, y> is linear in the weak block, so for any direction V the derivative
    <dW_weak, V> equals <dy, y(W_hat = 0, W_weak = V)> exactly (the forward product pinned
    above, with the dense part switched off)."""
    d, r, W_hat, dy = _wct_case(3, 256, k, M, seed=90 + k)
    g = oracle.weak_grad(d["x"], dy, r["idx"])
    assert g.shape == (12, k)
    rng = np.random.default_rng(9)
    zero = np.zeros_like(W_hat)
    for _ in range(3):
        V = rng.standard_normal((12, k)).astype(F16)
        y = oracle.matmul(zero, V, r["idx"], d["x"])
        assert float((g * V.astype(F64)).sum()) == pytest.approx(float((dy.astype(F64) * y).sum()), rel=1e-12)
    # a unit direction isolates one entry
    for i, t in [(0, 0), (11, k - 1), (5, k // 2)]:
        V = np.zeros((12, k), dtype=F16)
        V[i, t] = 1
        y = oracle.matmul(zero, V, r["idx"], d["x"])
        assert g[i, t] == pytest.approx(float((dy.astype(F64) * y).sum()), rel=1e-12, abs=1e-14)


# ------------------------------------------------------------------ OPTQ and the parameter search
def _rtn_error(w, s, z, bits):
    """Squared reconstruction error of one group's weights under RTN with the given (s, z)
    (test-side evaluation of a candidate; the oracle's RTN is pinned above)."""
    s32, z32 = np.float32(s), np.float32(z)
    q = np.clip(np.rint(w.astype(np.float32) / s32) + z32, 0, (1 << bits) - 1)
    w_hat = (s32 * (q - z32)).astype(F16).astype(F64)
    return float(((w.astype(F64) - w_hat) ** 2).sum())


def test_optq_with_diagonal_hessian_is_rtn():
    """With X^T X diagonal, H^-1 has no off-diagonal terms, so no column compensates another:
    OPTQ gives exactly the RTN codes of the same parameters and keeps the weak columns."""
    d = owq_synth.draw_small(6, 32, 1, 8, seed=120)
    c = np.linspace(0.5, 3.0, 32).astype(F16)
    X = np.diag(c).astype(F16)
    weak = [3, 17, 30]
    codes, s, z = oracle.quantize_rtn(d["W"], 3, 32, weak)
    r = oracle.optq_quantize(d["W"], X, 3, 32, weak, s, z, damp=0.0)
    assert np.array_equal(r["codes"], codes)
    assert np.array_equal(r["w_weak"].view(np.uint16), d["W"][:, weak].view(np.uint16))


@pytest.mark.parametrize("bits,group", [(3, 32), (4, 16)])
def test_optq_weak_columns_are_least_squares_optimum(bits, group):
    """The compensated weak columns minimise the row's output error ||X (w - w_hat)||^2 given the
    quantised dense columns: checked against numpy's least-squares solve on X itself."""
    rng = np.random.default_rng(130 + bits)
    N, K, T = 5, 32, 96
    W = (rng.standard_normal((N, K)) * 0.02).astype(F16)
    X = rng.standard_normal((T, K)).astype(F16)
    weak = [2, 9, 25]
    s, z = oracle.search_params(W, bits, group, weak)
    r = oracle.optq_quantize(W, X, bits, group, weak, s, z, damp=0.0)
    W_hat = oracle.dequant(r["codes"], s, z).astype(F64)
    dense = np.setdiff1d(np.arange(K), weak)
    X64 = X.astype(F64)
    for i in range(N):
        target = X64 @ W[i].astype(F64) - X64[:, dense] @ W_hat[i, dense]
        v, *_ = np.linalg.lstsq(X64[:, weak], target, rcond=None)
        assert np.allclose(r["w_weak64"][i], v, rtol=1e-9, atol=1e-12)
    # and the compensation is real: the optimum differs from the original weak values
    assert not np.allclose(r["w_weak64"], W[:, weak].astype(F64), atol=1e-6)


def test_search_params_never_worse_than_minmax_and_exact_on_grid_rows():
    d = owq_synth.draw_small(8, 64, 1, 8, seed=140)
    weak = [5]
    s, z = oracle.search_params(d["W"], 3, 32, weak)
    _, s0, z0 = oracle.quantize_rtn(d["W"], 3, 32, weak)
    dense = np.ones(64, bool)
    dense[weak] = False
    for i in range(8):
        for g in range(2):
            cols = np.arange(32 * g, 32 * g + 32)
            w = d["W"][i, cols[dense[cols]]]
            assert _rtn_error(w, s[i, g], z[i, g], 3) <= _rtn_error(w, s0[i, g], z0[i, g], 3)
    # a row that lies exactly on a 3-bit grid (codes 0..7, step 1/16, zero point 3) is
    # reproduced with zero error by its own min-max parameters, which the search keeps
    q = np.array([0, 7, 3, 1, 5, 2, 6, 4] * 4, dtype=np.float32)
    row = ((q - 3) / 16).astype(F16)[None, :]
    s1, z1 = oracle.search_params(row, 3, 32)
    assert float(s1[0, 0]) == 1 / 16 and float(z1[0, 0]) == 3
    assert _rtn_error(row[0], s1[0, 0], z1[0, 0], 3) == 0.0


def test_search_params_truncates_a_planted_outlier():
    """One large weight among small ones: clamping it lowers the total squared error, so the
    search picks a step below the min-max step."""
    rng = np.random.default_rng(150)
    row = (rng.standard_normal(128) * 0.01).astype(F16)
    row[77] = F16(0.5)
    s, z = oracle.search_params(row[None, :], 3, 128)
    _, s0, _ = oracle.quantize_rtn(row[None, :], 3, 128)
    assert float(s[0, 0]) < float(s0[0, 0])
    assert _rtn_error(row, s[0, 0], z[0, 0], 3) < _rtn_error(row, s0[0, 0], oracle.quantize_rtn(row[None, :], 3, 128)[2][0, 0], 3)


# ------------------------------------------------------------------ storage-favoured layout
@pytest.mark.parametrize("bits,group,k", [(3, 128, 5), (4, 256, 0), (3, 256, 11)])
def test_storage_layout_round_trip_matches_latency_layout(bits, group, k):
    """Both layouts hold the same quantised matrix: the storage-favoured stream, unpacked,
    gives exactly the zero-filled codes the latency-favoured blocks hold."""
    d = owq_synth.draw_small(7, 256, 1, 32, seed=160 + k)
    r = oracle.owq_quantize(d["W"], d["X"], bits, group, k)
    words = oracle.pack_storage(r["codes"], r["idx"], bits)
    assert words.shape == (7, ((256 - k) * bits + 31) // 32)
    back = oracle.unpack_storage(words, 256, r["idx"], bits, r["zeros"], group)
    lat = oracle.unpack(oracle.pack(r["codes"], bits), 256, bits)
    assert np.array_equal(back, lat)
    assert np.array_equal(back, r["codes"])


def test_storage_layout_single_code_moves_its_own_bits():
    """A code of all ones at dense position p sets exactly bits [3p, 3p + 3) of the row's
    stream, positions counted after the weak columns are removed (p = 10 starts at bit 30
    and straddles words 0 and 1)."""
    for p in (0, 5, 10, 11, 40):
        codes = np.zeros((1, 128), dtype=np.uint8)
        idx = [3, 64]
        dense_cols = [j for j in range(128) if j not in idx]
        codes[0, dense_cols[p]] = 7
        words = oracle.pack_storage(codes, idx, 3)
        bits = int(sum(int(w) << (32 * i) for i, w in enumerate(words[0])))
        assert bits == 7 << (3 * p)


def test_storage_layout_bytes_reproduce_storage_bits_per_weight():
    """With (K - k) b a multiple of 32 there is no padding, and the layout's bits per weight
    (stream + fp16 weak block) equal the pages' storage-favoured b + (16 - b) k / K."""
    N, K, k, b = 4, 512, 32, 4
    codes = np.zeros((N, K), dtype=np.uint8)
    words = oracle.pack_storage(codes, np.arange(0, K, K // k)[:k], b)
    bits = (words.size * 32 + N * k * 16) / (N * K)
    assert bits == pytest.approx(oracle.bits_per_weight(K, b, k, layout="storage"), abs=1e-12)
    assert bits < oracle.bits_per_weight(K, b, k, layout="latency")


def test_owq_quantize_optq_end_to_end():
    """The full quantiser selects the planted outlier channels, and its stored weak columns
    (before fp16 rounding) are the least-squares optimum given its quantised dense columns."""
    rng = np.random.default_rng(170)
    N, K, T = 6, 64, 160
    W = (rng.standard_normal((N, K)) * 0.02).astype(F16)
    X = rng.standard_normal((T, K)).astype(np.float32)
    planted = [7, 40]
    X[:, planted] *= 50
    X = X.astype(F16)
    r = oracle.owq_quantize_optq(W, X, 3, K, 2, damp=0.0)
    assert r["idx"].tolist() == planted
    W_hat = oracle.dequant(r["codes"], r["scales"], r["zeros"]).astype(F64)
    dense = np.setdiff1d(np.arange(K), planted)
    X64 = X.astype(F64)
    for i in range(N):
        target = X64 @ W[i].astype(F64) - X64[:, dense] @ W_hat[i, dense]
        v, *_ = np.linalg.lstsq(X64[:, planted], target, rcond=None)
        assert np.allclose(r["w_weak64"][i], v, rtol=1e-8, atol=1e-12)
    # the output error of the full quantiser is below that of the RTN oracle quantiser
    base = oracle.owq_quantize(W, X, 3, K, 2)
    y_ref = X64 @ W.astype(F64).T
    e_optq = np.linalg.norm(oracle.matmul(W_hat.astype(F16), r["w_weak"], r["idx"], X) - y_ref)
    W_hat_b = oracle.dequant(base["codes"], base["scales"], base["zeros"])
    e_rtn = np.linalg.norm(oracle.matmul(W_hat_b, base["w_weak"], base["idx"], X) - y_ref)
    assert e_optq < e_rtn
