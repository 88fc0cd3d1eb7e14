"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one.

Every mutant replaces one oracle function for the duration of a test; the pins of
test_oracle_pins.py must then fail.
"""
import numpy as np
import pytest

import oracle
import oracle.owq_oracle as oo
import tests.test_oracle_pins as pins

F16, F32, F64 = np.float16, np.float32, np.float64


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(oo, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def test_mutant_select_ascending_is_caught(monkeypatch):
    def bad(sens, k):
        return np.sort(np.argsort(np.asarray(sens), kind="stable")[:k]).astype(np.int32)
    _patch(monkeypatch, "select_weak", bad)
    with pytest.raises(AssertionError):
        pins.test_planted_outlier_channels_are_selected()


def test_mutant_sensitivity_without_hessian_is_caught(monkeypatch):
    orig = oo.sensitivity

    def bad(W, W_hat0, lam):
        return orig(W, W_hat0, np.ones_like(np.asarray(lam)))
    _patch(monkeypatch, "sensitivity", bad)
    with pytest.raises(AssertionError):
        pins.test_sensitivity_is_output_error_of_one_column()


def test_mutant_sensitivity_on_weights_not_perturbation_is_caught(monkeypatch):
    def bad(W, W_hat0, lam):
        d = np.asarray(W, dtype=F16).astype(F64)
        return np.asarray(lam) * (d * d).sum(axis=0)
    _patch(monkeypatch, "sensitivity", bad)
    with pytest.raises(AssertionError):
        pins.test_sensitivity_is_output_error_of_one_column()


def test_mutant_round_half_up_is_caught(monkeypatch, golden_dir):
    orig_rint = np.rint

    def half_up(v):
        return np.floor(np.asarray(v) + F32(0.5)).astype(np.asarray(v).dtype)
    monkeypatch.setattr(oo.np, "rint", half_up)
    try:
        with pytest.raises(AssertionError):
            pins.test_rtn_hand_worked_rows(golden_dir)
    finally:
        monkeypatch.setattr(oo.np, "rint", orig_rint)


def test_mutant_weak_code_zero_is_caught(monkeypatch):
    orig = oo.quantize_rtn

    def bad(W, bits, group, weak_idx=None):
        c, s, z = orig(W, bits, group, weak_idx)
        if weak_idx is not None and len(weak_idx):
            c = c.copy()
            c[:, np.asarray(weak_idx)] = 0
        return c, s, z
    _patch(monkeypatch, "quantize_rtn", bad)
    with pytest.raises(AssertionError):
        pins.test_rtn_invariants_and_error_bound(3, 64)


def test_mutant_dropped_weak_term_is_caught(monkeypatch):
    def bad(W_hat, w_weak, idx, x):
        return np.ascontiguousarray((np.asarray(W_hat, F16).astype(F64) @ np.asarray(x, F16).astype(F64).T).T)
    _patch(monkeypatch, "matmul", bad)
    with pytest.raises(AssertionError):
        pins.test_all_columns_weak_is_exact_full_precision_product()


def test_mutant_transposed_weak_block_is_caught(monkeypatch):
    orig = oo.matmul

    def bad(W_hat, w_weak, idx, x):
        ww = np.asarray(w_weak)
        return orig(W_hat, ww[::-1] if ww.shape[0] > 1 else ww, idx, x)
    _patch(monkeypatch, "matmul", bad)
    with pytest.raises(AssertionError):
        pins.test_split_product_equals_patched_matrix_brute_force(3, 16, 2)


def test_mutant_swapped_pair_halves_is_caught(monkeypatch, golden_dir):
    orig = oo.pack

    def bad(codes, bits):
        c = np.asarray(codes).copy()
        c[:, 0::2], c[:, 1::2] = np.asarray(codes)[:, 1::2], np.asarray(codes)[:, 0::2]
        return orig(c, bits)
    _patch(monkeypatch, "pack", bad)
    with pytest.raises(AssertionError):
        pins.test_pack_hand_derived_words(golden_dir)


def test_mutant_swapped_slots_is_caught(monkeypatch, golden_dir):
    slots = list(oo.SLOT3)
    slots[13], slots[15] = slots[15], slots[13]
    monkeypatch.setattr(oo, "SLOT3", slots)
    with pytest.raises(AssertionError):
        pins.test_pack_hand_derived_words(golden_dir)


def test_mutant_chunk_of_consecutive_pairs_is_caught(monkeypatch, golden_dir):
    orig = oo.pack

    def bad(codes, bits):
        c = np.asarray(codes)
        N, K = c.shape
        # chunk q taking pairs 16q..16q+15 instead of 4j + q
        perm = np.arange(K).reshape(K // 128, 16, 4, 2).transpose(0, 2, 1, 3).reshape(K)
        return orig(c[:, perm], bits)
    _patch(monkeypatch, "pack", bad)
    with pytest.raises(AssertionError):
        pins.test_pack_hand_derived_words(golden_dir)


def test_mutant_latency_bits_without_zero_fill_is_caught(monkeypatch):
    orig = oo.bits_per_weight

    def bad(K, bits, k, layout="latency", group=None, N=None):
        return orig(K, bits, k, "storage" if layout == "latency" else layout, group, N)
    _patch(monkeypatch, "bits_per_weight", bad)
    with pytest.raises(AssertionError):
        pins.test_bits_per_weight_reproduces_page_numbers()


def test_mutant_input_grad_without_weak_term_is_caught(monkeypatch):
    def bad(W_hat, w_weak, idx, dy):
        return np.asarray(dy, dtype=F16).astype(F64) @ np.asarray(W_hat, dtype=F16).astype(F64)
    _patch(monkeypatch, "input_grad", bad)
    with pytest.raises(AssertionError):
        pins.test_input_grad_is_adjoint_of_forward_product(3, 256, 5, 3)


def test_mutant_input_grad_weak_term_at_wrong_columns_is_caught(monkeypatch):
    orig = oo.input_grad

    def bad(W_hat, w_weak, idx, dy):
        return orig(W_hat, w_weak, np.minimum(np.asarray(idx) + 1, np.asarray(W_hat).shape[1] - 1), dy)
    _patch(monkeypatch, "input_grad", bad)
    with pytest.raises(AssertionError):
        pins.test_input_grad_is_adjoint_of_forward_product(4, 128, 9, 1)


def test_mutant_weak_grad_wrong_gather_is_caught(monkeypatch):
    def bad(x, dy, idx):
        k = len(idx)
        return np.asarray(dy, dtype=F16).astype(F64).T @ np.asarray(x, dtype=F16).astype(F64)[:, :k]
    _patch(monkeypatch, "weak_grad", bad)
    with pytest.raises(AssertionError):
        pins.test_weak_grad_is_directional_derivative_of_forward_product(5, 3)


def test_mutant_optq_without_compensation_is_caught(monkeypatch):
    orig = oo.optq_quantize

    def bad(W, X, bits, group, weak_idx, scales, zeros, damp=0.01):
        # an identity Hessian: every column is quantised on its own, nothing is compensated
        K = np.asarray(W).shape[1]
        return orig(W, np.eye(K, dtype=F16), bits, group, weak_idx, scales, zeros, damp=0.0)
    _patch(monkeypatch, "optq_quantize", bad)
    with pytest.raises(AssertionError):
        pins.test_optq_weak_columns_are_least_squares_optimum(3, 32)


def test_mutant_optq_weak_columns_first_is_caught(monkeypatch):
    orig = oo.optq_quantize

    def bad(W, X, bits, group, weak_idx, scales, zeros, damp=0.01):
        # weak columns taken out of the compensation (their values never move)
        r = orig(W, X, bits, group, weak_idx, scales, zeros, damp)
        r["w_weak64"] = np.asarray(W, dtype=F16)[:, np.sort(weak_idx)].astype(F64)
        return r
    _patch(monkeypatch, "optq_quantize", bad)
    with pytest.raises(AssertionError):
        pins.test_optq_weak_columns_are_least_squares_optimum(4, 16)


def test_mutant_search_without_truncation_is_caught(monkeypatch):
    orig = oo.search_params

    def bad(W, bits, group, weak_idx=None, alphas=None):
        return orig(W, bits, group, weak_idx, alphas=(1.0,))
    _patch(monkeypatch, "search_params", bad)
    with pytest.raises(AssertionError):
        pins.test_search_params_truncates_a_planted_outlier()


def test_mutant_storage_stream_keeping_weak_columns_is_caught(monkeypatch):
    orig = oo.pack_storage

    def bad(codes, idx, bits):
        return orig(codes, [], bits)
    _patch(monkeypatch, "pack_storage", bad)
    with pytest.raises(AssertionError):
        pins.test_storage_layout_round_trip_matches_latency_layout(3, 128, 5)
