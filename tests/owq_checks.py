"""Shared helpers of the GPU parity tests: the output tolerance and oracle caches."""
import numpy as np

F64 = np.float64

REL_L2 = 1e-3
MAX_ABS = 1e-2


def check_output(y_gpu_fp16: np.ndarray, y64: np.ndarray, where: str = "") -> dict:
    """fp16 outputs against the oracle's unrounded fp64 outputs.

    rel-L2 <= 1e-3 over all outputs, and per output |err| <= 1e-2.  Where |y| >= 32 the fp16
    grid alone can be 0.0156 away from y (half a spacing), so there the per-output bound is
    half an fp16 spacing plus 2^-13 |y| of accumulation slack; the number of such outputs is
    reported.
    """
    yg = np.asarray(y_gpu_fp16, dtype=np.float16).astype(F64)
    y64 = np.asarray(y64, dtype=F64)
    assert yg.shape == y64.shape, (yg.shape, y64.shape)
    assert np.all(np.isfinite(yg)), where
    err = np.abs(yg - y64)
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(y64), 1e-300))
    big = np.abs(y64) >= 32.0
    half_ulp = 0.5 * np.spacing(np.abs(y64).astype(np.float16)).astype(F64)
    allowed = np.where(big, half_ulp + np.abs(y64) * 2.0 ** -13, MAX_ABS)
    worst = float(err.max()) if err.size else 0.0
    bad = err > allowed
    assert rel <= REL_L2, f"{where}: rel-L2 {rel:.3e} > {REL_L2}"
    assert not bad.any(), f"{where}: {int(bad.sum())} outputs over the bound, worst {worst:.4g}"
    return {"rel_l2": rel, "max_abs": worst, "n_relaxed": int(big.sum())}


def check_output_short(y_gpu_fp16: np.ndarray, W_hat: np.ndarray, w_weak: np.ndarray, idx: np.ndarray,
                       x: np.ndarray, y64: np.ndarray, where: str = "") -> None:
    """A product with a single output element, where the rel-L2 criterion becomes the relative
    error of one possibly near-cancelled dot product.

    The 1-8 token decode product applies each segment's scale and zero point to its integer
    sums, i.e. it multiplies the unrounded dequantised weights s (q - z); the oracle multiplies
    W_hat = fp16_rn(s (q - z)).  Each weight then differs by at most half an fp16 spacing,
    2^-11 of its magnitude (2^-25 absolute below the normal range), so per output
    |y - y64| <= 2^-11 sum_j |W_hat_ij x_j| + 2^-25 sum_j |x_j| + half an fp16 spacing of y64
    + 2^-20 (|W_hat| |x| + |W_weak| |x_w|) (fp32 accumulation).  The max-abs bound of
    check_output holds as well.
    """
    yg = np.asarray(y_gpu_fp16, dtype=np.float16).astype(F64)
    y64 = np.asarray(y64, dtype=F64)
    ax = np.abs(np.asarray(x, dtype=F64))
    terms = ax @ np.abs(W_hat.astype(F64)).T
    weak = ax[:, idx] @ np.abs(w_weak.astype(F64)).T if len(idx) else np.zeros_like(y64)
    bound = (2.0 ** -11 * terms + 2.0 ** -25 * ax.sum(axis=1, keepdims=True)
             + 0.5 * np.spacing(np.abs(y64).astype(np.float16)).astype(F64) + 2.0 ** -20 * (terms + weak))
    err = np.abs(yg - y64)
    assert np.all(err <= MAX_ABS), f"{where}: max-abs {float(err.max()):.4g}"
    assert np.all(err <= bound), f"{where}: error {float(err.max()):.4g} over the bound {float(bound.min()):.4g}"

