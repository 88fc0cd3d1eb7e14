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
