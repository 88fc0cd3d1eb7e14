"""OWQ oracle: a plain, slow, obviously-correct CPU implementation of the mixed-precision
weight-only matmul and of the quantiser that produces its operands.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The CUDA library never calls it, and it shares
no code with the CUDA library: it imports numpy and nothing else of this repository.

Sources (five web pages about the OWQ paper, Lee et al., arXiv:2306.02272):
  [SUM]  "OWQ -- paper by Lee et al. (2023) -- summary and ideas" (research.elamur.ai):
         sections "Key points" and "Interesting ideas".
  [PL]   "OWQ: Outlier-Aware Weight Quantization for Efficient Fine-Tuning and Inference of
         Large Language Models" (paperlayer.ai), whose items name the paper's sections:
         "Problem Definition and Motivation" (p.3), "Layer-wise Quantization and Hessian"
         (p.3), "OWQ: Outlier-aware Weight Quantization" (p.4), "Acceleration on Real
         Device" (p.6), appendix "§1" (p.10, Eq. (10)) and "§2 Storage Methods" (pp.10-11).

Every floating-point reduction is fp64 in a fixed order (index ascending). Every decision
that turns a float into an integer (a quantised code, the zero point, the top-k order) is
taken in the precision stated at that step, with IEEE round-to-nearest-even.

Readings of the pages where they are silent (each is listed with its reason in the design
notes): the sensitivity uses the perturbation of an all-column RTN pre-quantisation; the
quantisation range always contains 0; a degenerate range becomes [-1, 1]; rounding is
half-to-even; the dequantised weight is fp16_rn(s * (q - z)); weak positions carry the code
q = z (so they dequantise to exactly 0); groups are contiguous blocks of the original column
order; top-k ties go to the lower column index and the index list is stored ascending.

Parity status of each function (what pins it, in tests/test_oracle_pins.py):
  hessian_diag, sensitivity   pinned: brute-force output error of a one-column perturbation.
  select_weak                 pinned: exhaustive subset search; planted outlier channel.
  quantize_rtn                pinned: hand-worked rows (tests/golden/rtn_rows.txt), RTN error
                              bound, range/zero-point invariants.  The exact choice of
                              scale/zero among valid min-max RTN variants is a reading, not a
                              page value (the pages print no quantised example).
  pack / unpack               pinned: hand-derived packed words (tests/golden/pack_words.txt).
  dequant                     pinned: exact small-integer cases and the RTN error bound.
  matmul                      pinned: k = K reproduces W x exactly; k = 0 is the plain quantised
                              product; the RTN error bound; brute force on tiny shapes.
  bits_per_weight             pinned: the pages' 3.01 -> 3.012 and 0.21% figures.
  weak_grad                   pinned: directional derivative of the pinned forward product
                              (the loss is linear in the weak block).
  input_grad                  pinned: adjoint identity against the pinned forward product.
  pack_storage /
  unpack_storage              pinned: the round trip gives the latency layout's codes (z at
                              the weak columns); each code moves exactly its own bits; the
                              layout's bytes reproduce the storage-favoured bits per weight.
  search_params               pinned: never worse than min-max RTN (whose parameters are a
                              grid point); exact rows reproduced with zero error; a planted
                              outlier is truncated.  The grid itself is a reading.
  owq_quantize_optq           composition of pinned steps; pinned end to end: the planted
                              outlier channels are selected and its weak columns are the
                              least-squares optimum.
  optq_quantize               pinned: a diagonal Hessian reduces it to RTN; the compensated
                              weak columns equal the least-squares optimum given the
                              quantised dense columns (a different route: lstsq on X).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "hessian_diag",
    "quantize_rtn",
    "dequant",
    "sensitivity",
    "select_weak",
    "owq_quantize",
    "pack",
    "unpack",
    "matmul",
    "matmul_rows",
    "weak_grad",
    "input_grad",
    "pack_storage",
    "unpack_storage",
    "search_params",
    "optq_quantize",
    "owq_quantize_optq",
    "bits_per_weight",
    "layer_bytes",
]

F16 = np.float16
F32 = np.float32
F64 = np.float64


# ----------------------------------------------------------------------------------------
# Calibration statistics and sensitivity
# ----------------------------------------------------------------------------------------
def hessian_diag(X: np.ndarray) -> np.ndarray:
    """lambda_j = sum_t X[t, j]^2, the diagonal of X^T X (fp64, t ascending).

    [PL] "Error Analysis" / appendix §1 Eq. (10): the per-output-channel error is
    dW_i H dW_i^T with H built from the calibration inputs; [PL] "Error Decomposition":
    one C_in x C_in Hessian is shared by all output rows. OPTQ's H = 2 X^T X differs from
    X^T X by a constant factor, which does not change any ranking, so the oracle keeps
    X^T X.  Only the diagonal enters the weak-column score ([PL] "Weak-column selection").
    """
    X64 = np.asarray(X, dtype=F16).astype(F64)
    lam = np.zeros(X64.shape[1], dtype=F64)
    for t in range(X64.shape[0]):
        lam += X64[t] * X64[t]
    return lam


def sensitivity(W: np.ndarray, W_hat0: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """sens_j = lambda_j * sum_i (W_ij - W_hat0_ij)^2 (fp64, i ascending).

    [PL] "Weak-column selection" (paper p.4): the score of a column combines its
    perturbation norm with the matching Hessian diagonal element; with a diagonal H the
    second-order error of appendix Eq. (10) summed over rows is exactly this product.
    [SUM] "Interesting ideas": the metric multiplies Hessian sensitivity by the weight
    perturbation.
    """
    d = np.asarray(W, dtype=F16).astype(F64) - np.asarray(W_hat0, dtype=F16).astype(F64)
    col = np.zeros(d.shape[1], dtype=F64)
    for i in range(d.shape[0]):
        col += d[i] * d[i]
    return np.asarray(lam, dtype=F64) * col


def select_weak(sens: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k most sensitive columns, returned in ascending order (int32).

    [PL] "Weak-column selection": OWQ keeps the top-k columns by sensitivity in fp16 and
    excludes them from quantisation. Order: sensitivity descending, ties to the lower
    column index; the stored list is ascending.
    """
    sens = np.asarray(sens, dtype=F64)
    K = sens.size
    if not 0 <= k <= K:
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(K), -sens))      # primary: -sens ascending; then index
    return np.sort(order[:k]).astype(np.int32)


# ----------------------------------------------------------------------------------------
# Min-max round-to-nearest quantiser
# ----------------------------------------------------------------------------------------
def quantize_rtn(W: np.ndarray, bits: int, group: int, weak_idx=None):
    """Asymmetric min-max RTN, per output row and per group of `group` contiguous columns.

    Returns (codes uint8 N x K, scales fp16 N x G, zeros fp16 N x G), G = K / group.
    [SUM] "Key points" names min-max RTN as the simple quantiser OWQ is compared with;
    [PL] "Weak-column selection": weak columns are excluded from quantisation, so they are
    left out of their group's min/max and get the code q = z ([PL] "Storage Methods": the
    latency-favoured matrix is zero-filled at the weak columns).

    For each (row, group), over the group's dense (non-weak) columns, in fp32:
        mn = min(0, min w), mx = max(0, max w)
        if mn == mx: mn, mx = -1, 1
        s  = fp16_rn((mx - mn) / (2^b - 1))         (fp32 subtract and divide, then fp16)
        if s == 0:  mn, mx = -1, 1 and s recomputed (a range below fp16 resolution)
        z  = clamp(rint(-mn / s), 0, 2^b - 1)       (an exactly-integral fp16, +0 for zero)
        q  = clamp(rint(w / s) + z, 0, 2^b - 1)     (rint = round half to even)
    """
    W = np.asarray(W, dtype=F16)
    N, K = W.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    G = K // group
    qmax = (1 << bits) - 1
    dense = np.ones(K, dtype=bool)
    if weak_idx is not None and len(weak_idx):
        dense[np.asarray(weak_idx, dtype=np.int64)] = False

    W32 = W.astype(F32).reshape(N, G, group)
    # 0 is always inside the range, so a weak column replaced by 0 leaves min/max unchanged.
    Wm = np.where(dense.reshape(1, G, group), W32, F32(0))
    mn = np.minimum(Wm.min(axis=2), F32(0))
    mx = np.maximum(Wm.max(axis=2), F32(0))
    deg = mn == mx
    mn = np.where(deg, F32(-1), mn).astype(F32)
    mx = np.where(deg, F32(1), mx).astype(F32)
    s16 = ((mx - mn) / F32(qmax)).astype(F16)
    tiny = s16 == 0
    if tiny.any():
        mn = np.where(tiny, F32(-1), mn).astype(F32)
        mx = np.where(tiny, F32(1), mx).astype(F32)
        s16 = ((mx - mn) / F32(qmax)).astype(F16)
    s32 = s16.astype(F32)
    # the zero point is an integer: "+ 0" maps a -0.0 (from mn == 0) to the canonical +0
    z32 = (np.clip(np.rint(-mn / s32), F32(0), F32(qmax)) + F32(0)).astype(F32)
    q32 = np.clip(np.rint(W32 / s32[:, :, None]) + z32[:, :, None], F32(0), F32(qmax))
    q32 = np.where(dense.reshape(1, G, group), q32, z32[:, :, None])
    codes = q32.reshape(N, K).astype(np.uint8)
    return codes, s16, z32.astype(F16)


def dequant(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray) -> np.ndarray:
    """W_hat = fp16_rn(s * (q - z)) with the (row, group) scale and zero of each entry.

    q - z is an exact small integer and s * (q - z) is exact in fp32 (an 11-bit times a
    5-bit significand), so the only rounding is the final one to fp16.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    G = np.asarray(scales).shape[1]
    group = K // G
    s = np.repeat(np.asarray(scales, dtype=F16).astype(F32), group, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=F16).astype(F32), group, axis=1)
    return (s * (codes.astype(F32) - z)).astype(F16)


def owq_quantize(W: np.ndarray, X: np.ndarray, bits: int, group: int, k: int) -> dict:
    """The OWQ quantiser used by the oracle: selection, then RTN of the dense part.

    1. lambda = diag(X^T X)                                   (hessian_diag)
    2. W_hat0 = RTN of W over all columns                      (quantize_rtn, no exclusion)
    3. sens_j = lambda_j * ||W[:, j] - W_hat0[:, j]||^2        (sensitivity)
    4. idx = top-k of sens, ascending                          (select_weak)
    5. codes/scales/zeros = RTN with idx excluded, q = z there (quantize_rtn)
    6. W_weak = W[:, idx], bit-exact fp16                      ([PL] "Storage Methods")
    The selection precedes the exclusion, so the score has to come from a quantisation
    that still includes every column; [PL] "Weak-column selection" then "Low-precision
    quantization" give that order.
    """
    W = np.asarray(W, dtype=F16)
    lam = hessian_diag(X)
    c0, s0, z0 = quantize_rtn(W, bits, group, None)
    sens = sensitivity(W, dequant(c0, s0, z0), lam)
    idx = select_weak(sens, k)
    codes, scales, zeros = quantize_rtn(W, bits, group, idx)
    w_weak = np.ascontiguousarray(W[:, idx])
    return {"codes": codes, "scales": scales, "zeros": zeros, "idx": idx, "w_weak": w_weak,
            "lam": lam, "sens": sens}


# ----------------------------------------------------------------------------------------
# Packed layout (latency-favoured, zero-filled; the format of this library)
# ----------------------------------------------------------------------------------------
# A row of K codes is cut into blocks of 128 consecutive codes; block b of row i is
# 4 * bits little-endian 32-bit words at word offset (i * K/128 + b) * 4 * bits.  Codes 2p and
# 2p+1 of a block form pair p (p = 0..63).  The block is four chunks of `bits` words; chunk q
# (words q*bits .. q*bits + bits - 1) holds the sixteen pairs p = 4j + q, j = 0..15.  Pair j
# of a chunk sits at a slot (word w, bit offset o): the even code in bits o.., the odd code in
# bits 16 + o.. of word w.
#   bits = 4: w = 2 (j // 8) + (j % 2), o = 4 ((j % 8) // 2).
#   bits = 3: slots of j = 0..15: (0,0) (1,0) (0,3) (1,3) (0,6) (1,6) (0,9) (1,9) (0,12) (1,12)
#             (2,6) D (2,3) (2,12) (2,0) (2,9); slot D (j = 11) spreads its codes over the
#             chunk: bit e of the even code is bit 15 of word e, bit e of the odd code is bit 31
#             of word e (e = 0, 1, 2).
SLOT3 = [(0, 0), (1, 0), (0, 3), (1, 3), (0, 6), (1, 6), (0, 9), (1, 9), (0, 12), (1, 12),
         (2, 6), None, (2, 3), (2, 12), (2, 0), (2, 9)]
SLOT4 = [(2 * (j // 8) + (j % 2), 4 * ((j % 8) // 2)) for j in range(16)]


def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack N x K codes into N x (K * bits / 32) uint32 words (format above)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    if K % 128:
        raise ValueError("K must be a multiple of 128")
    if bits not in (3, 4):
        raise ValueError("bits must be 3 or 4")
    B = K // 128
    c = codes.reshape(N, B, 64, 2).astype(np.uint32)          # [row, block, pair, even/odd]
    words = np.zeros((N, B, 4, bits), dtype=np.uint32)        # [row, block, chunk, word]
    slots = SLOT3 if bits == 3 else SLOT4
    for q in range(4):
        for j in range(16):
            ev, od = c[:, :, 4 * j + q, 0], c[:, :, 4 * j + q, 1]
            if slots[j] is None:
                for e in range(3):
                    words[:, :, q, e] |= (((ev >> e) & 1) << 15) | (((od >> e) & 1) << 31)
            else:
                w, o = slots[j]
                words[:, :, q, w] |= (ev << o) | (od << (16 + o))
    return words.reshape(N, B * 4 * bits)


def unpack(words: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Inverse of pack: N x (K * bits / 32) uint32 words -> N x K uint8 codes."""
    words = np.asarray(words, dtype=np.uint32)
    N = words.shape[0]
    B = K // 128
    w4 = words.reshape(N, B, 4, bits)
    c = np.zeros((N, B, 64, 2), dtype=np.uint32)
    mask = (1 << bits) - 1
    slots = SLOT3 if bits == 3 else SLOT4
    for q in range(4):
        for j in range(16):
            if slots[j] is None:
                for e in range(3):
                    c[:, :, 4 * j + q, 0] |= ((w4[:, :, q, e] >> 15) & 1) << e
                    c[:, :, 4 * j + q, 1] |= ((w4[:, :, q, e] >> 31) & 1) << e
            else:
                w, o = slots[j]
                c[:, :, 4 * j + q, 0] = (w4[:, :, q, w] >> o) & mask
                c[:, :, 4 * j + q, 1] = (w4[:, :, q, w] >> (16 + o)) & mask
    return c.reshape(N, K).astype(np.uint8)


def pack_storage(codes: np.ndarray, idx, bits: int) -> np.ndarray:
    """The storage-favoured dense stream: per row, only the codes of the K - k dense columns,
    in column order, as one little-endian bit stream of `bits` bits per code (code p of the
    stream at bits [p b, p b + b)), padded with zero bits to whole uint32 words.

    [PL] "Storage Methods" (appendix §2, pp.10-11): the storage-favoured form drops the weak
    columns from the low-precision matrix (b + (16 - b) k / K bits per weight) instead of
    keeping them zero-filled (the latency-favoured form of ``pack``).  The bit order inside the
    stream is not given on the pages; a plain LSB-first stream is the reading taken.
    Returns uint32 N x ceil((K - k) b / 32).
    """
    codes = np.asarray(codes, dtype=np.uint8)
    N, K = codes.shape
    dense = np.ones(K, dtype=bool)
    idx = np.asarray(idx if idx is not None else [], dtype=np.int64)
    dense[idx] = False
    nd = int(dense.sum())
    W = (nd * bits + 31) // 32
    out = np.zeros((N, W), dtype=np.uint64)
    dc = codes[:, dense].astype(np.uint64)
    for p in range(nd):
        bit = p * bits
        w, o = divmod(bit, 32)
        v = dc[:, p] << np.uint64(o)
        out[:, w] |= v & np.uint64(0xFFFFFFFF)
        if o + bits > 32:
            out[:, w + 1] |= v >> np.uint64(32)
    return out.astype(np.uint32)


def unpack_storage(words: np.ndarray, K: int, idx, bits: int, zeros: np.ndarray, group: int) -> np.ndarray:
    """Inverse of ``pack_storage``, back to full N x K codes with the weak columns set to their
    group's zero point (the latency-favoured, zero-filled codes)."""
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    N = words.shape[0]
    dense = np.ones(K, dtype=bool)
    idx = np.asarray(idx if idx is not None else [], dtype=np.int64)
    dense[idx] = False
    mask = np.uint64((1 << bits) - 1)
    codes = np.zeros((N, K), dtype=np.uint8)
    for p, j in enumerate(np.flatnonzero(dense)):
        w, o = divmod(p * bits, 32)
        v = words[:, w] >> np.uint64(o)
        if o + bits > 32:
            v |= words[:, w + 1] << np.uint64(32 - o)
        codes[:, j] = (v & mask).astype(np.uint8)
    z = np.asarray(zeros, dtype=F16).astype(np.uint8)
    for j in idx:
        codes[:, j] = z[:, j // group]
    return codes


# ----------------------------------------------------------------------------------------
# The product
# ----------------------------------------------------------------------------------------
def matmul(W_hat: np.ndarray, w_weak: np.ndarray, idx: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y64[m, i] = sum_j W_hat[i, j] x[m, j] + sum_t W_weak[i, t] x[m, idx[t]]   (fp64).

    [PL] "Real-device acceleration" (paper "Acceleration on Real Device", p.6): a low-bit
    dense product plus an fp16 product over the weak-column activation channels gathered
    on the fly.  W_hat is zero at the weak columns, so the two terms together are the
    full-precision weak columns times their activations plus the quantised rest.
    Every fp16 value converts to fp64 exactly; the library matmul accumulates in fp64.
    """
    x64 = np.asarray(x, dtype=F16).astype(F64)
    y = np.asarray(W_hat, dtype=F16).astype(F64) @ x64.T
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size:
        y += np.asarray(w_weak, dtype=F16).astype(F64) @ x64[:, idx].T
    return np.ascontiguousarray(y.T)


def matmul_rows(codes, scales, zeros, w_weak, idx, x, rows) -> np.ndarray:
    """y64 restricted to the output rows `rows` (for sampled checks of large layers).

    Returns an M x len(rows) array; the same arithmetic as ``matmul`` on those rows.
    """
    rows = np.asarray(rows, dtype=np.int64)
    W_hat = dequant(np.asarray(codes)[rows], np.asarray(scales)[rows], np.asarray(zeros)[rows])
    return matmul(W_hat, np.asarray(w_weak)[rows], idx, x)


# ----------------------------------------------------------------------------------------
# The paper's own dense quantiser: truncation-aware parameter search, then OPTQ with the weak
# columns last
# ----------------------------------------------------------------------------------------
DEFAULT_ALPHAS = tuple(1.0 - 0.02 * i for i in range(26))   # range shrink factors 1.00 .. 0.50


def _dequant_one(q: np.ndarray, s: np.float16, z: np.float16) -> np.ndarray:
    return (np.float32(s) * (q.astype(F32) - np.float32(z))).astype(F16)


def search_params(W: np.ndarray, bits: int, group: int, weak_idx=None, alphas=DEFAULT_ALPHAS):
    """Truncation-aware 2-D grid search of (step size, zero point) per (row, group).

    [PL] "Low-precision quantization" (paper "Quantization Configuration Search", pp.4-5):
    before OPTQ, OWQ searches a 2-D grid over the step size and the zero point, with nearest
    rounding and truncation (clamping), so that the range may shrink below min-max and the
    reconstruction error drops.  Readings (the pages give no grid): the step sizes are the
    min-max step of the range [min(0, min w), max(0, max w)] (the quantize_rtn rules) times a
    shrink factor alpha in `alphas`, rounded to fp16; the zero points are every integer in
    [0, 2^b - 1]; the error is sum_j (w_j - fp16_rn(s (q_j - z)))^2 in fp64 over the group's
    dense columns, with q = clamp(rint(w / s) + z, 0, 2^b - 1) in fp32; the first minimum in
    the order (alpha descending, z ascending) wins; the error is a running fp64 sum in ascending
    column order, each square rounded before it is added.  Weak columns are left out of the
    search.
    Returns (scales fp16 N x G, zeros fp16 N x G).
    """
    W = np.asarray(W, dtype=F16)
    N, K = W.shape
    G = K // group
    qmax = (1 << bits) - 1
    dense = np.ones(K, dtype=bool)
    if weak_idx is not None and len(weak_idx):
        dense[np.asarray(weak_idx, dtype=np.int64)] = False
    scales = np.zeros((N, G), dtype=F16)
    zeros = np.zeros((N, G), dtype=F16)
    for i in range(N):
        for gi in range(G):
            cols = np.arange(gi * group, (gi + 1) * group)
            w = W[i, cols[dense[cols]]].astype(F32)
            mn = min(F32(0), w.min()) if w.size else F32(0)
            mx = max(F32(0), w.max()) if w.size else F32(0)
            if mn == mx:
                mn, mx = F32(-1), F32(1)
            best = None
            for a in alphas:
                s16 = F16((mx - mn) * F32(a) / F32(qmax))
                if s16 == 0:
                    continue
                s32 = F32(s16)
                for z in range(qmax + 1):
                    q = np.clip(np.rint(w / s32) + F32(z), F32(0), F32(qmax))
                    e = w.astype(F64) - _dequant_one(q, s16, F16(z)).astype(F64)
                    # fp64 sum of the squares in ascending column order (a running sum)
                    err = float(np.cumsum(e * e)[-1]) if e.size else 0.0
                    if best is None or err < best[0]:
                        best = (err, s16, z)
            if best is None:   # a range below fp16 resolution: fall back to [-1, 1]
                best = (0.0, F16(F32(2) / F32(qmax)), (qmax + 1) // 2)
            scales[i, gi] = best[1]
            zeros[i, gi] = F16(best[2])
    return scales, zeros


def optq_quantize(W: np.ndarray, X: np.ndarray, bits: int, group: int, weak_idx,
                  scales: np.ndarray, zeros: np.ndarray, damp: float = 0.01) -> dict:
    """OPTQ sequential column-wise quantisation with the weak columns moved to the end.

    [PL] "Low-precision quantization" (paper p.4): the dense weights go through OPTQ's
    column-by-column quantisation; the weak columns are moved to the end of the order, are
    never quantised, and absorb the compensation of the columns before them, so the stored
    fp16 weak block holds their compensated values.  [PL] "Layer-wise Quantization and
    Hessian": each row's error is dW H dW^T with H built from the calibration inputs
    (H = X^T X here; OPTQ's factor 2 cancels in every update).

    Each step is the optimal-brain-surgeon update written from its definition: with F the
    columns not yet quantised (the current column j first) and H_F^-1 the inverse of H
    restricted to F (recomputed at every step; no Cholesky form, no blocking), quantise column
    j with the given (scale, zero) of its group, then move the remaining columns of F by
    -(w_j - w_hat_j) / [H_F^-1]_jj * [H_F^-1]_{j, F without j}, which keeps them at the minimum of
    the row's error given the columns already fixed.  H gets damp * mean(diag H) added to its
    diagonal (a reading: OPTQ's usual dampening; damp = 0 for an exact solve).  The code
    decision is taken in fp32 on the current fp64 weight: q = clamp(rint(fp32(w) / s) + z).

    Returns codes (uint8 N x K; z at the weak columns), the weak block fp16 N x k (compensated
    values), and the compensated weak values in fp64 ("w_weak64") for checks.
    """
    W = np.asarray(W, dtype=F16)
    N, K = W.shape
    qmax = (1 << bits) - 1
    weak = np.asarray(weak_idx if weak_idx is not None else [], dtype=np.int64)
    is_weak = np.zeros(K, dtype=bool)
    is_weak[weak] = True
    order = np.concatenate([np.flatnonzero(~is_weak), np.sort(weak)])
    X64 = np.asarray(X, dtype=F16).astype(F64)
    H = X64.T @ X64
    if damp:
        H = H + damp * float(np.mean(np.diag(H))) * np.eye(K)
    Wc = W.astype(F64)
    codes = np.zeros((N, K), dtype=np.uint8)
    n_dense = K - len(weak)
    for step in range(n_dense):
        j = order[step]
        F = order[step:]
        Hinv = np.linalg.inv(H[np.ix_(F, F)])
        gi = j // group
        s16, z16 = scales[:, gi], zeros[:, gi]
        q = np.clip(np.rint(Wc[:, j].astype(F32) / s16.astype(F32)) + z16.astype(F32), F32(0), F32(qmax))
        w_hat = (s16.astype(F32) * (q - z16.astype(F32))).astype(F16).astype(F64)
        err = (Wc[:, j] - w_hat) / Hinv[0, 0]
        Wc[:, F[1:]] -= err[:, None] * Hinv[0, 1:][None, :]
        Wc[:, j] = w_hat
        codes[:, j] = q.astype(np.uint8)
    for t in weak:
        codes[:, t] = zeros[:, t // group].astype(np.uint8)
    w_weak64 = Wc[:, np.sort(weak)]
    return {"codes": codes, "scales": np.asarray(scales, dtype=F16), "zeros": np.asarray(zeros, dtype=F16),
            "idx": np.sort(weak).astype(np.int32), "w_weak": w_weak64.astype(F16), "w_weak64": w_weak64}


def owq_quantize_optq(W: np.ndarray, X: np.ndarray, bits: int, group: int, k: int,
                      damp: float = 0.01, alphas=DEFAULT_ALPHAS) -> dict:
    """The paper's full quantiser: weak-column selection, truncation-aware parameter search,
    then OPTQ with the weak columns last ([PL] "Weak-column selection", "Low-precision
    quantization").

    1. lambda, the all-column RTN perturbation, the sensitivity and the top-k selection exactly
       as in ``owq_quantize`` (steps 1-4);
    2. (scale, zero) per (row, group) by ``search_params`` over the dense columns;
    3. ``optq_quantize`` with those parameters; the weak block holds the compensated values.
    """
    W = np.asarray(W, dtype=F16)
    lam = hessian_diag(X)
    c0, s0, z0 = quantize_rtn(W, bits, group, None)
    sens = sensitivity(W, dequant(c0, s0, z0), lam)
    idx = select_weak(sens, k)
    scales, zeros = search_params(W, bits, group, idx, alphas)
    r = optq_quantize(W, X, bits, group, idx, scales, zeros, damp)
    r["lam"], r["sens"] = lam, sens
    return r


# ----------------------------------------------------------------------------------------
# Weak column tuning: the two gradients a frozen OWQ layer passes back
# ----------------------------------------------------------------------------------------
def weak_grad(x: np.ndarray, dy: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """dW_weak[i, t] = sum_m dy[m, i] x[m, idx[t]]   (fp64, N x k).

    [PL] "Weak Column Tuning" (paper "PEFT with Weak Column Tuning", p.5) and "WCT-based
    fine-tuning" (p.7): only the fp16 weak columns are trained, the packed low-bit matrix stays
    frozen.  The forward term that holds them is sum_t W_weak[i, t] x[m, idx[t]], so the
    gradient of a loss with output gradient dy is the product of dy^T and the gathered
    activation columns.
    """
    dy64 = np.asarray(dy, dtype=F16).astype(F64)
    x64 = np.asarray(x, dtype=F16).astype(F64)
    idx = np.asarray(idx, dtype=np.int64)
    return dy64.T @ x64[:, idx]


def input_grad(W_hat: np.ndarray, w_weak: np.ndarray, idx: np.ndarray, dy: np.ndarray) -> np.ndarray:
    """dX[m, j] = sum_i dy[m, i] W_hat[i, j] + sum_{t: idx[t] = j} sum_i dy[m, i] W_weak[i, t]
    (fp64, M x K).

    The gradient a frozen OWQ layer passes to the layer below during weak column tuning
    ([PL] "Weak Column Tuning", p.5: the dense matrix stays frozen, earlier layers' weak
    columns still need it): the transpose of the forward product of [PL] "Real-device
    acceleration", with the weak columns' fp16 values in place of the zero-filled codes.
    """
    dy64 = np.asarray(dy, dtype=F16).astype(F64)
    dx = dy64 @ np.asarray(W_hat, dtype=F16).astype(F64)
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size:
        dx[:, idx] += dy64 @ np.asarray(w_weak, dtype=F16).astype(F64)
    return dx


# ----------------------------------------------------------------------------------------
# Storage accounting
# ----------------------------------------------------------------------------------------
def layer_bytes(N: int, K: int, bits: int, group: int, k: int) -> dict:
    """Bytes of the latency-favoured layout: packed codes, fp16 scale + zero per (row,
    group), fp16 weak block N x k, int32 index list."""
    G = K // group
    return {"packed": N * K * bits // 8, "scales_zeros": N * G * 4, "weak": N * k * 2, "idx": 4 * k}


def bits_per_weight(K: int, bits: int, k: float, layout: str = "latency",
                    group: int | None = None, N: int | None = None) -> float:
    """Effective bits per weight.

    [PL] "Storage Methods" (appendix §2, pp.10-11): the storage-favoured form keeps only
    the dense codes plus the fp16 weak columns, b + (16 - b) k / K; the latency-favoured
    form also keeps the zero-filled codes of the weak columns, b + 16 k / K.  With
    `group` given, the fp16 scale and zero (32 bits per group) are added; with N also
    given, the int32 index list (32 k bits over N K weights).
    """
    if layout == "storage":
        b = bits + (16 - bits) * k / K
    elif layout == "latency":
        b = bits + 16.0 * k / K
    else:
        raise ValueError(layout)
    if group is not None:
        b += 32.0 / group
        if N is not None:
            b += 32.0 * k / (N * K)
    return b
