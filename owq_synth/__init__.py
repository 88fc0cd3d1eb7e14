"""Seeded synthetic inputs for the OWQ mixed-precision matmul.

This module is shared by the CUDA path's tests and benchmark and by the CPU oracle.
It only draws random numbers: it holds none of the method's arithmetic (no
quantisation, no sensitivity score, no packing, no product).

What it draws follows the workloads the OWQ pages describe (OPT / LLaMA decoder
layers, activations with a few large "outlier" input channels):

* the weight W of a linear layer, N output channels x K input channels, fp16,
  drawn as N(0, 0.02^2) in fp32 and rounded to fp16;
* a calibration matrix X, T tokens x K channels, fp16, N(0, 1) with the outlier
  channels multiplied by their factor (these are what make some weight columns
  "weak": Problem Definition / Sensitivity to Outliers, OWQ p.3);
* the activations x, M tokens x K, fp16, drawn the same way with the same outlier
  channels.

All draws use numpy's PCG64 generator seeded explicitly, in fp32, then rounded to
fp16 (round-to-nearest-even, numpy's cast).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "LayerSpec",
    "WorkloadSpec",
    "WORKLOADS",
    "rng",
    "outlier_channels",
    "draw_weight",
    "draw_activations",
    "draw_layer",
    "seed_for",
]


def rng(seed: int) -> np.random.Generator:
    """A PCG64 generator with an explicit seed."""
    return np.random.Generator(np.random.PCG64(int(seed)))


def seed_for(workload_id: int, layer_id: int) -> int:
    """Seed of one layer of one workload: 1234 + 100 * workload + layer."""
    return 1234 + 100 * int(workload_id) + int(layer_id)


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer of a workload: y = x W^T with W of shape N x K."""

    name: str
    N: int
    K: int
    bits: int
    group: int          # K for per-output-channel, 128 for per-group
    k: int              # number of weak (fp16) columns


@dataclass(frozen=True)
class WorkloadSpec:
    """A set of layers sharing a quantisation recipe and an activation recipe."""

    wid: int
    name: str
    layers: tuple
    Ms: tuple                     # token counts exercised
    outlier: str                  # "count" | "frac" | "heavy"
    outlier_arg: float            # count, fraction, or fraction (heavy)
    outlier_factor: float         # multiplier for "count"/"frac"
    T: int = 256                  # calibration tokens
    n_sets: int = 1               # distinct resident copies streamed per step
    extra: dict = field(default_factory=dict)


def _set(prefix, shapes, bits, group):
    out = []
    for name, N, K in shapes:
        out.append(LayerSpec(f"{prefix}.{name}", N, K, bits, K if group == "K" else group, K // 128))
    return tuple(out)


_OPT67 = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("out", 4096, 4096),
          ("fc1", 16384, 4096), ("fc2", 4096, 16384)]
_LLAMA7 = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
           ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
_OPT66 = [("q", 9216, 9216), ("k", 9216, 9216), ("v", 9216, 9216), ("out", 9216, 9216),
          ("fc1", 36864, 9216), ("fc2", 9216, 36864)]
_LLAMA13 = [("up", 13824, 5120), ("down", 5120, 13824)]

# Workload 0 is the small single layer the oracle finishes in seconds; 1-4 take the
# shapes of the OPT / LLaMA models the OWQ pages evaluate (Experimental Setup, p.5).
WORKLOADS = {
    0: WorkloadSpec(0, "single-512", (LayerSpec("single", 512, 512, 3, 512, 4),), (1,),
                    "count", 4, 50.0),
    1: WorkloadSpec(1, "opt-6.7b-decode", _set("opt6.7b", _OPT67, 3, "K"), (1,),
                    "frac", 0.005, 30.0),
    2: WorkloadSpec(2, "llama-7b-decode", _set("llama7b", _LLAMA7, 4, 128), (1, 2, 4, 8, 16),
                    "heavy", 0.01, 0.0),
    3: WorkloadSpec(3, "opt-66b-decode", _set("opt66b", _OPT66, 3, "K"), (1,),
                    "frac", 0.005, 30.0, n_sets=64),
    4: WorkloadSpec(4, "llama-13b-prefill", _set("llama13b", _LLAMA13, 3, 128),
                    (64, 128, 256, 512, 2048), "frac", 0.005, 50.0),
}


def outlier_channels(g: np.random.Generator, K: int, kind: str, arg: float) -> np.ndarray:
    """Indices (ascending) of the input channels that carry activation outliers."""
    if kind == "count":
        n = int(arg)
    else:
        n = int(math.ceil(arg * K))
    n = max(0, min(K, n))
    return np.sort(g.choice(K, size=n, replace=False)).astype(np.int64)


def _channel_gain(g: np.random.Generator, K: int, chans: np.ndarray, kind: str, factor: float) -> np.ndarray:
    """Per-channel multiplier c_j: the outlier factor on the chosen channels, 1 elsewhere.

    For the "heavy" recipe each chosen channel draws its own factor
    exp(U[ln 10, ln 100]) (a heavy tail between x10 and x100).
    """
    gain = np.ones(K, dtype=np.float32)
    if kind == "heavy":
        gain[chans] = np.exp(g.uniform(math.log(10.0), math.log(100.0), size=chans.size)).astype(np.float32)
    else:
        gain[chans] = np.float32(factor)
    return gain


def draw_weight(g: np.random.Generator, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """W ~ N(0, std^2), drawn in fp32, rounded to fp16; shape N x K (row = output channel)."""
    return (g.standard_normal((N, K), dtype=np.float32) * np.float32(std)).astype(np.float16)


def draw_activations(g: np.random.Generator, rows: int, gain: np.ndarray) -> np.ndarray:
    """rows x K activations: N(0,1) times the per-channel gain, fp32 then fp16."""
    K = gain.size
    a = g.standard_normal((rows, K), dtype=np.float32) * gain[None, :]
    return a.astype(np.float16)


def draw_layer(spec: LayerSpec, workload: WorkloadSpec, M: int, seed: int, T: int | None = None) -> dict:
    """Draw W, the calibration X and the activations x for one layer.

    Returns a dict with fp16 arrays ``W`` (N x K), ``X`` (T x K), ``x`` (M x K) and
    the int64 array ``outliers`` (the outlier channel indices).
    The draw order is fixed (channels, gains, W, X, x) so a seed fixes every array.
    """
    g = rng(seed)
    T = workload.T if T is None else T
    chans = outlier_channels(g, spec.K, workload.outlier, workload.outlier_arg)
    gain = _channel_gain(g, spec.K, chans, workload.outlier, workload.outlier_factor)
    W = draw_weight(g, spec.N, spec.K)
    X = draw_activations(g, T, gain)
    x = draw_activations(g, M, gain)
    return {"W": W, "X": X, "x": x, "outliers": chans}


def draw_small(N: int, K: int, M: int, T: int, seed: int, n_outliers: int = 2,
               factor: float = 50.0) -> dict:
    """A small ad-hoc layer (for parity tests on odd shapes): same recipe as workload 0."""
    g = rng(seed)
    chans = outlier_channels(g, K, "count", min(n_outliers, K))
    gain = _channel_gain(g, K, chans, "count", factor)
    W = draw_weight(g, N, K)
    X = draw_activations(g, T, gain)
    x = draw_activations(g, M, gain)
    return {"W": W, "X": X, "x": x, "outliers": chans}


def draw_codes(g: np.random.Generator, N: int, K: int, bits: int) -> np.ndarray:
    """Uniform random integer codes in [0, 2^bits - 1] (for layout round-trip tests)."""
    return g.integers(0, 1 << bits, size=(N, K), dtype=np.uint8)
