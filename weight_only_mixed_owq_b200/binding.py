"""ctypes binding of libowq_b200.so (include/owq.h): same names, argument marshalling only.

Every function here forwards to the C ABI; PyTorch is used only to allocate device memory
and to name streams.  There is no CPU fallback: if the library is missing this module
raises at import time.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# OWQ_LIB_VARIANT=bounds loads the debug-bounds build (libowq_b200_bounds.so) built beside it
VARIANTS = {"": "libowq_b200.so", "bounds": "libowq_b200_bounds.so"}
_variant = os.environ.get("OWQ_LIB_VARIANT", "")
if _variant not in VARIANTS:
    raise ImportError(f"OWQ_LIB_VARIANT={_variant!r}: expected one of {sorted(VARIANTS)}")
LIB_PATH = os.path.join(PKG, VARIANTS[_variant])

OWQ_OK = 0
STATUS_NAMES = {
    0: "OWQ_OK", 1: "OWQ_ERR_NULL", 2: "OWQ_ERR_SHAPE", 3: "OWQ_ERR_BITS", 4: "OWQ_ERR_GROUP",
    5: "OWQ_ERR_INDEX", 6: "OWQ_ERR_ALIGN", 7: "OWQ_ERR_CUDA", 8: "OWQ_ERR_TIMEOUT",
    9: "OWQ_ERR_NOMEM", 10: "OWQ_ERR_HANDLE", 11: "OWQ_ERR_DEVICE", 12: "OWQ_ERR_ARG", 13: "OWQ_ERR_BOUNDS",
}
OWQ_INJECT_NONE, OWQ_INJECT_GEMV_TAG, OWQ_INJECT_GEMM_ARRIVE, OWQ_INJECT_BOUNDS = 0, 1, 2, 3

# (name, restype, argtypes) of every exported symbol of include/owq.h
_P, _I, _SZ, _S = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t), ctypes.c_char_p
PROTOTYPES = [
    ("owq_quantize", _I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    ("owq_quantize_noalloc", _I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    ("owq_pack", _I, [_P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P, ctypes.POINTER(_P)]),
    ("owq_search_params", _I, [_P, _I, _I, _I, _I, _P, _I, _P, _P, _P]),
    ("owq_optq", _I, [_P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _P, ctypes.c_double, _P, _P, _P]),
    ("owq_quantize_optq", _I, [_P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_double, _P, _P, _P, _P, _P, _P]),
    ("owq_storage_words", _I, [_I, _I, _I, ctypes.POINTER(_I)]),
    ("owq_storage_pack", _I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    ("owq_storage_unpack", _I, [_P, _I, _I, _I, _I, _P, _I, _P, _P, _P]),
    ("owq_pack_storage", _I, [_P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P, ctypes.POINTER(_P)]),
    ("owq_gemv", _I, [_P, _P, _P, _I, _P]),
    ("owq_gemv_multi", _I, [ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P), _I, _I, _P]),
    ("owq_gemm", _I, [_P, _P, _P, _I, _P]),
    ("owq_gemm_plan", _I, [_I, _I, _I, _I, ctypes.POINTER(_I)]),
    ("owq_weak_grad", _I, [_P, _P, _P, _P, _I, _P]),
    ("owq_input_grad", _I, [_P, _P, _P, _I, _P]),
    ("owq_dequant", _I, [_P, _P, _P, _P]),
    ("owq_layer_info", _I, [_P] + [ctypes.POINTER(_I)] * 5),
    ("owq_layer_bytes", _I, [_P, _SZ, _SZ, _SZ, _SZ]),
    ("owq_layer_free", _I, [_P]),
    ("owq_device_status", _I, []),
    ("owq_debug_inject", _I, [_I, ctypes.c_longlong]),
    ("owq_status_string", _S, [_I]),
    ("owq_version", _S, []),
]


class OwqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m weight_only_mixed_owq_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, res, args in PROTOTYPES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _ptr(a) -> int | None:
    """Device address of a tensor (or an int address, or None)."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int, where: str) -> None:
    if st != OWQ_OK:
        raise OwqError(st, where)


# ------------------------------------------------------------------ raw C-ABI mirrors
def owq_quantize(W, X, N, K, T, bits, group, k, codes, scales, zeros, idx, w_weak, stream=None) -> int:
    return LIB.owq_quantize(_ptr(W), _ptr(X), N, K, T, bits, group, k, _ptr(codes), _ptr(scales),
                            _ptr(zeros), _ptr(idx), _ptr(w_weak), _stream(stream))


def owq_quantize_noalloc(W, X, N, K, T, bits, group, k, codes, scales, zeros, idx, w_weak, stream=None) -> int:
    return LIB.owq_quantize_noalloc(_ptr(W), _ptr(X), N, K, T, bits, group, k, _ptr(codes), _ptr(scales),
                                    _ptr(zeros), _ptr(idx), _ptr(w_weak), _stream(stream))


def owq_pack(codes, N, K, bits, group, scales, zeros, idx, k, w_weak, stream=None):
    """Returns (status, handle)."""
    h = ctypes.c_void_p()
    st = LIB.owq_pack(_ptr(codes), N, K, bits, group, _ptr(scales), _ptr(zeros), _ptr(idx), k,
                      _ptr(w_weak), _stream(stream), ctypes.byref(h))
    return st, h.value


def owq_search_params(W, N, K, bits, group, idx, k, scales, zeros, stream=None) -> int:
    return LIB.owq_search_params(_ptr(W), N, K, bits, group, _ptr(idx), k, _ptr(scales), _ptr(zeros), _stream(stream))


def owq_optq(W, X, N, K, T, bits, group, idx, k, scales, zeros, damp, codes, w_weak, stream=None) -> int:
    return LIB.owq_optq(_ptr(W), _ptr(X), N, K, T, bits, group, _ptr(idx), k, _ptr(scales), _ptr(zeros),
                        float(damp), _ptr(codes), _ptr(w_weak), _stream(stream))


def owq_quantize_optq(W, X, N, K, T, bits, group, k, damp, codes, scales, zeros, idx, w_weak, stream=None) -> int:
    return LIB.owq_quantize_optq(_ptr(W), _ptr(X), N, K, T, bits, group, k, float(damp), _ptr(codes), _ptr(scales),
                                 _ptr(zeros), _ptr(idx), _ptr(w_weak), _stream(stream))


def owq_storage_words(K, bits, k):
    """Returns (status, uint32 words per row of the storage-favoured stream)."""
    w = ctypes.c_int()
    st = LIB.owq_storage_words(K, bits, k, ctypes.byref(w))
    return st, w.value


def owq_storage_pack(codes, N, K, bits, idx, k, words, stream=None) -> int:
    return LIB.owq_storage_pack(_ptr(codes), N, K, bits, _ptr(idx), k, _ptr(words), _stream(stream))


def owq_storage_unpack(words, N, K, bits, group, idx, k, zeros, codes, stream=None) -> int:
    return LIB.owq_storage_unpack(_ptr(words), N, K, bits, group, _ptr(idx), k, _ptr(zeros), _ptr(codes),
                                  _stream(stream))


def owq_pack_storage(words, N, K, bits, group, scales, zeros, idx, k, w_weak, stream=None):
    """Returns (status, handle)."""
    h = ctypes.c_void_p()
    st = LIB.owq_pack_storage(_ptr(words), N, K, bits, group, _ptr(scales), _ptr(zeros), _ptr(idx), k,
                              _ptr(w_weak), _stream(stream), ctypes.byref(h))
    return st, h.value


def owq_gemv(layer, x, y, M, stream=None) -> int:
    return LIB.owq_gemv(layer, _ptr(x), _ptr(y), M, _stream(stream))


def owq_gemv_multi(layers, xs, ys, M, stream=None) -> int:
    n = len(layers)
    arr_l = (ctypes.c_void_p * n)(*layers)
    arr_x = (ctypes.c_void_p * n)(*[_ptr(v) for v in xs])
    arr_y = (ctypes.c_void_p * n)(*[_ptr(v) for v in ys])
    return LIB.owq_gemv_multi(arr_l, arr_x, arr_y, n, M, _stream(stream))


def owq_gemm(layer, x, y, M, stream=None) -> int:
    return LIB.owq_gemm(layer, _ptr(x), _ptr(y), M, _stream(stream))


def owq_gemm_plan(N, K, M, sms):
    """Returns (status, {tile_tokens, splits, tail_tiles, tail_splits}): owq_gemm's launch shape."""
    out = (ctypes.c_int * 4)()
    st = LIB.owq_gemm_plan(N, K, M, sms, out)
    return st, dict(zip(("tile_tokens", "splits", "tail_tiles", "tail_splits"), out))


def owq_weak_grad(layer, x, dy, dw_weak, M, stream=None) -> int:
    return LIB.owq_weak_grad(layer, _ptr(x), _ptr(dy), _ptr(dw_weak), M, _stream(stream))


def owq_input_grad(layer, dy, dx, M, stream=None) -> int:
    return LIB.owq_input_grad(layer, _ptr(dy), _ptr(dx), M, _stream(stream))


def owq_dequant(layer, w_hat, codes=None, stream=None) -> int:
    return LIB.owq_dequant(layer, _ptr(w_hat), _ptr(codes), _stream(stream))


def owq_layer_info(layer):
    vals = [ctypes.c_int() for _ in range(5)]
    st = LIB.owq_layer_info(layer, *[ctypes.byref(v) for v in vals])
    return st, tuple(v.value for v in vals)


def owq_layer_bytes(layer):
    vals = [ctypes.c_size_t() for _ in range(4)]
    st = LIB.owq_layer_bytes(layer, *[ctypes.byref(v) for v in vals])
    return st, dict(zip(("packed", "scales_zeros", "weak", "idx"), (v.value for v in vals)))


def owq_layer_free(layer) -> int:
    return LIB.owq_layer_free(layer)


def owq_device_status() -> int:
    return LIB.owq_device_status()


def owq_debug_inject(what: int, wait_cycles: int) -> int:
    return LIB.owq_debug_inject(what, wait_cycles)


def owq_status_string(st: int) -> str:
    return LIB.owq_status_string(st).decode()


def owq_version() -> str:
    return LIB.owq_version().decode()


# ------------------------------------------------------------------ torch-facing helpers
def quantize(W, X, bits: int, group: int, k: int, stream=None) -> dict:
    """Run owq_quantize on fp16 CUDA tensors W (N x K) and X (T x K); allocates the outputs."""
    import torch
    N, K = W.shape
    T = X.shape[0]
    dev = W.device
    out = {
        "codes": torch.empty((N, K), dtype=torch.uint8, device=dev),
        "scales": torch.empty((N, K // group), dtype=torch.float16, device=dev),
        "zeros": torch.empty((N, K // group), dtype=torch.float16, device=dev),
        "idx": torch.empty((k,), dtype=torch.int32, device=dev),
        "w_weak": torch.empty((N, k), dtype=torch.float16, device=dev),
    }
    _check(owq_quantize(W, X, N, K, T, bits, group, k, out["codes"], out["scales"], out["zeros"],
                        out["idx"] if k else None, out["w_weak"] if k else None, stream), "owq_quantize")
    return out


class OwqLayer:
    """A packed layer owned by the C library (freed on close() / garbage collection)."""

    def __init__(self, codes, scales, zeros, idx, w_weak, bits: int, group: int, stream=None):
        N, K = codes.shape
        k = 0 if idx is None else int(idx.numel())
        st, h = owq_pack(codes, N, K, bits, group, scales, zeros, idx if k else None, k,
                         w_weak if k else None, stream)
        _check(st, "owq_pack")
        self.handle = h
        self.N, self.K, self.bits, self.group, self.k = N, K, bits, group, k

    def gemv(self, x, y=None, stream=None):
        import torch
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=x.device)
        _check(owq_gemv(self.handle, x, y, M, stream), "owq_gemv")
        return y

    def gemm(self, x, y=None, stream=None):
        import torch
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float16, device=x.device)
        _check(owq_gemm(self.handle, x, y, M, stream), "owq_gemm")
        return y

    def weak_grad(self, x, dy, dw=None, stream=None):
        """dW_weak = dy^T x[:, idx] (fp32 N x k)."""
        import torch
        M = x.shape[0]
        if dw is None:
            dw = torch.empty((self.N, self.k), dtype=torch.float32, device=x.device)
        _check(owq_weak_grad(self.handle, x, dy, dw if self.k else None, M, stream), "owq_weak_grad")
        return dw

    def input_grad(self, dy, dx=None, stream=None):
        """dX = dy W_eff (fp16 M x K)."""
        import torch
        M = dy.shape[0]
        if dx is None:
            dx = torch.empty((M, self.K), dtype=torch.float16, device=dy.device)
        _check(owq_input_grad(self.handle, dy, dx, M, stream), "owq_input_grad")
        return dx

    def dequant(self, with_codes: bool = False, stream=None):
        import torch
        dev = torch.device("cuda")
        w = torch.empty((self.N, self.K), dtype=torch.float16, device=dev)
        c = torch.empty((self.N, self.K), dtype=torch.uint8, device=dev) if with_codes else None
        _check(owq_dequant(self.handle, w, c, stream), "owq_dequant")
        return (w, c) if with_codes else w

    def nbytes(self) -> dict:
        st, b = owq_layer_bytes(self.handle)
        _check(st, "owq_layer_bytes")
        return b

    def close(self):
        if getattr(self, "handle", None):
            owq_layer_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize_optq(W, X, bits: int, group: int, k: int, damp: float = 0.01, stream=None) -> dict:
    """Run owq_quantize_optq (selection, parameter search, OPTQ with the weak columns last) on
    fp16 CUDA tensors W (N x K) and X (T x K); allocates the outputs."""
    import torch
    N, K = W.shape
    T = X.shape[0]
    dev = W.device
    out = {
        "codes": torch.empty((N, K), dtype=torch.uint8, device=dev),
        "scales": torch.empty((N, K // group), dtype=torch.float16, device=dev),
        "zeros": torch.empty((N, K // group), dtype=torch.float16, device=dev),
        "idx": torch.empty((k,), dtype=torch.int32, device=dev),
        "w_weak": torch.empty((N, k), dtype=torch.float16, device=dev),
    }
    _check(owq_quantize_optq(W, X, N, K, T, bits, group, k, damp, out["codes"], out["scales"], out["zeros"],
                             out["idx"] if k else None, out["w_weak"] if k else None, stream), "owq_quantize_optq")
    return out


def quantize_pack(W, X, bits: int, group: int, k: int, stream=None) -> tuple[OwqLayer, dict]:
    """owq_quantize then owq_pack (both on the GPU)."""
    q = quantize(W, X, bits, group, k, stream)
    layer = OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"], q["w_weak"], bits, group, stream)
    return layer, q
