"""ctypes binding of libawq.so (declared in include/awq.h).

Argument marshalling only: every function here passes device pointers,
sizes and the current CUDA stream to the C ABI of the same name and raises
AwqError on a non-zero status.  Every step of the search runs in the
library's sm_100a kernels; there is no fallback.  If the library is missing
the import of this module fails with a message saying how to build it.
"""

from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_uint8, c_void_p
from typing import Optional

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
# AWQ_LIB=debug loads the debug library (index checks in the kernels,
# awq_bounds_status); the default is the release library
LIB_PATH = os.path.join(PKG_DIR, "libawq_debug.so" if os.environ.get("AWQ_LIB") == "debug"
                        else "libawq.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG_DIR), "include", "awq.h")

STATUS = {
    0: "AWQ_OK",
    1: "AWQ_ERR_INVALID_ARG",
    2: "AWQ_ERR_UNSUPPORTED",
    3: "AWQ_ERR_WORKSPACE",
    4: "AWQ_ERR_CUDA",
    5: "AWQ_ERR_TIMEOUT",
    6: "AWQ_ERR_NONFINITE",
}


class AwqError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        self.status = status
        self.status_name = STATUS.get(status, str(status))
        super().__init__(f"{func}: {self.status_name}: {message}")


SEARCH_DIRECT, SEARCH_GRAM, SEARCH_CACHED_Y, SEARCH_FUSED = 0, 1, 2, 3


class AwqConfig(ctypes.Structure):
    """awq_config: w_bit, group_size, zero_point ("05 — AWQ" §9 quant_config),
    n_alpha, n_clip, clip_min ("05 — AWQ" §4), search_form (0 direct scored
    GEMM, 1 Gram form, 2 cached fp16 output, 3 candidates made inside the
    GEMM)."""

    _fields_ = [
        ("w_bit", c_int32),
        ("group_size", c_int32),
        ("zero_point", c_int32),
        ("n_alpha", c_int32),
        ("n_clip", c_int32),
        ("clip_min", c_float),
        ("search_form", c_int32),
    ]

    @classmethod
    def make(cls, w_bit=4, group_size=128, zero_point=1, n_alpha=20, n_clip=0, clip_min=0.5,
             search_form=0):
        return cls(int(w_bit), int(group_size), int(zero_point), int(n_alpha), int(n_clip),
                   float(clip_min), int(search_form))


_SIGNATURES = {
    "awq_version": (c_char_p, []),
    "awq_last_error": (c_char_p, []),
    "awq_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, POINTER(AwqConfig)]),
    "awq_workspace_size_min": (c_size_t, [c_int64, c_int64, c_int64, POINTER(AwqConfig)]),
    "awq_act_stats": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p]),
    "awq_scale_grid": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_void_p]),
    "awq_search_scale": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_void_p,
                                   POINTER(AwqConfig), c_void_p, c_size_t, c_void_p, c_void_p,
                                   c_void_p, c_void_p]),
    "awq_search_clip": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64, c_void_p,
                                  POINTER(AwqConfig), c_void_p, c_size_t, c_void_p, c_void_p,
                                  c_void_p]),
    "awq_search_clip_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64,
                                          c_void_p, POINTER(AwqConfig), c_void_p, c_void_p,
                                          c_void_p]),
    "awq_candidate_codes": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, POINTER(AwqConfig),
                                      c_void_p, c_size_t, c_void_p, c_void_p, c_void_p, c_void_p]),
    "awq_clip_candidate_codes": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p,
                                           POINTER(AwqConfig), c_void_p, c_size_t, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p]),
    "awq_quant_pack": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, POINTER(AwqConfig),
                                 c_void_p, c_void_p, c_void_p, c_void_p]),
    "awq_fold_inv_scale": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    "awq_w4a16_gemm": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                 c_int64, POINTER(AwqConfig), c_void_p, c_int64, c_void_p, c_size_t,
                                 c_void_p]),
    "awq_w4a16_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, POINTER(AwqConfig)]),
    "awq_act_sums": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p]),
    "awq_act_stats_finish": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p]),
    "awq_search_scale_sse": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_int64,
                                       c_void_p, POINTER(AwqConfig), c_void_p, c_size_t, c_void_p,
                                       c_void_p]),
    "awq_select_scale": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_void_p, POINTER(AwqConfig),
                                   c_void_p, c_size_t, c_void_p, c_void_p, c_void_p, c_void_p]),
    "awq_block_grams": (c_int32, [c_void_p, c_int64, c_int64, c_int64, POINTER(AwqConfig), c_void_p,
                                  c_size_t, c_void_p, c_void_p]),
    "awq_search_clip_grams": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p,
                                        POINTER(AwqConfig), c_void_p, c_size_t, c_void_p, c_void_p,
                                        c_void_p]),
    "awq_device_status": (c_int32, [c_void_p, c_void_p]),
    "awq_profile_enable": (c_int32, [c_int32]),
    "awq_profile_read": (c_int32, [c_char_p, POINTER(c_double), POINTER(c_int64)]),
    "awq_profile_reset": (c_int32, []),
    "awq_bounds_checks_enabled": (c_int32, []),
    "awq_bounds_status": (c_int32, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m post_weight_quantization_awq_b200.build` "
            "(nvcc, sm_100a); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        try:
            fn = getattr(lib, name)
        except AttributeError as e:
            raise ImportError(f"{LIB_PATH} does not export {name}: rebuild it") from e
        fn.restype = res
        fn.argtypes = args
    return lib


class _Lib:
    """libawq.so, loaded on first use (so that the build module can be
    imported before the library exists); a missing or stale library raises
    ImportError at the first call."""

    _lib = None

    def _get(self) -> ctypes.CDLL:
        if _Lib._lib is None:
            _Lib._lib = _load()
        return _Lib._lib

    def __getattr__(self, name):
        return getattr(self._get(), name)

    def __getitem__(self, name):
        return self._get()[name]


LIB = _Lib()


def header_functions(path: str = HEADER_PATH):
    """Names of the functions include/awq.h declares."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(awq_[a-z0-9_]+)\s*\(", text)))


def version() -> str:
    return LIB.awq_version().decode()


def last_error() -> str:
    return LIB.awq_last_error().decode()


def _check(func: str, status: int) -> None:
    if status != 0:
        raise AwqError(func, status, last_error())


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is not None:
        return int(stream)
    import torch
    return torch.cuda.current_stream().cuda_stream


def awq_workspace_size(T: int, inn: int, out: int, cfg: AwqConfig) -> int:
    n = LIB.awq_workspace_size(T, inn, out, ctypes.byref(cfg))
    if n == 0:
        raise AwqError("awq_workspace_size", 1, last_error())
    return int(n)


def awq_workspace_size_min(T: int, inn: int, out: int, cfg: AwqConfig) -> int:
    """The smallest workspace the search and clip calls accept (the alpha
    search then runs its candidates in chunks)."""
    n = LIB.awq_workspace_size_min(T, inn, out, ctypes.byref(cfg))
    if n == 0:
        raise AwqError("awq_workspace_size_min", 1, last_error())
    return int(n)


def awq_act_stats(X, abar, stream=None) -> None:
    """X: CUDA fp16 [T, in] (row stride X.stride(0)); abar: CUDA fp64 [in]."""
    _check("awq_act_stats", LIB.awq_act_stats(_ptr(X), X.shape[0], X.shape[1], X.stride(0),
                                              _ptr(abar), _stream(stream)))


def awq_scale_grid(abar, n_alpha: int, s, stream=None) -> None:
    _check("awq_scale_grid", LIB.awq_scale_grid(_ptr(abar), abar.shape[0], n_alpha, _ptr(s),
                                                _stream(stream)))


def awq_search_scale(X, W, abar, cfg: AwqConfig, ws, s_best, mse, best_idx, stream=None) -> None:
    _check("awq_search_scale", LIB.awq_search_scale(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), _ptr(W), W.shape[0], _ptr(abar),
        ctypes.byref(cfg), _ptr(ws), ws.numel() * ws.element_size(), _ptr(s_best), _ptr(mse),
        _ptr(best_idx), _stream(stream)))


def awq_search_clip(X, W, s, cfg: AwqConfig, ws, clip_idx, err=None, stream=None) -> None:
    _check("awq_search_clip", LIB.awq_search_clip(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), _ptr(W), W.shape[0], _ptr(s),
        ctypes.byref(cfg), _ptr(ws), ws.numel() * ws.element_size(), _ptr(clip_idx), _ptr(err),
        _stream(stream)))


def awq_search_clip_noalloc(X, W, s, cfg: AwqConfig, clip_idx, err=None, stream=None) -> None:
    """awq_search_clip without a workspace (scratch in the library's static
    device array; in <= 16384; overlapping calls race)."""
    _check("awq_search_clip_noalloc", LIB.awq_search_clip_noalloc(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), _ptr(W), W.shape[0], _ptr(s),
        ctypes.byref(cfg), _ptr(clip_idx), _ptr(err), _stream(stream)))


def awq_quant_pack(W, s, clip_idx, cfg: AwqConfig, qweight, qzeros, scales, stream=None) -> None:
    _check("awq_quant_pack", LIB.awq_quant_pack(
        _ptr(W), W.shape[0], W.shape[1], _ptr(s), _ptr(clip_idx), ctypes.byref(cfg),
        _ptr(qweight), _ptr(qzeros), _ptr(scales), _stream(stream)))


def awq_fold_inv_scale(v, s, stream=None) -> None:
    rows = v.shape[0]
    cols = v.numel() // rows
    _check("awq_fold_inv_scale", LIB.awq_fold_inv_scale(_ptr(v), rows, cols, _ptr(s),
                                                        _stream(stream)))


def awq_act_sums(X, sums, stream=None) -> None:
    """Exact sums of |X| over these tokens, int64 [in] in units of 2^-24."""
    _check("awq_act_sums", LIB.awq_act_sums(_ptr(X), X.shape[0], X.shape[1], X.stride(0),
                                            _ptr(sums), _stream(stream)))


def awq_act_stats_finish(sums, T_total: int, abar, stream=None) -> None:
    _check("awq_act_stats_finish", LIB.awq_act_stats_finish(_ptr(sums), int(T_total), sums.shape[0],
                                                            _ptr(abar), _stream(stream)))


def awq_search_scale_sse(X, W, abar, cfg: AwqConfig, ws, sse, stream=None) -> None:
    _check("awq_search_scale_sse", LIB.awq_search_scale_sse(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), _ptr(W), W.shape[0], _ptr(abar),
        ctypes.byref(cfg), _ptr(ws), ws.numel() * ws.element_size(), _ptr(sse), _stream(stream)))


def awq_select_scale(sse, T_total: int, out: int, abar, cfg: AwqConfig, ws, s_best, mse, best_idx,
                     stream=None) -> None:
    _check("awq_select_scale", LIB.awq_select_scale(
        _ptr(sse), int(T_total), abar.shape[0], int(out), _ptr(abar), ctypes.byref(cfg), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(s_best), _ptr(mse), _ptr(best_idx), _stream(stream)))


def awq_block_grams(X, cfg: AwqConfig, ws, G, stream=None) -> None:
    _check("awq_block_grams", LIB.awq_block_grams(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), ctypes.byref(cfg), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(G), _stream(stream)))


def awq_search_clip_grams(W, s, G, cfg: AwqConfig, ws, clip_idx, err=None, stream=None) -> None:
    _check("awq_search_clip_grams", LIB.awq_search_clip_grams(
        _ptr(W), W.shape[0], W.shape[1], _ptr(s), _ptr(G), ctypes.byref(cfg), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(clip_idx), _ptr(err), _stream(stream)))


def awq_candidate_codes(W, abar, cfg: AwqConfig, ws, q, z, delta, stream=None) -> None:
    """Codes q uint8 [n_alpha, out, in], zero points z uint8 and steps delta
    fp32 [n_alpha, out, in/g] of every candidate of the alpha search."""
    _check("awq_candidate_codes", LIB.awq_candidate_codes(
        _ptr(W), W.shape[0], W.shape[1], _ptr(abar), ctypes.byref(cfg), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(q), _ptr(z), _ptr(delta), _stream(stream)))


def awq_clip_candidate_codes(W, s, G, cfg: AwqConfig, ws, clip_idx, err, q, z, stream=None) -> None:
    """awq_search_clip_grams that also stores the clip candidates' codes q
    uint8 [out, n_clip, in] and zero points z uint8 [out, n_clip, in/128]."""
    _check("awq_clip_candidate_codes", LIB.awq_clip_candidate_codes(
        _ptr(W), W.shape[0], W.shape[1], _ptr(s), _ptr(G), ctypes.byref(cfg), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(clip_idx), _ptr(err), _ptr(q), _ptr(z),
        _stream(stream)))


def awq_w4a16_gemm(X, qweight, qzeros, scales, cfg: AwqConfig, Y, ws, stream=None) -> None:
    """Y [T, out] fp16 = X [T, in] times the packed weights, dequantised on the fly."""
    _check("awq_w4a16_gemm", LIB.awq_w4a16_gemm(
        _ptr(X), X.shape[0], X.shape[1], X.stride(0), _ptr(qweight), _ptr(qzeros), _ptr(scales),
        Y.shape[1], ctypes.byref(cfg), _ptr(Y), Y.stride(0), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def awq_w4a16_workspace_size(T: int, inn: int, out: int, cfg: AwqConfig) -> int:
    """Workspace bytes that let awq_w4a16_gemm split K for few tokens."""
    n = LIB.awq_w4a16_workspace_size(T, inn, out, ctypes.byref(cfg))
    if n == 0:
        raise AwqError("awq_w4a16_workspace_size", 1, last_error())
    return int(n)


def awq_device_status(ws, stream=None) -> None:
    """Raises AwqError if the device status in workspace ``ws`` records a
    failure; ws=None reads the library's own status word (the calls that take
    no workspace: awq_quant_pack, awq_search_clip_noalloc)."""
    _check("awq_device_status", LIB.awq_device_status(_ptr(ws), _stream(stream)))


def awq_bounds_checks_enabled() -> bool:
    """True in the debug library (index checks compiled into the kernels)."""
    return bool(LIB.awq_bounds_checks_enabled())


def awq_bounds_status() -> None:
    """Raises AwqError if a kernel index check failed since the last call
    (debug library); clears the record.  A no-op in the release library."""
    _check("awq_bounds_status", LIB.awq_bounds_status())


def profile_enable(on: bool) -> None:
    _check("awq_profile_enable", LIB.awq_profile_enable(1 if on else 0))


def profile_read(name: str):
    ms, n = c_double(0.0), c_int64(0)
    _check("awq_profile_read", LIB.awq_profile_read(name.encode(), ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def profile_reset() -> None:
    _check("awq_profile_reset", LIB.awq_profile_reset())
