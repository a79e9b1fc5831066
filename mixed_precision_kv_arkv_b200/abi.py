"""Python binding of libarkv (include/arkv.h): ctypes marshalling only.

Every function here has the name of the C entry point it calls and passes its
arguments through unchanged; all computation happens in the CUDA library.  The
library must have been built (`python -m mixed_precision_kv_arkv_b200.build`);
loading fails loudly otherwise -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libarkv.so")

ARKV_OK, ARKV_EINVAL, ARKV_ECAPACITY, ARKV_ECUDA = 0, -1, -2, -3
ARKV_STATUS_BF16_FULL, ARKV_STATUS_FP8_FULL = 1, 2
ARKV_TIER_ORIGINAL, ARKV_TIER_QUANTIZED, ARKV_TIER_EVICTED = 0, 1, 2
ARKV_WS_DECODE, ARKV_WS_REASSIGN, ARKV_WS_PREFILL = 0, 1, 2
ARKV_FMT_E4M3, ARKV_FMT_E5M2 = 0, 1
FORMATS = {"e4m3": ARKV_FMT_E4M3, "e5m2": ARKV_FMT_E5M2}
ARKV_NOALLOC_SCRATCH_BYTES = 24 << 20


class arkv_cfg(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("window", ctypes.c_int32), ("n_obs", ctypes.c_int32),
                ("gamma", ctypes.c_float), ("budget_frac", ctypes.c_float),
                ("cap_bf16", ctypes.c_int32), ("cap_fp8", ctypes.c_int32),
                ("quant_format", ctypes.c_int32),
                ("early_start", ctypes.c_int32)]


class arkv_layer_cache(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("k16", "v16", "pos16", "mu16", "m2_16", "k8", "v8", "sk", "sv", "pos8", "mu8",
                 "m2_8", "n_bf16", "n_fp8", "status")]


class ArkvError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} returned {code}: {msg}")
        self.code = code


_P = ctypes.c_void_p
_SIG = {
    "arkv_workspace_bytes": (ctypes.c_size_t, [_P, ctypes.c_int, ctypes.c_int32]),
    "arkv_row_capacity": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_float, ctypes.c_int32, _P, _P]),
    "arkv_prefill_stats": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "arkv_oq_ratio": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_double, _P]),
    "arkv_quantize_pack": (ctypes.c_int, [_P, ctypes.c_float, _P, _P, ctypes.c_int32, _P, _P, _P, _P,
                                          _P, _P, ctypes.c_size_t, _P]),
    "arkv_decode_attn": (ctypes.c_int, [_P, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "arkv_score_update": (ctypes.c_int, [_P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]),
    "arkv_reassign": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_float, _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "arkv_fp8_encode": (ctypes.c_int, [ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "arkv_copy_async": (ctypes.c_int, [_P, _P, ctypes.c_size_t, _P]),
    "arkv_reassign_noalloc": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_float, _P, _P, _P, _P]),
    "arkv_last_error_string": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libarkv (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libarkv.so is not built at {LIB_PATH}; run "
                              "`python -m mixed_precision_kv_arkv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _ref(x):
    return ctypes.byref(x) if x is not None else None


def _check(fn: str, rc: int) -> int:
    if rc != ARKV_OK:
        raise ArkvError(fn, rc, lib().arkv_last_error_string().decode())
    return rc


def arkv_last_error_string() -> str:
    return lib().arkv_last_error_string().decode()


def arkv_workspace_bytes(cfg: arkv_cfg, which: int, n_ctx_max: int = 0) -> int:
    return lib().arkv_workspace_bytes(_ref(cfg), which, n_ctx_max)


def arkv_row_capacity(cfg: arkv_cfg, n_ctx_max: int, r: float, reassign_interval: int):
    a, b = ctypes.c_int32(), ctypes.c_int32()
    _check("arkv_row_capacity", lib().arkv_row_capacity(_ref(cfg), n_ctx_max, r, reassign_interval,
                                                        ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def arkv_oq_ratio(stats_ptr: int, layers: int, r_bar: float, r_out_ptr: int, check=True) -> int:
    rc = lib().arkv_oq_ratio(stats_ptr, layers, r_bar, r_out_ptr)
    return _check("arkv_oq_ratio", rc) if check else rc


def arkv_prefill_stats(cfg, q_obs, k, n_ctx_max, ctx_len, stats_out, query_stats, mu0, m2_0, ws,
                       ws_bytes, stream, check=True) -> int:
    rc = lib().arkv_prefill_stats(_ref(cfg), q_obs, k, n_ctx_max, ctx_len, stats_out, query_stats,
                                  mu0, m2_0, ws, ws_bytes, stream)
    return _check("arkv_prefill_stats", rc) if check else rc


def arkv_quantize_pack(cfg, r, k, v, n_ctx_max, ctx_len, mu0, m2_0, cache, tier_out, ws, ws_bytes,
                       stream, check=True) -> int:
    rc = lib().arkv_quantize_pack(_ref(cfg), r, k, v, n_ctx_max, ctx_len, mu0, m2_0, _ref(cache),
                                  tier_out, ws, ws_bytes, stream)
    return _check("arkv_quantize_pack", rc) if check else rc


def arkv_decode_attn(cfg, step, q, k_new, v_new, ctx_len, cache, o, ws, ws_bytes, stream,
                     check=True) -> int:
    rc = lib().arkv_decode_attn(_ref(cfg), step, q, k_new, v_new, ctx_len, _ref(cache), o, ws,
                                ws_bytes, stream)
    return _check("arkv_decode_attn", rc) if check else rc


def arkv_score_update(cfg, step, ctx_len, cache, ws, ws_bytes, stream, check=True) -> int:
    rc = lib().arkv_score_update(_ref(cfg), step, ctx_len, _ref(cache), ws, ws_bytes, stream)
    return _check("arkv_score_update", rc) if check else rc


def arkv_reassign(cfg, step, r, ctx_len, cache, tier_dbg, ws, ws_bytes, stream, check=True) -> int:
    rc = lib().arkv_reassign(_ref(cfg), step, r, ctx_len, _ref(cache), tier_dbg, ws, ws_bytes, stream)
    return _check("arkv_reassign", rc) if check else rc


def arkv_reassign_noalloc(cfg, step, r, ctx_len, cache, tier_dbg, stream, check=True) -> int:
    """arkv_reassign without a workspace (scratch in the library's static device array)."""
    rc = lib().arkv_reassign_noalloc(_ref(cfg), step, r, ctx_len, _ref(cache), tier_dbg, stream)
    return _check("arkv_reassign_noalloc", rc) if check else rc


def arkv_copy_async(dst, src, nbytes, stream, check=True) -> int:
    rc = lib().arkv_copy_async(dst, src, nbytes, stream)
    return _check("arkv_copy_async", rc) if check else rc


def arkv_fp8_encode(fmt, x, out, n, stream, check=True) -> int:
    rc = lib().arkv_fp8_encode(fmt, x, out, n, stream)
    return _check("arkv_fp8_encode", rc) if check else rc
