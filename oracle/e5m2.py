"""ctypes binding of the oracle's E5M2 codec (oracle/e5m2.c). Test infrastructure only."""
import ctypes

import numpy as np

from .build import build

_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.arkv_oracle_e5m2_encode.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        _lib.arkv_oracle_e5m2_decode.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        _lib.arkv_oracle_e5m2_encode_bits_range.argtypes = [ctypes.c_uint32, ctypes.c_int64,
                                                            ctypes.c_void_p]
    return _lib


MAX = 57344.0


def encode(x) -> np.ndarray:
    """float32 values -> E5M2 codes (round to nearest even, saturate to +-57344)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().arkv_oracle_e5m2_encode(x.ctypes.data, out.ctypes.data, x.size)
    return out


def decode(c) -> np.ndarray:
    """E5M2 codes -> their exact values as float64 (+-inf for S.11111.00, NaN for S.11111.mm, mm != 0)."""
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().arkv_oracle_e5m2_decode(c.ctypes.data, out.ctypes.data, c.size)
    return out


def encode_bits_range(start: int, n: int) -> np.ndarray:
    """Codes of the float32 values with bit patterns start .. start+n-1."""
    out = np.empty(n, np.uint8)
    _load().arkv_oracle_e5m2_encode_bits_range(start, n, out.ctypes.data)
    return out
