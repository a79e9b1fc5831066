"""The C-ABI library loads, exports every entry point include/arkv.h declares, and
its host-only calls agree with the oracle; bad arguments are rejected before any
launch.  No CUDA device is touched."""
import ctypes
import os
import re

import numpy as np
import pytest

from mixed_precision_kv_arkv_b200 import abi, build
from oracle import arkv as A

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "arkv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.lib()


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(arkv_\w+)\s*\(", src, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_oq_ratio_matches_oracle(lib):
    rng = np.random.default_rng(0)
    for L in (1, 3, 28, 36):
        st = np.stack([rng.uniform(0, 1, L), rng.uniform(0, 5000, L), rng.uniform(-2, 3e4, L)], 1)
        out = np.zeros(L, np.float32)
        abi.arkv_oq_ratio(st.ctypes.data, L, 0.55, out.ctypes.data)
        np.testing.assert_allclose(out, A.oq_ratio(st, 0.55).astype(np.float32), rtol=2e-7)


def cfg(**kw):
    base = dict(batch=1, hq=8, hkv=2, head_dim=64, window=64, n_obs=64, gamma=1.0, budget_frac=0.25,
                cap_bf16=1000, cap_fp8=1000, quant_format=abi.ARKV_FMT_E4M3, early_start=0)
    base.update(kw)
    return abi.arkv_cfg(*[base[n] for n, _ in abi.arkv_cfg._fields_])


def test_row_capacity_matches_oracle_budget(lib):
    for D, W, n, r, beta, T in [(64, 64, 2064, 0.5, 0.25, 1), (128, 128, 32896, 0.55, 0.25, 16),
                                (128, 64, 16640, 0.3, 0.3, 16), (128, 256, 131136, 0.9, 0.25, 16)]:
        c = cfg(head_dim=D, window=W, budget_frac=beta)
        cap_o, cap_q = abi.arkv_row_capacity(c, n, r, T)
        n_sel, n_o = A.budget_counts(beta, n, r, D, W, 10 ** 9)
        assert (cap_o, cap_q) == (n_o + W + T, n_sel)


def test_workspace_sizes(lib):
    c = cfg()
    for which in (abi.ARKV_WS_DECODE, abi.ARKV_WS_REASSIGN):
        assert abi.arkv_workspace_bytes(c, which) > 0
    assert abi.arkv_workspace_bytes(c, abi.ARKV_WS_PREFILL, 2048) > 0
    assert abi.arkv_workspace_bytes(c, 99) == 0
    assert abi.arkv_workspace_bytes(cfg(head_dim=96), abi.ARKV_WS_DECODE) == 0


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(hq=7), dict(hq=16, hkv=2), dict(window=0),
                                 dict(budget_frac=0.0), dict(budget_frac=1.5), dict(gamma=-1.0),
                                 dict(cap_fp8=0), dict(quant_format=2), dict(quant_format=-1),
                                 dict(early_start=2), dict(early_start=-1)])
def test_bad_config_rejected_before_launch(lib, bad):
    c = cfg(**bad)
    dummy = ctypes.c_void_p(256)
    rc = abi.arkv_decode_attn(c, 0, dummy, dummy, dummy, dummy, abi.arkv_layer_cache(), dummy,
                              dummy, 1 << 20, None, check=False)
    assert rc == abi.ARKV_EINVAL
    assert abi.arkv_last_error_string()


def test_null_cache_buffers_and_small_workspace_rejected(lib):
    c = cfg()
    cache = abi.arkv_layer_cache(*[256 * (i + 1) for i in range(15)])
    p = 4096
    assert abi.arkv_decode_attn(c, 0, p, p, p, p, abi.arkv_layer_cache(), p, p, 1 << 30, None,
                                check=False) == abi.ARKV_EINVAL
    need = abi.arkv_workspace_bytes(c, abi.ARKV_WS_DECODE)
    assert abi.arkv_decode_attn(c, 0, p, p, p, p, cache, p, p, need - 1, None,
                                check=False) == abi.ARKV_EINVAL
    assert "workspace" in abi.arkv_last_error_string()
    assert abi.arkv_decode_attn(c, -1, p, p, p, p, cache, p, p, need, None,
                                check=False) == abi.ARKV_EINVAL
    assert abi.arkv_reassign(c, 0, 1.5, p, cache, None, p, 1 << 30, None,
                             check=False) == abi.ARKV_EINVAL
    # the attention output is written in 16-byte words
    assert abi.arkv_decode_attn(c, 0, p, p, p, p, cache, p + 4, p, need, None,
                                check=False) == abi.ARKV_EINVAL
    assert "aligned" in abi.arkv_last_error_string()
    # unknown FP8 format of the debug encoder
    assert abi.arkv_fp8_encode(7, p, p, 16, None, check=False) == abi.ARKV_EINVAL
    # capacities below the kept counts at the longest context are refused up front
    small = cfg(cap_bf16=10, cap_fp8=10)
    assert abi.arkv_quantize_pack(small, 0.5, p, p, 2048, p, p, p, cache, None, p, 1 << 30, None,
                                  check=False) == abi.ARKV_ECAPACITY


def test_copy_async_rejects_bad_arguments_before_any_launch(lib):
    """Alignment, size and overlap are checked on the host, before the pointers are
    even inspected (no GPU needed)."""
    a, b = ctypes.c_void_p(4096), ctypes.c_void_p(1 << 20)
    assert abi.arkv_copy_async(a, b, 0, None) == abi.ARKV_OK           # nothing to copy
    assert abi.arkv_copy_async(None, b, 16, None, check=False) == abi.ARKV_EINVAL
    assert abi.arkv_copy_async(a, b, 24, None, check=False) == abi.ARKV_EINVAL                # size % 16
    assert abi.arkv_copy_async(ctypes.c_void_p(4104), b, 32, None, check=False) == abi.ARKV_EINVAL   # dst % 16
    assert abi.arkv_copy_async(a, ctypes.c_void_p(4096 + 16), 64, None, check=False) == abi.ARKV_EINVAL  # overlap
    assert "arkv_copy_async" in abi.arkv_last_error_string()
