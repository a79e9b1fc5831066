"""Pins of the oracle's E5M2 codec (the second FP8 format of the Quantization
tier): the format definition's values, torch's own float8_e5m2 conversion (an
independent library routine), and round trips."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import e5m2

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "e5m2_ocp_values.json")))


def test_decode_matches_format_definition():
    for code, val in GOLD["decode"]:
        got = e5m2.decode(np.array([int(code, 16)], np.uint8))[0]
        assert got == val and np.signbit(got) == np.signbit(val), code
    for code, sign in GOLD["inf_codes"]:
        assert e5m2.decode(np.array([int(code, 16)], np.uint8))[0] == sign * np.inf
    for code in GOLD["nan_codes"]:
        assert np.isnan(e5m2.decode(np.array([int(code, 16)], np.uint8))[0])


def test_decode_all_codes_match_torch():
    c = np.arange(256, dtype=np.uint8)
    ours = e5m2.decode(c)
    ref = torch.from_numpy(c.copy()).view(torch.float8_e5m2).double().numpy()
    assert ((ours == ref) | (np.isnan(ours) & np.isnan(ref))).all()
    assert (np.signbit(ours[~np.isnan(ours)]) == np.signbit(ref[~np.isnan(ref)])).all()


def test_encode_rne_and_saturation_cases():
    for x, code, why in GOLD["encode_rne"]:
        assert e5m2.encode(np.array([x], np.float32))[0] == int(code, 16), why
    assert e5m2.encode(np.array([np.inf], np.float32))[0] == 0x7B
    assert e5m2.encode(np.array([-np.inf], np.float32))[0] == 0xFB
    c = e5m2.encode(np.array([np.nan], np.float32))[0]
    assert (c & 0x7C) == 0x7C and (c & 0x03) != 0


def test_round_trip_every_finite_code():
    c = np.arange(256, dtype=np.uint8)
    v = e5m2.decode(c)
    fin = np.isfinite(v)
    back = e5m2.encode(v[fin].astype(np.float32))
    assert (back == c[fin]).all()


def _midpoints():
    v = np.unique(np.abs(e5m2.decode(np.arange(0, 0x7C, dtype=np.uint8))))
    mids = (v[:-1] + v[1:]) / 2
    eps = np.float32(1.0 + 2.0 ** -20)
    pts = np.concatenate([mids, mids * eps, mids / eps, v])
    return np.concatenate([pts, -pts]).astype(np.float32)


# torch's (non-saturating) cast sends values at or beyond the rounding boundary
# above 57344 (61440) to infinity; below it the two conversions must agree
_TORCH_OK = 61440.0


def test_encode_matches_torch_where_torch_does_not_saturate():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        _midpoints(),
        (rng.standard_normal(200_000) * 8000).astype(np.float32),
        (rng.standard_normal(200_000) * 1e-4).astype(np.float32),
        rng.integers(0, 2 ** 32, 400_000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ])
    x = x[np.isfinite(x) & (np.abs(x) < _TORCH_OK)]
    ours = e5m2.encode(x)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert (ours == ref).all()


def test_bits_range_matches_elementwise():
    start = 0x3F7F0000
    got = e5m2.encode_bits_range(start, 1 << 16)
    x = (np.arange(1 << 16, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
    assert (got == e5m2.encode(x)).all()


# float32 exponent fields of the binades the format spans: below its smallest
# subnormal (2^-17), its subnormals (2^-16, 2^-15), its smallest normal (2^-14), 1,
# and its top binades ([16384, 32768) and [32768, 65536), where 57344 saturates),
# plus the float32 subnormals
@pytest.mark.parametrize("exp_bits", [0x00, 0x6E, 0x6F, 0x70, 0x71, 0x7F, 0x8D, 0x8E])
def test_exhaustive_mantissa_sweep_against_torch(exp_bits):
    """Every float32 in selected binades (all 2^23 mantissas each), positive and negative."""
    for sign in (0, 1):
        start = (sign << 31) | (exp_bits << 23)
        codes = e5m2.encode_bits_range(start, 1 << 23)
        x = (np.arange(1 << 23, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
        ok = np.isfinite(x) & (np.abs(x) < _TORCH_OK)
        ref = torch.from_numpy(x[ok].copy()).to(torch.float8_e5m2).view(torch.uint8).numpy()
        assert (codes[ok] == ref).all()
        assert (codes[~ok & np.isfinite(x)] & 0x7F == 0x7B).all()
