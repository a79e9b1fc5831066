"""Pins of the oracle's E4M3 codec: the format definition's values, torch's own
float8_e4m3fn conversion (an independent library routine), and round trips."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import e4m3

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_values.json")))


def test_decode_matches_format_definition():
    for code, val in GOLD["decode"]:
        got = e4m3.decode(np.array([int(code, 16)], np.uint8))[0]
        assert got == val and np.signbit(got) == np.signbit(val), code
    for code in GOLD["nan_codes"]:
        assert np.isnan(e4m3.decode(np.array([int(code, 16)], np.uint8))[0])


def test_decode_all_codes_match_torch():
    c = np.arange(256, dtype=np.uint8)
    ours = e4m3.decode(c)
    ref = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()
    assert (np.signbit(ours[~np.isnan(ours)]) == np.signbit(ref[~np.isnan(ref)])).all()


def test_encode_rne_and_saturation_cases():
    for x, code, why in GOLD["encode_rne"]:
        assert e4m3.encode(np.array([x], np.float32))[0] == int(code, 16), why
    assert e4m3.encode(np.array([np.inf], np.float32))[0] == 0x7E
    assert e4m3.encode(np.array([-np.inf], np.float32))[0] == 0xFE
    assert e4m3.encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_round_trip_every_finite_code():
    c = np.arange(256, dtype=np.uint8)
    v = e4m3.decode(c)
    fin = ~np.isnan(v)
    back = e4m3.encode(v[fin].astype(np.float32))
    assert (back == c[fin]).all()


def _midpoints():
    v = np.unique(np.abs(e4m3.decode(np.arange(0, 0x7F, dtype=np.uint8))))
    mids = (v[:-1] + v[1:]) / 2
    eps = np.float32(1.0 + 2.0 ** -20)
    pts = np.concatenate([mids, mids * eps, mids / eps, v])
    return np.concatenate([pts, -pts]).astype(np.float32)


def test_encode_matches_torch_where_torch_does_not_saturate():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        _midpoints(),
        (rng.standard_normal(200_000) * 60).astype(np.float32),
        (rng.standard_normal(200_000) * 0.01).astype(np.float32),
        rng.integers(0, 2 ** 32, 400_000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ])
    x = x[np.isfinite(x) & (np.abs(x) < 464)]   # torch maps |x| >= 464 to NaN, not 448
    ours = e4m3.encode(x)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (ours == ref).all()


def test_bits_range_matches_elementwise():
    start = 0x3F7F0000
    got = e4m3.encode_bits_range(start, 1 << 16)
    x = (np.arange(1 << 16, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
    assert (got == e4m3.encode(x)).all()


# float32 exponent fields of the binades the format spans: below its smallest
# subnormal (2^-10), its subnormals (2^-9 .. 2^-7), its smallest normal (2^-6), 1,
# and its top binades ([128, 256) and [256, 512), where 448 saturates), plus the
# float32 subnormals
@pytest.mark.parametrize("exp_bits", [0x00, 0x75, 0x76, 0x77, 0x78, 0x79, 0x7F, 0x86, 0x87])
def test_exhaustive_mantissa_sweep_against_torch(exp_bits):
    """Every float32 in selected binades (all 2^23 mantissas each), positive and negative."""
    for sign in (0, 1):
        start = (sign << 31) | (exp_bits << 23)
        codes = e4m3.encode_bits_range(start, 1 << 23)
        x = (np.arange(1 << 23, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
        ok = np.isfinite(x) & (np.abs(x) < 464)
        ref = torch.from_numpy(x[ok].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert (codes[ok] == ref).all()
        assert (codes[~ok & np.isfinite(x)] & 0x7F == 0x7E).all()
