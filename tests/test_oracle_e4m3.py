"""Pins of the oracle's e4m3 codec against torch.float8_e4m3fn (a library
routine): exhaustive decode, round trip of every finite code, and encode of
in-range values including ties and subnormals."""
import math

import numpy as np
import torch

from oracle import e4m3 as e4


def _torch_decode_all():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_all_codes_match_torch():
    ref = _torch_decode_all()
    ours = e4.decode(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_roundtrip_every_finite_code():
    vals = e4.decode(np.arange(256, dtype=np.uint8))
    for c in range(256):
        if math.isnan(vals[c]):
            continue
        if c == 0x80:  # -0 keeps its sign
            assert e4.encode_scalar(-0.0) == 0x80
            continue
        assert e4.encode_scalar(vals[c]) == c
        assert int(e4.encode(np.array([vals[c]]))[0]) == c


def test_encode_matches_torch_in_range():
    r = np.random.default_rng(5)
    v = np.concatenate([
        r.standard_normal(20000) * 100.0,
        r.standard_normal(20000) * 1e-2,
        r.uniform(-2.0 ** -6, 2.0 ** -6, 20000),
        # exact midpoints between neighbouring codes (ties to even)
        (e4.decode(np.arange(0, 0x7D, dtype=np.uint8)) + e4.decode(np.arange(1, 0x7E, dtype=np.uint8))) / 2,
    ])
    v = v[np.abs(v) < 464.0]  # beyond this torch rounds to NaN; we saturate (tested below)
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = e4.encode(v32.astype(np.float64))
    assert np.array_equal(ours, ref)
    scalar = np.array([e4.encode_scalar(float(t)) for t in v32[:3000]], dtype=np.uint8)
    assert np.array_equal(scalar, ref[:3000])


def test_saturation_and_nan():
    for v in (448.0, 463.9, 464.0, 500.0, 1e30):
        assert e4.encode_scalar(v) == 0x7E and e4.encode_scalar(-v) == 0xFE
    assert np.array_equal(e4.encode(np.array([1e30, -1e30, 470.0])), np.array([0x7E, 0xFE, 0x7E], np.uint8))
    assert e4.encode_scalar(float("nan")) & 0x7F == 0x7F
    assert int(e4.encode(np.array([np.nan]))[0]) & 0x7F == 0x7F
