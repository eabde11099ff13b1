"""Pins of the oracle's number formats (bf16 decoding, E4M3 codec) against their definitions."""

import os

import numpy as np
import pytest
import torch

from oracle import formats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spec_points.txt")


def _golden_points():
    pts = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            val, code = line.split()[:2]
            pts.append((float(val), int(code, 16)))
    return pts


@pytest.mark.parametrize("value,code", _golden_points())
def test_e4m3_spec_points(value, code):
    got = int(formats.e4m3_encode(np.array([value], dtype=np.float32))[0])
    assert got == code, f"{value}: got {got:#04x}, want {code:#04x}"


def test_e4m3_decode_closed_form_every_code():
    codes = np.arange(256, dtype=np.uint8)
    dec = formats.e4m3_decode(codes)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            assert np.isnan(dec[c])
            continue
        want = s * (m / 8.0 * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
        assert dec[c] == want, c


def test_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    back = formats.e4m3_encode(formats.e4m3_decode(codes).astype(np.float32))
    assert np.array_equal(back, codes)


def test_e4m3_nearest_and_monotone():
    # every float32 maps to one of its two E4M3 neighbours, the nearer one
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-1, 1, 20000),
                        rng.uniform(-0.02, 0.02, 20000)]).astype(np.float32)
    got = formats.e4m3_decode(formats.e4m3_encode(x))
    finite = formats.e4m3_decode(np.array([c for c in range(128) if c != 0x7F], dtype=np.uint8))
    grid = np.unique(np.concatenate([finite, -finite]))
    idx = np.searchsorted(grid, x.astype(np.float64))
    lo = grid[np.clip(idx - 1, 0, len(grid) - 1)]
    hi = grid[np.clip(idx, 0, len(grid) - 1)]
    err = np.abs(got - x)
    assert np.all(err <= np.minimum(np.abs(x - lo), np.abs(hi - x)) + 0.0)
    xs = np.sort(x)
    assert np.all(np.diff(formats.e4m3_decode(formats.e4m3_encode(xs))) >= 0)


def test_e4m3_matches_torch_cast_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(50000) * 50, rng.standard_normal(50000) * 1e-2,
                        rng.uniform(-448, 448, 50000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(formats.e4m3_encode(x), ref)


def test_bf16_decode():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x7F7F, 0x0001], dtype=np.uint16)
    want = np.array([1.0, -2.0, 0.0, float(np.float32(3.3895314e38)), 2.0 ** -133])
    got = formats.bf16_to_f64(bits)
    assert np.allclose(got[:3], want[:3], rtol=0, atol=0)
    assert got[3] == np.float64(np.array([0x7F7F0000], dtype=np.uint32).view(np.float32)[0])
    assert got[4] == 2.0 ** -133
