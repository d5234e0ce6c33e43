"""Pins for the oracle's number formats (CPU only).

The E4M3 and E2M1 rounders are checked against (a) hand-derived encodings
from the format definitions (tests/golden), (b) brute-force nearest-value
search over every finite code with ties to the even mantissa, and (c) the
independent casts of the ml_dtypes library.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import gift_oracle as O


def _read_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            v, c = line.split()[:2]
            rows.append((float(v), int(c, 16)))
    return rows


def test_e4m3_hand_values(golden_dir):
    rows = _read_golden(os.path.join(golden_dir, "e4m3_hand_values.txt"))
    assert len(rows) >= 20
    vals = np.array([v for v, _ in rows])
    want = np.array([c for _, c in rows], dtype=np.uint8)
    got = O.e4m3_encode(vals)
    assert np.array_equal(got, want), list(zip(vals, got, want))


def test_e2m1_hand_values(golden_dir):
    rows = _read_golden(os.path.join(golden_dir, "e2m1_hand_values.txt"))
    vals = np.array([v for v, _ in rows])
    want = np.array([c for _, c in rows], dtype=np.uint8)
    got = O.e2m1_encode(vals)
    assert np.array_equal(got, want), list(zip(vals, got, want))


def test_e4m3_decode_all_codes_vs_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], lib[~nan])
    assert np.nanmax(ours) == 448.0
    assert ours[1] == 2.0 ** -9


def test_e2m1_decode_all_codes_vs_library():
    codes = np.arange(16, dtype=np.uint8)
    ours = O.e2m1_decode(codes)
    # ml_dtypes stores float4 one per byte in the low nibble
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, lib)


def _brute_force_nearest(x, table_vals, table_codes, mant_bits):
    """Nearest finite value; ties broken toward the even mantissa (code LSB 0)."""
    out = np.empty(x.shape, dtype=np.uint8)
    for i, xi in enumerate(x):
        d = np.abs(table_vals - xi)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            even = [b for b in best if (table_codes[b] & 1) == 0]
            b = even[0]
        else:
            b = best[0]
        out[i] = table_codes[b]
    return out


def test_e4m3_encode_brute_force():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    pos = (codes < 0x80) & ~np.isnan(vals)
    tv, tc = vals[pos], codes[pos]
    rng = np.random.default_rng(7)
    # random magnitudes over the whole range, every midpoint, and values just off midpoints
    x = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 4000)),
        rng.uniform(0, 2.0 ** -6, 500),
    ])
    tvs = np.sort(tv)
    mids = 0.5 * (tvs[1:] + tvs[:-1])
    x = np.concatenate([x, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9)])
    x = x[x <= 448.0]
    want = _brute_force_nearest(x, tv, tc, 3)
    assert np.array_equal(O.e4m3_encode(x), want)
    assert np.array_equal(O.e4m3_encode(-x), want | 0x80)


def test_e4m3_encode_vs_library_cast():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-8, 5, 200000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    lib = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ours = O.e4m3_encode(x)
    assert np.array_equal(ours, lib)
    # torch's cast is a second independent implementation
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, t)


def test_e4m3_saturation_and_signed_zero():
    x = np.array([448.0, 449.0, 463.999, 464.0, 500.0, 1e30, -1e30, -0.0, 0.0, -1e-30])
    got = O.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x00, 0x80]


def test_e2m1_encode_brute_force():
    codes = np.arange(8, dtype=np.uint8)
    tv = O.e2m1_decode(codes)
    x = np.concatenate([np.linspace(0, 6, 6001), 0.5 * (tv[1:] + tv[:-1])])
    want = _brute_force_nearest(x, tv, codes, 1)
    assert np.array_equal(O.e2m1_encode(x), want)
    assert np.array_equal(O.e2m1_encode(-x[x > 0]), want[x > 0] | 0x8)


def test_e2m1_encode_vs_library_cast():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(50000) * 2.5).astype(np.float32)
    x = x[np.abs(x) <= 6]
    lib = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(O.e2m1_encode(x), lib)


def test_bf16_round_vs_torch():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(3.7)
    ours = O.bf16_round(x)
    t = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours, t)
