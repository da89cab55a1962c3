"""Pins of the oracle's E4M3 codec against things other than itself.

- torch.float8_e4m3fn (an independent library implementation of the same OCP
  format; its cast rounds to nearest even but does not saturate, so inputs
  are clamped to +-448 first),
- the published constants of the format (tests/golden/e4m3_points.txt),
- exact properties: round trip of every finite code, monotonicity, sign
  symmetry.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def torch_encode(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = torch.clamp(t, -448.0, 448.0)  # saturating reading; NaN passes through clamp
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_all_256_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros
    assert math.copysign(1.0, ours[0x80]) == -1.0 and ours[0x00] == 0.0


def test_decode_range_constants():
    v = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = v[np.isfinite(v)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert np.min(np.abs(finite[finite != 0])) == 2.0 ** -9
    assert np.isinf(v).sum() == 0


def test_golden_points():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((float(a), int(b, 16)))
    x = np.array([r[0] for r in rows], dtype=np.float32)
    want = np.array([r[1] for r in rows], dtype=np.uint8)
    got = oracle.e4m3_encode(x)
    bad = [(float(x[i]), hex(want[i]), hex(got[i])) for i in range(len(rows)) if got[i] != want[i]]
    assert not bad, bad


def test_nan_encodes_to_canonical_nan():
    x = np.array([np.nan, -np.nan], dtype=np.float32)
    assert oracle.e4m3_encode(x).tolist() == [0x7F, 0x7F]


def test_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)  # exact in float32
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_encode_all_bf16_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    ours = oracle.e4m3_encode(x)
    ref = torch_encode(x)
    nan = np.isnan(x)
    assert np.all(ours[nan] == 0x7F)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_encode_near_every_midpoint_matches_torch():
    """Every tie between adjacent codes, and the floats 1..8 ulps either side."""
    pos = np.array(sorted(set(oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).tolist())))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)  # exact in float32
    mids = np.concatenate([mids, np.float32([464.0, 2.0 ** -10])])
    offs = np.arange(-8, 9, dtype=np.int64)
    b = mids.view(np.uint32).astype(np.int64)[:, None] + offs[None, :]
    x = np.concatenate([b.ravel()]).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, -x])
    assert np.array_equal(oracle.e4m3_encode(x), torch_encode(x))


def test_encode_random_float_patterns_match_torch():
    r = np.random.default_rng(12345)
    bits = r.integers(0, 2**32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    keep = ~np.isnan(x)
    x = x[keep]
    assert np.array_equal(oracle.e4m3_encode(x), torch_encode(x))
    # magnitudes where the grid is dense
    y = (r.standard_normal(1 << 20) * np.exp2(r.uniform(-12, 10, 1 << 20))).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(y), torch_encode(y))


def test_encode_bits_range_equals_elementwise():
    start = 0x3F7FFF00
    a = oracle.e4m3_encode_bits_range(start, 4096)
    x = (np.arange(4096, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
    assert np.array_equal(a, oracle.e4m3_encode(x))


def test_encode_monotone_and_sign_symmetric():
    x = np.linspace(0, 500, 200001, dtype=np.float32)
    c = oracle.e4m3_encode(x)
    v = oracle.e4m3_decode(c)
    assert np.all(np.diff(v) >= 0)
    assert np.array_equal(oracle.e4m3_encode(-x[1:]), c[1:] | 0x80)


def test_scale_from_amax():
    assert oracle.scale_from_amax(0.0) == 1.0
    assert oracle.scale_from_amax(448.0) == 1.0
    # the amax element always lands on the largest code
    r = np.random.default_rng(7)
    for amax in np.abs(r.standard_normal(2000)).astype(np.float32) * 10 + 1e-3:
        s = np.float32(oracle.scale_from_amax(float(amax)))
        assert s == np.float32(amax) / np.float32(448.0)
        code = oracle.e4m3_encode(np.array([np.float32(amax) / s], dtype=np.float32))[0]
        assert code == 0x7E, (amax, s, hex(code))
