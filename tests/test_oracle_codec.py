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


QUANT_SCALES = [3.7 / 448, 0.0123, 2.0 ** -6, 3.0e-11, 7.5e8, 2.0 ** -50]


@pytest.mark.parametrize("scale", QUANT_SCALES)
def test_quantize_bits_range_matches_ieee_quotient_and_torch_cast(scale):
    """The quantize step (reading R3: code = E4M3 of the IEEE binary32
    quotient x / s) against numpy's float32 division and torch's E4M3 cast,
    on a strided sample of all 2^32 float bit patterns plus random ones.
    The scales are the ones the exhaustive device check uses."""
    s = np.float32(scale)
    stride = (1 << 12) + 1                       # ~1M patterns spread over the whole range
    start = 0x1234
    count = (1 << 32) // stride
    got = oracle.e4m3_quantize_bits_range(start, count, float(s))
    x = ((np.arange(count, dtype=np.uint64) * 1 + start).astype(np.uint32)).view(np.float32)
    # the oracle function takes consecutive patterns: compare on that block, then
    # on a strided sample through e4m3_encode of numpy's quotient
    with np.errstate(all="ignore"):
        qd = x / s
    nan = np.isnan(qd)
    assert np.all(got[nan] == 0x7F)
    assert np.array_equal(got[~nan], torch_encode(qd[~nan]))
    bits = (np.arange(count, dtype=np.uint64) * stride + 7).astype(np.uint32)
    xs = bits.view(np.float32)
    r = np.random.default_rng(int(s.view(np.uint32)))
    xs = np.concatenate([xs, r.integers(0, 2**32, 1 << 18, dtype=np.uint64).astype(np.uint32)
                         .view(np.float32)])
    with np.errstate(all="ignore"):
        qs = xs / s
        prod = xs * (np.float32(1.0) / s)
    want = np.where(np.isnan(qs), np.uint8(0x7F), 0).astype(np.uint8)
    fin = ~np.isnan(qs)
    want[fin] = torch_encode(qs[fin])
    got_s = np.array([oracle.e4m3_quantize_bits_range(int(b), 1, float(s))[0] for b in
                      xs.view(np.uint32)[:: 257]], np.uint8)
    assert np.array_equal(got_s, want[:: 257])


@pytest.mark.parametrize("scale", QUANT_SCALES)
def test_quantize_bits_range_near_code_midpoints(scale):
    """Inputs whose quotient x / s lies within a few float ulps of a tie
    between two E4M3 codes, where x / s and the product x * (1/s) can round
    to different codes: the oracle must give the codes of the quotient."""
    s = np.float32(scale)
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    pos = np.array(sorted(set(pos.tolist())))
    mids = (pos[:-1] + pos[1:]) / 2
    with np.errstate(all="ignore"):
        centre = (mids * np.float64(s)).astype(np.float32)
    offs = np.arange(-6, 7, dtype=np.int64)
    b = centre.view(np.uint32).astype(np.int64)[:, None] + offs[None, :]
    x = b.ravel().astype(np.uint32).view(np.float32)
    x = np.concatenate([x, -x])
    got = np.array([oracle.e4m3_quantize_bits_range(int(v), 1, float(s))[0]
                    for v in x.view(np.uint32)], np.uint8)
    with np.errstate(all="ignore"):
        q = x / s
        prod = x * (np.float32(1.0) / s)
    want = torch_encode(q)
    assert np.array_equal(got, want)
    # negative control: for amax/448-like scales the product by the rounded
    # reciprocal lands on the other side of some of these ties, so this
    # sample tells the quotient from the product
    if scale in QUANT_SCALES[:2]:
        fin = np.isfinite(prod)
        assert not np.array_equal(torch_encode(prod[fin]), want[fin])


def test_quantize_bits_range_consecutive_block_is_elementwise_quotient():
    """A consecutive block across the normal/subnormal boundary of the quotient."""
    s = np.float32(3.7 / 448)
    start = 0x00700000
    got = oracle.e4m3_quantize_bits_range(start, 1 << 20, float(s))
    x = (np.arange(1 << 20, dtype=np.uint64) + start).astype(np.uint32).view(np.float32)
    with np.errstate(all="ignore"):
        q = x / s
    assert np.array_equal(got, torch_encode(q))
