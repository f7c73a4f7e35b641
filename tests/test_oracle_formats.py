"""Pins of the oracle's scalar format functions against definitions and
library routines that do not share its code (CPU only).

- e4m3 decode: all 256 bytes against torch.float8_e4m3fn.
- e4m3 encode: a dense sweep against torch's float -> float8_e4m3fn cast
  (round to nearest even), inside the finite range where torch agrees with
  the saturating rule; saturation beyond it.
- e2m1 encode: a dense sweep against a second, independent rounding routine
  (quantum + rint, itself pinned against torch / numpy below).
- e8m0 round-up: the defining inequalities 2^(b-128) < v <= 2^(b-127).
- rounding to bf16 / fp16: against torch and numpy conversions.
"""
import math
import struct

import numpy as np
import pytest
import torch


def f32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def all_bf16_as_f32():
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[np.isfinite(v)]


def test_e4m3_decode_all_bytes_match_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        v = orc.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(v), b
        else:
            assert v == ref[b], (b, v, ref[b])


def test_format_maxima_are_the_pages_constants(orc):
    # fp_quantize.cu ("mlx 0.30.7.2 -> 0.30.7.6", page 7): F8E4M3_MAX = 448,
    # F4E2M1_MAX = 6, and the encode constant 448 * 6 = 2688.
    e2 = [orc.e2m1_value(c) for c in range(16)]
    e4 = [orc.e4m3_value(b) for b in range(256)]
    assert max(e2) == 6.0 and min(e2) == -6.0
    assert max(v for v in e4 if not math.isnan(v)) == 448.0
    assert sum(math.isnan(v) for v in e4) == 2  # 0x7F and 0xFF only
    # e2m1: 16 codes, 15 distinct values (+0 and -0), sign in bit 3
    assert len({v for v in e2}) == 15
    for c in range(8):
        assert e2[c | 8] == -e2[c]


def test_e8m0_decode_is_power_of_two(orc):
    for b in range(255):
        assert orc.e8m0_value(b) == math.ldexp(1.0, b - 127)
    assert math.isnan(orc.e8m0_value(255))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_encode_decode_round_trip_every_code(orc, fmt):
    """decode(encode(decode(c))) == decode(c) for every non-NaN code."""
    n, dec, enc = (16, orc.e2m1_value, orc.e2m1_encode) if fmt == "e2m1" else \
                  (256, orc.e4m3_value, orc.e4m3_encode)
    for c in range(n):
        v = dec(c)
        if math.isnan(v):
            continue
        assert dec(enc(v)) == v
        assert math.copysign(1.0, dec(enc(v))) == math.copysign(1.0, v)


def _e4m3_sweep():
    vals = [v for v in all_bf16_as_f32() if abs(v) <= 464.0]
    finite = sorted({orc_v for orc_v in
                     torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
                     .to(torch.float64).numpy() if np.isfinite(orc_v)})
    for a, b in zip(finite[:-1], finite[1:]):
        m = np.float32((a + b) / 2)  # midpoints are exact in fp32
        vals += [m, np.nextafter(m, np.float32(-np.inf)), np.nextafter(m, np.float32(np.inf))]
    return np.array(vals, dtype=np.float32)


def test_e4m3_encode_matches_torch_cast(orc):
    vals = _e4m3_sweep()
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(got[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_encode_saturates(orc):
    for v in [464.0001, 480.0, 1e6, 3e38, float("inf")]:
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE
    # below half the smallest subnormal (2^-10) -> 0; exactly 2^-10 ties to 0
    assert orc.e4m3_encode(2.0 ** -10) == 0
    assert orc.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 1


def _e2m1_by_quantum_rounding(orc, v):
    r = orc.round_to_format(float(v), 2, 0, 6.0)  # 2 significand bits, emin 0
    if math.isinf(r):
        r = math.copysign(6.0, r)
    return r


def test_e2m1_encode_matches_independent_rounding(orc):
    vals = [v for v in all_bf16_as_f32() if abs(v) <= 16.0]
    grid = [0, .5, 1, 1.5, 2, 3, 4, 6]
    for a, b in zip(grid[:-1], grid[1:]):
        m = np.float32((a + b) / 2)
        vals += [m, np.nextafter(m, np.float32(-1)), np.nextafter(m, np.float32(7))]
        vals += [-m, -np.nextafter(m, np.float32(-1)), -np.nextafter(m, np.float32(7))]
    vals += [np.float32(100.0), np.float32(-1e30)]
    for v in vals:
        got = orc.e2m1_value(orc.e2m1_encode(float(v)))
        want = _e2m1_by_quantum_rounding(orc, v)
        assert got == want, (float(v), got, want)


def test_e2m1_ties_and_signs(orc):
    # Midpoints round to the neighbour with an even code (mantissa bit 0).
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert orc.e2m1_value(orc.e2m1_encode(v)) == want
        assert orc.e2m1_value(orc.e2m1_encode(-v)) == -want
    assert orc.e2m1_encode(float("inf")) == 0x7
    assert orc.e2m1_encode(-float("inf")) == 0xF
    # sign-preserving zero: a negative value that rounds to 0 gives code 0x8
    assert orc.e2m1_encode(-0.1) == 0x8
    assert orc.e2m1_encode(-0.0) == 0x8
    assert orc.e2m1_encode(0.0) == 0x0


def test_e8m0_ceil_defining_inequalities(orc):
    rng = np.random.default_rng(0)
    exps = rng.uniform(-140, 130, size=4000)
    with np.errstate(over="ignore"):  # draws above 2^128 become inf and are skipped below
        vals = np.float32(np.exp2(exps))
    vals = np.concatenate([vals, np.float32(np.exp2(np.arange(-126, 128)))])
    for v in vals:
        v = float(v)
        if not (v > 0) or math.isinf(v):
            continue
        b = orc.e8m0_encode_ceil(v)
        assert 0 <= b <= 254
        if v <= 2.0 ** 127:
            assert math.ldexp(1.0, b - 127) >= v, (v, b)
        else:
            assert b == 254
        if b > 0:
            assert math.ldexp(1.0, b - 128) < v, (v, b)
    assert orc.e8m0_encode_ceil(0.0) == 0
    assert orc.e8m0_encode_ceil(1.0) == 127
    assert orc.e8m0_encode_ceil(f32(1.0000001)) == 128


def test_round_to_bf16_matches_torch(orc):
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        np.float32(np.exp2(rng.uniform(-140, 127, 5000))),
        np.array([3.3895314e38, 3.39e38, 1e-45, -1e-44, 0.0, -0.0], dtype=np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.uint16).numpy()
    got = orc.round_to(v.astype(np.float64), "bf16")
    assert np.array_equal(got, want)


def test_round_to_f16_matches_numpy(orc):
    rng = np.random.default_rng(2)
    v = np.concatenate([
        rng.standard_normal(20000) * 1e3,
        np.exp2(rng.uniform(-26, 16.1, 5000)),
        np.array([65504.0, 65519.99, 65520.0, 2.0 ** -25, 2.0 ** -24 * 1.5, -0.0]),
    ])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16)
    got = orc.round_to(v, "f16")
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_round_to_f32_is_ieee_cast(orc):
    rng = np.random.default_rng(3)
    v = rng.standard_normal(10000) * 1e5
    assert np.array_equal(orc.round_to(v, "f32"), v.astype(np.float32))


def test_load_of_each_type_is_exact(orc):
    rng = np.random.default_rng(4)
    x = rng.standard_normal(1000).astype(np.float32)
    assert np.array_equal(orc.to_f64(x, "f32"), x.astype(np.float64))
    h = x.astype(np.float16)
    assert np.array_equal(orc.to_f64(h, "f16"), h.astype(np.float64))
    b = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(orc.to_f64(b.view(torch.uint16).numpy(), "bf16"),
                          b.to(torch.float64).numpy())
