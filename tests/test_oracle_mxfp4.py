"""Pins of the oracle's MXFP4 functions (4-bit e2m1 codes with the mx e8m0
scale, 32-element blocks) against hand-derived blocks, closed forms and brute
force (CPU only).

Source: "mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, fp_quantize.cu
(fp_quantize_rowwise / fp_quantize_dequantize with bits = 4 and the mx
scale), and the E8M0 round-up recorded on the "[Metal] global scale for qmm"
page.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _codes(words, K):
    w = np.asarray(words, dtype=np.uint32).reshape(-1)
    return np.array([(int(w[i // 8]) >> (4 * (i % 8))) & 15 for i in range(K)])


def _golden_blocks():
    out = []
    for line in open(os.path.join(GOLDEN, "mxfp4_blocks.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        out.append((f[0], [float(v) for v in f[1:5]], int(f[5]), [int(v) for v in f[6:10]]))
    return out


@pytest.mark.parametrize("name,x4,s,c4", _golden_blocks())
def test_mxfp4_hand_derived_blocks(orc, name, x4, s, c4):
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, :4] = x4
    codes, scales = orc.mxfp4_quantize(x, "f32")
    assert int(scales[0, 0]) == s, name
    assert list(_codes(codes, 32)[:4]) == c4, name
    assert not _codes(codes, 32)[4:].any()


def _brute_code(t):
    """Nearest e2m1 code to t by exhaustive search, ties to the even code,
    magnitudes above 6 saturated."""
    mag = min(abs(t), 6.0)
    best = min(range(8), key=lambda c: (abs(E2M1[c] - mag), c & 1))
    return best | (8 if t < 0 and best != 0 else 0) if best != 0 else (8 if np.signbit(t) else 0)


def test_mxfp4_scale_is_smallest_power_of_two_covering_max_over_6(orc):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((16, 256)) * np.exp2(rng.integers(-20, 20, (16, 1)))).astype(np.float32)
    codes, scales = orc.mxfp4_quantize(x, "f32")
    for r in range(16):
        for b in range(8):
            v = np.float32(np.abs(x[r, 32 * b:32 * b + 32]).max()) / np.float32(6.0)
            p = 2.0 ** (int(scales[r, b]) - 127)
            assert p / 2 < v <= p, (r, b)


def test_mxfp4_codes_match_brute_force_nearest(orc):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((4, 64)) * 3).astype(np.float32)
    x[0, :8] = [2.5, -2.5, 0.75, -0.25, 5.0, 1.25, 1.75, -3.5]  # ties in a block of max 6-ish
    codes, scales = orc.mxfp4_quantize(x, "f32")
    for r in range(4):
        c = _codes(codes[r], 64)
        for k in range(64):
            t = float(x[r, k]) * 2.0 ** (127 - int(scales[r, k // 32]))
            assert c[k] == _brute_code(t), (r, k, t, c[k])


def test_mxfp4_grid_values_round_trip_exactly(orc):
    rng = np.random.default_rng(5)
    mags = np.array(E2M1, dtype=np.float64)
    x = mags[rng.integers(0, 8, (8, 96))] * np.where(rng.random((8, 96)) < 0.5, -1.0, 1.0)
    x[:, ::32] = 6.0  # a +6 in every block: the scale is exactly the block's power of two
    x *= np.exp2(rng.integers(-10, 10, (8, 1)))
    x = x.astype(np.float32)
    codes, scales = orc.mxfp4_quantize(x, "f32")
    np.testing.assert_array_equal(orc.mxfp4_decode_exact(codes, scales), x.astype(np.float64))
    np.testing.assert_array_equal(orc.mxfp4_dequantize(codes, scales, "f32"), x)


def test_mxfp4_zero_block_and_ones_matmul(orc):
    x = np.zeros((2, 64), dtype=np.float32)
    x[1] = 1.0
    codes, scales = orc.mxfp4_quantize(x, "f32")
    assert not codes[0].any() and int(scales[1, 0]) == 125  # 1/6 rounded up to 1/4
    # all-ones operands: every product is exactly 1, y = K
    r = orc.qqmm(codes[1:], scales[1:], codes[1:], scales[1:], mode="mxfp4", out_dt="f32")
    assert float(r["y_ref"][0, 0]) == 64.0


def test_mxfp4_dequantize_rounds_once_to_bf16(orc):
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    codes, scales = orc.mxfp4_quantize(x, "f32")
    exact = orc.mxfp4_decode_exact(codes, scales)
    # e2m1 (2 significant bits) times a power of two is a bf16 value: no rounding
    np.testing.assert_array_equal(orc.to_f64(orc.mxfp4_dequantize(codes, scales, "bf16"), "bf16"), exact)


# ---------------------------------------------------------------------------
# Mutation checks: plant a mistake in a copy of an MXFP4 step, see a pin fail
# ---------------------------------------------------------------------------
def _golden_scale_with(mistake):
    """Scale byte of each hand-derived block computed with a planted mistake."""
    out = []
    for name, x4, s, _ in _golden_blocks():
        a = np.float32(max(abs(v) for v in x4))
        if mistake == "round_nearest":     # e8m0 of max/6 to the nearest power, not up
            v = a / np.float32(6.0)
            e = int(np.round(np.log2(float(v)))) if v > 0 else -127
        elif mistake == "divisor_448":     # the MXFP8 divisor
            v = a / np.float32(448.0)
            e = int(np.ceil(np.log2(float(v)))) if v > 0 else -127
        else:
            v = a / np.float32(6.0)
            e = int(np.ceil(np.log2(float(v)))) if v > 0 else -127
        out.append((name, e + 127, s))
    return out


def test_mutation_mxfp4_round_nearest_scale_fails_golden():
    assert any(got != want for _, got, want in _golden_scale_with("round_nearest"))
    assert all(got == want for _, got, want in _golden_scale_with(None))  # the unmutated step agrees


def test_mutation_mxfp4_mxfp8_divisor_fails_golden():
    assert any(got != want for _, got, want in _golden_scale_with("divisor_448"))


def test_mutation_mxfp4_ties_away_fails_golden(orc):
    """Mistake: round ties away from zero instead of to the even code; the
    max6 block's 2.5 would become 3 (code 5) where the pin expects code 4."""
    name, x4, s, c4 = _golden_blocks()[0]
    k = 2.0 ** (127 - s)
    t = abs(x4[1]) * k
    lo = max(m for m in E2M1 if m <= t)
    hi = min(m for m in E2M1 if m >= t)
    away = hi if (t - lo) >= (hi - t) else lo
    assert E2M1.index(away) != c4[1]
