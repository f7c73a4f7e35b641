"""Pins of the oracle's stochastic-rounding NVFP4 quantizer (CPU only).

The pages reserve stochastic rounding ("mlx 0.30.7.2 -> 0.30.7.6" diff,
page 7, fp_quantize_rowwise<..., USE_SR> with rbits "reserved for future
use"); the reading pinned here: scales as in the round-to-nearest quantizer,
each scaled value rounded to one of its two e2m1 neighbours, up with
probability equal to its relative position between them, decided by 32
random bits per element: byte i % 4 of one Philox4x32-10 word per group of
4 elements (the pages pass one 32-bit rbits word to each 4-value conversion,
scale_cvt_Tx4_to_fp4x4<T, USE_SR>)."""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _kat():
    out = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        f = line.split()
        v = [int(h, 16) for h in f[1:]]
        out.append((f[0], v[0:4], v[4:6], v[6:10]))
    return out


@pytest.mark.parametrize("name,ctr,key,want", _kat())
def test_philox_known_answers(orc, name, ctr, key, want):
    assert list(orc.philox4x32_10(ctr, key)) == want, name


def _val(code):
    return (-1.0 if code & 8 else 1.0) * MAGS[code & 7]


@pytest.mark.parametrize("t,r,code", [
    (2.5, 0, 5),              # u = 0 < 1/2: up to 3
    (2.5, 0xFF, 4),           # u = 255/256 >= 1/2: down to 2
    (5.0, 0x80, 6),           # u = 1/2, not < 1/2: down to 4
    (5.0, 0x7F, 7),           # u = 127/256 < 1/2: up to 6
    (2.25, 0x3F, 5),          # frac 1/4: u = 63/256 < 1/4: up
    (2.25, 0x40, 4),          # u = 1/4: down
    (-0.25, 0, 9),            # sign kept: -0.5
    (-0.25, 0xFF, 8),         # -0 (code 8), as the round-to-nearest path keeps the sign
    (7.0, 0, 7),              # saturates at 6
    (1.5, 123, 3),            # on the grid: kept
    (0.0, 0, 0),
])
def test_sr_hand_cases(orc, t, r, code):
    assert orc.e2m1_sr(t, r) == code


def test_sr_bits_are_bytes_of_philox_words(orc):
    """Element i takes byte i % 4 of word i / 4; word w is output w % 4 of
    Philox at counter w / 4 (16 elements per generator call)."""
    seed = 0x0123456789ABCDEF
    for i in [0, 1, 2, 3, 4, 7, 15, 16, 17, 1000003, 2**33 + 5]:
        w = i // 4
        out = orc.philox4x32_10([w // 4 & 0xFFFFFFFF, w // 4 >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        assert orc.sr_bits(seed, i) == (int(out[w % 4]) >> (8 * (i % 4))) & 0xFF


def test_sr_only_neighbours_and_unbiased(orc):
    rng = np.random.default_rng(1)
    for t in [0.3, 0.75, 1.2, 1.75, 2.9, 3.5, 5.1, -4.7]:
        codes = np.array([orc.e2m1_sr(t, int(orc.sr_bits(7, i))) for i in range(20000)])
        vals = np.array([_val(c) for c in codes])
        a = abs(t)
        lo = max(m for m in MAGS if m <= a)
        hi = min(m for m in MAGS if m >= a)
        assert set(np.abs(vals)) <= {lo, hi}
        p = (a - lo) / (hi - lo)
        sigma = (hi - lo) * np.sqrt(p * (1 - p) / len(vals))
        assert abs(np.abs(vals).mean() - a) < 5 * sigma + 1e-12, t


def test_sr_quantizer_scales_match_rne_and_codes_are_neighbours(orc):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    g = float(np.abs(x).max())
    c_rn, s_rn = orc.nvfp4_quantize(x, "f32", g)
    c_sr, s_sr = orc.nvfp4_quantize_sr(x, "f32", g, seed=123)
    assert np.array_equal(s_rn, s_sr)
    exact = orc.to_f64(x, "f32")
    d_sr = orc.nvfp4_decode_exact(c_sr, s_sr, g)
    d_rn = orc.nvfp4_decode_exact(c_rn, s_rn, g)
    # every SR value is one of the two grid neighbours of x; RNE picks the nearer one
    assert np.all(np.abs(d_sr - exact) <= np.abs(d_rn - exact) + np.abs(d_sr - d_rn) + 1e-12)
    assert np.all((d_sr == d_rn) | (np.sign(d_sr - exact) != np.sign(d_rn - exact)) | (d_rn == exact))


def test_sr_is_deterministic_per_seed_and_seed_dependent(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    a = orc.nvfp4_quantize_sr(x, "f32", None, seed=5)[0]
    b = orc.nvfp4_quantize_sr(x, "f32", None, seed=5)[0]
    c = orc.nvfp4_quantize_sr(x, "f32", None, seed=6)[0]
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_sr_grid_values_unchanged(orc):
    """Values exactly on the e2m1 grid with a 6 per block (scale 1): SR
    returns the round-to-nearest codes for every seed."""
    rng = np.random.default_rng(4)
    x = np.array(MAGS, dtype=np.float32)[rng.integers(0, 8, (4, 64))] * np.where(rng.random((4, 64)) < .5, -1, 1)
    x[:, ::16] = 6.0
    x = x.astype(np.float32)
    c_rn, _ = orc.nvfp4_quantize(x, "f32", None)
    for seed in (0, 1, 2**40 + 3):
        assert np.array_equal(orc.nvfp4_quantize_sr(x, "f32", None, seed=seed)[0], c_rn)


# ---------------------------------------------------------------------------
# Mutation checks: plant a mistake in a copy of an SR step, see a pin fail
# ---------------------------------------------------------------------------
def test_mutation_sr_comparison_reversed_is_biased(orc):
    """Mistake: round up when u >= frac (the complementary event).  The mean
    of many draws then sits at the mirror position, which the unbiasedness
    pin rejects."""
    t, lo, hi = 2.25, 2.0, 3.0
    frac = (t - lo) / (hi - lo)
    ups = sum(1 for i in range(20000) if ((orc.sr_bits(7, i) / 256.0) >= frac))
    mean = lo + (hi - lo) * ups / 20000
    sigma = (hi - lo) * np.sqrt(frac * (1 - frac) / 20000)
    assert abs(mean - t) > 5 * sigma


def test_mutation_sr_wrong_byte_fails_extraction_pin(orc):
    """Mistake: every element of a group of 4 takes byte 0 of the word."""
    seed = 0x0123456789ABCDEF
    diffs = 0
    for i in range(1, 64, 4):
        w = i // 4
        out = orc.philox4x32_10([w // 4 & 0xFFFFFFFF, w // 4 >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        diffs += orc.sr_bits(seed, i) != (int(out[w % 4]) & 0xFF)
    assert diffs > 0
