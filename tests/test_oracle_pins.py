"""Pins of the oracle's method-level functions against values the pages fix,
closed forms and invariants (CPU only).

Golden values live in tests/golden/, each file citing its page and section.
The mutation tests at the end plant a mistake in a copy of an oracle step
(on the CPU) and show that one of these pins fails on it.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        out[k] = v[0] if len(v) == 1 else v
    return out


def bf16(t):
    """numpy bf16 bit patterns of a float tensor / array."""
    return torch.as_tensor(np.asarray(t, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def bf16_value(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


def pack_codes(code_rows):
    """uint32 words of 4-bit codes, element 8w+i in bits 4i..4i+3 of word w."""
    c = np.asarray(code_rows, dtype=np.uint32)
    rows, K = c.shape
    c = c.reshape(rows, K // 8, 8)
    return np.bitwise_or.reduce(c << (4 * np.arange(8, dtype=np.uint32)), axis=2).astype(np.uint32)


# ---------------------------------------------------------------------------
# Worked example: "[Metal] global scale for qmm" (ml-explore/mlx pull 4458)
# ---------------------------------------------------------------------------
def _worked_example_weights(orc, K, g):
    codes = pack_codes(np.full((1, K), 0x7))  # e2m1 code 0x7 = 6
    scales = np.full((1, K // 16), 0x30, dtype=np.uint8)  # e4m3 0x30 = 0.5
    return codes, scales


def test_worked_example_block_values(orc):
    G = golden("worked_example_global_scale.txt")
    assert orc.e2m1_value(0x7) == float(G["code_value"])
    assert orc.e4m3_value(0x30) == float(G["block_scale"])


def test_worked_example_dequantize(orc):
    """w_hat = bf16(6 * 0.5 * 0.1) = 0.30078125; without the global scale 3.0.
    The page's decode factor 0.1 is g / 2688, so g = 268.8."""
    G = golden("worked_example_global_scale.txt")
    K = int(G["K"])
    g = float(np.float32(float(G["decode_factor"]) * 2688.0))
    codes, scales = _worked_example_weights(orc, K, g)
    w = bf16_value(orc.nvfp4_dequantize(codes, scales, g, "bf16"))
    assert np.all(w == float(G["w_with_global_bf16"]))
    w0 = bf16_value(orc.nvfp4_dequantize(codes, scales, None, "bf16"))
    assert np.all(w0 == float(G["w_without_global_bf16"]))


def test_worked_example_qmv_and_scale_after(orc):
    """qmv with x = ones: the bf16 result is 1232.0; scaling the bf16 product
    of the unscaled weights by the fp32 decode factor gives 1228.8000488
    (the page's "scale after")."""
    G = golden("worked_example_global_scale.txt")
    K = int(G["K"])
    g = float(np.float32(float(G["decode_factor"]) * 2688.0))
    codes, scales = _worked_example_weights(orc, K, g)
    x = bf16(np.ones((1, K)))
    g_x = orc.amax(x, "bf16")
    assert g_x == 1.0
    # x = ones survives quantize-dequantize with g_x = amax exactly
    assert np.array_equal(orc.nvfp4_quantize_dequantize(x, "bf16", g_x), x)
    r = orc.qmv(x, "bf16", g_x, codes, scales, g)
    assert bf16_value(r["y"])[0, 0] == float(G["y_scale_inside"])
    # the page's "scale after": bf16 product of the unscaled weights, times
    # the fp32 decode factor
    r0 = orc.qmv(x, "bf16", g_x, codes, scales, None)
    after = np.float32(bf16_value(r0["y"])[0, 0]) * np.float32(float(G["decode_factor"]))
    assert float(after) == float(G["y_scale_after"])
    assert float(np.float32(after) - np.float32(float(G["y_scale_inside"]))) == float(G["difference"])


def test_worked_example_in_gather_layout(orc):
    """Two experts, per-expert global scales (g shaped (E,1,1) on the page,
    [E] here): expert 0 decodes with 0.1 as in the example, expert 1 with
    g = 2688 (decode factor 1)."""
    K = 4096
    codes, scales = _worked_example_weights(orc, K, None)
    wc = np.stack([np.repeat(codes, 3, 0)] * 2)  # [E=2, N=3, K/8]
    ws = np.stack([np.repeat(scales, 3, 0)] * 2)
    g = np.array([np.float32(268.8), 2688.0], dtype=np.float32)
    x = bf16(np.ones((3, K)))
    idx = np.array([[0, 1], [1, 0], [0, 1]], dtype=np.int32)
    r = orc.gather_qmm(x, wc, ws, g, idx)
    y = bf16_value(r["y"])
    for t in range(3):
        for j in range(2):
            assert np.all(y[t, j] == (1232.0 if idx[t, j] == 0 else 4096 * 3.0))


def test_scale_inside_differs_from_scale_after_at_K96(orc):
    """Derived from the worked example, in the gather_qmm layout where the
    weight is rounded to bf16 before the matmul: with K = 96, y = 96 *
    0.30078125 = 28.875 exactly, while scaling after the matmul gives
    bf16(28.8) = 28.75.  This separates the two orders in a bf16 result."""
    K = 96
    g = np.array([np.float32(268.8)], dtype=np.float32)
    codes, scales = _worked_example_weights(orc, K, None)
    x = bf16(np.ones((1, K)))
    r = orc.gather_qmm(x, codes[None], scales[None], g, np.zeros((1, 1), dtype=np.int32))
    assert bf16_value(r["y"])[0, 0, 0] == 28.875


def test_qmv_does_not_round_the_weight(orc):
    """qmv keeps w_hat = e2m1 * fp32(f8(s) * d): K = 96, x = ones gives
    96 * 6 * fp32(0.5 * fp32(268.8/2688)) = 28.799998..., bf16 28.75."""
    K = 96
    g = float(np.float32(268.8))
    codes, scales = _worked_example_weights(orc, K, g)
    x = bf16(np.ones((1, K)))
    r = orc.qmv(x, "bf16", 1.0, codes, scales, g)
    sd = np.float32(np.float32(0.5) * (np.float32(g) / np.float32(2688.0)))
    assert r["y_ref"][0, 0] == 96 * 6 * float(sd)
    assert bf16_value(r["y"])[0, 0] == 28.75


# ---------------------------------------------------------------------------
# Cases A-D: osaurus-ai/mlx pull 31, "The test"
# ---------------------------------------------------------------------------
GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])


def grid_matrix(rows, K, seed):
    """Values on the e2m1 grid; every group of 16 holds +6 and -6."""
    rng = np.random.default_rng(seed)
    v = GRID[rng.integers(0, 8, size=(rows, K))] * rng.choice([-1.0, 1.0], size=(rows, K))
    for g0 in range(0, K, 16):
        v[:, g0] = 6.0
        v[:, g0 + 1] = -6.0
    return v


def _case(orc, name):
    x = grid_matrix(1, 32, 11)
    w = grid_matrix(4, 32, 12)
    if name == "A":
        return x, w, "f32", 2688.0, 336.0
    if name == "B":
        return x * 2.0 ** -12, w, "f32", 0.65625, 2688.0
    if name == "C":
        return x, w, "f32", None, None
    if name == "D":
        return w[:1].copy(), w, "f16", 2688.0, 10.5
    raise KeyError(name)


def _as(v, dt):
    return v.astype(np.float32) if dt == "f32" else v.astype(np.float16)


@pytest.mark.parametrize("name", ["A", "B", "C", "D"])
def test_cases_round_trip_and_exact_product(orc, name):
    x, w, dt, g_x, g_w = _case(orc, name)
    xq, xs = orc.nvfp4_quantize(_as(x, dt), dt, g_x)
    wq, ws = orc.nvfp4_quantize(_as(w, "f32"), "f32", g_w)
    # every dequantize gives x and w back exactly
    assert np.array_equal(orc.to_f64(orc.nvfp4_dequantize(xq, xs, g_x, dt), dt), x)
    assert np.array_equal(orc.to_f64(orc.nvfp4_dequantize(wq, ws, g_w, "f32"), "f32"), w)
    # qqmm equals the exact product of the original values
    r = orc.qqmm(xq, xs, wq, ws, "nvfp4", g_x, g_w, dt)
    assert np.array_equal(r["y_ref"], x @ w.T)
    assert np.array_equal(orc.to_f64(r["y"], dt), x @ w.T)  # exact in T too


def test_case_A_block_scale_is_8(orc):
    _, w, _, _, g_w = _case(orc, "A")
    _, ws = orc.nvfp4_quantize(w.astype(np.float32), "f32", g_w)
    assert np.all(ws == 0x50) and orc.e4m3_value(0x50) == 8.0


def test_case_B_encode_factor_rescues_underflow(orc):
    x, _, _, g_x, _ = _case(orc, "B")
    assert np.float32(2688.0) / np.float32(g_x) == 4096.0
    _, xs = orc.nvfp4_quantize(x.astype(np.float32), "f32", g_x)
    assert np.all(xs == 0x38)  # 1.0
    # without the global scale the block scales (2^-12) underflow e4m3 to 0
    xq0, xs0 = orc.nvfp4_quantize(x.astype(np.float32), "f32", None)
    assert np.all(xs0 == 0x00) and np.all(xq0 == 0)
    assert np.all(orc.to_f64(orc.nvfp4_dequantize(xq0, xs0, None, "f32"), "f32") == 0)


def test_case_D_scale_256_decoded_by_2_pow_minus_8(orc):
    _, w, _, _, g_w = _case(orc, "D")
    _, ws = orc.nvfp4_quantize(w.astype(np.float32), "f32", g_w)
    assert np.all(ws == 0x78) and orc.e4m3_value(0x78) == 256.0
    assert np.float32(g_w) / np.float32(2688.0) == 2.0 ** -8
    assert orc.nvfp4_block_scale(0x78, g_w) == 1.0


def test_case_D_product_needs_the_per_block_scale_in_f16(orc):
    """256 times the product overflows float16 for at least one element
    of a 32-long dot product with +-6 pairs (the page's point for case D)."""
    x, w, dt, g_x, g_w = _case(orc, "D")
    y = x @ w.T
    assert np.all(np.abs(y) <= 65504) and np.any(np.abs(y * 256) > 65504)


# ---------------------------------------------------------------------------
# MXFP8: E8M0 scale rounded up (mlxcel pull 1772 text on the pull 4458 page)
# ---------------------------------------------------------------------------
def test_mxfp8_round_up_case(orc):
    G = golden("mxfp8_round_up.txt")
    m = float(G["block_max"])
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = m
    x[0, 1:] = np.linspace(-1, 1, 31, dtype=np.float32)
    q, s = orc.mxfp8_quantize(x, "f32")
    assert s[0, 0] == 121  # 2^-6: the smallest power of two >= m / 448
    # the maximum scales to 307.5 and encodes as 320 (0x7A), unsaturated
    assert m * 2.0 ** 6 == 307.5
    assert (q[0, 0] & 0xFF) == 0x7A and orc.e4m3_value(0x7A) == 320.0
    # round-to-nearest would have chosen 2^-7, scaling the maximum to 615
    assert round(math.log2(m / 448.0)) == -7
    assert m * 2.0 ** 7 == float(G["round_nearest_scaled_max"])
    assert orc.e4m3_encode(np.float32(615.0)) == 0x7E  # saturates at 448


def test_mxfp8_block_max_within_448_scale(orc):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((64, 256)) * np.exp2(rng.uniform(-20, 20, (64, 1)))).astype(np.float32)
    q, s = orc.mxfp8_quantize(x, "f32")
    gm = np.abs(x).reshape(64, 8, 32).max(axis=2)
    scale = np.exp2(s.astype(np.float64) - 127)
    assert np.all(gm <= 448.0 * scale)
    assert np.all(gm > 448.0 * scale / 2)  # and the scale is the smallest such
    # decode error bounded by half an e4m3 step at the element's magnitude
    xd = orc.mxfp8_decode_exact(q, s)
    assert np.all(np.abs(xd - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * np.repeat(scale, 32, 1)))


def test_mxfp8_zero_block(orc):
    q, s = orc.mxfp8_quantize(np.zeros((2, 64), dtype=np.float32), "f32")
    assert np.all(s == 0) and np.all(q == 0)


# (e4m3 code byte, e8m0 scale byte, value) from the two formats' definitions:
# e4m3 (-1)^s 2^(e-7) (1 + m/8), subnormal (e = 0) 2^-6 m/8; e8m0 2^(b-127).
MXFP8_DECODE_CASES = [
    (0x38, 127, 1.0),                 # e=7 m=0
    (0x7E, 127, 448.0),               # e=15 m=6: 2^8 * 1.75, the largest e4m3
    (0x01, 127, 0.001953125),         # subnormal m=1: 2^-6 / 8 = 2^-9
    (0xB8, 130, -8.0),                # sign, 1.0 * 2^3
    (0x7A, 121, 5.0),                 # 320 * 2^-6: the round-up case decoded
    (0x00, 200, 0.0),
    (0x80, 127, -0.0),                # signed zero keeps its sign
    (0x3C, 254, 1.5 * 2.0 ** 127),    # e=7 m=4, the largest e8m0 scale
    (0x38, 0, 2.0 ** -127),           # the smallest e8m0 scale
]


@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
def test_mxfp8_dequantize_hand_decoded_bytes(orc, out_dt):
    """One row per case: element 0 holds the case's code, the other 31 hold
    0x38 (1.0), all under the case's scale; the product is exact in f32 and
    bf16 for every case, so the dequantize returns it exactly."""
    rows = len(MXFP8_DECODE_CASES)
    code_bytes = np.full((rows, 32), 0x38, dtype=np.uint32)
    scales = np.zeros((rows, 1), dtype=np.uint8)
    want = np.zeros((rows, 32))
    for r, (c, sb, v) in enumerate(MXFP8_DECODE_CASES):
        code_bytes[r, 0] = c
        scales[r, 0] = sb
        want[r, 0] = v
        want[r, 1:] = 2.0 ** (sb - 127)
    words = code_bytes.reshape(rows, 8, 4)
    codes = np.bitwise_or.reduce(words << (8 * np.arange(4, dtype=np.uint32)), axis=2).astype(np.uint32)
    got = orc.to_f64(orc.mxfp8_dequantize(codes, scales, out_dt), out_dt)
    np.testing.assert_array_equal(got, want)
    assert np.signbit(got[6, 0]) and not np.signbit(got[5, 0])
    np.testing.assert_array_equal(orc.mxfp8_decode_exact(codes, scales), want)


def test_mxfp8_dequantize_of_quantize_round_up_case(orc):
    """The round-up case's block maximum (4.8046875) comes back as 5.0: code
    320 under scale 2^-6."""
    G = golden("mxfp8_round_up.txt")
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0] = float(G["block_max"])
    q, s = orc.mxfp8_quantize(x, "f32")
    assert orc.to_f64(orc.mxfp8_dequantize(q, s, "f32"), "f32")[0, 0] == 5.0


# ---------------------------------------------------------------------------
# Scale layout: the page's index table ("mlx 0.30.7" diff page 71)
# ---------------------------------------------------------------------------
def test_swizzle_index_table(orc):
    lines = [l.split() for l in open(os.path.join(GOLDEN, "swizzle_tile_128x4.txt"))
             if l.strip() and not l.startswith("#")]
    idx = np.arange(512).reshape(128, 4)
    lo = orc.swizzle_scales((idx & 0xFF).astype(np.uint8)).reshape(-1).astype(np.int64)
    hi = orc.swizzle_scales((idx >> 8).astype(np.uint8)).reshape(-1).astype(np.int64)
    packed = lo | (hi << 8)
    for line in lines:
        n = int(line[0])
        assert packed[16 * n:16 * n + 16].tolist() == [int(v) for v in line[1:]]


@pytest.mark.parametrize("rows,cols", [(67, 16), (128, 4), (200, 5), (1, 1), (256, 256)])
def test_swizzle_padding_is_zero_and_permutation(orc, rows, cols):
    rng = np.random.default_rng(rows * 1000 + cols)
    lin = rng.integers(1, 256, size=(rows, cols), dtype=np.uint8)
    sw = orc.swizzle_scales(lin)
    Rp, Cp = (rows + 127) // 128 * 128, (cols + 3) // 4 * 4
    assert sw.shape == (Rp, Cp)
    assert np.count_nonzero(sw) == rows * cols  # every real byte once, padding 0
    assert sorted(sw[sw != 0].tolist()) == sorted(lin.reshape(-1).tolist())


# ---------------------------------------------------------------------------
# Closed forms and invariants of the NVFP4 quantizer
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_amax_block_gets_scale_448_and_code_6(orc, dt):
    for seed in range(5):
        rng = np.random.default_rng(seed)
        v = rng.standard_normal((8, 64)) * 10 ** rng.uniform(-3, 3)
        x = v.astype(np.float32) if dt == "f32" else (v.astype(np.float16) if dt == "f16" else bf16(v))
        xf = orc.to_f64(x, dt)
        g = orc.amax(x, dt)
        assert g == np.abs(xf).max()
        q, s = orc.nvfp4_quantize(x, dt, g)
        r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        assert s[r, c // 16] == 0x7E
        code = (q[r, c // 8] >> (4 * (c % 8))) & 0xF
        assert code == (0x7 if xf[r, c] > 0 else 0xF)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_no_global_scale_equals_g_2688(orc, dt):
    rng = np.random.default_rng(7)
    v = rng.standard_normal((16, 128)) * 3
    x = v.astype(np.float32) if dt == "f32" else (v.astype(np.float16) if dt == "f16" else bf16(v))
    q0, s0 = orc.nvfp4_quantize(x, dt, None)
    q1, s1 = orc.nvfp4_quantize(x, dt, 2688.0)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1)


def test_nvfp4_scale_byte_is_e4m3_of_scaled_block_amax(orc):
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    g = orc.amax(x, "f32")
    q, s = orc.nvfp4_quantize(x, "f32", g)
    a = np.abs(x).reshape(32, 16, 16).max(axis=2)
    t = (a.astype(np.float32) / np.float32(6.0)) * (np.float32(2688.0) / np.float32(g))
    # the stored byte is within half an e4m3 step of t (relative 2^-4)
    sv = np.vectorize(orc.e4m3_value)(s)
    assert np.all(np.abs(sv - t) <= np.maximum(t * 2.0 ** -4, 2.0 ** -10))
    # and each element's decoded value is within one e2m1 half-step of x
    xd = orc.nvfp4_decode_exact(q, s, g)
    blk = np.repeat(sv * (np.float32(g) / np.float32(2688.0)), 16, axis=1)
    assert np.all(np.abs(xd - x) <= blk * 1.0 + 1e-30)


def test_quantize_dequantize_equals_dequantize_of_quantize(orc):
    rng = np.random.default_rng(9)
    x = bf16(rng.standard_normal((4, 512)))
    g = orc.amax(x, "bf16")
    q, s = orc.nvfp4_quantize(x, "bf16", g)
    assert np.array_equal(orc.nvfp4_quantize_dequantize(x, "bf16", g),
                          orc.nvfp4_dequantize(q, s, g, "bf16"))


def test_tiny_workload_oracle_runs(orc):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("tiny")
    x, w = d["x"].numpy(), d["w"].numpy()
    gx, gw = orc.amax(x, "f32"), orc.amax(w, "f32")
    xq, xs = orc.nvfp4_quantize(x, "f32", gx)
    wq, ws = orc.nvfp4_quantize(w, "f32", gw)
    r = orc.qqmm(xq, xs, wq, ws, "nvfp4", gx, gw, "f32")
    assert r["y"].shape == (4, 64)
    # quantization error of a K=256 dot product of N(0,1) data stays small
    # against the magnitude scale of the exact product
    assert np.max(np.abs(r["y_ref"] - x.astype(np.float64) @ w.T.astype(np.float64))) < 0.25 * np.sqrt(256) * 4


# ---------------------------------------------------------------------------
# Mutation checks: plant a mistake in a copy of an oracle step, see a pin fail
# ---------------------------------------------------------------------------
def test_mutation_global_scale_on_the_sum_fails_K96_pin(orc):
    """Mistake (gather_qmm): decode w without g into bf16, apply g to the
    bf16 result of the sum."""
    K = 96
    g = np.array([np.float32(268.8)], dtype=np.float32)
    codes, scales = _worked_example_weights(orc, K, None)
    x = bf16(np.ones((1, K)))
    r0 = orc.gather_qmm(x, codes[None], scales[None], None, np.zeros((1, 1), dtype=np.int32))
    mutated = orc.round_to(np.array([r0["y_ref"][0, 0, 0] * float(g[0] / np.float32(2688.0))]), "bf16")
    assert bf16_value(mutated)[0] != 28.875  # the pin catches it


def test_mutation_dropped_g_w_fails_case_A(orc):
    x, w, dt, g_x, g_w = _case(orc, "A")
    xq, xs = orc.nvfp4_quantize(_as(x, dt), dt, g_x)
    wq, ws = orc.nvfp4_quantize(_as(w, "f32"), "f32", g_w)
    r = orc.qqmm(xq, xs, wq, ws, "nvfp4", g_x, 2688.0, dt)  # g_w dropped
    assert not np.array_equal(r["y_ref"], x @ w.T)
    assert np.array_equal(r["y_ref"], 8 * (x @ w.T))


def test_mutation_amax_over_16_not_scaled_by_E_fails_case_B(orc):
    """Mistake: ignore the encode factor in the scale (t = a/6)."""
    x, _, _, g_x, _ = _case(orc, "B")
    a = np.abs(x).reshape(1, 2, 16).max(axis=2).astype(np.float32)
    t = a / np.float32(6.0)  # missing * 2688/g
    bytes_ = np.vectorize(lambda v: orc.e4m3_encode(float(v)))(t)
    assert not np.all(bytes_ == 0x38)


# ---------------------------------------------------------------------------
# MX modes of qqmm on exactly representable operands
# ---------------------------------------------------------------------------
def _mx_exact_operand(rng, rows, K, mags, top, ks):
    """rows x K values: per 32-block a power of two 2^k (k from ks), each
    element a random signed magnitude from ``mags`` times 2^k, and one
    element +-top*2^k setting the block maximum.  With top = the format's
    largest magnitude (448 for e4m3, 6 for e2m1) the e8m0 scale of the block
    is 2^k exactly and every element's code represents it exactly."""
    v = np.empty((rows, K))
    kblk = rng.choice(ks, size=(rows, K // 32))
    for r in range(rows):
        for b in range(K // 32):
            blk = rng.choice(mags, 32) * np.where(rng.random(32) < 0.5, -1.0, 1.0)
            blk[rng.integers(0, 32)] = top * (1.0 if rng.random() < 0.5 else -1.0)
            v[r, 32 * b:32 * b + 32] = blk * 2.0 ** kblk[r, b]
    return v.astype(np.float32), kblk


def _e4m3_magnitudes():
    """Every finite e4m3 magnitude from the format's definition: subnormals
    m/8 2^-6, normals (1 + m/8) 2^(e-7) for e = 1..15 except the NaN code."""
    vals = [m / 8 * 2.0 ** -6 for m in range(8)]
    vals += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    return np.array(vals)


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
def test_mx_qqmm_exact_on_representable_operands(orc, mode):
    rng = np.random.default_rng(41)
    M, N, K = 5, 7, 96
    if mode == "mxfp8":
        mags, top, quant = _e4m3_magnitudes(), 448.0, orc.mxfp8_quantize
    else:
        mags, top, quant = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]), 6.0, orc.mxfp4_quantize
    x, kx = _mx_exact_operand(rng, M, K, mags, top, [-3, 0, 2])
    w, kw = _mx_exact_operand(rng, N, K, mags, top, [-1, 1, 4])
    xq, xs = quant(x, "f32")
    wq, ws = quant(w, "f32")
    assert np.array_equal(xs, 127 + kx) and np.array_equal(ws, 127 + kw)
    r = orc.qqmm(xq, xs, wq, ws, mode, out_dt="f32")
    assert r["y_ref"].shape == (M, N)
    np.testing.assert_array_equal(r["y_ref"], x.astype(np.float64) @ w.astype(np.float64).T)


def test_mutation_mx_qqmm_without_block_scales_fails_exact_pin(orc):
    """Mistake: contract the codes' values without the per-block 2^(s-127)
    (here: decode with every scale byte forced to 127)."""
    rng = np.random.default_rng(42)
    x, _ = _mx_exact_operand(rng, 4, 64, _e4m3_magnitudes(), 448.0, [-3, 0, 2])
    w, _ = _mx_exact_operand(rng, 6, 64, _e4m3_magnitudes(), 448.0, [-1, 1, 4])
    xq, xs = orc.mxfp8_quantize(x, "f32")
    wq, ws = orc.mxfp8_quantize(w, "f32")
    wrong = orc.qqmm(xq, np.full_like(xs, 127), wq, np.full_like(ws, 127), "mxfp8", out_dt="f32")["y_ref"]
    assert not np.array_equal(wrong, x.astype(np.float64) @ w.astype(np.float64).T)


def test_qmv_quantizes_x_first(orc):
    """qmv contracts x_hat, not x.  One 16-block x = [6, 2.9, 1.2, 0.7, 0 ...]
    (bf16), a zero second block, g_x = amax = 6: E = 2688/6 = 448, block scale
    e4m3(6/6 * 448) = 448, encode factor 1, codes e2m1 of [6, 2.90625,
    1.203125, 0.69921875] = [6, 3, 1, 0.5] (0.699 is below the 0.75
    midpoint), decode factor 448 * 6/2688 = 1: x_hat = [6, 3, 1, 0.5].  With
    every weight 1 (code 0x2, scale 1.0, no global scale) y = 10.5, where the
    raw x would give bf16(10.80859375) = 10.8125."""
    K = 32
    xv = np.zeros((1, K))
    xv[0, :4] = [6.0, 2.9, 1.2, 0.7]
    x = bf16(xv)
    g_x = orc.amax(x, "bf16")
    assert g_x == 6.0
    codes = pack_codes(np.full((2, K), 0x2))
    scales = np.full((2, K // 16), 0x38, dtype=np.uint8)
    r = orc.qmv(x, "bf16", g_x, codes, scales, None)
    assert np.all(bf16_value(r["y"]) == 10.5)
    assert float(bf16_value(x).sum()) == 10.80859375
