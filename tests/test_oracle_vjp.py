"""Pins of the oracle's qqmm backward pass ([P1] primitives.cpp QQMatmul::vjp:
dx from the cotangent and w^T, both quantized along N; dw from cotan^T and
x^T, both quantized along M; the cotangent's global scale is its amax) on
the CPU.  Inputs are chosen so that every quantization in the pass is exact,
each operand with a different global scale; the pass must then return the
exact gradient."""
import numpy as np
import pytest
import torch

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16(t):
    return torch.as_tensor(np.asarray(t, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def exact_operand(rng, rows, cols, unit):
    """unit * (e2m1-grid values), with unit * 6 at every (r, c) where
    r % 16 == c % 16: every 16-block along a row and along a column holds the
    tensor's amax (6 unit), so with g = amax every block scale is 448 and the
    codes are the grid values themselves (encode factor E = 2688 / g, block
    scale (6 unit / 6) E = 448, decode factor g / 2688 a power of two for the
    units used here)."""
    v = GRID[rng.integers(0, 7, (rows, cols))] * np.where(rng.random((rows, cols)) < 0.5, -1.0, 1.0)
    for r in range(rows):
        v[r, (r % 16)::16] = 6.0
    return v * unit


def raw(v, dt):
    return v.astype(np.float32) if dt == "f32" else bf16(v)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_vjp_is_the_exact_gradient_on_exact_operands(orc, dt):
    rng = np.random.default_rng(31)
    M, N, K = 48, 32, 80
    cotan = exact_operand(rng, M, N, 448.0)   # amax 2688: decode factor 1
    x = exact_operand(rng, M, K, 896.0)       # amax 5376: decode factor 2
    w = exact_operand(rng, N, K, 224.0)       # amax 1344: decode factor 1/2
    g_x, g_w = orc.amax(raw(x, dt), dt), orc.amax(raw(w, dt), dt)
    assert (g_x, g_w) == (5376.0, 1344.0)
    dx, dw = orc.qqmm_vjp(raw(x, dt), raw(w, dt), raw(cotan, dt), dt, g_x, g_w)
    assert dx["y_ref"].shape == (M, K) and dw["y_ref"].shape == (N, K)
    np.testing.assert_array_equal(dx["y_ref"], cotan @ w)
    np.testing.assert_array_equal(dw["y_ref"], cotan.T @ x)


def test_vjp_scale_blocks_are_448(orc):
    """The premise of the exact pin: each operand quantized along the axis
    the pass uses has every block scale 448 (e4m3 byte 0x7E) and its codes
    decode to the operand exactly."""
    rng = np.random.default_rng(32)
    for unit, shape in [(448.0, (48, 32)), (896.0, (48, 80)), (224.0, (32, 80))]:
        v = exact_operand(rng, *shape, unit)
        for a in (v, np.ascontiguousarray(v.T)):
            g = float(np.abs(a).max())
            c, s = orc.nvfp4_quantize(a.astype(np.float32), "f32", g)
            assert np.all(s == 0x7E)
            np.testing.assert_array_equal(orc.nvfp4_decode_exact(c, s, g), a)


def _vjp_planted(orc, x, w, cotan, dt, g_x, g_w, mistake):
    """The backward pass with one plausible mistake planted (CPU only)."""
    g_c = orc.amax(cotan, dt)
    if mistake == "swap_global_scales":
        g_x, g_w = g_w, g_x
    c, cs = orc.nvfp4_quantize(cotan, dt, g_c)
    w_op = w if mistake == "w_not_transposed" else np.ascontiguousarray(w.T)
    wt, wts = orc.nvfp4_quantize(w_op, dt, g_w)
    dx = orc.qqmm(c, cs, wt, wts, "nvfp4", g_c, g_w, dt)
    ct, cts = orc.nvfp4_quantize(np.ascontiguousarray(cotan.T), dt, g_c)
    x_op = x if mistake == "x_not_transposed" else np.ascontiguousarray(x.T)
    gx_used = g_w if mistake == "g_w_for_x" else g_x
    xt, xts = orc.nvfp4_quantize(x_op, dt, gx_used)
    dw = orc.qqmm(ct, cts, xt, xts, "nvfp4", g_c, gx_used, dt)
    return dx, dw


@pytest.mark.parametrize("mistake", ["swap_global_scales", "w_not_transposed", "x_not_transposed", "g_w_for_x"])
def test_mutations_fail_the_exact_pin(orc, mistake):
    """Each planted mistake changes the result on the exact operands (square
    shapes, so that the transposition mistakes still give defined products)."""
    rng = np.random.default_rng(33)
    M = N = K = 32
    cotan = exact_operand(rng, M, N, 448.0)
    x = exact_operand(rng, M, K, 896.0)
    w = exact_operand(rng, N, K, 224.0)
    dt = "f32"
    right = orc.qqmm_vjp(raw(x, dt), raw(w, dt), raw(cotan, dt), dt, 5376.0, 1344.0)
    np.testing.assert_array_equal(right[0]["y_ref"], cotan @ w)
    np.testing.assert_array_equal(right[1]["y_ref"], cotan.T @ x)
    dx, dw = _vjp_planted(orc, raw(x, dt), raw(w, dt), raw(cotan, dt), dt, 5376.0, 1344.0, mistake)
    assert not (np.array_equal(dx["y_ref"], cotan @ w) and np.array_equal(dw["y_ref"], cotan.T @ x))
