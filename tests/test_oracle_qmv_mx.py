"""Pins of the oracle's qmv in the MX modes (CPU only): the M = 1 route of
"mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, qqmm.cpp QQMatmul::eval_gpu, which
quantize-dequantizes x with the mode's group size and bits before fp_qmv.
Each case is a hand-derived 32-element block whose quantize-dequantize
differs from x, against unit weights, so y is the sum of x_hat."""
import numpy as np
import pytest
import torch


def bf16(v):
    return torch.as_tensor(np.asarray(v, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def bf16_value(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


def unit_weights(mode, n, K):
    """Every weight 1.0: MXFP4 code 0x2 (8 per word), MXFP8 byte 0x38 (4 per
    word), every e8m0 scale byte 127 (2^0)."""
    word = 0x22222222 if mode == "mxfp4" else 0x38383838
    per_word = 8 if mode == "mxfp4" else 4
    codes = np.full((n, K // per_word), word, dtype=np.uint32)
    scales = np.full((n, K // 32), 127, dtype=np.uint8)
    return codes, scales


def test_mxfp4_qmv_quantizes_x_first(orc):
    """x = [6, 2.9, 1.2, 0.7, 0, ...] (bf16: 6, 2.90625, 1.203125,
    0.69921875): amax / 6 = 1, rounded up to the power of two 2^0 (scale
    byte 127); codes e2m1 of [6, 2.90625, 1.203125, 0.69921875] =
    [6, 3, 1, 0.5] (0.699 is below the 0.75 midpoint, 1.2 below 1.25), so
    x_hat = [6, 3, 1, 0.5] and y = 10.5; the raw x would give bf16(10.80859375)
    = 10.8125."""
    K = 32
    xv = np.zeros((1, K))
    xv[0, :4] = [6.0, 2.9, 1.2, 0.7]
    x = bf16(xv)
    codes, scales = unit_weights("mxfp4", 3, K)
    r = orc.qmv_mx(x, "bf16", codes, scales, "mxfp4")
    assert np.all(bf16_value(r["y"]) == 10.5)
    assert float(bf16_value(x).sum()) == 10.80859375


def test_mxfp8_qmv_quantizes_x_first(orc):
    """x = [3.3, 1, 0, ...] (bf16: 3.296875, 1): amax / 448 = 0.00735...,
    rounded up to 2^-7 (scale byte 120); 3.296875 * 2^7 = 422 lies between
    the e4m3 values 416 and 448 below their midpoint 432, so its code is 416
    and x_hat = 416 / 128 = 3.25; 1 * 2^7 = 128 is exact.  y = 4.25 (the raw
    x: 4.296875)."""
    K = 64
    xv = np.zeros((1, K))
    xv[0, :2] = [3.3, 1.0]
    x = bf16(xv)
    xc, xs = orc.mxfp8_quantize(x, "bf16")
    assert xs[0, 0] == 120
    codes, scales = unit_weights("mxfp8", 2, K)
    r = orc.qmv_mx(x, "bf16", codes, scales, "mxfp8")
    assert np.all(bf16_value(r["y"]) == 4.25)
    assert float(bf16_value(x).sum()) == 4.296875


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
def test_qmv_mx_weight_scales_apply_per_block(orc, mode):
    """With x = ones (x_hat = x exactly: amax 1 is a power of two times the
    format's max only through the rounded-up scale, and 1 is on both grids),
    unit codes and scale bytes 127 + j for block j, y = 32 * sum_j 2^j."""
    K = 96
    x = bf16(np.ones((1, K)))
    codes, scales = unit_weights(mode, 1, K)
    scales[0, :] = [127, 128, 129]
    r = orc.qmv_mx(x, "bf16", codes, scales, mode)
    assert float(bf16_value(r["y"])[0, 0]) == 32 * (1 + 2 + 4)
