"""GPU parity of the NVFP4 quantizer with stochastic rounding (Philox4x32-10
random bits keyed by a 64-bit seed) against the oracle, bit-exact codes and
scales, through the C ABI."""
import numpy as np
import pytest
import torch

from helpers import TORCH_DT, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    assert torch.cuda.is_available()
    return nvfp4


def make_x(shape, dt, seed, std=1.0):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    return workloads.normal(shape, std, seed, TORCH_DT[dt], "cpu")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (67, 256), (200, 1040), (257, 64)])
@pytest.mark.parametrize("use_g", [False, True])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_sr_quantize_parity(nv, orc, dt, shape, use_g, layout):
    x = make_x(shape, dt, 500 + shape[0] + shape[1], std=0.02 if dt != "f16" else 1.0)
    xg = x.cuda()
    g = nv.amax(xg) if use_g else None
    seed = 0x1234_5678_9ABC + shape[0]
    codes, scales = nv.nvfp4_quantize_sr(xg, g, seed, layout)
    nv.check_device_errors()
    oc, os_ = orc.nvfp4_quantize_sr(raw(x), dt, None if g is None else g.item(), seed=seed)
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)


@pytest.mark.parametrize("seed", [0, 1, 2**32 - 1, 2**32, 2**63 + 12345])
def test_sr_seeds(nv, orc, seed):
    x = make_x((64, 512), "bf16", 9)
    codes, _ = nv.nvfp4_quantize_sr(x.cuda(), None, seed, "linear")
    oc, _ = orc.nvfp4_quantize_sr(raw(x), "bf16", None, seed=seed)
    assert np.array_equal(raw(codes), oc)


def test_sr_scales_equal_rne_and_mean_is_unbiased(nv, orc):
    """Scales equal the round-to-nearest quantizer's; averaged over 64 seeds
    the dequantized values approach x (each draw is one of x's two grid
    neighbours, so the mean's error shrinks like 1/sqrt(draws))."""
    x = make_x((32, 256), "f32", 11)
    xg = x.cuda()
    c_rn, s_rn = nv.nvfp4_quantize(xg, None, "linear")
    acc = torch.zeros(32, 256, dtype=torch.float64, device="cuda")
    for seed in range(64):
        c, s = nv.nvfp4_quantize_sr(xg, None, seed, "linear")
        assert torch.equal(s, s_rn)
        acc += nv.nvfp4_dequantize(c, s, None, "linear", torch.float32).double()
    mean = acc / 64
    err_sr = (mean - xg.double()).abs().mean().item()
    err_rn = (nv.nvfp4_dequantize(c_rn, s_rn, None, "linear", torch.float32).double() - xg.double()).abs().mean().item()
    assert err_sr < 0.5 * err_rn, (err_sr, err_rn)


def test_sr_full_size_sampled_rows(nv, orc):
    """The 1 GiB quantize config [32768, 16384] bf16 N(0,1): 8 rows checked,
    the first and last among them (counters up to 2^26)."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.make("quant1g", device="cuda")["x"]
    g = nv.amax(x)
    codes, scales = nv.nvfp4_quantize_sr(x, g, 99, "linear")
    nv.check_device_errors()
    rows = [0, 1, 4095, 16384, 20000, 30001, 32766, 32767]
    xs = raw(x[rows].cpu())
    del x
    # rows checked through the scalar oracle steps
    xs_f = orc.to_f64(xs, "bf16").astype(np.float32)
    codes_c = raw(codes[rows].cpu())
    scales_c = raw(scales[rows].cpu())
    c_rn, s_rn = orc.nvfp4_quantize(xs, "bf16", g.item())
    assert np.array_equal(scales_c, s_rn)
    E = np.float32(2688.0) / np.float32(g.item())
    for n, r in enumerate(rows):
        for b in (0, 5, 1023):
            fs = np.float32(orc.e4m3_value(int(s_rn[n, b])))
            if fs == 0:
                continue
            kf = np.float32(E / fs)
            for j in range(16):
                kk = b * 16 + j
                t = np.float32(xs_f[n, kk] * kf)
                want = orc.e2m1_sr(float(t), orc.sr_bits(99, r * 16384 + kk))
                got = (int(codes_c[n, kk // 8]) >> (4 * (kk % 8))) & 15
                assert got == want, (r, kk)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(16, 1), (48, 3), (256, 67), (1040, 200), (4096, 130)])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_sr_columnwise_parity(nv, orc, dt, shape, layout):
    """Column-wise stochastic rounding equals the oracle's stochastic
    rounding of the transposed, contiguous matrix with the same seed."""
    x = make_x(shape, dt, 900 + shape[0] + shape[1], std=0.02)
    xg = x.cuda()
    g = nv.amax(xg)
    seed = 0xDEAD_BEEF_0000 + shape[1]
    codes, scales = nv.nvfp4_quantize_columnwise(xg, g, layout, seed=seed)
    nv.check_device_errors()
    oc, os_ = orc.nvfp4_quantize_sr(raw(x.t().contiguous()), dt, g.item(), seed=seed)
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)
