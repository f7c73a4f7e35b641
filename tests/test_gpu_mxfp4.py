"""GPU parity of the MXFP4 mode (4-bit e2m1 codes with e8m0 scales per 32
elements) against the CPU oracle, through the C ABI: quantize and dequantize
bit-exact, the dense block-scaled GEMM in mxfp4 mode within the GEMM
tolerance, ragged shapes, every dtype."""
import numpy as np
import pytest
import torch

from helpers import TORCH_DT, check_gemm_output, raw

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
@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (67, 256), (130, 4128), (257, 64)])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_mxfp4_quantize_parity(nv, orc, dt, shape, layout):
    x = make_x(shape, dt, 300 + shape[0] * 3 + shape[1])
    codes, scales = nv.mxfp4_quantize(x.cuda(), layout)
    nv.check_device_errors()
    oc, os_ = orc.mxfp4_quantize(raw(x), dt)
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)


def test_mxfp4_quantize_wide_range_and_zero_rows(nv, orc):
    """Rows scaled by 2^-60 .. 2^60 (e8m0 scales far from 127), a zero row,
    values exactly on ties and at the saturation edge."""
    x = make_x((64, 128), "f32", 9)
    x = x * torch.exp2(torch.arange(-60, 68, 2, dtype=torch.float32)).reshape(64, 1)
    x[5] = 0.0
    x[6, :8] = torch.tensor([6.0, 2.5, -5.0, 0.25, 3.0, -1.5, 1.25, 5.9999])
    codes, scales = nv.mxfp4_quantize(x.cuda(), "linear")
    oc, os_ = orc.mxfp4_quantize(raw(x), "f32")
    assert np.array_equal(raw(codes), oc)
    assert np.array_equal(raw(scales), os_)


@pytest.mark.parametrize("out_dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_mxfp4_dequantize_parity(nv, orc, out_dt, layout):
    x = make_x((67, 288), "bf16", 4)
    codes, scales = nv.mxfp4_quantize(x.cuda(), layout)
    out = nv.mxfp4_dequantize(codes, scales, layout, TORCH_DT[out_dt])
    oc, os_ = orc.mxfp4_quantize(raw(x), "bf16")
    want = orc.mxfp4_dequantize(oc, os_, out_dt)
    assert np.array_equal(raw(out).view(np.uint8), want.view(np.uint8))


def _qqmm(nv, orc, M, N, K, out_dt, seed, in_dt=torch.bfloat16, rows=None):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal((M, K), 1.0, seed, in_dt)
    w = workloads.normal((N, K), 1.0, seed + 1, in_dt)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[in_dt]
    xc, xs = nv.mxfp4_quantize(x.cuda(), "swizzled")
    wc, ws = nv.mxfp4_quantize(w.cuda(), "swizzled")
    y = nv.qqmm(xc, xs, wc, ws, K, "mxfp4", out_dtype=TORCH_DT[out_dt])
    nv.check_device_errors()
    (oxc, oxs), (owc, ows) = orc.mxfp4_quantize(raw(x), dt), orc.mxfp4_quantize(raw(w), dt)
    assert np.array_equal(raw(xc), oxc) and np.array_equal(raw(wc), owc)
    r = orc.qqmm(oxc, oxs, owc, ows, "mxfp4", None, None, out_dt, rows=rows)
    return check_gemm_output(raw(y) if rows is None else raw(y)[rows], r, out_dt, orc)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (67, 300, 1056), (256, 256, 4096), (200, 72, 96),
                                   (1, 256, 512), (130, 520, 160), (384, 136, 2048)])
@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
def test_mxfp4_qqmm_parity(nv, orc, M, N, K, out_dt):
    _qqmm(nv, orc, M, N, K, out_dt, seed=M + 3 * N + K)


@pytest.mark.parametrize("in_dt", [torch.float32, torch.float16])
def test_mxfp4_qqmm_input_dtypes_f16_out(nv, orc, in_dt):
    _qqmm(nv, orc, 130, 260, 512, "f16", seed=5, in_dt=in_dt)


def test_mxfp4_qqmm_4096_sampled_rows(nv, orc):
    rows = np.sort(np.random.default_rng(2).choice(4096, 48, replace=False))
    _qqmm(nv, orc, 4096, 4096, 4096, "bf16", seed=21, rows=rows)


def test_mxfp4_qqmm_rejects_global_scales(nv):
    x = torch.randn(128, 256, device="cuda", dtype=torch.bfloat16)
    xc, xs = nv.mxfp4_quantize(x, "swizzled")
    g = nv.amax(x)
    with pytest.raises(RuntimeError, match="only supported for 'nvfp4'"):
        nv.qqmm(xc, xs, xc, xs, 256, "mxfp4", g, g)
