"""GPU parity of the column-wise NVFP4 quantize and of the qqmm backward
pass (QQMatmul::vjp) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from helpers import TORCH_DT, check_gemm_output, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4


def make_x(shape, dt, seed, std=1.0):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    return workloads.normal(shape, std, seed, TORCH_DT[dt], "cpu")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", [(16, 1), (48, 3), (256, 67), (4096, 128), (1040, 200), (64, 257), (144, 64)])
@pytest.mark.parametrize("use_g", [False, True])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_quantize_columnwise_parity(nv, orc, dt, shape, use_g, layout):
    """Column-wise quantize of x [R, C] == the oracle's quantize of x^T along R."""
    x = make_x(shape, dt, 500 + shape[0] + 3 * shape[1], std=0.02 if dt != "f16" else 1.0)
    xg = x.cuda()
    g = nv.amax(xg) if use_g else None
    codes, scales = nv.nvfp4_quantize_columnwise(xg, g, layout)
    torch.cuda.synchronize()
    xt = x.t().contiguous()
    oc, os_ = orc.nvfp4_quantize(raw(xt), dt, None if g is None else g.item())
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)


def test_quantize_columnwise_equals_rowwise_of_transpose(nv):
    """[4096, 4096] bf16 with outliers: bit-identical to nvfp4_quantize(x^T)."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal_with_outliers((4096, 4096), 0.02, 0.01, 50.0, 91, torch.bfloat16, "cuda")
    g = nv.amax(x)
    c1, s1 = nv.nvfp4_quantize_columnwise(x, g, "swizzled")
    c2, s2 = nv.nvfp4_quantize(x.t().contiguous(), g, "swizzled")
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(s1, s2)


def test_quantize_columnwise_rejects_rows_not_multiple_of_16(nv):
    with pytest.raises(nv.Nvfp4Error):
        nv.nvfp4_quantize_columnwise(torch.ones(24, 32, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("M,N,K", [(64, 96, 128), (256, 128, 512), (160, 320, 256)])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_qqmm_vjp_parity(nv, orc, M, N, K, dt):
    """dx = cotan_hat . (w^T)_hat^T and dw = (cotan^T)_hat . (x^T)_hat^T with
    g_c = amax(cotan), against the oracle's quantize + float64 qqmm."""
    x = make_x((M, K), dt, 11 + M, 1.0)
    w = make_x((N, K), dt, 12 + N, 0.02)
    cotan = make_x((M, N), dt, 13 + K, 0.1)
    xg, wg, cg = x.cuda(), w.cuda(), cotan.cuda()
    g_x, g_w = nv.amax(xg), nv.amax(wg)
    dx, dw = nv.qqmm_vjp(xg, wg, cg, g_x, g_w)
    nv.check_device_errors()
    # dx: cotan and w^T quantized along N; dw: cotan^T and x^T along M
    r_dx, r_dw = orc.qqmm_vjp(raw(x), raw(w), raw(cotan), dt, g_x.item(), g_w.item())
    check_gemm_output(raw(dx), r_dx, dt, orc)
    check_gemm_output(raw(dw), r_dw, dt, orc)
