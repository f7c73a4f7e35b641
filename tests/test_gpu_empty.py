"""Empty inputs through the binding on the GPU: every call with an empty
output returns empty results without error, and amax of nothing is 0."""
import pytest
import torch

pytestmark = pytest.mark.gpu

bf16, i32, u8 = torch.bfloat16, torch.int32, torch.uint8


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4


def z(*shape, dtype=u8):
    return torch.zeros(*shape, dtype=dtype, device="cuda")


def test_amax_of_nothing_is_zero(nv):
    g = torch.full((1,), 5.0, device="cuda")
    nv.amax(z(0, dtype=bf16), g)
    assert g.item() == 0.0


@pytest.mark.parametrize("layout", ["linear", "swizzled"])
@pytest.mark.parametrize("shape", [(0, 64), (5, 0)])
def test_quantizers(nv, layout, shape):
    x = z(*shape, dtype=bf16)
    rows, K = shape
    for fn, cw, sc in [(lambda: nv.nvfp4_quantize(x, None, layout), K // 8, K // 16),
                       (lambda: nv.nvfp4_quantize_sr(x, None, 7, layout), K // 8, K // 16),
                       (lambda: nv.mxfp8_quantize(x, layout), K // 4, K // 32),
                       (lambda: nv.mxfp4_quantize(x, layout), K // 8, K // 32)]:
        codes, scales = fn()
        assert codes.shape == (rows, cw) and scales.numel() == nv.scale_bytes(rows, sc, layout)
    codes, scales = nv.nvfp4_quantize_columnwise(z(K, rows, dtype=bf16), None, layout)  # x^T of the same shape
    assert codes.numel() == 0
    torch.cuda.synchronize()
    nv.check_device_errors()


def test_dequantizers_and_swizzle(nv):
    out = nv.nvfp4_dequantize(z(0, 8, dtype=i32), z(0, 4))
    assert out.shape == (0, 64)
    assert nv.mxfp8_dequantize(z(0, 16, dtype=i32), z(0, 2)).shape == (0, 64)
    assert nv.mxfp4_dequantize(z(0, 8, dtype=i32), z(0, 2)).shape == (0, 64)
    assert nv.swizzle_scales(z(0, 4)).shape == (0, 4)
    torch.cuda.synchronize()


@pytest.mark.parametrize("mode", ["nvfp4", "mxfp8", "mxfp4"])
def test_qqmm_empty_output(nv, mode):
    K = 256
    cw = K // 4 if mode == "mxfp8" else K // 8
    sc = K // 16 if mode == "nvfp4" else K // 32
    full_c, full_s = z(128, cw, dtype=i32), z(128, sc)
    y = nv.qqmm(z(0, cw, dtype=i32), z(0, sc), full_c, full_s, K, mode)      # M = 0
    assert y.shape == (0, 128)
    y = nv.qqmm(full_c, full_s, z(0, cw, dtype=i32), z(0, sc), K, mode)      # N = 0
    assert y.shape == (128, 0)
    torch.cuda.synchronize()
    nv.check_device_errors()


def test_qmv_no_weight_rows(nv):
    y = nv.qmv(torch.ones(1, 256, dtype=bf16, device="cuda"), z(0, 32, dtype=i32), z(0, 16))
    assert y.shape == (1, 0)
    torch.cuda.synchronize()


@pytest.mark.parametrize("transpose", [True, False])
def test_gather_no_tokens(nv, transpose):
    E, N, K, topk = 4, 64, 128, 2
    wc = z(E, N, K // 8, dtype=i32) if transpose else z(E, K, N // 8, dtype=i32)
    ws = z(E, N, K // 16) if transpose else z(E, K, N // 16)
    y = nv.gather_qmm(z(0, K, dtype=bf16), wc, ws, None, z(0, topk, dtype=i32), transpose=transpose)
    assert y.shape == (0, topk, N)
    if transpose:
        y = nv.gather_qmm_noalloc(z(0, K, dtype=bf16), wc, ws, None, z(0, topk, dtype=i32))
        assert y.shape == (0, topk, N)
    torch.cuda.synchronize()
    nv.check_device_errors()
