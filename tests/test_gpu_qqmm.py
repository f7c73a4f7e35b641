"""GPU parity of the dense block-scaled GEMM (tcgen05) against the oracle,
through the C ABI: NVFP4 with and without global scales, MXFP8, ragged M, N
and K, every output dtype; full-size configs on sampled rows."""
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


def quantized_operands(nv, orc, x, w, mode, use_g):
    """GPU-quantized operands (SWIZZLED) and the oracle's own (LINEAR)."""
    xg, wg = x.cuda(), w.cuda()
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[x.dtype]
    if mode == "nvfp4":
        g_x = nv.amax(xg) if use_g else None
        g_w = nv.amax(wg) if use_g else None
        xc, xs = nv.nvfp4_quantize(xg, g_x, "swizzled")
        wc, ws = nv.nvfp4_quantize(wg, g_w, "swizzled")
        gx = None if g_x is None else g_x.item()
        gw = None if g_w is None else g_w.item()
        o = (orc.nvfp4_quantize(raw(x), dt, gx), orc.nvfp4_quantize(raw(w), dt, gw), gx, gw)
    else:
        g_x = g_w = None
        xc, xs = nv.mxfp8_quantize(xg, "swizzled")
        wc, ws = nv.mxfp8_quantize(wg, "swizzled")
        o = (orc.mxfp8_quantize(raw(x), dt), orc.mxfp8_quantize(raw(w), dt), None, None)
    return (xc, xs, wc, ws, g_x, g_w), o


def run(nv, orc, M, N, K, mode, use_g, out_dt, seed, in_dt=torch.bfloat16, rows=None):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal((M, K), 1.0, seed, in_dt)
    w = workloads.normal((N, K), 0.02 if mode == "nvfp4" else 1.0, seed + 1, in_dt)
    (xc, xs, wc, ws, g_x, g_w), ((oxc, oxs), (owc, ows), gx, gw) = quantized_operands(nv, orc, x, w, mode, use_g)
    y = nv.qqmm(xc, xs, wc, ws, K, mode, g_x, g_w, out_dtype=TORCH_DT[out_dt])
    nv.check_device_errors()
    if rows is None:
        r = orc.qqmm(oxc, oxs, owc, ows, mode, gx, gw, out_dt)
        return check_gemm_output(raw(y), r, out_dt, orc)
    r = orc.qqmm(oxc, oxs, owc, ows, mode, gx, gw, out_dt, rows=rows)
    return check_gemm_output(raw(y)[rows], r, out_dt, orc)


def test_tiny_config(nv, orc):
    """x [4,256], w [64,256] fp32 N(0,1) (seed 0), g = amax, y fp32."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("tiny")
    x, w = d["x"], d["w"]
    (xc, xs, wc, ws, g_x, g_w), ((oxc, oxs), (owc, ows), gx, gw) = quantized_operands(nv, orc, x, w, "nvfp4", True)
    assert np.array_equal(raw(xc), oxc) and np.array_equal(raw(wc), owc)
    y = nv.qqmm(xc, xs, wc, ws, 256, "nvfp4", g_x, g_w, out_dtype=torch.float32)
    nv.check_device_errors()
    r = orc.qqmm(oxc, oxs, owc, ows, "nvfp4", gx, gw, "f32")
    check_gemm_output(raw(y), r, "f32", orc)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (67, 64, 256), (130, 300, 1056), (256, 512, 4096),
                                   (1, 256, 512), (200, 520, 96), (384, 136, 2048)])
@pytest.mark.parametrize("use_g", [True, False])
@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
def test_nvfp4_qqmm_parity(nv, orc, M, N, K, use_g, out_dt):
    run(nv, orc, M, N, K, "nvfp4", use_g, out_dt, seed=M + 7 * N + K)


@pytest.mark.parametrize("mode", ["nvfp4", "mxfp8"])
def test_qqmm_split_last_wave(nv, orc, mode):
    """20 x 9 = 180 tiles of 128 x 256 on 148 SMs: the last 32 run as 128 x
    128 halves (wide and narrow units in one launch), with ragged M and N
    (the last narrow half holds 28 columns), compared in full."""
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the tile count is chosen for 148 SMs")
    run(nv, orc, 2555, 2204, 256, mode, mode == "nvfp4", "bf16", seed=11)


@pytest.mark.parametrize("in_dt", [torch.float32, torch.float16])
def test_nvfp4_qqmm_input_dtypes_f16_out(nv, orc, in_dt):
    run(nv, orc, 130, 260, 512, "nvfp4", True, "f16", seed=3, in_dt=in_dt)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (67, 300, 1056), (256, 256, 4096), (200, 72, 96)])
@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
def test_mxfp8_qqmm_parity(nv, orc, M, N, K, out_dt):
    run(nv, orc, M, N, K, "mxfp8", False, out_dt, seed=M + N + K)


def test_prefill_config_sampled_rows(nv, orc):
    """x [4096,4096] bf16 N(0,1), W [4096,4096] bf16 N(0,0.02) with 1% x50
    outliers, g = amax, SWIZZLED scales, y bf16: 64 random rows x all N."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("prefill")
    x, w = d["x"], d["w"]
    (xc, xs, wc, ws, g_x, g_w), ((oxc, oxs), (owc, ows), gx, gw) = quantized_operands(nv, orc, x, w, "nvfp4", True)
    assert np.array_equal(raw(wc), owc) and np.array_equal(raw(xc), oxc)
    y = nv.qqmm(xc, xs, wc, ws, 4096, "nvfp4", g_x, g_w, out_dtype=torch.bfloat16)
    nv.check_device_errors()
    rows = np.sort(np.random.default_rng(1).choice(4096, 64, replace=False))
    r = orc.qqmm(oxc, oxs, owc, ows, "nvfp4", gx, gw, "bf16", rows=rows)
    n_floor = check_gemm_output(raw(y)[rows], r, "bf16", orc)
    # The same GEMM with fp32 output: every sampled element within the fp32
    # tolerance (no bf16 slack), and the bf16 output equal, bit for bit, to
    # the round-to-nearest-even bf16 of the fp32 output everywhere.  So the
    # elements the bf16 check accepted only through the fp32 floor are fp32
    # sums within tolerance that sit next to a bf16 rounding boundary.
    y32 = nv.qqmm(xc, xs, wc, ws, 4096, "nvfp4", g_x, g_w, out_dtype=torch.float32)
    nv.check_device_errors()
    r32 = orc.qqmm(oxc, oxs, owc, ows, "nvfp4", gx, gw, "f32", rows=rows)
    check_gemm_output(raw(y32)[rows], r32, "f32", orc)
    assert torch.equal(y32.to(torch.bfloat16).view(torch.int16), y.view(torch.int16))
    print(f"prefill bf16: {n_floor} of {rows.size * 4096} sampled outputs accepted through the fp32 floor")


def test_mxfp8_config_sampled_rows(nv, orc):
    """x, W [8192,8192] bf16 N(0,1), E8M0 round-up, e4m3 codes, y bf16:
    32 random rows x all N."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("mxfp8", device="cuda")
    x, w = d["x"], d["w"]
    xc, xs = nv.mxfp8_quantize(x, "swizzled")
    wc, ws = nv.mxfp8_quantize(w, "swizzled")
    y = nv.qqmm(xc, xs, wc, ws, 8192, "mxfp8", out_dtype=torch.bfloat16)
    nv.check_device_errors()
    rows = np.sort(np.random.default_rng(2).choice(8192, 32, replace=False))
    oxc, oxs = orc.mxfp8_quantize(raw(x[torch.from_numpy(rows).cuda()]), "bf16")
    owc, ows = orc.mxfp8_quantize(raw(w), "bf16")
    r = orc.qqmm(oxc, oxs, owc, ows, "mxfp8", None, None, "bf16")
    check_gemm_output(raw(y)[rows], r, "bf16", orc)
