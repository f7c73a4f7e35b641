"""GPU parity of qmv (small-M route of qqmm with a pre-quantized NVFP4
weight) against the oracle, through the C ABI."""
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


def run_case(nv, orc, M, N, K, dt, use_g, seed):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal((M, K), 1.0, seed, TORCH_DT[dt])
    w = workloads.normal((N, K), 0.02, seed + 1, TORCH_DT[dt])
    xg, wg = x.cuda(), w.cuda()
    g_x = nv.amax(xg) if use_g else None
    g_w = nv.amax(wg) if use_g else None
    wc, ws = nv.nvfp4_quantize(wg, g_w, "linear")
    y = nv.qmv(xg, wc, ws, g_x, g_w)
    # the oracle quantizes w itself (bit-exactness of that step is tested
    # separately); its qmv uses its own codes
    gx = None if g_x is None else g_x.item()
    gw = None if g_w is None else g_w.item()
    owc, ows = orc.nvfp4_quantize(raw(w), dt, gw)
    assert np.array_equal(raw(wc), owc) and np.array_equal(raw(ws), ows)
    r = orc.qmv(raw(x), dt, gx, owc, ows, gw)
    return check_gemm_output(raw(y), r, dt, orc)


@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("M,N,K", [(1, 64, 256), (1, 200, 1056), (2, 130, 512), (3, 130, 512), (8, 257, 2048),
                                   (1, 33, 32), (5, 1000, 4096)])
@pytest.mark.parametrize("use_g", [True, False])
def test_qmv_parity(nv, orc, dt, M, N, K, use_g):
    run_case(nv, orc, M, N, K, dt, use_g, seed=M * 100 + N + K)


def test_qmv_decode_gemv_full_size(nv, orc):
    """The decode GEMV config: x [1,4096] bf16 N(0,1), W [14336,4096] bf16
    N(0,0.02), g = amax; every output element compared."""
    floor_count = run_case(nv, orc, 1, 14336, 4096, "bf16", True, seed=1)
    assert floor_count < 14336 * 0.01


def test_qmv_worked_example(nv):
    """K = 4096, x = ones, codes 6, block scale 0.5, decode factor 0.1:
    y = 1232.0 ("[Metal] global scale for qmm"); K = 96 gives bf16(28.8)."""
    for K, want in [(4096, 1232.0), (96, 28.75)]:
        x = torch.ones(1, K, dtype=torch.bfloat16).cuda()
        wc = torch.full((2, K // 8), 0x77777777, dtype=torch.int32).cuda()
        ws = torch.full((2, K // 16), 0x30, dtype=torch.uint8).cuda()
        g_x = nv.amax(x)
        g_w = torch.tensor([268.8], dtype=torch.float32).cuda()
        y = nv.qmv(x, wc, ws, g_x, g_w)
        assert torch.all(y.float() == want), (K, y)


def test_qmv_rejects_K_not_multiple_of_32(nv):
    x = torch.ones(1, 48, dtype=torch.bfloat16).cuda()
    wc = torch.zeros(4, 6, dtype=torch.int32).cuda()
    ws = torch.zeros(4, 3, dtype=torch.uint8).cuda()
    with pytest.raises(nv.Nvfp4Error):
        nv.qmv(x, wc, ws)


# Shapes that take the tensor-core path (M <= 2, K % 256 == 0): the weight
# goes to block-scaled MMAs in its stored form, x_hat as two e2m1 planes.
@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("M,N,K", [(1, 130, 4096), (2, 257, 2048), (1, 128, 8192), (2, 384, 256), (1, 1, 512)])
@pytest.mark.parametrize("use_g", [True, False])
def test_qmv_tensor_path_parity(nv, orc, dt, M, N, K, use_g):
    run_case(nv, orc, M, N, K, dt, use_g, seed=7 * M + N + K)


def test_qmv_tensor_path_falls_back_on_subnormal_x_hat(nv, orc):
    """fp16 x around 1e-6 with g_x = amax(x): x_hat lands in fp16's subnormal
    range, where the two-plane form is not exact, so the kernel computes
    these rows on the SIMT cores; the result still matches the oracle."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    M, N, K = 1, 256, 1024
    x = (workloads.normal((M, K), 1.0, 5, torch.float32) * 1e-6).to(torch.float16)
    w = workloads.normal((N, K), 0.02, 6, torch.float16)
    xg, wg = x.cuda(), w.cuda()
    g_x, g_w = nv.amax(xg), nv.amax(wg)
    wc, ws = nv.nvfp4_quantize(wg, g_w, "linear")
    y = nv.qmv(xg, wc, ws, g_x, g_w)
    owc, ows = orc.nvfp4_quantize(raw(w), "f16", g_w.item())
    r = orc.qmv(raw(x), "f16", g_x.item(), owc, ows, g_w.item())
    # the two-plane form really is inexact for this input
    xh = orc.to_f64(orc.nvfp4_quantize_dequantize(raw(x), "f16", g_x.item()), "f16")
    assert np.any((np.abs(xh) < 2.0 ** -14) & (xh != 0))
    check_gemm_output(raw(y), r, "f16", orc)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("M,N,K", [(1, 200, 1024), (2, 130, 512), (1, 14336, 4096)])
def test_qmv_pdl_equals_qmv(nv, dt, M, N, K):
    """qmv_pdl (programmatic dependent launch, weight streamed before the
    previous kernel finishes) computes exactly what qmv computes."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal((M, K), 1.0, 60 + M, TORCH_DT[dt]).cuda()
    w = workloads.normal((N, K), 0.02, 61, TORCH_DT[dt]).cuda()
    g_x, g_w = nv.amax(x), nv.amax(w)
    wc, ws = nv.nvfp4_quantize(w, g_w, "linear")
    torch.cuda.synchronize()  # the weight is written before any qmv_pdl call
    y = nv.qmv(x, wc, ws, g_x, g_w)
    y2 = nv.qmv(x, wc, ws, g_x, g_w, pdl=True)
    nv.check_device_errors()
    assert torch.equal(y.view(torch.int16) if dt == "bf16" else y, y2.view(torch.int16) if dt == "bf16" else y2)


def test_qmv_pdl_chain_orders_reads_and_writes(nv):
    """A chain of qmv_pdl calls where each call's x is the previous call's
    output (read after write) and the last call writes over the first
    call's input (write after read), launched back to back: the same bits as
    the same chain of qmv calls."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    K = 4096
    ws_ = [workloads.normal((K, K), 0.02, 70 + i, torch.bfloat16).cuda() for i in range(3)]
    q = [nv.nvfp4_quantize(w, None, "linear") for w in ws_]
    torch.cuda.synchronize()

    def chain(pdl):
        a = workloads.normal((1, K), 1.0, 80, torch.bfloat16).cuda()
        b = torch.empty_like(a)
        c = torch.empty_like(a)
        torch.cuda.synchronize()
        for _ in range(4):
            nv.qmv(a, *q[0], out=b, pdl=pdl)   # b = f(a)
            nv.qmv(b, *q[1], out=c, pdl=pdl)   # c = f(b): reads what the call before wrote
            nv.qmv(c, *q[2], out=a, pdl=pdl)   # a = f(c): overwrites the first call's input
        torch.cuda.synchronize()
        return a, b, c
    want = chain(False)
    got = chain(True)
    nv.check_device_errors()
    for u, v in zip(want, got):
        assert torch.equal(u.view(torch.int16), v.view(torch.int16))


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("M,N,K", [(1, 200, 256), (2, 130, 1024), (3, 77, 96), (8, 257, 2048), (1, 4096, 4096)])
def test_qmv_mx_parity(nv, orc, mode, dt, M, N, K):
    """qmv in the MX modes against the oracle (x quantize-dequantized with
    the mode's 32-blocks and e8m0 scales, the weight decoded exactly)."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.normal((M, K), 1.0, 90 + M + K, TORCH_DT[dt])
    w = workloads.normal((N, K), 0.02, 91 + N, TORCH_DT[dt])
    quant = nv.mxfp8_quantize if mode == "mxfp8" else nv.mxfp4_quantize
    oquant = orc.mxfp8_quantize if mode == "mxfp8" else orc.mxfp4_quantize
    wc, ws = quant(w.cuda(), "linear")
    y = nv.qmv_mx(x.cuda(), wc, ws, mode)
    nv.check_device_errors()
    owc, ows = oquant(raw(w), dt)
    assert np.array_equal(raw(wc), owc) and np.array_equal(raw(ws), ows)
    r = orc.qmv_mx(raw(x), dt, owc, ows, mode)
    check_gemm_output(raw(y), r, dt, orc)
