"""GPU parity of gather_qmm with transpose=False (weights stored [E, K, N],
quantized along N; the tensor-core kernel reads the dequantized weight as an
MN-major operand) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from helpers import check_gemm_output, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4


def make_case(nv, orc, T, topk, E, N, K, use_g, seed, idx=None):
    """w [E, K, N] bf16, quantized per expert along N on the GPU; the
    oracle's own quantization of the same values."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    w = workloads.normal((E, K, N), 0.02, seed, torch.bfloat16)
    x = workloads.normal((T, K), 1.0, seed + 1, torch.bfloat16)
    if idx is None:
        idx = workloads.routing(T, E, topk, seed + 2)
    wg = w.cuda()
    g = torch.stack([nv.amax(wg[e]) for e in range(E)]).view(E) if use_g else None
    wc = torch.empty(E, K, N // 8, dtype=torch.int32, device="cuda")
    ws = torch.empty(E, K, N // 16, dtype=torch.uint8, device="cuda")
    for e in range(E):
        nv.nvfp4_quantize(wg[e], None if g is None else g[e:e + 1], "linear", wc[e], ws[e])
    gs = None if g is None else g.cpu().numpy()
    oc, os_ = zip(*[orc.nvfp4_quantize(raw(w[e]), "bf16", None if gs is None else float(gs[e])) for e in range(E)])
    oc, os_ = np.stack(oc), np.stack(os_)
    assert np.array_equal(raw(wc).reshape(oc.shape), oc) and np.array_equal(raw(ws), os_)
    return x, idx, g, wc, ws, oc, os_, gs


@pytest.mark.parametrize("T,topk,E,N,K", [(64, 2, 4, 256, 256), (200, 3, 7, 288, 192), (130, 1, 3, 512, 2048),
                                          (300, 8, 16, 1408, 128), (5, 2, 4, 96, 64), (1, 1, 2, 32, 512)])
@pytest.mark.parametrize("use_g", [True, False])
def test_gather_qmm_kn_parity(nv, orc, T, topk, E, N, K, use_g):
    x, idx, g, wc, ws, oc, os_, gs = make_case(nv, orc, T, topk, E, N, K, use_g, seed=T + E + N + K)
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda(), transpose=False)
    nv.check_device_errors()
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy(), transpose=False)
    check_gemm_output(raw(y), r, "bf16", orc)


def test_gather_qmm_kn_worked_example(nv):
    """The pages' worked example laid out [K, N]: codes 6, block scale 0.5
    (blocks along N), decode factor 0.1 for expert 0 and 1 for expert 1;
    x = ones, K = 192: the weight rounds to bf16 0.30078125 first, so
    y = 192 * 0.30078125 = 57.75 (expert 0) and 192 * 3 = 576 (expert 1)."""
    K, N, E = 192, 64, 2
    wc = torch.full((E, K, N // 8), 0x77777777, dtype=torch.int32).cuda()
    ws = torch.full((E, K, N // 16), 0x30, dtype=torch.uint8).cuda()
    g = torch.tensor([268.8, 2688.0], dtype=torch.float32).cuda()
    x = torch.ones(3, K, dtype=torch.bfloat16).cuda()
    idx = torch.tensor([[0, 1], [1, 0], [0, 1]], dtype=torch.int32).cuda()
    y = nv.gather_qmm(x, wc, ws, g, idx, transpose=False).float().cpu()
    nv.check_device_errors()
    want = torch.where(idx.cpu() == 0, 57.75, 576.0)
    assert torch.equal(y, want[:, :, None].expand(3, 2, N))


def test_gather_qmm_kn_full_size_sampled_tokens(nv, orc):
    """The MoE config with the weights stored [E, K, N]: 64 experts [2048, 1408],
    4096 tokens top-8; 48 sampled tokens checked against the oracle."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    T, topk, E, N, K = 4096, 8, 64, 1408, 2048
    x, idx, g, wc, ws, oc, os_, gs = make_case(nv, orc, T, topk, E, N, K, True, seed=5)
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda(), transpose=False)
    nv.check_device_errors()
    tok = np.sort(np.random.default_rng(4).choice(T, 48, replace=False))
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy(), tokens=tok, transpose=False)
    check_gemm_output(raw(y)[tok], r, "bf16", orc)


def test_gather_qmm_kn_rejects_n_not_multiple_of_32(nv):
    x = torch.ones(4, 64, dtype=torch.bfloat16, device="cuda")
    wc = torch.zeros(1, 64, 2, dtype=torch.int32, device="cuda")
    ws = torch.zeros(1, 64, 1, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(4, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="N of 32"):
        nv.gather_qmm(x, wc, ws, None, idx, transpose=False)
