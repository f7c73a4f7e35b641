"""GPU parity of gather_qmm (MoE matmul with per-expert NVFP4 weights and
per-expert global scales) against the oracle, through the C ABI."""
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


def make_case(nv, T, topk, E, N, K, use_g, seed, idx=None):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    w = workloads.normal((E, N, K), 0.02, seed, torch.bfloat16)
    x = workloads.normal((T, K), 1.0, seed + 1, torch.bfloat16)
    if idx is None:
        idx = workloads.routing(T, E, topk, seed + 2)
    wg = w.cuda()
    g = torch.stack([nv.amax(wg[e]) for e in range(E)]).view(E) if use_g else None
    wc = torch.empty(E, N, K // 8, dtype=torch.int32, device="cuda")
    ws = torch.empty(E, N, K // 16, dtype=torch.uint8, device="cuda")
    for e in range(E):
        nv.nvfp4_quantize(wg[e], None if g is None else g[e:e + 1], "linear", wc[e], ws[e])
    return x, w, idx, g, wc, ws


def oracle_operands(orc, w, g):
    E = w.shape[0]
    gs = None if g is None else g.cpu().numpy()
    oc, os_ = [], []
    for e in range(E):
        c, s = orc.nvfp4_quantize(raw(w[e]), "bf16", None if gs is None else float(gs[e]))
        oc.append(c)
        os_.append(s)
    return np.stack(oc), np.stack(os_), gs


@pytest.mark.parametrize("T,topk,E,N,K", [(64, 2, 4, 128, 256), (200, 3, 7, 272, 192), (130, 1, 3, 512, 2048),
                                          (300, 8, 16, 1408, 128)])
@pytest.mark.parametrize("use_g", [True, False])
@pytest.mark.parametrize("staged", [True, False])  # SM-pair kernel on staged rows / single-SM gathering kernel
def test_gather_qmm_parity(nv, orc, T, topk, E, N, K, use_g, staged):
    x, w, idx, g, wc, ws = make_case(nv, T, topk, E, N, K, use_g, seed=T + E + N)
    size = (nv.gather_qmm_staged_workspace_size if staged else
            lambda T, topk, E, K: nv.gather_qmm_workspace_size(T, topk, E))(T, topk, E, K)
    work = torch.empty(size, dtype=torch.uint8, device="cuda")
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda(), workspace=work)
    nv.check_device_errors()
    oc, os_, gs = oracle_operands(orc, w, g)
    assert np.array_equal(raw(wc).reshape(oc.shape), oc)
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy())
    check_gemm_output(raw(y), r, "bf16", orc)


def test_gather_qmm_experts_without_tokens(nv, orc):
    """Only experts 1 and 5 of 8 receive tokens."""
    T, topk, E, N, K = 40, 2, 8, 64, 128
    idx = torch.tensor([[1, 5]] * T, dtype=torch.int32)
    x, w, idx, g, wc, ws = make_case(nv, T, topk, E, N, K, True, seed=9, idx=idx)
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda())
    nv.check_device_errors()
    oc, os_, gs = oracle_operands(orc, w, g)
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy())
    check_gemm_output(raw(y), r, "bf16", orc)


@pytest.mark.parametrize("T", [3, 24])  # the decode kernel and the tensor-core kernel
def test_gather_worked_example_bf16_before_the_sum(nv, T):
    """"[Metal] global scale for qmm": codes 6, block scale 0.5, decode factor
    0.1; the weight rounds to bf16 0.30078125 before the matmul, so x = ones
    with K = 192 gives 192 * 0.30078125 = 57.75 (scaling after the matmul
    would give bf16(57.6) = 57.5)."""
    K, N, E = 192, 16, 2
    wc = torch.full((E, N, K // 8), 0x77777777, dtype=torch.int32).cuda()
    ws = torch.full((E, N, K // 16), 0x30, dtype=torch.uint8).cuda()
    g = torch.tensor([268.8, 2688.0], dtype=torch.float32).cuda()
    x = torch.ones(T, K, dtype=torch.bfloat16).cuda()
    idx = torch.tensor([[t % 2, 1 - t % 2] for t in range(T)], dtype=torch.int32).cuda()
    y = nv.gather_qmm(x, wc, ws, g, idx).float().cpu()
    for t in range(T):
        for j in range(2):
            want = 57.75 if idx[t, j].item() == 0 else 192 * 3.0
            assert torch.all(y[t, j] == want), (t, j, y[t, j, :4])


@pytest.mark.parametrize("T", [8, 40])  # the decode kernel and the tensor-core kernel
def test_gather_out_of_range_expert_sets_error_and_zero_rows(nv, T):
    topk, E, N, K = 2, 4, 32, 64
    x, w, idx, g, wc, ws = make_case(nv, T, topk, E, N, K, True, seed=4)
    idx = idx.clone()
    idx[3, 1] = E  # out of range
    idx[5, 0] = -1
    y = torch.full((T, topk, N), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda(), out=y)
    with pytest.raises(nv.Nvfp4Error) as ei:
        nv.check_device_errors()
    assert ei.value.status == nv.ERR_DEVICE_INDEX
    assert torch.all(y[3, 1] == 0) and torch.all(y[5, 0] == 0)
    assert torch.all(y[3, 0] != 7.0)
    nv.check_device_errors()  # the error word was cleared


def test_moe_config_sampled_tokens(nv, orc):
    """64 experts W_e [1408, 2048] N(0,0.02), g_e = amax(W_e); x [4096, 2048]
    bf16 N(0,1); top-8 uniform routing; 48 random tokens compared."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    d = workloads.make("moe", device="cpu")
    x, w, idx = d["x"], d["w"], d["idx"]
    E, N, K = w.shape
    wg = w.cuda()
    g = torch.stack([nv.amax(wg[e]) for e in range(E)]).view(E)
    wc = torch.empty(E, N, K // 8, dtype=torch.int32, device="cuda")
    ws = torch.empty(E, N, K // 16, dtype=torch.uint8, device="cuda")
    for e in range(E):
        nv.nvfp4_quantize(wg[e], g[e:e + 1], "linear", wc[e], ws[e])
    del wg
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda())
    nv.check_device_errors()
    tokens = np.sort(np.random.default_rng(3).choice(x.shape[0], 48, replace=False))
    oc, os_, gs = oracle_operands(orc, w, g)
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy(), tokens=tokens)
    check_gemm_output(raw(y)[tokens], r, "bf16", orc)


# Decode: T <= 16 tokens take the gather_qmv kernel (a warp per expert weight
# row, the same bf16 rounding of the dequantized weight); same oracle.
@pytest.mark.parametrize("T,topk,E,N,K", [(1, 8, 64, 192, 256), (2, 4, 8, 272, 512), (4, 8, 16, 128, 2048),
                                          (16, 2, 5, 64, 128), (3, 3, 7, 1408, 192)])
@pytest.mark.parametrize("use_g", [True, False])
def test_gather_qmv_decode_parity(nv, orc, T, topk, E, N, K, use_g):
    x, w, idx, g, wc, ws = make_case(nv, T, topk, E, N, K, use_g, seed=3 * T + E + N)
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda())
    nv.check_device_errors()
    oc, os_, gs = oracle_operands(orc, w, g)
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy())
    check_gemm_output(raw(y), r, "bf16", orc)


def test_gather_qmv_decode_full_size_experts(nv, orc):
    """64 experts W_e [1408, 2048] N(0,0.02), g_e = amax(W_e), 4 tokens, top-8:
    every output element compared."""
    x, w, idx, g, wc, ws = make_case(nv, 4, 8, 64, 1408, 2048, True, seed=41)
    y = nv.gather_qmm(x.cuda(), wc, ws, g, idx.cuda())
    nv.check_device_errors()
    oc, os_, gs = oracle_operands(orc, w, g)
    r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy())
    check_gemm_output(raw(y), r, "bf16", orc)


def test_gather_qmv_repeated_expert_and_boundary(nv, orc):
    """A token routed twice to the same expert (more pairs per expert than
    tokens), and T = 16 (decode kernel) vs T = 17 (MMA kernel) on the same
    weights: both match the oracle."""
    E, N, K, topk = 6, 96, 256, 3
    idx = torch.tensor([[2, 2, 5]] + [[i % E, (i + 1) % E, 2] for i in range(16)], dtype=torch.int32)
    x, w, _, g, wc, ws = make_case(nv, 17, topk, E, N, K, True, seed=77, idx=idx)
    oc, os_, gs = oracle_operands(orc, w, g)
    for T in (16, 17):
        y = nv.gather_qmm(x[:T].cuda(), wc, ws, g, idx[:T].cuda())
        nv.check_device_errors()
        r = orc.gather_qmm(raw(x[:T]), oc, os_, gs, idx[:T].numpy())
        check_gemm_output(raw(y), r, "bf16", orc)
