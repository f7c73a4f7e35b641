"""The allocation-free gather_qmm entry point (gather_qmm_noalloc).

Some callers cannot allocate device memory themselves -- a host program
that fixes its device memory budget at start-up, or plugin code with no
handle on its framework's allocator -- so the library offers a gather_qmm
that works out of a static scratch array it owns.  These tests call it
through the C ABI and check its output against gather_qmm with a
caller-provided workspace, on two calls in a row with different routings
(the scratch keeps the first call's contents, which the second call must
not see).  This file is named to be collected last.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4


def _case(nv, T, topk, E, N, K, seed):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    w = workloads.normal((E, N, K), 0.02, seed, torch.bfloat16, "cuda")
    x = workloads.normal((T, K), 1.0, seed + 1, torch.bfloat16, "cuda")
    idx = workloads.routing(T, E, topk, seed + 2, "cuda")
    g = torch.stack([nv.amax(w[e]) for e in range(E)]).view(E)
    wc = torch.empty(E, N, K // 8, dtype=torch.int32, device="cuda")
    ws = torch.empty(E, N, K // 16, dtype=torch.uint8, device="cuda")
    for e in range(E):
        nv.nvfp4_quantize(w[e], g[e:e + 1], "linear", wc[e], ws[e])
    return x, wc, ws, g, idx


def _noalloc_raw(nv, x, wc, ws, g, idx, y):
    """Direct C-ABI call of gather_qmm_noalloc (ctypes, device pointers)."""
    L = nv.lib()
    T, K = x.shape
    E, N = wc.shape[0], wc.shape[1]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return L.gather_qmm_noalloc(p(x), p(wc), p(ws), p(g), p(idx), T, idx.shape[1], E, N, K, p(y),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b):
    """Within one bf16 ulp elementwise (the output tolerance of the GEMM tests)."""
    a, b = a.float(), b.float()
    ulp = torch.exp2(torch.floor(torch.log2(b.abs().clamp_min(2.0 ** -126))) - 7)
    return bool(torch.all((a - b).abs() <= ulp))


def test_noalloc_matches_workspace_entry_point_twice(nv):
    # calls in a row with different routing: the decode path (T <= 16 tokens,
    # its tile list and permutation in the static scratch) first, then larger
    # calls that would read any stale tile entries it left
    cases = [(8, 4, 8, 256, 256, 10), (256, 8, 16, 512, 256, 11), (96, 2, 5, 128, 512, 12)]
    for T, topk, E, N, K, seed in cases:
        x, wc, ws, g, idx = _case(nv, T, topk, E, N, K, seed)
        want = nv.gather_qmm(x, wc, ws, g, idx)
        got = torch.full_like(want, float("nan"))
        st = _noalloc_raw(nv, x, wc, ws, g, idx, got)
        assert st == nv.OK, nv.lib().nvfp4_last_error_message()
        nv.check_device_errors()
        assert _close(got, want)


def test_noalloc_rejects_scratch_beyond_its_size(nv):
    T, topk, E, N, K = 65536, 8, 64, 128, 256  # ~2.2 MB of routing scratch > 1 MiB
    assert nv.gather_qmm_workspace_size(T, topk, E) > (1 << 20)
    x = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")  # never read: rejected first
    wc = torch.zeros(E, N, K // 8, dtype=torch.int32, device="cuda")
    ws = torch.zeros(E, N, K // 16, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(16, topk, dtype=torch.int32, device="cuda")
    y = torch.zeros(16, topk, N, dtype=torch.bfloat16, device="cuda")
    L = nv.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = L.gather_qmm_noalloc(p(x), p(wc), p(ws), None, p(idx), T, topk, E, N, K, p(y),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nv.ERR_UNSUPPORTED
    assert "static scratch" in L.nvfp4_last_error_message().decode()


def test_noalloc_against_the_oracle(nv, orc):
    """One decode-size and one tensor-core-size call compared with the CPU
    oracle's gather_qmm on the oracle's own quantization of the same seeded
    weights (the tolerance of the other GEMM tests)."""
    import numpy as np
    from helpers import check_gemm_output, raw
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    for T, topk, E, N, K, seed in [(12, 2, 6, 128, 256, 21), (80, 3, 7, 272, 192, 22)]:
        w = workloads.normal((E, N, K), 0.02, seed, torch.bfloat16)
        x = workloads.normal((T, K), 1.0, seed + 1, torch.bfloat16)
        idx = workloads.routing(T, E, topk, seed + 2)
        wg = w.cuda()
        g = torch.stack([nv.amax(wg[e]) for e in range(E)]).view(E)
        wc = torch.empty(E, N, K // 8, dtype=torch.int32, device="cuda")
        ws = torch.empty(E, N, K // 16, dtype=torch.uint8, device="cuda")
        for e in range(E):
            nv.nvfp4_quantize(wg[e], g[e:e + 1], "linear", wc[e], ws[e])
        y = torch.empty(T, topk, N, dtype=torch.bfloat16, device="cuda")
        assert _noalloc_raw(nv, x.cuda(), wc, ws, g, idx.cuda(), y) == nv.OK
        nv.check_device_errors()
        gs = np.array([orc.amax(raw(w[e]), "bf16") for e in range(E)], dtype=np.float32)
        q = [orc.nvfp4_quantize(raw(w[e]), "bf16", float(gs[e])) for e in range(E)]
        oc, os_ = np.stack([c for c, _ in q]), np.stack([s for _, s in q])
        assert np.array_equal(raw(wc).reshape(oc.shape), oc)
        r = orc.gather_qmm(raw(x), oc, os_, gs, idx.numpy())
        check_gemm_output(raw(y), r, "bf16", orc)


def test_noalloc_leaves_free_device_memory_unchanged(nv):
    """After a warm-up call, a call changes nothing in the device's free
    memory (cudaMemGetInfo): the entry point allocates nothing."""
    x, wc, ws, g, idx = _case(nv, 64, 4, 8, 256, 256, 31)
    y = torch.empty(64, 4, 256, dtype=torch.bfloat16, device="cuda")
    assert _noalloc_raw(nv, x, wc, ws, g, idx, y) == nv.OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc_raw(nv, x, wc, ws, g, idx, y) == nv.OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    nv.check_device_errors()
