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
    cases = [(256, 8, 16, 512, 256, 11), (96, 2, 5, 128, 512, 12)]
    for T, topk, E, N, K, seed in cases:  # two calls in a row, different routing
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
