"""The bounded-wait timeout path of the dense GEMM, exercised on the GPU.

Every mbarrier wait in the tensor-core kernels gives up after a fixed number
of polls, sets the device error word and lets the kernel drain and free its
tensor memory, so a stuck pipeline ends in NVFP4_ERR_TIMEOUT instead of a
hang.  Here a test build of the library (compiled by the test into a
temporary directory) lowers the poll limit and withholds one pipeline stage
of CTA 0: neither its arrival nor any copy is issued, so the MMA warp's wait
on that stage runs out.  Nothing faults, nothing hangs, no copy is left in
flight (nothing is issued for the withheld stage).  The test expects
NVFP4_ERR_TIMEOUT from nvfp4_check_device_errors, a cleared word on the next
check, and a normal GEMM through the library afterwards.
"""
import ctypes
import os
import subprocess

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


@pytest.fixture(scope="module")
def withheld_lib(tmp_path_factory):
    """libnvfp4 built with a 65536-poll wait limit and stage 1 of CTA 0's
    GEMM pipeline withheld."""
    from mxfp8_block_scaled_nvfp4_b200 import build
    from mxfp8_block_scaled_nvfp4_b200 import nvfp4 as nvmod
    out = str(tmp_path_factory.mktemp("withheld") / "libnvfp4_withheld.so")
    cmd = [build.NVCC, *build.FLAGS, "-DNVFP4_WAIT_LIMIT=65536u", "-DNVFP4_TEST_WITHHOLD_STAGE=1",
           "-I", build.INCLUDE, "-I", build.CSRC, os.path.join(build.CSRC, "nvfp4_abi.cu"), "-o", out]
    subprocess.check_call(cmd)
    L = ctypes.CDLL(out)
    for name, res, args in nvmod.SIGNATURES:
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


def test_withheld_stage_ends_in_timeout_status(nv, orc, withheld_lib):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    M, N, K = 128, 256, 2048  # 8 pipeline stages per tile
    x = workloads.normal((M, K), 1.0, 41, torch.bfloat16)
    w = workloads.normal((N, K), 0.02, 42, torch.bfloat16)
    xg, wg = x.cuda(), w.cuda()
    g_x, g_w = nv.amax(xg), nv.amax(wg)
    xc, xs = nv.nvfp4_quantize(xg, g_x, "swizzled")
    wc, ws = nv.nvfp4_quantize(wg, g_w, "swizzled")
    y = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    L = withheld_lib
    st = L.qqmm(0, M, N, K, p(xc), p(xs), p(wc), p(ws), p(g_x), p(g_w), p(y), 0, stream)
    assert st == nv.OK, L.nvfp4_last_error_message()
    st = L.nvfp4_check_device_errors(stream)
    assert st == nv.ERR_TIMEOUT, (st, L.nvfp4_last_error_message())
    assert b"bounded wait" in L.nvfp4_last_error_message()
    assert L.nvfp4_check_device_errors(stream) == nv.OK  # the word was cleared
    # the context is still usable: the library's own GEMM on the same operands
    y2 = nv.qqmm(xc, xs, wc, ws, K, "nvfp4", g_x, g_w, out_dtype=torch.float32)
    nv.check_device_errors()
    gx, gw = g_x.item(), g_w.item()
    oxc, oxs = orc.nvfp4_quantize(raw(x), "bf16", gx)
    owc, ows = orc.nvfp4_quantize(raw(w), "bf16", gw)
    assert np.array_equal(raw(xc), oxc) and np.array_equal(raw(wc), owc)
    check_gemm_output(raw(y2), orc.qqmm(oxc, oxs, owc, ows, "nvfp4", gx, gw, "f32"), "f32", orc)
