"""The C-ABI library loads, exports every symbol include/nvfp4.h declares, and
rejects bad arguments on the host (no GPU needed: argument checks run before
any device call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ["nvfp4_amax", "nvfp4_quantize", "nvfp4_dequantize", "mxfp8_quantize", "qqmm", "qmv",
              "gather_qmm", "gather_qmm_workspace_size", "nvfp4_check_device_errors"]:
        assert s in syms


def test_library_exports_every_declared_symbol(L):
    for s in declared_symbols():
        assert hasattr(L, s), s


def test_binding_signatures_cover_the_header():
    from mxfp8_block_scaled_nvfp4_b200 import nvfp4
    assert sorted(n for n, _, _ in nvfp4.SIGNATURES) == declared_symbols()


def test_status_strings(L):
    assert L.nvfp4_status_string(0) == b"ok"
    assert b"invalid" in L.nvfp4_status_string(1)


A = 0x10000  # a fake, 16-byte aligned device address: never dereferenced


def msg(L):
    return L.nvfp4_last_error_message().decode()


def test_qqmm_requires_both_global_scales_or_neither(L):
    st = L.qqmm(0, 128, 128, 256, A, A, A, A, A, None, A, 2, None)
    assert st == 1
    assert msg(L) == ("[qqmm] For nvfp4 mode, either both global_scale_x and global_scale_w "
                      "must be provided, or neither.")
    st = L.qqmm(0, 128, 128, 256, A, A, A, A, None, A, A, 2, None)
    assert st == 1


def test_global_scale_only_for_nvfp4(L):
    st = L.qqmm(1, 128, 128, 256, A, A, A, A, A, A, A, 2, None)
    assert st == 1 and "only supported for 'nvfp4'" in msg(L)


def test_qqmm_K_multiple_of_32(L):
    assert L.qqmm(0, 128, 128, 48, A, A, A, A, None, None, A, 2, None) == 1


def test_quantize_group_divisibility_and_alignment(L):
    assert L.nvfp4_quantize(A, 2, 4, 24, None, A, A, 0, None) == 1
    assert "divisible by the quantization group size 16" in msg(L)
    assert L.mxfp8_quantize(A, 2, 4, 48, A, A, 0, None) == 1
    assert L.nvfp4_quantize(A + 8, 2, 4, 32, None, A, A, 0, None) == 1
    assert "aligned" in msg(L)


def test_bad_dtype_and_layout(L):
    assert L.nvfp4_quantize(A, 7, 4, 32, None, A, A, 0, None) == 2
    assert L.nvfp4_quantize(A, 2, 4, 32, None, A, A, 5, None) == 1
    assert L.nvfp4_dequantize(A, A, 0, 4, 32, None, A, 9, None) == 2


def test_qmv_bounds(L):
    assert L.qmv(A, 2, None, A, A, None, 9, 64, 256, A, None) == 1  # M > 8
    assert L.qmv(A, 2, A, A, A, None, 1, 64, 256, A, None) == 1  # one global scale only
    assert L.qmv(A, 2, None, A, A, None, 1, 64, 65536, A, None) == 2  # x_hat too large


def test_gather_workspace_and_shape_checks(L):
    ws = L.gather_qmm_workspace_size(4096, 8, 64)
    assert ws > 0
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 4, 64, 96, A, A, ws, None) == 1  # K % 64
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 4, 64, 128, A, A, 0, None) == 1  # workspace


def test_header_declares_the_next_rows():
    syms = declared_symbols()
    for sname in ["nvfp4_quantize_columnwise", "nvfp4_quantize_sr", "mxfp4_quantize", "mxfp4_dequantize",
                  "mxfp8_dequantize", "gather_qmm_kn"]:
        assert sname in syms


def test_mxfp4_checks(L):
    # 32-element groups
    assert L.mxfp4_quantize(A, 2, 4, 48, A, A, 0, None) == 1
    assert "group size 32" in msg(L)
    assert L.mxfp4_dequantize(A, A, 0, 4, 48, A, 2, None) == 1
    assert L.mxfp4_quantize(A, 7, 4, 64, A, A, 0, None) == 2  # dtype
    # qqmm in mxfp4 mode takes no global scale; an unknown mode is rejected
    assert L.qqmm(2, 128, 128, 256, A, A, A, A, A, A, A, 2, None) == 1
    assert "only supported for 'nvfp4'" in msg(L)
    assert L.qqmm(3, 128, 128, 256, A, A, A, A, None, None, A, 2, None) == 1
    assert "'mxfp4'" in msg(L)


def test_quantize_sr_checks(L):
    assert L.nvfp4_quantize_sr(A, 2, 4, 24, None, 7, A, A, 0, None) == 1
    assert "divisible by the quantization group size 16" in msg(L)
    assert L.nvfp4_quantize_sr(A, 2, 4, 32, None, 7, A, A, 5, None) == 1  # layout
    assert L.nvfp4_quantize_sr(A + 8, 2, 4, 32, None, 7, A, A, 0, None) == 1
    assert "aligned" in msg(L)
    # column-wise: the quantized dimension is the rows of x
    assert L.nvfp4_quantize_columnwise_sr(A, 2, 24, 4, None, 7, A, A, 0, None) == 1
    assert "group size 16" in msg(L)
    assert L.nvfp4_quantize_columnwise_sr(A, 2, 32, 4, None, 7, A, A, 5, None) == 1  # layout
    assert L.nvfp4_quantize_columnwise_sr(None, 2, 32, 0, None, 7, None, None, 1, None) == 0  # empty
    assert L.nvfp4_quantize_columnwise_sr(A, 2, 32, 4, None, 7, A, A, 0, None) not in (0, 1, 2)  # needs a device


def test_gather_kn_checks(L):
    ws = L.gather_qmm_workspace_size(64, 2, 4)
    assert L.gather_qmm_kn(A, A, A, A, A, 64, 2, 4, 48, 128, A, A, ws, None) == 1  # N % 32
    assert "N of 32" in msg(L)
    assert L.gather_qmm_kn(A, A, A, A, A, 64, 2, 4, 64, 96, A, A, ws, None) == 1  # K % 64
    assert L.gather_qmm_kn(A, A, A, A, A, 64, 2, 4, 64, 128, A, A, 0, None) == 1  # workspace
    assert "workspace" in msg(L)


def test_scale_bytes(L):
    assert L.nvfp4_scale_bytes(67, 16, 0) == 67 * 16
    assert L.nvfp4_scale_bytes(67, 16, 1) == 128 * 16
    assert L.nvfp4_scale_bytes(200, 5, 1) == 256 * 8


def test_binding_refuses_cpu_tensors():
    import torch
    from mxfp8_block_scaled_nvfp4_b200 import nvfp4
    with pytest.raises(ValueError):
        nvfp4.amax(torch.ones(16))


def test_empty_outputs_return_ok_without_a_device(L):
    """A call with nothing to write returns NVFP4_OK after its argument checks,
    with NULL pointers and no device present; the same call with work needs
    the device (here: none, so it fails)."""
    N0 = None
    assert L.nvfp4_quantize(N0, 2, 0, 64, N0, N0, N0, 0, N0) == 0
    assert L.nvfp4_quantize(N0, 2, 7, 0, N0, N0, N0, 1, N0) == 0
    assert L.nvfp4_quantize_sr(N0, 2, 0, 64, N0, 5, N0, N0, 1, N0) == 0
    assert L.nvfp4_quantize_columnwise(N0, 2, 32, 0, N0, N0, N0, 1, N0) == 0
    assert L.nvfp4_quantize_columnwise(N0, 2, 0, 5, N0, N0, N0, 0, N0) == 0
    assert L.mxfp8_quantize(N0, 2, 0, 64, N0, N0, 1, N0) == 0
    assert L.mxfp4_quantize(N0, 2, 3, 0, N0, N0, 0, N0) == 0
    assert L.nvfp4_dequantize(N0, N0, 1, 0, 64, N0, N0, 2, N0) == 0
    assert L.mxfp8_dequantize(N0, N0, 0, 5, 0, N0, 0, N0) == 0
    assert L.mxfp4_dequantize(N0, N0, 1, 0, 32, N0, 1, N0) == 0
    assert L.nvfp4_swizzle_scales(N0, 0, 4, N0, N0) == 0
    for mode in (0, 1, 2):
        assert L.qqmm(mode, 0, 128, 256, N0, N0, N0, N0, N0, N0, N0, 2, N0) == 0
        assert L.qqmm(mode, 64, 0, 0, N0, N0, N0, N0, N0, N0, N0, 0, N0) == 0
    assert L.qmv(N0, 2, N0, N0, N0, N0, 1, 0, 256, N0, N0) == 0
    ws = L.gather_qmm_workspace_size(0, 2, 4)
    assert L.gather_qmm(N0, N0, N0, N0, N0, 0, 2, 4, 64, 128, N0, N0, ws, N0) == 0
    assert L.gather_qmm(N0, N0, N0, N0, N0, 16, 2, 4, 0, 128, N0, N0, L.gather_qmm_workspace_size(16, 2, 4), N0) == 0
    assert L.gather_qmm_kn(N0, N0, N0, N0, N0, 0, 2, 4, 64, 128, N0, N0, ws, N0) == 0
    assert L.gather_qmm_noalloc(N0, N0, N0, N0, N0, 0, 2, 4, 64, 128, N0, N0) == 0
    # argument checks still run for empty outputs
    assert L.nvfp4_quantize(N0, 2, 0, 24, N0, N0, N0, 0, N0) == 1
    assert L.qqmm(0, 0, 128, 48, N0, N0, N0, N0, N0, N0, N0, 2, N0) == 1
    assert L.gather_qmm_noalloc(N0, N0, N0, N0, N0, 0, 2, 4, -16, 128, N0, N0) == 1
    # the same shapes with work to do reach the device query (no device here)
    assert L.nvfp4_quantize(A, 2, 4, 64, N0, A, A, 0, N0) not in (0, 1, 2)
    assert L.qqmm(0, 128, 128, 256, A, A, A, A, N0, N0, A, 2, N0) not in (0, 1, 2)


def test_gemms_reject_K_zero_with_an_output(L):
    for mode in (0, 1, 2):
        assert L.qqmm(mode, 128, 128, 0, A, A, A, A, None, None, A, 2, None) == 1
        assert "K must be positive" in msg(L)
    ws = L.gather_qmm_workspace_size(16, 2, 4)
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 4, 64, 0, A, A, ws, None) == 1
    assert "K must be positive" in msg(L)
    assert L.gather_qmm_kn(A, A, A, A, A, 16, 2, 4, 64, 0, A, A, ws, None) == 1
    assert L.gather_qmm_noalloc(A, A, A, A, A, 16, 2, 4, 64, 0, A, None) == 1
    assert L.qmv(A, 2, None, A, A, None, 1, 64, 0, A, None) == 1


def test_size_limits_without_overflow(L):
    """Sizes whose products overflow int64 are rejected, not wrapped: the
    checks bound each factor before multiplying."""
    big = 1 << 40
    assert L.nvfp4_quantize(A, 2, big, big, None, A, A, 0, None) == 1
    assert L.nvfp4_quantize(A, 2, (1 << 33) + 1, 1 << 31, None, A, A, 0, None) == 1  # product wraps to 2^31
    assert L.nvfp4_dequantize(A, A, 0, (1 << 33) + 1, 1 << 31, None, A, 2, None) == 1
    assert L.mxfp8_quantize(A, 2, 1 << 62, 64, A, A, 0, None) == 1
    assert L.nvfp4_quantize_columnwise(A, 2, 1 << 31, 1 << 40, None, A, A, 0, None) == 1
    assert L.nvfp4_swizzle_scales(A, 1 << 40, 1 << 40, A, None) == 1
    assert L.qqmm(0, (1 << 30) + 1, 128, 256, A, A, A, A, None, None, A, 2, None) == 1
    ws = L.gather_qmm_workspace_size(16, 2, 4)
    assert L.gather_qmm(A, A, A, A, A, 1 << 62, 4, 4, 64, 128, A, A, ws, None) == 1  # T*topk wraps to 0
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 4, 1 << 40, 128, A, A, ws, None) == 1
    assert L.gather_qmm_noalloc(A, A, A, A, A, 1 << 62, 4, 4, 64, 128, A, None) == 1
    # the largest accepted sizes pass the argument checks and reach the device query
    assert L.nvfp4_quantize(A, 2, 1 << 20, 1 << 14, None, A, A, 0, None) not in (0, 1, 2)
    assert L.nvfp4_quantize(A, 2, (1 << 20) + 1, 1 << 14, None, A, A, 0, None) == 1


def test_gather_expert_limit_and_workspace_size(L):
    ws = L.gather_qmm_workspace_size(16, 2, 1025)
    assert ws == 0
    big = L.gather_qmm_workspace_size(16, 2, 1024)
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 1025, 64, 128, A, A, big, None) == 2
    assert "at most 1024 experts" in msg(L)
    assert L.gather_qmm_noalloc(A, A, A, A, A, 16, 2, 1025, 64, 128, A, None) == 2
    for bad in [(-1, 2, 4), (16, 0, 4), (16, 2, 0), (1 << 62, 4, 4)]:
        assert L.gather_qmm_workspace_size(*bad) == 0
    # monotone in T and covers at least the permutation (4 bytes per routed row)
    sizes = [L.gather_qmm_workspace_size(t, 8, 64) for t in (1, 64, 4096)]
    assert sizes == sorted(sizes) and sizes[-1] >= 4 * 4096 * 8


def test_gather_weight_rows_fit_32_bit_coordinates(L):
    """The weight tensor map's rows (E*N, or E*K for [E, K, N]) are addressed
    by 32-bit signed TMA coordinates: more are refused, not wrapped."""
    ws = L.gather_qmm_workspace_size(16, 2, 1024)
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 1024, 1 << 21, 128, A, A, ws, None) == 2  # E*N = 2^31
    assert "rows" in msg(L)
    assert L.gather_qmm_kn(A, A, A, A, A, 16, 2, 1024, 64, 1 << 21, A, A, ws, None) == 2  # E*K = 2^31
    # just under the limit passes the checks (and reaches the device query)
    assert L.gather_qmm(A, A, A, A, A, 16, 2, 1024, (1 << 21) - 16, 128, A, A, ws, None) not in (0, 1, 2)


def test_plain_c_caller(L):
    """The header compiles as strict C99 and a C program links the library
    and sees the host-side contract (no CUDA or torch headers involved)."""
    import shutil
    import subprocess
    from mxfp8_block_scaled_nvfp4_b200 import nvfp4
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_abi_example")
    lib_dir = os.path.dirname(nvfp4.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_example.c"), "-o", exe, "-L", lib_dir,
                    "-l:" + os.path.basename(nvfp4.LIB_PATH), "-Wl,-rpath," + lib_dir], check=True)
    r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok")
    assert "or neither" in r.stdout


def test_multi_tensor_entries_check_every_item(L):
    """nvfp4_amax_multi / nvfp4_quantize_multi: 1 to 4 items, each checked as
    the single-tensor call checks it; items with no element are skipped, so
    a call whose items are all empty returns OK without a device, while
    amax_multi (which zeroes its outputs) always needs one."""
    from mxfp8_block_scaled_nvfp4_b200.nvfp4 import AmaxItem, QuantizeItem
    N0 = None

    def q(*items):
        arr = (QuantizeItem * max(1, len(items)))(*items)
        return L.nvfp4_quantize_multi(arr, len(items), 2, N0)

    def am(*items):
        arr = (AmaxItem * max(1, len(items)))(*items)
        return L.nvfp4_amax_multi(arr, len(items), 2, N0)

    good = QuantizeItem(A, 4, 64, N0, A, A, 0)
    empty = QuantizeItem(N0, 0, 64, N0, N0, N0, 1)
    assert q() == 1 and "between 1 and 4" in msg(L)
    assert q(good, good, good, good, good) == 1
    assert q(empty, empty) == 0
    assert q(empty, QuantizeItem(A, 4, 24, N0, A, A, 0)) == 1 and "group size 16" in msg(L)
    assert q(good, QuantizeItem(A + 8, 4, 64, N0, A, A, 0)) == 1 and "16-byte aligned" in msg(L)
    assert q(good, QuantizeItem(A, 4, 64, N0, A, A, 7)) == 1 and "layout" in msg(L)
    assert q(good, empty) not in (0, 1, 2)  # work to do: reaches the device query (no device here)
    assert L.nvfp4_quantize_multi(None, 1, 2, N0) == 1
    assert L.nvfp4_quantize_multi((QuantizeItem * 1)(good), 1, 7, N0) == 2

    assert am() == 1
    assert am(AmaxItem(A, 16, A), AmaxItem(A, 16, A)) == 1 and "share one output" in msg(L)
    assert am(AmaxItem(A, -1, A)) == 1
    assert am(AmaxItem(A, 16, A + 2)) == 1 and "4-byte aligned" in msg(L)
    assert am(AmaxItem(A, 16, A), AmaxItem(A, 0, A + 4)) not in (0, 1, 2)


def test_qmv_mx_checks(L):
    N0 = None
    assert L.qmv_mx(0, A, 2, A, A, 1, 64, 256, A, N0) == 1 and "mxfp8 or mxfp4" in msg(L)  # nvfp4 mode
    assert L.qmv_mx(1, A, 2, A, A, 9, 64, 256, A, N0) == 1 and "M must be" in msg(L)
    assert L.qmv_mx(2, A, 2, A, A, 1, 64, 48, A, N0) == 1 and "K % 32" in msg(L)
    assert L.qmv_mx(2, A, 7, A, A, 1, 64, 256, A, N0) == 2
    assert L.qmv_mx(1, A + 8, 2, A, A, 1, 64, 256, A, N0) == 1 and "aligned" in msg(L)
    assert L.qmv_mx(1, A, 2, A, A, 8, 64, 8192, A, N0) == 2 and "160 KiB" in msg(L)
    assert L.qmv_mx(2, N0, 2, N0, N0, 1, 0, 256, N0, N0) == 0  # empty output
    assert L.qmv_mx(2, A, 2, A, A, 1, 64, 256, A, N0) not in (0, 1, 2)  # needs a device


def test_gather_staged_workspace_size(L):
    """The staged workspace holds the routing workspace, 256-byte aligned,
    then a bf16 copy of every routed x row (T*topk rows of K elements)."""
    for T, topk, E, K in [(4096, 8, 64, 2048), (17, 3, 5, 192), (1, 1, 1, 64), (0, 2, 4, 128)]:
        base = L.gather_qmm_workspace_size(T, topk, E)
        staged = L.gather_qmm_staged_workspace_size(T, topk, E, K)
        assert staged == ((base + 255) // 256) * 256 + T * topk * K * 2
    for bad in [(-1, 2, 4, 64), (16, 0, 4, 64), (16, 2, 0, 64), (16, 2, 1025, 64), (16, 2, 4, -64),
                (16, 2, 4, (1 << 30) + 64), (1 << 62, 4, 4, 64)]:
        assert L.gather_qmm_staged_workspace_size(*bad) == 0
