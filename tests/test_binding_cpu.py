"""Host-side checks of the Python binding (CPU only): buffers the library
would read or write through raw pointers are refused when they are too small
or of the wrong type, before any CUDA call; buffers of the right size pass
those checks and reach the CUDA-tensor check (no CPU fallback)."""
import pytest
import torch

from mxfp8_block_scaled_nvfp4_b200 import nvfp4 as nv

bf16, f32, i32, u8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def e(*shape, dtype=u8):
    return torch.empty(*shape, dtype=dtype)


def refused(fn, *a, match, **k):
    with pytest.raises(ValueError, match=match):
        fn(*a, **k)


def reaches_cuda_check(fn, *a, **k):
    refused(fn, *a, match="CUDA tensors", **k)


def test_quantize_output_buffers():
    x = e(256, 64, dtype=bf16)
    reaches_cuda_check(nv.nvfp4_quantize, x, None, "swizzled", e(256, 8, dtype=i32), e(256, 4))
    refused(nv.nvfp4_quantize, x, None, "linear", e(256, 7, dtype=i32), None, match="codes")
    refused(nv.nvfp4_quantize, x, None, "linear", None, e(255, 4), match="scales")
    # SWIZZLED scales are padded to 128 rows x 4 columns: 256 x 4 bytes
    refused(nv.nvfp4_quantize, e(200, 64, dtype=bf16), None, "swizzled", None, e(200, 4), match="scales")
    reaches_cuda_check(nv.nvfp4_quantize, e(200, 64, dtype=bf16), None, "swizzled", None, e(256, 4))
    refused(nv.nvfp4_quantize_sr, x, None, 3, "linear", e(10, dtype=i32), match="codes")
    refused(nv.nvfp4_quantize_columnwise, x, None, "linear", e(64, 31, dtype=i32), match="codes")
    reaches_cuda_check(nv.nvfp4_quantize_columnwise, x, None, "linear", e(64, 32, dtype=i32), e(64, 16))
    refused(nv.mxfp8_quantize, x, "linear", e(256, 15, dtype=i32), match="codes")
    refused(nv.mxfp8_quantize, x, "linear", None, e(256, 1), match="scales")
    refused(nv.mxfp4_quantize, x, "swizzled", None, e(256, 3), match="scales")
    reaches_cuda_check(nv.mxfp4_quantize, x, "swizzled", e(256, 8, dtype=i32), e(256, 4))


def test_global_scales_are_fp32_scalars():
    x = e(16, 64, dtype=bf16)
    refused(nv.nvfp4_quantize, x, torch.ones(1, dtype=torch.float64), match="float32")
    refused(nv.nvfp4_quantize, x, torch.ones(0, dtype=f32), match="global scale")
    refused(nv.amax, x, torch.empty(1, dtype=bf16), match="float32")
    reaches_cuda_check(nv.amax, x, torch.empty(1, dtype=f32))


def test_dequantize_buffers():
    codes, scales = e(64, 4, dtype=i32), e(64, 2)
    reaches_cuda_check(nv.nvfp4_dequantize, codes, scales)
    refused(nv.nvfp4_dequantize, codes, e(64, 1), match="scales")
    refused(nv.nvfp4_dequantize, codes, scales, None, "swizzled", match="scales")  # needs 128 x 4
    refused(nv.nvfp4_dequantize, codes, scales, out=e(64, 31, dtype=bf16), match="out")
    refused(nv.mxfp4_dequantize, codes, e(63, 1), match="scales")
    refused(nv.mxfp8_dequantize, e(64, 8, dtype=i32), e(64, 0), match="scales")


def test_qqmm_operands():
    M, N, K = 128, 256, 512
    a, sa = e(M, K // 8, dtype=i32), e(M, K // 16)
    b, sb = e(N, K // 8, dtype=i32), e(N, K // 16)
    reaches_cuda_check(nv.qqmm, a, sa, b, sb, K)
    refused(nv.qqmm, a, sa, b, sb, 2 * K, match="a_codes")  # K larger than the codes hold
    refused(nv.qqmm, a, sa, b[:, :-1].contiguous(), sb, K, match="b_codes")
    refused(nv.qqmm, a, sa[:, :-1].contiguous(), b, sb, K, match="a_scales")
    refused(nv.qqmm, a, sa, b, sb, K, out=e(M, N - 1, dtype=bf16), match="out")
    refused(nv.qqmm, a, sa, b, sb, K, "nvfp4", torch.ones(1, dtype=torch.float64), torch.ones(1), match="float32")
    # MXFP8 codes hold one byte per element, 32-element scale groups
    reaches_cuda_check(nv.qqmm, e(M, K // 4, dtype=i32), e(M, K // 32), e(N, K // 4, dtype=i32), e(N, K // 32), K,
                       "mxfp8")
    refused(nv.qqmm, a, e(M, K // 32), e(N, K // 4, dtype=i32), e(N, K // 32), K, "mxfp8", match="a_codes")


def test_qmv_operands():
    x = e(1, 4096, dtype=bf16)
    wc, ws = e(64, 512, dtype=i32), e(64, 256)
    reaches_cuda_check(nv.qmv, x, wc, ws)
    refused(nv.qmv, x, wc, e(64, 255), match="w_scales")
    refused(nv.qmv, x, e(64, 511, dtype=i32), ws, match="w_codes")
    refused(nv.qmv, x, wc, ws, out=e(1, 64, dtype=f32), match="out")


def test_gather_operands():
    T, topk, E, N, K = 16, 2, 4, 64, 128
    x, idx = e(T, K, dtype=bf16), e(T, topk, dtype=i32)
    wc, ws, g = e(E, N, K // 8, dtype=i32), e(E, N, K // 16), e(E, dtype=f32)
    reaches_cuda_check(nv.gather_qmm, x, wc, ws, g, idx)
    refused(nv.gather_qmm, x.float(), wc, ws, g, idx, match="bfloat16")
    refused(nv.gather_qmm, x, wc, ws, g, idx.long(), match="int32")
    refused(nv.gather_qmm, x, wc, ws, g[:3], idx, match="g")
    refused(nv.gather_qmm, x, wc, ws[:, :, :-1].contiguous(), g, idx, match="w_scales")
    refused(nv.gather_qmm, x, wc, ws, g, idx, out=e(T, topk, N - 8, dtype=bf16), match="out")
    refused(nv.gather_qmm_noalloc, x, wc[:, :, :-1].contiguous(), ws, g, idx, match="w_codes")
    # [E, K, N] weights
    wkn, skn = e(E, K, N // 8, dtype=i32), e(E, K, N // 16)
    reaches_cuda_check(nv.gather_qmm, x, wkn, skn, None, idx, transpose=False)
    refused(nv.gather_qmm, x, wkn, skn[:, :-1].contiguous(), None, idx, transpose=False, match="w_scales")


class _OnDevice:
    """Stand-in for a contiguous CUDA tensor on a given device (no GPU here)."""
    is_cuda = True

    def __init__(self, index):
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True


def test_tensors_on_another_device_are_refused(monkeypatch):
    # the library launches on the current device: a tensor of another GPU
    # would be read there through a pointer that device cannot use
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    nv._need_cuda(_OnDevice(0), None, _OnDevice(0))
    refused(nv._need_cuda, _OnDevice(0), _OnDevice(1), match="current device is cuda:0")
    refused(nv._need_cuda, _OnDevice(1), match="torch.cuda.device")
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    nv._need_cuda(_OnDevice(1), _OnDevice(1))
