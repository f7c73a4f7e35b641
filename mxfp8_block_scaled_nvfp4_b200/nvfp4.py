"""Thin Python binding of libnvfp4.so (include/nvfp4.h).

Argument marshalling only: every step of the method runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  There
is no CPU fallback: if the shared library is missing or the device is not a
B200 (sm_100), calls raise.

The raw C functions are available as ``lib().<name>`` (ctypes), with the same
names and arguments as the header; the wrappers below allocate outputs with
torch and pass device pointers plus ``torch.cuda.current_stream()``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_INDEX = range(6)
DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
LAYOUT = {"linear": 0, "swizzled": 1}
MODE = {"nvfp4": 0, "mxfp8": 1, "mxfp4": 2}

# (name, restype, argtypes) of every symbol declared in include/nvfp4.h
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class AmaxItem(ctypes.Structure):
    """nvfp4_amax_item"""
    _fields_ = [("x", _P), ("n", _I64), ("g_out", _P)]


class QuantizeItem(ctypes.Structure):
    """nvfp4_quantize_item (the layout enum is a C int)"""
    _fields_ = [("x", _P), ("rows", _I64), ("K", _I64), ("g", _P), ("codes", _P), ("scales", _P),
                ("layout", _I)]


SIGNATURES = [
    ("nvfp4_status_string", ctypes.c_char_p, [_I]),
    ("nvfp4_last_error_message", ctypes.c_char_p, []),
    ("nvfp4_check_device_errors", _I, [_P]),
    ("nvfp4_scale_bytes", _SZ, [_I64, _I64, _I]),
    ("nvfp4_amax", _I, [_P, _I, _I64, _P, _P]),
    ("nvfp4_amax_multi", _I, [ctypes.POINTER(AmaxItem), _I, _I, _P]),
    ("nvfp4_quantize", _I, [_P, _I, _I64, _I64, _P, _P, _P, _I, _P]),
    ("nvfp4_quantize_multi", _I, [ctypes.POINTER(QuantizeItem), _I, _I, _P]),
    ("nvfp4_quantize_columnwise", _I, [_P, _I, _I64, _I64, _P, _P, _P, _I, _P]),
    ("nvfp4_dequantize", _I, [_P, _P, _I, _I64, _I64, _P, _P, _I, _P]),
    ("nvfp4_quantize_sr", _I, [_P, _I, _I64, _I64, _P, ctypes.c_uint64, _P, _P, _I, _P]),
    ("nvfp4_quantize_columnwise_sr", _I, [_P, _I, _I64, _I64, _P, ctypes.c_uint64, _P, _P, _I, _P]),
    ("mxfp8_quantize", _I, [_P, _I, _I64, _I64, _P, _P, _I, _P]),
    ("mxfp8_dequantize", _I, [_P, _P, _I, _I64, _I64, _P, _I, _P]),
    ("mxfp4_quantize", _I, [_P, _I, _I64, _I64, _P, _P, _I, _P]),
    ("mxfp4_dequantize", _I, [_P, _P, _I, _I64, _I64, _P, _I, _P]),
    ("nvfp4_swizzle_scales", _I, [_P, _I64, _I64, _P, _P]),
    ("qqmm", _I, [_I, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    ("qmv", _I, [_P, _I, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    ("qmv_pdl", _I, [_P, _I, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    ("qmv_mx", _I, [_I, _P, _I, _P, _P, _I64, _I64, _I64, _P, _P]),
    ("gather_qmm", _I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    ("gather_qmm_kn", _I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    ("gather_qmm_workspace_size", _SZ, [_I64, _I64, _I64]),
    ("gather_qmm_staged_workspace_size", _SZ, [_I64, _I64, _I64, _I64]),
    ("gather_qmm_noalloc", _I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P]),
]

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


def lib():
    """The loaded libnvfp4.so (ctypes.CDLL) with argument types set."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m mxfp8_block_scaled_nvfp4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        L = lib()
        msg = L.nvfp4_last_error_message().decode() or L.nvfp4_status_string(status).decode()
        raise Nvfp4Error(status, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need_cuda(*ts):
    """Every tensor is a contiguous CUDA tensor on the current device: the
    library launches on the current device and the current stream, so a
    tensor of another GPU would be read through a pointer that GPU's kernels
    cannot use."""
    dev = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be CUDA tensors (no CPU fallback)")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")
            if dev is None:
                dev = torch.cuda.current_device()
            if t.device.index != dev:
                raise ValueError(f"tensor on {t.device}, but the current device is cuda:{dev}; "
                                 "call under torch.cuda.device(tensor.device)")


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _need_bytes(t, nbytes: int, what: str):
    """The library takes raw pointers and cannot see a buffer's size: refuse
    one smaller than the bytes the call reads or writes through it."""
    if t is not None and _nbytes(t) < nbytes:
        raise ValueError(f"{what} holds {_nbytes(t)} bytes; the call needs {nbytes}")


def _need_dtype(t, dtype, what: str):
    if t is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")


def _need_g(g, n: int = 1, what: str = "global scale"):
    """Global scales are fp32 device scalars (n of them for per-expert g)."""
    _need_dtype(g, torch.float32, what)
    _need_bytes(g, 4 * n, what)


def _scale_nbytes(rows: int, cols: int, layout: str) -> int:
    r, c = scale_shape(rows, cols, layout)
    return r * c


def check_device_errors():
    _check(lib().nvfp4_check_device_errors(_stream()))


def scale_bytes(rows: int, cols: int, layout: str) -> int:
    return int(lib().nvfp4_scale_bytes(rows, cols, LAYOUT[layout]))


def scale_shape(rows: int, cols: int, layout: str):
    if layout == "linear":
        return (rows, cols)
    return ((rows + 127) // 128 * 128, (cols + 3) // 4 * 4)


# ---------------------------------------------------------------------------
def amax(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 [1] tensor holding max |x| (the global scale g)."""
    _need_g(out, 1, "out")
    _need_cuda(x, out)
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    _check(lib().nvfp4_amax(_ptr(x), DT[x.dtype], x.numel(), _ptr(out), _stream()))
    return out


def nvfp4_quantize(x: torch.Tensor, g: torch.Tensor | None = None, layout: str = "linear",
                   codes: torch.Tensor | None = None, scales: torch.Tensor | None = None):
    """(codes uint32 [rows, K/8] viewed as int32, scales uint8) of a 2-D x."""
    rows, K = x.shape
    _need_g(g)
    _need_bytes(codes, rows * (K // 8) * 4, "codes")
    _need_bytes(scales, _scale_nbytes(rows, K // 16, layout), "scales")
    _need_cuda(x, g, codes, scales)
    if codes is None:
        codes = torch.empty(rows, K // 8, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(rows, K // 16, layout), dtype=torch.uint8, device=x.device)
    _check(lib().nvfp4_quantize(_ptr(x), DT[x.dtype], rows, K, _ptr(g), _ptr(codes), _ptr(scales),
                                LAYOUT[layout], _stream()))
    return codes, scales


def amax_multi(xs, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 [len(xs)] tensor: out[i] = max |xs[i]|, one launch (1 to 4
    tensors of one dtype)."""
    n = len(xs)
    if not 1 <= n <= 4:
        raise ValueError("amax_multi takes 1 to 4 tensors")
    if any(x.dtype != xs[0].dtype for x in xs):
        raise ValueError("amax_multi: every tensor must have the same dtype")
    _need_g(out, n, "out")
    _need_cuda(*xs, out)
    out = torch.empty(n, dtype=torch.float32, device=xs[0].device) if out is None else out
    items = (AmaxItem * n)(*[AmaxItem(x.data_ptr(), x.numel(), out.data_ptr() + 4 * i) for i, x in enumerate(xs)])
    _check(lib().nvfp4_amax_multi(items, n, DT[xs[0].dtype], _stream()))
    return out


def nvfp4_quantize_multi(jobs):
    """nvfp4_quantize of 1 to 4 tensors of one dtype in one launch.  jobs:
    (x, g, layout[, codes, scales]) tuples, as nvfp4_quantize's arguments.
    Returns [(codes, scales), ...] in the same order."""
    n = len(jobs)
    if not 1 <= n <= 4:
        raise ValueError("nvfp4_quantize_multi takes 1 to 4 tensors")
    outs, items = [], []
    for job in jobs:
        x, g, layout = job[0], job[1], job[2]
        codes, scales = (job[3], job[4]) if len(job) > 3 else (None, None)
        if x.dtype != jobs[0][0].dtype:
            raise ValueError("nvfp4_quantize_multi: every tensor must have the same dtype")
        rows, K = x.shape
        _need_g(g)
        _need_bytes(codes, rows * (K // 8) * 4, "codes")
        _need_bytes(scales, _scale_nbytes(rows, K // 16, layout), "scales")
        _need_cuda(x, g, codes, scales)
        if codes is None:
            codes = torch.empty(rows, K // 8, dtype=torch.int32, device=x.device)
        if scales is None:
            scales = torch.empty(scale_shape(rows, K // 16, layout), dtype=torch.uint8, device=x.device)
        outs.append((codes, scales))
        items.append(QuantizeItem(x.data_ptr(), rows, K, None if g is None else g.data_ptr(), codes.data_ptr(),
                                  scales.data_ptr(), LAYOUT[layout]))
    arr = (QuantizeItem * n)(*items)
    _check(lib().nvfp4_quantize_multi(arr, n, DT[jobs[0][0].dtype], _stream()))
    return outs


def nvfp4_quantize_columnwise(x: torch.Tensor, g: torch.Tensor | None = None, layout: str = "linear",
                              codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                              seed: int | None = None):
    """(codes [cols, rows/8], scales) of x^T quantized along the rows of a 2-D x
    (equal to nvfp4_quantize(x.T.contiguous(), g, layout)); with a seed,
    nvfp4_quantize_columnwise_sr (equal to nvfp4_quantize_sr of x^T)."""
    rows, cols = x.shape
    _need_g(g)
    _need_bytes(codes, cols * (rows // 8) * 4, "codes")
    _need_bytes(scales, _scale_nbytes(cols, rows // 16, layout), "scales")
    _need_cuda(x, g, codes, scales)
    if codes is None:
        codes = torch.empty(cols, rows // 8, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(cols, rows // 16, layout), dtype=torch.uint8, device=x.device)
    if seed is None:
        _check(lib().nvfp4_quantize_columnwise(_ptr(x), DT[x.dtype], rows, cols, _ptr(g), _ptr(codes), _ptr(scales),
                                               LAYOUT[layout], _stream()))
    else:
        _check(lib().nvfp4_quantize_columnwise_sr(_ptr(x), DT[x.dtype], rows, cols, _ptr(g), seed, _ptr(codes),
                                                  _ptr(scales), LAYOUT[layout], _stream()))
    return codes, scales


def nvfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, g: torch.Tensor | None = None,
                     layout: str = "linear", dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    rows, K = codes.shape[0], codes.shape[1] * 8
    _need_g(g)
    _need_bytes(scales, _scale_nbytes(rows, K // 16, layout), "scales")
    _need_bytes(out, rows * K * (out.element_size() if out is not None else 0), "out")
    _need_cuda(codes, scales, g, out)
    if out is None:
        out = torch.empty(rows, K, dtype=dtype, device=codes.device)
    dtype = out.dtype
    _check(lib().nvfp4_dequantize(_ptr(codes), _ptr(scales), LAYOUT[layout], rows, K, _ptr(g), _ptr(out),
                                  DT[dtype], _stream()))
    return out


def nvfp4_quantize_sr(x: torch.Tensor, g: torch.Tensor | None = None, seed: int = 0, layout: str = "linear",
                      codes: torch.Tensor | None = None, scales: torch.Tensor | None = None):
    """nvfp4_quantize with stochastic rounding of the codes (Philox4x32-10
    random bits keyed by ``seed``); scales as nvfp4_quantize."""
    rows, K = x.shape
    _need_g(g)
    _need_bytes(codes, rows * (K // 8) * 4, "codes")
    _need_bytes(scales, _scale_nbytes(rows, K // 16, layout), "scales")
    _need_cuda(x, g, codes, scales)
    if codes is None:
        codes = torch.empty(rows, K // 8, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(rows, K // 16, layout), dtype=torch.uint8, device=x.device)
    _check(lib().nvfp4_quantize_sr(_ptr(x), DT[x.dtype], rows, K, _ptr(g), seed, _ptr(codes), _ptr(scales),
                                   LAYOUT[layout], _stream()))
    return codes, scales


def mxfp8_quantize(x: torch.Tensor, layout: str = "linear", codes=None, scales=None):
    rows, K = x.shape
    _need_bytes(codes, rows * (K // 4) * 4, "codes")
    _need_bytes(scales, _scale_nbytes(rows, K // 32, layout), "scales")
    _need_cuda(x, codes, scales)
    if codes is None:
        codes = torch.empty(rows, K // 4, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(rows, K // 32, layout), dtype=torch.uint8, device=x.device)
    _check(lib().mxfp8_quantize(_ptr(x), DT[x.dtype], rows, K, _ptr(codes), _ptr(scales), LAYOUT[layout],
                                _stream()))
    return codes, scales


def mxfp4_quantize(x: torch.Tensor, layout: str = "linear", codes=None, scales=None):
    """(codes int32 [rows, K/8], e8m0 scales uint8) of a 2-D x, 32-element blocks."""
    rows, K = x.shape
    _need_bytes(codes, rows * (K // 8) * 4, "codes")
    _need_bytes(scales, _scale_nbytes(rows, K // 32, layout), "scales")
    _need_cuda(x, codes, scales)
    if codes is None:
        codes = torch.empty(rows, K // 8, dtype=torch.int32, device=x.device)
    if scales is None:
        scales = torch.empty(scale_shape(rows, K // 32, layout), dtype=torch.uint8, device=x.device)
    _check(lib().mxfp4_quantize(_ptr(x), DT[x.dtype], rows, K, _ptr(codes), _ptr(scales), LAYOUT[layout],
                                _stream()))
    return codes, scales


def mxfp4_dequantize(codes, scales, layout: str = "linear", dtype=torch.bfloat16) -> torch.Tensor:
    rows, K = codes.shape[0], codes.shape[1] * 8
    _need_bytes(scales, _scale_nbytes(rows, K // 32, layout), "scales")
    _need_cuda(codes, scales)
    out = torch.empty(rows, K, dtype=dtype, device=codes.device)
    _check(lib().mxfp4_dequantize(_ptr(codes), _ptr(scales), LAYOUT[layout], rows, K, _ptr(out), DT[dtype],
                                  _stream()))
    return out


def mxfp8_dequantize(codes, scales, layout: str = "linear", dtype=torch.bfloat16) -> torch.Tensor:
    rows, K = codes.shape[0], codes.shape[1] * 4
    _need_bytes(scales, _scale_nbytes(rows, K // 32, layout), "scales")
    _need_cuda(codes, scales)
    out = torch.empty(rows, K, dtype=dtype, device=codes.device)
    _check(lib().mxfp8_dequantize(_ptr(codes), _ptr(scales), LAYOUT[layout], rows, K, _ptr(out), DT[dtype],
                                  _stream()))
    return out


def swizzle_scales(lin: torch.Tensor) -> torch.Tensor:
    _need_cuda(lin)
    rows, cols = lin.shape
    out = torch.empty(scale_shape(rows, cols, "swizzled"), dtype=torch.uint8, device=lin.device)
    _check(lib().nvfp4_swizzle_scales(_ptr(lin), rows, cols, _ptr(out), _stream()))
    return out


def qqmm(a_codes, a_scales, b_codes, b_scales, K: int, mode: str = "nvfp4", g_x=None, g_w=None,
         out_dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """y [M, N] = x_hat . w_hat^T from quantized operands with SWIZZLED scales."""
    M, N = a_codes.shape[0], b_codes.shape[0]
    if mode in MODE:
        row_bytes = K if mode == "mxfp8" else K // 2
        group = 16 if mode == "nvfp4" else 32
        _need_bytes(a_codes, M * row_bytes, "a_codes")
        _need_bytes(b_codes, N * row_bytes, "b_codes")
        _need_bytes(a_scales, _scale_nbytes(M, K // group, "swizzled"), "a_scales")
        _need_bytes(b_scales, _scale_nbytes(N, K // group, "swizzled"), "b_scales")
    _need_g(g_x, 1, "g_x")
    _need_g(g_w, 1, "g_w")
    _need_bytes(out, M * N * (out.element_size() if out is not None else 0), "out")
    _need_cuda(a_codes, a_scales, b_codes, b_scales, g_x, g_w, out)
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=a_codes.device)
    _check(lib().qqmm(MODE[mode], M, N, K, _ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales),
                      _ptr(g_x), _ptr(g_w), _ptr(out), DT[out.dtype], _stream()))
    return out


def qqmm_raw(x: torch.Tensor, w: torch.Tensor, out_dtype=None, out: torch.Tensor | None = None, buffers=None):
    """y [M, N] = qqmm of raw operands x [M, K] and w [N, K] (one dtype),
    NVFP4 with g = amax of each ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 8,
    ops.cpp qqmm on unquantized inputs): both amaxes in one launch, both
    quantizations (SWIZZLED scales) in one launch, then the GEMM.  y has x's
    dtype unless out_dtype or out says otherwise.  buffers: optional
    preallocated (g [2] fp32, x codes, x scales, w codes, w scales)."""
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K or w.dtype != x.dtype:
        raise ValueError("x [M, K] and w [N, K] must share K and dtype")
    if buffers is None:
        dev = x.device
        g = torch.empty(2, dtype=torch.float32, device=dev)
        xc, wc = (torch.empty(r, K // 8, dtype=torch.int32, device=dev) for r in (M, N))
        xs, ws = (torch.empty(scale_shape(r, K // 16, "swizzled"), dtype=torch.uint8, device=dev) for r in (M, N))
    else:
        g, xc, xs, wc, ws = buffers
    amax_multi([x, w], g)
    nvfp4_quantize_multi([(x, g[0:1], "swizzled", xc, xs), (w, g[1:2], "swizzled", wc, ws)])
    return qqmm(xc, xs, wc, ws, K, "nvfp4", g[0:1], g[1:2], out_dtype=out_dtype or x.dtype, out=out)


def qqmm_vjp(x: torch.Tensor, w: torch.Tensor, cotan: torch.Tensor, g_x: torch.Tensor, g_w: torch.Tensor):
    """(dx, dw) of y = qqmm(x, w) ("mlx 0.30.7.2 -> 0.30.7.6" diff, page 8,
    QQMatmul::vjp, NVFP4 with global scales): with g_c = amax(cotan),
      dx = qqmm(cotan, w^T)   -- cotan quantized along N with g_c, w^T along N with g_w
      dw = qqmm(cotan^T, x^T) -- both quantized along M, with g_c and g_x.
    x [M, K], w [N, K], cotan [M, N] bf16/fp16/fp32; M, N multiples of 32.
    Every step is one ABI call (amax, quantize, column-wise quantize, qqmm)."""
    _need_cuda(x, w, cotan, g_x, g_w)
    M, N = x.shape[0], w.shape[0]
    g_c = amax(cotan)
    c_codes, c_scales = nvfp4_quantize(cotan, g_c, "swizzled")                # [M, N/8]
    wt_codes, wt_scales = nvfp4_quantize_columnwise(w, g_w, "swizzled")      # w^T [K, N/8]
    dx = qqmm(c_codes, c_scales, wt_codes, wt_scales, N, "nvfp4", g_c, g_w, out_dtype=x.dtype)
    ct_codes, ct_scales = nvfp4_quantize_columnwise(cotan, g_c, "swizzled")  # cotan^T [N, M/8]
    xt_codes, xt_scales = nvfp4_quantize_columnwise(x, g_x, "swizzled")      # x^T [K, M/8]
    dw = qqmm(ct_codes, ct_scales, xt_codes, xt_scales, M, "nvfp4", g_c, g_x, out_dtype=w.dtype)
    return dx, dw


def qmv(x: torch.Tensor, w_codes, w_scales, g_x=None, g_w=None, out=None, pdl: bool = False) -> torch.Tensor:
    """y [M, N] (x's dtype) = x_hat . w_hat^T, M <= 8, w pre-quantized (LINEAR scales).
    pdl=True calls qmv_pdl: for chains of decode calls whose weight (codes,
    scales, g_w) is not written by work still pending on the device."""
    M, K = x.shape
    N = w_codes.shape[0]
    _need_bytes(w_codes, N * (K // 8) * 4, "w_codes")
    _need_bytes(w_scales, N * (K // 16), "w_scales")
    _need_g(g_x, 1, "g_x")
    _need_g(g_w, 1, "g_w")
    _need_dtype(out, x.dtype, "out")
    _need_bytes(out, M * N * x.element_size(), "out")
    _need_cuda(x, w_codes, w_scales, g_x, g_w, out)
    if out is None:
        out = torch.empty(M, N, dtype=x.dtype, device=x.device)
    fn = lib().qmv_pdl if pdl else lib().qmv
    _check(fn(_ptr(x), DT[x.dtype], _ptr(g_x), _ptr(w_codes), _ptr(w_scales), _ptr(g_w), M, N, K, _ptr(out),
              _stream()))
    return out


def qmv_mx(x: torch.Tensor, w_codes, w_scales, mode: str, out=None) -> torch.Tensor:
    """y [M, N] (x's dtype) = x_hat . w_hat^T in an MX mode ("mxfp8": codes
    [N, K/4], "mxfp4": codes [N, K/8]; e8m0 scales LINEAR [N, K/32]), M <= 8."""
    if mode not in ("mxfp8", "mxfp4"):
        raise ValueError("qmv_mx: mode must be mxfp8 or mxfp4")
    M, K = x.shape
    N = w_codes.shape[0]
    _need_bytes(w_codes, N * (K if mode == "mxfp8" else K // 2), "w_codes")
    _need_bytes(w_scales, N * (K // 32), "w_scales")
    _need_dtype(out, x.dtype, "out")
    _need_bytes(out, M * N * x.element_size(), "out")
    _need_cuda(x, w_codes, w_scales, out)
    if out is None:
        out = torch.empty(M, N, dtype=x.dtype, device=x.device)
    _check(lib().qmv_mx(MODE[mode], _ptr(x), DT[x.dtype], _ptr(w_codes), _ptr(w_scales), M, N, K, _ptr(out),
                        _stream()))
    return out


def gather_qmm_workspace_size(T: int, topk: int, E: int) -> int:
    return int(lib().gather_qmm_workspace_size(T, topk, E))


def gather_qmm_staged_workspace_size(T: int, topk: int, E: int, K: int) -> int:
    return int(lib().gather_qmm_staged_workspace_size(T, topk, E, K))


def _need_gather(x, w_codes, w_scales, g, idx, out, T, topk, E, N, K, transpose):
    """Types and sizes the gather entries read and write through raw pointers."""
    _need_dtype(x, torch.bfloat16, "x")
    _need_dtype(idx, torch.int32, "idx")
    _need_bytes(idx, T * topk * 4, "idx")
    if transpose:
        _need_bytes(w_codes, E * N * (K // 8) * 4, "w_codes")
        _need_bytes(w_scales, E * N * (K // 16), "w_scales")
    else:
        _need_bytes(w_codes, E * K * (N // 8) * 4, "w_codes")
        _need_bytes(w_scales, E * K * (N // 16), "w_scales")
    _need_g(g, E, "g")
    _need_dtype(out, torch.bfloat16, "out")
    _need_bytes(out, T * topk * N * 2, "out")


def gather_qmm(x, w_codes, w_scales, g, idx, workspace=None, out=None, transpose: bool = True) -> torch.Tensor:
    """y [T, topk, N] bf16.  transpose=True: w_codes [E, N, K/8], w_scales
    LINEAR [E, N, K/16] (y = x . w_hat^T); transpose=False: w_codes
    [E, K, N/8], w_scales LINEAR [E, K, N/16] (y = x . w_hat)."""
    T, K = x.shape
    topk = idx.shape[1]
    E = w_codes.shape[0]
    N = w_codes.shape[1] if transpose else w_codes.shape[2] * 8
    _need_gather(x, w_codes, w_scales, g, idx, out, T, topk, E, N, K, transpose)
    _need_cuda(x, w_codes, w_scales, g, idx, workspace, out)
    if workspace is None:  # the staged form where it applies (weights [E, N, K])
        size = gather_qmm_staged_workspace_size(T, topk, E, K) if transpose else gather_qmm_workspace_size(T, topk, E)
        workspace = torch.empty(size, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty(T, topk, N, dtype=torch.bfloat16, device=x.device)
    fn = lib().gather_qmm if transpose else lib().gather_qmm_kn
    _check(fn(_ptr(x), _ptr(w_codes), _ptr(w_scales), _ptr(g), _ptr(idx), T, topk, E, N, K,
              _ptr(out), _ptr(workspace), _nbytes(workspace), _stream()))
    return out


def gather_qmm_noalloc(x, w_codes, w_scales, g, idx, out=None) -> torch.Tensor:
    """gather_qmm using the library's own static scratch instead of a
    workspace (for callers that cannot allocate device memory); see
    include/nvfp4.h for its size limit and the rule that overlapping calls
    must be serialized."""
    T, K = x.shape
    topk = idx.shape[1]
    E, N = w_codes.shape[0], w_codes.shape[1]
    _need_gather(x, w_codes, w_scales, g, idx, out, T, topk, E, N, K, True)
    _need_cuda(x, w_codes, w_scales, g, idx, out)
    if out is None:
        out = torch.empty(T, topk, N, dtype=torch.bfloat16, device=x.device)
    _check(lib().gather_qmm_noalloc(_ptr(x), _ptr(w_codes), _ptr(w_scales), _ptr(g), _ptr(idx), T, topk, E, N, K,
                                    _ptr(out), _stream()))
    return out
