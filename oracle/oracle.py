"""Plain, slow CPU oracle for NVFP4 / MXFP8 block-scaled quantize, dequantize
and quantized matmuls.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA path (``mxfp8_block_scaled_nvfp4_b200``); neither imports
the other.

Element-wise steps (encode, decode, rounding to an output type) run in the C
file ``nvfp4_oracle.c`` beside this one, in strict IEEE fp32 where the method
computes in fp32.  Contractions are a float64 ``numpy.matmul`` of exactly
decoded operands, then one rounding to the output type.

Sources (page title, then file / section):
  [P1] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 8: ops.cpp (qqmm validation,
       fp_quantize / fp_dequantize fallbacks), primitives.cpp QQMatmul::vjp.
  [P2] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 7: fp_quantize.cu kernels;
       qqmm.cpp QQMatmul::eval_gpu (M=1 route, dense route, alpha).
  [P3] "[Metal] global scale for qmm" (ml-explore/mlx pull 4458): the worked
       example (global scale applied before the cast to bf16).
  [P4] osaurus-ai/mlx pull 31: cases A-D; "The fix" (scale per block).
  [P5] "mlx 0.30.7" diff, page 71: qqmm_utils.cu 128x4 scale tiles.

Every function here is pinned by ``tests/test_oracle_*.py``; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")

# Oracle-local element-type tags (the C file's ORC_F32 / ORC_F16 / ORC_BF16).
DT = {"f32": 0, "f16": 1, "bf16": 2}
# numpy containers of raw elements; bf16 is carried as its uint16 bit pattern.
NP_CONTAINER = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c with gcc (strict IEEE: no FMA contraction, no
    fast-math) into oracle/_build/liboracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        compile_source(_SRC, tmp)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def compile_source(src: str, out: str) -> None:
    """gcc with the oracle's flags: C11, no FMA contraction, no fast-math,
    float expressions evaluated in their own type.  The mutation tests build
    edited copies of nvfp4_oracle.c with it."""
    subprocess.check_call([
        "gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
        "-fno-fast-math", "-fexcess-precision=standard", "-o", out, src, "-lm",
    ])


def _L():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
        return _lib


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sig = {
        "orc_e2m1_value": (ctypes.c_double, [I]),
        "orc_e4m3_value": (ctypes.c_double, [I]),
        "orc_e8m0_value": (ctypes.c_double, [I]),
        "orc_e2m1_rne_satfinite": (I, [ctypes.c_float]),
        "orc_e4m3_rne_satfinite": (I, [ctypes.c_float]),
        "orc_e8m0_ceil": (I, [ctypes.c_float]),
        "orc_round_to_format": (ctypes.c_double, [ctypes.c_double, I, I, ctypes.c_double]),
        "orc_round_to_type": (ctypes.c_double, [ctypes.c_double, I]),
        "orc_amax": (ctypes.c_float, [P, I, I64]),
        "orc_nvfp4_quantize": (None, [P, I, I64, I64, P, P, P]),
        "orc_nvfp4_block_scale": (ctypes.c_float, [ctypes.c_uint8, P]),
        "orc_nvfp4_dequantize": (None, [P, P, I64, I64, P, P, I]),
        "orc_nvfp4_decode_exact": (None, [P, P, I64, I64, P, P]),
        "orc_nvfp4_decode_blockscale": (None, [P, P, I64, I64, P, P]),
        "orc_nvfp4_quantize_dequantize": (None, [P, I, I64, I64, P, P]),
        "orc_mxfp8_quantize": (None, [P, I, I64, I64, P, P]),
        "orc_mxfp8_dequantize": (None, [P, P, I64, I64, P, I]),
        "orc_mxfp8_decode_exact": (None, [P, P, I64, I64, P]),
        "orc_mxfp4_quantize": (None, [P, I, I64, I64, P, P]),
        "orc_philox4x32_10": (None, [P, P, P]),
        "orc_sr_bits": (ctypes.c_uint32, [ctypes.c_uint64, ctypes.c_uint64]),
        "orc_e2m1_sr_satfinite": (I, [ctypes.c_float, ctypes.c_uint32]),
        "orc_nvfp4_quantize_sr": (None, [P, I, I64, I64, P, ctypes.c_uint64, P, P]),
        "orc_mxfp4_dequantize": (None, [P, P, I64, I64, P, I]),
        "orc_mxfp4_decode_exact": (None, [P, P, I64, I64, P]),
        "orc_swizzle_scales": (None, [P, I64, I64, P]),
        "orc_load_array": (None, [P, I, I64, P]),
        "orc_store_array": (None, [P, I64, I, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _g(g):
    """Global scale as a pointer to one fp32, or NULL."""
    if g is None:
        return None, None
    buf = np.array([g], dtype=np.float32)
    return buf, _p(buf)


def _raw(x: np.ndarray, dt: str) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == NP_CONTAINER[dt], (x.dtype, dt)
    return x


# --------------------------------------------------------------------------
# scalar format functions (exposed for the pins)
# --------------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return _L().orc_e2m1_value(code)


def e4m3_value(byte: int) -> float:
    return _L().orc_e4m3_value(byte)


def e8m0_value(byte: int) -> float:
    return _L().orc_e8m0_value(byte)


def e2m1_encode(v: float) -> int:
    return _L().orc_e2m1_rne_satfinite(v)


def e4m3_encode(v: float) -> int:
    return _L().orc_e4m3_rne_satfinite(v)


def e8m0_encode_ceil(v: float) -> int:
    return _L().orc_e8m0_ceil(v)


def round_to_format(v: float, p: int, emin: int, maxv: float) -> float:
    return _L().orc_round_to_format(v, p, emin, maxv)


# --------------------------------------------------------------------------
# element type conversion
# --------------------------------------------------------------------------
def to_f64(x: np.ndarray, dt: str) -> np.ndarray:
    """Exact float64 values of a raw array of element type dt."""
    x = _raw(x, dt)
    out = np.empty(x.shape, dtype=np.float64)
    _L().orc_load_array(_p(x), DT[dt], x.size, _p(out))
    return out


def round_to(v: np.ndarray, dt: str) -> np.ndarray:
    """Round float64 values to element type dt (RNE, IEEE overflow), raw."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=NP_CONTAINER[dt])
    _L().orc_store_array(_p(v), v.size, DT[dt], _p(out))
    return out


# --------------------------------------------------------------------------
# a1: tensor amax
# --------------------------------------------------------------------------
def amax(x: np.ndarray, dt: str) -> float:
    """g = max|x| as fp32 ([P1] QQMatmul::vjp's cotangent amax)."""
    x = _raw(x, dt)
    return float(_L().orc_amax(_p(x), DT[dt], x.size))


# --------------------------------------------------------------------------
# a2-a4: NVFP4 quantize, scale layout
# --------------------------------------------------------------------------
def nvfp4_quantize(x: np.ndarray, dt: str, g: float | None = None):
    """NVFP4 two-level quantize of a [rows, K] array ([P2] fp_quantize_rowwise
    with global scale).  Returns (codes uint32 [rows, K/8], scales uint8
    [rows, K/16] in the LINEAR layout)."""
    x = _raw(x, dt)
    rows, K = x.shape
    assert K % 16 == 0
    codes = np.zeros((rows, K // 8), dtype=np.uint32)
    scales = np.zeros((rows, K // 16), dtype=np.uint8)
    gb, gp = _g(g)
    _L().orc_nvfp4_quantize(_p(x), DT[dt], rows, K, gp, _p(codes), _p(scales))
    return codes, scales


def swizzle_scales(lin: np.ndarray) -> np.ndarray:
    """128x4-tile layout of a [rows, cols] scale matrix ([P5] qqmm_utils.cu),
    padded to [ceil128(rows), ceil4(cols)] with zeros."""
    lin = np.ascontiguousarray(lin, dtype=np.uint8)
    rows, cols = lin.shape
    Rp, Cp = (rows + 127) // 128 * 128, (cols + 3) // 4 * 4
    out = np.empty((Rp, Cp), dtype=np.uint8)
    _L().orc_swizzle_scales(_p(lin), rows, cols, _p(out))
    return out


# --------------------------------------------------------------------------
# a5: dequantize
# --------------------------------------------------------------------------
def nvfp4_dequantize(codes, scales, g=None, out_dt="bf16") -> np.ndarray:
    """w_hat = T(e2m1(q) * (f8(s) * g/2688)) ([P2] fp_dequantize)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 8
    out = np.empty((rows, K), dtype=NP_CONTAINER[out_dt])
    gb, gp = _g(g)
    _L().orc_nvfp4_dequantize(_p(codes), _p(scales), rows, K, gp, _p(out), DT[out_dt])
    return out


def nvfp4_block_scale(s: int, g=None) -> float:
    gb, gp = _g(g)
    return _L().orc_nvfp4_block_scale(s, gp)


def nvfp4_decode_exact(codes, scales, g=None) -> np.ndarray:
    """Exact float64 e2m1(q) * f8(s) * d(g) per element."""
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 8
    out = np.empty((rows, K), dtype=np.float64)
    gb, gp = _g(g)
    _L().orc_nvfp4_decode_exact(_p(codes), _p(scales), rows, K, gp, _p(out))
    return out


# --------------------------------------------------------------------------
# a6: quantize-dequantize (x_hat)
# --------------------------------------------------------------------------
def nvfp4_quantize_dequantize(x: np.ndarray, dt: str, g=None) -> np.ndarray:
    """x_hat in x's type ([P2] fp_quantize_dequantize with global scale)."""
    x = _raw(x, dt)
    rows, K = x.shape
    out = np.empty_like(x)
    gb, gp = _g(g)
    _L().orc_nvfp4_quantize_dequantize(_p(x), DT[dt], rows, K, gp, _p(out))
    return out


# --------------------------------------------------------------------------
# a11: MXFP8 quantize / dequantize
# --------------------------------------------------------------------------
def mxfp8_quantize(x: np.ndarray, dt: str):
    """MXFP8 quantize: 32-blocks, E8M0 scale rounded up, e4m3 codes
    ([P2] fp_quantize_rowwise with bits 8; [P3] mlxcel round-up note).
    Returns (codes uint32 [rows, K/4], scales uint8 [rows, K/32] LINEAR)."""
    x = _raw(x, dt)
    rows, K = x.shape
    assert K % 32 == 0
    codes = np.zeros((rows, K // 4), dtype=np.uint32)
    scales = np.zeros((rows, K // 32), dtype=np.uint8)
    _L().orc_mxfp8_quantize(_p(x), DT[dt], rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp8_dequantize(codes, scales, out_dt="bf16") -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 4
    out = np.empty((rows, K), dtype=NP_CONTAINER[out_dt])
    _L().orc_mxfp8_dequantize(_p(codes), _p(scales), rows, K, _p(out), DT[out_dt])
    return out


def mxfp8_decode_exact(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 4
    out = np.empty((rows, K), dtype=np.float64)
    _L().orc_mxfp8_decode_exact(_p(codes), _p(scales), rows, K, _p(out))
    return out


# --------------------------------------------------------------------------
# NVFP4 quantize with stochastic rounding of the codes
# --------------------------------------------------------------------------
def philox4x32_10(ctr, key):
    """Philox4x32-10 (Salmon et al., SC 2011): 4 counter words, 2 key words."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    _L().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_bits(seed: int, i: int) -> int:
    return int(_L().orc_sr_bits(seed, i))


def e2m1_sr(t: float, r: int) -> int:
    return int(_L().orc_e2m1_sr_satfinite(t, r))


def nvfp4_quantize_sr(x: np.ndarray, dt: str, g: float | None = None, seed: int = 0):
    """NVFP4 quantize whose codes are rounded stochastically (the scales as in
    nvfp4_quantize; random bits from Philox4x32-10 keyed by ``seed``, counter
    = flat element index / 4).  Returns (codes, scales LINEAR)."""
    x = _raw(x, dt)
    rows, K = x.shape
    assert K % 16 == 0
    codes = np.zeros((rows, K // 8), dtype=np.uint32)
    scales = np.zeros((rows, K // 16), dtype=np.uint8)
    gb, gp = _g(g)
    _L().orc_nvfp4_quantize_sr(_p(x), DT[dt], rows, K, gp, seed, _p(codes), _p(scales))
    return codes, scales


# --------------------------------------------------------------------------
# MXFP4 quantize / dequantize (the 4-bit codes with the mx scale)
# --------------------------------------------------------------------------
def mxfp4_quantize(x: np.ndarray, dt: str):
    """MXFP4 quantize: 32-blocks, E8M0 scale of max|x|/6 rounded up, e2m1
    codes ([P2] fp_quantize_rowwise with bits 4 and the mx scale).
    Returns (codes uint32 [rows, K/8], scales uint8 [rows, K/32] LINEAR)."""
    x = _raw(x, dt)
    rows, K = x.shape
    assert K % 32 == 0
    codes = np.zeros((rows, K // 8), dtype=np.uint32)
    scales = np.zeros((rows, K // 32), dtype=np.uint8)
    _L().orc_mxfp4_quantize(_p(x), DT[dt], rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp4_dequantize(codes, scales, out_dt="bf16") -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 8
    out = np.empty((rows, K), dtype=NP_CONTAINER[out_dt])
    _L().orc_mxfp4_dequantize(_p(codes), _p(scales), rows, K, _p(out), DT[out_dt])
    return out


def mxfp4_decode_exact(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 8
    out = np.empty((rows, K), dtype=np.float64)
    _L().orc_mxfp4_decode_exact(_p(codes), _p(scales), rows, K, _p(out))
    return out


# --------------------------------------------------------------------------
# a8-a9, a12: dense block-scaled matmul y = x_hat . w_hat^T
# --------------------------------------------------------------------------
def qqmm(a_codes, a_scales, b_codes, b_scales, mode="nvfp4", g_x=None, g_w=None,
         out_dt="bf16", rows=None):
    """Dense quantized matmul of two quantized operands, w given as [N, K]
    ([P2] QQMatmul::eval_gpu dense route; alpha = g_x g_w / 2688^2).

    Operands are decoded exactly in float64 (per-block scale times the global
    decode factor; no rounding to T anywhere before the sum), the contraction
    is a float64 matmul, the result is rounded once to out_dt.
    ``rows`` optionally selects a subset of output rows.
    Returns dict(y_ref=float64 [M', N], abs_ref=sum |x_hat w_hat|, y=raw T)."""
    a_codes = np.asarray(a_codes)
    a_scales = np.asarray(a_scales)
    if rows is not None:
        a_codes, a_scales = a_codes[rows], a_scales[rows]
    if mode == "nvfp4":
        xh = nvfp4_decode_exact(a_codes, a_scales, g_x)
        wh = nvfp4_decode_exact(b_codes, b_scales, g_w)
    elif mode == "mxfp8":
        assert g_x is None and g_w is None
        xh = mxfp8_decode_exact(a_codes, a_scales)
        wh = mxfp8_decode_exact(b_codes, b_scales)
    elif mode == "mxfp4":
        assert g_x is None and g_w is None
        xh = mxfp4_decode_exact(a_codes, a_scales)
        wh = mxfp4_decode_exact(b_codes, b_scales)
    else:
        raise ValueError(mode)
    y_ref = xh @ wh.T
    abs_ref = np.abs(xh) @ np.abs(wh).T
    return {"y_ref": y_ref, "abs_ref": abs_ref, "y": round_to(y_ref, out_dt)}


def qqmm_vjp(x, w, cotan, dt: str, g_x: float, g_w: float):
    """Backward pass of y = qqmm(x, w) in NVFP4 mode ([P1] primitives.cpp
    QQMatmul::vjp), each product a fresh quantize of both operands followed by
    the dense quantized matmul above:
      dx [M, K] = cotan_hat . ((w^T)_hat)^T, cotan quantized along N with
                  g_c = amax(cotan), w^T [K, N] quantized along N with g_w;
      dw [N, K] = (cotan^T)_hat . ((x^T)_hat)^T, cotan^T [N, M] and x^T [K, M]
                  quantized along M, with g_c and g_x.
    x [M, K], w [N, K], cotan [M, N] are raw arrays of dt.  Returns
    (dx, dw), each qqmm's dict with the output in dt."""
    x, w, cotan = np.asarray(x), np.asarray(w), np.asarray(cotan)
    g_c = amax(cotan, dt)
    c_codes, c_scales = nvfp4_quantize(cotan, dt, g_c)
    wt_codes, wt_scales = nvfp4_quantize(np.ascontiguousarray(w.T), dt, g_w)
    dx = qqmm(c_codes, c_scales, wt_codes, wt_scales, "nvfp4", g_c, g_w, dt)
    ct_codes, ct_scales = nvfp4_quantize(np.ascontiguousarray(cotan.T), dt, g_c)
    xt_codes, xt_scales = nvfp4_quantize(np.ascontiguousarray(x.T), dt, g_x)
    dw = qqmm(ct_codes, ct_scales, xt_codes, xt_scales, "nvfp4", g_c, g_x, dt)
    return dx, dw


# --------------------------------------------------------------------------
# a6-a7: qmv (small-M route of qqmm with pre-quantized w)
# --------------------------------------------------------------------------
def nvfp4_decode_blockscale(codes, scales, g=None) -> np.ndarray:
    """float64 e2m1(q) * fp32(f8(s) * d(g)) per element (exact product)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 8
    out = np.empty((rows, K), dtype=np.float64)
    gb, gp = _g(g)
    _L().orc_nvfp4_decode_blockscale(_p(codes), _p(scales), rows, K, gp, _p(out))
    return out


def qmv(x, x_dt, g_x, w_codes, w_scales, g_w):
    """y = x_hat . w_hat^T for a small number of rows of x ([P2] qqmm.cpp M=1
    route: fp_quantize_dequantize then fp_qmv).  x_hat is x quantize-
    dequantized with g_x, in x's type (materialized, as the kernel writes
    it); w_hat = e2m1(q) * (f8(s) * g_w / 2688) with the block scale formed
    in fp32 and the global scale on each block scale ([P4] "The fix"); the
    weight is not rounded to T on this route.  float64 sum, one rounding
    to T."""
    xh = to_f64(nvfp4_quantize_dequantize(x, x_dt, g_x), x_dt)
    wh = nvfp4_decode_blockscale(w_codes, w_scales, g_w)
    y_ref = xh @ wh.T
    abs_ref = np.abs(xh) @ np.abs(wh).T
    return {"y_ref": y_ref, "abs_ref": abs_ref, "y": round_to(y_ref, x_dt)}


def qmv_mx(x, x_dt, w_codes, w_scales, mode):
    """qmv in an MX mode ([P2] qqmm.cpp M=1 route: fp_quantize_dequantize of x
    with the mode's group size 32 and bits, then fp_qmv; no global scales,
    [P1] validate_global_scale).  x_hat = the mode's quantize then dequantize
    of x, in x's type (materialized); w_hat = code * 2^(s-127) decoded
    exactly.  float64 sum, one rounding to T."""
    if mode == "mxfp8":
        quant, deq, dec = mxfp8_quantize, mxfp8_dequantize, mxfp8_decode_exact
    elif mode == "mxfp4":
        quant, deq, dec = mxfp4_quantize, mxfp4_dequantize, mxfp4_decode_exact
    else:
        raise ValueError(mode)
    xc, xs = quant(x, x_dt)
    xh = to_f64(deq(xc, xs, x_dt), x_dt)
    wh = dec(w_codes, w_scales)
    y_ref = xh @ wh.T
    abs_ref = np.abs(xh) @ np.abs(wh).T
    return {"y_ref": y_ref, "abs_ref": abs_ref, "y": round_to(y_ref, x_dt)}


# --------------------------------------------------------------------------
# a10: gather_qmm (MoE) with per-expert global scales
# --------------------------------------------------------------------------
def gather_qmm(x, w_codes, w_scales, g, idx, tokens=None, x_dt="bf16", transpose=True):
    """y[t, j, :] = x[t] . w_hat_e^T with e = idx[t, j] ([P3] "[Metal] global
    scale for qmm": the per-expert global scale multiplies each block scale
    inside dequantization, before the cast to T).  transpose=True: w is
    [E, N, K] (transposed weights, quantized along K); transpose=False
    (the other layout the pull's tests loop over): w is [E, K, N], quantized
    along N, and y[t, j, :] = x[t] . w_hat_e.  g is [E] or None.  float64
    sum, one rounding to T.  ``tokens`` optionally selects a subset of tokens.
    Returns dict(y_ref float64 [T', topk, N], abs_ref, y raw)."""
    x = _raw(x, x_dt)
    idx = np.asarray(idx)
    tok = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    E = w_codes.shape[0]
    N = w_codes.shape[1] if transpose else w_codes.shape[2] * 8
    topk = idx.shape[1]
    xf = to_f64(np.ascontiguousarray(x[tok]), x_dt)
    y_ref = np.zeros((len(tok), topk, N), dtype=np.float64)
    abs_ref = np.zeros_like(y_ref)
    used = np.unique(idx[tok])
    for e in used:
        ge = None if g is None else float(g[e])
        wh = to_f64(nvfp4_dequantize(w_codes[e], w_scales[e], ge, x_dt), x_dt)
        if not transpose:
            wh = wh.T  # [K, N] decoded along its rows (N): the matmul takes w_hat itself
        ti, ji = np.nonzero(idx[tok] == e)
        y_ref[ti, ji] = xf[ti] @ wh.T
        abs_ref[ti, ji] = np.abs(xf[ti]) @ np.abs(wh).T
    return {"y_ref": y_ref, "abs_ref": abs_ref, "y": round_to(y_ref, x_dt)}
