"""Pins of the order of the fp32 operations in the oracle's NVFP4 quantizer
(CPU only).

"mlx 0.30.7.2 -> 0.30.7.6" diff, page 7, fp_quantize.cu fp_quantize_rowwise
computes the block scale as (amax / 6) * E and the code input as
x * (E / float(s)); the page-8 fallback (ops.cpp fp_quantize) orders the
code step as (x / float(s)) * E.  Real arithmetic cannot tell the orders
apart; fp32 rounding can.  tests/golden/quantize_operation_order.txt holds
two hand-derived blocks on which the orders give different scale bytes (R1)
or codes (R2), with every rounding written out.

The tests below (1) re-check each written-out rounding of that file with
numpy fp32 arithmetic and torch's e4m3 decode, (2) pin the oracle's scale
bytes and codes to the file, and (3) build edited copies of
oracle/nvfp4_oracle.c, each with one step in another order, and show that
the pin fails on every one of them while an unedited copy passes.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_operation_order.txt")
ORACLE_C = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "nvfp4_oracle.c")

f32 = np.float32


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        out[k] = v
    return out


G = _golden()


def _block(tag):
    g = float(G[f"{tag}_g"][0])
    x = np.array([[float(v) for v in G[f"{tag}_x"]]], dtype=np.float32)
    scale = int(G[f"{tag}_scale"][0], 16)
    codes = [int(c, 16) for c in G[f"{tag}_codes"]]
    return g, x, scale, codes


def _unpack(words):
    w = np.asarray(words, dtype=np.uint32).reshape(-1)
    return [int((w[i // 8] >> (4 * (i % 8))) & 15) for i in range(8 * w.size)]


def _e4m3(byte):
    return float(torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


# ---------------------------------------------------------------------------
# (1) the file's written-out roundings
# ---------------------------------------------------------------------------
def test_r1_derivation():
    g, x, scale, _ = _block("r1")
    a = f32(np.abs(x).max())
    E = f32(f32(2688.0) / f32(g))
    assert E == f32(float.fromhex("0x1.333334p+8"))
    t = f32(f32(a / f32(6.0)) * E)
    assert t == f32(float.fromhex(G["r1_t"][0]))
    other = f32(float.fromhex(G["r1_t_other_orders"][0]))
    assert f32(a * f32(E / f32(6.0))) == other
    assert f32(f32(a * E) / f32(6.0)) == other
    # 200 is the midpoint of the e4m3 neighbours 0x74 and 0x75
    assert (_e4m3(0x74) + _e4m3(0x75)) / 2 == float(other) == 200.0
    assert float(t) > 200.0 and _e4m3(scale) == 208.0


def test_r2_derivation():
    g, x, scale, _ = _block("r2")
    E = f32(f32(2688.0) / f32(g))
    a = f32(np.abs(x).max())
    t = f32(f32(a / f32(6.0)) * E)
    assert _e4m3(0x3C) < t < (_e4m3(0x3C) + _e4m3(0x3D)) / 2 and _e4m3(scale) == 1.5
    fs = f32(_e4m3(scale))
    xe = f32(x[0, 1])
    v = f32(xe * f32(E / fs))
    assert v == f32(float.fromhex(G["r2_v"][0]))
    other = f32(float.fromhex(G["r2_v_other_orders"][0]))
    assert f32(f32(xe / fs) * E) == other == f32(3.5)
    assert f32(f32(xe * f32(f32(1.0) / fs)) * E) == other
    assert float(v) < 3.5


# ---------------------------------------------------------------------------
# (2) the oracle against the file
# ---------------------------------------------------------------------------
def _check(quantize, tag):
    """True when quantize(x, g) gives the file's scale byte and codes."""
    g, x, scale, codes = _block(tag)
    q, s = quantize(x, g)
    return int(s.reshape(-1)[0]) == scale and _unpack(q) == codes


@pytest.mark.parametrize("tag", ["r1", "r2"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_oracle_matches_operation_order_blocks(orc, tag, dt):
    # every value of both blocks is exact in bf16, so the input type does not matter
    def quantize(x, g):
        xin = x if dt == "f32" else torch.from_numpy(x).to(torch.bfloat16).view(torch.uint16).numpy()
        return orc.nvfp4_quantize(xin, dt, g)
    assert _check(quantize, tag)


@pytest.mark.parametrize("tag", ["r1", "r2"])
def test_oracle_sr_scale_bytes_follow_the_same_order(orc, tag):
    g, x, scale, _ = _block(tag)
    _, s = orc.nvfp4_quantize_sr(x, "f32", g, seed=7)
    assert int(s.reshape(-1)[0]) == scale


# ---------------------------------------------------------------------------
# (3) edited copies of the oracle's C source
# ---------------------------------------------------------------------------
SCALE_STEP = "  float t = a / 6.0f;\n  t = t * E;\n"
CODE_STEP = "  float k = E / fs;\n  return x * k;\n"
MUTANTS = {
    # R1: the encode factor divided by 6 first, as one factor
    "scale_a_times_E_over_6": (SCALE_STEP, "  float t = a * (E / 6.0f);\n", "r1"),
    # R1: amax times the encode factor, then divided by 6
    "scale_aE_over_6": (SCALE_STEP, "  float t = (a * E) / 6.0f;\n", "r1"),
    # R2: the page-8 fallback's order, x / float(s) first
    "code_x_over_s_times_E": (CODE_STEP, "  return (x / fs) * E;\n", "r2"),
    # R2: the reciprocal of the scale first, as older code did
    "code_x_times_inv_s_times_E": (CODE_STEP, "  return (x * (1.0f / fs)) * E;\n", "r2"),
}


def _build_copy(orc, tmp_path, name, edit=None):
    src = open(ORACLE_C).read()
    if edit is not None:
        old, new = edit
        assert src.count(old) == 1, "the edited step must occur exactly once"
        src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    orc.compile_source(str(c), str(so))
    return orc.bind(ctypes.CDLL(str(so)))


def _quantize_with(lib):
    def quantize(x, g):
        x = np.ascontiguousarray(x, dtype=np.float32)
        rows, K = x.shape
        q = np.zeros((rows, K // 8), dtype=np.uint32)
        s = np.zeros((rows, K // 16), dtype=np.uint8)
        gb = np.array([g], dtype=np.float32)
        P = ctypes.c_void_p
        lib.orc_nvfp4_quantize(x.ctypes.data_as(P), 0, rows, K, gb.ctypes.data_as(P),
                               q.ctypes.data_as(P), s.ctypes.data_as(P))
        return q, s
    return quantize


def test_unedited_copy_passes(orc, tmp_path):
    lib = _build_copy(orc, tmp_path, "control")
    assert _check(_quantize_with(lib), "r1") and _check(_quantize_with(lib), "r2")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutation_of_the_operation_order_fails_its_pin(orc, tmp_path, name):
    old, new, tag = MUTANTS[name]
    lib = _build_copy(orc, tmp_path, name, (old, new))
    assert not _check(_quantize_with(lib), tag)
