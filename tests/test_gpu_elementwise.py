"""GPU parity of amax, NVFP4 / MXFP8 quantize and dequantize and the scale
re-layout against the CPU oracle (bit-exact), through the C ABI."""
import numpy as np
import pytest
import torch

from helpers import TORCH_DT, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    assert torch.cuda.is_available()
    return nvfp4


def make_x(shape, dt, seed, std=1.0):
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    return workloads.normal(shape, std, seed, TORCH_DT[dt], "cpu")


SHAPES = [(1, 16), (3, 48), (67, 256), (128, 4096), (200, 1040), (257, 64)]


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("n", [1, 7, 8, 4096, 100003])
def test_amax_parity(nv, orc, dt, n):
    x = make_x((n,), dt, 20 + n)
    g = nv.amax(x.cuda())
    assert g.item() == orc.amax(raw(x), dt)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("use_g", [False, True])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_nvfp4_quantize_parity(nv, orc, dt, shape, use_g, layout):
    x = make_x(shape, dt, 1000 + shape[0] * 7 + shape[1], std=0.02 if dt != "f16" else 1.0)
    xg = x.cuda()
    g = nv.amax(xg) if use_g else None
    codes, scales = nv.nvfp4_quantize(xg, g, layout)
    torch.cuda.synchronize()
    oc, os_ = orc.nvfp4_quantize(raw(x), dt, None if g is None else g.item())
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)


@pytest.mark.parametrize("tag", ["r1", "r2"])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_nvfp4_quantize_operation_order_blocks(nv, tag, dt):
    """The hand-derived blocks on which the fp32 order of the scale step (r1)
    or the code step (r2) changes the result: the kernel gives the bytes and
    codes of "mlx 0.30.7.2 -> 0.30.7.6" page 7 fp_quantize_rowwise's order
    (tests/golden/quantize_operation_order.txt), with round-to-nearest and,
    for the scale byte, with stochastic rounding."""
    from test_oracle_operation_order import _block, _unpack
    g, x, scale, codes = _block(tag)
    xg = torch.from_numpy(x).to(TORCH_DT[dt]).cuda()
    gg = torch.tensor([g], dtype=torch.float32, device="cuda")
    q, s = nv.nvfp4_quantize(xg, gg, "linear")
    torch.cuda.synchronize()
    assert int(raw(s).reshape(-1)[0]) == scale
    assert _unpack(raw(q)) == codes
    _, s_sr = nv.nvfp4_quantize_sr(xg, gg, 7, "linear")
    torch.cuda.synchronize()
    assert int(raw(s_sr).reshape(-1)[0]) == scale


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("out_dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_nvfp4_dequantize_parity(nv, orc, dt, out_dt, layout):
    x = make_x((67, 272), dt, 5)
    xg = x.cuda()
    g = nv.amax(xg)
    codes, scales = nv.nvfp4_quantize(xg, g, layout)
    out = nv.nvfp4_dequantize(codes, scales, g, layout, TORCH_DT[out_dt])
    oc, os_ = orc.nvfp4_quantize(raw(x), dt, g.item())
    want = orc.nvfp4_dequantize(oc, os_, g.item(), out_dt)
    assert np.array_equal(raw(out).view(np.uint8), want.view(np.uint8))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 32), (67, 256), (130, 4128), (256, 8192)])
@pytest.mark.parametrize("layout", ["linear", "swizzled"])
def test_mxfp8_quantize_parity(nv, orc, dt, shape, layout):
    x = make_x(shape, dt, 77 + shape[0])
    codes, scales = nv.mxfp8_quantize(x.cuda(), layout)
    oc, os_ = orc.mxfp8_quantize(raw(x), dt)
    assert np.array_equal(raw(codes), oc)
    want_s = os_ if layout == "linear" else orc.swizzle_scales(os_)
    assert np.array_equal(raw(scales), want_s)


@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
def test_mxfp8_dequantize_parity(nv, orc, out_dt):
    x = make_x((67, 256), "bf16", 3)
    codes, scales = nv.mxfp8_quantize(x.cuda(), "linear")
    out = nv.mxfp8_dequantize(codes, scales, "linear", TORCH_DT[out_dt])
    oc, os_ = orc.mxfp8_quantize(raw(x), "bf16")
    want = orc.mxfp8_dequantize(oc, os_, out_dt)
    assert np.array_equal(raw(out).view(np.uint8), want.view(np.uint8))


@pytest.mark.parametrize("rows,cols", [(1, 1), (67, 16), (128, 4), (200, 5), (300, 256)])
def test_swizzle_scales_parity(nv, orc, rows, cols):
    lin = torch.randint(0, 256, (rows, cols), dtype=torch.uint8, generator=torch.Generator().manual_seed(rows))
    out = nv.swizzle_scales(lin.cuda())
    assert np.array_equal(raw(out), orc.swizzle_scales(raw(lin)))


# --- sweeps that drive every conversion through its rounding boundaries ----

def _all_bf16_in(lo, hi):
    bits = np.arange(65536, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) >= lo) & (np.abs(v) <= hi)]
    return v


def test_e2m1_conversion_sweep(nv, orc):
    """Blocks whose amax is 6 (scale byte 1.0, encode factor 1): the codes are
    e2m1(x) of every bf16 value in [-6, 6] plus midpoints and their fp32
    neighbours; checks rounding, ties-to-even, saturation and -0."""
    vals = list(_all_bf16_in(0, 6.0))
    grid = [0, .5, 1, 1.5, 2, 3, 4, 6]
    for a, b in zip(grid[:-1], grid[1:]):
        m = np.float32((a + b) / 2)
        for v in (m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(7))):
            vals += [v, -v]
    vals += [np.float32(-0.0), np.float32(-1e-30), np.float32(1e-30)]
    vals = np.array(vals, dtype=np.float32)
    n15 = (len(vals) + 14) // 15
    x = np.zeros((n15, 16), dtype=np.float32)
    x[:, 0] = 6.0
    x.reshape(-1)[np.arange(n15 * 16).reshape(n15, 16)[:, 1:].reshape(-1)[:len(vals)]] = vals
    xt = torch.from_numpy(x)
    codes, scales = nv.nvfp4_quantize(xt.cuda(), None, "linear")
    oc, os_ = orc.nvfp4_quantize(x, "f32", None)
    assert np.all(os_ == 0x38)
    got, want = raw(codes), oc
    if not np.array_equal(got, want):
        diff = np.nonzero(got != want)
        r, w = diff[0][0], diff[1][0]
        pytest.fail(f"e2m1 mismatch in row {r} word {w}: got {got[r, w]:08x} want {want[r, w]:08x}; "
                    f"inputs {x[r, 8 * w:8 * w + 8]}")
    assert np.array_equal(raw(scales), os_)


def test_e4m3_scale_conversion_sweep(nv, orc):
    """One block per amax value: amax over all positive bf16 values (no
    global scale), so the scale byte is e4m3(amax / 6) across subnormals,
    normals and saturation."""
    a = _all_bf16_in(1e-38, 3e38)
    a = a[a > 0]
    x = np.zeros((len(a), 16), dtype=np.float32)
    x[:, 3] = a
    x[:, 7] = -a / 3
    codes, scales = nv.nvfp4_quantize(torch.from_numpy(x).cuda(), None, "linear")
    oc, os_ = orc.nvfp4_quantize(x, "f32", None)
    assert np.array_equal(raw(scales), os_)
    assert np.array_equal(raw(codes), oc)


def test_ue8m0_scale_conversion_sweep(nv, orc):
    """MXFP8: amax over all positive bf16 values, so the scale byte is the
    rounded-up e8m0 of amax / 448 across the whole range (tiny values give
    fp32 subnormal quotients)."""
    a = _all_bf16_in(1e-38, 3e38)
    a = a[a > 0]
    x = np.zeros((len(a), 32), dtype=np.float32)
    x[:, 5] = a
    x[:, 6] = -a * np.float32(0.7)
    codes, scales = nv.mxfp8_quantize(torch.from_numpy(x).cuda(), "linear")
    oc, os_ = orc.mxfp8_quantize(x, "f32")
    assert np.array_equal(raw(scales), os_)
    assert np.array_equal(raw(codes), oc)


def test_global_scale_worked_example_on_gpu(nv, orc):
    """Dequantize of the "[Metal] global scale for qmm" example on the GPU:
    code 6, block scale 0.5, decode factor 0.1 gives bf16 0.30078125."""
    K = 4096
    codes = torch.full((1, K // 8), 0x77777777, dtype=torch.int32).cuda()
    scales = torch.full((1, K // 16), 0x30, dtype=torch.uint8).cuda()
    g = torch.tensor([268.8], dtype=torch.float32).cuda()
    w = nv.nvfp4_dequantize(codes, scales, g, "linear", torch.bfloat16)
    assert torch.all(w.float() == 0.30078125)


def test_full_size_quantize_sampled_rows(nv, orc):
    """The 1 GiB bf16 tensor [32768, 16384], g = amax, SWIZZLED scales, in the
    launch configuration the benchmark times; 48 random rows compared with
    the oracle, plus the amax against torch's own reduction."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    x = workloads.make("quant1g", device="cuda")["x"]
    R, K = x.shape
    g = nv.amax(x)
    assert g.item() == x.abs().max().float().item()
    codes, scales = nv.nvfp4_quantize(x, g, "swizzled")
    rows = np.sort(np.random.default_rng(0).choice(R, 48, replace=False))
    xs = raw(x[torch.from_numpy(rows).cuda()])
    oc, os_ = orc.nvfp4_quantize(xs, "bf16", g.item())
    assert np.array_equal(raw(codes[torch.from_numpy(rows).cuda()]), oc)
    sc = raw(scales).reshape(-1)
    Cp = K // 16
    r = rows[:, None]
    c = np.arange(K // 16)[None, :]
    off = ((r // 128) * (Cp // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    assert np.array_equal(sc[off], os_)
    del x, codes, scales
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_amax_multi_parity(nv, orc, dt):
    """Several tensors in one launch (ragged lengths, an empty one): each
    output equals the oracle's amax of its tensor, with consecutive and with
    separate output buffers."""
    import ctypes
    xs = [make_x((n,), dt, 300 + n) for n in (100003, 7, 4096 * 3)]
    xs[1] = xs[1] * 40.0  # the largest values in the shortest tensor
    want = [orc.amax(raw(x), dt) for x in xs]
    gs = nv.amax_multi([x.cuda() for x in xs])
    assert gs.cpu().tolist() == want
    # separate outputs (one memset each) and an empty tensor, through the C ABI
    xg = [x.cuda() for x in xs] + [torch.empty(0, dtype=xs[0].dtype, device="cuda")]
    outs = [torch.full((1,), 7.0, device="cuda") for _ in xg]
    items = (nv.AmaxItem * 4)(*[nv.AmaxItem(x.data_ptr(), x.numel(), o.data_ptr()) for x, o in zip(xg, outs)])
    st = nv.lib().nvfp4_amax_multi(items, 4, nv.DT[xg[0].dtype], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert [o.item() for o in outs] == want + [0.0]


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_quantize_multi_parity(nv, orc, dt):
    """Four tensors of different shapes, layouts and global scales in one
    launch: every code and scale byte equals the oracle's (as one
    nvfp4_quantize per tensor), padding of the tile layout zero."""
    shapes = [(67, 256), (200, 1040), (1, 16), (257, 48)]
    layouts = ["swizzled", "linear", "linear", "swizzled"]
    xs = [make_x(s, dt, 500 + i, std=0.02 if dt != "f16" else 1.0) for i, s in enumerate(shapes)]
    xg = [x.cuda() for x in xs]
    gs = [nv.amax(xg[0]), None, nv.amax(xg[2]), nv.amax(xg[3])]
    # poison the outputs: every byte must be written
    jobs = []
    for x, g, lay in zip(xg, gs, layouts):
        rows, K = x.shape
        codes = torch.full((rows, K // 8), -1, dtype=torch.int32, device="cuda")
        scales = torch.full(nv.scale_shape(rows, K // 16, lay), 0xAB, dtype=torch.uint8, device="cuda")
        jobs.append((x, g, lay, codes, scales))
    outs = nv.nvfp4_quantize_multi(jobs)
    torch.cuda.synchronize()
    for x, g, lay, (codes, scales) in zip(xs, gs, layouts, outs):
        oc, os_ = orc.nvfp4_quantize(raw(x), dt, None if g is None else g.item())
        assert np.array_equal(raw(codes), oc)
        assert np.array_equal(raw(scales), os_ if lay == "linear" else orc.swizzle_scales(os_))


def test_qqmm_raw_matches_the_separate_calls(nv):
    """qqmm_raw (amax and quantize of both operands, one launch each, then
    the GEMM) gives bit for bit the result of the single-tensor calls."""
    x = make_x((300, 512), "bf16", 71).cuda()
    w = make_x((520, 512), "bf16", 72, std=0.02).cuda()
    y = nv.qqmm_raw(x, w)
    g_x, g_w = nv.amax(x), nv.amax(w)
    xc, xs = nv.nvfp4_quantize(x, g_x, "swizzled")
    wc, ws = nv.nvfp4_quantize(w, g_w, "swizzled")
    y2 = nv.qqmm(xc, xs, wc, ws, 512, "nvfp4", g_x, g_w)
    nv.check_device_errors()
    assert y.dtype == torch.bfloat16 and torch.equal(y.view(torch.int16), y2.view(torch.int16))
