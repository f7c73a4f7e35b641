"""Pins of the oracle's gather_qmm with transpose=False (weights stored
[E, K, N], quantized along N), the other layout the tests of "[Metal] global
scale for qmm" (ml-explore/mlx pull 4458) loop over (CPU only)."""
import numpy as np
import torch


def bf16(t):
    return torch.as_tensor(np.asarray(t, dtype=np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def bf16_value(bits):
    return torch.from_numpy(np.asarray(bits, dtype=np.uint16).copy()).view(torch.bfloat16).to(torch.float64).numpy()


def test_worked_example_in_kn_layout(orc):
    """The page's worked example with the weight laid out [K, N]: every code
    6, block scale 0.5 (blocks of 16 along N), global scale 0.1 (g = 268.8):
    w_hat = bf16(6 * fp32(0.5 * 0.1)) = 0.30078125 and, with x = 1 and
    K = 4096, y = 1232.0 in every output column; expert 1 decodes with
    g = 2688 (factor 1): y = 4096 * 3."""
    K, N = 4096, 48
    codes = np.full((2, K, N // 8), 0x77777777, dtype=np.uint32)     # code 7 = 6.0
    scales = np.full((2, K, N // 16), 0x30, dtype=np.uint8)           # e4m3 0.5
    g = np.array([np.float32(268.8), 2688.0], dtype=np.float32)
    x = bf16(np.ones((3, K)))
    idx = np.array([[0, 1], [1, 0], [0, 1]], dtype=np.int32)
    r = orc.gather_qmm(x, codes, scales, g, idx, transpose=False)
    y = bf16_value(r["y"])
    assert y.shape == (3, 2, N)
    for t in range(3):
        for j in range(2):
            assert np.all(y[t, j] == (1232.0 if idx[t, j] == 0 else 4096 * 3.0))


def _grid_weight(rng, K, N):
    """e2m1-grid values with a +6 in every 16-block of every row and every
    column, so that quantizing along N (rows of W) and along K (rows of W^T)
    are both exact with block scale 1."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    w = mags[rng.integers(0, 7, (K, N))] * np.where(rng.random((K, N)) < 0.5, -1.0, 1.0)
    for k in range(K):
        w[k, (k % 16)::16] = 6.0
    return w.astype(np.float32)


def test_kn_layout_equals_transposed_layout_on_exact_weights(orc):
    rng = np.random.default_rng(8)
    E, K, N, T, topk = 3, 64, 48, 5, 2
    W = [_grid_weight(rng, K, N) for _ in range(E)]
    kn = [orc.nvfp4_quantize(W[e], "f32") for e in range(E)]              # along N
    nk = [orc.nvfp4_quantize(np.ascontiguousarray(W[e].T), "f32") for e in range(E)]  # along K
    assert all(np.all(s == 0x38) for _, s in kn) and all(np.all(s == 0x38) for _, s in nk)
    x = bf16(rng.standard_normal((T, K)))
    idx = np.array([rng.permutation(E)[:topk] for _ in range(T)], dtype=np.int32)
    g = np.array([2688.0, 1344.0, 5376.0], dtype=np.float32)  # decode factors 1, 1/2, 2: exact
    r_kn = orc.gather_qmm(x, np.stack([c for c, _ in kn]), np.stack([s for _, s in kn]), g, idx, transpose=False)
    r_nk = orc.gather_qmm(x, np.stack([c for c, _ in nk]), np.stack([s for _, s in nk]), g, idx)
    np.testing.assert_array_equal(r_kn["y_ref"], r_nk["y_ref"])
    # and both equal x . (W_e * g_e / 2688) computed directly
    xf = bf16_value(x)
    for t in range(T):
        for j in range(topk):
            e = idx[t, j]
            np.testing.assert_allclose(r_kn["y_ref"][t, j], xf[t] @ (W[e].astype(np.float64) * g[e] / 2688.0),
                                       rtol=0, atol=1e-9)


def test_mutation_kn_without_transposing_fails(orc):
    """Mistake: take the [K, N] decode as if it were [N, K] (no transpose of
    the decoded weight).  With K != N the product is not even defined; with
    K == N it gives x . w_hat^T, which the exact-weights pin rejects."""
    rng = np.random.default_rng(9)
    K = N = 48
    W = _grid_weight(rng, K, N)
    c, s = orc.nvfp4_quantize(W, "f32")
    x = bf16(rng.standard_normal((3, K)))
    idx = np.zeros((3, 1), dtype=np.int32)
    right = orc.gather_qmm(x, c[None], s[None], None, idx, transpose=False)["y_ref"]
    wrong = orc.gather_qmm(x, c[None], s[None], None, idx, transpose=True)["y_ref"]  # w_hat used as [N, K]
    assert not np.array_equal(right, wrong)
    xf = bf16_value(x)
    np.testing.assert_allclose(right[:, 0], xf @ W.astype(np.float64), rtol=0, atol=1e-9)
