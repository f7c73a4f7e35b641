"""The documented argument rules of include/nvfp4.h, restated in Python, give
the status the library returns for random sizes (CPU only).  Without a GPU a
call that passes every host check reaches the device query and fails with a
CUDA status, so each call lands in one of three classes: refused on the host
(invalid / unsupported), done on the host (an empty output: OK), or needing
the device."""
import pytest
from hypothesis import given, settings, strategies as st

A = 0x10000  # a fake, 16-byte aligned device address: never dereferenced
OK, INVALID, UNSUPPORTED = 0, 1, 2
MAX_ELEMS = 1 << 34


@pytest.fixture(scope="module")
def L():
    from mxfp8_block_scaled_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4.lib()


def cls(status):
    return status if status in (OK, INVALID, UNSUPPORTED) else "device"


dims = st.one_of(st.integers(-3, 3), st.sampled_from([16, 32, 48, 64, 96, 256, 4096]),
                 st.integers(-(1 << 40), 1 << 40), st.sampled_from([1 << 30, (1 << 30) + 1, 1 << 34, 1 << 62]))


def quantize_rule(rows, K, group):
    if rows < 0 or K < 0 or (K and rows > MAX_ELEMS // K):
        return INVALID
    if K % group:
        return INVALID
    return OK if rows * K == 0 else "device"


@settings(max_examples=300, deadline=None)
@given(rows=dims, K=dims)
def test_quantize_family_rules(L, rows, K):
    assert cls(L.nvfp4_quantize(A, 2, rows, K, None, A, A, 0, None)) == quantize_rule(rows, K, 16)
    assert cls(L.nvfp4_quantize_sr(A, 2, rows, K, None, 1, A, A, 1, None)) == quantize_rule(rows, K, 16)
    assert cls(L.mxfp8_quantize(A, 2, rows, K, A, A, 0, None)) == quantize_rule(rows, K, 32)
    assert cls(L.mxfp4_quantize(A, 2, rows, K, A, A, 1, None)) == quantize_rule(rows, K, 32)
    assert cls(L.nvfp4_dequantize(A, A, 0, rows, K, None, A, 2, None)) == quantize_rule(rows, K, 16)
    assert cls(L.mxfp8_dequantize(A, A, 1, rows, K, A, 0, None)) == quantize_rule(rows, K, 32)


def qqmm_rule(M, N, K):
    lim = 1 << 30
    if M < 0 or N < 0 or K < 0 or M > lim or N > lim or K > lim or K % 32:
        return INVALID
    if K == 0 and M * N > 0:
        return INVALID
    return OK if M * N == 0 else "device"


@settings(max_examples=300, deadline=None)
@given(M=dims, N=dims, K=dims, mode=st.sampled_from([0, 1, 2]))
def test_qqmm_rules(L, M, N, K, mode):
    assert cls(L.qqmm(mode, M, N, K, A, A, A, A, None, None, A, 2, None)) == qqmm_rule(M, N, K)


def gather_rule(T, topk, E, N, K, kn):
    lim = 1 << 30
    if T < 0 or topk < 1 or E < 1 or N < 0 or K < 0 or T > lim // topk or N > lim or K > lim:
        return INVALID
    if K % 64 or N % (32 if kn else 16):
        return INVALID
    if K == 0 and T * N > 0:
        return INVALID
    if E > 1024 or E * (K if kn else N) > (1 << 31) - 1:
        return UNSUPPORTED
    return OK if T * N == 0 else "device"


@settings(max_examples=300, deadline=None)
@given(T=dims, topk=st.sampled_from([-1, 0, 1, 2, 8, 1 << 31]), E=st.sampled_from([0, 1, 4, 64, 1024, 1025]),
       N=dims, K=dims, kn=st.booleans())
def test_gather_rules(L, T, topk, E, N, K, kn):
    ws = 1 << 62  # a workspace size no valid call exceeds
    fn = L.gather_qmm_kn if kn else L.gather_qmm
    assert cls(fn(A, A, A, A, A, T, topk, E, N, K, A, A, ws, None)) == gather_rule(T, topk, E, N, K, kn)
