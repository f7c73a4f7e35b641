"""Shared helpers of the test suite: tensor <-> numpy raw conversions and the
output tolerances stated for the method.

Tolerances (written here once, used by every parity test):
- codes, scale bytes, amax, dequantized values: bit-exact;
- fp32 GEMM outputs: |y - y_ref| <= 1e-5 * sum_k |x_hat_k w_hat_k| + 1e-30;
- bf16 / fp16 GEMM outputs: within one ulp (of the output type) of the
  correctly rounded oracle value; near cancellation the fp32 floor
  1e-5 * sum_k |x_hat_k w_hat_k| also accepts (the count is reported).
"""
import numpy as np
import torch

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
NAME_DT = {v: k for k, v in TORCH_DT.items()}


def raw(t: torch.Tensor) -> np.ndarray:
    """numpy raw container of a CPU/GPU tensor: float32, float16 or bf16 bits."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float16:
        return t.numpy()
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype == torch.int32:
        return t.numpy().view(np.uint32)
    if t.dtype == torch.uint8:
        return t.numpy()
    raise TypeError(t.dtype)


def ulp(v: np.ndarray, dt: str) -> np.ndarray:
    """Spacing of the output type at |v| (v already representable)."""
    p, emin = {"bf16": (8, -126), "f16": (11, -14), "f32": (24, -126)}[dt]
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return np.exp2(e - (p - 1))


def check_gemm_output(y_gpu_raw, r, dt, orc, floor_rel=1e-5):
    """Compare a GEMM result with the oracle's dict(y_ref, abs_ref, y).
    Returns the number of elements accepted only through the fp32 floor."""
    y = orc.to_f64(np.ascontiguousarray(y_gpu_raw), dt)
    y_ref, abs_ref = r["y_ref"], r["abs_ref"]
    floor = floor_rel * abs_ref + 1e-30
    if dt == "f32":
        bad = np.abs(y - y_ref) > floor
        assert not bad.any(), _report(y, y_ref, abs_ref, bad)
        return 0
    yr = orc.to_f64(r["y"], dt)
    within_ulp = np.abs(y - yr) <= ulp(yr, dt)
    within_floor = np.abs(y - y_ref) <= floor
    bad = ~(within_ulp | within_floor)
    assert not bad.any(), _report(y, y_ref, abs_ref, bad)
    return int(np.count_nonzero(~within_ulp & within_floor))


def _report(y, y_ref, abs_ref, bad):
    i = np.argwhere(bad)[:8]
    return f"{int(bad.sum())} mismatches, e.g. " + ", ".join(
        f"{tuple(j)}: got {y[tuple(j)]!r} want {y_ref[tuple(j)]!r} (sum|.|={abs_ref[tuple(j)]:.4g})" for j in i)
