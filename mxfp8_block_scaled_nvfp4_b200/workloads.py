"""Seeded synthetic inputs for the NVFP4 / MXFP8 hot path.

This module only draws random numbers and shapes; it holds none of the
method's arithmetic (no amax, no scale, no rounding to a quantized format),
so that the CUDA path and the CPU oracle can both take their inputs from it.

Every generator takes a seed and a device and uses its own
``torch.Generator``; the same (seed, device) always gives the same tensor.

Workloads (shapes and distributions of the pages' tests and of the
decode / prefill / MoE / training settings the method serves):

=========  ==========================================================  =====
name       tensors                                                     seeds
=========  ==========================================================  =====
tiny       x [4,256] fp32 N(0,1); w [64,256] fp32 N(0,1), one stream   0
gemv       x [1,4096] bf16 N(0,1); W [14336,4096] bf16 N(0,0.02)       1, 2
prefill    x [4096,4096] bf16 N(0,1); W [4096,4096] bf16 N(0,0.02)     3, 4
           with exactly 1% of W's entries (randperm) multiplied by 50
moe        64 experts W_e [1408,2048] bf16 N(0,0.02); x [4096,2048]    5, 6
           bf16 N(0,1); per token 8 distinct experts (randperm(64))    7
mxfp8      x, W [8192,8192] bf16 N(0,1)                                8, 9
quant1g    x [32768,16384] bf16 N(0,1) (1 GiB)                         10
prefill_bwd  the prefill x and W, upstream gradient [4096,4096] bf16    3, 4, 11
           N(0,1) (synthetic: no model produces it here)
=========  ==========================================================  =====
"""
from __future__ import annotations

import torch

WORKLOADS = {
    "tiny": {"M": 4, "N": 64, "K": 256, "dtype": torch.float32, "seeds": (0,)},
    "gemv": {"M": 1, "N": 14336, "K": 4096, "dtype": torch.bfloat16, "seeds": (1, 2)},
    "prefill": {"M": 4096, "N": 4096, "K": 4096, "dtype": torch.bfloat16, "seeds": (3, 4)},
    "moe": {"T": 4096, "E": 64, "topk": 8, "N": 1408, "K": 2048, "dtype": torch.bfloat16,
            "seeds": (5, 6, 7)},
    "mxfp8": {"M": 8192, "N": 8192, "K": 8192, "dtype": torch.bfloat16, "seeds": (8, 9)},
    # the mxfp8 GEMM's operands quantized in the MXFP4 mode instead
    "mxfp4": {"M": 8192, "N": 8192, "K": 8192, "dtype": torch.bfloat16, "seeds": (8, 9)},
    "quant1g": {"R": 32768, "K": 16384, "dtype": torch.bfloat16, "seeds": (10,)},
    "prefill_bwd": {"M": 4096, "N": 4096, "K": 4096, "dtype": torch.bfloat16, "seeds": (3, 4, 11)},
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32, then stored as ``dtype``."""
    t = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def normal_with_outliers(shape, std: float, frac: float, factor: float, seed: int,
                         dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, std^2) with exactly round(frac * numel) entries, chosen by a
    random permutation, multiplied by ``factor`` (the prefill weight)."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    n = t.numel()
    k = int(round(frac * n))
    pos = torch.randperm(n, generator=g, device=device)[:k]
    t.view(-1)[pos] *= factor
    return t.to(dtype)


def routing(T: int, E: int, topk: int, seed: int, device="cpu") -> torch.Tensor:
    """int32 [T, topk]: for each token, ``topk`` distinct experts, uniformly
    at random (the first topk entries of a fresh permutation of E)."""
    g = _gen(seed, device)
    keys = torch.rand(T, E, generator=g, device=device)
    return torch.argsort(keys, dim=1)[:, :topk].to(torch.int32).contiguous()


def make(name: str, device="cpu", scale_down: int = 1, seed_offset: int = 0) -> dict:
    """Inputs of a named workload.  ``scale_down`` > 1 divides the large
    dimensions (for CPU-sized variants with the same distributions).
    ``seed_offset`` k > 0 draws another instance of the same workload (every
    seed s becomes s + 1000 k): one per rank when each rank solves its own
    problem; k = 0 is the workload itself."""
    w = WORKLOADS[name]
    sd = max(1, int(scale_down))
    seeds = tuple(s + 1000 * int(seed_offset) for s in w["seeds"])
    if name == "tiny":
        g = _gen(seeds[0], device)
        x = torch.randn(w["M"], w["K"], generator=g, device=device, dtype=torch.float32)
        W = torch.randn(w["N"], w["K"], generator=g, device=device, dtype=torch.float32)
        return {"x": x, "w": W}
    if name in ("gemv", "prefill", "mxfp8", "mxfp4"):
        M, N, K = w["M"], w["N"], w["K"]
        if sd > 1:
            M, N = max(1, M // sd), max(1, N // sd)
        s0, s1 = seeds
        std_w = 0.02 if name in ("gemv", "prefill") else 1.0
        x = normal((M, K), 1.0, s0, w["dtype"], device)
        if name == "prefill":
            W = normal_with_outliers((N, K), 0.02, 0.01, 50.0, s1, w["dtype"], device)
        else:
            W = normal((N, K), std_w, s1, w["dtype"], device)
        return {"x": x, "w": W}
    if name == "moe":
        T, E, topk, N, K = w["T"], w["E"], w["topk"], w["N"], w["K"]
        if sd > 1:
            T, N = max(1, T // sd), max(8, N // sd)
        s_w, s_x, s_i = seeds
        W = normal((E, N, K), 0.02, s_w, w["dtype"], device)
        x = normal((T, K), 1.0, s_x, w["dtype"], device)
        idx = routing(T, E, topk, s_i, device)
        return {"x": x, "w": W, "idx": idx}
    if name == "prefill_bwd":
        d = make("prefill", device=device, scale_down=sd, seed_offset=seed_offset)
        M, N = d["x"].shape[0], d["w"].shape[0]
        d["cotan"] = normal((M, N), 1.0, seeds[2], w["dtype"], device)
        return d
    if name == "quant1g":
        R, K = w["R"], w["K"]
        if sd > 1:
            R = max(1, R // sd)
        return {"x": normal((R, K), 1.0, seeds[0], w["dtype"], device)}
    raise KeyError(name)
