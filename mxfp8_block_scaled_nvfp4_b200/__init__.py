"""B200 (sm_100a) NVFP4 / MXFP8 block-scaled quantize, dequantize, qmv, qqmm
and gather_qmm: hand-written CUDA kernels behind the C ABI of include/nvfp4.h,
with a thin ctypes binding (``nvfp4``) and seeded synthetic inputs
(``workloads``)."""
from . import nvfp4  # noqa: F401
