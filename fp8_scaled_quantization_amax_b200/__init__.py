"""FP8 scaled quantization for NVIDIA B200 (sm_100a).

amax -> scale (per tensor, per row with power-of-two scales, per 1x128 /
128x128 block) -> saturating round-to-nearest-even cast to E4M3 / E5M2 ->
FP8 scaled GEMM (tcgen05 tensor cores, fp32 accumulation, bf16 epilogue),
plus the delayed-scaling amax history and the FP8 KV cache.

The product is the C-ABI library ``libfp8q.so`` (``include/fp8q.h``); the
module :mod:`.fp8q` is its Python binding.  ``inputs`` holds the seeded
synthetic workloads.
"""
from . import fp8q  # noqa: F401  (binding; loads the library on first call)
