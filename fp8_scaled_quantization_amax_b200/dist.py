"""Data-parallel plumbing for per-tensor FP8 scaling across ranks.

"DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.2 and §5.1: when each rank
scales its own gradients, the all-reduced result mixes scales; all ranks must
share one global scale (the global maximum) before the exchange.  For
per-tensor scaling that is a 4-byte MAX all-reduce of the amax; per-row,
per-block and KV-cache scaling need no exchange (each row / block / (b, h)
slice lives on one rank).

Every arithmetic step stays in the library's kernels: local amax
(``fp8_amax``), MAX all-reduce (NCCL through ``torch.distributed``), the scale
from the global amax (``fp8_amax_history_update`` with a one-entry history,
i.e. s = fmax / amax), and the cast with that scale
(``fp8_quantize_tensorwise`` with ``scale_in``).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In-place MAX all-reduce of a per-tensor amax (fp32 [1]) over the group."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Largest value over all ranks (used for max-over-ranks timings)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def quantize_tensorwise_global(x: torch.Tensor, fmt: int, group=None, counts=None):
    """Per-tensor quantization of this rank's shard with the scale of the
    global amax over all ranks.  Returns (q, scale_inv [1], global amax [1])."""
    from . import fp8q
    amax = fp8q.amax(x, counts)
    allreduce_amax_(amax, group)
    state = fp8q.AmaxHistory(1, fmt, device=x.device)
    state.update(amax)                         # scale = fmax / global amax
    q, scale_inv, _ = fp8q.quantize_tensorwise(x, fmt, scale_in=state.scale, want_amax=False)
    return q, scale_inv, amax
