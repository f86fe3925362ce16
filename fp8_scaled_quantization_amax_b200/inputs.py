"""Seeded synthetic inputs shaped like the workloads of the FP8 pages.

This module holds NO arithmetic of the method (no amax, scale, cast or GEMM):
it only draws random bf16 tensors.  Both the CUDA path and the CPU oracle are
fed from it, so each side sees exactly the same bytes.

Workloads (Llama/Qwen-style linear layers and KV caches):
  * per-tensor:   A, B [256, 256] ~ N(0, 1)
  * rowwise:      activations [4096, 4096] ~ N(0, 1) with 0.1 % of the entries
                  (chosen uniformly without replacement) multiplied by 100,
                  weights [4096, 4096] ~ N(0, 0.02)
  * blockwise MLP: X [8192, 4096] ~ N(0, 1); W_up [11008, 4096] and
                  W_down [4096, 11008] ~ N(0, 0.02)
  * dgrad:        dY_t [8192, 4096] with |g| = 10**u, u ~ N(-2, (4/3)^2)
                  clipped to [-6, 2] (log-normal over 1e-6 .. 1e2), random
                  sign, seed = base + t; W [4096, 4096] ~ N(0, 0.02)
  * KV cache:     K, V [32, 32, 8192, 128] ~ N(0, 1)
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """bf16 tensor ~ N(0, std^2), drawn in fp32 then rounded to bf16."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def outlier_activations_bf16(shape, seed: int, frac: float = 1e-3, factor: float = 100.0,
                             device="cpu") -> torch.Tensor:
    """N(0, 1) activations with ``frac`` of the entries multiplied by ``factor``."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    n = x.numel()
    k = max(1, int(round(frac * n)))
    idx = torch.randperm(n, generator=g, device=device)[:k]
    x.view(-1)[idx] *= factor
    return x.to(torch.bfloat16)


def lognormal_grads_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """Gradients with |g| = 10**u, u ~ N(-2, (4/3)^2) clipped to [-6, 2],
    random sign."""
    g = _gen(seed, device)
    u = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    u.mul_(4.0 / 3.0).add_(-2.0).clamp_(-6.0, 2.0)
    mag = torch.pow(10.0, u)
    sign = torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.int8)
    mag = torch.where(sign.bool(), -mag, mag)
    return mag.to(torch.bfloat16)


def bf16_bits(x: torch.Tensor):
    """Raw uint16 bit patterns of a bf16 tensor as a numpy array (CPU copy)."""
    import numpy as np
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bf16_bits(bits, device="cpu") -> torch.Tensor:
    """bf16 tensor from uint16 bit patterns."""
    import numpy as np
    a = np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(a.copy()).view(torch.bfloat16).to(device)


# Named workloads: shapes only (the tests and the bench pick sizes from here).
PER_TENSOR = dict(M=256, N=256, K=256)
ROWWISE = dict(M=4096, N=4096, K=4096)
BLOCK_MLP = dict(M=8192, D=4096, F=11008)
DGRAD = dict(M=8192, N=4096, K=4096, steps=16)
KV = dict(B=32, H=32, S=8192, Dh=128)
