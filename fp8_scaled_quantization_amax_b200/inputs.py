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
  * paged KV:     K [32 sequences x 8192 tokens, 32 heads, 128] ~ N(0, 1)
                  written into 16-token pages, each sequence's pages drawn at
                  random from the pool (a shuffled block table, as a cache
                  that has served many requests looks)
  * scale health: per-layer scale snapshots, log10(s) ~ N(1, 0.5^2), and a
                  next snapshot with every entry drifted by a factor
                  10**N(0, 0.05^2) and ``jump_frac`` of them multiplied or
                  divided by ``jump`` (the step changes a health check flags)
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


def scale_snapshots_f32(n: int, seed: int, jump_frac: float = 1e-3, jump: float = 16.0, device="cpu"):
    """Two fp32 snapshots (prev, cur) of n positive scale factors."""
    g = _gen(seed, device)
    prev = torch.pow(10.0, torch.randn(n, generator=g, device=device).mul_(0.5).add_(1.0))
    cur = prev * torch.pow(10.0, torch.randn(n, generator=g, device=device).mul_(0.05))
    k = int(round(jump_frac * n))
    if k:
        idx = torch.randperm(n, generator=g, device=device)[:k]
        up = torch.randint(0, 2, (k,), generator=g, device=device).bool()
        cur[idx] = torch.where(up, cur[idx] * jump, cur[idx] / jump)
    return prev.float(), cur.float()


def paged_layout(seq_lens, block_size: int, num_blocks: int, seed: int):
    """Block table [B, max_blocks] int32 (-1 = unused entry) giving every
    sequence ceil(len / block_size) distinct pages drawn at random from the
    pool, and the slot of every token, sequence-major: slot_mapping [sum(len)]
    int64 (= page * block_size + offset)."""
    g = _gen(seed, "cpu")
    lens = [int(n) for n in seq_lens]
    need = [(n + block_size - 1) // block_size for n in lens]
    if sum(need) > num_blocks:
        raise ValueError("pool too small for the sequences")
    mb = max(need) if need else 0
    perm = torch.randperm(num_blocks, generator=g)
    table = torch.full((len(lens), mb), -1, dtype=torch.int32)
    slots = []
    k = 0
    for b, n in enumerate(lens):
        pages = perm[k:k + need[b]]
        k += need[b]
        table[b, :need[b]] = pages.to(torch.int32)
        t = torch.arange(n)
        slots.append(pages[t // block_size].to(torch.int64) * block_size + t % block_size)
    slot_mapping = torch.cat(slots) if slots else torch.zeros(0, dtype=torch.int64)
    return table, slot_mapping


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
PAGED_KV = dict(B=32, S=8192, H=32, Dh=128, block_size=16)
# scale health check: the rowwise scales of every linear input of a 32-layer
# model (7 projections per layer) at 8192 tokens
SCALE_HEALTH = dict(layers=32 * 7, per_layer=8192)
KV = dict(B=32, H=32, S=8192, Dh=128)
