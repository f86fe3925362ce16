"""GPU parity of the paged FP8 KV cache against the CPU oracle (bit-exact).

Sources: "ms-swift全链路能力解析：训练、推理、评测、量化与部署一体化解决方案" (KV cache in
fixed-size blocks allocated on demand) and "DeepL押注FP8：大模型训练与推理统一
精度实战解析" §3.1 (K and V kept in FP8, dequantized when read).  Every case
starts the device cache and the oracle's from the same stale bytes, so pages
the write must not touch are checked too.
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_codes_equal, assert_f32_equal, need_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _case(orc, fmt, H, Dh, lens, bs, NB, seed, S_out=None, specials=False):
    table, slots = inputs.paged_layout(lens, bs, NB, seed)
    T = slots.numel()
    slots = torch.cat([slots, torch.tensor([-1, NB * bs + 3], dtype=torch.int64)])   # padding tokens
    x = inputs.normal_bf16((T + 2, H, Dh), 2.0, seed=seed + 1)
    if specials and T > 3:
        x[0, 0, 1] = float("inf")
        x[1, H - 1, 2] = float("nan")
        x[2, 0] = 0.0
    rng = np.random.default_rng(seed)
    c0 = rng.integers(0, 256, (NB, bs, H, Dh)).astype(np.uint8)
    s0 = np.full((NB, bs, H), 3.0, np.float32)
    kv = fp8q.PagedKVCache(NB, bs, H, Dh, fmt)
    kv.cache.copy_(torch.from_numpy(c0))
    kv.scale_inv.copy_(torch.from_numpy(s0))
    kv.write(x.cuda(), slots.cuda())
    rc, rs = orc.paged_kv_write(inputs.bf16_bits(x), slots.numpy(), c0, s0, fmt)
    assert_codes_equal(to_np(kv.cache), rc, fmt, "cache")
    assert_f32_equal(to_np(kv.scale_inv), rs, "scale_cache")
    S_out = S_out if S_out is not None else max(lens) + 3
    lens_t = torch.tensor(lens, dtype=torch.int32)
    out = kv.gather(table.cuda(), lens_t.cuda(), S_out)
    ref = orc.paged_kv_gather(rc, rs, table.numpy(), lens_t.numpy(), S_out, fmt)
    got = inputs.bf16_bits(out)
    nan = (ref & 0x7FFF) > 0x7F80
    assert np.array_equal(nan, (got & 0x7FFF) > 0x7F80)
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("H,Dh", [(3, 32), (2, 80), (8, 128), (1, 256), (4, 512), (2, 8), (64, 128)])
def test_paged_write_gather_small(orc, fmt, H, Dh):
    _case(orc, fmt, H, Dh, [37, 5, 0, 16, 1], bs=16, NB=10, seed=H * 1000 + Dh, specials=True)


@pytest.mark.parametrize("bs", [1, 7, 32])
def test_paged_block_sizes_and_short_output(orc, bs):
    lens = [50, 3, 64]
    NB = sum((n + bs - 1) // bs for n in lens) + 2
    _case(orc, 0, 4, 64, lens, bs=bs, NB=NB, seed=bs)
    _case(orc, 0, 4, 64, lens, bs=bs, NB=NB, seed=bs + 1, S_out=20)   # output shorter than the sequences


def test_paged_decode_step(orc):
    """One new token per sequence (a decode step) appended after a prefill."""
    H, Dh, bs = 8, 128, 16
    lens = [100, 31, 64, 1]
    NB = 40
    table, slots = inputs.paged_layout([n + 1 for n in lens], bs, NB, seed=9)
    kv = fp8q.PagedKVCache(NB, bs, H, Dh, 0)
    rc = np.zeros((NB, bs, H, Dh), np.uint8)
    rs = np.zeros((NB, bs, H), np.float32)
    x = inputs.normal_bf16((slots.numel(), H, Dh), 1.0, seed=10)
    starts = np.cumsum([0] + [n + 1 for n in lens])
    prefill = np.concatenate([np.arange(starts[b], starts[b] + lens[b]) for b in range(len(lens))])
    decode = starts[1:] - 1
    for idx in (prefill, decode):
        idx_t = torch.from_numpy(idx)
        kv.write(x[idx_t].cuda(), slots[idx_t].cuda())
        rc, rs = orc.paged_kv_write(inputs.bf16_bits(x[idx_t]), slots[idx_t].numpy(), rc, rs, 0)
    assert_codes_equal(to_np(kv.cache), rc, 0, "cache")
    assert_f32_equal(to_np(kv.scale_inv), rs, "scale_cache")
    lens1 = torch.tensor([n + 1 for n in lens], dtype=torch.int32)
    out = kv.gather(table.cuda(), lens1.cuda(), 101)
    ref = orc.paged_kv_gather(rc, rs, table.numpy(), lens1.numpy(), 101, 0)
    assert np.array_equal(inputs.bf16_bits(out), ref)


def test_paged_full_size_sampled(orc):
    """K of 32 sequences x 8192 tokens, 32 heads x 128, 16-token pages on a
    shuffled table (the size the bench times): the whole cache is written in
    one launch and gathered in one launch; 64 sampled tokens are checked
    against the oracle run on their inputs alone (codes and scales at their
    slots, and the gathered rows)."""
    P = inputs.PAGED_KV
    B, S, H, Dh, bs = P["B"], P["S"], P["H"], P["Dh"], P["block_size"]
    NB = B * S // bs
    table, slots = inputs.paged_layout([S] * B, bs, NB, seed=21)
    x = inputs.normal_bf16((B * S, H, Dh), 1.0, seed=22, device="cuda")
    kv = fp8q.PagedKVCache(NB, bs, H, Dh, 0)
    kv.write(x, slots.cuda())
    lens = torch.full((B,), S, dtype=torch.int32)
    out = kv.gather(table.cuda(), lens.cuda(), S)
    rng = np.random.default_rng(0)
    pick = np.concatenate([[0, B * S - 1, S - 1, S], rng.integers(0, B * S, 60)])
    n = len(pick)
    xs = inputs.bf16_bits(x[torch.from_numpy(pick).cuda()])
    # the oracle writes the picked tokens into a fresh n-slot cache ...
    rc, rs = orc.paged_kv_write(xs, np.arange(n, dtype=np.int64), np.zeros((n, 1, H, Dh), np.uint8),
                                np.zeros((n, 1, H), np.float32), 0)
    sl = torch.from_numpy(slots.numpy()[pick]).cuda()
    assert_codes_equal(to_np(kv.cache.view(NB * bs, H, Dh)[sl]), rc[:, 0], 0, "cache")
    assert_f32_equal(to_np(kv.scale_inv.view(NB * bs, H)[sl]), rs[:, 0], "scales")
    # ... and reads them back as one sequence of n one-token pages
    ref = orc.paged_kv_gather(rc, rs, np.arange(n, dtype=np.int32)[None], np.array([n], np.int32), n, 0)[0]
    b, t = torch.from_numpy(pick // S).cuda(), torch.from_numpy(pick % S).cuda()
    assert np.array_equal(inputs.bf16_bits(out[b, t]), ref)
