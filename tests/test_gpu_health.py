"""GPU parity of the scale health check against the CPU oracle.

Source: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §6.2 (min / max /
mean of each layer's scales at intervals; a step change flags an outlier or a
distribution drift).  min, max and both counts are compared bit for bit; the
mean (an fp64 sum whose order differs from the oracle's, rounded to fp32) to
one fp32 ulp.
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import need_gpu, to_np

pytestmark = pytest.mark.gpu


def _check(orc, s, prev, offs, r, stats, counts):
    st, ct = to_np(stats), to_np(counts).view(np.uint32)
    for g in range(len(offs) - 1):
        lo, hi = offs[g], offs[g + 1]
        rs, rc = orc.scale_stats(s[lo:hi], None if prev is None else prev[lo:hi], r)
        assert st[g, 0].view(np.uint32) == rs[0].view(np.uint32), (g, st[g], rs)
        assert st[g, 1].view(np.uint32) == rs[1].view(np.uint32), (g, st[g], rs)
        assert abs(float(st[g, 2]) - float(rs[2])) <= float(np.spacing(np.float32(rs[2]))), (g, st[g], rs)
        assert list(ct[g]) == list(rc), (g, ct[g], rc)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("n", [0, 1, 7, 2048, 2049, 100003])
def test_single_segment_with_invalid_entries(orc, n):
    prev, cur = inputs.scale_snapshots_f32(n, seed=n, jump_frac=0.01)
    c = cur.numpy().copy()
    if n >= 7:
        c[[0, 3, 6]] = [np.nan, -2.0, np.inf]
        c[n // 2] = 0.0
    s = torch.from_numpy(c).cuda()
    p = prev.cuda()
    stats, counts = fp8q.scale_stats(s, prev=p, jump_ratio=4.0)
    _check(orc, c, prev.numpy(), [0, n], 4.0, stats, counts)
    stats, counts = fp8q.scale_stats(s)            # no previous snapshot
    _check(orc, c, None, [0, n], 4.0, stats, counts)


def test_segments_ragged_and_empty(orc):
    sizes = [1, 0, 4096, 8191, 3, 0, 70000, 129]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    prev, cur = inputs.scale_snapshots_f32(int(offs[-1]), seed=3, jump_frac=0.002)
    stats, counts = fp8q.scale_stats(cur.cuda(), torch.from_numpy(offs).cuda(), prev.cuda(), 8.0)
    _check(orc, cur.numpy(), prev.numpy(), offs, 8.0, stats, counts)


def test_full_size_every_layer(orc):
    """224 segments of 8192 scales (rowwise scales of every linear input of a
    32-layer model at 8192 tokens), the size the bench times."""
    L, n = inputs.SCALE_HEALTH["layers"], inputs.SCALE_HEALTH["per_layer"]
    offs = (np.arange(L + 1) * n).astype(np.int64)
    prev, cur = inputs.scale_snapshots_f32(L * n, seed=11)
    stats, counts = fp8q.scale_stats(cur.cuda(), torch.from_numpy(offs).cuda(), prev.cuda(), 4.0)
    _check(orc, cur.numpy(), prev.numpy(), offs, 4.0, stats, counts)
    assert int(to_np(counts)[:, 0].sum()) > 0       # the planted jumps are seen


def test_offsets_beyond_the_array_are_clamped(orc):
    prev, cur = inputs.scale_snapshots_f32(1000, seed=5)
    offs = torch.tensor([0, 600, 5000, 7000], dtype=torch.int64)
    stats, counts = fp8q.scale_stats(cur.cuda(), offs.cuda(), prev.cuda(), 4.0)
    _check(orc, cur.numpy(), prev.numpy(), [0, 600, 1000, 1000], 4.0, stats, counts)


@pytest.mark.parametrize("r", [4.0, 1.0, 3.3, 1.0000001, 16777215.0])
def test_step_change_decisions_at_the_threshold(orc, r):
    """Ratios placed on and next to the threshold (one fp32 step either way,
    both directions): the kernel's division-free test must take exactly the
    decisions of the oracle's rounded fp32 division."""
    rng = np.random.default_rng(int(r * 1000) % 2**31)
    p = (2.0 ** rng.uniform(-20, 20, 6000)).astype(np.float32)
    q = (p.astype(np.float64) * np.float64(np.float32(r))).astype(np.float32)
    v = np.concatenate([q, np.nextafter(q, np.float32(np.inf)), np.nextafter(q, np.float32(0)),
                        (p / np.float32(r)).astype(np.float32), np.nextafter(p / np.float32(r), np.float32(0))])
    prev = np.concatenate([p] * 5)
    ok = np.isfinite(v) & (v > 0)
    v, prev = v[ok], prev[ok]
    stats, counts = fp8q.scale_stats(torch.from_numpy(v).cuda(), prev=torch.from_numpy(prev).cuda(), jump_ratio=r)
    _check(orc, v, prev, [0, len(v)], r, stats, counts)
    assert 0 < int(to_np(counts)[0, 0]) < len(v)
