"""Multi-rank host logic on CPU (gloo, world size 2): the global-scale
exchange of per-tensor scaling ("DeepL押注FP8：…" §2.2, §5.1) and the
max-over-ranks timing reduction.  The arithmetic on each rank is the
oracle's (no GPU here); the exchange is the library's own code."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from fp8_scaled_quantization_amax_b200 import dist as fdist, inputs
        from oracle import oracle as orc
        # each rank holds a different shard; rank 1's has a larger outlier
        x = inputs.normal_bf16((64, 32), 1.0 + rank, seed=rank)
        bits = inputs.bf16_bits(x)
        local, _ = orc.amax(bits)
        a = torch.tensor([local], dtype=torch.float32)
        fdist.allreduce_amax_(a)
        s = orc.scale_from_amax(float(a[0]), 0)
        q, sinv, _, _ = orc.quantize_tensorwise(bits, 0, scale_in=s)
        t = fdist.max_over_ranks(10.0 * (rank + 1))
        results[rank] = (float(local), float(a[0]), s, q.tobytes(), t)
    finally:
        dist.destroy_process_group()


def test_global_amax_scale_shared_by_all_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()   # no fork of a process that may hold threads
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    r0, r1 = results[0], results[1]
    # both ranks see the max of the local amaxes and derive the same scale
    assert r0[1] == r1[1] == max(r0[0], r1[0])
    assert r0[2] == r1[2]
    # the shared scale equals the oracle's scale of the union of the shards
    from fp8_scaled_quantization_amax_b200 import inputs
    from oracle import oracle as orc
    union = np.concatenate([inputs.bf16_bits(inputs.normal_bf16((64, 32), 1.0 + r, seed=r)) for r in range(world)])
    ua, _ = orc.amax(union)
    assert r0[2] == orc.scale_from_amax(ua, 0)
    # max-over-ranks timing
    assert r0[4] == r1[4] == 20.0


def test_single_process_helpers_without_a_group():
    from fp8_scaled_quantization_amax_b200 import dist as fdist
    a = torch.tensor([3.0])
    assert fdist.allreduce_amax_(a) is a and float(a) == 3.0
    assert fdist.max_over_ranks(1.5) == 1.5
