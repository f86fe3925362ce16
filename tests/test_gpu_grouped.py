"""GPU parity of the grouped (mixture-of-experts) FP8 GEMM with the oracle.

Source: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §3.2 (MoE inference
routes each token to a few experts; the per-expert matrix products become one
grouped GEMM over the token groups).  Operands come from the oracle's own
quantizer on seeded inputs; group sizes are ragged, with empty groups.
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_gemm_close, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def _grouped_operands(orc, mode, sizes, N, K, seed):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    G, M = len(sizes), int(off[-1])
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((max(M, 1), K), seed=seed))[:M]
    w = inputs.bf16_bits(inputs.normal_bf16((G * N, K), 0.02, seed=seed + 1)).reshape(G, N, K)
    if mode == orc.SCALE_TENSOR:
        A = np.empty((M, K), np.uint8)
        da = np.empty(G, np.float32)
        for e in range(G):
            r0, r1 = off[e], off[e + 1]
            if r1 > r0:
                q, s, _, _ = orc.quantize_tensorwise(np.ascontiguousarray(a[r0:r1]), 0)
                A[r0:r1], da[e] = q, s
            else:
                da[e] = 1.0
        B = np.empty((G, N, K), np.uint8)
        db = np.empty(G, np.float32)
        for e in range(G):
            B[e], db[e], _, _ = orc.quantize_tensorwise(np.ascontiguousarray(w[e]), 0)
    else:
        A, da = orc.quantize_rowwise(np.ascontiguousarray(a), 0, True)
        Bf, db = orc.quantize_rowwise(np.ascontiguousarray(w.reshape(G * N, K)), 0, True)
        B = Bf.reshape(G, N, K)
    return off, A, da, B, db


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("sizes,N,K", [([0, 37, 256, 300, 1], 264, 400), ([130], 512, 256),
                                       ([513, 0, 0, 255], 128, 128)])
def test_grouped_full_compare(orc, mode, sizes, N, K):
    off, A, da, B, db = _grouped_operands(orc, mode, sizes, N, K, seed=sum(sizes) + N)
    D = fp8q.gemm_grouped(_cuda(A), 0, _cuda(B), 0, _cuda(off), mode, _cuda(da), _cuda(db))
    ref, mag = orc.gemm_grouped(A, 0, B, 0, off, mode, da, db)
    assert_gemm_close(D.float().cpu().numpy().astype(np.float64), ref, mag)
    D2 = fp8q.gemm_grouped(_cuda(A), 0, _cuda(B), 0, _cuda(off), mode, _cuda(da), _cuda(db))
    assert torch.equal(D, D2)


def test_grouped_moe_sized_sampled(orc):
    """8 experts, ~8192 routed tokens with ragged counts, N = 1408, K = 2048."""
    rng = np.random.default_rng(5)
    sizes = list(rng.multinomial(8192, np.full(8, 1 / 8)))
    off, A, da, B, db = _grouped_operands(orc, 1, sizes, 1408, 2048, seed=77)
    D = fp8q.gemm_grouped(_cuda(A), 0, _cuda(B), 0, _cuda(off), 1, _cuda(da), _cuda(db))
    G, N, K = B.shape
    im = rng.integers(0, int(off[-1]), 1500)
    inn = rng.integers(0, N, 1500)
    e_of = np.searchsorted(off, im, side="right") - 1
    got = D.float().cpu().numpy().astype(np.float64)[im, inn]
    ref = np.empty(im.size)
    mag = np.empty(im.size)
    for e in range(G):
        sel = np.where(e_of == e)[0]
        if sel.size == 0:
            continue
        v, mg = orc.gemm_scaled_sampled(A, 0, B[e], 0, 1, da, db.reshape(G, N)[e], im[sel], inn[sel])
        ref[sel], mag[sel] = v, mg
    assert_gemm_close(got, ref, mag)


def test_grouped_rejects_block_mode():
    z = torch.zeros((256, 128), dtype=torch.uint8, device="cuda")
    off = torch.tensor([0, 256], dtype=torch.int64, device="cuda")
    s = torch.ones(256, device="cuda")
    D = torch.empty((256, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8q.Fp8Error, match="INVALID_ARG"):
        fp8q.fp8_gemm_grouped(z, 0, z[:128], 0, 1, off, 256, 128, 128, 2, s, s, D, 128)
