"""GPU parity of the power-of-two block scales applied by the tensor core
(E8M0 scale images + tcgen05.mma.kind::mxf8f6f4.block_scale) against the CPU
oracle.

Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-block
scales: 1x128 activation blocks, 128x128 weight blocks);
"FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section "FP8 三种缩放
配方怎么选" (power-of-two scales).  With power-of-two scales the block-scaled
GEMM is the oracle's per-block GEMM exactly (scaling by 2^e is exact), so the
oracle is its BLOCK mode fed with the oracle's own power-of-two scales; the
scale images fed to the GPU GEMM are written here from those scales with the
layout the C header states.
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_codes_equal, assert_gemm_close, bf16_to_f64, need_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _e8m0(d):
    """Biased exponent of a power-of-two factor d (fp32), from frexp."""
    f, e = np.frexp(np.asarray(d, np.float64))
    assert np.all(f == 0.5), "factor is not a power of two"
    return (e - 1 + 127).astype(np.int64)


def _image(scale_inv, rows, cols, block_rows, fill=127):
    """E8M0 image (header layout) from the oracle's fp32 power-of-two factors;
    bytes of K blocks past the last one hold `fill`."""
    nkb, rt = (cols + 127) // 128, (rows + 127) // 128
    img = np.full(((nkb + 3) // 4) * rt * 512, fill, np.uint8)
    r = np.arange(rt * 128)
    for kb in range(nkb):
        if block_rows == 1:
            e = np.full(rt * 128, 127)
            e[:rows] = _e8m0(scale_inv[kb, :rows])
        else:
            e = _e8m0(scale_inv[r // 128, kb])
        img[((kb // 4) * rt + r // 128) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4] = e
    return img


def _written(rows, cols):
    """Mask of the image bytes the quantizer defines."""
    nkb, rt = (cols + 127) // 128, (rows + 127) // 128
    m = np.zeros(((nkb + 3) // 4) * rt * 512, bool)
    r = np.arange(rt * 128)
    for kb in range(nkb):
        m[((kb // 4) * rt + r // 128) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4] = True
    return m


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("block_rows", [1, 128])
@pytest.mark.parametrize("shape", [(128, 128), (300, 400), (1, 16), (257, 1040)])
def test_quantize_e8m0_matches_oracle(orc, fmt, block_rows, shape):
    rows, cols = shape
    x = inputs.outlier_activations_bf16((rows, cols), seed=rows + cols)
    bits = inputs.bf16_bits(x)
    q, img = fp8q.quantize_blockwise_e8m0(x.cuda(), fmt, block_rows)
    rq, rs = orc.quantize_blockwise(bits, fmt, block_rows, pow2=True)
    assert_codes_equal(to_np(q), rq, fmt)
    w = _written(rows, cols)
    assert np.array_equal(to_np(img)[w], _image(rs, rows, cols, block_rows)[w])


def _operands(orc, M, N, K, fa=0, fb=0, seed=0):
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((M, K), seed=seed))
    b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=seed + 1))
    A, da = orc.quantize_blockwise(a, fa, 1, pow2=True)
    B, db = orc.quantize_blockwise(b, fb, 128, pow2=True)
    return A, da, B, db


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


@pytest.mark.parametrize("fa,fb", [(0, 0), (1, 0)])
@pytest.mark.parametrize("shape", [(256, 256, 256), (300, 272, 400), (64, 520, 1024), (1, 8, 16),
                                   (520, 776, 640), (1024, 768, 2048)])
def test_gemm_e8m0_full_compare(orc, fa, fb, shape):
    M, N, K = shape
    A, da, B, db = _operands(orc, M, N, K, fa, fb, seed=M + N + K)
    D = fp8q.gemm_block_e8m0(_cuda(A), fa, _cuda(B), fb, _cuda(_image(da, M, K, 1)), _cuda(_image(db, N, K, 128)))
    ref, mag = orc.gemm_scaled(A, fa, B, fb, orc.SCALE_BLOCK, da, db)
    assert_gemm_close(bf16_to_f64(D), ref, mag, "e8m0 gemm")
    # deterministic: repeated calls are bit-identical
    D2 = fp8q.gemm_block_e8m0(_cuda(A), fa, _cuda(B), fb, _cuda(_image(da, M, K, 1)), _cuda(_image(db, N, K, 128)))
    assert torch.equal(D, D2)


def test_gemm_e8m0_end_to_end_gpu_quantizer(orc):
    """GPU quantizer -> GPU GEMM against oracle quantizer -> oracle GEMM."""
    M, N, K = 768, 1280, 1152
    x = inputs.outlier_activations_bf16((M, K), seed=7)
    w = inputs.normal_bf16((N, K), 0.02, seed=8)
    qa, ia = fp8q.quantize_blockwise_e8m0(x.cuda(), 0, 1)
    qb, ib = fp8q.quantize_blockwise_e8m0(w.cuda(), 0, 128)
    D = fp8q.gemm_block_e8m0(qa, 0, qb, 0, ia, ib)
    A, da = orc.quantize_blockwise(inputs.bf16_bits(x), 0, 1, pow2=True)
    B, db = orc.quantize_blockwise(inputs.bf16_bits(w), 0, 128, pow2=True)
    ref, mag = orc.gemm_scaled(A, 0, B, 0, orc.SCALE_BLOCK, da, db)
    assert_gemm_close(bf16_to_f64(D), ref, mag, "e2e e8m0")


def test_gemm_e8m0_mlp_up_sampled(orc):
    """[8192, 4096] x W_up[11008, 4096]^T, the block MLP's up projection:
    2048 sampled outputs against the oracle."""
    M, N, K = 8192, 11008, 4096
    x = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=5, device="cuda"))
    w = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=6, device="cuda"))
    A, da = orc.quantize_blockwise(x, 0, 1, pow2=True)
    B, db = orc.quantize_blockwise(w, 0, 128, pow2=True)
    D = fp8q.gemm_block_e8m0(_cuda(A), 0, _cuda(B), 0, _cuda(_image(da, M, K, 1)), _cuda(_image(db, N, K, 128)))
    rng = np.random.default_rng(0)
    im = np.concatenate([[0, M - 1, 255, 256], rng.integers(0, M, 2044)])
    inn = np.concatenate([[0, N - 1, 255, 256], rng.integers(0, N, 2044)])
    ref, mag = orc.gemm_scaled_sampled(A, 0, B, 0, orc.SCALE_BLOCK, da, db, im, inn)
    got = bf16_to_f64(D[_cuda(im), _cuda(inn)])
    assert_gemm_close(got, ref, mag, "e8m0 mlp up sampled")


def test_gemm_e8m0_mlp_down_sampled(orc):
    """[8192, 11008] x W_down[4096, 11008]^T, the block MLP's down projection
    (the input a seeded bf16 tensor of the up projection's output shape):
    2048 sampled outputs against the oracle."""
    M, N, K = 8192, 4096, 11008
    h = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=15, device="cuda"))
    w = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=16, device="cuda"))
    A, da = orc.quantize_blockwise(h, 0, 1, pow2=True)
    B, db = orc.quantize_blockwise(w, 0, 128, pow2=True)
    D = fp8q.gemm_block_e8m0(_cuda(A), 0, _cuda(B), 0, _cuda(_image(da, M, K, 1)), _cuda(_image(db, N, K, 128)))
    rng = np.random.default_rng(2)
    im = np.concatenate([[0, M - 1, 255, 256], rng.integers(0, M, 2044)])
    inn = np.concatenate([[0, N - 1, 255, 256], rng.integers(0, N, 2044)])
    ref, mag = orc.gemm_scaled_sampled(A, 0, B, 0, orc.SCALE_BLOCK, da, db, im, inn)
    got = bf16_to_f64(D[_cuda(im), _cuda(inn)])
    assert_gemm_close(got, ref, mag, "e8m0 mlp down sampled")


def test_e8m0_accuracy_against_fp32_block_scales(orc):
    """What power-of-two block scales cost in accuracy on the block MLP's up
    projection ([8192, 4096] x W_up[11008, 4096]^T): both recipes' GPU
    outputs on 64 sampled rows x every column, against the unquantized
    product of the same bf16 inputs (fp64).  Power-of-two factors are up to
    2x coarser than fp32 block scales (the codes use as little as half the
    range below fmax, so values near the underflow end lose bits), but FP8's
    relative precision does not depend on the scale elsewhere, so the two
    errors must stay within a factor of two of each other.  FP8_ACCURACY_LOG, when set,
    names a file that receives the two relative errors."""
    import json
    import os
    M, N, K = 8192, 11008, 4096
    x = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=5, device="cuda"))
    w = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=6, device="cuda"))
    rows = np.sort(np.random.default_rng(3).choice(M, 64, replace=False))
    truth = bf16_to_f64(inputs.from_bf16_bits(x[rows])) @ bf16_to_f64(inputs.from_bf16_bits(w)).T
    err = {}
    for name, pow2 in (("fp32 block scales", False), ("E8M0 block scales", True)):
        A, da = orc.quantize_blockwise(x, 0, 1, pow2=pow2)
        B, db = orc.quantize_blockwise(w, 0, 128, pow2=pow2)
        if pow2:
            D = fp8q.gemm_block_e8m0(_cuda(A), 0, _cuda(B), 0, _cuda(_image(da, M, K, 1)),
                                     _cuda(_image(db, N, K, 128)))
        else:
            D = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, 2, _cuda(da), _cuda(db))
        got = bf16_to_f64(D[_cuda(rows)])
        err[name] = float(np.linalg.norm(got - truth) / np.linalg.norm(truth))
    e32, e8 = err["fp32 block scales"], err["E8M0 block scales"]
    if os.environ.get("FP8_ACCURACY_LOG"):
        with open(os.environ["FP8_ACCURACY_LOG"], "a") as f:
            f.write(json.dumps({"shape": [M, N, K], "rows": 64, "relative_rms_error": err}) + "\n")
    assert 0 < e32 < 0.1, err          # E4M3 keeps ~3 significand bits: a few % of the output norm
    assert 0.5 * e32 <= e8 <= 2.0 * e32, err   # relative FP8 precision does not depend on the scale, except near underflow
