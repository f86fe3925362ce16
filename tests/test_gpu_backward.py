"""GPU parity of the backward-pass pieces of the rowwise recipes against the
CPU oracle: rowwise quantization of transposed operands (bit-exact) and the
weight-gradient GEMM kept in high precision (rowwise_with_gw_hp).

Source: "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
"FP8 三种缩放配方怎么选" (tensorwise / rowwise / rowwise_with_gw_hp: rowwise
scales, and the weight gradient kept in high precision in the last one);
"DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.1 (E5M2 gradients).

Tolerance of the bf16 GEMM: exact bf16 products summed in fp32, so within
T * 2^-22 of sum_t |dY x| (twice the worst-case bound of a T-term fp32 sum).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_codes_equal, assert_f32_equal, assert_gemm_close, bf16_to_f64, need_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("pow2", [True, False])
@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (1040, 272), (512, 4096)])
def test_rowwise_transpose_matches_oracle(orc, fmt, pow2, shape):
    rows, cols = shape
    x = (inputs.lognormal_grads_bf16((rows, cols), seed=rows + cols) if fmt == 1
         else inputs.outlier_activations_bf16((rows, cols), seed=rows + cols, frac=0.01))
    bits = inputs.bf16_bits(x).copy()
    bits[rows // 2, 3] = 0x7F80        # +Inf: skipped by the amax, saturates in the cast
    bits[1, cols - 1] = 0xFFC0         # NaN
    bits[:, 5] = 0                     # an all-zero column
    qT, sinv, am = fp8q.quantize_rowwise_transpose(inputs.from_bf16_bits(bits, "cuda"), fmt, pow2)
    rq, rs = orc.quantize_rowwise_transpose(bits, fmt, pow2)
    assert_codes_equal(to_np(qT), rq, fmt)
    assert_f32_equal(to_np(sinv), rs)
    xf = bf16_to_f64(inputs.from_bf16_bits(bits))
    ref_am = np.where(np.isfinite(xf), np.abs(xf), 0).max(axis=0).astype(np.float32)
    assert_f32_equal(to_np(am), ref_am, "column amax")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(16384, 2112), (2064, 16400), (16400, 48)])
def test_rowwise_transpose_schedules_strided(orc, fmt, shape):
    """Both schedules of the transposed per-row quantizer against the oracle
    ("FP8训练与QAT…Soup", section "FP8 三种缩放配方怎么选": rowwise scales of
    the backward GEMMs' K-major operands): the single-pass strip kernel with
    clusters that each take several strips (16384 rows: the strips in flight
    are capped by L2; 16400 columns: more strips than clusters, a ragged last
    strip and ranks with no rows) and the two-pass path for columns longer
    than 16384 rows, on a strided input whose padding columns hold +Inf and
    NaN, with the non-finite and saturation counts."""
    rows, cols = shape
    pad = 24
    wide = inputs.bf16_bits(inputs.outlier_activations_bf16((rows, cols + pad), seed=rows + fmt, frac=0.01)).copy()
    wide[:, cols::2] = 0x7F80
    wide[:, cols + 1::2] = 0x7FC0
    wide[rows // 3, 7] = 0xFF80        # -Inf in the data
    wide[rows - 1, cols - 16] = 0x7FC1  # NaN in the last row
    bits = np.ascontiguousarray(wide[:, :cols])
    x = inputs.from_bf16_bits(wide, "cuda")   # [rows, cols + pad]; the quantizer reads cols of each row
    for pow2 in (True, False):
        c = torch.zeros(2, dtype=torch.int32, device="cuda")
        qT = torch.empty((cols, rows), dtype=torch.uint8, device="cuda")
        sinv = torch.empty(cols, dtype=torch.float32, device="cuda")
        am = torch.empty(cols, dtype=torch.float32, device="cuda")
        fp8q.fp8_quantize_rowwise_transpose(x, rows, cols, cols + pad, fmt, pow2, qT, sinv, am, counts=c)
        rq, rs, rc = orc.quantize_rowwise_transpose(bits, fmt, pow2, counts=True)
        assert_codes_equal(to_np(qT), rq, fmt)
        assert_f32_equal(to_np(sinv), rs)
        assert (int(c[0]), int(c[1])) == rc
        xf = bf16_to_f64(inputs.from_bf16_bits(bits))
        ref_am = np.where(np.isfinite(xf), np.abs(xf), 0).max(axis=0).astype(np.float32)
        assert_f32_equal(to_np(am), ref_am, "column amax")


def _tol_check(got, ref, mag, T, what):
    err = np.abs(got - ref)
    bound = T * 2.0 ** -22 * mag + 1e-30
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs off, worst {float((err / bound).max()):.3g} x bound"


@pytest.mark.parametrize("shape", [(64, 256, 256), (100, 64, 40), (1, 8, 8), (640, 520, 776), (4096, 512, 1024)])
def test_bf16_wgrad_full_compare(orc, shape):
    T, M, N = shape
    dy = inputs.lognormal_grads_bf16((T, M), seed=T + M)
    x = inputs.normal_bf16((T, N), 1.0, seed=T + N)
    dW = fp8q.gemm_bf16_wgrad(dy.cuda(), x.cuda())
    ref, mag = orc.gemm_bf16_wgrad(inputs.bf16_bits(dy), inputs.bf16_bits(x))
    _tol_check(to_np(dW).astype(np.float64), ref, mag, T, "dW")
    # deterministic, and accumulate adds to what is there
    again = fp8q.gemm_bf16_wgrad(dy.cuda(), x.cuda())
    assert torch.equal(dW, again)
    acc = dW.clone()
    fp8q.gemm_bf16_wgrad(dy.cuda(), x.cuda(), out=acc, accumulate=True)
    assert torch.equal(acc, dW + again)


def test_bf16_wgrad_full_size_sampled(orc):
    """dW [4096, 4096] over 8192 tokens (the dgrad workload's layer),
    2048 sampled outputs."""
    T, M, N = 8192, 4096, 4096
    dy = inputs.lognormal_grads_bf16((T, M), seed=90, device="cuda")
    x = inputs.normal_bf16((T, N), 1.0, seed=91, device="cuda")
    dW = fp8q.gemm_bf16_wgrad(dy, x)
    rng = np.random.default_rng(1)
    im = np.concatenate([[0, M - 1, 255, 256], rng.integers(0, M, 2044)])
    inn = np.concatenate([[0, N - 1, 255, 256], rng.integers(0, N, 2044)])
    ref, mag = orc.gemm_bf16_wgrad_sampled(inputs.bf16_bits(dy), inputs.bf16_bits(x), im, inn)
    got = to_np(dW[_cuda(im), _cuda(inn)]).astype(np.float64)
    _tol_check(got, ref, mag, T, "dW sampled")


def test_linear_backward_rowwise_recipes(orc):
    """A linear layer's backward under the rowwise recipes, every GEMM through
    the library: dX = dY W with rowwise FP8 scales (dY E5M2 per token, W^T E4M3
    per input channel), dW in FP8 (rowwise: dY^T and X^T quantized per row of
    the transpose) and in bf16 (rowwise_with_gw_hp); each against the oracle
    running the same recipe."""
    T, Nin, Nout = 512, 384, 256
    x = inputs.normal_bf16((T, Nin), 1.0, seed=80)
    w = inputs.normal_bf16((Nout, Nin), 0.02, seed=81)
    dy = inputs.lognormal_grads_bf16((T, Nout), seed=82)
    xb, wb, dyb = (inputs.bf16_bits(t) for t in (x, w, dy))
    # dgrad: A = dY [T, Nout] (K = Nout), B = W^T [Nin, Nout]
    qdy, sdy = fp8q.quantize_rowwise(dy.cuda(), 1, True)
    qwT, swT, _ = fp8q.quantize_rowwise_transpose(w.cuda(), 0, True)
    dX = fp8q.gemm(qdy, 1, qwT, 0, fp8q.SCALE_ROW, sdy, swT)
    rqdy, rsdy = orc.quantize_rowwise(dyb, 1, True)
    rqwT, rswT = orc.quantize_rowwise_transpose(wb, 0, True)
    assert_codes_equal(to_np(qwT), rqwT, 0, "W^T")
    ref, mag = orc.gemm_scaled(rqdy, 1, rqwT, 0, orc.SCALE_ROW, rsdy, rswT)
    assert_gemm_close(bf16_to_f64(dX), ref, mag, "dX")
    # wgrad in FP8: A = dY^T [Nout, T], B = X^T [Nin, T] (K = tokens)
    qdyT, sdyT, _ = fp8q.quantize_rowwise_transpose(dy.cuda(), 1, True)
    qxT, sxT, _ = fp8q.quantize_rowwise_transpose(x.cuda(), 0, True)
    dW8 = fp8q.gemm(qdyT, 1, qxT, 0, fp8q.SCALE_ROW, sdyT, sxT)
    rqdyT, rsdyT = orc.quantize_rowwise_transpose(dyb, 1, True)
    rqxT, rsxT = orc.quantize_rowwise_transpose(xb, 0, True)
    ref8, mag8 = orc.gemm_scaled(rqdyT, 1, rqxT, 0, orc.SCALE_ROW, rsdyT, rsxT)
    assert_gemm_close(bf16_to_f64(dW8), ref8, mag8, "dW fp8")
    # wgrad in bf16 (rowwise_with_gw_hp)
    dWh = fp8q.gemm_bf16_wgrad(dy.cuda(), x.cuda())
    refh, magh = orc.gemm_bf16_wgrad(dyb, xb)
    _tol_check(to_np(dWh).astype(np.float64), refh, magh, T, "dW bf16")
    # the high-precision weight gradient is the more accurate one
    e8 = np.abs(bf16_to_f64(dW8) - refh).mean()
    eh = np.abs(to_np(dWh).astype(np.float64) - refh).mean()
    assert eh < e8
