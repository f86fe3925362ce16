"""GPU parity of the block-scaled GEMM that requantizes its own output
(fp8_gemm_block_requant): the MLP chain H = bf16(up(X)), quantized with
1 x 128 blocks for the down projection, in one launch.

The expected codes, scales and counts come from the oracle's chain on
oracle-side data only: integer FP8 codes with power-of-two scales make the
GEMM exact (the same construction as tests/test_gpu_gemm_exact.py), so the
oracle's exact product rounded to bf16 IS the GEMM output, and the oracle's
1 x 128 quantizer applied to it gives the codes the fused epilogue must
produce bit for bit.

Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-block scales
on every GEMM operand), §5.1 (overflow and NaN are what a run must catch).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q
from tests.gpu_util import assert_codes_equal, assert_f32_equal, need_gpu, to_np
from tests.test_gpu_gemm_exact import _cuda, _exact_bf16, _operands, _rows_touching_every_tile, _scale_maps

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _bits(d_bf16):
    return d_bf16.contiguous().view(torch.int16).numpy().view(np.uint16)


def _requant(A, B, da, db, fo, store_d):
    c = torch.zeros(2, dtype=torch.int32, device="cuda")
    q, qs, D = fp8q.gemm_block_requant(_cuda(A), 0, _cuda(B), 0, _cuda(da), _cuda(db), fo, store_d=store_d, counts=c)
    return q, qs, D, (int(c[0]), int(c[1]))


@pytest.mark.parametrize("fo", [0, 1])
@pytest.mark.parametrize("shape", [(300, 272, 400), (520, 784, 640), (1024, 1040, 896), (64, 272, 256),
                                   (129, 272, 144), (300, 272, 48)])
def test_requant_equals_the_oracle_chain(orc, fo, shape):
    """Fused GEMM + 1x128 requantization against the oracle's exact GEMM
    rounded to bf16 and quantized by the oracle: codes, scales, counts and
    the stored bf16 output bit for bit; ragged M, N and K, both output
    formats; M = 64 takes the two-launch path (GEMM, then the quantizer)."""
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=M + N + K + 3 * fo)
    SA, SB = _scale_maps(2, M, N, K, da, db)
    ref = _exact_bf16(va, vb, SA, SB)
    rq, rs, rc = orc.quantize_blockwise(_bits(ref), fo, 1, counts=True)
    q, qs, D, c = _requant(A, B, da, db, fo, store_d=True)
    assert torch.equal(D.cpu(), ref)
    assert_codes_equal(to_np(q), rq, fo)
    assert_f32_equal(to_np(qs), rs)
    assert c == rc
    if M > 128:   # the fused path without the bf16 store gives the same codes
        q2, qs2, D2, c2 = _requant(A, B, da, db, fo, store_d=False)
        assert D2 is None
        assert torch.equal(q2, q) and torch.equal(qs2, qs) and c2 == c


def test_requant_nan_columns_are_counted_and_excluded(orc):
    """A NaN code in a row of B makes that output column NaN: every row's
    block holding it takes its amax over the other 127 values, casts the NaN
    to a NaN code and counts one non-finite element (as the 1x128 quantizer
    does on the same bf16 values)."""
    M, N, K = 384, 528, 512
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=11)
    nan_cols = [5, 300, 527]
    B = B.copy()
    for n in nan_cols:
        B[n, 17] = 0x7F   # E4M3 NaN
    SA, SB = _scale_maps(2, M, N, K, da, db)
    vbf = vb.astype(np.float64)
    for n in nan_cols:
        vbf[n, 17] = np.nan
    exact = (va.astype(np.float64) * SA) @ (vbf * SB).T
    ref = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16)
    rq, rs, rc = orc.quantize_blockwise(_bits(ref), 0, 1, counts=True)
    assert rc[0] == M * len(nan_cols)
    q, qs, D, c = _requant(A, B, da, db, 0, store_d=True)
    got = D.cpu().float().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref.float().numpy()))
    assert np.array_equal(got[~np.isnan(got)], ref.float().numpy()[~np.isnan(got)])
    assert_codes_equal(to_np(q), rq, 0)
    assert_f32_equal(to_np(qs), rs)
    assert c == rc


@pytest.mark.parametrize("fo", [0])
def test_requant_mlp_up_full_size(orc, fo):
    """The MLP's up projection [8192, 4096] x W_up[11008, 4096]^T with its
    output requantized for the down projection (86 blocks per row, the last
    one 128 wide as 11008 = 86 x 128): rows touching every row tile, every
    column, against the oracle chain."""
    M, N, K = 8192, 11008, 4096
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=21, vmax=8)
    SA, SB = _scale_maps(2, M, N, K, da, db)
    rows = _rows_touching_every_tile(M, n=256, seed=2)
    ref = _exact_bf16(va, vb, SA, SB, rows)
    rq, rs, rc = orc.quantize_blockwise(_bits(ref), fo, 1, counts=True)
    q, qs, D, _ = _requant(A, B, da, db, fo, store_d=False)
    r = torch.from_numpy(rows)
    assert_codes_equal(to_np(q.cpu()[r]), rq, fo)
    assert_f32_equal(to_np(qs.cpu()[:, r]), rs)


def test_requant_needs_d_where_it_does_not_fuse():
    """M <= 128 runs the GEMM into D, then the quantizer: D is required."""
    M, N, K = 64, 256, 256
    _, A, da, _, B, db = _operands(M, N, K, 2, seed=5)
    q = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    qs = torch.empty((2, M), dtype=torch.float32, device="cuda")
    with pytest.raises(fp8q.Fp8Error):
        fp8q.fp8_gemm_block_requant(_cuda(A), 0, _cuda(B), 0, M, N, K, _cuda(da), _cuda(db), None, N, 0, q, qs)


@pytest.mark.parametrize("fo", [0, 1])
@pytest.mark.parametrize("shape", [(300, 272, 400), (520, 784, 640), (64, 272, 256), (1024, 1040, 896),
                                   (129, 272, 144)])
def test_e8m0_requant_equals_the_oracle_chain(orc, fo, shape):
    """The E8M0 GEMM (power-of-two block scales in the MMA) with its output
    requantized 1x128 with power-of-two scales into the next GEMM's E8M0
    image, against the oracle's exact GEMM -> bf16 -> power-of-two 1x128
    quantizer: codes, every image byte the quantizer defines (rows past M in
    the last 128-row group hold e = 127), counts and the bf16 output."""
    from tests.test_gpu_block_e8m0 import _image, _written
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=M + 7 * N + K + fo)
    img_a, img_b = _image(da, M, K, 1), _image(db, N, K, 128)
    SA, SB = _scale_maps(2, M, N, K, da, db)
    ref = _exact_bf16(va, vb, SA, SB)
    rq, rs, rc = orc.quantize_blockwise(_bits(ref), fo, 1, pow2=True, counts=True)
    want, mask = _image(rs, M, N, 1), _written(M, N)
    for store_d in (True, False):
        c = torch.zeros(2, dtype=torch.int32, device="cuda")
        q, qsf, D = fp8q.gemm_block_e8m0_requant(_cuda(A), 0, _cuda(B), 0, _cuda(img_a), _cuda(img_b), fo,
                                                 store_d=store_d, counts=c)
        if store_d:
            assert torch.equal(D.cpu(), ref)
        assert_codes_equal(to_np(q), rq, fo)
        got = to_np(qsf)
        assert np.array_equal(got[mask], want[mask]), f"{int((got[mask] != want[mask]).sum())} image bytes differ"
        assert (int(c[0]), int(c[1])) == rc


def test_block_mlp_step_replays_in_a_cuda_graph():
    """The block-scaled MLP step -- X quantized 1x128, W_up and W_down
    128x128, the up GEMM requantizing H in its epilogue, the down GEMM --
    captured once in a CUDA graph (its launches use programmatic dependent
    launch and thread-block clusters) and replayed with new inputs copied
    into the captured buffers: every replay equals the eager step on the same
    inputs, bit for bit."""
    from fp8_scaled_quantization_amax_b200 import inputs
    M, Dm, F = 512, 1024, 2816
    X_ = torch.empty((M, Dm), dtype=torch.bfloat16, device="cuda")
    Wu_ = torch.empty((F, Dm), dtype=torch.bfloat16, device="cuda")
    Wd_ = torch.empty((Dm, F), dtype=torch.bfloat16, device="cuda")

    def step(X, Wu, Wd):
        qx, sx = fp8q.quantize_blockwise(X, 0, 1)
        qwu, swu = fp8q.quantize_blockwise(Wu, 0, 128)
        qh, sh, _ = fp8q.gemm_block_requant(qx, 0, qwu, 0, sx, swu, 0)
        qwd, swd = fp8q.quantize_blockwise(Wd, 0, 128)
        return fp8q.gemm(qh, 0, qwd, 0, fp8q.SCALE_BLOCK, sh, swd)

    sets = [(inputs.normal_bf16((M, Dm), 1.0, seed=40 + i, device="cuda"),
             inputs.normal_bf16((F, Dm), 0.02, seed=50 + i, device="cuda"),
             inputs.normal_bf16((Dm, F), 0.02, seed=60 + i, device="cuda")) for i in range(3)]
    for t, v in zip((X_, Wu_, Wd_), sets[0]):
        t.copy_(v)
    step(X_, Wu_, Wd_)   # warm-up outside the capture (per-device set-up of every kernel)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            Y_ = step(X_, Wu_, Wd_)
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(6):
        X, Wu, Wd = sets[rep % 3]
        X_.copy_(X); Wu_.copy_(Wu); Wd_.copy_(Wd)
        g.replay()
        torch.cuda.synchronize()
        ref = step(X, Wu, Wd)
        torch.cuda.synchronize()
        assert torch.equal(Y_, ref), rep
