"""The GEMM entry point that allocates nothing (fp8_gemm_scaled_noalloc).

It exists for callers that cannot allocate device memory where they run the
GEMM -- code inside a framework whose caching allocator owns all device
memory, or latency-critical paths that cannot take cudaMalloc's implicit
device synchronisation.  Its split-K scratch is an array built into the
library instead of a caller workspace.

Checked through the C ABI on two calls in a row (the second reuses the
scratch the first left behind): against the CPU oracle on sampled outputs,
within the GEMM tolerance every other test uses, and against the existing
entry point (fp8_gemm_scaled with a caller workspace), bit for bit, since
both run the same split schedule and summation order.  The shapes that are
meant to use the scratch are asserted to need it; the others run without it.
The FP8 operands come from the CPU oracle's quantizer applied to seeded
inputs.

This file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_gemm_close, need_gpu

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 10 << 20


def _noalloc_via_c_abi(A, fa, B, fb, mode, da, db, D):
    L = fp8q.lib()
    fn = L.fp8_gemm_scaled_noalloc
    P = ctypes.c_void_p
    M, K = A.shape
    N = B.shape[0]
    st = fn(P(A.data_ptr()), fa, P(B.data_ptr()), fb, M, N, K, mode, P(da.data_ptr()), P(db.data_ptr()),
            P(D.data_ptr()), D.stride(0), P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.fp8_status_string(st)


# (shape, uses the scratch): the pair split (K >= 64 blocks, with few 256 x
# 256 tiles or a last wave of tiles at most half full) needs it; shorter K,
# cluster-split shapes and grids of whole waves do not.
_SHAPES = [((1000, 1288, 8208), True), ((1024, 1536, 16384), True), ((4096, 4096, 8192), True),
           ((4096, 4096, 4096), False),
           ((1024, 1024, 16384), False), ((300, 272, 400), False)]


@pytest.mark.parametrize("shape,uses_scratch", _SHAPES)
def test_noalloc_gemm_matches_oracle_and_workspace_entry_point(orc, shape, uses_scratch):
    need_gpu()
    M, N, K = shape
    need = fp8q.fp8_gemm_workspace_size(M, N, K, fp8q.SCALE_ROW)
    assert (need > 0) == uses_scratch, need
    assert need <= SCRATCH_BYTES
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((M, K), seed=M + K))
    b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=N + K))
    A, da = orc.quantize_rowwise(a, 0, True)
    B, db = orc.quantize_rowwise(b, 0, True)
    cuda = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda")
    A_, B_, da_, db_ = cuda(A), cuda(B), cuda(da), cuda(db)

    ws = fp8q.gemm_workspace(M, N, K, fp8q.SCALE_ROW)
    ref_gpu = fp8q.gemm(A_, 0, B_, 0, fp8q.SCALE_ROW, da_, db_, workspace=ws)

    rng = np.random.default_rng(M + N)
    im = rng.integers(0, M, 2048)
    inn = rng.integers(0, N, 2048)
    im[:4] = [0, M - 1, M - 1, 0]
    inn[:4] = [0, N - 1, 0, N - 1]
    ref, mag = orc.gemm_scaled_sampled(A, 0, B, 0, orc.SCALE_ROW, da, db, im, inn)

    for call in range(2):   # two calls in a row share the built-in scratch
        D = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        _noalloc_via_c_abi(A_, 0, B_, 0, fp8q.SCALE_ROW, da_, db_, D)
        torch.cuda.synchronize()
        got = D.float().cpu().numpy().astype(np.float64)[im, inn]
        assert_gemm_close(got, ref, mag, f"noalloc call {call} vs oracle")
        assert torch.equal(D, ref_gpu), f"call {call}: differs from the workspace entry point"
    assert fp8q.fp8_device_error(clear=True) == 0


def test_noalloc_largest_split_fits_the_scratch(orc):
    """The largest split this device can run (half of its CTA pairs' worth of
    256 x 256 tiles, all in one row of tiles) fits the built-in scratch, so
    the entry point never rejects a shape here; its output matches the
    oracle on sampled entries."""
    need_gpu()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = (sms // 2) // 2                     # r <= pairs / 2 split tiles
    M, N, K = 256, 256 * tiles, 8192
    need = fp8q.fp8_gemm_workspace_size(M, N, K, fp8q.SCALE_ROW)
    assert 0 < need <= SCRATCH_BYTES, need
    a = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=3))
    b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=4))
    A, da = orc.quantize_rowwise(a, 0, True)
    B, db = orc.quantize_rowwise(b, 0, True)
    cuda = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda")
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    _noalloc_via_c_abi(cuda(A), 0, cuda(B), 0, fp8q.SCALE_ROW, cuda(da), cuda(db), D)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    im, inn = rng.integers(0, M, 1024), rng.integers(0, N, 1024)
    ref, mag = orc.gemm_scaled_sampled(A, 0, B, 0, orc.SCALE_ROW, da, db, im, inn)
    assert_gemm_close(D.float().cpu().numpy().astype(np.float64)[im, inn], ref, mag, "largest split")
    assert fp8q.fp8_device_error(clear=True) == 0
