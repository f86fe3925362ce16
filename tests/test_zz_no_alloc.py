"""The GEMM entry point that allocates nothing (fp8_gemm_scaled_noalloc).

It exists for callers that cannot allocate device memory where they run the
GEMM -- code inside a framework whose caching allocator owns all device
memory, or latency-critical paths that cannot take cudaMalloc's implicit
device synchronisation.  Its split-K scratch is an array built into the
library instead of a caller workspace.

Checked through the C ABI against the existing entry point (fp8_gemm_scaled
with a workspace) on two calls in a row: the outputs must agree within the
GEMM tolerance every other test uses (and, with the same split schedule and
summation order, bit for bit).  The FP8 operands come from the CPU oracle's
quantizer applied to seeded inputs.

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


def _noalloc_via_c_abi(A, fa, B, fb, mode, da, db, D):
    L = fp8q.lib()
    fn = L.fp8_gemm_scaled_noalloc
    P = ctypes.c_void_p
    M, K = A.shape
    N = B.shape[0]
    st = fn(P(A.data_ptr()), fa, P(B.data_ptr()), fb, M, N, K, mode, P(da.data_ptr()), P(db.data_ptr()),
            P(D.data_ptr()), D.stride(0), P(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.fp8_status_string(st)


@pytest.mark.parametrize("shape", [(1000, 1288, 8208), (1024, 1024, 16384), (300, 272, 400), (4096, 4096, 4096)])
def test_noalloc_gemm_matches_workspace_entry_point(orc, shape):
    need_gpu()
    M, N, K = shape
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((M, K), seed=M + K))
    b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=N + K))
    A, da = orc.quantize_rowwise(a, 0, True)
    B, db = orc.quantize_rowwise(b, 0, True)
    cuda = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda")
    A_, B_, da_, db_ = cuda(A), cuda(B), cuda(da), cuda(db)

    ws = fp8q.gemm_workspace(M, N, K, fp8q.SCALE_ROW)
    ref = fp8q.gemm(A_, 0, B_, 0, fp8q.SCALE_ROW, da_, db_, workspace=ws)
    torch.cuda.synchronize()

    # tolerance basis: sum_k |a b| with the scales (the magnitude every GEMM test uses)
    t = np.abs(orc.decode_table(0)).astype(np.float32)
    mag = (t[A] @ t[B].T).astype(np.float64) * da.astype(np.float64)[:, None] * db.astype(np.float64)[None, :]
    ref64 = ref.float().cpu().numpy().astype(np.float64)

    for _ in range(2):   # two calls in a row share the built-in scratch
        D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        _noalloc_via_c_abi(A_, 0, B_, 0, fp8q.SCALE_ROW, da_, db_, D)
        torch.cuda.synchronize()
        assert_gemm_close(D.float().cpu().numpy().astype(np.float64), ref64, mag, "noalloc vs workspace entry")
        assert torch.equal(D, ref)
    assert fp8q.fp8_device_error(clear=True) == 0
