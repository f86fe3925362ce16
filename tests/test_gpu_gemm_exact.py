"""Exact GEMM parity on every schedule of the library's FP8 GEMMs.

FP8 codes of small integers (|v| <= 16 for E4M3, <= 8 for E5M2; every such
integer is a code) with power-of-two scales make every partial sum the
tensor cores form exact in fp32: the K-block partials, their promotion in
the block-scaled epilogue, the split-K hand-offs and the scale products.  The
GPU result must therefore equal the exact product -- integer matmul in fp64
times the scales -- rounded once to bf16, bit for bit.  A dropped, doubled
or misplaced K block, a swapped half tile, a wrong scale index or a lost
split-K partial changes an exact integer and fails, at any K; the
magnitude-based tolerance of the other GEMM tests cannot see such errors at
K = 4096 and beyond.

Each shape is one the library dispatches to a particular schedule: the CTA
pair kernel over several waves, the pair split with a workspace, the cluster
split of the one-SM kernel, the block-scaled pair kernel, the E8M0 kernel and
the grouped kernel.  Full-size shapes compare every column of a spread of
rows that touches every row tile.

Sources: "H100 FP8加速实测：新一代计算架构的飞跃" (FP8 multiply-accumulate on
the tensor cores); "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.1 (E5M2
gradients against E4M3 weights), §2.3 (per-tensor, per-row and per-block
scaling), §3.2 (grouped GEMM for experts), §5.3 (results must not depend on
how the GEMM is split); "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍",
section "FP8 三种缩放配方怎么选" (tensorwise / rowwise scaled matmul).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

TORCH_FP8 = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}
VMAX = {0: 16, 1: 8}


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def _int_codes(rng, shape, fmt, vmax=None):
    """(integer values, their FP8 codes); torch's float8 conversion of an
    exactly representable value is that value's code."""
    top = VMAX[fmt] if vmax is None else vmax
    v = rng.integers(-top, top + 1, shape).astype(np.int64)
    codes = torch.from_numpy(v.astype(np.float32)).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    return v, codes


def _pow2(rng, shape, lo, hi):
    return np.exp2(rng.integers(lo, hi + 1, shape)).astype(np.float32)


def _scale_maps(mode, M, N, K, da, db):
    """Per-element scale factors SA [M, K] and SB [N, K] with D = (A*SA) (B*SB)^T."""
    if mode == 0:
        return np.full((M, K), da[0], np.float64), np.full((N, K), db[0], np.float64)
    if mode == 1:
        return np.repeat(da.astype(np.float64)[:, None], K, 1), np.repeat(db.astype(np.float64)[:, None], K, 1)
    kb = np.arange(K) // 128
    SA = da.astype(np.float64).T[:, kb]                                   # da [nkb, M]
    SB = db.astype(np.float64)[(np.arange(N) // 128)[:, None], kb[None, :]]   # db [ceil(N/128), nkb]
    return SA, SB


def _exact_bf16(va, vb, SA, SB, rows=None):
    """The exact product (fp64; every term and partial sum is an integer
    times a power of two well inside 2^53) rounded once to bf16."""
    a = va.astype(np.float64) * SA
    if rows is not None:
        a = a[rows]
    exact = a @ (vb.astype(np.float64) * SB).T
    f32 = exact.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), exact), "reference not exact in fp32"
    return torch.from_numpy(f32).to(torch.bfloat16)


def _operands(M, N, K, mode, fa=0, fb=0, seed=0, vmax=None):
    rng = np.random.default_rng(seed)
    va, A = _int_codes(rng, (M, K), fa, vmax)
    vb, B = _int_codes(rng, (N, K), fb, vmax)
    nkb = (K + 127) // 128
    if mode == 0:
        da, db = np.float32([0.5]), np.float32([2.0])
    elif mode == 1:
        da, db = _pow2(rng, M, -2, 2), _pow2(rng, N, -2, 2)
    else:   # every product da * db in {1/2, 1, 2}: promoted sums stay multiples of 1/2 below 2^23
        da, db = _pow2(rng, (nkb, M), -1, 0), _pow2(rng, ((N + 127) // 128, nkb), 0, 1)
    return va, A, da, vb, B, db


def _rows_touching_every_tile(M, n=512, seed=0):
    rng = np.random.default_rng(seed)
    r = np.unique(np.concatenate([rng.integers(0, M, n), np.arange(0, M, 128), np.arange(127, M, 128), [M - 1]]))
    return r[r < M]


def _check(D, va, vb, SA, SB, rows=None, what=""):
    ref = _exact_bf16(va, vb, SA, SB, rows)
    got = D.cpu() if rows is None else D.cpu()[torch.from_numpy(rows)]
    if not torch.equal(got, ref):
        bad = (got != ref).nonzero()[:4].tolist()
        raise AssertionError(f"{what}: {int((got != ref).sum())} outputs differ from the exact result, first {bad}")


# --------------------------------------------------- tensor and row modes --

@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("shape", [(4096, 4096, 4096), (300, 272, 400), (520, 776, 640), (129, 272, 144), (300, 272, 48)])
def test_exact_pair_kernel(mode, shape):
    """CTA-pair kernel: 4096^3 runs 256 tiles over several waves of pairs."""
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, mode, seed=M + N + K + mode)
    D = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, mode, _cuda(da), _cuda(db))
    SA, SB = _scale_maps(mode, M, N, K, da, db)
    _check(D, va, vb, SA, SB, what=f"pair {shape}")


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("shape", [(1000, 1288, 8208), (1024, 1536, 16384), (4096, 4096, 8192)])
def test_exact_pair_split_with_workspace(mode, shape):
    """Long K, few 256 x 256 tiles: each tile's K halves run on two pairs and
    the first hands its fp32 partial to the second through the workspace
    (ragged K included: 8208 = 64 blocks + 16); 4096 x 4096 x 8192: only the
    last wave's tiles are split (their first halves run first, their second halves
    last).  Repeated calls reuse the workspace and must give the same exact
    result."""
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, mode, seed=7 + mode, vmax=8)
    ws = fp8q.gemm_workspace(M, N, K, mode)
    assert ws is not None and ws.numel() > 0, "this shape is meant to take the pair split"
    A_, B_, da_, db_ = _cuda(A), _cuda(B), _cuda(da), _cuda(db)
    SA, SB = _scale_maps(mode, M, N, K, da, db)
    for rep in range(2):
        D = fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, workspace=ws)
        _check(D, va, vb, SA, SB, what=f"pair split {shape} call {rep}")


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1024, 1024, 16384), (16, 4096, 4096), (1, 4096, 4096), (100, 776, 1424)])
def test_exact_cluster_split(mode, shape):
    """Few output tiles: each 128 x 256 tile shared by a thread-block cluster
    splitting K, the parts summed through distributed shared memory."""
    M, N, K = shape
    if mode == 1 or mode == 0:
        assert fp8q.fp8_gemm_workspace_size(M, N, K, mode) == 0
    va, A, da, vb, B, db = _operands(M, N, K, mode, seed=11 + mode + M, vmax=8)
    D = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, mode, _cuda(da), _cuda(db))
    SA, SB = _scale_maps(mode, M, N, K, da, db)
    _check(D, va, vb, SA, SB, what=f"cluster split {shape}")


def test_exact_dgrad_e5m2_times_e4m3():
    """The data-gradient shape: E5M2 gradients [8192, 4096] x E4M3 W^T [4096, 4096], rowwise."""
    M, N, K = 8192, 4096, 4096
    va, A, da, vb, B, db = _operands(M, N, K, 1, fa=1, fb=0, seed=21)
    D = fp8q.gemm(_cuda(A), 1, _cuda(B), 0, 1, _cuda(da), _cuda(db))
    SA, SB = _scale_maps(1, M, N, K, da, db)
    rows = _rows_touching_every_tile(M)
    _check(D, va, vb, SA, SB, rows, what="dgrad")


# ------------------------------------------------------ block-scaled mode --

@pytest.mark.parametrize("shape", [(300, 272, 400), (520, 776, 640), (4096, 4096, 4096), (640, 1024, 896),
                                   (129, 272, 144), (300, 272, 48), (520, 784, 16)])
def test_exact_block_scaled_pair_kernel(shape):
    """fp32 per-block scales (1x128 of A, 128x128 of B): each K block's
    partial promoted by the epilogue; ragged M, N and K, K below one block
    (48, 16: a single partial K block) and M = 129 (the odd CTA of the pair
    holds one row)."""
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=31 + M)
    A_, B_, da_, db_ = _cuda(A), _cuda(B), _cuda(da), _cuda(db)
    D = fp8q.gemm(A_, 0, B_, 0, 2, da_, db_)
    SA, SB = _scale_maps(2, M, N, K, da, db)
    _check(D, va, vb, SA, SB, what=f"block {shape}")
    assert torch.equal(fp8q.gemm(A_, 0, B_, 0, 2, da_, db_), D)   # bit-identical repeat


@pytest.mark.parametrize("which", ["up", "down"])
def test_exact_block_scaled_mlp_full_size(which):
    """The MLP GEMMs at full size: [8192, 4096] x W_up[11008, 4096]^T and
    [8192, 11008] x W_down[4096, 11008]^T (86 K blocks)."""
    M, N, K = (8192, 11008, 4096) if which == "up" else (8192, 4096, 11008)
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=41 if which == "up" else 42, vmax=8)
    D = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, 2, _cuda(da), _cuda(db))
    SA, SB = _scale_maps(2, M, N, K, da, db)
    rows = _rows_touching_every_tile(M, n=256)
    _check(D, va, vb, SA, SB, rows, what=f"block mlp {which}")


# ------------------------------------------------ E8M0 block scales (MMA) --

@pytest.mark.parametrize("shape", [(300, 272, 400), (4096, 4096, 4096)])
def test_exact_e8m0_kernel(shape):
    """Power-of-two block scales applied inside the tensor core: the same
    exact result as the per-block promotion."""
    from tests.test_gpu_block_e8m0 import _image
    M, N, K = shape
    va, A, da, vb, B, db = _operands(M, N, K, 2, seed=51 + M)
    img_a = _image(da, M, K, 1)
    img_b = _image(db, N, K, 128)
    D = fp8q.gemm_block_e8m0(_cuda(A), 0, _cuda(B), 0, _cuda(img_a), _cuda(img_b))
    SA, SB = _scale_maps(2, M, N, K, da, db)
    rows = None if M <= 1024 else _rows_touching_every_tile(M)
    _check(D, va, vb, SA, SB, rows, what=f"e8m0 {shape}")


# ------------------------------------------------------------ grouped GEMM --

@pytest.mark.parametrize("mode", [0, 1])
def test_exact_grouped(mode):
    """Ragged token groups (with empty ones) against per-expert weights."""
    sizes, N, K = [0, 37, 600, 300, 1, 0, 1030], 528, 1024
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    M = int(off[-1])
    rng = np.random.default_rng(61 + mode)
    va, A = _int_codes(rng, (M, K), 0)
    vb, B = _int_codes(rng, (G, N, K), 0)
    if mode == 0:
        da, db = _pow2(rng, G, -2, 2), _pow2(rng, G, -2, 2)
    else:
        da, db = _pow2(rng, M, -2, 2), _pow2(rng, G * N, -2, 2)
    D = fp8q.gemm_grouped(_cuda(A), 0, _cuda(B), 0, _cuda(off), mode, _cuda(da), _cuda(db))
    ref = np.zeros((M, N), np.float64)
    for e in range(G):
        r0, r1 = off[e], off[e + 1]
        if r1 == r0:
            continue
        sa = da[e] if mode == 0 else da[r0:r1].astype(np.float64)[:, None]
        sb = db[e] if mode == 0 else db[e * N:(e + 1) * N].astype(np.float64)[None, :]
        ref[r0:r1] = (va[r0:r1].astype(np.float64) @ vb[e].astype(np.float64).T) * sa * sb
    f32 = ref.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), ref)
    assert torch.equal(D.cpu(), torch.from_numpy(f32).to(torch.bfloat16))
