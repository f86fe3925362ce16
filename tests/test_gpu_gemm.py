"""GPU parity of the FP8 scaled GEMM (tcgen05 kernel) against the CPU oracle.

The FP8 operands and scales fed to BOTH sides come from the oracle's own
quantizer applied to seeded bf16 inputs (never from the CUDA path).  The
oracle sums exact products in fp64; the tolerance per element is
1e-2 x sum_k |a_k b_k| (scaled) plus the bf16 rounding of the output.

Sources: "H100 FP8加速实测：新一代计算架构的飞跃" (FP8 multiply-accumulate on
tensor cores); "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
"FP8 三种缩放配方怎么选" (tensorwise / rowwise scaled matmul);
"DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.1 (E5M2 gradients x E4M3
weights), §2.3 (per-block scales), §5.3 (determinism).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_gemm_close, bf16_to_f64, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def _operands(orc, mode, M, N, K, fa=0, fb=0, seed=0, wstd=0.02):
    """Oracle-quantized operands: A from N(0,1) activations, B from N(0,wstd) weights."""
    a_bits = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=seed))
    b_bits = inputs.bf16_bits(inputs.normal_bf16((N, K), wstd, seed=seed + 1))
    if mode == orc.SCALE_TENSOR:
        A, da, _, _ = orc.quantize_tensorwise(a_bits, fa)
        B, db, _, _ = orc.quantize_tensorwise(b_bits, fb)
        da, db = np.float32([da]), np.float32([db])
    elif mode == orc.SCALE_ROW:
        A, da = orc.quantize_rowwise(a_bits, fa, True)
        B, db = orc.quantize_rowwise(b_bits, fb, True)
    else:
        A, da = orc.quantize_blockwise(a_bits, fa, 1)
        B, db = orc.quantize_blockwise(b_bits, fb, 128)
    return A, da, B, db


def _run(A, fa, B, fb, mode, da, db):
    return fp8q.gemm(_cuda(A), fa, _cuda(B), fb, mode, _cuda(da), _cuda(db))


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", [(256, 256, 256), (300, 272, 400), (128, 512, 1024), (1, 8, 16),
                                   (129, 264, 144), (520, 776, 640)])
def test_gemm_full_compare(orc, mode, shape):
    M, N, K = shape
    A, da, B, db = _operands(orc, mode, M, N, K, seed=M + N + K)
    D = _run(A, 0, B, 0, mode, da, db)
    ref, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
    assert_gemm_close(bf16_to_f64(D), ref, mag)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_gemm_e5m2_grad_times_e4m3_weight(orc, mode):
    M, N, K = 264, 320, 512
    g = inputs.bf16_bits(inputs.lognormal_grads_bf16((M, K), seed=7))
    w = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=8))
    if mode == 0:
        A, da, _, _ = orc.quantize_tensorwise(g, 1)
        B, db, _, _ = orc.quantize_tensorwise(w, 0)
        da, db = np.float32([da]), np.float32([db])
    elif mode == 1:
        A, da = orc.quantize_rowwise(g, 1, True)
        B, db = orc.quantize_rowwise(w, 0, True)
    else:
        A, da = orc.quantize_blockwise(g, 1, 1)
        B, db = orc.quantize_blockwise(w, 0, 128)
    D = _run(A, 1, B, 0, mode, da, db)
    ref, mag = orc.gemm_scaled(A, 1, B, 0, mode, da, db)
    assert_gemm_close(bf16_to_f64(D), ref, mag)


def test_gemm_integer_values_exact(orc):
    """Codes of small integers with unit scales: every partial sum is an
    integer below 2^24, so the GPU result is exact (up to bf16 output)."""
    rng = np.random.default_rng(3)
    M, N, K = 192, 264, 384
    enc = {v: orc.encode(float(v), 0) for v in range(-16, 17)}
    va = rng.integers(-16, 17, (M, K))
    vb = rng.integers(-16, 17, (N, K))
    A = np.vectorize(enc.get)(va).astype(np.uint8)
    B = np.vectorize(enc.get)(vb).astype(np.uint8)
    one = np.ones(1, np.float32)
    D = _run(A, 0, B, 0, 0, one, one)
    exact = (va @ vb.T).astype(np.float32)
    bf = torch.from_numpy(exact).to(torch.bfloat16).float().numpy()
    assert np.array_equal(D.float().cpu().numpy(), bf)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_gemm_against_the_naive_fp32_sum(orc, mode):
    """How far the tensor cores' accumulation sits from the naive sequential
    fp32 sum (the oracle's fp32-accumulate variant), both against the fp64
    reference: the GPU's worst error relative to max |ref| is no larger than
    that of the naive fp32 sum rounded to bf16 the same way (both are
    dominated by the output's bf16 rounding), and the two bf16 results agree
    on almost every output (they can differ where an fp32 rounding
    difference lands on a bf16 rounding boundary).  The figures are logged
    with the other GEMM error figures."""
    M, N, K = 520, 776, 640
    A, da, B, db = _operands(orc, mode, M, N, K, seed=90 + mode)
    D = _run(A, 0, B, 0, mode, da, db)
    ref, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
    f32 = orc.gemm_scaled_f32acc(A, 0, B, 0, mode, da, db)
    naive = torch.from_numpy(f32.astype(np.float32)).to(torch.bfloat16)
    got = D.cpu()
    e_gpu = assert_gemm_close(bf16_to_f64(D), ref, mag, f"gpu mode {mode}")
    e_naive = assert_gemm_close(naive.double().numpy(), ref, mag, f"naive fp32 sum mode {mode}")
    assert e_gpu <= 1.5 * e_naive + 1e-12
    assert float((got != naive).float().mean()) < 0.01


def test_gemm_identity_weight(orc):
    K = 256
    A, da, _, _ = orc.quantize_tensorwise(inputs.bf16_bits(inputs.normal_bf16((200, K), 1.0, seed=9)), 0)
    B = np.zeros((K, K), np.uint8)
    B[np.arange(K), np.arange(K)] = 0x38      # 1.0
    D = _run(A, 0, B, 0, 0, np.float32([da]), np.float32([1.0]))
    t = orc.decode_table(0)
    ref = torch.from_numpy((t[A] * np.float64(np.float32(da))).astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(D.cpu(), ref)


def test_gemm_deterministic_and_zero_k(orc):
    A, da, B, db = _operands(orc, 1, 384, 512, 1024, seed=4)
    D1 = _run(A, 0, B, 0, 1, da, db)
    D2 = _run(A, 0, B, 0, 1, da, db)
    assert torch.equal(D1, D2)
    D0 = torch.full((5, 16), 7.0, dtype=torch.bfloat16, device="cuda")
    z = torch.empty((5, 0), dtype=torch.uint8, device="cuda")
    fp8q.fp8_gemm_scaled(z, 0, torch.empty((16, 0), dtype=torch.uint8, device="cuda"), 0, 5, 16, 0, 0,
                         torch.ones(1, device="cuda"), torch.ones(1, device="cuda"), D0, 16)
    assert torch.count_nonzero(D0).item() == 0


def test_gemm_invalid_shapes_rejected():
    A = torch.zeros((64, 40), dtype=torch.uint8, device="cuda")
    s = torch.ones(64, device="cuda")
    D = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8q.Fp8Error, match="SHAPE"):
        fp8q.fp8_gemm_scaled(A, 0, A, 0, 64, 64, 40, 1, s, s, D, 64)      # K % 16
    with pytest.raises(fp8q.Fp8Error, match="ALIGNMENT"):
        fp8q.fp8_gemm_scaled(A, 0, A, 0, 64, 60, 32, 1, s, s, D, 64)      # N % 8
    with pytest.raises(fp8q.Fp8Error, match="INVALID_ARG"):
        fp8q.fp8_gemm_scaled(A, 0, A, 0, 64, 64, 32, 7, s, s, D, 64)      # mode


# ---------------------------------------------------- full-size, sampled --

def _sampled_check(orc, D, A, fa, B, fb, mode, da, db, n=4096, seed=0):
    rng = np.random.default_rng(seed)
    M, N = D.shape
    im = rng.integers(0, M, n)
    inn = rng.integers(0, N, n)
    # always include the corners of the last (ragged) tiles
    im[:4] = [0, M - 1, M - 1, 0]
    inn[:4] = [0, N - 1, 0, N - 1]
    ref, mag = orc.gemm_scaled_sampled(A, fa, B, fb, mode, da, db, im, inn)
    got = D.float().cpu().numpy().astype(np.float64)[im, inn]
    return assert_gemm_close(got, ref, mag)


def test_gemm_rowwise_4096_cube_sampled(orc):
    """Rowwise pow2 E4M3 GEMM at M = N = K = 4096 (activations with 0.1 %
    x100 outliers, N(0, 0.02) weights)."""
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((4096, 4096), seed=1, device="cuda"))
    b = inputs.bf16_bits(inputs.normal_bf16((4096, 4096), 0.02, seed=2, device="cuda"))
    A, da = orc.quantize_rowwise(a, 0, True)
    B, db = orc.quantize_rowwise(b, 0, True)
    D = _run(A, 0, B, 0, 1, da, db)
    _sampled_check(orc, D, A, 0, B, 0, 1, da, db)


@pytest.mark.parametrize("which", ["up", "down"])
def test_gemm_blockwise_mlp_sampled(orc, which):
    """Block-scaled MLP GEMMs: [8192, 4096] x W_up[11008, 4096]^T and
    [8192, 11008] x W_down[4096, 11008]^T (the second GEMM's input is a seeded
    bf16 tensor of the same shape, so no oracle input comes from the GPU)."""
    if which == "up":
        M, N, K = 8192, 11008, 4096
    else:
        M, N, K = 8192, 4096, 11008
    x = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=5, device="cuda"))
    w = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=6, device="cuda"))
    A, da = orc.quantize_blockwise(x, 0, 1)
    B, db = orc.quantize_blockwise(w, 0, 128)
    D = _run(A, 0, B, 0, 2, da, db)
    _sampled_check(orc, D, A, 0, B, 0, 2, da, db, n=2048)


# ------------------------------------- split-K over CTA pairs (workspace) --

_PAIR_SPLIT_SHAPES = [(1000, 1288, 8208), (1024, 1280, 8192)]   # 20-24 pair tiles, K >= 64 blocks, 40-48 1-SM tiles


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("shape", _PAIR_SPLIT_SHAPES)
def test_gemm_pair_split_sampled_and_repeatable(orc, mode, shape):
    """With a workspace, a long-K problem whose 256 x 256 tiles fill at most
    half of the CTA pairs computes each tile as two K halves on two pairs
    (the first half hands its fp32 partial to the second through the
    workspace); sampled against the oracle (ragged M, N and K included),
    bit-identical over repeated calls (a fresh hand-off epoch per call, so a
    reused workspace is safe), and too small a workspace gives the unsplit
    schedule, still correct."""
    M, N, K = shape
    A, da, B, db = _operands(orc, mode, M, N, K, seed=M + 3 * N + K)
    ws = fp8q.gemm_workspace(M, N, K, mode)
    assert ws is not None and ws.numel() > 0
    A_, B_, da_, db_ = _cuda(A), _cuda(B), _cuda(da), _cuda(db)
    D1 = fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, workspace=ws)
    _sampled_check(orc, D1, A, 0, B, 0, mode, da, db, n=2048, seed=mode)
    for _ in range(3):
        assert torch.equal(fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, workspace=ws), D1)
    small = torch.zeros(ws.numel() - 256, dtype=torch.uint8, device="cuda")
    D0 = fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, workspace=small)
    _sampled_check(orc, D0, A, 0, B, 0, mode, da, db, n=2048, seed=mode + 2)


def test_gemm_long_k_few_tiles_cluster_split_sampled(orc):
    """A skinny, long-K GEMM (1024 x 1024 x 16384: 32 tiles of 128 x 256)
    needs no workspace: each tile is shared by a cluster of CTAs splitting K
    (32 K blocks each); sampled against the oracle.  Shapes that split this
    way, or whose last wave of tiles is more than half full, ask for no
    workspace."""
    M, N, K = 1024, 1024, 16384
    a = inputs.bf16_bits(inputs.outlier_activations_bf16((M, K), seed=11, device="cuda"))
    b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=12, device="cuda"))
    A, da = orc.quantize_rowwise(a, 0, True)
    B, db = orc.quantize_rowwise(b, 0, True)
    assert fp8q.fp8_gemm_workspace_size(M, N, K, 1) == 0
    D = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, 1, _cuda(da), _cuda(db))
    _sampled_check(orc, D, A, 0, B, 0, 1, da, db, n=1024, seed=4)
    # several waves whose last one is more than half full: no split
    assert fp8q.fp8_gemm_workspace_size(8192, 11008, 4096, 1) == 0


def test_launch_chain_keeps_stream_order(orc):
    """The quantizers and GEMMs are launched with programmatic dependent
    launch: each may start before its predecessor ends and waits for it
    before touching memory.  Reusing the same FP8 buffers for two different
    inputs back to back (quantize -> GEMM -> quantize over the same buffers
    -> GEMM ...) must give every GEMM the operands quantized just before it
    (a read-after-write and a write-after-read hazard on every step)."""
    M, N, K = 512, 768, 1024
    xs = [inputs.outlier_activations_bf16((M, K), seed=200 + i, device="cuda") for i in range(2)]
    ws = [inputs.normal_bf16((N, K), 0.02, seed=210 + i, device="cuda") for i in range(2)]
    refs = []
    for i in range(2):
        (qa, sa), (qb, sb) = fp8q.quantize_rowwise_pair(xs[i], ws[i], 0, True)
        refs.append(fp8q.gemm(qa, 0, qb, 0, fp8q.SCALE_ROW, sa, sb).clone())
    torch.cuda.synchronize()
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    qb = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, dtype=torch.float32, device="cuda")
    sb = torch.empty(N, dtype=torch.float32, device="cuda")
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(40)]
    for j, out in enumerate(outs):
        i = j % 2
        fp8q.fp8_quantize_rowwise_pair(xs[i], M, K, qa, sa, ws[i], N, K, qb, sb, K, 0, True)
        fp8q.fp8_gemm_scaled(qa, 0, qb, 0, M, N, K, fp8q.SCALE_ROW, sa, sb, out, N)
    torch.cuda.synchronize()
    for j, out in enumerate(outs):
        assert torch.equal(out, refs[j % 2]), j


def test_split_k_gemm_replays_in_a_cuda_graph(orc):
    """A split-K GEMM (the workspace hand-off between CTA pairs) captured in a
    CUDA graph and replayed with new operands copied into the captured
    buffers: each replay must match the eager call on the same operands (the
    launch clears its hand-off flags, so a replay, which reuses the captured
    epoch, never sees the previous replay's flag)."""
    M, N, K = _PAIR_SPLIT_SHAPES[0]
    mode = fp8q.SCALE_ROW
    ws = fp8q.gemm_workspace(M, N, K, mode)
    assert ws is not None and ws.numel() > 0
    ops = [_operands(orc, mode, M, N, K, seed=500 + i) for i in range(3)]
    A_, da_ = _cuda(ops[0][0]), _cuda(ops[0][1])
    B_, db_ = _cuda(ops[0][2]), _cuda(ops[0][3])
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, out=D, workspace=ws)   # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, out=D, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(6):
        A, da, B, db = ops[rep % 3]
        A_.copy_(_cuda(A)); da_.copy_(_cuda(da)); B_.copy_(_cuda(B)); db_.copy_(_cuda(db))
        g.replay()
        torch.cuda.synchronize()
        ref = fp8q.gemm(_cuda(A), 0, _cuda(B), 0, mode, _cuda(da), _cuda(db), workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(D, ref), rep
        if rep < 3:
            _sampled_check(orc, D, A, 0, B, 0, mode, da, db, n=512, seed=rep)
    del g


# ------------------------------------ few-row GEMMs: K split over a cluster --

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", [(1, 4096, 4096), (17, 2048, 2048), (100, 776, 1424), (64, 264, 528),
                                   (16, 9736, 768), (260, 520, 1040)])
def test_gemm_few_tiles_cluster_split_full_compare(orc, mode, shape):
    """Few output tiles: each 128 x 256 tile is shared by a cluster of CTAs,
    each accumulating a K range, and the partial tiles are summed through
    distributed shared memory in rank order.  M <= 128 splits into 2 to 8 K
    parts (3 at 39 tiles), larger M when S >= 4 fits (260 rows: 9 tiles,
    4 parts); ragged M, N and K (a last K block of 16); full compare with the
    oracle and bit-identical repeats."""
    M, N, K = shape
    A, da, B, db = _operands(orc, mode, M, N, K, seed=M + 5 * N + K)
    A_, B_, da_, db_ = _cuda(A), _cuda(B), _cuda(da), _cuda(db)
    D = fp8q.gemm(A_, 0, B_, 0, mode, da_, db_)
    ref, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
    assert_gemm_close(bf16_to_f64(D), ref, mag)
    for _ in range(2):
        assert torch.equal(fp8q.gemm(A_, 0, B_, 0, mode, da_, db_), D)


def test_gemm_few_rows_takes_the_cluster_split_and_replays_in_a_graph(orc):
    """The decode-shaped GEMM (16 x 4096 x 4096) launches the cluster
    split-K kernel (checked by kernel name in the profiler's trace), and the
    launch, captured in a CUDA graph, replays to the eager result on new
    operands copied into the captured buffers."""
    from torch.profiler import ProfilerActivity, profile
    M, N, K = 16, 4096, 4096
    mode = fp8q.SCALE_ROW
    ops = [_operands(orc, mode, M, N, K, seed=700 + i) for i in range(2)]
    A_, da_, B_, db_ = (_cuda(x) for x in ops[0])
    D = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, out=D)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if "k_gemm_fp8" in e.name]
    # k_gemm_fp8<MODE = 1, SPLIT = true>, demangled or not
    assert names and all("k_gemm_fp8<1, true>" in n or "ILi1ELb1E" in n for n in names), names
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            fp8q.gemm(A_, 0, B_, 0, mode, da_, db_, out=D)
    torch.cuda.current_stream().wait_stream(s)
    for rep in range(4):
        A, da, B, db = ops[rep % 2]
        A_.copy_(_cuda(A)); da_.copy_(_cuda(da)); B_.copy_(_cuda(B)); db_.copy_(_cuda(db))
        g.replay()
        torch.cuda.synchronize()
        ref, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
        assert_gemm_close(bf16_to_f64(D), ref, mag)
        assert torch.equal(D, fp8q.gemm(_cuda(A), 0, _cuda(B), 0, mode, _cuda(da), _cuda(db))), rep
    del g
