"""GPU parity of amax and the three quantizers against the CPU oracle:
bit-exact FP8 codes, scales and amax, through the C ABI.

Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-tensor,
per-row, per-block scaling; delayed scaling), §4.2 (amax);
"FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
"FP8 三种缩放配方怎么选" (rowwise power-of-two scales).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_codes_equal, assert_f32_equal, need_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


def _dev(x):
    return x.to("cuda")


def _special_values(n, seed, huge=True):
    """bf16 inputs with edge values mixed in: zeros of both signs, bf16
    subnormals, exact powers of two, and (huge=True) the largest bf16."""
    x = inputs.normal_bf16((n,), 1.0, seed=seed)
    bits = inputs.bf16_bits(x).copy()
    rng = np.random.default_rng(seed)
    special = [0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x3F80, 0xBF80, 0x4300]
    if huge:
        special += [0x7F7F, 0xFF7F]
    special = np.array(special, np.uint16)
    pos = rng.choice(n, special.size * 3, replace=False)
    bits[pos] = np.tile(special, 3)
    return bits


# ---------------------------------------------------------------- amax ----

@pytest.mark.parametrize("n", [0, 1, 7, 8, 1000, 1_000_003, 33_554_432])
def test_amax_matches_oracle(orc, n):
    x = inputs.normal_bf16((max(n, 1),), 2.0, seed=n)[:n]
    bits = inputs.bf16_bits(x)
    a = fp8q.amax(_dev(x))
    ref, _ = orc.amax(bits)
    assert_f32_equal(to_np(a), np.float32([ref]), "amax")


def test_amax_nonfinite_and_signed_zero(orc):
    bits = _special_values(100_001, 3)
    bits[[10, 20, 30, 40]] = [0x7FC0, 0xFFC0, 0x7F80, 0xFF80]
    x = inputs.from_bf16_bits(bits, "cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    a = fp8q.amax(x, counts)
    ref, nf = orc.amax(bits)
    assert_f32_equal(to_np(a), np.float32([ref]), "amax")
    assert int(counts[0]) == nf == 4
    z = inputs.from_bf16_bits(np.array([0x8000] * 40 + [0] * 9, np.uint16), "cuda")
    assert float(fp8q.amax(z)) == 0.0


# -------------------------------------------------------------- tensorwise --

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 17), (3, 1000), (256, 256), (1, 1_048_583)])
def test_tensorwise_current_scaling(orc, fmt, shape):
    x = inputs.normal_bf16(shape, 3.0, seed=11 + fmt)
    bits = inputs.bf16_bits(x)
    q, sinv, am = fp8q.quantize_tensorwise(_dev(x), fmt)
    rq, rsinv, ramax, _ = orc.quantize_tensorwise(bits, fmt)
    assert_codes_equal(to_np(q).reshape(rq.shape), rq, fmt)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]), "scale_inv")
    assert_f32_equal(to_np(am), np.float32([ramax]), "amax")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("n", [65535, 65536, 65537, 65544, 8, 9])
def test_tensorwise_small_tensor_path_boundary(orc, fmt, n):
    """Current scaling of up to 65536 elements runs in one launch (the whole
    tensor in one CTA's registers); longer tensors take the amax pass and the
    cast pass.  Both sides of the boundary, with an element count that is
    not a multiple of 8 inside the small path (65535, 9: the scalar tail),
    a NaN and an Inf in the tensor and a huge element so that the scale is
    set by it: codes, amax, scale and both counters against the oracle."""
    bits = _special_values(n, 40 + n % 7, huge=False) if n >= 64 else inputs.bf16_bits(
        inputs.normal_bf16((n,), 2.0, seed=n)).copy()
    bits[n // 2] = 0x7FC0            # NaN
    bits[n - 1] = 0xFF80             # -Inf, in the tail when n % 8 != 0
    bits[n // 3] = 0x4700            # 32768: the amax
    x = inputs.from_bf16_bits(bits, "cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    q, sinv, am = fp8q.quantize_tensorwise(x, fmt, counts=counts)
    rq, rsinv, ramax, (nf, sat) = orc.quantize_tensorwise(bits, fmt)
    assert_codes_equal(to_np(q).reshape(rq.shape), rq, fmt)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]), "scale_inv")
    assert_f32_equal(to_np(am), np.float32([ramax]), "amax")
    assert (int(counts[0]), int(counts[1])) == (nf, sat) and nf == 2


@pytest.mark.parametrize("fmt", [0, 1])
def test_tensorwise_edge_values(orc, fmt):
    bits = _special_values(50_000, 5 + fmt, huge=False).reshape(500, 100)
    bits[3, 4] = 0x7FC0       # NaN
    bits[7, 9] = 0xFF80       # -Inf
    x = inputs.from_bf16_bits(bits, "cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    q, sinv, am = fp8q.quantize_tensorwise(x, fmt, counts=counts)
    rq, rsinv, ramax, (nf, sat) = orc.quantize_tensorwise(bits, fmt)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]))
    assert_f32_equal(to_np(am), np.float32([ramax]))
    assert (int(counts[0]), int(counts[1])) == (nf, sat)


# bf16 values that are exact round-to-nearest-even ties (or saturate) at scale 1
TIES = {0: [0x3F88, 0x3F98, 0x43E8, 0x43EB, 0x43FA, 0x3A80, 0x3B40, 0x4000, 0x3F8C, 0x7F80, 0x7FC0],
        1: [0x3F90, 0x3FB0, 0x4770, 0x4771, 0x3700, 0x37C0, 0x3F98, 0x7F80, 0x7FC0]}


@pytest.mark.parametrize("fmt", [0, 1])
def test_tensorwise_rne_ties_and_saturation_at_scale_one(orc, fmt):
    """Delayed scale 1: the cast sees the bf16 values themselves, so the
    hardware convert meets exact ties, values past fmax, Inf and NaN."""
    t = np.array(TIES[fmt], np.uint16)
    bits = np.concatenate([t, t | 0x8000, np.tile(t, 20)]).astype(np.uint16)
    bits = np.concatenate([bits, np.zeros((-bits.size) % 16 + 16, np.uint16)])
    x = inputs.from_bf16_bits(bits, "cuda")
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    q, sinv, am = fp8q.quantize_tensorwise(x, fmt, scale_in=one, counts=counts)
    rq, rsinv, ramax, (nf, sat) = orc.quantize_tensorwise(bits, fmt, scale_in=1.0)
    assert_codes_equal(to_np(q).reshape(rq.shape), rq, fmt)
    assert_f32_equal(to_np(am), np.float32([ramax]))
    assert (int(counts[0]), int(counts[1])) == (nf, sat)


@pytest.mark.parametrize("fmt", [0, 1])
def test_tensorwise_delayed_scale_counts_and_amax(orc, fmt):
    x = inputs.lognormal_grads_bf16((640, 384), seed=21)
    bits = inputs.bf16_bits(x).copy()
    bits[0, 0] = 0x7FC0
    x = inputs.from_bf16_bits(bits, "cuda")
    s_in = 2.0 ** 20 if fmt == 1 else 300.0    # forces saturation of the large gradients
    scale = torch.tensor([s_in], dtype=torch.float32, device="cuda")
    counts = torch.zeros(2, dtype=torch.int32, device="cuda")
    q, sinv, am = fp8q.quantize_tensorwise(x, fmt, scale_in=scale, counts=counts)
    rq, rsinv, ramax, (nf, sat) = orc.quantize_tensorwise(bits, fmt, scale_in=s_in)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]))
    assert_f32_equal(to_np(am), np.float32([ramax]))
    assert sat > 0 and (int(counts[0]), int(counts[1])) == (nf, sat)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(64, 64), (96, 208), (4096, 4096)])
def test_tensorwise_transpose(orc, fmt, shape):
    x = inputs.normal_bf16(shape, 0.02, seed=31)
    bits = inputs.bf16_bits(x)
    q, sinv, am = fp8q.quantize_tensorwise(_dev(x), fmt, transpose=True)
    rq, rsinv, ramax, _ = orc.quantize_tensorwise(bits, fmt, transpose_out=True)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]))


# ----------------------------------------------------------------- rowwise --

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("pow2", [True, False])
@pytest.mark.parametrize("shape", [(1, 16), (37, 48), (300, 2048), (5, 4112), (3, 20000)])
def test_rowwise(orc, fmt, pow2, shape):
    x = inputs.outlier_activations_bf16(shape, seed=41, frac=2e-3)
    bits = inputs.bf16_bits(x)
    q, sinv = fp8q.quantize_rowwise(_dev(x), fmt, pow2)
    rq, rsinv = orc.quantize_rowwise(bits, fmt, pow2)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), rsinv)


def test_rowwise_strided_rows_and_special_rows(orc):
    rows, cols, ld = 40, 160, 200
    base = inputs.normal_bf16((rows, ld), 1.0, seed=51)
    bits = inputs.bf16_bits(base).copy()
    bits[3, :] = 0            # all-zero row -> scale 1
    bits[5, 7] = 0x7F80       # +Inf in a row
    bits[6, :cols] = 0x0001   # row of bf16 subnormals -> clamped pow2 scale
    x = inputs.from_bf16_bits(bits, "cuda")
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    sinv = torch.empty(rows, dtype=torch.float32, device="cuda")
    fp8q.fp8_quantize_rowwise(x, rows, cols, ld, 0, True, q, sinv)
    rq, rsinv = orc.quantize_rowwise(np.ascontiguousarray(bits[:, :cols]), 0, True)
    assert_codes_equal(to_np(q), rq, 0)
    assert_f32_equal(to_np(sinv), rsinv)


def test_rowwise_full_size_outlier_activations(orc):
    """4096 x 4096 activations with 0.1 % x100 outliers, pow2 E4M3, bit-exact."""
    x = inputs.outlier_activations_bf16((4096, 4096), seed=1, device="cuda")
    q, sinv = fp8q.quantize_rowwise(x, 0, True)
    rq, rsinv = orc.quantize_rowwise(inputs.bf16_bits(x), 0, True)
    assert_codes_equal(to_np(q), rq, 0)
    assert_f32_equal(to_np(sinv), rsinv)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shapes", [((300, 512), (257, 512)), ((1, 16), (0, 16)), ((0, 64), (33, 64)),
                                    ((4096, 4096), (4096, 4096)), ((3000, 4096), (11008, 4096))])
def test_rowwise_pair_one_launch(orc, fmt, shapes):
    """Both GEMM operands in one launch: each bit-exact against the oracle's
    per-tensor rowwise quantization (the tensors are read with their own
    row counts; a zero count leaves that side alone)."""
    (ra, k), (rb, _) = shapes
    a = inputs.outlier_activations_bf16((max(ra, 1), k), seed=ra + 3)[:ra]
    b = inputs.normal_bf16((max(rb, 1), k), 0.02, seed=rb + 4)[:rb]
    (qa, sa), (qb, sb) = fp8q.quantize_rowwise_pair(_dev(a), _dev(b), fmt, True)
    for q, s, t in ((qa, sa, a), (qb, sb, b)):
        if t.shape[0] == 0:
            continue
        rq, rs = orc.quantize_rowwise(inputs.bf16_bits(t), fmt, True)
        assert_codes_equal(to_np(q), rq, fmt)
        assert_f32_equal(to_np(s), rs)


# --------------------------------------------------------------- blockwise --

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("block_rows", [1, 128])
@pytest.mark.parametrize("shape", [(1, 16), (7, 400), (200, 300 - 300 % 16), (130, 1024), (257, 2064)])
def test_blockwise(orc, fmt, block_rows, shape):
    rng = np.random.default_rng(61)
    x = inputs.normal_bf16(shape, 1.0, seed=61)
    xf = x.float() * torch.from_numpy(10.0 ** rng.integers(-3, 4, shape).astype(np.float32))
    x = xf.to(torch.bfloat16)
    bits = inputs.bf16_bits(x)
    q, sinv = fp8q.quantize_blockwise(_dev(x), fmt, block_rows)
    rq, rsinv = orc.quantize_blockwise(bits, fmt, block_rows)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), rsinv)


def test_blockwise_full_size_mlp_operands(orc):
    """X [8192, 4096] in 1x128 blocks and W_up [11008, 4096] in 128x128 blocks."""
    X = inputs.normal_bf16((8192, 4096), 1.0, seed=2, device="cuda")
    qx, sx = fp8q.quantize_blockwise(X, 0, 1)
    rq, rs = orc.quantize_blockwise(inputs.bf16_bits(X), 0, 1)
    assert_codes_equal(to_np(qx), rq, 0)
    assert_f32_equal(to_np(sx), rs)
    W = inputs.normal_bf16((11008, 4096), 0.02, seed=3, device="cuda")
    qw, sw = fp8q.quantize_blockwise(W, 0, 128)
    rq, rs = orc.quantize_blockwise(inputs.bf16_bits(W), 0, 128)
    assert_codes_equal(to_np(qw), rq, 0)
    assert_f32_equal(to_np(sw), rs)


# ----------------------------------------------------------- error paths --

def test_invalid_arguments_rejected_before_launch():
    x = torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((4, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(fp8q.Fp8Error, match="SHAPE"):
        fp8q.fp8_quantize_rowwise(x, 4, 24, 32, 0, True, q, s)           # cols % 16
    with pytest.raises(fp8q.Fp8Error, match="ALIGNMENT"):
        fp8q.fp8_quantize_rowwise(x, 4, 16, 20, 0, True, q, s)           # ld % 8
    with pytest.raises(fp8q.Fp8Error, match="INVALID_ARG"):
        fp8q.fp8_quantize_blockwise(x, 4, 32, 32, 0, 64, q, s)           # block_rows
    with pytest.raises(fp8q.Fp8Error, match="INVALID_ARG"):
        fp8q.fp8_quantize_tensorwise(x, 4, 32, 0, None, q, 0, s[:1], None)   # current scaling needs amax_out
    with pytest.raises(fp8q.Fp8Error, match="ALIGNMENT"):
        fp8q.fp8_amax(x.view(-1)[1:], s[:1])                             # 2-byte offset pointer


def test_quantize_tensorwise_global_single_rank(orc):
    """Global-scale per-tensor path with one rank: library amax -> (no-op
    exchange) -> scale from the history kernel -> cast; equals the oracle's
    current scaling bit for bit."""
    from fp8_scaled_quantization_amax_b200 import dist as fdist
    x = inputs.normal_bf16((300, 512), 2.0, seed=77)
    q, sinv, am = fdist.quantize_tensorwise_global(x.to("cuda"), 0)
    rq, rsinv, ramax, _ = orc.quantize_tensorwise(inputs.bf16_bits(x), 0)
    assert_codes_equal(to_np(q), rq, 0)
    assert_f32_equal(to_np(sinv), np.float32([rsinv]))
    assert_f32_equal(to_np(am), np.float32([ramax]))


# ------------------------------------------- non-finite / saturation counters --

def _with_nonfinite(bits, seed, k=12):
    """Copy of bf16 bits with NaN, +Inf and -Inf written at seeded positions
    (one whole row NaN when the tensor has more than 4 rows)."""
    b = bits.copy()
    flat = b.reshape(-1)
    rng = np.random.default_rng(seed)
    pos = rng.choice(flat.size, k, replace=False)
    flat[pos] = np.resize(np.array([0x7FC0, 0x7F80, 0xFF80, 0xFFC1], np.uint16), k)
    if b.ndim == 2 and b.shape[0] > 4:
        b[3, :] = 0x7FC0
    return b


def _counts_dev():
    return torch.zeros(2, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(300, 400), (2048, 4096), (7, 8192), (5, 16400)])
def test_counts_rowwise_pair_and_transpose(orc, fmt, shape):
    """Non-finite and saturated counts of the per-row quantizer (pow2 and fp32
    scales), the two-tensor launch and the transposed per-row quantizer equal
    the oracle's ("DeepL押注FP8" §5.1: overflow and NaN are what a run must
    catch); codes and scales stay bit-exact on these inputs."""
    rows, cols = shape
    bits = _with_nonfinite(inputs.bf16_bits(inputs.outlier_activations_bf16(shape, seed=rows + fmt)), rows)
    x = inputs.from_bf16_bits(bits, "cuda")
    for pow2 in (True, False):
        c = _counts_dev()
        q, sinv = fp8q.quantize_rowwise(x, fmt, pow2, counts=c)
        rq, rs, rc = orc.quantize_rowwise(bits, fmt, pow2, counts=True)
        assert_codes_equal(to_np(q), rq, fmt)
        assert_f32_equal(to_np(sinv), rs)
        assert (int(c[0]), int(c[1])) == rc and rc[0] >= cols
    bits_b = _with_nonfinite(inputs.bf16_bits(inputs.normal_bf16((96, cols), 0.02, seed=5)), 9, k=5)
    c = _counts_dev()
    (qa, sa), (qb, sb) = fp8q.quantize_rowwise_pair(x, inputs.from_bf16_bits(bits_b, "cuda"), fmt, True, counts=c)
    ra, rb = orc.quantize_rowwise(bits, fmt, True, counts=True), orc.quantize_rowwise(bits_b, fmt, True, counts=True)
    assert_codes_equal(to_np(qb), rb[0], fmt)
    assert (int(c[0]), int(c[1])) == (ra[2][0] + rb[2][0], ra[2][1] + rb[2][1])
    if rows % 16 == 0:
        c = _counts_dev()
        qT, sT, _ = fp8q.quantize_rowwise_transpose(x, fmt, True, counts=c)
        rqT, rsT, rcT = orc.quantize_rowwise_transpose(bits, fmt, True, counts=True)
        assert_codes_equal(to_np(qT), rqT, fmt)
        assert (int(c[0]), int(c[1])) == rcT


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("block_rows", [1, 128])
@pytest.mark.parametrize("shape", [(300, 400), (1024, 4096)])
def test_counts_blockwise_and_e8m0(orc, fmt, block_rows, shape):
    """Counts of the per-block quantizers (fp32 scales and power-of-two scales
    written as E8M0) against the oracle, codes bit-exact."""
    bits = _with_nonfinite(inputs.bf16_bits(inputs.normal_bf16(shape, 1.0, seed=shape[0] + block_rows)), 77)
    x = inputs.from_bf16_bits(bits, "cuda")
    c = _counts_dev()
    q, sinv = fp8q.quantize_blockwise(x, fmt, block_rows, counts=c)
    rq, rs, rc = orc.quantize_blockwise(bits, fmt, block_rows, counts=True)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), rs)
    assert (int(c[0]), int(c[1])) == rc and rc[0] > 0 and rc[1] > 0
    c = _counts_dev()
    q, _ = fp8q.quantize_blockwise_e8m0(x, fmt, block_rows, counts=c)
    rq, _, rc = orc.quantize_blockwise(bits, fmt, block_rows, pow2=True, counts=True)
    assert_codes_equal(to_np(q), rq, fmt)
    assert (int(c[0]), int(c[1])) == rc


@pytest.mark.parametrize("fmt", [0, 1])
def test_counts_kv_quant(orc, fmt):
    """Counts of the per-(b, h) KV quantizer against the oracle, codes bit-exact;
    a NaN-only slice quantizes with scale 1."""
    kv = inputs.normal_bf16((2, 4, 512, 128), 1.0, seed=13 + fmt)
    bits = _with_nonfinite(inputs.bf16_bits(kv).reshape(8, -1), 21, k=20).reshape(2, 4, 512, 128)
    bits[1, 2] = 0x7FC0
    c = _counts_dev()
    q, sinv = fp8q.kv_quant(inputs.from_bf16_bits(bits, "cuda"), fmt, counts=c)
    rq, rs, rc = orc.kv_quant(bits, fmt, counts=True)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), rs)
    assert (int(c[0]), int(c[1])) == rc and rc[0] >= 512 * 128
