"""Pins for the CPU oracle: each test checks it against something other than
itself -- values the pages print, the format definition's fixed points,
library routines that compute a special case (torch's CPU float8 / bf16
casts, numpy / integer matmul), closed forms, invariants and brute force.

Pages cited:
  "DeepL押注FP8：大模型训练与推理统一精度实战解析" (§2.1 formats, §2.3 scaling
  granularity and delayed scaling, §3.1 FP8 KV cache, §4.2 amax statistics);
  "H100 FP8加速实测：新一代计算架构的飞跃" (E5M2 range +-57344);
  "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
  "FP8 三种缩放配方怎么选" (rowwise power-of-two scales).
"""
import math
import os

import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FMTS = {"e4m3": 0, "e5m2": 1}
TORCH_FP8 = {0: torch.float8_e4m3fn, 1: torch.float8_e5m2}


def _golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        if line.startswith("#") or not line.strip():
            continue
        rows.append(line.split())
    return rows


def _bits(x: torch.Tensor) -> np.ndarray:
    return inputs.bf16_bits(x)


# ----------------------------------------------------------------- decode --

@pytest.mark.parametrize("fmt", [0, 1])
def test_decode_matches_torch_float8_views(orc, fmt):
    """All 256 codes against torch's own float8 dtypes (a library decode)."""
    ours = orc.decode_table(fmt)
    lib = torch.arange(256, dtype=torch.uint8).view(TORCH_FP8[fmt]).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    # signed zero survives
    assert math.copysign(1.0, ours[0x80]) == -1.0


def test_decode_code_counts(orc):
    """E4M3: 254 finite (with +-0) + 2 NaN, no Inf.  E5M2: 248 finite + 2 Inf + 6 NaN."""
    e4 = orc.decode_table(0)
    e5 = orc.decode_table(1)
    assert np.isfinite(e4).sum() == 254 and np.isnan(e4).sum() == 2 and np.isinf(e4).sum() == 0
    assert np.isfinite(e5).sum() == 248 and np.isnan(e5).sum() == 6 and np.isinf(e5).sum() == 2


def test_decode_golden_points(orc):
    """Fixed points of the formats, incl. the E5M2 range the H100 page prints."""
    for fmt_s, code, val, *_ in _golden("fp8_format_points.txt"):
        got = orc.decode(int(code, 16), FMTS[fmt_s])
        exp = float(val)
        if math.isnan(exp):
            assert math.isnan(got), (fmt_s, code)
        else:
            assert got == exp and math.copysign(1, got) == math.copysign(1, exp), (fmt_s, code, got)
    assert orc.fmax(1) == 57344.0 and orc.fmax(0) == 448.0


@pytest.mark.parametrize("fmt", [0, 1])
def test_decode_monotone_positive_codes(orc, fmt):
    t = orc.decode_table(fmt)
    top = 0x7E if fmt == 0 else 0x7B
    pos = t[: top + 1]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80: 0x80 + top + 1], -pos)


# ----------------------------------------------------------------- encode --

def test_encode_golden_cases(orc):
    for fmt_s, x, code, *_ in _golden("fp8_encode_cases.txt"):
        assert orc.encode(float(x), FMTS[fmt_s]) == int(code, 16), (fmt_s, x)


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_roundtrip_all_finite_codes(orc, fmt):
    t = orc.decode_table(fmt)
    for c in range(256):
        if np.isfinite(t[c]):
            assert orc.encode(t[c], fmt) == c, hex(c)


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_matches_torch_in_range(orc, fmt):
    """In range, torch's CPU fp32 -> float8 conversion is RNE; it only differs
    from the saturating cast above fmax (it overflows to NaN / Inf there)."""
    rng = np.random.default_rng(11 + fmt)
    fm = orc.fmax(fmt)
    # log-uniform magnitudes across the whole range incl. subnormals, both signs
    e = rng.uniform(-20 if fmt == 0 else -19, math.log2(fm), 20000)
    y = (np.exp2(e) * rng.choice([-1.0, 1.0], e.size)).astype(np.float32)
    # plus exact midpoints between neighbouring codes (ties)
    t = orc.decode_table(fmt)
    top = 0x7E if fmt == 0 else 0x7B
    mids = ((t[: top] + t[1: top + 1]) / 2).astype(np.float32)
    y = np.concatenate([y, mids, -mids])
    y = y[np.abs(y) <= fm]
    ours = orc.encode_array(y, fmt)
    lib = torch.from_numpy(y).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)


@pytest.mark.parametrize("fmt", [0, 1])
def test_encode_is_nearest_by_brute_force(orc, fmt):
    """Brute force over all finite codes: the chosen code is a nearest one."""
    rng = np.random.default_rng(5)
    t = orc.decode_table(fmt)
    fin = np.isfinite(t)
    fm = orc.fmax(fmt)
    y = (rng.standard_normal(3000) * rng.choice([1e-4, 1e-2, 1.0, 100.0], 3000)).astype(np.float32)
    for v in y:
        c = orc.encode(v, fmt)
        if abs(v) >= fm:
            assert abs(t[c]) == fm
            continue
        best = np.min(np.abs(t[fin] - np.float64(v)))
        assert abs(t[c] - np.float64(v)) == best


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-30, 30, 20000)).astype(np.float32)
    # exact ties: bf16 values plus half an ulp
    base = torch.from_numpy(rng.standard_normal(2000).astype(np.float32)).to(torch.bfloat16)
    bb = base.float().numpy().view(np.uint32)
    ties = (bb | np.uint32(0x8000)).view(np.float32)
    f = np.concatenate([f, ties, np.array([3.3895e38, 3.4e38], np.float32)])
    ours = np.array([orc.f32_to_bf16(v) for v in f], np.uint16)
    lib = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


# ------------------------------------------------------------ amax, scale --

def test_amax_against_numpy_and_nonfinite(orc):
    x = inputs.normal_bf16((1000,), 3.0, seed=1)
    bits = _bits(x).copy()
    assert orc.amax(bits)[0] == np.abs(x.float().numpy()).max()
    bits[[3, 50, 700]] = [0x7FC0, 0x7F80, 0xFF80]   # NaN, +Inf, -Inf
    ref = np.abs(x.float().numpy())
    ref[[3, 50, 700]] = 0
    a, nf = orc.amax(bits)
    assert a == ref.max() and nf == 3
    assert orc.amax(np.zeros(17, np.uint16))[0] == 0.0
    assert orc.amax(np.array([0x8000, 0x0000], np.uint16))[0] == 0.0


@pytest.mark.parametrize("fmt", [0, 1])
def test_scale_closed_forms(orc, fmt):
    fm = orc.fmax(fmt)
    assert orc.scale_from_amax(0.0, fmt) == 1.0
    assert orc.scale_from_amax(1.0, fmt) == fm
    assert orc.scale_from_amax(fm, fmt) == 1.0
    assert orc.scale_from_amax(1e-38, fmt) == np.finfo(np.float32).max   # overflow clamps
    assert orc.scale_pow2_from_amax(1.0, fmt) == (256.0 if fmt == 0 else 32768.0)
    assert orc.scale_pow2_from_amax(fm, fmt) == 1.0
    assert orc.scale_pow2_from_amax(0.0, fmt) == 1.0
    assert orc.scale_pow2_from_amax(float(np.nextafter(np.float32(fm), np.float32(1e9))), fmt) == 0.5


@pytest.mark.parametrize("fmt", [0, 1])
def test_pow2_scale_property_on_bf16_amax(orc, fmt):
    """s is a power of two with amax*s <= fmax < amax*2s (the largest such)."""
    fm = orc.fmax(fmt)
    x = inputs.normal_bf16((4000,), 1.0, seed=2)
    vals = np.abs(x.float().numpy()) * 10.0 ** np.random.default_rng(0).uniform(-30, 30, 4000)
    vals = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).float().numpy()
    for a in vals[vals > 0]:
        s = orc.scale_pow2_from_amax(float(a), fmt)
        m, e = math.frexp(s)
        assert m == 0.5
        if s < 2.0 ** 127:
            assert np.float64(a) * s <= fm < np.float64(a) * 2 * s


# --------------------------------------------------------------- quantize --

@pytest.mark.parametrize("fmt", [0, 1])
def test_tensorwise_invariants(orc, fmt):
    """The amax element maps to +-fmax; every element is the cast of x*s, and
    the dequantized value is within half a code step of x."""
    x = inputs.normal_bf16((96, 80), 2.0, seed=3)
    bits = _bits(x)
    q, sinv, amax, (nf, sat) = orc.quantize_tensorwise(bits, fmt)
    xf = x.float().numpy()
    assert amax == np.abs(xf).max() and nf == 0 and sat == 0
    s = np.float32(orc.fmax(fmt)) / np.float32(amax)
    assert sinv == np.float32(1.0) / s
    t = orc.decode_table(fmt)
    i = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert abs(t[q[i]]) == orc.fmax(fmt)
    # relative error of the dequantized tensor: at most half a mantissa step
    deq = t[q].astype(np.float64) * sinv
    rel = 2.0 ** -(4 if fmt == 0 else 3)
    tiny = orc.decode(1, fmt) * sinv
    assert np.all(np.abs(deq - xf) <= rel * np.abs(xf) + tiny)
    # transposed output is the transpose
    qt, *_ = orc.quantize_tensorwise(bits, fmt, transpose_out=True)
    assert np.array_equal(qt, q.T)
    # lib cross-check of the whole cast (values in range, no saturation)
    y = (xf * s).astype(np.float32)
    lib = torch.from_numpy(y).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(q, lib)


def test_tensorwise_delayed_scale_saturation(orc):
    x = inputs.normal_bf16((64, 64), 1.0, seed=4)
    bits = _bits(x)
    q, sinv, amax, (nf, sat) = orc.quantize_tensorwise(bits, 0, scale_in=1000.0)
    xf = x.float().numpy()
    assert sat == int((np.abs(xf.astype(np.float32) * np.float32(1000.0)) > 448).sum()) > 0
    assert sinv == np.float32(1.0) / np.float32(1000.0)
    assert amax == np.abs(xf).max()
    t = orc.decode_table(0)
    assert np.all(np.abs(t[q]) <= 448)


@pytest.mark.parametrize("fmt", [0, 1])
def test_rowwise_pow2_per_row(orc, fmt):
    """Per-row pow2 scales; with outlier rows the per-row scale keeps the
    ordinary rows precise where a per-tensor scale would not (the outlier
    claim of the DeepL page §2.3)."""
    x = inputs.outlier_activations_bf16((64, 256), seed=5, frac=2e-3)
    bits = _bits(x)
    q, sinv = orc.quantize_rowwise(bits, fmt, pow2=True)
    xf = x.float().numpy()
    t = orc.decode_table(fmt)
    fm = orc.fmax(fmt)
    for r in range(64):
        a = np.abs(xf[r]).max()
        s = 1.0 / sinv[r]
        assert math.frexp(s)[0] == 0.5 and a * s <= fm < a * 2 * s
        row = torch.from_numpy((xf[r] * np.float32(s)).astype(np.float32))
        assert np.array_equal(q[r], row.to(TORCH_FP8[fmt]).view(torch.uint8).numpy())
    # one extreme outlier row: under one tensor scale the ordinary rows fall
    # into the subnormal range and lose precision; per-row scales keep them
    xo = inputs.normal_bf16((64, 256), 1.0, seed=15).float()
    xo[0, 7] = 1.0e5 if fmt == 0 else 1.0e11   # pushes ordinary values to subnormals
    ob = _bits(xo.to(torch.bfloat16))
    xof = xo.to(torch.bfloat16).float().numpy()
    qr, sr = orc.quantize_rowwise(ob, fmt, pow2=True)
    qt, st, *_ = orc.quantize_tensorwise(ob, fmt)
    err_row = np.abs(t[qr[1:]] * sr[1:, None] - xof[1:]).sum()
    err_ten = np.abs(t[qt[1:]] * st - xof[1:]).sum()
    assert err_row < 0.5 * err_ten


@pytest.mark.parametrize("block_rows", [1, 128])
def test_blockwise_layout_and_invariants(orc, block_rows):
    """Blocks with very different magnitudes: each block's scale follows its
    own amax (checked against a numpy reshape-max), the block's amax element
    maps to fmax, and the scale layout is the documented one."""
    rows, cols = (200, 300) if block_rows == 128 else (7, 400)
    rng = np.random.default_rng(6)
    xf = rng.standard_normal((rows, cols)).astype(np.float32)
    nrb, nkb = -(-rows // block_rows), -(-cols // 128)
    mult = 10.0 ** rng.integers(-3, 4, (nrb, nkb))
    xf *= np.kron(mult, np.ones((block_rows, 128)))[:rows, :cols]
    x = torch.from_numpy(xf).to(torch.bfloat16)
    bits = _bits(x)
    q, sinv = orc.quantize_blockwise(bits, 0, block_rows)
    xb = x.float().numpy()
    pad = np.zeros((nrb * block_rows, nkb * 128), np.float32)
    pad[:rows, :cols] = np.abs(xb)
    bam = pad.reshape(nrb, block_rows, nkb, 128).max(axis=(1, 3))
    exp_s = np.float32(448.0) / bam.astype(np.float32)
    exp_inv = (np.float32(1.0) / exp_s).astype(np.float32)
    if block_rows == 1:
        assert sinv.shape == (nkb, rows)
        assert np.array_equal(sinv, exp_inv.T)
    else:
        assert sinv.shape == (nrb, nkb)
        assert np.array_equal(sinv, exp_inv)
    t = orc.decode_table(0)
    deq = np.abs(t[q])
    dpad = np.zeros_like(pad)
    dpad[:rows, :cols] = deq
    assert np.all(dpad.reshape(nrb, block_rows, nkb, 128).max(axis=(1, 3)) == 448.0)


def _pow2_scale_by_comparison(a, fm):
    """Largest 2^k (k clamped to [-126, 127]) with a * 2^k <= fm, by exact
    fp64 comparisons (a * 2^k is exact); 1 for a == 0."""
    if a == 0:
        return 1.0
    k = math.floor(math.log2(fm / a))
    while a * 2.0 ** (k + 1) <= fm:
        k += 1
    while a * 2.0 ** k > fm:
        k -= 1
    return 2.0 ** min(max(k, -126), 127)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("block_rows", [1, 128])
@pytest.mark.parametrize("pow2", [False, True])
def test_blockwise_every_code_against_torch(orc, fmt, block_rows, pow2):
    """Every code and scale of the per-block quantizer (the DeepL page §2.3:
    the tensor is cut into blocks, each with its own scale; power-of-two
    block scales follow the Soup page's rowwise rule), recomputed
    independently: the block amax by numpy over the block's finite valid
    elements, s = fmax / amax as an fp32 division (or the largest power of
    two with amax * s <= fmax, by exact comparisons), and the codes by
    torch's float8 conversion of clamp(fp32(x) * s, -fmax, fmax).  The input
    lives in a wider buffer (ld > cols) whose padding holds huge values and
    NaN, so reading a padding element, or indexing the input with the
    output's row pitch, changes a scale or a code.  Blocks differ in
    magnitude by up to 10^+-3; one NaN and one -Inf sit in valid blocks
    (NaN stays NaN, -Inf saturates to -fmax, neither counts in the amax)."""
    rows, cols = (200, 300) if block_rows == 128 else (7, 400)
    ld = cols + 40
    fm = orc.fmax(fmt)
    rng = np.random.default_rng(20 + 4 * fmt + 2 * (block_rows == 128) + pow2)
    nrb, nkb = -(-rows // block_rows), -(-cols // 128)
    xf = rng.standard_normal((rows, cols)).astype(np.float32)
    mult = 10.0 ** rng.integers(-3, 4, (nrb, nkb))
    xf *= np.kron(mult, np.ones((block_rows, 128)))[:rows, :cols].astype(np.float32)
    x = torch.from_numpy(xf).to(torch.bfloat16)
    bits = _bits(x).copy()
    bits[1, 5] = 0x7FC0                      # NaN
    bits[rows - 1, cols - 3] = 0xFF80        # -Inf
    wide = np.full((rows, ld), 0x7F00, np.uint16)   # 1.7e38 in the padding
    wide[:, cols + 1] = 0x7FC0                       # and NaN
    wide[:, :cols] = bits
    q, sinv = orc.quantize_blockwise(wide, fmt, block_rows, pow2=pow2, cols=cols)
    assert q.shape == (rows, cols)

    xv = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    fin = np.where(np.isfinite(xv), np.abs(xv), 0.0)
    pad = np.zeros((nrb * block_rows, nkb * 128), np.float32)
    pad[:rows, :cols] = fin
    bam = pad.reshape(nrb, block_rows, nkb, 128).max(axis=(1, 3))
    if pow2:
        s = np.array([[_pow2_scale_by_comparison(float(a), fm) for a in r] for r in bam], np.float32)
    else:
        s = np.where(bam > 0, np.float32(fm) / np.maximum(bam, np.float32(1e-38)).astype(np.float32),
                     np.float32(1.0)).astype(np.float32)
    s_full = np.kron(s, np.ones((block_rows, 128), np.float32))[:rows, :cols]
    y = np.clip((xv * s_full).astype(np.float32), -fm, fm)
    ref = torch.from_numpy(y).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    nan = np.isnan(xv)
    assert np.all(np.isnan(orc.decode_table(fmt)[q[nan]]))
    assert np.array_equal(q[~nan], ref[~nan])
    assert orc.decode_table(fmt)[q[rows - 1, cols - 3]] == -fm
    inv = (np.float32(1.0) / s).astype(np.float32)
    assert np.array_equal(sinv, inv.T if block_rows == 1 else inv)
    # counts: the NaN and the -Inf are non-finite; saturated = |fp32(x) * s| > fmax (the -Inf among them)
    _, _, (nf, sat) = orc.quantize_blockwise(wide, fmt, block_rows, pow2=pow2, cols=cols, counts=True)
    with np.errstate(invalid="ignore", over="ignore"):
        y = (xv * s_full).astype(np.float32)
    assert nf == 2 and sat == int(np.sum(np.abs(y) > fm)) >= 1


def _counts_reference(xv, s_full, fm):
    """(non-finite inputs, elements with |fp32(x) * s| > fmax): NaN is not
    saturated, +-Inf is."""
    with np.errstate(invalid="ignore", over="ignore"):
        y = (xv * s_full).astype(np.float32)
    return int(np.sum(~np.isfinite(xv))), int(np.sum(np.abs(y) > fm))


@pytest.mark.parametrize("fmt", [0, 1])
def test_rowwise_kv_transpose_counts(orc, fmt):
    """Non-finite and saturation counts of the per-row, per-(b,h)-slice and
    per-column quantizers ("DeepL押注FP8" §5.1: overflow and NaN are the
    failures a run must notice) against numpy on inputs with NaN and +-Inf
    (an element whose fp32(x) * s rounds above fmax counts as saturated on
    both sides); the scales are recomputed independently (numpy maxima, the
    fp32 division or the exact power-of-two comparison)."""
    fm = orc.fmax(fmt)
    rng = np.random.default_rng(70 + fmt)
    xf = rng.standard_normal((24, 96)).astype(np.float32)
    bits = _bits(torch.from_numpy(xf).to(torch.bfloat16)).copy()
    bits[2, 5], bits[7, 1], bits[7, 2], bits[20, 95] = 0x7FC0, 0x7F80, 0xFF80, 0xFFC0
    xv = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    fin = np.where(np.isfinite(xv), np.abs(xv), 0.0)

    def s_of(a, pow2):
        if pow2:
            return np.float32(_pow2_scale_by_comparison(float(a), fm))
        return np.float32(1.0) if a == 0 else np.float32(fm) / np.float32(a)

    for pow2 in (False, True):
        _, _, c = orc.quantize_rowwise(bits, fmt, pow2, counts=True)
        s_full = np.array([s_of(a, pow2) for a in fin.max(axis=1)], np.float32)[:, None] * np.ones((1, 96), np.float32)
        assert c == _counts_reference(xv, s_full, fm)
        _, _, c = orc.quantize_rowwise_transpose(bits, fmt, pow2, counts=True)
        s_full = np.ones((24, 1), np.float32) * np.array([s_of(a, pow2) for a in fin.max(axis=0)], np.float32)[None, :]
        assert c == _counts_reference(xv, s_full, fm)
    kv = bits.reshape(2, 3, 4, 96)
    _, _, c = orc.kv_quant(kv, fmt, counts=True)
    sl = fin.reshape(6, -1).max(axis=1)
    s_full = np.repeat(np.array([s_of(a, False) for a in sl], np.float32), 4 * 96).reshape(24, 96)
    assert c == _counts_reference(xv, s_full, fm) and c[0] == 4


# -------------------------------------------------------------------- GEMM --

def _int_codes(rng, shape, fmt):
    """Codes of small integers (exactly representable): |v| <= 16 (E4M3), <= 8 (E5M2)."""
    top = 16 if fmt == 0 else 8
    vals = rng.integers(-top, top + 1, shape)
    enc = np.vectorize(lambda v: _enc_cache(fmt, int(v)))
    return vals, enc(vals).astype(np.uint8)


_CACHE = {}


def _enc_cache(fmt, v):
    from oracle import oracle
    k = (fmt, v)
    if k not in _CACHE:
        _CACHE[k] = oracle.encode(float(v), fmt)
    return _CACHE[k]


@pytest.mark.parametrize("fa,fb", [(0, 0), (1, 0)])
def test_gemm_integer_special_case(orc, fa, fb):
    """Codes of small integers with unit scales give an exact integer GEMM."""
    rng = np.random.default_rng(7)
    M, N, K = 24, 40, 72
    va, A = _int_codes(rng, (M, K), fa)
    vb, B = _int_codes(rng, (N, K), fb)
    one = np.ones(1, np.float32)
    D, mag = orc.gemm_scaled(A, fa, B, fb, orc.SCALE_TENSOR, one, one)
    exact = va.astype(np.int64) @ vb.astype(np.int64).T
    assert np.array_equal(D, exact.astype(np.float64))
    assert np.array_equal(mag, (np.abs(va) @ np.abs(vb).T).astype(np.float64))


def test_gemm_random_codes_against_numpy(orc):
    """Non-square shapes so a transposed operand fails; rowwise scales."""
    rng = np.random.default_rng(8)
    M, N, K = 19, 33, 100
    t = orc.decode_table(0)
    fin = np.where(np.isfinite(t))[0]
    A = rng.choice(fin, (M, K)).astype(np.uint8)
    B = rng.choice(fin, (N, K)).astype(np.uint8)
    da = rng.uniform(0.5, 2, M).astype(np.float32)
    db = rng.uniform(0.5, 2, N).astype(np.float32)
    D, mag = orc.gemm_scaled(A, 0, B, 0, orc.SCALE_ROW, da, db)
    ref = (t[A] @ t[B].T) * da[:, None].astype(np.float64) * db[None, :].astype(np.float64)
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-9)
    ref_mag = (np.abs(t[A]) @ np.abs(t[B]).T) * da[:, None] * db[None, :]
    assert np.allclose(mag, ref_mag, rtol=1e-12)
    # identity B: D = A's values times the scales
    Bi = np.zeros((K, K), np.uint8)
    Bi[np.arange(K), np.arange(K)] = 0x38
    Di, _ = orc.gemm_scaled(A, 0, Bi, 0, orc.SCALE_TENSOR, np.float32([0.5]), np.float32([1.0]))
    assert np.array_equal(Di, t[A] * 0.5)
    # sampled entries equal the full product
    im = rng.integers(0, M, 50)
    inn = rng.integers(0, N, 50)
    v, mg = orc.gemm_scaled_sampled(A, 0, B, 0, orc.SCALE_ROW, da, db, im, inn)
    assert np.array_equal(v, D[im, inn]) and np.array_equal(mg, mag[im, inn])


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_gemm_f32acc_variant_exact_on_integers_and_within_the_summation_bound(orc, mode):
    """The naive fp32-accumulate variant: on small-integer codes with
    power-of-two scales every sum is exact in fp32, so it equals the fp64
    GEMM (and the int64 matmul); on random codes it stays within the
    classical bound of sequential fp32 summation, (K + 2) u sum|scaled
    products| with u = 2^-24."""
    rng = np.random.default_rng(30 + mode)
    M, N, K = 9, 260, 300
    nkb = -(-K // 128)
    va, A = _int_codes(rng, (M, K), 0)
    vb, B = _int_codes(rng, (N, K), 0)
    if mode == orc.SCALE_TENSOR:
        da, db = np.float32([0.25]), np.float32([2.0])
    elif mode == orc.SCALE_ROW:
        da = np.exp2(rng.integers(-2, 3, M)).astype(np.float32)
        db = np.exp2(rng.integers(-2, 3, N)).astype(np.float32)
    else:
        da = np.exp2(rng.integers(-1, 2, (nkb, M))).astype(np.float32)
        db = np.exp2(rng.integers(-1, 2, (-(-N // 128), nkb))).astype(np.float32)
    D, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
    F = orc.gemm_scaled_f32acc(A, 0, B, 0, mode, da, db)
    assert np.array_equal(F, D)
    if mode != orc.SCALE_BLOCK:
        sa = da if mode == orc.SCALE_ROW else np.repeat(da, M)
        sb = db if mode == orc.SCALE_ROW else np.repeat(db, N)
        exact = (va.astype(np.int64) @ vb.astype(np.int64).T).astype(np.float64)
        assert np.array_equal(D, exact * sa[:, None].astype(np.float64) * sb[None, :].astype(np.float64))
    t = orc.decode_table(0)
    fin = np.where(np.isfinite(t))[0]
    A = rng.choice(fin, (M, K)).astype(np.uint8)
    B = rng.choice(fin, (N, K)).astype(np.uint8)
    if mode == orc.SCALE_BLOCK:
        da = rng.uniform(0.1, 3, (nkb, M)).astype(np.float32)
        db = rng.uniform(0.1, 3, (-(-N // 128), nkb)).astype(np.float32)
    elif mode == orc.SCALE_ROW:
        da = rng.uniform(0.5, 2, M).astype(np.float32)
        db = rng.uniform(0.5, 2, N).astype(np.float32)
    D, mag = orc.gemm_scaled(A, 0, B, 0, mode, da, db)
    F = orc.gemm_scaled_f32acc(A, 0, B, 0, mode, da, db)
    assert np.all(np.abs(F - D) <= (K + 2) * 2.0 ** -24 * mag)
    assert not np.array_equal(F, D)   # the rounding is really fp32


def test_gemm_blockwise_against_numpy(orc):
    """Per-(row, 128-K block) A scales and per-(128x128) B scales, ragged K."""
    rng = np.random.default_rng(9)
    M, N, K = 9, 260, 300
    nkb = -(-K // 128)
    t = orc.decode_table(0)
    fin = np.where(np.isfinite(t))[0]
    A = rng.choice(fin, (M, K)).astype(np.uint8)
    B = rng.choice(fin, (N, K)).astype(np.uint8)
    da = rng.uniform(0.1, 3, (nkb, M)).astype(np.float32)
    db = rng.uniform(0.1, 3, (-(-N // 128), nkb)).astype(np.float32)
    D, _ = orc.gemm_scaled(A, 0, B, 0, orc.SCALE_BLOCK, da, db)
    sa = np.repeat(da.T.astype(np.float64), 128, axis=1)[:, :K]          # [M, K]
    sb = np.repeat(np.repeat(db.astype(np.float64), 128, axis=0)[:N], 128, axis=1)[:, :K]  # [N, K]
    ref = np.einsum("mk,nk->mn", t[A] * sa, t[B] * sb)
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-9)
    # with all scales equal it is the tensorwise GEMM
    D1, _ = orc.gemm_scaled(A, 0, B, 0, orc.SCALE_BLOCK, np.ones_like(da), np.ones_like(db))
    D2, _ = orc.gemm_scaled(A, 0, B, 0, orc.SCALE_TENSOR, np.ones(1, np.float32), np.ones(1, np.float32))
    assert np.allclose(D1, D2, rtol=1e-13)


# --------------------------------------------------------- delayed scaling --

def test_history_constant_amax_and_spike_window(orc):
    """Constant amax: step 0 uses s = 1 (empty history), then s = fmax/amax.
    A spike stays in the window for exactly `len` steps."""
    h = orc.AmaxHistory(16, 0)
    assert h.update(2.0) == 0            # s_0 = 1: 2 * 1 <= 448
    assert h.scale[0] == np.float32(224.0)
    for _ in range(5):
        assert h.update(2.0) == 0
        assert h.scale[0] == np.float32(224.0)
    assert h.update(16.0) == 1           # spike: 16 * 224 > 448 -> saturation flag
    assert h.scale[0] == np.float32(28.0)
    for i in range(15):
        h.update(2.0)
        assert h.scale[0] == np.float32(28.0), i      # spike still in the window
    h.update(2.0)
    assert h.scale[0] == np.float32(224.0)            # 16 steps later it has left
    assert h.scale_inv[0] == np.float32(1.0) / np.float32(224.0)
    assert h.pos[0] == (6 + 1 + 16) % 16


def test_history_checkpoint_resume(orc):
    """The state is (history, pos, scale): save at step 8 and resume."""
    amaxes = np.random.default_rng(1).uniform(0.1, 5, 24).astype(np.float32)
    a = orc.AmaxHistory(16, 1)
    for v in amaxes:
        a.update(v)
    b = orc.AmaxHistory(16, 1)
    for v in amaxes[:8]:
        b.update(v)
    saved = (b.history.copy(), b.pos.copy(), b.scale.copy(), b.scale_inv.copy())
    c = orc.AmaxHistory(16, 1)
    c.history[:], c.pos[:], c.scale[:], c.scale_inv[:] = saved
    for v in amaxes[8:]:
        c.update(v)
    assert np.array_equal(a.history, c.history) and a.pos[0] == c.pos[0]
    assert a.scale[0] == c.scale[0] and a.scale_inv[0] == c.scale_inv[0]
    assert a.scale[0] == np.float32(57344.0) / np.float32(amaxes[-16:].max())


# ---------------------------------------------------------------- KV cache --

def test_kv_round_trip(orc):
    """Per-(b, h) scales; the round trip stays within half an E4M3 step plus
    the bf16 rounding; K8 memory halves (1 byte per element)."""
    x = inputs.normal_bf16((2, 3, 64, 128), 1.0, seed=10)
    bits = _bits(x)
    q, sinv = orc.kv_quant(bits)
    assert q.dtype == np.uint8 and q.nbytes * 2 == bits.nbytes
    xf = x.float().numpy().reshape(6, -1)
    for i in range(6):
        assert sinv[i] == np.float32(1.0) / (np.float32(448.0) / np.float32(np.abs(xf[i]).max()))
        qi, si, *_ = orc.quantize_tensorwise(bits.reshape(6, -1)[i], 0)
        assert np.array_equal(q.reshape(6, -1)[i], qi.ravel()) and si == sinv[i]
    back = orc.kv_dequant(q, sinv)
    bf = torch.from_numpy(back.view(np.int16)).view(torch.bfloat16).float().numpy().reshape(6, -1)
    tiny = 2.0 ** -9 * sinv[:, None]
    assert np.all(np.abs(bf - xf) <= (2.0 ** -4 + 2.0 ** -8) * np.abs(xf) + tiny)
    # dequant equals bf16(decoded * d) computed by torch's own bf16 cast
    t = orc.decode_table(0).astype(np.float32)
    y = (t[q.reshape(6, -1)] * sinv[:, None]).astype(np.float32)
    lib = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(back.reshape(6, -1), lib)


def test_grouped_gemm_is_the_per_group_gemm(orc):
    """The grouped oracle equals numpy's per-group products (empty groups and
    ragged sizes included) -- catches a swapped expert index or row offset."""
    rng = np.random.default_rng(21)
    sizes = [0, 5, 3, 0, 7]
    off = np.concatenate([[0], np.cumsum(sizes)])
    G, N, K = len(sizes), 6, 40
    t = orc.decode_table(0)
    fin = np.where(np.isfinite(t))[0]
    A = rng.choice(fin, (off[-1], K)).astype(np.uint8)
    B = rng.choice(fin, (G, N, K)).astype(np.uint8)
    da = rng.uniform(0.5, 2, G).astype(np.float32)
    db = rng.uniform(0.5, 2, G).astype(np.float32)
    D, _ = orc.gemm_grouped(A, 0, B, 0, off, orc.SCALE_TENSOR, da, db)
    for e in range(G):
        r0, r1 = off[e], off[e + 1]
        ref = (t[A[r0:r1]] @ t[B[e]].T) * np.float64(da[e]) * np.float64(db[e])
        assert np.allclose(D[r0:r1], ref, rtol=1e-12, atol=1e-12)
    dra = rng.uniform(0.5, 2, off[-1]).astype(np.float32)
    drb = rng.uniform(0.5, 2, G * N).astype(np.float32)
    D2, _ = orc.gemm_grouped(A, 0, B, 0, off, orc.SCALE_ROW, dra, drb)
    for e in range(G):
        r0, r1 = off[e], off[e + 1]
        ref = (t[A[r0:r1]] @ t[B[e]].T) * dra[r0:r1, None] * drb.reshape(G, N)[e][None, :]
        assert np.allclose(D2[r0:r1], ref, rtol=1e-12, atol=1e-12)


def test_scale_stats_closed_forms(orc):
    """Health check of scale factors (DeepL page §6.2): min / max / mean over
    the valid scales, step changes against a previous snapshot, invalid ones."""
    s = np.array([1.0, 4.0, 2.0, 0.5, np.nan, -1.0, 0.0, np.inf, 8.0], np.float32)
    st, c = orc.scale_stats(s)
    assert list(st) == [0.5, 8.0, np.float32(15.5 / 5)] and list(c) == [0, 4]
    prev = np.array([1.0, 1.0, 2.0, 0.25, 1.0, 1.0, 1.0, 1.0, 64.0], np.float32)
    st, c = orc.scale_stats(s, prev, 3.0)
    assert list(c) == [2, 4]        # 4/1 > 3 and 64/8 > 3; 0.5/0.25 = 2 is not
    st, c = orc.scale_stats(np.zeros(0, np.float32))
    assert list(st) == [0, 0, 0] and list(c) == [0, 0]
    rng = np.random.default_rng(0)
    v = (10.0 ** rng.uniform(-3, 3, 10000)).astype(np.float32)
    st, c = orc.scale_stats(v)
    assert st[0] == v.min() and st[1] == v.max() and np.isclose(st[2], v.astype(np.float64).mean(), rtol=1e-7)


@pytest.mark.parametrize("fmt", [0, 1])
def test_paged_kv_write_and_gather(orc, fmt):
    """Paged FP8 KV cache (block KV cache of "ms-swift全链路能力解析：训练、推理、评测、量化与部署一体化解决方案"; FP8 KV of the
    DeepL page §3.1), against torch built independently: per (token, head) the
    amax by torch, s = fmax / amax as one fp32 division, the cast by torch's
    float8 conversion of the clamped product, the read-back by torch's bf16
    cast.  Pages are scattered through a shuffled block table; padding slots
    (-1) write nothing; positions past a sequence's length read as 0."""
    rng = np.random.default_rng(40 + fmt)
    H, Dh, bs, NB = 3, 32, 16, 12
    fm = np.float32(orc.fmax(fmt))
    lens = np.array([37, 5, 0, 16], np.int32)
    B, mb = len(lens), 4
    table = np.full((B, mb), -1, np.int32)
    perm = rng.permutation(NB).astype(np.int32)
    k = 0
    for b in range(B):
        for j in range((lens[b] + bs - 1) // bs):
            table[b, j] = perm[k]
            k += 1
    # token list: every position of every sequence plus two padding tokens
    seq_of = np.concatenate([np.full(n, b) for b, n in enumerate(lens)] + [[0, 0]]).astype(np.int64)
    pos_of = np.concatenate([np.arange(n) for n in lens] + [[0, 0]]).astype(np.int64)
    T = len(seq_of)
    slot = table[seq_of, pos_of // bs].astype(np.int64) * bs + pos_of % bs
    slot[-2:] = -1
    x = inputs.normal_bf16((T, H, Dh), 3.0, seed=50 + fmt)
    x.view(-1)[7] = 0.0
    x[1, 1] = 0.0                                   # an all-zero row: scale 1
    c0 = rng.integers(0, 256, (NB, bs, H, Dh)).astype(np.uint8)   # stale pages
    s0 = np.full((NB, bs, H), 7.0, np.float32)
    cache, sc = orc.paged_kv_write(_bits(x), slot, c0, s0, fmt)

    xf = x.float()
    amax = xf.abs().amax(dim=-1)                    # [T, H]
    s = torch.where(amax > 0, torch.tensor(float(fm)) / amax, torch.tensor(1.0))
    y = (xf * s[..., None]).clamp(-float(fm), float(fm))
    qref = y.to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
    sinv = (1.0 / s).numpy().astype(np.float32)
    written = np.zeros(NB * bs, bool)
    for t in range(T):
        if slot[t] < 0:
            continue
        written[slot[t]] = True
        assert np.array_equal(cache.reshape(NB * bs, H, Dh)[slot[t]], qref[t]), t
        assert np.array_equal(sc.reshape(NB * bs, H)[slot[t]], sinv[t]), t
    assert np.array_equal(cache.reshape(NB * bs, H, Dh)[~written], c0.reshape(NB * bs, H, Dh)[~written])
    assert np.all(sc.reshape(NB * bs, H)[~written] == 7.0)

    S_out = 40
    out = orc.paged_kv_gather(cache, sc, table, lens, S_out, fmt)
    deq = torch.from_numpy(qref).view(TORCH_FP8[fmt]).float()
    ref = (deq * torch.from_numpy(sinv)[..., None]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    for b in range(B):
        for t in range(S_out):
            if t < lens[b]:
                i = int(np.flatnonzero((seq_of[:-2] == b) & (pos_of[:-2] == t))[0])
                assert np.array_equal(out[b, t], ref[i]), (b, t)
            else:
                assert not out[b, t].any(), (b, t)


def _bf16_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("pow2", [True, False])
def test_rowwise_transpose_per_column(orc, fmt, pow2):
    """Rowwise quantization of x^T (the Soup page's rowwise recipes applied to
    the backward GEMMs' transposed operands), built independently: column
    amax by torch over the finite entries, the scale from its closed form,
    the cast by torch's float8 conversion of the clamped product."""
    rows, cols = 45, 70
    x = inputs.outlier_activations_bf16((rows, cols), seed=60 + fmt, frac=0.02)
    bits = _bits(x).copy()
    bits[3, 5] = 0x7FC0            # NaN: skipped by the amax, cast to NaN
    bits[:, 9] = 0                 # an all-zero column: scale 1
    qT, sinv = orc.quantize_rowwise_transpose(bits, fmt, pow2)
    assert qT.shape == (cols, rows) and sinv.shape == (cols,)
    xf = _bf16_f64(bits)
    fm = orc.fmax(fmt)
    for c in range(cols):
        col = xf[:, c]
        a = np.max(np.abs(col[np.isfinite(col)]), initial=0.0)
        if a == 0:
            s = 1.0
        elif pow2:
            k = math.floor(math.log2(fm / a))
            while a * 2.0 ** (k + 1) <= fm:   # exact fix-ups of the float log
                k += 1
            while a * 2.0 ** k > fm:
                k -= 1
            s = 2.0 ** max(-126, min(127, k))
        else:
            s = float(np.float32(np.float32(fm) / np.float32(a)))
        assert sinv[c] == np.float32(1.0) / np.float32(s), c
        y = torch.from_numpy((col.astype(np.float32) * np.float32(s)).astype(np.float32))
        ref = y.clamp(-fm, fm).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()
        fin = np.isfinite(col)
        assert np.array_equal(qT[c][fin], ref[fin]), c
        assert np.all(np.isin(qT[c][~fin], [0x7F, 0xFF, 0x7D, 0x7E, 0xFD, 0xFE]))
    # the same numbers as the rowwise quantizer applied to the transpose
    q2, s2 = orc.quantize_rowwise(np.ascontiguousarray(bits.T), fmt, pow2)
    assert np.array_equal(q2, qT) and np.array_equal(s2, sinv)


def test_bf16_wgrad_against_numpy(orc):
    """dW = dY^T X from the bf16 tensors as stored (token-major), against
    numpy's fp64 matmul of the same values on a non-square shape (a swapped
    operand or index fails it), and exactly on small integers."""
    T, M, N = 37, 24, 40
    dy = _bits(inputs.lognormal_grads_bf16((T, M), seed=70))
    x = _bits(inputs.normal_bf16((T, N), 1.0, seed=71))
    D, mag = orc.gemm_bf16_wgrad(dy, x)
    ref = _bf16_f64(dy).T @ _bf16_f64(x)
    assert D.shape == (M, N)
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(mag, np.abs(_bf16_f64(dy)).T @ np.abs(_bf16_f64(x)), rtol=1e-12)
    rng = np.random.default_rng(72)
    ai = rng.integers(-8, 9, (T, M)).astype(np.float32)
    bi = rng.integers(-8, 9, (T, N)).astype(np.float32)
    abits = _bits(torch.from_numpy(ai).to(torch.bfloat16))
    bbits = _bits(torch.from_numpy(bi).to(torch.bfloat16))
    Di, _ = orc.gemm_bf16_wgrad(abits, bbits)
    assert np.array_equal(Di, (ai.astype(np.int64).T @ bi.astype(np.int64)).astype(np.float64))
