"""CPU oracle for the FP8 scaled-quantization path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

This is a thin ctypes wrapper over ``fp8_oracle.c`` (plain C, fp64 sums,
fp32 where the method fixes fp32).  Arrays are numpy: bf16 tensors are passed
as their raw ``uint16`` bit patterns, FP8 tensors as ``uint8`` codes.
Which page and section each function follows is stated in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

E4M3 = 0
E5M2 = 1
SCALE_TENSOR = 0
SCALE_ROW = 1
SCALE_BLOCK = 2


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE arithmetic: no fast-math, no FMA
    contraction) into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        F = ctypes.c_float
        L.orc_decode.restype = ctypes.c_double
        L.orc_decode.argtypes = [ctypes.c_uint8, I]
        L.orc_encode.restype = ctypes.c_uint8
        L.orc_encode.argtypes = [F, I]
        L.orc_fmax.restype = ctypes.c_double
        L.orc_fmax.argtypes = [I]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_bf16.argtypes = [F]
        L.orc_amax_bf16.restype = F
        L.orc_amax_bf16.argtypes = [P, I64, P]
        L.orc_scale_from_amax.restype = F
        L.orc_scale_from_amax.argtypes = [F, I]
        L.orc_scale_pow2_from_amax.restype = F
        L.orc_scale_pow2_from_amax.argtypes = [F, I]
        L.orc_inverse.restype = F
        L.orc_inverse.argtypes = [F]
        L.orc_quantize_tensorwise.restype = None
        L.orc_quantize_tensorwise.argtypes = [P, I64, I64, I, P, I, P, P, P, P]
        L.orc_quantize_rowwise.restype = None
        L.orc_quantize_rowwise.argtypes = [P, I64, I64, I64, I, I, P, P, P]
        L.orc_quantize_blockwise.restype = None
        L.orc_quantize_blockwise.argtypes = [P, I64, I64, I64, I, I, I, P, P, P]
        L.orc_gemm_scaled.restype = None
        L.orc_gemm_scaled.argtypes = [P, I, P, I, I64, I64, I64, I, P, P, P, P]
        L.orc_gemm_scaled_sampled.restype = None
        L.orc_gemm_scaled_sampled.argtypes = [P, I, P, I, I64, I64, I64, I, P, P, P, P, I64, P, P]
        L.orc_gemm_scaled_f32acc_sampled.restype = None
        L.orc_gemm_scaled_f32acc_sampled.argtypes = [P, I, P, I, I64, I64, I64, I, P, P, P, P, I64, P]
        L.orc_amax_history_update.restype = None
        L.orc_amax_history_update.argtypes = [P, P, I, F, I, P, P, P]
        L.orc_kv_quant.restype = None
        L.orc_kv_quant.argtypes = [P, I64, I64, I, P, P, P]
        L.orc_kv_dequant.restype = None
        L.orc_kv_dequant.argtypes = [P, P, I64, I64, I, P]
        L.orc_paged_kv_write.restype = None
        L.orc_paged_kv_write.argtypes = [P, P, I64, I64, I64, I64, I, P, P]
        L.orc_paged_kv_gather.restype = None
        L.orc_paged_kv_gather.argtypes = [P, P, P, P, I64, I64, I64, I64, I64, I64, I64, I, P]
        L.orc_quantize_rowwise_transpose.restype = None
        L.orc_quantize_rowwise_transpose.argtypes = [P, I64, I64, I64, I, I, P, P, P]
        L.orc_gemm_bf16_wgrad_sampled.restype = None
        L.orc_gemm_bf16_wgrad_sampled.argtypes = [P, P, I64, I64, I64, P, P, I64, P, P]
        L.orc_scale_stats.restype = None
        L.orc_scale_stats.argtypes = [P, P, I64, F, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u16(x) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return x


# ------------------------------------------------------------------ formats --

def decode(code: int, fmt: int) -> float:
    return lib().orc_decode(code, fmt)


def decode_table(fmt: int) -> np.ndarray:
    """All 256 code values of a format (fp64), index == code."""
    return np.array([decode(c, fmt) for c in range(256)], dtype=np.float64)


def encode(y: float, fmt: int) -> int:
    return int(lib().orc_encode(float(y), fmt))


def encode_array(y: np.ndarray, fmt: int) -> np.ndarray:
    y = np.asarray(y, dtype=np.float32).ravel()
    return np.array([encode(v, fmt) for v in y], dtype=np.uint8)


def fmax(fmt: int) -> float:
    return lib().orc_fmax(fmt)


def f32_to_bf16(f: float) -> int:
    return int(lib().orc_f32_to_bf16(float(f)))


# ------------------------------------------------------------ amax / scale --

def amax(x_bits: np.ndarray) -> tuple[float, int]:
    x = _u16(x_bits)
    nf = ctypes.c_uint64(0)
    a = lib().orc_amax_bf16(_p(x), x.size, ctypes.byref(nf))
    return float(np.float32(a)), int(nf.value)


def scale_from_amax(a: float, fmt: int) -> float:
    return float(np.float32(lib().orc_scale_from_amax(a, fmt)))


def scale_pow2_from_amax(a: float, fmt: int) -> float:
    return float(np.float32(lib().orc_scale_pow2_from_amax(a, fmt)))


def inverse(s: float) -> float:
    return float(np.float32(lib().orc_inverse(s)))


# ---------------------------------------------------------------- quantize --

def quantize_tensorwise(x_bits: np.ndarray, fmt: int, scale_in: float | None = None,
                        transpose_out: bool = False):
    """Returns (q [rows, cols] or [cols, rows], scale_inv, amax, (nonfinite, saturated))."""
    x = _u16(x_bits)
    rows, cols = (1, x.size) if x.ndim == 1 else x.shape
    q = np.empty((cols, rows) if transpose_out else (rows, cols), dtype=np.uint8)
    sinv = np.zeros(1, np.float32)
    am = np.zeros(1, np.float32)
    counts = np.zeros(2, np.uint64)
    s_in = None if scale_in is None else np.array([scale_in], np.float32)
    lib().orc_quantize_tensorwise(_p(x), rows, cols, fmt, None if s_in is None else _p(s_in),
                                  int(transpose_out), _p(q), _p(sinv), _p(am), _p(counts))
    return q, float(sinv[0]), float(am[0]), (int(counts[0]), int(counts[1]))


def _rows_cols_ld(x: np.ndarray, cols):
    """A [rows, ld] array read as [rows, cols] rows of a wider buffer."""
    rows, ld = x.shape
    cols = ld if cols is None else int(cols)
    assert 0 <= cols <= ld
    return rows, cols, ld


def _with_counts(res, counts, want):
    return (*res, (int(counts[0]), int(counts[1]))) if want else res


def quantize_rowwise(x_bits: np.ndarray, fmt: int, pow2: bool = True, cols=None, counts: bool = False):
    """x [rows, ld] (the first ``cols`` columns of each row are the tensor;
    cols=None: all) -> (q [rows, cols], scale_inv [rows]) and, with
    counts=True, (non-finite inputs, saturated elements)."""
    x = _u16(x_bits)
    rows, cols, ld = _rows_cols_ld(x, cols)
    q = np.empty((rows, cols), np.uint8)
    sinv = np.empty(rows, np.float32)
    c = np.zeros(2, np.uint64)
    lib().orc_quantize_rowwise(_p(x), rows, cols, ld, fmt, int(pow2), _p(q), _p(sinv), _p(c))
    return _with_counts((q, sinv), c, counts)


def quantize_blockwise(x_bits: np.ndarray, fmt: int, block_rows: int, pow2: bool = False, cols=None,
                       counts: bool = False):
    """x [rows, ld] (the first ``cols`` columns of each row are the tensor;
    cols=None: all) -> (q [rows, cols], scales) and, with counts=True,
    (non-finite inputs, saturated elements).  block_rows 1: scales
    [ceil(cols/128), rows]; block_rows 128: scales [ceil(rows/128), ceil(cols/128)]."""
    x = _u16(x_bits)
    rows, cols, ld = _rows_cols_ld(x, cols)
    nkb = (cols + 127) // 128
    q = np.empty((rows, cols), np.uint8)
    if block_rows == 1:
        sinv = np.empty((nkb, rows), np.float32)
    else:
        sinv = np.empty(((rows + block_rows - 1) // block_rows, nkb), np.float32)
    c = np.zeros(2, np.uint64)
    lib().orc_quantize_blockwise(_p(x), rows, cols, ld, fmt, block_rows, int(pow2), _p(q), _p(sinv), _p(c))
    return _with_counts((q, sinv), c, counts)


# -------------------------------------------------------------------- GEMM --

def gemm_scaled(A: np.ndarray, fa: int, B: np.ndarray, fb: int, mode: int,
                da: np.ndarray, db: np.ndarray):
    """Full reference D (fp64 [M, N]) and magnitude mag (fp64 [M, N])."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    da = np.ascontiguousarray(da, np.float32)
    db = np.ascontiguousarray(db, np.float32)
    D = np.empty((M, N), np.float64)
    mag = np.empty((M, N), np.float64)
    lib().orc_gemm_scaled(_p(A), fa, _p(B), fb, M, N, K, mode, _p(da), _p(db), _p(D), _p(mag))
    return D, mag


def gemm_scaled_sampled(A: np.ndarray, fa: int, B: np.ndarray, fb: int, mode: int,
                        da: np.ndarray, db: np.ndarray, idx_m: np.ndarray, idx_n: np.ndarray):
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    M, K = A.shape
    N, _ = B.shape
    da = np.ascontiguousarray(da, np.float32)
    db = np.ascontiguousarray(db, np.float32)
    im = np.ascontiguousarray(idx_m, np.int64)
    inn = np.ascontiguousarray(idx_n, np.int64)
    val = np.empty(im.size, np.float64)
    mag = np.empty(im.size, np.float64)
    lib().orc_gemm_scaled_sampled(_p(A), fa, _p(B), fb, M, N, K, mode, _p(da), _p(db),
                                  _p(im), _p(inn), im.size, _p(val), _p(mag))
    return val, mag


def gemm_scaled_f32acc_sampled(A: np.ndarray, fa: int, B: np.ndarray, fb: int, mode: int,
                               da: np.ndarray, db: np.ndarray, idx_m: np.ndarray, idx_n: np.ndarray):
    """The naive sequential fp32-accumulate GEMM at the listed outputs (fp64
    values of fp32 results, before any bf16 rounding)."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    M, K = A.shape
    N, _ = B.shape
    da = np.ascontiguousarray(da, np.float32)
    db = np.ascontiguousarray(db, np.float32)
    im = np.ascontiguousarray(idx_m, np.int64)
    inn = np.ascontiguousarray(idx_n, np.int64)
    val = np.empty(im.size, np.float64)
    lib().orc_gemm_scaled_f32acc_sampled(_p(A), fa, _p(B), fb, M, N, K, mode, _p(da), _p(db),
                                         _p(im), _p(inn), im.size, _p(val))
    return val


def gemm_scaled_f32acc(A: np.ndarray, fa: int, B: np.ndarray, fb: int, mode: int,
                       da: np.ndarray, db: np.ndarray):
    """Full [M, N] naive fp32-accumulate GEMM (fp64 values of fp32 results)."""
    M, N = np.asarray(A).shape[0], np.asarray(B).shape[0]
    im = np.repeat(np.arange(M), N)
    inn = np.tile(np.arange(N), M)
    return gemm_scaled_f32acc_sampled(A, fa, B, fb, mode, da, db, im, inn).reshape(M, N)


def gemm_grouped(A: np.ndarray, fa: int, B: np.ndarray, fb: int, offsets, mode: int,
                 da: np.ndarray, db: np.ndarray):
    """Grouped (mixture-of-experts) GEMM: rows [offsets[e], offsets[e+1]) of A
    times expert e's weight B[e] ([G, N, K]); tensor mode takes da[e], db[e],
    row mode da[row], db[e, col].  Each group is the plain scaled GEMM above
    ("DeepL押注FP8：…" §3.2: one GEMM per expert's token group)."""
    G, N, K = B.shape
    M = A.shape[0]
    D = np.zeros((M, N), np.float64)
    mag = np.zeros((M, N), np.float64)
    for e in range(G):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        if mode == SCALE_TENSOR:
            sa, sb = np.float32([da[e]]), np.float32([db[e]])
        else:
            sa, sb = np.ascontiguousarray(da[r0:r1]), np.ascontiguousarray(np.asarray(db).reshape(G, N)[e])
        D[r0:r1], mag[r0:r1] = gemm_scaled(A[r0:r1], fa, B[e], fb, mode, sa, sb)
    return D, mag


# --------------------------------------------------------- delayed scaling --

class AmaxHistory:
    """Host-side delayed-scaling state: history ring, position, scale."""

    def __init__(self, length: int, fmt: int):
        self.history = np.zeros(length, np.float32)
        self.pos = np.zeros(1, np.int32)
        self.scale = np.ones(1, np.float32)
        self.scale_inv = np.ones(1, np.float32)
        self.fmt = fmt

    def update(self, amax_cur: float) -> int:
        sat = np.zeros(1, np.uint32)
        lib().orc_amax_history_update(_p(self.history), _p(self.pos), self.history.size,
                                      float(amax_cur), self.fmt, _p(self.scale),
                                      _p(self.scale_inv), _p(sat))
        return int(sat[0])


# ---------------------------------------------------------------- KV cache --

def kv_quant(x_bits: np.ndarray, fmt: int = E4M3, counts: bool = False):
    """x [B, H, S, Dh] bf16 bits -> (q same shape, scale_inv [B*H]) and, with
    counts=True, (non-finite inputs, saturated elements)."""
    x = _u16(x_bits)
    B, H, S, Dh = x.shape
    q = np.empty(x.shape, np.uint8)
    sinv = np.empty(B * H, np.float32)
    c = np.zeros(2, np.uint64)
    lib().orc_kv_quant(_p(x), B * H, S * Dh, fmt, _p(q), _p(sinv), _p(c))
    return _with_counts((q, sinv), c, counts)


def kv_dequant(q: np.ndarray, scale_inv: np.ndarray, fmt: int = E4M3) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    B, H, S, Dh = q.shape
    sinv = np.ascontiguousarray(scale_inv, np.float32)
    out = np.empty(q.shape, np.uint16)
    lib().orc_kv_dequant(_p(q), _p(sinv), B * H, S * Dh, fmt, _p(out))
    return out


# ------------------------------------------ backward operands, wgrad GEMM --

def quantize_rowwise_transpose(x_bits: np.ndarray, fmt: int, pow2: bool = True, counts: bool = False):
    """x [rows, cols] -> (qT [cols, rows], scale_inv [cols]): rowwise
    quantization of x^T (one scale per column of x); with counts=True also
    (non-finite inputs, saturated elements)."""
    x = _u16(x_bits)
    rows, cols = x.shape
    qT = np.empty((cols, rows), np.uint8)
    sinv = np.empty(cols, np.float32)
    c = np.zeros(2, np.uint64)
    lib().orc_quantize_rowwise_transpose(_p(x), rows, cols, cols, fmt, int(pow2), _p(qT), _p(sinv), _p(c))
    return _with_counts((qT, sinv), c, counts)


def gemm_bf16_wgrad_sampled(dY_bits: np.ndarray, X_bits: np.ndarray, idx_m, idx_n):
    """dW[m, n] = sum_t dY[t, m] X[t, n] (fp64) at the sampled (m, n)."""
    dy = _u16(dY_bits)
    x = _u16(X_bits)
    T, M = dy.shape
    T2, N = x.shape
    assert T == T2
    im = np.ascontiguousarray(idx_m, np.int64)
    inn = np.ascontiguousarray(idx_n, np.int64)
    val = np.empty(im.size, np.float64)
    mag = np.empty(im.size, np.float64)
    lib().orc_gemm_bf16_wgrad_sampled(_p(dy), _p(x), T, M, N, _p(im), _p(inn), im.size, _p(val), _p(mag))
    return val, mag


def gemm_bf16_wgrad(dY_bits: np.ndarray, X_bits: np.ndarray):
    """Full dW [M, N] and magnitude (fp64)."""
    T, M = np.asarray(dY_bits).shape
    N = np.asarray(X_bits).shape[1]
    im = np.repeat(np.arange(M), N)
    inn = np.tile(np.arange(N), M)
    v, g = gemm_bf16_wgrad_sampled(dY_bits, X_bits, im, inn)
    return v.reshape(M, N), g.reshape(M, N)


# --------------------------------------------------------- paged KV cache --

def paged_kv_write(x_bits: np.ndarray, slot: np.ndarray, cache: np.ndarray, scale_cache: np.ndarray,
                   fmt: int = E4M3):
    """x [T, H, Dh] bf16 bits written into copies of cache [num_blocks,
    block_size, H, Dh] / scale_cache [num_blocks, block_size, H]; returns them."""
    x = _u16(x_bits)
    T, H, Dh = x.shape
    sl = np.ascontiguousarray(slot, np.int64)
    c = np.array(cache, np.uint8, copy=True, order="C")
    sc = np.array(scale_cache, np.float32, copy=True, order="C")
    nslots = c.shape[0] * c.shape[1]
    assert c.shape[2:] == (H, Dh) and sc.shape == c.shape[:3] and sl.shape == (T,)
    lib().orc_paged_kv_write(_p(x), _p(sl), T, H, Dh, nslots, fmt, _p(c), _p(sc))
    return c, sc


def paged_kv_gather(cache: np.ndarray, scale_cache: np.ndarray, block_table: np.ndarray,
                    seq_lens: np.ndarray, S_out: int, fmt: int = E4M3) -> np.ndarray:
    """Dequantized [B, S_out, H, Dh] bf16 bits of each sequence's tokens."""
    c = np.ascontiguousarray(cache, np.uint8)
    sc = np.ascontiguousarray(scale_cache, np.float32)
    bt = np.ascontiguousarray(block_table, np.int32)
    sl = np.ascontiguousarray(seq_lens, np.int32)
    NB, bs, H, Dh = c.shape
    B, mb = bt.shape
    out = np.empty((B, S_out, H, Dh), np.uint16)
    lib().orc_paged_kv_gather(_p(c), _p(sc), _p(bt), _p(sl), B, mb, H, Dh, bs, NB, S_out, fmt, _p(out))
    return out


# ------------------------------------------------------- scale health check --

def scale_stats(scales: np.ndarray, prev: np.ndarray | None = None, jump_ratio: float = 4.0):
    """(min, max, mean) over the finite positive scales, (jumps, invalid)."""
    s = np.ascontiguousarray(scales, np.float32)
    p = None if prev is None else np.ascontiguousarray(prev, np.float32)
    st = np.zeros(3, np.float32)
    c = np.zeros(2, np.uint32)
    lib().orc_scale_stats(_p(s), None if p is None else _p(p), s.size, float(jump_ratio), _p(st), _p(c))
    return st, c
