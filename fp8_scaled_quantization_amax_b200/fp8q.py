"""Python binding of the C ABI in ``include/fp8q.h`` (``libfp8q.so``).

Argument marshalling only: every function here checks tensor dtypes, devices
and contiguity, passes raw device pointers and the current CUDA stream to the
library function of the same name, and raises :class:`Fp8Error` on a non-OK
status.  All arithmetic runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback -- if the library is missing the first call raises.

The ``quantize_*`` / ``gemm`` / ``kv_*`` helpers at the bottom only allocate
the outputs with torch (device memory) and call the raw entry points.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

E4M3 = 0
E5M2 = 1
SCALE_TENSOR = 0
SCALE_ROW = 1
SCALE_BLOCK = 2
FMAX = {E4M3: 448.0, E5M2: 57344.0}

# every symbol the header declares, with (restype, argtypes)
_P, _I64, _I, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_S = ctypes.c_int
SIGNATURES = {
    "fp8_status_string": (ctypes.c_char_p, [_S]),
    "fp8_amax": (_S, [_P, _I64, _P, _P, _P]),
    "fp8_quantize_tensorwise": (_S, [_P, _I64, _I64, _I, _P, _P, _I, _P, _P, _P, _P]),
    "fp8_quantize_rowwise": (_S, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P]),
    "fp8_quantize_blockwise": (_S, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P]),
    "fp8_gemm_scaled": (_S, [_P, _I, _P, _I, _I64, _I64, _I64, _I, _P, _P, _P, _I64, _P, ctypes.c_size_t, _P]),
    "fp8_gemm_workspace_size": (_S, [_I64, _I64, _I64, _I, _P]),
    "fp8_gemm_grouped": (_S, [_P, _I, _P, _I, _I, _P, _I64, _I64, _I64, _I, _P, _P, _P, _I64, _P]),
    "fp8_gemm_scaled_noalloc": (_S, [_P, _I, _P, _I, _I64, _I64, _I64, _I, _P, _P, _P, _I64, _P]),
    "fp8_gemm_block_requant": (_S, [_P, _I, _P, _I, _I64, _I64, _I64, _P, _P, _P, _I64, _I, _P, _P, _P, _P]),
    "fp8_amax_history_update": (_S, [_P, _P, _I, _P, _I, _P, _P, _P, _P]),
    "fp8_kv_quant": (_S, [_P, _I64, _I64, _I64, _I64, _I, _P, _P, _P, _P]),
    "fp8_kv_dequant": (_S, [_P, _P, _I64, _I64, _I64, _I64, _I, _P, _P]),
    "fp8_quantize_rowwise_pair": (_S, [_P, _I64, _I64, _P, _P, _P, _I64, _I64, _P, _P, _I64, _I, _I, _P, _P]),
    "fp8_quantize_blockwise_e8m0": (_S, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P]),
    "fp8_quantize_rowwise_transpose": (_S, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _P, _P, _P]),
    "fp8_gemm_bf16_wgrad": (_S, [_P, _P, _I64, _I64, _I64, _I64, _I64, _P, _I64, _I, _P]),
    "fp8_gemm_block_e8m0": (_S, [_P, _I, _P, _I, _I64, _I64, _I64, _P, _P, _P, _I64, _P]),
    "fp8_gemm_block_e8m0_requant": (_S, [_P, _I, _P, _I, _I64, _I64, _I64, _P, _P, _P, _I64, _I, _P, _P, _P, _P]),
    "fp8_paged_kv_write": (_S, [_P, _P, _I64, _I64, _I64, _I64, _I, _P, _P, _P]),
    "fp8_paged_kv_gather": (_S, [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64, _I64, _I, _P, _P]),
    "fp8_scale_stats": (_S, [_P, _P, _I64, _P, _I64, _F, _P, _P, _P]),
    "fp8_device_error": (_S, [_P, _I]),
}


class Fp8Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().fp8_status_string(status)
        super().__init__(f"{fn} failed: {msg.decode() if msg else status}")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load ``libfp8q.so`` (built in-tree by ``build.py``); raise if absent."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m fp8_scaled_quantization_amax_b200.build` (no fallback exists)")
                L = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, status):
    if status != 0:
        raise Fp8Error(name, status)


def _dev(t, dtype, what):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{what}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")


# ------------------------------------------------------- raw entry points --

def fp8_amax(x, amax, counts=None, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(amax, torch.float32, "amax"); _dev(counts, torch.int32, "counts")
    _check("fp8_amax", lib().fp8_amax(_ptr(x), x.numel(), _ptr(amax), _ptr(counts), _stream(stream)))


def fp8_quantize_tensorwise(x, rows, cols, fmt, scale_in, q, transpose_out, scale_inv_out,
                            amax_out=None, counts=None, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(q, torch.uint8, "q")
    _dev(scale_in, torch.float32, "scale_in"); _dev(scale_inv_out, torch.float32, "scale_inv_out")
    _dev(amax_out, torch.float32, "amax_out"); _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_tensorwise", lib().fp8_quantize_tensorwise(
        _ptr(x), rows, cols, fmt, _ptr(scale_in), _ptr(q), int(transpose_out), _ptr(scale_inv_out),
        _ptr(amax_out), _ptr(counts), _stream(stream)))


def fp8_quantize_rowwise(x, rows, cols, ld, fmt, pow2, q, scale_inv, counts=None, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(q, torch.uint8, "q"); _dev(scale_inv, torch.float32, "scale_inv")
    _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_rowwise", lib().fp8_quantize_rowwise(
        _ptr(x), rows, cols, ld, fmt, int(pow2), _ptr(q), _ptr(scale_inv), _ptr(counts), _stream(stream)))


def fp8_quantize_blockwise(x, rows, cols, ld, fmt, block_rows, q, scale_inv, counts=None, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(q, torch.uint8, "q"); _dev(scale_inv, torch.float32, "scale_inv")
    _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_blockwise", lib().fp8_quantize_blockwise(
        _ptr(x), rows, cols, ld, fmt, block_rows, _ptr(q), _ptr(scale_inv), _ptr(counts), _stream(stream)))


def fp8_gemm_scaled(A, fa, B, fb, M, N, K, mode, a_scale_inv, b_scale_inv, D, ldd, workspace=None,
                    stream=None):
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(a_scale_inv, torch.float32, "a_scale_inv"); _dev(b_scale_inv, torch.float32, "b_scale_inv")
    _dev(workspace, torch.uint8, "workspace")
    _check("fp8_gemm_scaled", lib().fp8_gemm_scaled(
        _ptr(A), fa, _ptr(B), fb, M, N, K, mode, _ptr(a_scale_inv), _ptr(b_scale_inv), _ptr(D), ldd,
        _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream)))


def fp8_gemm_scaled_noalloc(A, fa, B, fb, M, N, K, mode, a_scale_inv, b_scale_inv, D, ldd, stream=None):
    """fp8_gemm_scaled with the split-K scratch built into the library (for
    callers that cannot allocate device memory; see include/fp8q.h)."""
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(a_scale_inv, torch.float32, "a_scale_inv"); _dev(b_scale_inv, torch.float32, "b_scale_inv")
    _check("fp8_gemm_scaled_noalloc", lib().fp8_gemm_scaled_noalloc(
        _ptr(A), fa, _ptr(B), fb, M, N, K, mode, _ptr(a_scale_inv), _ptr(b_scale_inv), _ptr(D), ldd,
        _stream(stream)))


def fp8_gemm_block_requant(A, fa, B, fb, M, N, K, a_scale_inv, b_scale_inv, D, ldd, fo, q, q_scale_inv,
                           counts=None, stream=None):
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(a_scale_inv, torch.float32, "a_scale_inv"); _dev(b_scale_inv, torch.float32, "b_scale_inv")
    _dev(q, torch.uint8, "q"); _dev(q_scale_inv, torch.float32, "q_scale_inv"); _dev(counts, torch.int32, "counts")
    _check("fp8_gemm_block_requant", lib().fp8_gemm_block_requant(
        _ptr(A), fa, _ptr(B), fb, M, N, K, _ptr(a_scale_inv), _ptr(b_scale_inv), _ptr(D), ldd, fo, _ptr(q),
        _ptr(q_scale_inv), _ptr(counts), _stream(stream)))


def fp8_gemm_grouped(A, fa, B, fb, G, group_offsets, total_M, N, K, mode, a_scale_inv, b_scale_inv, D, ldd,
                     stream=None):
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(group_offsets, torch.int64, "group_offsets")
    _dev(a_scale_inv, torch.float32, "a_scale_inv"); _dev(b_scale_inv, torch.float32, "b_scale_inv")
    _check("fp8_gemm_grouped", lib().fp8_gemm_grouped(
        _ptr(A), fa, _ptr(B), fb, G, _ptr(group_offsets), total_M, N, K, mode, _ptr(a_scale_inv),
        _ptr(b_scale_inv), _ptr(D), ldd, _stream(stream)))


def fp8_gemm_workspace_size(M, N, K, mode) -> int:
    b = ctypes.c_size_t(0)
    _check("fp8_gemm_workspace_size", lib().fp8_gemm_workspace_size(M, N, K, mode, ctypes.byref(b)))
    return int(b.value)


def fp8_amax_history_update(history, pos, amax_cur, fmt, scale, scale_inv, saturated, stream=None):
    _dev(history, torch.float32, "history"); _dev(pos, torch.int32, "pos")
    _dev(amax_cur, torch.float32, "amax_cur"); _dev(scale, torch.float32, "scale")
    _dev(scale_inv, torch.float32, "scale_inv"); _dev(saturated, torch.int32, "saturated")
    _check("fp8_amax_history_update", lib().fp8_amax_history_update(
        _ptr(history), _ptr(pos), history.numel(), _ptr(amax_cur), fmt, _ptr(scale), _ptr(scale_inv),
        _ptr(saturated), _stream(stream)))


def fp8_kv_quant(kv, B, H, S, Dh, fmt, q, scale_inv, counts=None, stream=None):
    _dev(kv, torch.bfloat16, "kv"); _dev(q, torch.uint8, "q"); _dev(scale_inv, torch.float32, "scale_inv")
    _dev(counts, torch.int32, "counts")
    _check("fp8_kv_quant", lib().fp8_kv_quant(_ptr(kv), B, H, S, Dh, fmt, _ptr(q), _ptr(scale_inv), _ptr(counts),
                                              _stream(stream)))


def fp8_kv_dequant(q, scale_inv, B, H, S, Dh, fmt, out, stream=None):
    _dev(q, torch.uint8, "q"); _dev(scale_inv, torch.float32, "scale_inv"); _dev(out, torch.bfloat16, "out")
    _check("fp8_kv_dequant", lib().fp8_kv_dequant(_ptr(q), _ptr(scale_inv), B, H, S, Dh, fmt, _ptr(out),
                                                  _stream(stream)))


def fp8_quantize_blockwise_e8m0(x, rows, cols, ld, fmt, block_rows, q, sf_image, counts=None, stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(q, torch.uint8, "q"); _dev(sf_image, torch.uint8, "sf_image")
    _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_blockwise_e8m0", lib().fp8_quantize_blockwise_e8m0(
        _ptr(x), rows, cols, ld, fmt, block_rows, _ptr(q), _ptr(sf_image), _ptr(counts), _stream(stream)))


def fp8_gemm_block_e8m0(A, fa, B, fb, M, N, K, a_sf, b_sf, D, ldd, stream=None):
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(a_sf, torch.uint8, "a_sf"); _dev(b_sf, torch.uint8, "b_sf")
    _check("fp8_gemm_block_e8m0", lib().fp8_gemm_block_e8m0(
        _ptr(A), fa, _ptr(B), fb, M, N, K, _ptr(a_sf), _ptr(b_sf), _ptr(D), ldd, _stream(stream)))


def fp8_quantize_rowwise_pair(a, rows_a, lda, qa, sa, b, rows_b, ldb, qb, sb, cols, fmt, pow2, counts=None,
                              stream=None):
    _dev(a, torch.bfloat16, "a"); _dev(qa, torch.uint8, "qa"); _dev(sa, torch.float32, "sa")
    _dev(b, torch.bfloat16, "b"); _dev(qb, torch.uint8, "qb"); _dev(sb, torch.float32, "sb")
    _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_rowwise_pair", lib().fp8_quantize_rowwise_pair(
        _ptr(a), rows_a, lda, _ptr(qa), _ptr(sa), _ptr(b), rows_b, ldb, _ptr(qb), _ptr(sb), cols, fmt, int(pow2),
        _ptr(counts), _stream(stream)))


def quantize_rowwise_pair(a, b, fmt=E4M3, pow2=True, counts=None):
    """((qa, sa), (qb, sb)) of a [Ma, K] and b [Mb, K] in one launch."""
    K = a.shape[1]
    if b.shape[1] != K:
        raise ValueError("both operands need the same row length")
    qa = torch.empty(a.shape, dtype=torch.uint8, device=a.device)
    qb = torch.empty(b.shape, dtype=torch.uint8, device=b.device)
    sa = torch.empty(a.shape[0], dtype=torch.float32, device=a.device)
    sb = torch.empty(b.shape[0], dtype=torch.float32, device=b.device)
    fp8_quantize_rowwise_pair(a, a.shape[0], a.stride(0), qa, sa, b, b.shape[0], b.stride(0), qb, sb, K, fmt, pow2,
                              counts)
    return (qa, sa), (qb, sb)


def fp8_quantize_rowwise_transpose(x, rows, cols, ld, fmt, pow2, qT, scale_inv, amax_out, counts=None,
                                   stream=None):
    _dev(x, torch.bfloat16, "x"); _dev(qT, torch.uint8, "qT")
    _dev(scale_inv, torch.float32, "scale_inv"); _dev(amax_out, torch.float32, "amax_out")
    _dev(counts, torch.int32, "counts")
    _check("fp8_quantize_rowwise_transpose", lib().fp8_quantize_rowwise_transpose(
        _ptr(x), rows, cols, ld, fmt, int(pow2), _ptr(qT), _ptr(scale_inv), _ptr(amax_out), _ptr(counts),
        _stream(stream)))


def quantize_rowwise_transpose(x, fmt, pow2=True, counts=None):
    """(qT [cols, rows], scale_inv [cols], amax [cols]) of x [rows, cols]."""
    rows, cols = x.shape
    qT = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    sinv = torch.empty(cols, dtype=torch.float32, device=x.device)
    am = torch.empty(cols, dtype=torch.float32, device=x.device)
    fp8_quantize_rowwise_transpose(x, rows, cols, x.stride(0), fmt, pow2, qT, sinv, am, counts)
    return qT, sinv, am


def fp8_gemm_bf16_wgrad(dY, X, T, M, N, ld_dy, ld_x, dW, ldd, accumulate=False, stream=None):
    _dev(dY, torch.bfloat16, "dY"); _dev(X, torch.bfloat16, "X"); _dev(dW, torch.float32, "dW")
    _check("fp8_gemm_bf16_wgrad", lib().fp8_gemm_bf16_wgrad(
        _ptr(dY), _ptr(X), T, M, N, ld_dy, ld_x, _ptr(dW), ldd, int(accumulate), _stream(stream)))


def gemm_bf16_wgrad(dY, X, out=None, accumulate=False):
    """dW [M, N] fp32 = (dW if accumulate) + dY^T X for token-major dY [T, M], X [T, N]."""
    T, M = dY.shape
    N = X.shape[1]
    dW = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=dY.device)
    fp8_gemm_bf16_wgrad(dY, X, T, M, N, dY.stride(0), X.stride(0), dW, dW.stride(0), accumulate)
    return dW


def e8m0_image_bytes(rows: int, cols: int) -> int:
    return ((cols + 511) // 512) * ((rows + 127) // 128) * 512


def quantize_blockwise_e8m0(x, fmt, block_rows, counts=None):
    """(q, sf_image) of x [rows, cols] with power-of-two block scales."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    img = torch.empty(e8m0_image_bytes(rows, cols), dtype=torch.uint8, device=x.device)
    fp8_quantize_blockwise_e8m0(x, rows, cols, x.stride(0), fmt, block_rows, q, img, counts)
    return q, img


def fp8_gemm_block_e8m0_requant(A, fa, B, fb, M, N, K, a_sf, b_sf, D, ldd, fo, q, q_sf, counts=None, stream=None):
    _dev(A, torch.uint8, "A"); _dev(B, torch.uint8, "B"); _dev(D, torch.bfloat16, "D")
    _dev(a_sf, torch.uint8, "a_sf"); _dev(b_sf, torch.uint8, "b_sf")
    _dev(q, torch.uint8, "q"); _dev(q_sf, torch.uint8, "q_sf"); _dev(counts, torch.int32, "counts")
    _check("fp8_gemm_block_e8m0_requant", lib().fp8_gemm_block_e8m0_requant(
        _ptr(A), fa, _ptr(B), fb, M, N, K, _ptr(a_sf), _ptr(b_sf), _ptr(D), ldd, fo, _ptr(q), _ptr(q_sf),
        _ptr(counts), _stream(stream)))


def gemm_block_e8m0_requant(A, fa, B, fb, a_sf, b_sf, fo, store_d=False, counts=None):
    """(q [M, N], q_sf E8M0 image, D or None): the E8M0 GEMM's output requantized 1 x 128 with
    power-of-two scales, as quantize_blockwise_e8m0(D, fo, 1) would."""
    M, K = A.shape
    N = B.shape[0]
    D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if store_d else None
    q = torch.empty((M, N), dtype=torch.uint8, device=A.device)
    q_sf = torch.empty(e8m0_image_bytes(M, N), dtype=torch.uint8, device=A.device)
    fp8_gemm_block_e8m0_requant(A, fa, B, fb, M, N, K, a_sf, b_sf, D, N, fo, q, q_sf, counts)
    return q, q_sf, D


def gemm_block_e8m0(A, fa, B, fb, a_sf, b_sf, out=None):
    M, K = A.shape
    N = B.shape[0]
    D = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    fp8_gemm_block_e8m0(A, fa, B, fb, M, N, K, a_sf, b_sf, D, D.stride(0))
    return D


def fp8_paged_kv_write(kv, slot_mapping, T, H, Dh, num_slots, fmt, cache, scale_cache, stream=None):
    _dev(kv, torch.bfloat16, "kv"); _dev(slot_mapping, torch.int64, "slot_mapping")
    _dev(cache, torch.uint8, "cache"); _dev(scale_cache, torch.float32, "scale_cache")
    _check("fp8_paged_kv_write", lib().fp8_paged_kv_write(
        _ptr(kv), _ptr(slot_mapping), T, H, Dh, num_slots, fmt, _ptr(cache), _ptr(scale_cache), _stream(stream)))


def fp8_paged_kv_gather(cache, scale_cache, block_table, seq_lens, B, max_blocks, H, Dh, block_size, num_blocks,
                        S_out, fmt, out, stream=None):
    _dev(cache, torch.uint8, "cache"); _dev(scale_cache, torch.float32, "scale_cache")
    _dev(block_table, torch.int32, "block_table"); _dev(seq_lens, torch.int32, "seq_lens")
    _dev(out, torch.bfloat16, "out")
    _check("fp8_paged_kv_gather", lib().fp8_paged_kv_gather(
        _ptr(cache), _ptr(scale_cache), _ptr(block_table), _ptr(seq_lens), B, max_blocks, H, Dh, block_size,
        num_blocks, S_out, fmt, _ptr(out), _stream(stream)))


def fp8_scale_stats(scales, prev, n, seg_offsets, num_segments, jump_ratio, stats, counts, stream=None):
    _dev(scales, torch.float32, "scales"); _dev(prev, torch.float32, "prev")
    _dev(seg_offsets, torch.int64, "seg_offsets")
    _dev(stats, torch.float32, "stats"); _dev(counts, torch.int32, "counts")
    _check("fp8_scale_stats", lib().fp8_scale_stats(
        _ptr(scales), _ptr(prev), n, _ptr(seg_offsets), num_segments, jump_ratio, _ptr(stats), _ptr(counts),
        _stream(stream)))


def fp8_device_error(clear: bool = False) -> int:
    v = ctypes.c_uint32(0)
    _check("fp8_device_error", lib().fp8_device_error(ctypes.byref(v), int(clear)))
    return int(v.value)


# ------------------------------------------------ allocating conveniences --

def amax(x, counts=None):
    out = torch.empty(1, dtype=torch.float32, device=x.device)
    fp8_amax(x, out, counts)
    return out


def quantize_tensorwise(x, fmt=E4M3, scale_in=None, transpose=False, counts=None, want_amax=True):
    """Returns (q, scale_inv[1], amax[1] or None).  x is 2-D [rows, cols] or 1-D."""
    rows, cols = (1, x.numel()) if x.dim() == 1 else tuple(x.shape)
    q = torch.empty((cols, rows) if transpose else (rows, cols), dtype=torch.uint8, device=x.device)
    if x.dim() == 1 and not transpose:
        q = q.view(-1)
    sinv = torch.empty(1, dtype=torch.float32, device=x.device)
    am = torch.empty(1, dtype=torch.float32, device=x.device) if (want_amax or scale_in is None) else None
    fp8_quantize_tensorwise(x, rows, cols, fmt, scale_in, q, transpose, sinv, am, counts)
    return q, sinv, am


def quantize_rowwise(x, fmt=E4M3, pow2=True, counts=None):
    """(q, scale_inv) of x [rows, cols]; counts: an int32 [2] device tensor
    the non-finite and saturated counts are added to, or None."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    sinv = torch.empty(rows, dtype=torch.float32, device=x.device)
    fp8_quantize_rowwise(x, rows, cols, x.stride(0), fmt, pow2, q, sinv, counts)
    return q, sinv


def quantize_blockwise(x, fmt=E4M3, block_rows=1, counts=None):
    rows, cols = x.shape
    nkb = (cols + 127) // 128
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if block_rows == 1:
        sinv = torch.empty((nkb, rows), dtype=torch.float32, device=x.device)
    else:
        sinv = torch.empty(((rows + block_rows - 1) // block_rows, nkb), dtype=torch.float32, device=x.device)
    fp8_quantize_blockwise(x, rows, cols, x.stride(0), fmt, block_rows, q, sinv, counts)
    return q, sinv


def gemm_workspace(M, N, K, mode, device="cuda"):
    """Zero-filled workspace of the size fp8_gemm_scaled can use (None if 0)."""
    n = fp8_gemm_workspace_size(M, N, K, mode)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def gemm(A, fa, B, fb, mode, a_scale_inv, b_scale_inv, out=None, workspace=None):
    M, K = A.shape
    N = B.shape[0]
    D = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    fp8_gemm_scaled(A, fa, B, fb, M, N, K, mode, a_scale_inv, b_scale_inv, D, D.stride(0), workspace)
    return D


def gemm_block_requant(A, fa, B, fb, a_scale_inv, b_scale_inv, fo, store_d=False, counts=None):
    """(q [M, N] codes of format fo, q_scale_inv [ceil(N/128), M], D [M, N] bf16 or None): the block-scaled
    GEMM's output requantized with 1 x 128 blocks, as quantize_blockwise(D, fo, 1) would."""
    M, K = A.shape
    N = B.shape[0]
    D = torch.empty((M, N), dtype=torch.bfloat16, device=A.device) if store_d else None
    q = torch.empty((M, N), dtype=torch.uint8, device=A.device)
    qs = torch.empty(((N + 127) // 128, M), dtype=torch.float32, device=A.device)
    fp8_gemm_block_requant(A, fa, B, fb, M, N, K, a_scale_inv, b_scale_inv, D, N, fo, q, qs, counts)
    return q, qs, D


def gemm_grouped(A, fa, B, fb, group_offsets, mode, a_scale_inv, b_scale_inv, out=None):
    """A [total_M, K], B [G, N, K], group_offsets int64 [G+1] on the device."""
    total_M, K = A.shape
    G, N, _ = B.shape
    D = out if out is not None else torch.empty((total_M, N), dtype=torch.bfloat16, device=A.device)
    fp8_gemm_grouped(A, fa, B.reshape(G * N, K), fb, G, group_offsets, total_M, N, K, mode, a_scale_inv,
                     b_scale_inv, D, D.stride(0))
    return D


def kv_quant(kv, fmt=E4M3, counts=None):
    B, H, S, Dh = kv.shape
    q = torch.empty(kv.shape, dtype=torch.uint8, device=kv.device)
    sinv = torch.empty(B * H, dtype=torch.float32, device=kv.device)
    fp8_kv_quant(kv, B, H, S, Dh, fmt, q, sinv, counts)
    return q, sinv


def kv_dequant(q, scale_inv, fmt=E4M3):
    B, H, S, Dh = q.shape
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    fp8_kv_dequant(q, scale_inv, B, H, S, Dh, fmt, out)
    return out


class PagedKVCache:
    """Device-resident paged FP8 cache of one tensor (K or V of one layer):
    codes [num_blocks, block_size, H, Dh] and 1/s per (slot, head)."""

    def __init__(self, num_blocks: int, block_size: int, H: int, Dh: int, fmt: int = E4M3, device="cuda"):
        self.fmt, self.block_size, self.H, self.Dh = fmt, block_size, H, Dh
        self.num_blocks = num_blocks
        self.cache = torch.zeros((num_blocks, block_size, H, Dh), dtype=torch.uint8, device=device)
        self.scale_inv = torch.zeros((num_blocks, block_size, H), dtype=torch.float32, device=device)

    def write(self, kv, slot_mapping):
        """kv [T, H, Dh] bf16 into the slots slot_mapping [T] (int64; < 0 = padding)."""
        T = kv.shape[0]
        fp8_paged_kv_write(kv, slot_mapping, T, self.H, self.Dh, self.num_blocks * self.block_size, self.fmt,
                           self.cache, self.scale_inv)

    def gather(self, block_table, seq_lens, S_out: int):
        """[B, S_out, H, Dh] bf16 of every sequence (0 past its length)."""
        B, mb = block_table.shape
        out = torch.empty((B, S_out, self.H, self.Dh), dtype=torch.bfloat16, device=self.cache.device)
        fp8_paged_kv_gather(self.cache, self.scale_inv, block_table, seq_lens, B, mb, self.H, self.Dh,
                            self.block_size, self.num_blocks, S_out, self.fmt, out)
        return out


def scale_stats(scales, seg_offsets=None, prev=None, jump_ratio=4.0):
    """Health check of scale factors: per segment {min, max, mean} (fp32 [G, 3])
    and {step changes against prev, invalid entries} (int32 [G, 2], read as
    unsigned).  seg_offsets: device int64 [G + 1] or None for one segment."""
    s = scales.reshape(-1)
    p = None if prev is None else prev.reshape(-1)
    if p is not None and p.numel() != s.numel():
        raise ValueError("prev must have as many entries as scales")
    G = 1 if seg_offsets is None else seg_offsets.numel() - 1
    stats = torch.empty((G, 3), dtype=torch.float32, device=s.device)
    counts = torch.empty((G, 2), dtype=torch.int32, device=s.device)
    fp8_scale_stats(s, p, s.numel(), seg_offsets, G, jump_ratio, stats, counts)
    return stats, counts


class AmaxHistory:
    """Device-resident delayed-scaling state (history ring, position, scale)."""

    def __init__(self, length: int, fmt: int, device="cuda"):
        self.fmt = fmt
        self.history = torch.zeros(length, dtype=torch.float32, device=device)
        self.pos = torch.zeros(1, dtype=torch.int32, device=device)
        self.scale = torch.ones(1, dtype=torch.float32, device=device)
        self.scale_inv = torch.ones(1, dtype=torch.float32, device=device)
        self.saturated = torch.zeros(1, dtype=torch.int32, device=device)

    def update(self, amax_cur):
        fp8_amax_history_update(self.history, self.pos, amax_cur, self.fmt, self.scale, self.scale_inv,
                                self.saturated)
