"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol ``include/fp8q.h`` declares, and rejects bad arguments before
touching the device; with no device a valid call fails loudly (no fallback)."""
import ctypes
import os
import re

import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, CUDA = range(6)


def declared_symbols():
    txt = open(HEADER).read()
    return re.findall(r"^FP8Q_API\s+[^;(]*?\b(fp8_\w+)\s*\(", txt, flags=re.M)


def test_header_declares_the_abi():
    names = declared_symbols()
    assert len(names) == len(set(names)) >= 10
    assert set(names) == set(fp8q.SIGNATURES)


def test_library_exports_every_declared_symbol():
    L = fp8q.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings():
    L = fp8q.lib()
    for s in range(6):
        assert L.fp8_status_string(s)
    assert b"sm_100a" in L.fp8_status_string(UNSUPPORTED)
    assert L.fp8_status_string(99) == b"FP8_ERR_UNKNOWN"


P = ctypes.c_void_p
FAKE = P(0x10000)          # a 16-byte aligned non-null address never dereferenced
FAKE_ODD = P(0x10002)


def test_validation_before_device_access():
    L = fp8q.lib()
    n = P(0)
    # GEMM: bad format, bad mode, K % 16, N % 8, null D, misaligned A
    assert L.fp8_gemm_scaled(FAKE, 3, FAKE, 0, 64, 64, 64, 0, FAKE, FAKE, FAKE, 64, None, 0, n) == INVALID
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 64, 64, 64, 5, FAKE, FAKE, FAKE, 64, None, 0, n) == INVALID
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 64, 64, 40, 0, FAKE, FAKE, FAKE, 64, None, 0, n) == SHAPE
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 64, 60, 64, 0, FAKE, FAKE, FAKE, 64, None, 0, n) == ALIGN
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 64, 64, 64, 0, FAKE, FAKE, None, 64, None, 0, n) == INVALID
    assert L.fp8_gemm_scaled(FAKE_ODD, 0, FAKE, 0, 64, 64, 64, 0, FAKE, FAKE, FAKE, 64, None, 0, n) == ALIGN
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, -1, 64, 64, 0, FAKE, FAKE, FAKE, 64, None, 0, n) == SHAPE
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 64, 64, 64, 0, FAKE, FAKE, FAKE, 32, None, 0, n) == SHAPE  # ldd < N
    # quantizers
    assert L.fp8_quantize_rowwise(FAKE, 4, 24, 32, 0, 1, FAKE, FAKE, None, n) == SHAPE
    assert L.fp8_quantize_rowwise(FAKE, 4, 16, 20, 0, 1, FAKE, FAKE, None, n) == ALIGN
    assert L.fp8_quantize_rowwise(FAKE, 4, 16, 16, 2, 1, FAKE, FAKE, None, n) == INVALID
    assert L.fp8_quantize_rowwise(FAKE, 4, 16, 16, 0, 1, FAKE, FAKE, FAKE_ODD, n) == ALIGN   # counts
    assert L.fp8_quantize_blockwise(FAKE, 4, 32, 32, 0, 64, FAKE, FAKE, None, n) == INVALID
    assert L.fp8_quantize_blockwise(FAKE, 4, 32, 32, 0, 1, FAKE, FAKE, FAKE_ODD, n) == ALIGN  # counts
    assert L.fp8_quantize_tensorwise(FAKE, 4, 32, 0, None, FAKE, 0, FAKE, None, None, n) == INVALID
    assert L.fp8_quantize_tensorwise(FAKE, 4, 40, 0, FAKE, FAKE, 1, FAKE, None, None, n) == SHAPE
    assert L.fp8_gemm_scaled(FAKE, 0, FAKE, 0, 256, 256, 256, 0, FAKE, FAKE, FAKE, 256, FAKE_ODD, 1024, n) == ALIGN
    assert L.fp8_gemm_workspace_size(64, 64, 64, 9, ctypes.byref(ctypes.c_size_t())) == INVALID
    assert L.fp8_gemm_workspace_size(-1, 64, 64, 0, ctypes.byref(ctypes.c_size_t())) == SHAPE
    assert L.fp8_gemm_workspace_size(64, 64, 64, 0, None) == INVALID
    assert L.fp8_amax(FAKE_ODD, 100, FAKE, None, n) == ALIGN
    assert L.fp8_amax(FAKE, -1, FAKE, None, n) == SHAPE
    assert L.fp8_amax(FAKE, 10, None, None, n) == INVALID
    # KV cache and history
    assert L.fp8_kv_quant(FAKE, 2, 2, 3, 5, 0, FAKE, FAKE, None, n) == SHAPE
    assert L.fp8_kv_quant(FAKE, 2, 2, 16, 8, 0, FAKE, FAKE, FAKE_ODD, n) == ALIGN   # counts
    assert L.fp8_kv_dequant(FAKE, FAKE, 2, 2, 16, 8, 7, FAKE, n) == INVALID
    assert L.fp8_amax_history_update(FAKE, FAKE, 0, FAKE, 0, FAKE, FAKE, FAKE, n) == SHAPE
    assert L.fp8_amax_history_update(FAKE, FAKE, 2000, FAKE, 0, FAKE, FAKE, FAKE, n) == SHAPE
    assert L.fp8_amax_history_update(None, FAKE, 16, FAKE, 0, FAKE, FAKE, FAKE, n) == INVALID
    # rowwise pair
    assert L.fp8_quantize_rowwise_pair(FAKE, 4, 32, FAKE, FAKE, FAKE, 4, 32, FAKE, FAKE, 24, 0, 1, None, n) == SHAPE
    assert L.fp8_quantize_rowwise_pair(FAKE, 4, 32, FAKE, FAKE, FAKE, 4, 16, FAKE, FAKE, 32, 0, 1, None, n) == SHAPE
    assert L.fp8_quantize_rowwise_pair(FAKE, 4, 32, FAKE, FAKE, None, 4, 32, FAKE, FAKE, 32, 0, 1, None, n) == INVALID
    assert L.fp8_quantize_rowwise_pair(FAKE, 4, 32, FAKE, FAKE, FAKE, 4, 32, FAKE, FAKE, 32, 5, 1, None, n) == INVALID
    # E8M0 block scales
    assert L.fp8_quantize_blockwise_e8m0(FAKE, 4, 32, 32, 0, 64, FAKE, FAKE, None, n) == INVALID    # block_rows
    assert L.fp8_quantize_blockwise_e8m0(FAKE, 4, 24, 32, 0, 1, FAKE, FAKE, None, n) == SHAPE       # cols % 16
    assert L.fp8_quantize_blockwise_e8m0(FAKE, 4, 32, 32, 0, 1, FAKE, FAKE_ODD, None, n) == ALIGN
    assert L.fp8_gemm_block_e8m0(FAKE, 0, FAKE, 0, 64, 64, 40, FAKE, FAKE, FAKE, 64, n) == SHAPE   # K % 16
    assert L.fp8_gemm_block_e8m0(FAKE, 2, FAKE, 0, 64, 64, 64, FAKE, FAKE, FAKE, 64, n) == INVALID
    assert L.fp8_gemm_block_e8m0(FAKE, 0, FAKE, 0, 64, 64, 64, None, FAKE, FAKE, 64, n) == INVALID
    assert L.fp8_gemm_block_e8m0(FAKE, 0, FAKE, 0, 64, 64, 64, FAKE_ODD, FAKE, FAKE, 64, n) == ALIGN
    # block-scaled GEMM with its output requantized 1x128
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 256, 264, 256, FAKE, FAKE, None, 264, 0, FAKE, FAKE, None, n) == SHAPE   # N % 16
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 256, 256, 256, FAKE, FAKE, None, 256, 3, FAKE, FAKE, None, n) == INVALID  # fo
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 256, 256, 256, FAKE, FAKE, None, 256, 0, None, FAKE, None, n) == INVALID  # q
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 64, 256, 256, FAKE, FAKE, None, 256, 0, FAKE, FAKE, None, n) == INVALID   # D needed
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 256, 256, 256, FAKE, FAKE, FAKE, 128, 0, FAKE, FAKE, None, n) == SHAPE   # ldd < N
    assert L.fp8_gemm_block_requant(FAKE, 0, FAKE, 0, 256, 256, 256, FAKE, FAKE, None, 256, 0, FAKE, FAKE, FAKE_ODD, n) == ALIGN
    # backward operands and the bf16 weight gradient
    assert L.fp8_quantize_rowwise_transpose(FAKE, 24, 32, 32, 0, 1, FAKE, FAKE, FAKE, None, n) == SHAPE   # rows % 16
    assert L.fp8_quantize_rowwise_transpose(FAKE, 32, 32, 32, 0, 1, FAKE, FAKE, None, None, n) == INVALID
    assert L.fp8_gemm_bf16_wgrad(FAKE, FAKE, 64, 12, 64, 12, 64, FAKE, 64, 0, n) == ALIGN    # M % 8
    assert L.fp8_gemm_bf16_wgrad(FAKE, FAKE, 64, 64, 64, 64, 64, None, 64, 0, n) == INVALID
    assert L.fp8_gemm_bf16_wgrad(FAKE, FAKE, 64, 64, 64, 32, 64, FAKE, 64, 0, n) == SHAPE    # ld_dy < M
    # paged KV cache
    assert L.fp8_paged_kv_write(FAKE, FAKE, 4, 2, 12, 64, 0, FAKE, FAKE, n) == SHAPE        # Dh % 8
    assert L.fp8_paged_kv_write(FAKE, FAKE, 4, 128, 128, 64, 0, FAKE, FAKE, n) == SHAPE     # H*Dh > 8192
    assert L.fp8_paged_kv_write(FAKE, FAKE, 4, 2, 64, 64, 3, FAKE, FAKE, n) == INVALID
    assert L.fp8_paged_kv_write(FAKE_ODD, FAKE, 4, 2, 64, 64, 0, FAKE, FAKE, n) == ALIGN
    assert L.fp8_paged_kv_write(FAKE, None, 4, 2, 64, 64, 0, FAKE, FAKE, n) == INVALID
    assert L.fp8_paged_kv_gather(FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 64, 0, 8, 16, 0, FAKE, n) == SHAPE
    assert L.fp8_paged_kv_gather(FAKE, FAKE, FAKE, FAKE, 70000, 4, 2, 64, 16, 8, 16, 0, FAKE, n) == SHAPE
    assert L.fp8_paged_kv_gather(FAKE, FAKE, FAKE, FAKE, 2, 4, 2, 64, 16, 8, 16, 0, FAKE_ODD, n) == ALIGN
    assert L.fp8_paged_kv_gather(FAKE, FAKE, FAKE, None, 2, 4, 2, 64, 16, 8, 16, 0, FAKE, n) == INVALID
    # scale health check
    assert L.fp8_scale_stats(FAKE, None, 16, None, 1, 0.5, FAKE, FAKE, n) == INVALID   # ratio < 1
    assert L.fp8_scale_stats(FAKE, None, 16, None, 1, float("nan"), FAKE, FAKE, n) == INVALID
    assert L.fp8_scale_stats(FAKE, None, 16, None, 1, 4.0, None, FAKE, n) == INVALID
    assert L.fp8_scale_stats(FAKE, None, 16, None, 2, 4.0, FAKE, FAKE, n) == SHAPE   # no table, 2 segments
    assert L.fp8_scale_stats(FAKE, None, 16, FAKE, 0, 4.0, FAKE, FAKE, n) == SHAPE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_fails_loudly():
    L = fp8q.lib()
    st = L.fp8_amax(FAKE, 64, FAKE, None, P(0))
    assert st in (UNSUPPORTED, CUDA)
    with pytest.raises((fp8q.Fp8Error, RuntimeError, ValueError)):
        fp8q.amax(torch.zeros(64, dtype=torch.bfloat16))


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_header_compiles_as_plain_c_and_cpp(tmp_path, lang):
    """The boundary is a C ABI: the header must compile as strict C99 (no C++
    types or overloads in the signatures) and as C++ (extern "C" guards)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "fp8q.h"\n'
                   "int main(void) { fp8_status s = FP8_OK; fp8_format f = FP8_E5M2;\n"
                   "  fp8_scale_mode m = FP8_SCALE_BLOCK; (void)s; (void)f; (void)m; return 0; }\n")
    std = ["-std=c99", "-pedantic", "-x", "c"] if lang == "c" else ["-std=c++17", "-x", "c++"]
    r = subprocess.run([cc, *std, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-c",
                        str(src), "-o", str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_e8m0_image_size_and_layout_are_one_to_one():
    """The E8M0 scale image that the GPU tests write for the block-scaled MMA
    (tests/test_gpu_block_e8m0.py) and the binding's image size agree: every
    (row, 128-column block) owns one byte of its own, the image holds nothing
    else but the unused slots of a last group of fewer than four blocks, and
    the exponent byte of a power-of-two factor 2^k is k + 127."""
    from tests.test_gpu_block_e8m0 import _e8m0, _written
    for rows, cols in [(1, 16), (128, 128), (300, 400), (257, 1040), (129, 2048), (8192, 11008)]:
        nkb, rt = (cols + 127) // 128, (rows + 127) // 128
        w = _written(rows, cols)
        assert w.size == fp8q.e8m0_image_bytes(rows, cols)
        assert int(w.sum()) == nkb * rt * 128          # no two (row, block) pairs share a byte
        assert w.size - int(w.sum()) == (-nkb % 4) * rt * 128
    assert list(_e8m0([1.0, 2.0, 0.5, 2.0 ** -126, 2.0 ** 127])) == [127, 128, 126, 1, 254]
