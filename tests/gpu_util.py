"""Helpers shared by the GPU parity tests (comparison rules only)."""
import json
import os

import numpy as np
import torch

NAN_CODES = {0: {0x7F, 0xFF}, 1: {0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF}}


def need_gpu():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_codes_equal(gpu: np.ndarray, ref: np.ndarray, fmt: int, what: str = "q"):
    """Bit-exact FP8 codes; NaN lanes compare NaN-ness only (the canonical NaN
    pattern is the hardware's choice)."""
    gpu = np.asarray(gpu, np.uint8)
    ref = np.asarray(ref, np.uint8)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    nan_ref = np.isin(ref, list(NAN_CODES[fmt]))
    nan_gpu = np.isin(gpu, list(NAN_CODES[fmt]))
    assert np.array_equal(nan_ref, nan_gpu), f"{what}: NaN positions differ"
    diff = (gpu != ref) & ~nan_ref
    if diff.any():
        idx = np.argwhere(diff)[:8]
        raise AssertionError(f"{what}: {int(diff.sum())} codes differ, first at {idx.tolist()}: "
                             f"gpu {[hex(gpu[tuple(i)]) for i in idx]} ref {[hex(ref[tuple(i)]) for i in idx]}")


def assert_f32_equal(gpu, ref, what="scale"):
    g = np.asarray(gpu, np.float32)
    r = np.asarray(ref, np.float32)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    if not np.array_equal(g.view(np.uint32), r.view(np.uint32)):
        bad = np.argwhere(g.view(np.uint32) != r.view(np.uint32))[:8]
        raise AssertionError(f"{what}: bits differ at {bad.tolist()}: gpu {g[tuple(bad[0])]!r} ref {r[tuple(bad[0])]!r}")


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def gemm_tolerance(ref: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """Per element: 1e-2 x the oracle's absolute dot-product magnitude (the
    fp32-accumulation allowance) plus the bf16 rounding of the output
    (2^-8 relative covers round-to-nearest at any binade)."""
    return 1e-2 * mag + np.abs(ref) * 2.0 ** -8 + 1e-30


def gemm_error_stats(gpu: np.ndarray, ref: np.ndarray, mag: np.ndarray) -> dict:
    """Global error figures of a GEMM output against the fp64 oracle:
    max |err| / max |ref|; the largest error in units of the per-element
    magnitude sum_k |a b| once the bf16 rounding of the output (2^-8 |ref|)
    is taken off; and the largest error relative to the bf16 rounding
    allowance alone."""
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    bf = np.abs(ref) * 2.0 ** -8
    m = np.maximum(mag, 1e-300)
    return {"n": int(err.size),
            "max_err_over_max_ref": float(err.max() / max(float(np.abs(ref).max()), 1e-300)),
            "max_excess_over_mag": float(np.max(np.maximum(err - bf, 0.0) / m)),
            "max_err_over_bf16_half_ulp": float(np.max(err / np.maximum(bf, 1e-300)))}


def _log_stats(what: str, stats: dict):
    """Append the figures to the JSON-lines file named by FP8Q_GEMM_ERR_LOG
    (unset: nothing is written)."""
    path = os.environ.get("FP8Q_GEMM_ERR_LOG")
    if not path:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, "what": what, **stats}) + "\n")


def gemm_tight_tolerance(ref: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """A structural bound inside the stated tolerance: the bf16 rounding of
    the output (2^-8 |ref|) plus 2^-14 x sum_k |a b|.  The tensor cores sum
    each 32-wide K step of exact FP8 products into an fp32 accumulator, one
    step after another, and the block-scaled epilogue adds one rounded FMA
    per 128-wide K block, so the accumulated rounding stays below
    (K/32 + K/128 + 2) x 2^-24 x sum_k |a b| <= 2^-14 x sum_k |a b| for
    K <= 16384 (measured on B200: at most 2.1e-7 x sum_k |a b| beyond the
    output rounding over every GEMM test).  One product lost or counted twice
    moves an output by about sum_k |a b| / K, far above this bound."""
    return np.abs(ref) * 2.0 ** -8 + 2.0 ** -14 * mag + 1e-30


def assert_gemm_close(gpu: np.ndarray, ref: np.ndarray, mag: np.ndarray, what="D"):
    tol = gemm_tolerance(ref, mag)
    err = np.abs(gpu - ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first {i.tolist()} "
                             f"gpu {gpu[tuple(i)]!r} ref {ref[tuple(i)]!r} tol {tol[tuple(i)]!r}")
    tight = gemm_tight_tolerance(ref, mag)
    bad = err > tight
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside the accumulation bound; first "
                             f"{i.tolist()} gpu {gpu[tuple(i)]!r} ref {ref[tuple(i)]!r} bound {tight[tuple(i)]!r}")
    stats = gemm_error_stats(gpu, ref, mag)
    _log_stats(what, stats)
    return stats["max_err_over_max_ref"]
