"""GPU parity of the FP8 KV cache and of the delayed-scaling history against
the CPU oracle (bit-exact), plus the delayed-scaling data-gradient loop.

Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §3.1 (FP8 KV cache),
§2.3 (delayed scaling from the previous steps' statistics; recompute when the
deviation passes a threshold), §2.1 (E5M2 gradients), §5.1 (overflow).
"""
import numpy as np
import pytest
import torch

from fp8_scaled_quantization_amax_b200 import fp8q, inputs
from tests.gpu_util import assert_codes_equal, assert_f32_equal, assert_gemm_close, need_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()
    yield
    assert fp8q.fp8_device_error(clear=True) == 0


# ---------------------------------------------------------------- KV cache --

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("shape", [(1, 1, 16, 1), (2, 3, 64, 128), (2, 8, 1000, 64), (1, 40, 257, 80)])
def test_kv_quant_dequant_small(orc, fmt, shape):
    x = inputs.normal_bf16(shape, 1.0, seed=sum(shape))
    bits = inputs.bf16_bits(x).copy()
    bits.reshape(-1)[5] = 0   # harmless edge: zero
    if shape[1] > 1:
        bits[0, 1] = 0        # an all-zero (b, h) slice -> scale 1
    x = inputs.from_bf16_bits(bits, "cuda")
    q, sinv = fp8q.kv_quant(x, fmt)
    rq, rsinv = orc.kv_quant(bits, fmt)
    assert_codes_equal(to_np(q), rq, fmt)
    assert_f32_equal(to_np(sinv), rsinv)
    back = fp8q.kv_dequant(q, sinv, fmt)
    rback = orc.kv_dequant(rq, rsinv, fmt)
    assert np.array_equal(inputs.bf16_bits(back), rback)


def test_kv_full_size_sampled_slices(orc):
    """K [32, 32, 8192, 128] bf16: every (b, h) scale and 8 whole slices."""
    B, H, S, Dh = 32, 32, 8192, 128
    k = inputs.normal_bf16((B, H, S, Dh), 1.0, seed=77, device="cuda")
    q, sinv = fp8q.kv_quant(k, 0)
    back = fp8q.kv_dequant(q, sinv, 0)
    rng = np.random.default_rng(0)
    picks = [(0, 0), (B - 1, H - 1)] + [tuple(v) for v in rng.integers(0, 32, (6, 2))]
    for b, h in picks:
        bits = inputs.bf16_bits(k[b:b + 1, h:h + 1])
        rq, rsinv = orc.kv_quant(bits, 0)
        assert_codes_equal(to_np(q[b:b + 1, h:h + 1]), rq, 0, f"q[{b},{h}]")
        assert_f32_equal(to_np(sinv[b * H + h: b * H + h + 1]), rsinv)
        assert np.array_equal(inputs.bf16_bits(back[b:b + 1, h:h + 1]), orc.kv_dequant(rq, rsinv, 0))
    # every slice's scale: amax of the slice from torch's own max (a library
    # reduction over exact bf16 magnitudes), then the oracle's scale rule
    am = k.view(B * H, -1).abs().amax(dim=1).float().cpu().numpy()
    ref = np.array([orc.inverse(orc.scale_from_amax(float(a), 0)) for a in am], np.float32)
    assert_f32_equal(to_np(sinv), ref)


# --------------------------------------------------------- delayed scaling --

@pytest.mark.parametrize("fmt", [0, 1])
def test_history_sequence_bit_exact(orc, fmt):
    rng = np.random.default_rng(5)
    amaxes = rng.uniform(0.5, 4.0, 40).astype(np.float32)
    amaxes[10] = 300.0 if fmt == 0 else 4e4       # a spike
    amaxes[25] = 0.0
    dev = fp8q.AmaxHistory(16, fmt)
    ref = orc.AmaxHistory(16, fmt)
    cur = torch.empty(1, dtype=torch.float32, device="cuda")
    for a in amaxes:
        cur.fill_(float(a))
        dev.update(cur)
        sat = ref.update(float(a))
        assert_f32_equal(to_np(dev.history), ref.history)
        assert int(dev.pos) == int(ref.pos[0])
        assert_f32_equal(to_np(dev.scale), ref.scale)
        assert_f32_equal(to_np(dev.scale_inv), ref.scale_inv)
        assert int(dev.saturated) == sat


@pytest.mark.parametrize("fmt", [0, 1])
def test_history_checkpoint_resume_on_device(orc, fmt):
    """The delayed-scaling state (history ring, position, scale) is the whole
    checkpoint ("DeepL押注FP8" §2.3: the scale of a step is predicted from
    the previous steps' statistics).  Run 8 steps on the device, save the
    state to the host, reload it into fresh device buffers and run 12 more:
    every step after the reload must equal, bit for bit, an uninterrupted
    device run and the oracle."""
    rng = np.random.default_rng(17 + fmt)
    amaxes = rng.uniform(0.25, 8.0, 20).astype(np.float32)
    amaxes[11] = 500.0 if fmt == 0 else 6e4          # a spike after the reload
    cur = torch.empty(1, dtype=torch.float32, device="cuda")
    full = fp8q.AmaxHistory(16, fmt)
    part = fp8q.AmaxHistory(16, fmt)
    ref = orc.AmaxHistory(16, fmt)
    for a in amaxes[:8]:
        cur.fill_(float(a))
        full.update(cur)
        part.update(cur)
        ref.update(float(a))
    saved = {k: getattr(part, k).cpu().clone() for k in ("history", "pos", "scale", "scale_inv")}
    del part
    resumed = fp8q.AmaxHistory(16, fmt)
    for k, v in saved.items():
        getattr(resumed, k).copy_(v.to("cuda"))
    for a in amaxes[8:]:
        cur.fill_(float(a))
        full.update(cur)
        resumed.update(cur)
        sat = ref.update(float(a))
        for k in ("history", "scale", "scale_inv"):
            assert_f32_equal(to_np(getattr(resumed, k)), to_np(getattr(full, k)), k)
            assert_f32_equal(to_np(getattr(resumed, k)), getattr(ref, k), k)
        assert int(resumed.pos) == int(full.pos) == int(ref.pos[0])
        assert int(resumed.saturated) == int(full.saturated) == sat


def test_dgrad_delayed_scaling_loop(orc):
    """Data-gradient GEMM with delayed scaling, reduced to [512, 256] x
    W[256, 384]: per step quantize dY_t (E5M2, scale from the history, amax
    fused), GEMM against the E4M3 W^T, update the history.  Every step is
    compared with the oracle running the same recipe; step 9 is an injected
    x8 spike that must raise the saturation flag."""
    M, N_out, K_in = 512, 256, 384
    W = inputs.normal_bf16((N_out, K_in), 0.02, seed=100)
    wb = inputs.bf16_bits(W)
    # E4M3 W^T [K_in, N_out] through the transposed tensorwise cast
    wq, wsinv, _ = fp8q.quantize_tensorwise(W.to("cuda"), 0, transpose=True)
    rwq, rwsinv, _, _ = orc.quantize_tensorwise(wb, 0, transpose_out=True)
    assert_codes_equal(to_np(wq), rwq, 0)
    hist = fp8q.AmaxHistory(16, 1)
    rh = orc.AmaxHistory(16, 1)
    for t in range(14):
        g = inputs.lognormal_grads_bf16((M, N_out), seed=1000 + t)
        if t == 9:
            g = (g.float() * 8).to(torch.bfloat16)
        gb = inputs.bf16_bits(g)
        q, sinv, am = fp8q.quantize_tensorwise(g.to("cuda"), 1, scale_in=hist.scale)
        rq, rsinv, ramax, _ = orc.quantize_tensorwise(gb, 1, scale_in=float(rh.scale[0]))
        assert_codes_equal(to_np(q), rq, 1, f"dY8 step {t}")
        assert_f32_equal(to_np(am), np.float32([ramax]))
        D = fp8q.gemm(q, 1, wq, 0, 0, sinv, wsinv)
        ref, mag = orc.gemm_scaled(rq, 1, rwq, 0, 0, np.float32([rsinv]), np.float32([rwsinv]))
        assert_gemm_close(D.float().cpu().numpy().astype(np.float64), ref, mag, f"dX step {t}")
        hist.update(am)
        sat = rh.update(ramax)
        assert int(hist.saturated) == sat
        assert_f32_equal(to_np(hist.scale), rh.scale)
        if t == 9:
            assert sat == 1


def test_dgrad_full_size_delayed_scaling_sampled(orc):
    """The dgrad workload at full size and in the bench's launch
    configuration: dY_t [8192, 4096] (log-normal magnitudes, E5M2 with the
    history's scale and fused amax) against W^T [4096, 4096] (E4M3
    per-tensor, transposed cast), split-K workspace passed as the bench does,
    16-step history; 5 steps, the third an x8 spike.  Codes and amax
    bit-exact per step, 512 sampled outputs per step against the oracle."""
    M, N_out, K_in = 8192, 4096, 4096
    W = inputs.normal_bf16((N_out, K_in), 0.02, seed=300, device="cuda")
    wq, wsinv, _ = fp8q.quantize_tensorwise(W, 0, transpose=True)
    rwq, rwsinv, _, _ = orc.quantize_tensorwise(inputs.bf16_bits(W), 0, transpose_out=True)
    assert_codes_equal(to_np(wq), rwq, 0)
    hist = fp8q.AmaxHistory(16, 1)
    rh = orc.AmaxHistory(16, 1)
    ws = fp8q.gemm_workspace(M, K_in, N_out, fp8q.SCALE_TENSOR)
    rng = np.random.default_rng(3)
    for t in range(5):
        g = inputs.lognormal_grads_bf16((M, N_out), seed=400 + t, device="cuda")
        if t == 2:
            g = (g.float() * 8).to(torch.bfloat16)
        gb = inputs.bf16_bits(g)
        q, sinv, am = fp8q.quantize_tensorwise(g, 1, scale_in=hist.scale)
        rq, rsinv, ramax, _ = orc.quantize_tensorwise(gb, 1, scale_in=float(rh.scale[0]))
        assert_codes_equal(to_np(q), rq, 1, f"dY8 step {t}")
        assert_f32_equal(to_np(am), np.float32([ramax]))
        D = fp8q.gemm(q, 1, wq, 0, 0, sinv, wsinv, workspace=ws)
        im = np.concatenate([[0, M - 1], rng.integers(0, M, 510)])
        inn = np.concatenate([[0, K_in - 1], rng.integers(0, K_in, 510)])
        ref, mag = orc.gemm_scaled_sampled(rq, 1, rwq, 0, 0, np.float32([rsinv]), np.float32([rwsinv]), im, inn)
        got = D.float().cpu().numpy().astype(np.float64)[im, inn]
        assert_gemm_close(got, ref, mag, f"dX step {t}")
        hist.update(am)
        sat = rh.update(ramax)
        assert int(hist.saturated) == sat
        assert_f32_equal(to_np(hist.scale), rh.scale)
        if t == 2:
            assert sat == 1
