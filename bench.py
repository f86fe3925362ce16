#!/usr/bin/env python
"""Benchmark of the FP8 scaled-quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One "step" is one pass of the whole hot path over one batch of synthetic
input already resident in HBM.  Default workload ``blockmlp``: the
block-scaled E4M3 MLP of a 7B-style layer -- X [8192, 4096] (N(0,1)) quantized
with 1x128 scales, W_up [11008, 4096] and W_down [4096, 11008] (N(0, 0.02))
with 128x128 scales, H = X8 W_up8^T in bf16 (fp32 accumulate, fp32 scales
promoted per 128-wide K block; the GEMM's epilogue rounds H to bf16 and
requantizes it 1x128 in the same launch), D = H8 W_down8^T.
Other workloads: ``rowwise`` (per-row power-of-two E4M3 quantization of A
[4096, 4096] with 0.1 % x100 outliers and B [4096, 4096], then the
rowwise-scaled GEMM), ``tensor`` (per-tensor E4M3, 256^3),
``blockmlp_e8m0`` (the MLP with power-of-two block scales applied in the
MMA), ``dgrad`` (E5M2 gradients [8192, 4096] x E4M3 W^T [4096, 4096] with
delayed scaling over a 16-step history), ``bwd_gw_hp`` (a layer's backward
under the rowwise_with_gw_hp recipe), ``kv`` (FP8 KV cache K, V [32, 32,
8192, 128] quantize + dequantize, GB/s), ``paged`` and ``health``.

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps, then K steps
bracketed by a barrier and a device synchronize; each step's kernels are
timed with CUDA events on the launching stream, L2 is flushed (a 256 MiB write
and a 256 MiB read)
before every step outside the events; multi-GPU takes the max over ranks.
Besides the mean the line carries the median and best per-step and
dominant-kernel times (rank 0's).
``--impl reference`` times the CPU oracle (the only reference this project
has) on a bounded sample of the same workload, on every host thread this
process may use; the GPU line's ``cpu_baseline`` gives that figure and the
one-thread figure of the same sample.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 scaled GEMM TFLOP/s (% dense FP8 peak); quantize/KV GB/s (% HBM)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0     # nominal dense ratio: 4.5 PFLOP/s fp8 / 2.25 PFLOP/s bf16
DEFAULT_STEPS = {"rowwise": 6000, "tensor": 6000, "blockmlp": 1500, "blockmlp_e8m0": 1500, "dgrad": 6000, "bwd_gw_hp": 2000, "kv": 600, "paged": 600, "health": 6000}


def peaks():
    """(HBM GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s or None, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        sus = d.get("bf16_tflops_sustained")
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), (float(sus) if sus else None), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, None, "fallback"


def choose_peak(bound: str, peak_dtype: str, clocks: dict, pk) -> tuple:
    """(peak, description) for the roofline of the dominant kernel.  pk is
    peaks().  Tensor-bound kernels: the sustained (power-capped) figure when
    the timed region ran under the power cap with the SM clock pulled down
    (median below 90 % of max; the sustained figure was measured near
    1.3 GHz), the burst figure otherwise; FP8 peaks are the bf16 figure times
    the nominal dense ratio 2.  Memory-bound kernels: the HBM copy rate."""
    hbm, bf16, bf16_sus, src = pk
    if bound != "tensor":
        return hbm, f"{src} HBM copy bandwidth {hbm} GB/s"
    mhz, mhz_max = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    pulled_down = mhz is None or not mhz_max or mhz < 0.9 * mhz_max
    capped = "sw_power_cap" in clocks.get("reasons", []) and pulled_down and bf16_sus is not None
    base = bf16_sus if capped else bf16
    kind = 'sustained' if capped else 'burst'
    note = '; sw_power_cap was active in the timed region' if capped else ''
    if peak_dtype == "bf16":
        return base, (f"bf16 dense peak = {src} cuBLAS bf16 {kind} {base} TFLOP/s (MEASURED_PEAKS.json){note}"
                      if src == "measured" else f"fallback bf16 {bf16}")
    return base * FP8_OVER_BF16, (f"FP8 dense peak = {src} bf16 {kind} {base} TFLOP/s x nominal fp8/bf16 ratio 2 "
                                  f"(MEASURED_PEAKS.json){note}" if src == "measured" else f"fallback bf16 {bf16} x 2")


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/roofline_traffic.json), or None when there is none or
    when the kernel's source has changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(workload)
    if not rec:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        fp = os.path.join(ROOT, f)
        if not os.path.exists(fp):
            return None
        h.update(open(fp, "rb").read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------- workloads --

def config_of(name: str, profile: bool = False) -> dict:
    """The workload description a bench line carries in "config" (both arms)."""
    from fp8_scaled_quantization_amax_b200 import inputs as inp
    small = 2048 if profile else 8192
    if name == "rowwise":
        return {"workload": "rowwise pow2 E4M3 GEMM", "M": 4096, "N": 4096, "K": 4096,
                "A": "N(0,1) bf16, 0.1% entries x100", "B": "N(0,0.02) bf16",
                "scales": "per-row A, per-row B (= per output column), powers of two"}
    if name == "tensor":
        return {"workload": "per-tensor E4M3 GEMM", "M": 256, "N": 256, "K": 256,
                "A": "N(0,1) bf16", "B": "N(0,1) bf16", "scales": "s = 448/amax per tensor"}
    if name == "blockmlp":
        return {"workload": "block-scaled E4M3 MLP (up then down)", "M": small, "D": 4096, "F": 11008,
                "X": "N(0,1) bf16", "W": "N(0,0.02) bf16",
                "scales": "1x128 activation blocks, 128x128 weight blocks, fp32",
                "chain": "H = up(X) rounded to bf16 and requantized 1x128 for the down GEMM in the up GEMM's epilogue "
                         "(fp8_gemm_block_requant: codes and scales equal the 1x128 quantizer's on bf16 H)"}
    if name == "blockmlp_e8m0":
        return {"workload": "block-scaled E4M3 MLP (up then down), E8M0 scales in the MMA", "M": small,
                "D": 4096, "F": 11008, "X": "N(0,1) bf16", "W": "N(0,0.02) bf16",
                "scales": "1x128 activation blocks, 128x128 weight blocks, powers of two (E8M0)",
                "chain": "H = up(X) rounded to bf16 and requantized 1x128 (E8M0 image) for the down GEMM in the up "
                         "GEMM's epilogue (fp8_gemm_block_e8m0_requant)"}
    if name == "dgrad":
        return {"workload": "dgrad E5M2 x E4M3, delayed scaling", "M": small, "N_out": 4096, "K_in": 4096,
                "dY": "|g| = 10^u, u ~ N(-2, (4/3)^2) clipped to [-6, 2], random sign, 16 seeded steps",
                "W": "N(0,0.02) bf16, E4M3 per-tensor, transposed once", "history": 16}
    if name == "bwd_gw_hp":
        return {"workload": "linear backward, rowwise_with_gw_hp (FP8 rowwise dgrad, bf16 wgrad)",
                "T": small, "N_out": 4096, "K_in": 4096,
                "dY": "|g| = 10^u, u ~ N(-2, (4/3)^2) clipped to [-6, 2], random sign; E5M2 per token",
                "W": "N(0,0.02) bf16; W^T E4M3 per input channel, requantized every step",
                "X": "N(0,1) bf16", "dW": "fp32, dY^T X from the bf16 tensors"}
    if name == "kv":
        return {"workload": "FP8 KV cache quantize + dequantize", "B": 8 if profile else 32, "H": 32, "S": 8192,
                "Dh": 128, "K,V": "N(0,1) bf16", "scale": "per (b, h): 448/amax, E4M3"}
    if name == "paged":
        P = inp.PAGED_KV
        B = 8 if profile else P["B"]
        return {"workload": "paged FP8 KV cache write + gather", "sequences": B, "tokens_per_seq": P["S"],
                "H": P["H"], "Dh": P["Dh"], "block_size": P["block_size"],
                "num_blocks": B * P["S"] // P["block_size"], "pages": "shuffled pool",
                "K,V": "N(0,1) bf16", "scale": "per (token, head): 448/amax, E4M3"}
    if name == "health":
        L = inp.SCALE_HEALTH["layers"] * (8 if profile else 1)
        return {"workload": "scale health check (min/max/mean + step changes)", "segments": L,
                "scales_per_segment": inp.SCALE_HEALTH["per_layer"],
                "scales": "log10 s ~ N(1, 0.25); next snapshot drifted, 0.1 % stepped x16 or /16",
                "jump_ratio": 4.0}
    raise ValueError(name)


class Workload:
    """Inputs resident on the device and the step as a list of library calls."""

    def __init__(self, name: str, device, seed: int, profile: bool = False):
        from fp8_scaled_quantization_amax_b200 import fp8q, inputs
        self.f, self.inp = fp8q, inputs
        self.name = name
        self.dev = device
        self.seed = seed
        # --profile: the same kernels on a case that holds at most ~2.5 GB of
        # device memory (for ncu captures); never a bench value
        self.profile = profile
        getattr(self, "_setup_" + name)()

    # per-row pow2 E4M3, M = N = K = 4096
    def _setup_rowwise(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        M = N = K = 4096
        self.A = inp.outlier_activations_bf16((M, K), seed=s, device=d)
        self.B = inp.normal_bf16((N, K), 0.02, seed=s + 1, device=d)
        self.qa = torch.empty((M, K), dtype=torch.uint8, device=d)
        self.qb = torch.empty((N, K), dtype=torch.uint8, device=d)
        self.sa = torch.empty(M, dtype=torch.float32, device=d)
        self.sb = torch.empty(N, dtype=torch.float32, device=d)
        self.D = torch.empty((M, N), dtype=torch.bfloat16, device=d)
        # the library's split-K workspace, as a caller would pass it (0 bytes, so None, for 4096^3)
        self.ws = f.gemm_workspace(M, N, K, f.SCALE_ROW, device=d)
        self.flops = 2.0 * M * N * K
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.launches = 2
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("A", self.A), ("B", self.B)]
        self.host_output = self.D

    def _step_rowwise(self, ev=None):
        f = self.f
        M, K = self.A.shape
        N = self.B.shape[0]
        # both operands in one launch
        f.fp8_quantize_rowwise_pair(self.A, M, K, self.qa, self.sa, self.B, N, K, self.qb, self.sb, K, f.E4M3, True)
        if ev:
            ev[0].record()
        f.fp8_gemm_scaled(self.qa, f.E4M3, self.qb, f.E4M3, M, N, K, f.SCALE_ROW, self.sa, self.sb, self.D, N, self.ws)
        if ev:
            ev[1].record()

    # per-tensor E4M3, 256^3
    def _setup_tensor(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        M = N = K = 256
        self.A = inp.normal_bf16((M, K), 1.0, seed=s, device=d)
        self.B = inp.normal_bf16((N, K), 1.0, seed=s + 1, device=d)
        self.qa = torch.empty((M, K), dtype=torch.uint8, device=d)
        self.qb = torch.empty((N, K), dtype=torch.uint8, device=d)
        self.sa, self.sb = (torch.empty(1, dtype=torch.float32, device=d) for _ in range(2))
        self.ama, self.amb = (torch.empty(1, dtype=torch.float32, device=d) for _ in range(2))
        self.D = torch.empty((M, N), dtype=torch.bfloat16, device=d)
        self.flops = 2.0 * M * N * K
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.launches = 3          # small tensors: amax and cast in one launch each, then the GEMM
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("A", self.A), ("B", self.B)]
        self.host_output = self.D

    def _step_tensor(self, ev=None):
        f = self.f
        M, K = self.A.shape
        N = self.B.shape[0]
        f.fp8_quantize_tensorwise(self.A, M, K, f.E4M3, None, self.qa, 0, self.sa, self.ama)
        f.fp8_quantize_tensorwise(self.B, N, K, f.E4M3, None, self.qb, 0, self.sb, self.amb)
        if ev:
            ev[0].record()
        f.fp8_gemm_scaled(self.qa, f.E4M3, self.qb, f.E4M3, M, N, K, f.SCALE_TENSOR, self.sa, self.sb, self.D, N)
        if ev:
            ev[1].record()

    # block-scaled MLP: X -> up -> H -> down
    def _setup_blockmlp(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        M, Dm, F = (2048 if self.profile else 8192), 4096, 11008
        self.X = inp.normal_bf16((M, Dm), 1.0, seed=s, device=d)
        self.Wu = inp.normal_bf16((F, Dm), 0.02, seed=s + 1, device=d)
        self.Wd = inp.normal_bf16((Dm, F), 0.02, seed=s + 2, device=d)
        self.qx = torch.empty((M, Dm), dtype=torch.uint8, device=d)
        self.sx = torch.empty(((Dm + 127) // 128, M), dtype=torch.float32, device=d)
        self.qwu = torch.empty((F, Dm), dtype=torch.uint8, device=d)
        self.swu = torch.empty(((F + 127) // 128, (Dm + 127) // 128), dtype=torch.float32, device=d)
        self.qh = torch.empty((M, F), dtype=torch.uint8, device=d)
        self.sh = torch.empty(((F + 127) // 128, M), dtype=torch.float32, device=d)
        self.qwd = torch.empty((Dm, F), dtype=torch.uint8, device=d)
        self.swd = torch.empty(((Dm + 127) // 128, (F + 127) // 128), dtype=torch.float32, device=d)
        self.Y = torch.empty((M, Dm), dtype=torch.bfloat16, device=d)
        self.dims = (M, Dm, F)
        self.flops = 2 * 2.0 * M * Dm * F
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.launches = 5
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("X", self.X), ("W_up", self.Wu), ("W_down", self.Wd)]
        self.host_output = self.Y

    def _step_blockmlp(self, ev=None):
        f = self.f
        M, Dm, F = self.dims
        f.fp8_quantize_blockwise(self.X, M, Dm, Dm, f.E4M3, 1, self.qx, self.sx)
        f.fp8_quantize_blockwise(self.Wu, F, Dm, Dm, f.E4M3, 128, self.qwu, self.swu)
        if ev:
            ev[0].record()
        # up projection; its epilogue rounds H to bf16 and requantizes it 1x128 (no bf16 H in HBM)
        f.fp8_gemm_block_requant(self.qx, f.E4M3, self.qwu, f.E4M3, M, F, Dm, self.sx, self.swu, None, F, f.E4M3,
                                 self.qh, self.sh)
        if ev:
            ev[1].record()
        f.fp8_quantize_blockwise(self.Wd, Dm, F, F, f.E4M3, 128, self.qwd, self.swd)
        f.fp8_gemm_scaled(self.qh, f.E4M3, self.qwd, f.E4M3, M, Dm, F, f.SCALE_BLOCK, self.sh, self.swd, self.Y, Dm)

    # the same MLP with power-of-two block scales applied by the tensor core
    def _setup_blockmlp_e8m0(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        M, Dm, F = (2048 if self.profile else 8192), 4096, 11008
        img = lambda r, c: torch.empty(f.e8m0_image_bytes(r, c), dtype=torch.uint8, device=d)
        self.X = inp.normal_bf16((M, Dm), 1.0, seed=s, device=d)
        self.Wu = inp.normal_bf16((F, Dm), 0.02, seed=s + 1, device=d)
        self.Wd = inp.normal_bf16((Dm, F), 0.02, seed=s + 2, device=d)
        self.qx, self.sx = torch.empty((M, Dm), dtype=torch.uint8, device=d), img(M, Dm)
        self.qwu, self.swu = torch.empty((F, Dm), dtype=torch.uint8, device=d), img(F, Dm)
        self.qh, self.sh = torch.empty((M, F), dtype=torch.uint8, device=d), img(M, F)
        self.qwd, self.swd = torch.empty((Dm, F), dtype=torch.uint8, device=d), img(Dm, F)
        self.Y = torch.empty((M, Dm), dtype=torch.bfloat16, device=d)
        self.dims = (M, Dm, F)
        self.flops = 2 * 2.0 * M * Dm * F
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.launches = 5
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("X", self.X), ("W_up", self.Wu), ("W_down", self.Wd)]
        self.host_output = self.Y

    def _step_blockmlp_e8m0(self, ev=None):
        f = self.f
        M, Dm, F = self.dims
        f.fp8_quantize_blockwise_e8m0(self.X, M, Dm, Dm, f.E4M3, 1, self.qx, self.sx)
        f.fp8_quantize_blockwise_e8m0(self.Wu, F, Dm, Dm, f.E4M3, 128, self.qwu, self.swu)
        if ev:
            ev[0].record()
        # up projection; its epilogue rounds H to bf16 and requantizes it 1x128 (E8M0 image, no bf16 H in HBM)
        f.fp8_gemm_block_e8m0_requant(self.qx, f.E4M3, self.qwu, f.E4M3, M, F, Dm, self.sx, self.swu, None, F,
                                      f.E4M3, self.qh, self.sh)
        if ev:
            ev[1].record()
        f.fp8_quantize_blockwise_e8m0(self.Wd, Dm, F, F, f.E4M3, 128, self.qwd, self.swd)
        f.fp8_gemm_block_e8m0(self.qh, f.E4M3, self.qwd, f.E4M3, M, Dm, F, self.sh, self.swd, self.Y, Dm)

    # dgrad with delayed scaling
    def _setup_dgrad(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        M, N_out, K_in, T = (2048 if self.profile else 8192), 4096, 4096, (4 if self.profile else 16)
        self.G = [inp.lognormal_grads_bf16((M, N_out), seed=s + 100 + t, device=d) for t in range(T)]
        W = inp.normal_bf16((N_out, K_in), 0.02, seed=s + 1, device=d)
        self.wq, self.wsinv, _ = f.quantize_tensorwise(W, f.E4M3, transpose=True)   # W^T [K_in, N_out]
        del W
        self.hist = f.AmaxHistory(16, f.E5M2, device=d)
        self.qg = torch.empty((M, N_out), dtype=torch.uint8, device=d)
        self.sg = torch.empty(1, dtype=torch.float32, device=d)
        self.am = torch.empty(1, dtype=torch.float32, device=d)
        self.DX = torch.empty((M, K_in), dtype=torch.bfloat16, device=d)
        self.ws = f.gemm_workspace(M, K_in, N_out, f.SCALE_TENSOR, device=d)
        self.t = 0
        self.dims = (M, N_out, K_in)
        self.flops = 2.0 * M * N_out * K_in
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.launches = 3
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("dY_t", self.G[0])]
        self.host_output = self.DX

    def _step_dgrad(self, ev=None):
        f = self.f
        M, N_out, K_in = self.dims
        g = self.G[self.t % len(self.G)]
        self.t += 1
        f.fp8_quantize_tensorwise(g, M, N_out, f.E5M2, self.hist.scale, self.qg, 0, self.sg, self.am)
        if ev:
            ev[0].record()
        f.fp8_gemm_scaled(self.qg, f.E5M2, self.wq, f.E4M3, M, K_in, N_out, f.SCALE_TENSOR, self.sg, self.wsinv,
                          self.DX, K_in, self.ws)
        if ev:
            ev[1].record()
        self.hist.update(self.am)

    # a linear layer's backward under the rowwise_with_gw_hp recipe
    def _setup_bwd_gw_hp(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        T, N_out, K_in = (2048 if self.profile else 8192), 4096, 4096
        self.dY = inp.lognormal_grads_bf16((T, N_out), seed=s + 100, device=d)
        self.X = inp.normal_bf16((T, K_in), 1.0, seed=s + 101, device=d)
        self.W = inp.normal_bf16((N_out, K_in), 0.02, seed=s + 1, device=d)
        self.qdy = torch.empty((T, N_out), dtype=torch.uint8, device=d)
        self.sdy = torch.empty(T, dtype=torch.float32, device=d)
        self.qwT = torch.empty((K_in, N_out), dtype=torch.uint8, device=d)
        self.swT = torch.empty(K_in, dtype=torch.float32, device=d)
        self.awT = torch.empty(K_in, dtype=torch.float32, device=d)
        self.DX = torch.empty((T, K_in), dtype=torch.bfloat16, device=d)
        self.DW = torch.empty((N_out, K_in), dtype=torch.float32, device=d)
        self.dims = (T, N_out, K_in)
        self.flops = 2 * 2.0 * T * N_out * K_in
        self.unit, self.bound = "TFLOP/s", "tensor"
        self.peak_dtype = "bf16"   # the dominant kernel is the bf16 weight-gradient GEMM
        self.launches = 4          # dY rowwise, W^T single-pass transposed rowwise, dgrad GEMM, wgrad GEMM
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("dY", self.dY), ("X", self.X)]
        self.host_output = self.DX

    def _step_bwd_gw_hp(self, ev=None):
        f = self.f
        T, N_out, K_in = self.dims
        f.fp8_quantize_rowwise(self.dY, T, N_out, N_out, f.E5M2, 1, self.qdy, self.sdy)
        f.fp8_quantize_rowwise_transpose(self.W, N_out, K_in, K_in, f.E4M3, 1, self.qwT, self.swT, self.awT)
        f.fp8_gemm_scaled(self.qdy, f.E5M2, self.qwT, f.E4M3, T, K_in, N_out, f.SCALE_ROW, self.sdy, self.swT,
                          self.DX, K_in)
        if ev:
            ev[0].record()
        f.fp8_gemm_bf16_wgrad(self.dY, self.X, T, N_out, K_in, N_out, K_in, self.DW, K_in)
        if ev:
            ev[1].record()

    # FP8 KV cache round trip
    def _setup_kv(self):
        f, inp, d, s = self.f, self.inp, self.dev, self.seed
        B, H, S, Dh = (8 if self.profile else 32), 32, 8192, 128
        self.K = inp.normal_bf16((B, H, S, Dh), 1.0, seed=s, device=d)
        self.V = inp.normal_bf16((B, H, S, Dh), 1.0, seed=s + 1, device=d)
        self.qk = torch.empty(self.K.shape, dtype=torch.uint8, device=d)
        self.qv = torch.empty(self.V.shape, dtype=torch.uint8, device=d)
        self.sk = torch.empty(B * H, dtype=torch.float32, device=d)
        self.sv = torch.empty(B * H, dtype=torch.float32, device=d)
        self.Kd = torch.empty_like(self.K)
        self.Vd = torch.empty_like(self.V)
        self.dims = (B, H, S, Dh)
        n = B * H * S * Dh
        self.bytes = 2 * (3.0 * n + 4 * B * H) * 2    # K and V: quantize (2 B in, 1 B out) + dequantize (1 B in, 2 B out)
        self.kernel_bytes = 3.0 * n + 4 * B * H       # one kv_quant launch
        self.unit, self.bound = "GB/s", "hbm"
        self.launches = 4
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("K", self.K), ("V", self.V)]
        self.host_output = self.Kd

    def _step_kv(self, ev=None):
        f = self.f
        B, H, S, Dh = self.dims
        if ev:
            ev[0].record()
        f.fp8_kv_quant(self.K, B, H, S, Dh, f.E4M3, self.qk, self.sk)
        if ev:
            ev[1].record()
        f.fp8_kv_quant(self.V, B, H, S, Dh, f.E4M3, self.qv, self.sv)
        f.fp8_kv_dequant(self.qk, self.sk, B, H, S, Dh, f.E4M3, self.Kd)
        f.fp8_kv_dequant(self.qv, self.sv, B, H, S, Dh, f.E4M3, self.Vd)

    # paged FP8 KV cache: prefill write of K and V into shuffled 16-token pages,
    # then both read back through the block table
    def _setup_paged(self):
        inp, d, s = self.inp, self.dev, self.seed
        P = inp.PAGED_KV
        B, S, H, Dh, bs = P["B"], P["S"], P["H"], P["Dh"], P["block_size"]
        if self.profile:
            B = 8
        NB = B * S // bs
        table, slots = inp.paged_layout([S] * B, bs, NB, seed=s + 3)
        self.table, self.slots = table.to(d), slots.to(d)
        self.lens = torch.full((B,), S, dtype=torch.int32, device=d)
        self.K = inp.normal_bf16((B * S, H, Dh), 1.0, seed=s, device=d)
        self.V = inp.normal_bf16((B * S, H, Dh), 1.0, seed=s + 1, device=d)
        self.kc = self.f.PagedKVCache(NB, bs, H, Dh, self.f.E4M3, device=d)
        self.vc = self.f.PagedKVCache(NB, bs, H, Dh, self.f.E4M3, device=d)
        self.Kd = torch.empty((B, S, H, Dh), dtype=torch.bfloat16, device=d)
        self.Vd = torch.empty_like(self.Kd)
        self.dims = (B, S, H, Dh, bs, NB)
        T = B * S
        wbytes = 3.0 * T * H * Dh + 4.0 * T * H + 8.0 * T            # bf16 in, FP8 + 1/s out, slot ids
        gbytes = 3.0 * T * H * Dh + 4.0 * T * H + 4.0 * table.numel() + 4.0 * B
        self.bytes = 2 * (wbytes + gbytes)
        self.kernel_bytes = wbytes                                    # one fp8_paged_kv_write launch
        self.unit, self.bound = "GB/s", "hbm"
        self.launches = 4
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("K", self.K), ("V", self.V)]
        self.host_output = self.Kd

    def _step_paged(self, ev=None):
        f = self.f
        B, S, H, Dh, bs, NB = self.dims
        if ev:
            ev[0].record()
        f.fp8_paged_kv_write(self.K, self.slots, B * S, H, Dh, NB * bs, f.E4M3, self.kc.cache, self.kc.scale_inv)
        if ev:
            ev[1].record()
        f.fp8_paged_kv_write(self.V, self.slots, B * S, H, Dh, NB * bs, f.E4M3, self.vc.cache, self.vc.scale_inv)
        mb = self.table.shape[1]
        f.fp8_paged_kv_gather(self.kc.cache, self.kc.scale_inv, self.table, self.lens, B, mb, H, Dh, bs, NB, S,
                              f.E4M3, self.Kd)
        f.fp8_paged_kv_gather(self.vc.cache, self.vc.scale_inv, self.table, self.lens, B, mb, H, Dh, bs, NB, S,
                              f.E4M3, self.Vd)

    # scale health check over every layer's rowwise scales
    def _setup_health(self):
        inp, d = self.inp, self.dev
        L, n = inp.SCALE_HEALTH["layers"], inp.SCALE_HEALTH["per_layer"]
        if self.profile:
            L *= 8     # inputs above L2 size for the DRAM counters
        prev, cur = inp.scale_snapshots_f32(L * n, seed=self.seed + 7)
        self.prev, self.cur = prev.to(d), cur.to(d)
        self.offs = (torch.arange(L + 1, dtype=torch.int64) * n).to(d)
        self.stats = torch.empty((L, 3), dtype=torch.float32, device=d)
        self.counts = torch.empty((L, 2), dtype=torch.int32, device=d)
        self.dims = (L, n)
        self.bytes = 2 * 4.0 * L * n + 8 * (L + 1) + 20 * L
        self.kernel_bytes = self.bytes
        self.unit, self.bound = "GB/s", "hbm"
        self.launches = 1
        self.config = config_of(self.name, self.profile)
        self.host_inputs = [("cur", self.cur)]
        self.host_output = self.stats

    def _step_health(self, ev=None):
        L, n = self.dims
        if ev:
            ev[0].record()
        self.f.fp8_scale_stats(self.cur, self.prev, L * n, self.offs, L, 4.0, self.stats, self.counts)
        if ev:
            ev[1].record()

    def step(self, ev=None):
        getattr(self, "_step_" + self.name)(ev)

    def next_inputs(self):
        """The device tensors the next step reads, in host_inputs order (the
        dgrad workload cycles through its 16 per-step gradients)."""
        if self.name == "dgrad":
            return [self.G[self.t % len(self.G)]]
        return [t for _, t in self.host_inputs]

    def work(self):
        return self.flops / 1e12 if self.unit == "TFLOP/s" else self.bytes / 1e9

    def kernel_work(self):
        """Work of one launch of the dominant kernel (events ev[0]..ev[1])."""
        if self.unit == "TFLOP/s":
            if self.name in ("blockmlp", "blockmlp_e8m0"):
                M, Dm, F = self.dims
                return 2.0 * M * Dm * F / 1e12
            if self.name == "bwd_gw_hp":
                T, N_out, K_in = self.dims
                return 2.0 * T * N_out * K_in / 1e12
            return self.flops / 1e12
        return self.kernel_bytes / 1e9


# --------------------------------------------------------- CPU (oracle) arm --

def host_cores() -> int:
    """Host threads this process may run on (its CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class _Phases:
    """Timed phases of the oracle sample.  Each phase is a list of independent
    jobs (oracle calls on disjoint rows, columns, outputs, slices or
    segments); the oracle is C called through ctypes, which releases the GIL,
    so a thread pool runs the jobs on separate cores.  A phase's wall time,
    times the phase's extrapolation factor, adds to the full-step estimate."""

    def __init__(self, pool):
        self.pool = pool
        self.total = 0.0

    def run(self, factor, jobs):
        t0 = time.perf_counter()
        out = [j() for j in jobs] if self.pool is None else list(self.pool.map(lambda j: j(), jobs))
        self.total += factor * (time.perf_counter() - t0)
        return out


def _chunks(n: int, parts: int):
    parts = max(1, min(n, parts))
    b = [n * i // parts for i in range(parts + 1)]
    return [(b[i], b[i + 1]) for i in range(parts) if b[i + 1] > b[i]]


def cpu_sample(name: str, seed: int = 0, pool=None, threads: int = 1):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload,
    on `threads` host threads (pool: a ThreadPoolExecutor of that size, or
    None for one thread); returns (value in the workload's unit for a full
    step, sample description)."""
    import numpy as np
    from fp8_scaled_quantization_amax_b200 import inputs
    from oracle import oracle as orc
    orc.lib()
    ph = _Phases(pool)
    parts = 4 * threads
    C = np.ascontiguousarray

    def rows_job(fn, x, r0, r1, *a):
        piece = C(x[r0:r1])
        return lambda: fn(piece, *a)

    def gemm_jobs(A, fa, B, fb, mode, da, db, im, inn):
        return [(lambda lo=lo, hi=hi: orc.gemm_scaled_sampled(A, fa, B, fb, mode, da, db, im[lo:hi], inn[lo:hi]))
                for lo, hi in _chunks(im.size, parts)]

    if name == "bwd_gw_hp":
        T, N_out, K_in = 8192, 4096, 4096
        r = 8
        g = inputs.bf16_bits(inputs.lognormal_grads_bf16((T, N_out), seed=seed))
        x = inputs.bf16_bits(inputs.normal_bf16((T, K_in), 1.0, seed=seed + 1))
        w = inputs.bf16_bits(inputs.normal_bf16((N_out, K_in), 0.02, seed=seed + 2))
        cols = [C(w[:, c0:c1]) for c0, c1 in _chunks(K_in, parts)]
        res = ph.run(1.0, [(lambda p=p: orc.quantize_rowwise_transpose(p, 0, True)) for p in cols])
        qwT, swT = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res])
        res = ph.run((T / r) * (K_in / 256), [rows_job(orc.quantize_rowwise, g, i, i + 1, 1, True) for i in range(r)])
        qg, sg = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res])
        im, inn = np.repeat(np.arange(r), 256), np.tile(np.arange(256), r)
        ph.run((T / r) * (K_in / 256), gemm_jobs(qg, 1, qwT, 0, 1, sg, swT, im, inn))
        wm, wn = np.repeat(np.arange(2), 64), np.tile(np.arange(64), 2)
        ph.run(N_out * K_in / 128, [(lambda lo=lo, hi=hi: orc.gemm_bf16_wgrad_sampled(g, x, wm[lo:hi], wn[lo:hi]))
                                    for lo, hi in _chunks(wm.size, parts)])
        return 4.0 * T * N_out * K_in / ph.total / 1e12, (
            f"all of W^T quantized, {r} dY rows quantized and {r}x256 dX outputs (K=4096), 128 dW outputs "
            "over all 8192 tokens; the dX and dW parts scaled to the full layer")
    if name == "blockmlp_e8m0":
        name = "blockmlp"   # the same per-block GEMM in the oracle (its cost does not depend on the scale rule)
    if name == "rowwise":
        M = N = K = 4096
        r = 8
        a = inputs.bf16_bits(inputs.outlier_activations_bf16((r, K), seed=seed))
        b = inputs.bf16_bits(inputs.normal_bf16((N, K), 0.02, seed=seed + 1))
        res = ph.run(1.0, [rows_job(orc.quantize_rowwise, b, r0, r1, 0, True) for r0, r1 in _chunks(N, parts)])
        qb, sb = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res])
        res = ph.run(M / r, [rows_job(orc.quantize_rowwise, a, i, i + 1, 0, True) for i in range(r)])
        qa, sa = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res])
        im, inn = np.repeat(np.arange(r), N), np.tile(np.arange(N), r)
        ph.run(M / r, gemm_jobs(qa, 0, qb, 0, 1, sa, sb, im, inn))
        return 2.0 * M * N * K / ph.total / 1e12, (
            f"rowwise-quantize all of B [4096,4096] + {r} rows of A, then those {r}x4096 outputs "
            f"(fp64 sums); full step extrapolated as t_B + (4096/{r}) x t_rows")
    if name == "tensor":
        M = N = K = 256
        a = inputs.bf16_bits(inputs.normal_bf16((M, K), 1.0, seed=seed))
        b = inputs.bf16_bits(inputs.normal_bf16((N, K), 1.0, seed=seed + 1))
        reps = 10
        im, inn = np.repeat(np.arange(M), N), np.tile(np.arange(N), M)
        for _ in range(reps):
            (qa, sa, _, _), (qb, sb, _, _) = ph.run(1.0 / reps, [lambda: orc.quantize_tensorwise(a, 0),
                                                                 lambda: orc.quantize_tensorwise(b, 0)])
            ph.run(1.0 / reps, gemm_jobs(qa, 0, qb, 0, 0, np.float32([sa]), np.float32([sb]), im, inn))
        return 2.0 * M * N * K / ph.total / 1e12, "the whole 256^3 per-tensor step, mean of 10"
    if name == "blockmlp":
        M, Dm, F = 8192, 4096, 11008
        r = 32
        wrows = 128 * max(2, min(threads, 86))
        x = inputs.bf16_bits(inputs.normal_bf16((r, Dm), 1.0, seed=seed))
        w = inputs.bf16_bits(inputs.normal_bf16((wrows, Dm), 0.02, seed=seed + 1))
        res = ph.run((F / wrows) * 2, [rows_job(orc.quantize_blockwise, w, r0, r0 + 128, 0, 128)
                                       for r0 in range(0, wrows, 128)])
        qw, sw = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res])
        res = ph.run((M / r) * (F / 256) * 2, [rows_job(orc.quantize_blockwise, x, i, i + 1, 0, 1) for i in range(r)])
        qx, sx = np.concatenate([q for q, _ in res]), np.concatenate([s_ for _, s_ in res], axis=1)
        im, inn = np.repeat(np.arange(r), 256), np.tile(np.arange(256), r)
        ph.run((M / r) * (F / 256) * 2, gemm_jobs(qx, 0, qw, 0, 2, C(sx), sw, im, inn))
        return 4.0 * M * Dm * F / ph.total / 1e12, (
            f"blockwise-quantize {wrows} W rows and {r} X rows, then {r}x256 outputs at K=4096; "
            "scaled to both MLP GEMMs")
    if name == "dgrad":
        M, N_out, K_in = 8192, 4096, 4096
        r = 128
        g = inputs.bf16_bits(inputs.lognormal_grads_bf16((r, N_out), seed=seed))
        w = inputs.bf16_bits(inputs.normal_bf16((256, N_out), 0.02, seed=seed + 1))
        f = (M / r) * (K_in / 256)
        jobs = [lambda: orc.quantize_tensorwise(w, 0)] + [
            (lambda p=C(g[r0:r1]): orc.quantize_tensorwise(p, 1, scale_in=1.0)) for r0, r1 in _chunks(r, parts)]
        res = ph.run(f, jobs)
        qw, sw = res[0][0], res[0][1]
        qg, sg = np.concatenate([q[0] for q in res[1:]]), res[1][1]
        im, inn = np.repeat(np.arange(r), 256), np.tile(np.arange(256), r)
        ph.run(f, gemm_jobs(qg, 1, qw, 0, 0, np.float32([sg]), np.float32([sw]), im, inn))
        return 2.0 * M * N_out * K_in / ph.total / 1e12, (
            f"quantize {r} gradient rows (E5M2) + 256 weight rows, then {r}x256 outputs; scaled to the step")
    if name == "paged":
        P = inputs.PAGED_KV
        B, S, H, Dh, bs = P["B"], P["S"], P["H"], P["Dh"], P["block_size"]
        per = 256
        nseq = max(8, min(2 * threads, 128))
        r = per * nseq
        x = inputs.bf16_bits(inputs.normal_bf16((r, H, Dh), 1.0, seed=seed))
        subs = []
        for i in range(nseq):
            table, slots = inputs.paged_layout([per], bs, per // bs, seed=seed + 3 + i)
            subs.append((C(x[i * per:(i + 1) * per]), slots.numpy(), table.numpy()))

        def one(xi, sl, tb):
            c, sc = orc.paged_kv_write(xi, sl, np.zeros((per // bs, bs, H, Dh), np.uint8),
                                       np.zeros((per // bs, bs, H), np.float32), 0)
            orc.paged_kv_gather(c, sc, tb, np.array([per], np.int32), per, 0)

        ph.run((B * S / r) * 2, [(lambda t=t: one(*t)) for t in subs])
        T = B * S
        full = 2 * (2 * (3.0 * T * H * Dh + 4.0 * T * H) + 8.0 * T + 4.0 * T / bs + 4.0 * B)
        return full / ph.total / 1e9, (f"{r} tokens of K ({nseq} sequences of {per}) written and gathered; "
                                       f"scaled to K and V of all {B}x{S} tokens")
    if name == "health":
        L, n = inputs.SCALE_HEALTH["layers"], inputs.SCALE_HEALTH["per_layer"]
        prev, cur = inputs.scale_snapshots_f32(L * n, seed=seed + 7)
        p, c = prev.numpy(), cur.numpy()
        reps = 20
        segs = [(C(c[g * n:(g + 1) * n]), C(p[g * n:(g + 1) * n])) for g in range(L)]

        def some(g0, g1):   # a job takes several segments: one is too little work for a thread hand-off
            for a, b in segs[g0:g1]:
                orc.scale_stats(a, b, 4.0)

        groups = _chunks(L, threads)
        for _ in range(reps):
            ph.run(1.0 / reps, [(lambda g0=g0, g1=g1: some(g0, g1)) for g0, g1 in groups])
        return (2 * 4.0 * L * n + 8 * (L + 1) + 20 * L) / ph.total / 1e9, "the whole step (all 224 segments), mean of 20"
    # kv
    B, H, S, Dh = 32, 32, 8192, 128
    ns = max(16, min(2 * threads, 256))
    k = inputs.bf16_bits(inputs.normal_bf16((1, ns, S, Dh), 1.0, seed=seed))
    slices = [C(k[:, i:i + 1]) for i in range(ns)]

    def kv_one(sl):
        q, sc = orc.kv_quant(sl, 0)
        orc.kv_dequant(q, sc, 0)

    ph.run(B * H * 2 / ns, [(lambda sl=sl: kv_one(sl)) for sl in slices])
    n = B * H * S * Dh
    return 2 * (3.0 * n) * 2 / ph.total / 1e9, f"{ns} of the 2048 (b,h) slices of K/V quantized and dequantized; scaled"


def cpu_baseline(name: str, seed: int = 0):
    """The oracle on all host threads this process may use and on one thread,
    on the same bounded sample: (value, threads, one-thread value,
    description), where value and threads are the faster of the two runs (a
    sample of many tiny oracle calls can run slower on many threads, whose
    hand-offs go through the interpreter lock)."""
    import concurrent.futures as cf
    threads = host_cores()
    v1, desc = cpu_sample(name, seed)
    if threads == 1:
        return v1, 1, v1, desc
    with cf.ThreadPoolExecutor(max_workers=threads) as pool:
        vall, desc = cpu_sample(name, seed, pool=pool, threads=threads)
    return (vall, threads, v1, desc) if vall >= v1 else (v1, 1, v1, desc)


# -------------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="blockmlp", choices=list(DEFAULT_STEPS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="reduced-size case for ncu captures (<= ~2.5 GB on the device); prints no bench value")
    args = ap.parse_args()
    steps = args.steps if args.steps is not None else DEFAULT_STEPS[args.workload]
    warmup = max(3, args.warmup)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    unit = "GB/s" if args.workload in ("kv", "paged", "health") else "TFLOP/s"

    if args.impl == "reference":
        if rank != 0:
            return
        # one untimed sample (the CPU oracle needs no more warm-up), then as many
        # timed samples as --steps asks for within a ~2.5 minute budget
        import concurrent.futures as cf
        threads = host_cores()
        vals = []
        desc = ""
        with cf.ThreadPoolExecutor(max_workers=threads) as pool:
            t0 = time.perf_counter()
            cpu_sample(args.workload, pool=pool, threads=threads)
            per = max(time.perf_counter() - t0, 1e-3)
            n = max(1, min(steps if args.steps is not None else 3, int(150.0 / per)))
            for i in range(n):
                v, desc = cpu_sample(args.workload, seed=i, pool=pool, threads=threads)
                vals.append(v)
        v = statistics.mean(vals)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
                "steps": len(vals), "warmup": 1, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64 sums / fp32 scales (CPU oracle)", "data": "synthetic",
                "config": config_of(args.workload),
                "cpu_baseline": {"value": v, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc},
                "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        from fp8_scaled_quantization_amax_b200.dist import max_over_ranks as mor
        return mor(x, device=dev)

    from fp8_scaled_quantization_amax_b200 import fp8q
    fp8q.lib()
    wl = Workload(args.workload, dev, seed=1000 * rank, profile=args.profile)
    # L2 flush before every step: write 256 MiB, then read another 256 MiB so
    # the flush's own dirty lines are written back before the step starts
    flush_w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    class _Flush:
        @staticmethod
        def zero_():
            flush_w.zero_()
            flush_r.sum()

    flush = _Flush()
    stream = torch.cuda.current_stream(dev)

    for _ in range(warmup):
        flush.zero_()
        wl.step()
    torch.cuda.synchronize(dev)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        t_wall0 = time.perf_counter()
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            wl.step(kev[i])
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall0
        barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kern_ms = [a.elapsed_time(b) for a, b in kev]
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / steps
    value = world * wl.work() * steps / (total_ms * 1e-3)
    kern_avg_ms = max_over_ranks(statistics.mean(kern_ms))
    # spread of the per-step device times (this rank's; the value above uses their sum)
    step_med_ms, step_best_ms = statistics.median(step_ms), min(step_ms)
    kern_med_ms, kern_best_ms = statistics.median(kern_ms), min(kern_ms)

    if args.profile:
        assert fp8q.fp8_device_error(clear=True) == 0, "a kernel gave up a bounded wait"
        if rank == 0:
            print(json.dumps({"profile": True, "workload": args.workload, "steps": steps,
                              "kernel_ms": kern_avg_ms, "config": wl.config}))
        return

    # end to end through the public API, run the way a training or serving
    # loop runs it: every step uploads its inputs from pinned host memory and
    # reads its result back, on copy streams of their own with two device
    # staging slots each way, so step i's upload overlaps step i-1's kernels
    # and step i's read-back overlaps step i+1's.  Each step's full input and
    # result bytes still cross PCIe inside the timed region (first upload to
    # last read-back).  No L2 flush here: each step's inputs arrive fresh.
    e2e_steps = min(steps, 20 if wl.unit == "TFLOP/s" and args.workload not in ("blockmlp", "blockmlp_e8m0") else 6)
    host_in = [t.detach().cpu().pin_memory() for _, t in wl.host_inputs]
    host_out = [torch.empty(wl.host_output.shape, dtype=wl.host_output.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out[0].numel() * host_out[0].element_size()
    stage_in = [[torch.empty_like(t) for _, t in wl.host_inputs] for _ in range(2)]
    stage_out = [torch.empty_like(wl.host_output) for _ in range(2)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_up, ev_in_free, ev_done, ev_back = ([ev() for _ in range(e2e_steps)] for _ in range(4))
    t_beg, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_beg.record(stream)
    s_up.wait_event(t_beg)
    for i in range(e2e_steps):
        slot = i % 2
        with torch.cuda.stream(s_up):   # upload step i's inputs into the staging slot
            if i >= 2:
                s_up.wait_event(ev_in_free[i - 2])
            for h, d in zip(host_in, stage_in[slot]):
                d.copy_(h, non_blocking=True)
            ev_up[i].record(s_up)
        stream.wait_event(ev_up[i])      # step i on the compute stream
        for d, w in zip(stage_in[slot], wl.next_inputs()):
            w.copy_(d, non_blocking=True)
        ev_in_free[i].record(stream)
        wl.step()
        if i >= 2:
            stream.wait_event(ev_back[i - 2])
        stage_out[slot].copy_(wl.host_output, non_blocking=True)
        ev_done[i].record(stream)
        with torch.cuda.stream(s_down):  # read step i's result back
            s_down.wait_event(ev_done[i])
            host_out[slot].copy_(stage_out[slot], non_blocking=True)
            ev_back[i].record(s_down)
    stream.wait_event(ev_back[e2e_steps - 1])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(t_beg.elapsed_time(t_end) / e2e_steps)
    e2e_value = world * wl.work() / (e2e_ms * 1e-3)
    assert fp8q.fp8_device_error(clear=True) == 0, "a kernel gave up a bounded wait"

    clocks = clk.summary()
    peak, peak_src = choose_peak(wl.bound, getattr(wl, "peak_dtype", "fp8"), clocks, peaks())
    achieved = wl.kernel_work() / (kern_avg_ms * 1e-3)

    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, threads, v1, desc = cpu_baseline(args.workload)
        cpu = {"value": v, "unit": wl.unit, "cores": threads, "kind": "oracle", "sample": desc,
               "value_1_core": v1}
    dtype = {"rowwise": "fp8_e4m3 x fp8_e4m3 -> f32 accumulate -> bf16",
             "tensor": "fp8_e4m3 x fp8_e4m3 -> f32 accumulate -> bf16",
             "blockmlp": "fp8_e4m3 x fp8_e4m3 -> f32 accumulate (per-128-K promotion) -> bf16",
             "blockmlp_e8m0": "fp8_e4m3 x fp8_e4m3, e8m0 block scales in the MMA -> f32 accumulate -> bf16",
             "dgrad": "fp8_e5m2 x fp8_e4m3 -> f32 accumulate -> bf16",
             "bwd_gw_hp": "dgrad fp8_e5m2 x fp8_e4m3 -> bf16; wgrad bf16 x bf16 -> f32",
             "kv": "bf16 <-> fp8_e4m3 (f32 scale)",
             "paged": "bf16 <-> fp8_e4m3 (f32 scale per token and head)",
             "health": "f32 scales, f64 sums"}[args.workload]
    cfg = dict(wl.config)
    cfg["l2"] = "flushed before every step (256 MiB write + 256 MiB read, outside the step's events)"
    line = {
        "metric": METRIC, "value": value, "unit": wl.unit, "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms_per_step, "ms_per_step_median": step_med_ms, "ms_per_step_best": step_best_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic (seeded, per rank)", "config": cfg,
        "roofline": {"bound": wl.bound, "achieved": achieved, "peak": peak, "unit": wl.unit,
                     "frac": achieved / peak, "traffic": recorded_traffic(args.workload),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                     "kernel": {"kv": "fp8_kv_quant", "paged": "fp8_paged_kv_write",
                                "health": "fp8_scale_stats", "bwd_gw_hp": "fp8_gemm_bf16_wgrad",
                                "blockmlp_e8m0": "fp8_gemm_block_e8m0_requant (up projection with its 1x128 requantization)",
                                "blockmlp": "fp8_gemm_block_requant (up projection with its 1x128 requantization)"
                                }.get(args.workload, "fp8_gemm_scaled"),
                     "kernel_ms": kern_avg_ms, "kernel_ms_median": kern_med_ms, "kernel_ms_best": kern_best_ms,
                     "peak_source": peak_src},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": wl.unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "schedule": "uploads and read-backs on their own streams, overlapping the neighbouring steps"},
        "gpu_launches": wl.launches * steps,
        "clocks": clocks,
        "wall_s_timed_region": t_wall,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    try:
        main()
    finally:
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
