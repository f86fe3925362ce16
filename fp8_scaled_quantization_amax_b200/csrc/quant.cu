// quant.cu -- amax and the three quantizers (per-tensor, per-row, per-block).
//
// Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-tensor,
// per-row and per-block scaling; delayed scaling), §4.2 (max-absolute-value
// statistics); "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
// "FP8 三种缩放配方怎么选" (tensorwise; rowwise with power-of-two e4m3 scales).
//
// All kernels are HBM-bound streams: 16-byte coalesced loads of bf16, 8- or
// 16-byte stores of FP8, the amax folded into the same pass wherever the scale
// does not depend on it (per-row and per-block data stays in registers between
// the amax and the cast, so each element is read from HBM exactly once).
#include <algorithm>

#include <cooperative_groups.h>
#include <type_traits>

#include "common.cuh"

using namespace fp8q;
using fp8q_host::pdl_launch;

namespace {

constexpr int kStreamThreads = 512;

// ------------------------------------------------------------------ amax --
// Grid-stride max over 8-element vectors; one atomicMax per CTA on the fp32
// bit pattern of the non-negative result (monotone as an unsigned integer).
__global__ void __launch_bounds__(kStreamThreads) k_amax(const uint4 *__restrict__ xv, int64_t nvec,
                                                         const uint16_t *__restrict__ xs, int64_t n,
                                                         uint32_t *__restrict__ amax_bits,
                                                         uint32_t *__restrict__ counts) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    __shared__ uint32_t red[32];
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m2 = 0;
    int64_t i = tid;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 a = ld_stream(xv + i), b = ld_stream(xv + i + stride);
        uint4 c = ld_stream(xv + i + 2 * stride), d = ld_stream(xv + i + 3 * stride);
        m2 = amax_fast8(amax_fast8(amax_fast8(amax_fast8(m2, a), b), c), d);
    }
    for (; i < nvec; i += stride) m2 = amax_fast8(m2, ld_stream(xv + i));
    uint32_t m = amax_fast_final(m2), bad = 0;
    if (m == 0xFFFFFFFFu) {   // a NaN or Inf among this thread's elements: exact pass
        m = 0;
        for (int64_t j = tid; j < nvec; j += stride) m = amax_exact8(m, ld_stream(xv + j), bad);
    }
    for (int64_t j = nvec * 8 + tid; j < n; j += stride) {   // tail (< 8 elements)
        uint32_t h = xs[j] & 0x7FFFu;
        if (h < 0x7F80u) m = h > m ? h : m; else ++bad;
    }
    m = block_max_u32(m, red);
    if (counts) bad = block_sum_u32(bad, red);
    if (threadIdx.x == 0) {
        atomicMax(amax_bits, m << 16);
        if (counts && bad) atomicAdd(counts, bad);
    }
}

// -------------------------------------------------- tensorwise cast pass --
// q = cast(x * s) over 16-element units (two 16-byte loads, one 16-byte
// store).  s comes from *scale_in (delayed scaling) or from *amax_in
// (current scaling, written by k_amax earlier on the same stream).
// AMAX: also reduce this tensor's amax into amax_bits (delayed scaling feeds
// it to the history).  COUNT: count non-finite and saturated elements.
template <int FMT, bool AMAX, bool COUNT>
__global__ void __launch_bounds__(kStreamThreads)
k_cast_tensor(const uint4 *__restrict__ xv, uint4 *__restrict__ qv, int64_t nunit,
              const uint16_t *__restrict__ xs, uint8_t *__restrict__ qs, int64_t n,
              const float *__restrict__ scale_in, const float *__restrict__ amax_in,
              float *__restrict__ scale_inv_out, uint32_t *__restrict__ amax_bits,
              uint32_t *__restrict__ nf_ctr, uint32_t *__restrict__ sat_ctr) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    __shared__ uint32_t red[32];
    constexpr float fm = fmax_of<FMT>();
    const float s = scale_in ? *scale_in : scale_from_amax(*amax_in, fm);
    if (blockIdx.x == 0 && threadIdx.x == 0) *scale_inv_out = __fdiv_rn(1.0f, s);
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t m2 = 0;
    int64_t i = tid;
    for (; i + stride < nunit; i += 2 * stride) {
        uint4 a0 = ld_stream(xv + 2 * i), a1 = ld_stream(xv + 2 * i + 1);
        uint4 b0 = ld_stream(xv + 2 * (i + stride)), b1 = ld_stream(xv + 2 * (i + stride) + 1);
        if (AMAX || COUNT) m2 = amax_fast8(amax_fast8(amax_fast8(amax_fast8(m2, a0), a1), b0), b1);
        uint2 qa0 = cast8<FMT>(a0, s), qa1 = cast8<FMT>(a1, s);
        uint2 qb0 = cast8<FMT>(b0, s), qb1 = cast8<FMT>(b1, s);
        qv[i] = make_uint4(qa0.x, qa0.y, qa1.x, qa1.y);
        qv[i + stride] = make_uint4(qb0.x, qb0.y, qb1.x, qb1.y);
    }
    for (; i < nunit; i += stride) {
        uint4 a0 = ld_stream(xv + 2 * i), a1 = ld_stream(xv + 2 * i + 1);
        if (AMAX || COUNT) m2 = amax_fast8(amax_fast8(m2, a0), a1);
        uint2 qa0 = cast8<FMT>(a0, s), qa1 = cast8<FMT>(a1, s);
        qv[i] = make_uint4(qa0.x, qa0.y, qa1.x, qa1.y);
    }
    // tail (< 16 elements), exact and scalar
    uint32_t mt = 0, badt = 0, satt = 0;
    for (int64_t j = nunit * 16 + tid; j < n; j += stride) {
        uint32_t h = xs[j];
        float y = __fmul_rn(__uint_as_float(h << 16), s);
        qs[j] = (uint8_t)(cvt2<FMT>(y, 0.0f) & 0xFFu);
        uint32_t a = h & 0x7FFFu;
        if (a < 0x7F80u) mt = a > mt ? a : mt; else ++badt;
        if (fabsf(y) > fm) ++satt;
    }
    if (AMAX || COUNT) {
        uint32_t m = amax_fast_final(m2), bad = 0, sat = 0;
        const bool nonfinite = (m == 0xFFFFFFFFu);
        const bool maybe_sat = COUNT && !nonfinite && __fmul_rn(bf16bits_to_float(m), s) > fm;
        if (nonfinite || maybe_sat) {   // rare: redo this thread's units exactly
            m = 0;
            for (int64_t j = tid; j < nunit; j += stride) {
                uint4 a0 = ld_stream(xv + 2 * j), a1 = ld_stream(xv + 2 * j + 1);
                m = amax_exact8(amax_exact8(m, a0, bad), a1, bad);
                if (COUNT) sat += count_sat8(a0, s, fm) + count_sat8(a1, s, fm);
            }
        }
        m = mt > m ? mt : m;
        bad += badt;
        sat += satt;
        m = block_max_u32(m, red);
        if (COUNT) {
            bad = block_sum_u32(bad, red);
            sat = block_sum_u32(sat, red);
        }
        if (threadIdx.x == 0) {
            if (AMAX) atomicMax(amax_bits, m << 16);
            if (COUNT && nf_ctr && bad) atomicAdd(nf_ctr, bad);
            if (COUNT && sat_ctr && sat) atomicAdd(sat_ctr, sat);
        }
    }
}

// ------------------------------------ small tensors: amax + cast fused --
// Current scaling of a small tensor (at most kSmallTensor elements) in one
// launch: a single 1024-thread CTA loads the whole tensor into registers
// (thread t holds the 8-element vectors t, t + 1024, ..., all loads in
// flight at once), takes the exact amax (the k_amax arithmetic), derives the
// scale and casts from the registers (the k_cast_tensor arithmetic), so HBM
// is read once.  The memset, amax and cast launches of the general path
// cost more than the work here.  Outputs and counters are the general
// path's: amax_out = max |x| over the finite elements, nf_ctr += non-finite
// count, sat_ctr += saturated count.
constexpr int kSmallThreads = 1024;
constexpr int kSmallVecs = 8;   // 8-element vectors per thread
constexpr int64_t kSmallTensor = (int64_t)kSmallThreads * kSmallVecs * 8;
template <int FMT>
__global__ void __launch_bounds__(kSmallThreads)
k_quant_tensor_small(const uint4 *__restrict__ xv, const uint16_t *__restrict__ xs, int64_t n,
                     uint8_t *__restrict__ q, uint32_t *__restrict__ amax_bits, float *__restrict__ scale_inv_out,
                     uint32_t *__restrict__ nf_ctr, uint32_t *__restrict__ sat_ctr) {
    pdl_trigger();
    pdl_wait();
    __shared__ uint32_t red[32];
    constexpr float fm = fmax_of<FMT>();
    const int tid = threadIdx.x;
    const int nvec = (int)(n / 8);
    uint4 v[kSmallVecs];
#pragma unroll
    for (int k = 0; k < kSmallVecs; ++k) {
        const int i = tid + k * kSmallThreads;
        v[k] = i < nvec ? ld_stream(xv + i) : make_uint4(0, 0, 0, 0);   // zeros do not move the max
    }
    uint32_t m2 = 0;
#pragma unroll
    for (int k = 0; k < kSmallVecs; ++k) m2 = amax_fast8(m2, v[k]);
    uint32_t m = amax_fast_final(m2), bad = 0;
    if (m == 0xFFFFFFFFu) {   // a NaN or Inf among this thread's elements: exact pass
        m = 0;
#pragma unroll
        for (int k = 0; k < kSmallVecs; ++k) m = amax_exact8(m, v[k], bad);
    }
    for (int64_t j = (int64_t)nvec * 8 + tid; j < n; j += kSmallThreads) {   // tail (< 8 elements)
        uint32_t h = xs[j] & 0x7FFFu;
        if (h < 0x7F80u) m = h > m ? h : m; else ++bad;
    }
    m = block_max_u32(m, red);
    if (nf_ctr) bad = block_sum_u32(bad, red);
    const float s = scale_from_amax(__uint_as_float(m << 16), fm);
    if (tid == 0) {
        *amax_bits = m << 16;
        *scale_inv_out = __fdiv_rn(1.0f, s);
        if (nf_ctr && bad) atomicAdd(nf_ctr, bad);
    }
    uint32_t sat = 0;
#pragma unroll
    for (int k = 0; k < kSmallVecs; ++k) {
        const int i = tid + k * kSmallThreads;
        if (i < nvec) {
            *reinterpret_cast<uint2 *>(q + (int64_t)i * 8) = cast8<FMT>(v[k], s);
            if (sat_ctr) sat += count_sat8(v[k], s, fm);
        }
    }
    for (int64_t j = (int64_t)nvec * 8 + tid; j < n; j += kSmallThreads) {   // tail, exact and scalar
        uint32_t h = xs[j];
        float y = __fmul_rn(__uint_as_float(h << 16), s);
        q[j] = (uint8_t)(cvt2<FMT>(y, 0.0f) & 0xFFu);
        if (fabsf(y) > fm) ++sat;
    }
    if (sat_ctr) {
        sat = block_sum_u32(sat, red);
        if (tid == 0 && sat) atomicAdd(sat_ctr, sat);
    }
}

// ---------------------------------------- tensorwise cast with transpose --
// 64x64 tiles: coalesced 16-byte bf16 loads, the FP8 codes written transposed
// into shared memory, then coalesced 16-byte stores of the [cols, rows] output.
template <int FMT, bool AMAX, bool COUNT>
__global__ void __launch_bounds__(256)
k_cast_transpose(const uint16_t *__restrict__ x, uint8_t *__restrict__ qt, int64_t rows, int64_t cols,
                 const float *__restrict__ scale_in, const float *__restrict__ amax_in,
                 float *__restrict__ scale_inv_out, uint32_t *__restrict__ amax_bits,
                 uint32_t *__restrict__ nf_ctr, uint32_t *__restrict__ sat_ctr) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    __shared__ __align__(16) uint8_t tile[64][64 + 16];
    __shared__ uint32_t red[32];
    constexpr float fm = fmax_of<FMT>();
    const float s = scale_in ? *scale_in : scale_from_amax(*amax_in, fm);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *scale_inv_out = __fdiv_rn(1.0f, s);
    const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
    uint32_t m = 0, bad = 0, sat = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int u = threadIdx.x + h * 256;
        const int row = u >> 3, cv = u & 7;
        const int64_t gr = r0 + row, gc = c0 + cv * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (gr < rows && gc < cols) v = ld_stream(reinterpret_cast<const uint4 *>(x + gr * cols + gc));
        if (AMAX || COUNT) {
            m = amax_exact8(m, v, bad);
            if (COUNT) sat += count_sat8(v, s, fm);
        }
        uint2 c = cast8<FMT>(v, s);
#pragma unroll
        for (int j = 0; j < 4; ++j) tile[cv * 8 + j][row] = (uint8_t)(c.x >> (8 * j));
#pragma unroll
        for (int j = 0; j < 4; ++j) tile[cv * 8 + 4 + j][row] = (uint8_t)(c.y >> (8 * j));
    }
    __syncthreads();
    {
        const int oc = threadIdx.x >> 2, part = threadIdx.x & 3;
        const int64_t go = c0 + oc, gi = r0 + part * 16;
        if (go < cols && gi < rows)
            *reinterpret_cast<uint4 *>(qt + go * rows + gi) = *reinterpret_cast<const uint4 *>(&tile[oc][part * 16]);
    }
    if (AMAX || COUNT) {
        m = block_max_u32(m, red);
        if (COUNT) {
            bad = block_sum_u32(bad, red);
            sat = block_sum_u32(sat, red);
        }
        if (threadIdx.x == 0) {
            if (AMAX) atomicMax(amax_bits, m << 16);
            if (COUNT && nf_ctr && bad) atomicAdd(nf_ctr, bad);
            if (COUNT && sat_ctr && sat) atomicAdd(sat_ctr, sat);
        }
    }
}

// ------------------------------------------- rowwise of the transpose ----
// The backward GEMMs contract over a dimension that is not contiguous in
// memory, so their K-major FP8 operands are transposes, quantized rowwise
// (one scale per row of x^T = per column of x).  Two passes: k_colamax
// reduces every column's amax over all rows into fp32 bits (atomicMax on
// non-negative floats as integers: order-independent, so deterministic);
// k_cast_transpose_col casts 64x64 tiles with per-column scales and writes
// them transposed.  The second pass re-reads x, from L2 when x fits.
constexpr int kColRows = 256;   // rows per k_colamax CTA

// |x| of two bf16, non-finite halves replaced by 0 (so they never win a max)
__device__ __forceinline__ uint32_t abs_finite2(uint32_t w) {
    const uint32_t a = w & 0x7FFF7FFFu;
    return a & __vcmpltu2(a, 0x7F807F80u);
}

__global__ void __launch_bounds__(256)
k_colamax(const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint32_t *__restrict__ amax_bits) {
    __shared__ uint4 red[8][32];
    const int cg = threadIdx.x & 31, sub = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 256 + cg * 8;
    const int64_t r0 = (int64_t)blockIdx.y * kColRows;
    const int64_t r1 = min(r0 + kColRows, rows);
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;   // packed per-column maxima (bf16 magnitude bits)
    const uint64_t keep = policy_evict_last();  // the cast pass reads x again, from L2 when it fits
    if (c < cols) {
        int64_t r = r0 + sub;
        for (; r + 24 < r1; r += 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = ld_hint(reinterpret_cast<const uint4 *>(x + (r + 8 * u) * ld + c), keep);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                m0 = __vmaxu2(m0, abs_finite2(v[u].x));
                m1 = __vmaxu2(m1, abs_finite2(v[u].y));
                m2 = __vmaxu2(m2, abs_finite2(v[u].z));
                m3 = __vmaxu2(m3, abs_finite2(v[u].w));
            }
        }
        for (; r < r1; r += 8) {
            const uint4 v = ld_hint(reinterpret_cast<const uint4 *>(x + r * ld + c), keep);
            m0 = __vmaxu2(m0, abs_finite2(v.x));
            m1 = __vmaxu2(m1, abs_finite2(v.y));
            m2 = __vmaxu2(m2, abs_finite2(v.z));
            m3 = __vmaxu2(m3, abs_finite2(v.w));
        }
    }
    red[sub][cg] = make_uint4(m0, m1, m2, m3);
    __syncthreads();
    if (sub == 0 && c < cols) {
#pragma unroll
        for (int k = 1; k < 8; ++k) {
            const uint4 o = red[k][cg];
            m0 = __vmaxu2(m0, o.x);
            m1 = __vmaxu2(m1, o.y);
            m2 = __vmaxu2(m2, o.z);
            m3 = __vmaxu2(m3, o.w);
        }
        const uint32_t w[4] = {m0, m1, m2, m3};
#pragma unroll
        for (int j = 0; j < 4; ++j) {   // bf16 magnitude bits << 16 = the fp32 bits of the same value
            if ((w[j] & 0xFFFFu) != 0u) atomicMax(&amax_bits[c + 2 * j], (w[j] & 0xFFFFu) << 16);
            if ((w[j] >> 16) != 0u) atomicMax(&amax_bits[c + 2 * j + 1], w[j] & 0xFFFF0000u);
        }
    }
}

// Four rows x eight columns of bf16 (v[k] = row k), cast with the columns'
// scales s8 and transposed in registers: colw[j] holds column j's four codes,
// row 0 in the low byte.
template <int FMT>
__device__ __forceinline__ void cast_transpose_4x8(const uint4 (&v)[4], const float (&s8)[8], uint32_t (&colw)[8]) {
    uint32_t lo[4], hi[4];   // row k's codes of columns 0-3 and 4-7
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
        uint32_t c2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {   // one rounded fp32 multiply per element, two per instruction
            const float2 y = __fmul2_rn(make_float2(bf_lo(w[j]), bf_hi(w[j])), make_float2(s8[2 * j], s8[2 * j + 1]));
            c2[j] = cvt2<FMT>(y.x, y.y);
        }
        lo[k] = c2[0] | (c2[1] << 16);
        hi[k] = c2[2] | (c2[3] << 16);
    }
    // 4 rows x 4 bytes -> 4 columns x 4 rows, for the low and the high half
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
        const uint32_t *R = hlf ? hi : lo;
        const uint32_t t01 = __byte_perm(R[0], R[1], 0x5140), t23 = __byte_perm(R[2], R[3], 0x5140);
        const uint32_t u01 = __byte_perm(R[0], R[1], 0x7362), u23 = __byte_perm(R[2], R[3], 0x7362);
        colw[4 * hlf + 0] = __byte_perm(t01, t23, 0x5410);
        colw[4 * hlf + 1] = __byte_perm(t01, t23, 0x7632);
        colw[4 * hlf + 2] = __byte_perm(u01, u23, 0x5410);
        colw[4 * hlf + 3] = __byte_perm(u01, u23, 0x7632);
    }
}

// Counters of the same 4 x 8 elements: non-finite inputs always, saturated
// elements exactly where a value is not finite or a column may saturate
// (bit j of cols8: column j has fp32(amax) * s > fmax).
template <int FMT>
__device__ __forceinline__ void count_4x8(const uint4 (&v)[4], const float (&s8)[8], uint32_t cols8, uint32_t &nf,
                                          uint32_t &sat) {
    constexpr float fm = fmax_of<FMT>();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t bad = count_nonfinite8(v[k]);
        nf += bad;
        if (bad || cols8) {
            const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sat += fabsf(__fmul_rn(bf_lo(w[j]), s8[2 * j])) > fm ? 1u : 0u;
                sat += fabsf(__fmul_rn(bf_hi(w[j]), s8[2 * j + 1])) > fm ? 1u : 0u;
            }
        }
    }
}

// 64x64 tiles, 128 threads.  The 64 column scales are computed once per CTA
// into shared memory.  Thread t loads rows 4(t/8) .. +3 of the 8 columns
// 8(t%8) .. +7 (four 16-byte loads), casts them, and transposes the 4 x 8
// bytes in registers (byte permutes) into eight 4-byte column words, stored
// to shared memory as the tile's transposed lines (64 bytes per column; the
// 16-byte chunk index XOR-swizzled by bits 3-4 of the column, so the eight
// column groups of a warp spread over the banks).  Each thread then stores
// two 16-byte chunks of output rows.  Row tile 0 also writes 1/s.
template <int FMT, bool POW2>
__global__ void __launch_bounds__(128)
k_cast_transpose_col(const uint16_t *__restrict__ x, uint8_t *__restrict__ qt, int64_t rows, int64_t cols,
                     int64_t ld, const uint32_t *__restrict__ amax_bits, float *__restrict__ scale_inv,
                     uint32_t *__restrict__ counts) {
    __shared__ __align__(16) uint32_t tile[64 * 16];   // [column][16 words of 4 rows]
    __shared__ float sc[64];
    __shared__ uint32_t maysat[2];   // bit j of word w: column c0 + 32w + j has fp32(amax) * s > fmax
    constexpr float fm = fmax_of<FMT>();
    const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
    if (threadIdx.x < 64) {
        const int64_t gc = c0 + threadIdx.x;
        const float a = gc < cols ? __uint_as_float(amax_bits[gc]) : 0.0f;
        const float s = POW2 ? pow2_scale_from_amax(a, fm) : scale_from_amax(a, fm);
        sc[threadIdx.x] = s;
        if (blockIdx.y == 0 && gc < cols) scale_inv[gc] = __fdiv_rn(1.0f, s);
        const uint32_t b = __ballot_sync(0xFFFFFFFFu, __fmul_rn(a, s) > fm);
        if ((threadIdx.x & 31) == 0) maysat[threadIdx.x >> 5] = b;
    }
    const int cv = threadIdx.x & 7, rg = threadIdx.x >> 3;
    const int64_t gc = c0 + cv * 8;
    const uint64_t drop = policy_evict_first();
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t gr = r0 + rg * 4 + k;
        v[k] = (gr < rows && gc < cols) ? ld_hint(reinterpret_cast<const uint4 *>(x + gr * ld + gc), drop)
                                        : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();   // the scales
    float s8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) s8[j] = sc[cv * 8 + j];
    uint32_t nf = 0, sat = 0;
    if (counts) count_4x8<FMT>(v, s8, (maysat[cv >> 2] >> ((cv & 3) * 8)) & 0xFFu, nf, sat);
    uint32_t colw[8];
    cast_transpose_4x8<FMT>(v, s8, colw);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int col = cv * 8 + j;
        const int chunk = (rg >> 2) ^ ((col >> 3) & 3);
        tile[col * 16 + chunk * 4 + (rg & 3)] = colw[j];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int q = threadIdx.x + 128 * i;
        const int col = q >> 2, part = q & 3;
        const int64_t go = c0 + col, gi = r0 + part * 16;
        const uint4 o = *reinterpret_cast<const uint4 *>(&tile[col * 16 + ((part ^ ((col >> 3) & 3)) * 4)]);
        if (go < cols && gi < rows) *reinterpret_cast<uint4 *>(qt + go * rows + gi) = o;
    }
    if (counts) flush_counts(counts, nf, sat);
}

// Single pass over x for the transposed rowwise quantizer: a cluster of
// kQtCtas CTAs owns a strip of 64 columns, CTA rank r a contiguous range of
// 128-row tiles of it.  Pass 1 reads the CTA's rows (loads kept in L2) and
// reduces the 64 column maxima of the finite magnitudes; the partial maxima
// are combined through distributed shared memory behind one cluster barrier;
// pass 2 re-reads the same rows (an L2 hit: the strip was read microseconds
// earlier) and casts and transposes them in 128 x 64 tiles.  x crosses HBM
// once; clusters loop over strips.  The grid is capped so that the strips
// in flight fit in L2 together.
// Split cluster barrier (every thread of every CTA of the cluster; arrive and
// wait alternate): release on arrive, acquire on wait.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

constexpr int kQtCtas = 8;
constexpr int kQtThreads = 256;
constexpr int kQtTile = 128;                      // rows per cast tile (4 per thread)
constexpr int64_t kQtMaxRows = 16384;             // strip of 2 MiB at most; longer columns take two passes

template <int FMT, bool POW2>
__global__ void __cluster_dims__(kQtCtas, 1, 1) __launch_bounds__(kQtThreads, 4)
k_qt_strip(const uint16_t *__restrict__ x, uint8_t *__restrict__ qt, int64_t rows, int64_t cols, int64_t ld,
           float *__restrict__ scale_inv, float *__restrict__ amax_out, uint32_t *__restrict__ counts) {
    __shared__ __align__(16) uint32_t tile[64 * 32];   // [column][32 words = 128 rows of codes], swizzled
    __shared__ uint4 red[8][8];                        // per warp: packed maxima of 8 x 8 columns
    __shared__ uint32_t part[64];                      // this CTA's column maxima (fp32 bits)
    __shared__ float sc[64];
    __shared__ uint32_t maysat[2];
    constexpr float fm = fmax_of<FMT>();
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank();
    const int64_t cid = blockIdx.x / kQtCtas, ncl = gridDim.x / kQtCtas;
    const int64_t nstrips = (cols + 63) / 64;
    const int64_t ntiles = (rows + kQtTile - 1) / kQtTile, tpc = (ntiles + kQtCtas - 1) / kQtCtas;
    const int64_t rb = min((int64_t)rank * tpc, ntiles) * kQtTile;
    const int64_t re = min(min((int64_t)rank * tpc + tpc, ntiles) * kQtTile, rows);
    const int cv = threadIdx.x & 7, rr = threadIdx.x >> 3;   // 8 columns x (rows rr, rr + 32, ...)
    const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
    uint32_t nf = 0, sat = 0;
    int it = 0;
    for (int64_t strip = cid; strip < nstrips; strip += ncl, ++it) {
        const int64_t c0 = strip * 64, gc = c0 + cv * 8;
        const bool cok = gc < cols;   // cols % 16 == 0: a vector of 8 columns is all in or all out
        // pass 1: column maxima of this CTA's rows.  Fast form: |x| by the
        // sign mask and a NaN-propagating bf16x2 max; if any column saw a
        // NaN or Inf the CTA redoes its rows with the finite-only maximum.
        uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;   // packed per-column maxima (bf16 magnitude bits)
        auto pass1 = [&](auto EXACT) {
            constexpr bool exact = decltype(EXACT)::value;
            auto acc4 = [&](const uint4 &v) {
                if (exact) {
                    m0 = __vmaxu2(m0, abs_finite2(v.x));
                    m1 = __vmaxu2(m1, abs_finite2(v.y));
                    m2 = __vmaxu2(m2, abs_finite2(v.z));
                    m3 = __vmaxu2(m3, abs_finite2(v.w));
                } else {
                    m0 = amax_fast_word(m0, v.x);
                    m1 = amax_fast_word(m1, v.y);
                    m2 = amax_fast_word(m2, v.z);
                    m3 = amax_fast_word(m3, v.w);
                }
            };
            if (!cok) return;
            const uint16_t *xc = x + gc;
            int64_t r = rb + rr;
            for (; r + 7 * 32 < re; r += 8 * 32) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = ld_hint(reinterpret_cast<const uint4 *>(xc + (r + 32 * u) * ld), keep);
#pragma unroll
                for (int u = 0; u < 8; ++u) acc4(v[u]);
            }
            for (; r < re; r += 32) acc4(ld_hint(reinterpret_cast<const uint4 *>(xc + r * ld), keep));
        };
        pass1(std::false_type{});
        const uint32_t hmax = max(max(m0 & 0xFFFFu, m0 >> 16), max(max(m1 & 0xFFFFu, m1 >> 16),
                                  max(max(m2 & 0xFFFFu, m2 >> 16), max(m3 & 0xFFFFu, m3 >> 16))));
        if (__syncthreads_or(hmax >= 0x7F80u)) {   // a NaN or Inf in this CTA's rows (rare)
            m0 = m1 = m2 = m3 = 0;
            pass1(std::true_type{});
        }
        // the four lanes of a warp with the same cv (lanes cv + 8i) first, by shuffles
#pragma unroll
        for (int o = 8; o < 32; o <<= 1) {
            m0 = __vmaxu2(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, o));
            m1 = __vmaxu2(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, o));
            m2 = __vmaxu2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, o));
            m3 = __vmaxu2(m3, __shfl_xor_sync(0xFFFFFFFFu, m3, o));
        }
        if ((threadIdx.x & 31) < 8) red[threadIdx.x >> 5][cv] = make_uint4(m0, m1, m2, m3);
        // the previous strip's peers have read part[] (their "reads done" arrive)
        if (it > 0) cluster_wait();
        __syncthreads();
        if (threadIdx.x < 64) {   // column j = 8 * (j >> 3) + (j & 7): word (j & 7) >> 1, half j & 1
            const int j = threadIdx.x, sh = (j & 1) * 16;
            uint32_t m = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 w = red[k][j >> 3];
                const uint32_t wj = ((j & 7) >> 1) == 0 ? w.x : ((j & 7) >> 1) == 1 ? w.y : ((j & 7) >> 1) == 2 ? w.z : w.w;
                m = max(m, (wj >> sh) & 0xFFFFu);
            }
            part[j] = m << 16;   // bf16 magnitude bits << 16 = the fp32 bits of the same value
        }
        cluster_arrive();   // every CTA's column maxima of this strip are published
        cluster_wait();
        if (threadIdx.x < 64) {
            const int j = threadIdx.x;
            uint32_t m = 0;
#pragma unroll
            for (int k = 0; k < kQtCtas; ++k) m = max(m, *cluster.map_shared_rank(&part[j], k));
            const float a = __uint_as_float(m);
            const float sj = POW2 ? pow2_scale_from_amax(a, fm) : scale_from_amax(a, fm);
            sc[j] = sj;
            if (rank == 0 && c0 + j < cols) {
                scale_inv[c0 + j] = __fdiv_rn(1.0f, sj);
                amax_out[c0 + j] = a;
            }
            const uint32_t b = __ballot_sync(0xFFFFFFFFu, __fmul_rn(a, sj) > fm);
            if ((j & 31) == 0) maysat[j >> 5] = b;
        }
        cluster_arrive();   // this CTA has read its peers' part[] ("reads done"; waited before the next write)
        __syncthreads();   // the scales
        float s8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) s8[j] = sc[cv * 8 + j];
        const uint32_t cols8 = (maysat[cv >> 2] >> ((cv & 3) * 8)) & 0xFFu;
        // pass 2: 128 x 64 tiles, thread (cv, rr) casts rows 4 rr .. + 3 of its 8 columns;
        // the next tile's loads are issued before this tile is cast.  re is a
        // multiple of 16, so a thread's four rows are all in or all out.
        const uint16_t *xp = x + (rb + rr * 4) * ld + gc;   // + k * ld: row k of this thread's group
        const int64_t tstep = (int64_t)kQtTile * ld;
        auto load_tile = [&](int64_t r0, const uint16_t *p, uint4 (&v)[4]) {
            const bool in = cok && r0 + rr * 4 < re;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                v[k] = in ? ld_hint(reinterpret_cast<const uint4 *>(p + k * ld), drop) : make_uint4(0, 0, 0, 0);
        };
        // output row c0 + col (col = q >> 3), bytes r0 + 16 (q & 7) .. + 15, for q = t and t + 256
        const int col0 = threadIdx.x >> 3, col1 = col0 + 32, ch = threadIdx.x & 7;
        uint8_t *qp = qt + (c0 + col0) * rows + rb + ch * 16;   // + 32 rows: output row c0 + col1
        const bool ok0 = c0 + col0 < cols, ok1 = c0 + col1 < cols;
        const int tl0 = col0 * 32 + ((ch ^ (col0 >> 3)) * 4), tl1 = col1 * 32 + ((ch ^ (col1 >> 3)) * 4);
        const int tw = (cv * 8) * 32 + (((rr >> 2) ^ cv) * 4) + (rr & 3);   // + 32 j: column cv * 8 + j
        auto cast_tile = [&](int64_t r0, const uint4 (&v)[4]) {
            if (counts) count_4x8<FMT>(v, s8, cols8, nf, sat);
            uint32_t colw[8];
            cast_transpose_4x8<FMT>(v, s8, colw);
#pragma unroll
            for (int j = 0; j < 8; ++j) tile[tw + 32 * j] = colw[j];
            __syncthreads();
            const bool rin = r0 + ch * 16 < re;
            const uint4 o0 = *reinterpret_cast<const uint4 *>(&tile[tl0]), o1 = *reinterpret_cast<const uint4 *>(&tile[tl1]);
            if (rin && ok0) st_hint(reinterpret_cast<uint4 *>(qp), o0, drop);
            if (rin && ok1) st_hint(reinterpret_cast<uint4 *>(qp + 32 * rows), o1, drop);
            qp += kQtTile;
            __syncthreads();   // the tile is rewritten by the next pass
        };
        uint4 nv[4];
        if (rb < re) load_tile(rb, xp, nv);
        for (int64_t r0 = rb; r0 < re; r0 += kQtTile) {
            uint4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = nv[k];
            xp += tstep;
            if (r0 + kQtTile < re) load_tile(r0 + kQtTile, xp, nv);
            cast_tile(r0, v);
        }
    }
    if (counts) flush_counts(counts, nf, sat);
    if (it > 0) cluster_wait();   // no CTA leaves while a peer may still read its column maxima
}

// Clusters of k_qt_strip that fit on the device at once (cached per device).
template <int FMT, bool POW2>
static int qt_active_clusters() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] > 0) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kQtCtas * 64);
    cfg.blockDim = dim3(kQtThreads);
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kQtCtas;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_qt_strip<FMT, POW2>, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

template <int FMT, bool POW2>
static cudaError_t launch_qt_strip(cudaStream_t s, const uint16_t *x, uint8_t *qt, int64_t rows, int64_t cols,
                                   int64_t ld, float *scale_inv, float *amax_out, uint32_t *counts) {
    const int active = qt_active_clusters<FMT, POW2>();
    if (active <= 0) return cudaErrorInvalidConfiguration;
    // strips in flight (rows x 128 bytes each) within 96 MiB of the 126 MB L2, so pass 2 finds them
    // there (measured: 64 MiB starved long columns of clusters, 112 MiB gained nothing more)
    const int64_t fit = std::max<int64_t>(1, ((int64_t)96 << 20) / std::max<int64_t>(1, rows * 128));
    const int64_t nstrips = (cols + 63) / 64;
    const int64_t ncl = std::min<int64_t>(std::min<int64_t>(nstrips, active), fit);
    k_qt_strip<FMT, POW2><<<(unsigned)(ncl * kQtCtas), kQtThreads, 0, s>>>(x, qt, rows, cols, ld, scale_inv, amax_out,
                                                                          counts);
    return cudaPeekAtLastError();
}

// --------------------------------------------------------------- rowwise --
// A CTA (128 threads) quantizes R rows at a time, every row held in registers
// (V vectors of 8 per thread) between its amax and its cast: one HBM read per
// element, and all R rows' loads are issued before the first reduction.
// V == 0: rows too long for registers, two passes (the second from L2).
constexpr int kRowThreads = 128;
// One tensor of a rowwise launch (a launch can quantize two, e.g. both GEMM
// operands, which share the row length).
struct RowJob {
    const uint16_t *x;
    int64_t rows, ld;
    uint8_t *q;
    float *scale_inv;
};
template <int FMT, bool POW2, int V, int R>
__global__ void __launch_bounds__(kRowThreads)
k_rowwise(RowJob ja, RowJob jb, int64_t cols, uint32_t *__restrict__ counts) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    __shared__ uint32_t red[R][32];
    constexpr float fm = fmax_of<FMT>();
    uint32_t nf = 0, sat = 0;   // counters (counts != NULL)
    const int64_t ncv = cols / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // groups of R rows: ja's first, then jb's
    const int64_t ga = (ja.rows + R - 1) / R, gtot = ga + (jb.rows + R - 1) / R;
    for (int64_t g = blockIdx.x; g < gtot; g += gridDim.x) {
        const bool first = g < ga;
        const uint16_t *x = first ? ja.x : jb.x;
        const int64_t rows = first ? ja.rows : jb.rows, ld = first ? ja.ld : jb.ld;
        uint8_t *q = first ? ja.q : jb.q;
        float *scale_inv = first ? ja.scale_inv : jb.scale_inv;
        const int64_t r0 = (first ? g : g - ga) * R;
        if constexpr (V > 0) {
            uint4 v[R][V];
            uint32_t m[R];
            bool nonfin[R];
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(x + (r0 + rr) * ld);
                const bool row_ok = r0 + rr < rows;
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const int64_t cv = threadIdx.x + j * kRowThreads;
                    v[rr][j] = (row_ok && cv < ncv) ? ld_stream(xr + cv) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                uint32_t m2 = 0;
#pragma unroll
                for (int j = 0; j < V; ++j) m2 = amax_fast8(m2, v[rr][j]);
                m[rr] = amax_fast_final(m2);
                nonfin[rr] = m[rr] == 0xFFFFFFFFu;
                if (nonfin[rr]) {
                    uint32_t bad = 0;
                    m[rr] = 0;
#pragma unroll
                    for (int j = 0; j < V; ++j) m[rr] = amax_exact8(m[rr], v[rr][j], bad);
                }
                m[rr] = __reduce_max_sync(0xFFFFFFFFu, m[rr]);
                if (lane == 0) red[rr][warp] = m[rr];
            }
            __syncthreads();
#pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                uint32_t mm = lane < kRowThreads / 32 ? red[rr][lane] : 0u;
                mm = __reduce_max_sync(0xFFFFFFFFu, mm);
                const float a = bf16bits_to_float(mm);
                const float s = POW2 ? pow2_scale_from_amax(a, fm) : scale_from_amax(a, fm);
                if (r0 + rr < rows) {
                    uint2 *qr = reinterpret_cast<uint2 *>(q + (r0 + rr) * cols);
#pragma unroll
                    for (int j = 0; j < V; ++j) {
                        const int64_t cv = threadIdx.x + j * kRowThreads;
                        if (cv < ncv) qr[cv] = cast8<FMT>(v[rr][j], s);
                    }
                    if (threadIdx.x == 0) scale_inv[r0 + rr] = __fdiv_rn(1.0f, s);
                    if (counts && may_saturate(nonfin[rr], a, s, fm)) {   // vectors past the row are zeros
#pragma unroll
                        for (int j = 0; j < V; ++j) {
                            nf += count_nonfinite8(v[rr][j]);
                            sat += count_sat8(v[rr][j], s, fm);
                        }
                    }
                }
            }
            __syncthreads();   // red[] is reused by the next rows
        } else {
            for (int rr = 0; rr < R && r0 + rr < rows; ++rr) {
                const int64_t r = r0 + rr;
                const uint4 *xr = reinterpret_cast<const uint4 *>(x + r * ld);
                uint2 *qr = reinterpret_cast<uint2 *>(q + r * cols);
                uint32_t bad = 0, mm = 0;
                for (int64_t cv = threadIdx.x; cv < ncv; cv += kRowThreads) mm = amax_exact8(mm, ld_stream(xr + cv), bad);
                mm = block_max_u32(mm, red[0]);
                const float a = bf16bits_to_float(mm);
                const float s = POW2 ? pow2_scale_from_amax(a, fm) : scale_from_amax(a, fm);
                const bool cnt = counts && may_saturate(bad > 0, a, s, fm);
                nf += bad;
                for (int64_t cv = threadIdx.x; cv < ncv; cv += kRowThreads) {
                    const uint4 w = xr[cv];
                    qr[cv] = cast8<FMT>(w, s);
                    if (cnt) sat += count_sat8(w, s, fm);
                }
                if (threadIdx.x == 0) scale_inv[r] = __fdiv_rn(1.0f, s);
                __syncthreads();
            }
        }
    }
    if (counts) flush_counts(counts, nf, sat);
}

// ---------------------------------------------------------- block 1x128 --
// Four lanes per 1x128 block, 32 elements each: a warp walks rows (warp,
// warp + nwarps, ...) and takes 8 blocks of a row per step, lanes 4g .. 4g+3
// block g, lane j its 16-byte pieces j, j+4, j+8, j+12 (each load instruction
// reads 64 contiguous bytes per block, each store writes 32).  Two steps'
// loads (8 x 16 bytes per lane) are issued before the first reduction.  The
// per-block work -- a two-shuffle max, the scale division, the scale store --
// is shared by four lanes' 32 elements (with 16 lanes of 8 elements it cost
// as many instructions as the cast itself: 15 per element against 5 now).
// scale_inv is stored [kb][row].
// SF = false: fp32 scale_inv[kb * rows + row], s = fmax / amax.
// SF = true:  E8M0 image (sf_image), s the pow2 rule; the image's padding rows
//             (up to a multiple of 128) get e = 127 (factor 1).
// COUNT: the non-finite / saturated counters.
template <int FMT, bool SF, bool COUNT>
__global__ void __launch_bounds__(256)
k_block1x128(const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
             uint8_t *__restrict__ q, float *__restrict__ scale_inv, uint8_t *__restrict__ sf_image,
             uint32_t *__restrict__ counts) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    constexpr float fm = fmax_of<FMT>();
    constexpr int STEPS = 2;                 // 8-block steps whose loads are in flight together
    const int lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
    const int64_t nkb = (cols + 127) / 128;
    const int64_t rt = (rows + 127) / 128;
    const int64_t row_end = SF ? rt * 128 : rows;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint32_t nf = 0, sat = 0;
    for (int64_t row = warp; row < row_end; row += nwarps) {
        const bool live = row < rows;
        const uint16_t *xr = x + (live ? row : 0) * ld;
        uint8_t *qr = q + row * cols;
        for (int64_t kb0 = 0; kb0 < nkb; kb0 += 8 * STEPS) {
            uint4 v[STEPS][4];
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int64_t c0 = (kb0 + 8 * t + g) * 128;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int64_t c = c0 + (j + 4 * p) * 8;
                    v[t][p] = (live && c < cols) ? ld_stream(reinterpret_cast<const uint4 *>(xr + c))
                                                 : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int t = 0; t < STEPS; ++t) {
                const int64_t kb = kb0 + 8 * t + g;
                uint32_t m = amax_fast_final(amax_fast8(amax_fast8(amax_fast8(amax_fast8(0u, v[t][0]), v[t][1]), v[t][2]), v[t][3]));
                const bool nonfin = m == 0xFFFFFFFFu;
                if (nonfin) {
                    uint32_t bad = 0;
                    m = amax_exact8(amax_exact8(amax_exact8(amax_exact8(0u, v[t][0], bad), v[t][1], bad), v[t][2], bad),
                                    v[t][3], bad);
                }
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                const float amax = bf16bits_to_float(m);
                const float s = SF ? pow2_scale_from_amax(amax, fm) : scale_from_amax(amax, fm);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int64_t c = kb * 128 + (j + 4 * p) * 8;
                    if (live && c < cols) *reinterpret_cast<uint2 *>(qr + c) = cast8<FMT>(v[t][p], s);
                }
                if (j == 0 && kb < nkb) {
                    if (SF) sf_image[e8m0_offset(kb, rt, row)] = live ? e8m0_of_scale(s) : (uint8_t)127;
                    else scale_inv[kb * rows + row] = __fdiv_rn(1.0f, s);
                }
                if (COUNT && live && may_saturate(nonfin, amax, s, fm)) {   // pieces past the row are zeros
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        nf += count_nonfinite8(v[t][p]);
                        sat += count_sat8(v[t][p], s, fm);
                    }
                }
            }
        }
    }
    if (COUNT) flush_counts(counts, nf, sat);
}

// -------------------------------------------------------- block 128x128 --
// One CTA (256 threads) per 128x128 tile, the tile held in registers (8
// vectors of 8 per thread: 16 threads across a 128-wide row, 16 rows per
// pass, 8 passes).
// SF = true: pow2 scale; the first 128 threads write the tile's exponent
// into the E8M0 image byte of each of its 128 rows (rows past `rows`
// included).
template <int FMT, bool SF>
__global__ void __launch_bounds__(256)
k_block128(const uint16_t *__restrict__ x, int64_t rows, int64_t cols, int64_t ld,
           uint8_t *__restrict__ q, float *__restrict__ scale_inv, uint8_t *__restrict__ sf_image,
           uint32_t *__restrict__ counts) {
    pdl_trigger();   // dependents are scheduled once all our CTAs have started
    pdl_wait();
    __shared__ uint32_t red[32];
    constexpr float fm = fmax_of<FMT>();
    uint32_t nf = 0, sat = 0;   // counters (counts != NULL)
    const int64_t nkb = (cols + 127) / 128, nrb = (rows + 127) / 128;
    const int rsub = threadIdx.x >> 4, cv = threadIdx.x & 15;
    for (int64_t t = blockIdx.x; t < nrb * nkb; t += gridDim.x) {
        const int64_t rb = t / nkb, kb = t - rb * nkb;
        const int64_t c = kb * 128 + cv * 8;
        uint4 v[8];
        uint32_t m2 = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int64_t r = rb * 128 + p * 16 + rsub;
            v[p] = (r < rows && c < cols) ? ld_stream(reinterpret_cast<const uint4 *>(x + r * ld + c))
                                          : make_uint4(0, 0, 0, 0);
            m2 = amax_fast8(m2, v[p]);
        }
        uint32_t m = amax_fast_final(m2);
        const bool nonfin = m == 0xFFFFFFFFu;
        if (nonfin) {
            uint32_t bad = 0;
            m = 0;
#pragma unroll
            for (int p = 0; p < 8; ++p) m = amax_exact8(m, v[p], bad);
        }
        m = block_max_u32(m, red);
        const float s = SF ? pow2_scale_from_amax(bf16bits_to_float(m), fm) : scale_from_amax(bf16bits_to_float(m), fm);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int64_t r = rb * 128 + p * 16 + rsub;
            if (r < rows && c < cols) *reinterpret_cast<uint2 *>(q + r * cols + c) = cast8<FMT>(v[p], s);
        }
        if (counts && may_saturate(nonfin, bf16bits_to_float(m), s, fm)) {   // out-of-range vectors are zeros
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                nf += count_nonfinite8(v[p]);
                sat += count_sat8(v[p], s, fm);
            }
        }
        if (SF) {
            if (threadIdx.x < 128) sf_image[e8m0_offset(kb, nrb, rb * 128 + threadIdx.x)] = e8m0_of_scale(s);
        } else if (threadIdx.x == 0) {
            scale_inv[rb * nkb + kb] = __fdiv_rn(1.0f, s);
        }
    }
    if (counts) flush_counts(counts, nf, sat);
}

int stream_grid(int sms, int64_t work_units, int threads) {
    int64_t want = (work_units + threads - 1) / threads;
    int64_t cap = (int64_t)sms * (2048 / threads);
    return (int)std::max<int64_t>(1, std::min(want, cap));
}

template <int FMT>
void launch_cast(cudaStream_t st, int sms, const void *x, int64_t rows, int64_t cols, const float *scale_in,
                 const float *amax_in, uint8_t *q, int transpose_out, float *scale_inv,
                 uint32_t *amax_bits, uint32_t *nf_ctr, uint32_t *sat_ctr) {
    const bool amax = amax_bits != nullptr, count = nf_ctr != nullptr || sat_ctr != nullptr;
    const uint16_t *xs = static_cast<const uint16_t *>(x);
    if (transpose_out) {
        dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
        if (amax && count) pdl_launch(k_cast_transpose<FMT, true, true>, dim3(grid), dim3(256), 0, st, xs, q, rows, cols, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
        else if (amax) pdl_launch(k_cast_transpose<FMT, true, false>, dim3(grid), dim3(256), 0, st, xs, q, rows, cols, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
        else if (count) pdl_launch(k_cast_transpose<FMT, false, true>, dim3(grid), dim3(256), 0, st, xs, q, rows, cols, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
        else pdl_launch(k_cast_transpose<FMT, false, false>, dim3(grid), dim3(256), 0, st, xs, q, rows, cols, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
        return;
    }
    const int64_t n = rows * cols, nunit = n / 16;
    const int grid = stream_grid(sms, std::max<int64_t>(nunit / 2, 1), kStreamThreads);
    const uint4 *xv = static_cast<const uint4 *>(x);
    uint4 *qv = reinterpret_cast<uint4 *>(q);
    if (amax && count) pdl_launch(k_cast_tensor<FMT, true, true>, dim3(grid), dim3(kStreamThreads), 0, st, xv, qv, nunit, xs, q, n, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
    else if (amax) pdl_launch(k_cast_tensor<FMT, true, false>, dim3(grid), dim3(kStreamThreads), 0, st, xv, qv, nunit, xs, q, n, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
    else if (count) pdl_launch(k_cast_tensor<FMT, false, true>, dim3(grid), dim3(kStreamThreads), 0, st, xv, qv, nunit, xs, q, n, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
    else pdl_launch(k_cast_tensor<FMT, false, false>, dim3(grid), dim3(kStreamThreads), 0, st, xv, qv, nunit, xs, q, n, scale_in, amax_in, scale_inv, amax_bits, nf_ctr, sat_ctr);
}

template <int FMT, bool POW2>
cudaError_t launch_rowwise(cudaStream_t st, int sms, const RowJob &ja, const RowJob &jb, int64_t cols,
                           uint32_t *counts) {
    const int64_t slots = (int64_t)sms * 16;   // resident 128-thread CTAs
    const int64_t ncv = cols / 8;
    const int64_t rows = ja.rows + jb.rows;
    const int T = kRowThreads;
    // two rows per CTA when that lets one wave of CTAs cover every row
    const bool two = rows > slots && ncv <= 4 * T;
    const int64_t groups = two ? (ja.rows + 1) / 2 + (jb.rows + 1) / 2 : rows;
    // the same number of row groups for every CTA (no half-empty last round)
    const int64_t rounds = (groups + slots - 1) / slots;
    const dim3 grid((unsigned)std::max<int64_t>(1, (groups + rounds - 1) / rounds)), block(T);
    if (two) {
        if (ncv <= T) return pdl_launch(k_rowwise<FMT, POW2, 1, 2>, grid, block, 0, st, ja, jb, cols, counts);
        if (ncv <= 2 * T) return pdl_launch(k_rowwise<FMT, POW2, 2, 2>, grid, block, 0, st, ja, jb, cols, counts);
        return pdl_launch(k_rowwise<FMT, POW2, 4, 2>, grid, block, 0, st, ja, jb, cols, counts);
    }
    if (ncv <= T) return pdl_launch(k_rowwise<FMT, POW2, 1, 1>, grid, block, 0, st, ja, jb, cols, counts);
    if (ncv <= 2 * T) return pdl_launch(k_rowwise<FMT, POW2, 2, 1>, grid, block, 0, st, ja, jb, cols, counts);
    if (ncv <= 4 * T) return pdl_launch(k_rowwise<FMT, POW2, 4, 1>, grid, block, 0, st, ja, jb, cols, counts);
    if (ncv <= 8 * T) return pdl_launch(k_rowwise<FMT, POW2, 8, 1>, grid, block, 0, st, ja, jb, cols, counts);
    if (ncv <= 16 * T) return pdl_launch(k_rowwise<FMT, POW2, 16, 1>, grid, block, 0, st, ja, jb, cols, counts);
    return pdl_launch(k_rowwise<FMT, POW2, 0, 1>, grid, block, 0, st, ja, jb, cols, counts);
}

template <int FMT, bool SF>
cudaError_t launch_block(cudaStream_t st, int sms, const void *x, int64_t rows, int64_t cols, int64_t ld,
                         int block_rows, uint8_t *q, float *scale_inv, uint8_t *sf_image, uint32_t *counts) {
    const uint16_t *xs = static_cast<const uint16_t *>(x);
    const int64_t nkb = (cols + 127) / 128;
    if (block_rows == 1) {
        const int64_t r = SF ? (rows + 127) / 128 * 128 : rows;
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((r + 7) / 8, (int64_t)sms * 8));
        if (counts)
            return pdl_launch(k_block1x128<FMT, SF, true>, dim3(grid), dim3(256), 0, st, xs, rows, cols, ld, q,
                              scale_inv, sf_image, counts);
        return pdl_launch(k_block1x128<FMT, SF, false>, dim3(grid), dim3(256), 0, st, xs, rows, cols, ld, q, scale_inv,
                          sf_image, counts);
    } else {
        const int64_t tiles = ((rows + 127) / 128) * nkb;
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, (int64_t)sms * 8));
        return pdl_launch(k_block128<FMT, SF>, dim3(grid), dim3(256), 0, st, xs, rows, cols, ld, q, scale_inv,
                          sf_image, counts);
    }
}

}  // namespace

using namespace fp8q_host;

extern "C" fp8_status fp8_amax(const void *x_bf16, int64_t n, float *amax, uint32_t *counts, void *stream) {
    if (!amax || (n > 0 && !x_bf16)) return FP8_ERR_INVALID_ARG;
    if (n < 0) return FP8_ERR_SHAPE;
    if ((n > 0 && !aligned16(x_bf16)) || (reinterpret_cast<uintptr_t>(amax) & 3u) ||
        (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)))
        return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return FP8_ERR_CUDA;
    const int64_t nvec = n / 8;
    const int grid = stream_grid(sms, std::max<int64_t>(nvec / 4, 1), kStreamThreads);
    pdl_launch(k_amax, dim3(grid), dim3(kStreamThreads), 0, s, static_cast<const uint4 *>(x_bf16), nvec,
                                            static_cast<const uint16_t *>(x_bf16), n,
                                            reinterpret_cast<uint32_t *>(amax), counts);
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_quantize_tensorwise(const void *x_bf16, int64_t rows, int64_t cols, fp8_format fmt,
                                              const float *scale_in, uint8_t *q, int transpose_out,
                                              float *scale_inv_out, float *amax_out, uint32_t *counts,
                                              void *stream) {
    if (rows < 0 || cols < 0) return FP8_ERR_SHAPE;
    const int64_t n = rows * cols;
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (!scale_inv_out || (n > 0 && (!x_bf16 || !q))) return FP8_ERR_INVALID_ARG;
    if (!scale_in && !amax_out) return FP8_ERR_INVALID_ARG;   // current scaling needs the amax buffer
    if (transpose_out && ((rows % 16) || (cols % 16))) return FP8_ERR_SHAPE;
    if (n > 0 && (!aligned16(x_bf16) || !aligned16(q))) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    uint32_t *amax_bits = reinterpret_cast<uint32_t *>(amax_out);
    const float *amax_in = nullptr;
    uint32_t *nf_ctr = counts, *sat_ctr = counts ? counts + 1 : nullptr;
    if (!scale_in && !transpose_out && n > 0 && n <= kSmallTensor) {   // one launch for a small tensor
        if ((reinterpret_cast<uintptr_t>(amax_out) & 3u) || (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)))
            return FP8_ERR_ALIGNMENT;
        const uint16_t *xs = static_cast<const uint16_t *>(x_bf16);
        const uint4 *xv = static_cast<const uint4 *>(x_bf16);
        cudaError_t e = (fmt == FP8_E4M3)
            ? pdl_launch(k_quant_tensor_small<FP8_E4M3>, dim3(1), dim3(kSmallThreads), 0, s, xv, xs, n, q,
                         amax_bits, scale_inv_out, nf_ctr, sat_ctr)
            : pdl_launch(k_quant_tensor_small<FP8_E5M2>, dim3(1), dim3(kSmallThreads), 0, s, xv, xs, n, q,
                         amax_bits, scale_inv_out, nf_ctr, sat_ctr);
        return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
    }
    if (!scale_in) {
        // Current scaling: an amax pass first (fills amax_out and counts the
        // non-finite inputs), then the cast pass reads the amax back.
        fp8_status a = fp8_amax(x_bf16, n, amax_out, counts, stream);
        if (a != FP8_OK) return a;
        amax_in = amax_out;
        amax_bits = nullptr;
        nf_ctr = nullptr;
    } else if (amax_bits) {
        if (cudaMemsetAsync(amax_bits, 0, sizeof(float), s) != cudaSuccess) return FP8_ERR_CUDA;
    }
    if (fmt == FP8_E4M3)
        launch_cast<FP8_E4M3>(s, sms, x_bf16, rows, cols, scale_in, amax_in, q, transpose_out, scale_inv_out, amax_bits, nf_ctr, sat_ctr);
    else
        launch_cast<FP8_E5M2>(s, sms, x_bf16, rows, cols, scale_in, amax_in, q, transpose_out, scale_inv_out, amax_bits, nf_ctr, sat_ctr);
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

static bool counts_ok(const uint32_t *counts) { return !counts || !(reinterpret_cast<uintptr_t>(counts) & 3u); }

static fp8_status dispatch_rowwise(cudaStream_t s, int sms, fp8_format fmt, int pow2, const RowJob &ja,
                                   const RowJob &jb, int64_t cols, uint32_t *counts) {
    cudaError_t e;
    if (fmt == FP8_E4M3) e = pow2 ? launch_rowwise<FP8_E4M3, true>(s, sms, ja, jb, cols, counts)
                                  : launch_rowwise<FP8_E4M3, false>(s, sms, ja, jb, cols, counts);
    else e = pow2 ? launch_rowwise<FP8_E5M2, true>(s, sms, ja, jb, cols, counts)
                  : launch_rowwise<FP8_E5M2, false>(s, sms, ja, jb, cols, counts);
    return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_quantize_rowwise(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                           fp8_format fmt, int pow2, uint8_t *q, float *scale_inv,
                                           uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return FP8_ERR_SHAPE;
    if (cols % 16) return FP8_ERR_SHAPE;
    if (rows == 0 || cols == 0) {
        if (rows > 0 && !scale_inv) return FP8_ERR_INVALID_ARG;
    } else if (!x_bf16 || !q || !scale_inv) {
        return FP8_ERR_INVALID_ARG;
    }
    if (ld % 8) return FP8_ERR_ALIGNMENT;
    if ((x_bf16 && !aligned16(x_bf16)) || (q && !aligned16(q)) || !counts_ok(counts)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (rows == 0) return FP8_OK;
    const RowJob ja{static_cast<const uint16_t *>(x_bf16), rows, ld, q, scale_inv}, jb{nullptr, 0, 0, nullptr, nullptr};
    return dispatch_rowwise(as_stream(stream), sms, fmt, pow2, ja, jb, cols, counts);
}

extern "C" fp8_status fp8_quantize_rowwise_pair(const void *a_bf16, int64_t rows_a, int64_t lda, uint8_t *qa,
                                                float *sa, const void *b_bf16, int64_t rows_b, int64_t ldb,
                                                uint8_t *qb, float *sb, int64_t cols, fp8_format fmt, int pow2,
                                                uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (rows_a < 0 || rows_b < 0 || cols < 0 || lda < cols || ldb < cols || (cols % 16)) return FP8_ERR_SHAPE;
    if ((rows_a > 0 && (!sa || (cols > 0 && (!a_bf16 || !qa)))) ||
        (rows_b > 0 && (!sb || (cols > 0 && (!b_bf16 || !qb)))))
        return FP8_ERR_INVALID_ARG;
    if (lda % 8 || ldb % 8) return FP8_ERR_ALIGNMENT;
    if ((a_bf16 && !aligned16(a_bf16)) || (qa && !aligned16(qa)) || (b_bf16 && !aligned16(b_bf16)) ||
        (qb && !aligned16(qb)) || !counts_ok(counts))
        return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (rows_a + rows_b == 0) return FP8_OK;
    const RowJob ja{static_cast<const uint16_t *>(a_bf16), rows_a, lda, qa, sa};
    const RowJob jb{static_cast<const uint16_t *>(b_bf16), rows_b, ldb, qb, sb};
    return dispatch_rowwise(as_stream(stream), sms, fmt, pow2, ja, jb, cols, counts);
}

extern "C" fp8_status fp8_quantize_blockwise(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                             fp8_format fmt, int block_rows, uint8_t *q, float *scale_inv,
                                             uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (block_rows != 1 && block_rows != 128) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols || (cols % 16)) return FP8_ERR_SHAPE;
    if (rows > 0 && cols > 0 && (!x_bf16 || !q || !scale_inv)) return FP8_ERR_INVALID_ARG;
    if (ld % 8) return FP8_ERR_ALIGNMENT;
    if ((x_bf16 && !aligned16(x_bf16)) || (q && !aligned16(q)) || !counts_ok(counts)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (rows == 0 || cols == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    const cudaError_t e =
        (fmt == FP8_E4M3)
            ? launch_block<FP8_E4M3, false>(s, sms, x_bf16, rows, cols, ld, block_rows, q, scale_inv, nullptr, counts)
            : launch_block<FP8_E5M2, false>(s, sms, x_bf16, rows, cols, ld, block_rows, q, scale_inv, nullptr, counts);
    return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_quantize_rowwise_transpose(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                                     fp8_format fmt, int pow2, uint8_t *qT, float *scale_inv,
                                                     float *amax_out, uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols || (cols % 16) || (rows % 16)) return FP8_ERR_SHAPE;
    if ((rows + 63) / 64 > 65535 || (rows + kColRows - 1) / kColRows > 65535) return FP8_ERR_SHAPE;
    if (rows > 0 && cols > 0 && (!x_bf16 || !qT || !scale_inv || !amax_out)) return FP8_ERR_INVALID_ARG;
    if (ld % 8) return FP8_ERR_ALIGNMENT;
    if ((x_bf16 && !aligned16(x_bf16)) || (qT && !aligned16(qT)) || !counts_ok(counts)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (rows == 0 || cols == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    const uint16_t *xs = static_cast<const uint16_t *>(x_bf16);
    if (rows <= kQtMaxRows) {   // one launch, one read of x from HBM
        cudaError_t e;
        if (fmt == FP8_E4M3)
            e = pow2 ? launch_qt_strip<FP8_E4M3, true>(s, xs, qT, rows, cols, ld, scale_inv, amax_out, counts)
                     : launch_qt_strip<FP8_E4M3, false>(s, xs, qT, rows, cols, ld, scale_inv, amax_out, counts);
        else
            e = pow2 ? launch_qt_strip<FP8_E5M2, true>(s, xs, qT, rows, cols, ld, scale_inv, amax_out, counts)
                     : launch_qt_strip<FP8_E5M2, false>(s, xs, qT, rows, cols, ld, scale_inv, amax_out, counts);
        return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
    }
    uint32_t *amax_bits = reinterpret_cast<uint32_t *>(amax_out);
    if (cudaMemsetAsync(amax_bits, 0, (size_t)cols * sizeof(uint32_t), s) != cudaSuccess) return FP8_ERR_CUDA;
    k_colamax<<<dim3((unsigned)((cols + 255) / 256), (unsigned)((rows + kColRows - 1) / kColRows)), 256, 0, s>>>(
        xs, rows, cols, ld, amax_bits);
    const dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
    if (fmt == FP8_E4M3) {
        if (pow2) k_cast_transpose_col<FP8_E4M3, true><<<grid, 128, 0, s>>>(xs, qT, rows, cols, ld, amax_bits, scale_inv, counts);
        else k_cast_transpose_col<FP8_E4M3, false><<<grid, 128, 0, s>>>(xs, qT, rows, cols, ld, amax_bits, scale_inv, counts);
    } else {
        if (pow2) k_cast_transpose_col<FP8_E5M2, true><<<grid, 128, 0, s>>>(xs, qT, rows, cols, ld, amax_bits, scale_inv, counts);
        else k_cast_transpose_col<FP8_E5M2, false><<<grid, 128, 0, s>>>(xs, qT, rows, cols, ld, amax_bits, scale_inv, counts);
    }
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_quantize_blockwise_e8m0(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                                  fp8_format fmt, int block_rows, uint8_t *q, uint8_t *sf_image,
                                                  uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (block_rows != 1 && block_rows != 128) return FP8_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols || (cols % 16)) return FP8_ERR_SHAPE;
    if (rows > 0 && cols > 0 && (!x_bf16 || !q || !sf_image)) return FP8_ERR_INVALID_ARG;
    if (ld % 8) return FP8_ERR_ALIGNMENT;
    if ((x_bf16 && !aligned16(x_bf16)) || (q && !aligned16(q)) || (sf_image && !aligned16(sf_image)) ||
        !counts_ok(counts))
        return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (rows == 0 || cols == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    const cudaError_t e =
        (fmt == FP8_E4M3)
            ? launch_block<FP8_E4M3, true>(s, sms, x_bf16, rows, cols, ld, block_rows, q, nullptr, sf_image, counts)
            : launch_block<FP8_E5M2, true>(s, sms, x_bf16, rows, cols, ld, block_rows, q, nullptr, sf_image, counts);
    return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
