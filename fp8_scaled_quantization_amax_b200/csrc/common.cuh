// common.cuh -- device helpers shared by the FP8 quantization kernels and the
// host-side validation used by every entry point.
//
// Numerics (bit-exact contract of the quantizers):
//   * amax is max |x| over the finite bf16 elements: exact, order independent.
//   * s = fmax / amax is one IEEE round-to-nearest fp32 division (__fdiv_rn);
//     amax == 0 gives 1, an overflowing quotient is clamped to FLT_MAX.
//   * the power-of-two scale keeps only the exponent of that quotient (the
//     largest 2^k not above it, clamped to [2^-126, 2^127]).
//   * the cast is y = x * s with one rounded fp32 multiply (__fmul_rn, never
//     contracted into an FMA), then the hardware's saturating
//     round-to-nearest-even convert (cvt.rn.satfinite.{e4m3,e5m2}x2.f32).
//   * no flush-to-zero anywhere (the library is built without fast math).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fp8q.h"

namespace fp8q {

// Largest finite magnitude of each format: E4M3 448, E5M2 57344.
template <int FMT>
__host__ __device__ constexpr float fmax_of() { return FMT == FP8_E4M3 ? 448.0f : 57344.0f; }

__device__ __forceinline__ float scale_from_amax(float amax, float fm) {
    if (!(amax > 0.0f)) return 1.0f;
    float s = __fdiv_rn(fm, amax);
    if (isinf(s)) s = 3.402823466e38f;
    return s;
}

__device__ __forceinline__ float pow2_scale_from_amax(float amax, float fm) {
    if (!(amax > 0.0f)) return 1.0f;
    uint32_t e = __float_as_uint(__fdiv_rn(fm, amax)) & 0x7F800000u;
    if (e == 0x7F800000u) e = 0x7F000000u;   // 2^127
    if (e == 0u) e = 0x00800000u;            // 2^-126
    return __uint_as_float(e);
}

// E8M0 scale image (the operand layout of the hardware block-scaled MMA,
// which reads one byte per row for every 32-wide K slice; a 32-bit word holds
// four such bytes).  Here a byte carries a whole 128-wide K block, so one word
// covers four K blocks: for K block kb and row r the byte at
//   ((kb / 4) * ceil(rows / 128) + r / 128) * 512 + (r % 32) * 16
//     + ((r % 128) / 32) * 4 + kb % 4
// holds the biased exponent e of the dequantization factor 2^(e - 127).  For
// a power-of-two scale s = 2^k the factor is 2^-k, so e = 127 - k
// = 254 - (biased exponent of s).
__device__ __forceinline__ uint8_t e8m0_of_scale(float s) {
    return (uint8_t)(254u - ((__float_as_uint(s) >> 23) & 0xFFu));
}
__device__ __forceinline__ int64_t e8m0_offset(int64_t kb, int64_t rt, int64_t r) {
    return ((kb >> 2) * rt + (r >> 7)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (kb & 3);
}

// Two bf16 in a 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Saturating RNE cast of two fp32 values to two FP8 codes; a lands in the low byte.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float a, float b) {
    uint16_t r;
    if (FMT == FP8_E4M3)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Cast one 32-bit word (two bf16) scaled by s to two FP8 codes (16 bits).
template <int FMT>
__device__ __forceinline__ uint32_t cast_word(uint32_t w, float s) {
    return cvt2<FMT>(__fmul_rn(bf_lo(w), s), __fmul_rn(bf_hi(w), s));
}

// Eight bf16 (uint4) -> eight FP8 codes (uint2).
template <int FMT>
__device__ __forceinline__ uint2 cast8(uint4 v, float s) {
    uint2 o;
    o.x = cast_word<FMT>(v.x, s) | (cast_word<FMT>(v.y, s) << 16);
    o.y = cast_word<FMT>(v.z, s) | (cast_word<FMT>(v.w, s) << 16);
    return o;
}

// Two FP8 codes (low 16 bits of c) -> two fp32 (exact, via f16x2).
template <int FMT>
__device__ __forceinline__ float2 fp8x2_to_float2(uint16_t c) {
    uint32_t h;
    if (FMT == FP8_E4M3)
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
    else
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(c));
    __half2 hh = *reinterpret_cast<__half2 *>(&h);
    return __half22float2(hh);
}

// fp32 pair -> packed bf16x2 (RNE), a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

// ---------------------------------------------------------------- amax ----
// Fast running max over packed bf16 pairs: |x| via the sign mask, then a
// NaN-propagating bf16x2 max.  If the result is non-finite (some element was
// NaN or Inf) the caller redoes its elements with amax_exact_word(), which
// skips non-finite values and counts them.
__device__ __forceinline__ uint32_t amax_fast_word(uint32_t m, uint32_t w) {
    uint32_t a = w & 0x7FFF7FFFu;
    uint32_t r;
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(a));
    return r;
}
__device__ __forceinline__ uint32_t amax_fast8(uint32_t m, uint4 v) {
    m = amax_fast_word(m, v.x);
    m = amax_fast_word(m, v.y);
    m = amax_fast_word(m, v.z);
    return amax_fast_word(m, v.w);
}
// Packed running max -> the max magnitude bits (of one bf16, as uint32), or
// 0xFFFFFFFF if a non-finite value was seen.
__device__ __forceinline__ uint32_t amax_fast_final(uint32_t m) {
    uint32_t lo = m & 0xFFFFu, hi = m >> 16;
    if (lo >= 0x7F80u || hi >= 0x7F80u) return 0xFFFFFFFFu;
    return lo > hi ? lo : hi;
}
// Exact: max over finite magnitudes (bf16 bits), counting non-finite ones.
__device__ __forceinline__ uint32_t amax_exact_word(uint32_t m, uint32_t w, uint32_t &bad) {
    uint32_t lo = w & 0x7FFFu, hi = (w >> 16) & 0x7FFFu;
    if (lo < 0x7F80u) { m = lo > m ? lo : m; } else { ++bad; }
    if (hi < 0x7F80u) { m = hi > m ? hi : m; } else { ++bad; }
    return m;
}
__device__ __forceinline__ uint32_t amax_exact8(uint32_t m, uint4 v, uint32_t &bad) {
    m = amax_exact_word(m, v.x, bad);
    m = amax_exact_word(m, v.y, bad);
    m = amax_exact_word(m, v.z, bad);
    return amax_exact_word(m, v.w, bad);
}
// bf16 magnitude bits -> fp32 value.
__device__ __forceinline__ float bf16bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// Number of elements among 8 (uint4 of bf16) whose scaled magnitude exceeds fm.
__device__ __forceinline__ uint32_t count_sat8(uint4 v, float s, float fm) {
    uint32_t c = 0;
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a = __fmul_rn(bf_lo(w[i]), s), b = __fmul_rn(bf_hi(w[i]), s);
        c += (fabsf(a) > fm) ? 1u : 0u;
        c += (fabsf(b) > fm) ? 1u : 0u;
    }
    return c;
}

// Non-finite elements among 8 bf16 (NaN or +-Inf: every exponent bit set).
__device__ __forceinline__ uint32_t count_nonfinite8(uint4 v) {
    uint32_t c = 0;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        c += ((w[i] & 0x7F80u) == 0x7F80u) ? 1u : 0u;
        c += ((w[i] & 0x7F800000u) == 0x7F800000u) ? 1u : 0u;
    }
    return c;
}

// Counters of the quantizers (counts[0] non-finite inputs, counts[1]
// saturated elements = |fp32(x) * s| > fmax, NaN excluded, +-Inf included):
// a unit (row, block, slice) can only have saturated elements when it holds
// a non-finite value or when fp32(amax) * s rounds above fmax, so the
// kernels count exactly only then.  The warp's per-thread counts are summed
// and added by lane 0 (warp-collective: all 32 lanes call it).
__device__ __forceinline__ bool may_saturate(bool nonfinite_seen, float amax, float s, float fm) {
    return nonfinite_seen || __fmul_rn(amax, s) > fm;
}
__device__ __forceinline__ void flush_counts(uint32_t *counts, uint32_t nf, uint32_t sat) {
    nf = __reduce_add_sync(0xFFFFFFFFu, nf);
    sat = __reduce_add_sync(0xFFFFFFFFu, sat);
    if ((threadIdx.x & 31) == 0) {
        if (nf) atomicAdd(counts, nf);
        if (sat) atomicAdd(counts + 1, sat);
    }
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// L2 eviction-priority policies and loads / stores carrying them.
__device__ __forceinline__ uint2 ld_stream_u2(const uint2 *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

// Programmatic dependent launch.  A kernel launched with pdl_launch() may
// start while the previous kernel in the stream is still running; it calls
// pdl_wait() before its first global-memory access, which returns once that
// kernel has completed and its writes are visible, so stream order is kept.
// pdl_trigger() lets the next kernel be scheduled (it will wait in turn):
// called once every CTA of this grid is resident, so a dependent grid never
// takes an SM one of our CTAs still needs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint4 *p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}
__device__ __forceinline__ void st_hint(uint4 *p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w), "l"(pol)
                 : "memory");
}

// Block-wide max of a uint32 (all threads get the result).  smem >= 32 words.
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t *smem) {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = (blockDim.x + 31) >> 5;
    __syncthreads();
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    uint32_t r = lane < nwarps ? smem[lane] : 0u;
    r = __reduce_max_sync(0xFFFFFFFFu, r);
    return r;
}
__device__ __forceinline__ uint32_t block_sum_u32(uint32_t v, uint32_t *smem) {
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = (blockDim.x + 31) >> 5;
    __syncthreads();
    if (lane == 0) smem[warp] = v;
    __syncthreads();
    uint32_t r = lane < nwarps ? smem[lane] : 0u;
    r = __reduce_add_sync(0xFFFFFFFFu, r);
    return r;
}

}  // namespace fp8q

// ------------------------------------------------------------- host side --
namespace fp8q_host {
// Launch with programmatic stream serialization allowed (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t pdl_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
// The same, with 1-D thread-block clusters of `cluster_x` CTAs chosen at launch.
template <typename... KArgs, typename... Args>
inline cudaError_t pdl_launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = cluster_x;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}


// Current device must be compute capability 10.0 (B200, sm_100a); cached
// per device ordinal.  Also returns the SM count.
fp8_status check_device(int *sm_count);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace fp8q_host
