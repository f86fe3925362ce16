// kv.cu -- FP8 KV cache: per-(batch, head) quantize and dequantize.
//
// Source: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §3.1 (K and V kept
// in FP8 halve the cache; each is dequantized when attention reads it).
//
// Quantize: a (b, h) slice (S*Dh elements, 2 MiB of bf16 at S=8192, Dh=128)
// needs its own amax before any element can be cast.  One 8-CTA thread-block
// cluster (two 512-thread CTAs per SM) owns one slice at a time: every CTA
// streams its eighth of the slice from HBM for the amax (loads marked L2
// evict-last), the eight partial maxima meet through distributed shared
// memory behind a cluster barrier, and the cast pass re-reads the same eighth
// from L2 (loads and FP8 stores marked evict-first, so the slices still
// waiting for their second pass stay resident; about 37 clusters x 2 MiB are
// in flight against the 126 MB L2).
// HBM traffic is the algorithmic 2 B in + 1 B out per element, in one
// launch, with no scratch memory and no grid-wide wait.
//
// Dequantize: each CTA streams a contiguous 256 KiB of FP8 codes (16 codes
// in per 16-byte load); the bf16 results go through shared memory and leave
// in 32 KiB bulk copies.  Contiguous per-CTA chunks keep the write-heavy
// stream at DRAM-page locality (a grid-stride layout measured ~20 % slower).
// One scale per (b, h) from the grid's y index.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"

namespace cg = cooperative_groups;
using namespace fp8q;

namespace {

constexpr int kClusterCtas = 8;
constexpr int kKvThreads = 512;

// COUNT: the non-finite / saturated counters (a separate instantiation, so
// the plain path keeps its registers).
template <int FMT, bool COUNT>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kKvThreads, 2)
k_kv_quant(const uint4 *__restrict__ x, uint4 *__restrict__ q, int64_t BH, int64_t nunit,
           float *__restrict__ scale_inv, uint32_t *__restrict__ counts) {
    __shared__ uint32_t red[32];
    __shared__ uint32_t slot[2];        // this CTA's partial amax, double-buffered by slice parity
    __shared__ uint32_t slice_amax;
    constexpr float fm = fmax_of<FMT>();
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank();
    const int64_t cid = blockIdx.x / kClusterCtas, ncl = gridDim.x / kClusterCtas;
    const int64_t per = (nunit + kClusterCtas - 1) / kClusterCtas;
    const int64_t u0 = min((int64_t)rank * per, nunit);
    const int64_t u1 = min(u0 + per, nunit);
    const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
    uint32_t nf = 0, sat = 0;   // counters (counts != NULL)
    int it = 0;
    for (int64_t sl = cid; sl < BH; sl += ncl, ++it) {
        const uint4 *xs = x + 2 * sl * nunit;   // a unit is 16 elements = two uint4 of bf16
        uint4 *qs = q + sl * nunit;             // and one uint4 of FP8
        // pass 1: amax of this CTA's part of the slice
        uint32_t m2 = 0;
        int64_t u = u0 + threadIdx.x;
        for (; u + 3 * kKvThreads < u1; u += 4 * kKvThreads) {
            uint4 v[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[2 * k] = ld_hint(xs + 2 * (u + k * kKvThreads), keep);
                v[2 * k + 1] = ld_hint(xs + 2 * (u + k * kKvThreads) + 1, keep);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) m2 = amax_fast8(m2, v[k]);
        }
        for (; u < u1; u += kKvThreads)
            m2 = amax_fast8(amax_fast8(m2, ld_hint(xs + 2 * u, keep)), ld_hint(xs + 2 * u + 1, keep));
        uint32_t m = amax_fast_final(m2);
        const bool nonfin = m == 0xFFFFFFFFu;
        if (nonfin) {
            uint32_t bad = 0;
            m = 0;
            for (int64_t j = u0 + threadIdx.x; j < u1; j += kKvThreads)
                m = amax_exact8(amax_exact8(m, xs[2 * j], bad), xs[2 * j + 1], bad);
        }
        m = block_max_u32(m, red);
        if (threadIdx.x == 0) slot[it & 1] = m;
        cluster.sync();   // every CTA's partial is published
        if (threadIdx.x < 32) {
            uint32_t v = 0;
            if (threadIdx.x < kClusterCtas) v = *cluster.map_shared_rank(&slot[it & 1], threadIdx.x);
            v = __reduce_max_sync(0xFFFFFFFFu, v);
            if (threadIdx.x == 0) slice_amax = v;
        }
        __syncthreads();
        const float s = scale_from_amax(bf16bits_to_float(slice_amax), fm);
        if (rank == 0 && threadIdx.x == 0) scale_inv[sl] = __fdiv_rn(1.0f, s);
        // exact counts where this thread saw a non-finite value or the slice may saturate
        const bool cnt = COUNT && may_saturate(nonfin, bf16bits_to_float(slice_amax), s, fm);
        // pass 2: cast (the re-read hits L2)
        int64_t j = u0 + threadIdx.x;
        for (; j + 3 * kKvThreads < u1; j += 4 * kKvThreads) {
            uint4 v[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[2 * k] = ld_hint(xs + 2 * (j + k * kKvThreads), drop);
                v[2 * k + 1] = ld_hint(xs + 2 * (j + k * kKvThreads) + 1, drop);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint2 c0 = cast8<FMT>(v[2 * k], s), c1 = cast8<FMT>(v[2 * k + 1], s);
                st_hint(qs + j + k * kKvThreads, make_uint4(c0.x, c0.y, c1.x, c1.y), drop);
                if (COUNT && cnt) {
                    nf += count_nonfinite8(v[2 * k]) + count_nonfinite8(v[2 * k + 1]);
                    sat += count_sat8(v[2 * k], s, fm) + count_sat8(v[2 * k + 1], s, fm);
                }
            }
        }
        for (; j < u1; j += kKvThreads) {
            uint4 a0 = ld_hint(xs + 2 * j, drop), a1 = ld_hint(xs + 2 * j + 1, drop);
            uint2 c0 = cast8<FMT>(a0, s), c1 = cast8<FMT>(a1, s);
            st_hint(qs + j, make_uint4(c0.x, c0.y, c1.x, c1.y), drop);
            if (COUNT && cnt) {
                nf += count_nonfinite8(a0) + count_nonfinite8(a1);
                sat += count_sat8(a0, s, fm) + count_sat8(a1, s, fm);
            }
        }
    }
    if (COUNT) flush_counts(counts, nf, sat);
    cluster.sync();   // no CTA leaves while a peer may still read its slots
}

template <int FMT>
__device__ __forceinline__ void dequant16(uint4 c, float d, uint4 &o0, uint4 &o1) {
    uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 lo = fp8x2_to_float2<FMT>((uint16_t)(w[i] & 0xFFFFu));
        float2 hi = fp8x2_to_float2<FMT>((uint16_t)(w[i] >> 16));
        o[2 * i] = pack_bf16x2(__fmul_rn(lo.x, d), __fmul_rn(lo.y, d));
        o[2 * i + 1] = pack_bf16x2(__fmul_rn(hi.x, d), __fmul_rn(hi.y, d));
    }
    o0 = make_uint4(o[0], o[1], o[2], o[3]);
    o1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// A CTA dequantizes the contiguous units [blockIdx.x * per, +per) of slice
// blockIdx.y (a unit = 16 codes = 32 bytes of bf16 out).  Per round each of
// the 256 threads loads four units' codes (16 KiB per CTA in flight), writes
// their bf16 values into one of two 32 KiB shared-memory buffers, and one
// thread sends the buffer to global memory with a single bulk copy
// (cp.async.bulk), so the write stream -- two thirds of the traffic -- costs
// no per-thread global stores: with two 16-byte stores per unit the
// load/store queue throttled the kernel (ncu: lg_throttle the top stall).
constexpr int64_t kDequantUnitsPerCta = 16384;   // 256 KiB of FP8 codes
constexpr int kDqThreads = 256;
constexpr int kDqRound = 4 * kDqThreads;          // units per round
constexpr int kDqBuf = kDqRound * 32;             // bytes of bf16 per round
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int FMT>
__global__ void __launch_bounds__(kDqThreads)
k_kv_dequant(const uint4 *__restrict__ q, const float *__restrict__ scale_inv, int64_t nunit,
             uint4 *__restrict__ out) {
    extern __shared__ __align__(128) uint8_t dq_smem[];   // two buffers of kDqBuf bytes
    const int64_t sl = blockIdx.y;
    const float d = scale_inv[sl];
    const uint4 *qs = q + sl * nunit;
    uint4 *os = out + 2 * sl * nunit;
    const int64_t u0 = blockIdx.x * kDequantUnitsPerCta;
    const int64_t u1 = min(u0 + kDequantUnitsPerCta, nunit);
    int buf = 0;
    for (int64_t r0 = u0; r0 < u1; r0 += kDqRound, buf ^= 1) {
        uint4 c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t u = r0 + threadIdx.x + k * kDqThreads;
            c[k] = u < u1 ? ld_stream(qs + u) : make_uint4(0, 0, 0, 0);
        }
        // the bulk copy issued from this buffer two rounds ago has read it
        if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncthreads();
        const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(dq_smem)) + (uint32_t)(buf * kDqBuf);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint4 o0, o1;
            dequant16<FMT>(c[k], d, o0, o1);
            const uint32_t a = base + (uint32_t)(threadIdx.x + k * kDqThreads) * 32u;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o0.x), "r"(o0.y), "r"(o0.z), "r"(o0.w)
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a + 16), "r"(o1.x), "r"(o1.y), "r"(o1.z),
                         "r"(o1.w)
                         : "memory");
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the bulk copy
        __syncthreads();
        if (threadIdx.x == 0) {
            const int64_t n = min((int64_t)kDqRound, u1 - r0);
            bulk_store(os + 2 * r0, base, (uint32_t)(n * 32));
        }
    }
    if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace

using namespace fp8q_host;

// Clusters of the quantize kernel that fit on the device at once (GPCs hold a
// whole number of 8-SM clusters, so this is below sm_count / 8); cached per
// device.  The grid never exceeds it, so no cluster waits for another to
// finish before it can start.
template <int FMT, bool COUNT>
static int max_active_clusters() {
    static int cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] > 0) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCtas * 64);
    cfg.blockDim = dim3(kKvThreads);
    cfg.dynamicSmemBytes = 0;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kClusterCtas;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_kv_quant<FMT, COUNT>, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

static fp8_status kv_check(int64_t B, int64_t H, int64_t S, int64_t Dh) {
    if (B < 0 || H < 0 || S < 0 || Dh < 0) return FP8_ERR_SHAPE;
    if ((S * Dh) % 16) return FP8_ERR_SHAPE;
    if (B * H > 65535 && S * Dh > 0) return FP8_ERR_SHAPE;   // one grid row per (b, h) slice
    return FP8_OK;
}

extern "C" fp8_status fp8_kv_quant(const void *kv_bf16, int64_t B, int64_t H, int64_t S, int64_t Dh,
                                   fp8_format fmt, uint8_t *q, float *scale_inv, uint32_t *counts, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    fp8_status c = kv_check(B, H, S, Dh);
    if (c != FP8_OK) return c;
    const int64_t BH = B * H, nunit = S * Dh / 16;
    if (BH > 0 && (!scale_inv || (nunit > 0 && (!kv_bf16 || !q)))) return FP8_ERR_INVALID_ARG;
    if ((kv_bf16 && !aligned16(kv_bf16)) || (q && !aligned16(q))) return FP8_ERR_ALIGNMENT;
    if (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (BH == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    const bool cnt = counts != nullptr;
    const int active = fmt == FP8_E4M3 ? (cnt ? max_active_clusters<FP8_E4M3, true>() : max_active_clusters<FP8_E4M3, false>())
                                       : (cnt ? max_active_clusters<FP8_E5M2, true>() : max_active_clusters<FP8_E5M2, false>());
    if (active <= 0) return FP8_ERR_CUDA;
    const int clusters = (int)std::max<int64_t>(1, std::min<int64_t>(BH, active));
    const dim3 grid(clusters * kClusterCtas);
    const uint4 *xv = static_cast<const uint4 *>(kv_bf16);
    uint4 *qv = reinterpret_cast<uint4 *>(q);
    if (fmt == FP8_E4M3) {
        if (cnt) k_kv_quant<FP8_E4M3, true><<<grid, kKvThreads, 0, s>>>(xv, qv, BH, nunit, scale_inv, counts);
        else k_kv_quant<FP8_E4M3, false><<<grid, kKvThreads, 0, s>>>(xv, qv, BH, nunit, scale_inv, counts);
    } else {
        if (cnt) k_kv_quant<FP8_E5M2, true><<<grid, kKvThreads, 0, s>>>(xv, qv, BH, nunit, scale_inv, counts);
        else k_kv_quant<FP8_E5M2, false><<<grid, kKvThreads, 0, s>>>(xv, qv, BH, nunit, scale_inv, counts);
    }
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_kv_dequant(const uint8_t *q, const float *scale_inv, int64_t B, int64_t H,
                                     int64_t S, int64_t Dh, fp8_format fmt, void *out_bf16, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    fp8_status c = kv_check(B, H, S, Dh);
    if (c != FP8_OK) return c;
    const int64_t BH = B * H, nunit = S * Dh / 16;
    if (BH > 0 && nunit > 0 && (!q || !scale_inv || !out_bf16)) return FP8_ERR_INVALID_ARG;
    if ((q && !aligned16(q)) || (out_bf16 && !aligned16(out_bf16))) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (BH == 0 || nunit == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    const int64_t per_slice = (nunit + kDequantUnitsPerCta - 1) / kDequantUnitsPerCta;
    if (per_slice > 2147483647LL) return FP8_ERR_SHAPE;
    const dim3 grid((unsigned)per_slice, (unsigned)BH);
    static bool attr_set[64][2];   // per device: the 64 KiB of shared memory needs the opt-in
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
    if (!attr_set[dev][fmt]) {
        const cudaError_t e = (fmt == FP8_E4M3)
            ? cudaFuncSetAttribute(k_kv_dequant<FP8_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kDqBuf)
            : cudaFuncSetAttribute(k_kv_dequant<FP8_E5M2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kDqBuf);
        if (e != cudaSuccess) return FP8_ERR_CUDA;
        attr_set[dev][fmt] = true;
    }
    if (fmt == FP8_E4M3)
        k_kv_dequant<FP8_E4M3><<<grid, kDqThreads, 2 * kDqBuf, s>>>(reinterpret_cast<const uint4 *>(q), scale_inv, nunit, static_cast<uint4 *>(out_bf16));
    else
        k_kv_dequant<FP8_E5M2><<<grid, kDqThreads, 2 * kDqBuf, s>>>(reinterpret_cast<const uint4 *>(q), scale_inv, nunit, static_cast<uint4 *>(out_bf16));
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
