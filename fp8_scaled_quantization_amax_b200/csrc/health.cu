// health.cu -- health check of scale factors.
//
// Source: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §6.2: print the
// min / max / mean of every layer's scale factors at intervals and check that
// they drift slowly; a step change in a scale is the early sign of an outlier
// or a shift of the data distribution.  Readings taken here: a scale is valid
// when finite and > 0; a step change is a ratio to the previous snapshot's
// scale above a caller threshold, in either direction.
//
// One CTA of 512 threads per segment (a layer's scales), two CTAs per SM, a
// thread's 16-byte loads of both snapshots for a batch of 4 vectors in flight
// together: one DRAM round trip covers 8192 scales.  Per entry the work is
// branch-free integer and fp64 arithmetic (no division).
// Segments averaging more than 32768 scales get a cluster of 8 CTAs each,
// every CTA reducing a contiguous eighth, combined by the leading CTA through
// distributed shared memory in rank order.  The sum is kept in fp64 and every
// reduction runs in a fixed order, so a result never depends on timing.
#include <cooperative_groups.h>

#include <cfloat>

#include "common.cuh"

namespace cg = cooperative_groups;
using namespace fp8q;

namespace {

constexpr int kThreads = 512;
constexpr int kUnroll = 4;   // float4 vectors per thread and snapshot in one batch
constexpr int kBigCluster = 8;
constexpr int64_t kBigSegment = 32768;   // average segment length above which clusters are used

struct Acc {
    uint32_t mn, mx;   // bit patterns of positive finite floats (ordered as integers)
    double sum;
    uint32_t nv, jumps, invalid;
};

// "RN(v / p) > r" for positive finite v, p without the division (the
// correctly rounded fp32 division is a long instruction sequence).  RN(q) > r
// exactly when q lies above the midpoint mid = r + ulp(r)/2 (q on the
// midpoint would need v = mid * p, whose odd significand has at least the
// 25 bits of mid's: no fp32 v is there, so there is no tie to break).  mid
// has 25 significant bits and p 24, so mid * p is exact in fp64 and so is
// the comparison with v.
__device__ __forceinline__ double ratio_midpoint(float r) {
    const uint32_t rb = __float_as_uint(r);
    const float up = __uint_as_float(rb + 1u);   // the next float above r (+inf above FLT_MAX)
    const double ulp = isinf(up) ? 20282409603651670423947251286016.0 /* 2^104 */ : (double)up - (double)r;
    return (double)r + 0.5 * ulp;
}

// One entry, branch-free.  Valid: the bits of a positive finite float, 1 ..
// 0x7F7FFFFF.  p is the previous snapshot's entry (NaN when there is none,
// which is never valid, so it never counts as a step change).  Invalid
// entries are counted at the end as (entries - valid).
__device__ __forceinline__ void visit(Acc &a, float v, float p, double mid) {
    const uint32_t b = __float_as_uint(v), pb = __float_as_uint(p);
    const bool ok = (b - 1u) < 0x7F7FFFFFu;
    const bool pok = (pb - 1u) < 0x7F7FFFFFu;
    a.mn = min(a.mn, ok ? b : 0xFFFFFFFFu);
    a.mx = max(a.mx, ok ? b : 0u);
    const double x = (double)v, y = (double)p;
    a.sum += ok ? x : 0.0;
    a.nv += ok ? 1u : 0u;
    a.jumps += (ok && pok && (x > mid * y || y > mid * x)) ? 1u : 0u;
}
__device__ __forceinline__ void visit4(Acc &a, float4 v, float4 p, double mid) {
    visit(a, v.x, p.x, mid);
    visit(a, v.y, p.y, mid);
    visit(a, v.z, p.z, mid);
    visit(a, v.w, p.w, mid);
}

__device__ __forceinline__ void warp_reduce(Acc &a) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint32_t mn = __shfl_down_sync(0xFFFFFFFFu, a.mn, o);
        const uint32_t mx = __shfl_down_sync(0xFFFFFFFFu, a.mx, o);
        a.sum += __shfl_down_sync(0xFFFFFFFFu, a.sum, o);
        a.nv += __shfl_down_sync(0xFFFFFFFFu, a.nv, o);
        a.jumps += __shfl_down_sync(0xFFFFFFFFu, a.jumps, o);
        a.invalid += __shfl_down_sync(0xFFFFFFFFu, a.invalid, o);
        a.mn = mn < a.mn ? mn : a.mn;
        a.mx = mx > a.mx ? mx : a.mx;
    }
}

template <int CL>
__global__ void __launch_bounds__(kThreads, 2)
k_scale_stats(const float *__restrict__ s, const float *__restrict__ prev, int64_t n,
              const int64_t *__restrict__ offsets, float r, float *__restrict__ stats,
              uint32_t *__restrict__ counts) {
    const unsigned rank = (CL > 1) ? cg::this_cluster().block_rank() : 0u;
    const int g = blockIdx.x / CL;
    int64_t lo = offsets ? offsets[g] : 0;
    int64_t hi = offsets ? offsets[g + 1] : n;
    lo = lo < 0 ? 0 : (lo > n ? n : lo);   // a corrupted table reads nothing out of range
    hi = hi < lo ? lo : (hi > n ? n : hi);
    const int64_t per = (hi - lo + CL - 1) / CL;
    const int64_t c0 = lo + min((int64_t)rank * per, hi - lo);
    const int64_t c1 = min(c0 + per, hi);

    Acc a{0xFFFFFFFFu, 0u, 0.0, 0u, 0u, 0u};
    const double mid = ratio_midpoint(r);
    const float nan = __int_as_float(0x7FC00000);
    // 16-byte vectors over [a4, b4); the up to 3 + 3 entries around them one by one
    const int64_t a4 = min((c0 + 3) & ~(int64_t)3, c1);
    const int64_t b4 = max(a4, c1 & ~(int64_t)3);
    if ((int64_t)threadIdx.x < a4 - c0) visit(a, s[c0 + threadIdx.x], prev ? prev[c0 + threadIdx.x] : nan, mid);
    if (threadIdx.x >= 4 && (int64_t)threadIdx.x - 4 < c1 - b4)
        visit(a, s[b4 + threadIdx.x - 4], prev ? prev[b4 + threadIdx.x - 4] : nan, mid);
    const float4 *s4 = reinterpret_cast<const float4 *>(s + a4);
    const float4 *p4 = prev ? reinterpret_cast<const float4 *>(prev + a4) : nullptr;
    const int64_t n4 = (b4 - a4) >> 2;
    const float4 nan4 = make_float4(nan, nan, nan, nan);
    int64_t j = threadIdx.x;
    for (; j + (kUnroll - 1) * kThreads < n4; j += (int64_t)kThreads * kUnroll) {
        float4 v[kUnroll], p[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {   // every load of the batch in flight at once
            v[u] = __ldg(s4 + j + u * kThreads);
            p[u] = p4 ? __ldg(p4 + j + u * kThreads) : nan4;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) visit4(a, v[u], p[u], mid);
    }
    {   // the ragged end of the vectors: its loads also issued together
        float4 v[kUnroll], p[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t k = j + u * kThreads;
            v[u] = k < n4 ? __ldg(s4 + k) : nan4;
            p[u] = (k < n4 && p4) ? __ldg(p4 + k) : nan4;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (j + u * kThreads < n4) visit4(a, v[u], p[u], mid);
    }

    warp_reduce(a);
    __shared__ Acc part[kThreads / 32];
    __shared__ Acc cta;   // this CTA's partial (read by the leading CTA of a cluster)
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) part[w] = a;
    __syncthreads();
    if (w == 0) {
        a = lane < kThreads / 32 ? part[lane] : Acc{0xFFFFFFFFu, 0u, 0.0, 0u, 0u, 0u};
        warp_reduce(a);
        a.invalid = (uint32_t)(c1 - c0) - a.nv;
        if (lane == 0) cta = a;
    }
    if (CL > 1) {
        cg::this_cluster().sync();   // every CTA's partial is published
        if (rank == 0 && w == 0) {
            a = lane < CL ? *cg::this_cluster().map_shared_rank(&cta, lane) : Acc{0xFFFFFFFFu, 0u, 0.0, 0u, 0u, 0u};
            warp_reduce(a);   // lanes >= CL hold the identity, so rank order fixes the sum
        }
    } else {
        __syncthreads();
    }
    if (rank == 0 && threadIdx.x == 0) {
        const bool any = a.nv != 0;
        stats[3 * g + 0] = any ? __uint_as_float(a.mn) : 0.0f;
        stats[3 * g + 1] = any ? __uint_as_float(a.mx) : 0.0f;
        stats[3 * g + 2] = any ? (float)(a.sum / (double)a.nv) : 0.0f;
        counts[2 * g + 0] = a.jumps;
        counts[2 * g + 1] = a.invalid;
    }
    if (CL > 1) cg::this_cluster().sync();   // no CTA leaves while the leading CTA may read its partial
}

}  // namespace

using namespace fp8q_host;

extern "C" fp8_status fp8_scale_stats(const float *scales, const float *prev, int64_t n,
                                      const int64_t *seg_offsets, int64_t num_segments, float jump_ratio,
                                      float *stats, uint32_t *counts, void *stream) {
    if (!stats || !counts || n < 0) return FP8_ERR_INVALID_ARG;
    if (n > 0 && !scales) return FP8_ERR_INVALID_ARG;
    if (!(jump_ratio >= 1.0f) || !(jump_ratio <= FLT_MAX)) return FP8_ERR_INVALID_ARG;
    if ((scales && !aligned16(scales)) || (prev && !aligned16(prev))) return FP8_ERR_ALIGNMENT;
    if (seg_offsets ? (num_segments < 1 || num_segments > 0x7FFFFFFF / kBigCluster) : num_segments != 1)
        return FP8_ERR_SHAPE;
    if (n > 0xFFFFFFFFll) return FP8_ERR_SHAPE;   // per-segment counters are 32-bit
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t cs = as_stream(stream);
    if (n / num_segments > kBigSegment) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(num_segments * kBigCluster));
        cfg.blockDim = dim3(kThreads);
        cfg.stream = cs;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = kBigCluster;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, k_scale_stats<kBigCluster>, scales, prev, n, seg_offsets, jump_ratio, stats,
                               counts) != cudaSuccess)
            return FP8_ERR_CUDA;
    } else {
        k_scale_stats<1><<<(unsigned)num_segments, kThreads, 0, cs>>>(scales, prev, n, seg_offsets, jump_ratio,
                                                                        stats, counts);
    }
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
