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
// thread's loads of both snapshots for a batch of 16 in flight together: one
// DRAM round trip covers 8192 scales.
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
constexpr int kUnroll = 16;
constexpr int kBigCluster = 8;
constexpr int64_t kBigSegment = 32768;   // average segment length above which clusters are used

struct Acc {
    uint32_t mn, mx;   // bit patterns of positive finite floats (ordered as integers)
    double sum;
    uint32_t nv, jumps, invalid;
};

// "RN(v / p) > r" for positive finite v, p without the division (the
// correctly rounded fp32 division is a long instruction sequence and made
// this kernel issue-bound).  RN(q) > r exactly when q lies above the midpoint
// mid = r + ulp(r)/2, or on it when the value above r has an even mantissa;
// mid needs 25 significant bits and p 24, so mid * p is exact in fp64 and the
// comparison with v is exact too.
struct Ratio {
    double mid;
    bool tie_up;
};
__device__ __forceinline__ Ratio ratio_threshold(float r) {
    const uint32_t rb = __float_as_uint(r);
    const float up = __uint_as_float(rb + 1u);   // the next float above r (+inf above FLT_MAX)
    const double ulp = isinf(up) ? 20282409603651670423947251286016.0 /* 2^104 */ : (double)up - (double)r;
    return Ratio{(double)r + 0.5 * ulp, (rb & 1u) != 0u};
}
__device__ __forceinline__ bool ratio_above(float v, float p, const Ratio &t) {
    const double x = (double)v, y = t.mid * (double)p;
    return x > y || (x == y && t.tie_up);
}

// p is the previous snapshot's entry, or NaN when there is none (NaN fails
// the validity test, so it never counts as a step change)
__device__ __forceinline__ void visit(Acc &a, float v, float p, const Ratio &t) {
    if (v > 0.0f && v <= FLT_MAX) {
        const uint32_t b = __float_as_uint(v);
        a.mn = b < a.mn ? b : a.mn;
        a.mx = b > a.mx ? b : a.mx;
        a.sum += (double)v;
        a.nv += 1;
        if (p > 0.0f && p <= FLT_MAX && (ratio_above(v, p, t) || ratio_above(p, v, t))) a.jumps += 1;
    } else {
        a.invalid += 1;
    }
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

    Acc a{0x7F800000u, 0u, 0.0, 0u, 0u, 0u};
    const Ratio rt = ratio_threshold(r);
    const int64_t step = (int64_t)kThreads * kUnroll;
    int64_t base = c0 + threadIdx.x;
    for (; base + (kUnroll - 1) * kThreads < c1; base += step) {
        float v[kUnroll], p[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {   // every load of the batch in flight at once
            v[u] = __ldg(s + base + u * kThreads);
            p[u] = prev ? __ldg(prev + base + u * kThreads) : __int_as_float(0x7FC00000);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) visit(a, v[u], p[u], rt);
    }
    {   // the ragged end: its loads also issued together
        float v[kUnroll], p[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = base + u * kThreads;
            v[u] = i < c1 ? __ldg(s + i) : 1.0f;
            p[u] = (i < c1 && prev) ? __ldg(prev + i) : __int_as_float(0x7FC00000);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (base + u * kThreads < c1) visit(a, v[u], p[u], rt);
    }

    warp_reduce(a);
    __shared__ Acc part[kThreads / 32];
    __shared__ Acc cta;   // this CTA's partial (read by the leading CTA of a cluster)
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) part[w] = a;
    __syncthreads();
    if (w == 0) {
        a = lane < kThreads / 32 ? part[lane] : Acc{0x7F800000u, 0u, 0.0, 0u, 0u, 0u};
        warp_reduce(a);
        if (lane == 0) cta = a;
    }
    if (CL > 1) {
        cg::this_cluster().sync();   // every CTA's partial is published
        if (rank == 0 && w == 0) {
            a = lane < CL ? *cg::this_cluster().map_shared_rank(&cta, lane) : Acc{0x7F800000u, 0u, 0.0, 0u, 0u, 0u};
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
