// gemm_bf16.cu -- the weight-gradient GEMM kept in high precision:
//   dW[m, n] (+)= sum_t dY[t, m] * X[t, n],   bf16 operands, fp32 accumulation
// and fp32 output.
//
// Source: "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
// "FP8 三种缩放配方怎么选": the rowwise_with_gw_hp recipe runs the forward and
// data-gradient GEMMs in FP8 with rowwise scales and keeps the weight
// gradient in high precision (the slowest and most accurate of the three).
//
// Both operands are read as stored, token-major (dY [T, M], X [T, N]): the
// contraction runs over tokens, which is the strided dimension, so A = dY^T
// and B = X^T are "MN-major" operands.  tcgen05.mma reads MN-major bf16 tiles
// directly: TMA boxes of 64 M (or N) elements (128 bytes, 128-byte swizzle) by
// 64 tokens, two boxes per 128-row operand half, and shared-memory
// descriptors with the MN-major canonical layout (64-element chunks LBO =
// 8 KiB apart, 8-token groups SBO = 1 KiB apart; each K step of 16 tokens
// advances 2 KiB).  No transpose pass.
//
// Structure as the FP8 pair kernel: a CTA pair (cluster of 2) per 256 x 256
// tile, tcgen05.mma.cta_group::2.kind::f16 256x256x16 issued by the even CTA,
// 6-stage TMA ring (32 KiB per stage and CTA), two 256-column TMEM
// accumulators so the epilogue of tile i overlaps the MMAs of tile i + 1,
// 8 epilogue warps storing fp32 rows (optionally adding the previous dW, for
// gradient accumulation over micro-batches).  Every wait is bounded as in
// the other GEMM files.
#include <algorithm>
#include <mutex>

#include "tc.cuh"

using namespace fp8q;
using fp8q_host::pdl_launch;

namespace {

namespace wg {
constexpr int BT = 64;                    // tokens (K) per stage
constexpr int HALF_TILE = 128 * BT * 2;   // 128 rows x 64 tokens of bf16 = 16 KiB
constexpr int STAGE = 2 * HALF_TILE;      // this CTA's A half and B half
constexpr int STAGES = 6;
constexpr int NBUF = 2;
constexpr int NBARS = 2 * STAGES + 2 * NBUF + 1;
// after the pipeline and the barriers: one store_rows_coalesced buffer per epilogue warp
constexpr size_t EPI_OFF = ((size_t)STAGES * STAGE + NBARS * 8 + 16 + 15) & ~(size_t)15;
constexpr size_t SMEM = 1024 + EPI_OFF + (size_t)sm2::EPI * kEpiBufBytes;
}  // namespace wg

// MN-major operand, 128-byte swizzle: 64-element (128-byte) rows, one per
// token; 8-token groups 1024 bytes apart (SBO); the second 64-element chunk
// of the 128-row half 8 KiB further (LBO).
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);            // start address (16-byte units)
    d |= (uint64_t)((wg::HALF_TILE / 2) >> 4) << 16;    // leading byte offset: next 64-element chunk
    d |= (uint64_t)(1024u >> 4) << 32;                  // stride byte offset: next 8 tokens
    d |= (uint64_t)1u << 46;                            // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                            // layout: SWIZZLE_128B
    return d;
}

__device__ __forceinline__ void tc_mma_pair_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(sm2::THREADS, 1)
k_gemm_bf16_wgrad_2sm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M,
                      int N, int T, uint32_t idesc, float *__restrict__ D, int64_t ldd, int accumulate) {
    constexpr int STG = wg::STAGES, NBUF = wg::NBUF;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)STG * wg::STAGE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + wg::NBARS);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = (rank == 0);
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (M + 255) / 256, num_n = (N + 255) / 256;
    const int tiles = num_m * num_n;
    const int nk = (T + wg::BT - 1) / wg::BT;
    const int n_items = (pair < tiles) ? (tiles - 1 - pair) / npairs + 1 : 0;

    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STG + s]); };
    auto accf_bar = [&](int b) { return smem_u32(&bars[2 * STG + b]); };
    auto acce_bar = [&](int b) { return smem_u32(&bars[2 * STG + NBUF + b]); };
    const uint32_t drain_bar = smem_u32(&bars[2 * STG + 2 * NBUF]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), 2 * sm2::EPI);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // both CTAs' barriers are initialised before any remote signal
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();      // inputs of the previous kernel in the stream are visible from here on
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            int last_round[STG];
            for (int s = 0; s < STG; ++s) last_round[s] = -1;
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_items; ++i) {
                const int t = pair + i * npairs;
                const int m0 = (t % num_m) * 256 + (int)rank * 128;   // this CTA's 128 rows of dW
                const int n0 = (t / num_m) * 256 + (int)rank * 128;   // and its half of the 256 columns
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(empty_bar(stage), (round & 1u) ^ 1u, abort_flag, kErrProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(full_bar(stage), 0);
                    if (leader) mbar_expect_tx(full_bar(stage), 2 * wg::STAGE);
                    const uint32_t a_dst = smem_u32(smem + (size_t)stage * wg::STAGE);
                    const uint32_t b_dst = a_dst + wg::HALF_TILE;
                    const int t0 = kc * wg::BT;
                    // 64-element boxes: x = the M (N) index (multiple of 64), y = the token
                    tma_load_2d_pair(a_dst, &tmA, full_leader, m0, t0);
                    tma_load_2d_pair(a_dst + wg::HALF_TILE / 2, &tmA, full_leader, m0 + 64, t0);
                    tma_load_2d_pair(b_dst, &tmB, full_leader, n0, t0);
                    tma_load_2d_pair(b_dst + wg::HALF_TILE / 2, &tmB, full_leader, n0 + 64, t0);
                    last_round[stage] = (int)round;
                }
            }
            if (leader && (!ok || *abort_flag)) {
                for (int s = 0; s < STG; ++s)
                    if (last_round[s] >= 0) wait_bar_drain(full_bar(s), (uint32_t)last_round[s] & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------- MMA issuer (leader only) --
        if (leader && lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_items; ++i) {
                const uint32_t ab = (uint32_t)i % NBUF, use = (uint32_t)i / NBUF;
                if (!wait_bar(acce_bar(ab), (use & 1u) ^ 1u, abort_flag, kErrMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * 256;
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(full_bar(stage), round & 1u, abort_flag, kErrMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)stage * wg::STAGE);
                    const uint64_t adesc = sdesc_mn_sw128(a_addr);
                    const uint64_t bdesc = sdesc_mn_sw128(a_addr + wg::HALF_TILE);
#pragma unroll
                    for (int k = 0; k < wg::BT / 16; ++k)   // 16 tokens = two 8-token groups = 2 KiB
                        tc_mma_pair_bf16(d_tmem, adesc + (uint64_t)(k * 2048 >> 4), bdesc + (uint64_t)(k * 2048 >> 4),
                                         idesc, (kc > 0 || k > 0) ? 1u : 0u);
                    tc_commit_pair_both(empty_bar(stage));
                }
                if (ok) tc_commit_pair_both(accf_bar(ab));
            }
            tc_commit_pair_self(drain_bar);
            wait_bar_drain(drain_bar, 0u);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // --------------------------------------------------- epilogue ----
        const int sp = warp & 3;
        const int ch = (warp - 4) >> 2;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        for (int i = 0; i < n_items; ++i) {
            const int t = pair + i * npairs;
            const uint32_t ab = (uint32_t)i % NBUF, use = (uint32_t)i / NBUF;
            const int64_t m = (int64_t)(t % num_m) * 256 + (int)rank * 128 + sp * 32 + lane;
            const int n_base = (t / num_m) * 256 + ch * 128;
            bool w = true;
            if (lane == 0) w = wait_bar(accf_bar(ab), use & 1u, abort_flag, kErrEpilogue);
            w = __shfl_sync(0xFFFFFFFFu, w, 0);
            if (!w) break;
            tc_fence_after();
            // two 32-column chunks per TMEM round trip; the buffer is released
            // once its last columns are in registers
            uint8_t *ebuf = smem + wg::EPI_OFF + (size_t)(warp - 4) * kEpiBufBytes;
#pragma unroll
            for (int c2 = 0; c2 < 4; c2 += 2) {
                uint32_t r[64];
                tmem_ld32_async(tmem + lane_base + ab * 256 + ch * 128 + c2 * 32, r);
                tmem_ld32_async(tmem + lane_base + ab * 256 + ch * 128 + c2 * 32 + 32, r + 32);
                tmem_wait64(r);
                if (c2 == 2) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar(ab), 0));
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = r[cc * 32 + j];
                    const int col0 = n_base + (c2 + cc) * 32;
                    if (accumulate) store_rows_coalesced<float, true>(ebuf, pk, lane, D, ldd, m - lane, M, col0, N);
                    else store_rows_coalesced<float, false>(ebuf, pk, lane, D, ldd, m - lane, M, col0, N);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();   // every TMEM read and MMA of both CTAs is done
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// 2-D map over a token-major bf16 matrix [T, cols] (row pitch ld elements),
// box 64 x 64 (64 contiguous elements = 128 bytes, 64 tokens), 128-byte
// swizzle; out-of-range boxes read zeros.
bool make_map_mn(CUtensorMap *map, const void *base, int64_t cols, int64_t T, int64_t ld) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)wg::BT};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int wgrad_pair_capacity() {
    static int cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(k_gemm_bf16_wgrad_2sm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wg::SMEM) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(sm2::THREADS);
    cfg.dynamicSmemBytes = wg::SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_gemm_bf16_wgrad_2sm, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

// kind::f16 instruction descriptor: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 and 10-12 = 1), both MN-major (bits 15 and 16), N >> 3, M >> 4.
uint32_t make_idesc_bf16_mn(int mma_m, int mma_n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(mma_n >> 3) << 17) |
           ((uint32_t)(mma_m >> 4) << 24);
}

}  // namespace

using namespace fp8q_host;

extern "C" fp8_status fp8_gemm_bf16_wgrad(const void *dY_bf16, const void *X_bf16, int64_t T, int64_t M, int64_t N,
                                          int64_t ld_dy, int64_t ld_x, float *dW, int64_t ldd, int accumulate,
                                          void *stream) {
    if (T < 0 || M < 0 || N < 0 || ld_dy < M || ld_x < N || ldd < N) return FP8_ERR_SHAPE;
    if (T > (1 << 30) || M > (1 << 30) || N > (1 << 30)) return FP8_ERR_SHAPE;
    if (M % 8 || N % 8 || ld_dy % 8 || ld_x % 8 || ldd % 4) return FP8_ERR_ALIGNMENT;
    int sms;
    if (M == 0 || N == 0) return check_device(&sms);
    if (!dW) return FP8_ERR_INVALID_ARG;
    if (T > 0 && (!dY_bf16 || !X_bf16)) return FP8_ERR_INVALID_ARG;
    if (!aligned16(dW) || (dY_bf16 && !aligned16(dY_bf16)) || (X_bf16 && !aligned16(X_bf16))) return FP8_ERR_ALIGNMENT;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (T == 0) {
        if (accumulate) return FP8_OK;
        return cudaMemset2DAsync(dW, (size_t)ldd * 4, 0, (size_t)N * 4, (size_t)M, s) == cudaSuccess ? FP8_OK
                                                                                                   : FP8_ERR_CUDA;
    }
    CUtensorMap ta, tb;
    if (!make_map_mn(&ta, dY_bf16, M, T, ld_dy) || !make_map_mn(&tb, X_bf16, N, T, ld_x)) return FP8_ERR_CUDA;
    const int cap = wgrad_pair_capacity();
    if (cap <= 0) return FP8_ERR_CUDA;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, cap));
    return pdl_launch(k_gemm_bf16_wgrad_2sm, dim3(2 * pairs), dim3(sm2::THREADS), wg::SMEM, s, ta, tb, (int)M,
                      (int)N, (int)T, make_idesc_bf16_mn(256, 256), dW, ldd, accumulate) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_CUDA;
}

// This file's device error word (read and optionally cleared by
// fp8_device_error together with the other GEMM files').
fp8_status fp8q_wgrad_device_error(uint32_t *out, int clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
    *out = v;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z)) != cudaSuccess) return FP8_ERR_CUDA;
    }
    return FP8_OK;
}
