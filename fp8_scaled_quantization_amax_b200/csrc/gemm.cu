// gemm.cu -- FP8 scaled GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Sources: "H100 FP8加速实测：新一代计算架构的飞跃" (the multiply-accumulate runs
// directly on 8-bit floating-point operands on the tensor cores);
// "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
// "FP8 三种缩放配方怎么选" (tensorwise and rowwise scaled matmuls);
// "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-block scales),
// §2.1 (E5M2 gradients against E4M3 weights), §5.3 (FP8 GEMM results depend
// on the tiling; here every tile has one fixed K order, and a tile split
// along K sums its parts in one fixed order, so results are deterministic
// run to run).
//
//   D[m, n] = bf16( epilogue( sum_k A[m, k] * B[n, k] ) )
//   A [M, K], B [N, K]: FP8 codes, K contiguous; fp32 accumulation in TMEM.
//
// Design (one CTA per SM, persistent over 128x256 output tiles; for few
// tiles, a cluster of CTAs per tile splitting K, see k_gemm_fp8's SPLIT):
//   warp 0      TMA producer: 128x128 A and 256x128 B tiles (128-byte
//               swizzle) into a 4-stage shared-memory ring, one mbarrier per
//               stage carrying the transaction byte count.
//   warp 1      TMEM allocator and MMA issuer: per 128-wide K chunk, four
//               tcgen05.mma.kind::f8f6f4 of 128x256x32 from shared-memory
//               descriptors; tcgen05.commit frees the stage when the tensor
//               core has read it.
//   warps 2-9   epilogue: tcgen05.ld of the fp32 accumulator (warp w reads
//               TMEM lanes 32*(w%4)..+31 = tile rows, columns split in two
//               128-wide halves), scales applied in fp32, RNE to bf16, 16-byte
//               stores.
//   TENSOR/ROW: the accumulator is double-buffered in TMEM (2 x 256 columns),
//               so the epilogue of tile i overlaps the mainloop of tile i+1.
//   BLOCK:      per-block scales vary along K, so each 128-wide K chunk is
//               accumulated alone into one of two TMEM partial buffers
//               (ping-pong); the epilogue warps read it, multiply by
//               sa[kb, m] * sb[n/128, kb] and add it into an fp32 register
//               accumulator ("promotion"); the MMA of chunk c+1 runs while
//               chunk c is promoted.
// Every wait on an mbarrier is bounded (about one second); on expiry the
// kernel records a bit in the library's device error word, stops issuing,
// waits (bounded) for its own copies and MMAs in flight, frees TMEM and
// returns.  No trap, no unbounded spin.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "tc.cuh"

using namespace fp8q;
using fp8q_host::pdl_launch;
using fp8q_host::pdl_launch_cluster;

namespace {

constexpr int BN = 256;                 // tile columns (TMEM columns per accumulator)
constexpr int STAGES = 4;
constexpr int B_TILE = BN * BK;         // 32 KiB
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr int NUM_BARS = 2 * STAGES + 5;   // full, empty, acc_full[2], acc_empty[2], drain
// after the pipeline and the barriers: one store_rows_coalesced buffer per epilogue warp
constexpr size_t EPI_OFF = ((size_t)STAGES * STAGE_BYTES + NUM_BARS * 8 + 16 + 15) & ~(size_t)15;
constexpr size_t SMEM_BYTES = 1024 + EPI_OFF + (size_t)EPI_WARPS * kEpiBufBytes;
// Split-K staging (SPLIT kernels): a CTA's fp32 partial tile, row-major with
// a 260-float pitch (rows 16 B apart modulo the 32 banks, so the eight lanes
// of a 16-byte store phase hit distinct banks), over the pipeline stages.
constexpr int kStagePitch = BN + 4;
static_assert((size_t)BM * kStagePitch * 4 <= (size_t)STAGES * STAGE_BYTES, "split-K stage exceeds the pipeline");
constexpr int kMaxSplit = 8;   // K parts per tile (portable cluster size)

enum { kModeTensor = 0, kModeRow = 1, kModeBlock = 2 };

// SPLIT reduction: CTA q of the cluster owns float4 column groups
// [q*64/S, (q+1)*64/S) of the tile; it sums that slice of every CTA's staged
// partial in rank order (so the result does not depend on timing), applies
// the output scales and stores bf16.  Threads 0..255 of the epilogue.
template <int MODE>
__device__ __forceinline__ void split_reduce_store(const float *stage, int S, int q, int et, int m_blk, int n_blk,
                                                   int M, int N, const float *__restrict__ sa,
                                                   const float *__restrict__ sb, __nv_bfloat16 *__restrict__ D,
                                                   int64_t ldd) {
    const int rows = min(M - m_blk * BM, BM);
    const int g0 = q * (BN / 4) / S, g1 = (q + 1) * (BN / 4) / S, G = g1 - g0;
    const uint32_t base = smem_u32(stage);
    const float rs = (MODE == kModeTensor) ? __fmul_rn(sa[0], sb[0]) : 0.0f;
    for (int i = et; i < rows * G; i += EPI_WARPS * 32) {
        const int row = i / G, g = g0 + i % G;
        const int n = n_blk * BN + g * 4;
        if (n >= N) continue;   // N % 8 == 0: a group is wholly inside or outside
        const uint32_t off = base + (uint32_t)(row * kStagePitch + g * 4) * 4u;
        float4 p[kMaxSplit];
#pragma unroll
        for (int r = 0; r < kMaxSplit; ++r)
            if (r < S) p[r] = ld_dsmem_f4(mapa_shared(off, (uint32_t)r));
        float4 v = p[0];
#pragma unroll
        for (int r = 1; r < kMaxSplit; ++r) {
            if (r < S) {
                v.x = v.x + p[r].x;
                v.y = v.y + p[r].y;
                v.z = v.z + p[r].z;
                v.w = v.w + p[r].w;
            }
        }
        const int64_t m = (int64_t)m_blk * BM + row;
        if (MODE == kModeRow) {
            const float a = sa[m];
            v.x = v.x * (a * sb[n + 0]);
            v.y = v.y * (a * sb[n + 1]);
            v.z = v.z * (a * sb[n + 2]);
            v.w = v.w * (a * sb[n + 3]);
        } else if (MODE == kModeTensor) {
            v.x = v.x * rs;
            v.y = v.y * rs;
            v.z = v.z * rs;
            v.w = v.w * rs;
        }
        uint2 o;
        o.x = pack_bf16x2(v.x, v.y);
        o.y = pack_bf16x2(v.z, v.w);
        *reinterpret_cast<uint2 *>(D + m * ldd + n) = o;
    }
}

// ------------------------------------------------------------- kernel ----
// SPLIT: launched in clusters of S CTAs (S chosen at launch); the cluster
// computes one output tile, CTA q accumulating K blocks [q*nk/S, (q+1)*nk/S),
// and the K parts are summed through distributed shared memory
// (split_reduce_store).  Otherwise the grid is persistent over whole tiles.
template <int MODE, bool SPLIT>
__global__ void __launch_bounds__(THREADS, 1)
k_gemm_fp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
           int K, uint32_t idesc, const float *__restrict__ sa, const float *__restrict__ sb,
           __nv_bfloat16 *__restrict__ D, int64_t ldd) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)STAGES * STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nk = (K + BK - 1) / BK;
    const int S = SPLIT ? (int)cluster_size() : 1;
    const int q = SPLIT ? (int)cluster_rank() : 0;
    const int t_first = SPLIT ? (int)blockIdx.x / S : (int)blockIdx.x;
    const int t_step = SPLIT ? num_tiles : (int)gridDim.x;   // SPLIT: exactly one tile per CTA
    const int k0 = (int)((int64_t)q * nk / S), k1 = (int)((int64_t)(q + 1) * nk / S);
    float *stage = reinterpret_cast<float *>(smem);

    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STAGES + s]); };
    auto accf_bar = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
    auto acce_bar = [&](int b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
    const uint32_t drain_bar = smem_u32(&bars[2 * STAGES + 4]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();      // inputs of the previous kernel in the stream are visible from here on
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            int last_round[STAGES];
            for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
            uint32_t it = 0;
            bool ok = true;
            for (int tile = t_first; ok && tile < num_tiles; tile += t_step) {
                const int m_blk = tile % num_m, n_blk = tile / num_m;
                for (int kc = k0; kc < k1; ++kc, ++it) {
                    const int stage = it % STAGES;
                    const uint32_t round = it / STAGES;
                    if (!wait_bar(empty_bar(stage), (round & 1u) ^ 1u, abort_flag, kErrProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + (size_t)stage * STAGE_BYTES);
                    mbar_expect_tx(full_bar(stage), STAGE_BYTES);
                    tma_load_2d(a_dst, &tmA, full_bar(stage), kc * BK, m_blk * BM);
                    tma_load_2d(a_dst + A_TILE, &tmB, full_bar(stage), kc * BK, n_blk * BN);
                    last_round[stage] = (int)round;
                }
            }
            if (!ok || *abort_flag) {   // copies in flight must land before the CTA exits
                for (int s = 0; s < STAGES; ++s)
                    if (last_round[s] >= 0) wait_bar_drain(full_bar(s), (uint32_t)last_round[s] & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (lane == 0) {
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int tile = t_first; ok && tile < num_tiles; tile += t_step, ++lt) {
                uint32_t d_tmem = tmem;
                if (MODE != kModeBlock) {
                    const uint32_t ab = lt & 1u, use = lt >> 1;
                    if (!wait_bar(acce_bar(ab), (use & 1u) ^ 1u, abort_flag, kErrMma)) break;
                    tc_fence_after();
                    d_tmem = tmem + ab * BN;
                }
                for (int kc = k0; kc < k1; ++kc, ++it) {
                    const int stage = it % STAGES;
                    const uint32_t round = it / STAGES;
                    if (MODE == kModeBlock) {
                        const uint32_t pb = it & 1u, use = it >> 1;
                        if (!wait_bar(acce_bar(pb), (use & 1u) ^ 1u, abort_flag, kErrMma)) { ok = false; break; }
                        d_tmem = tmem + pb * BN;
                    }
                    if (!wait_bar(full_bar(stage), round & 1u, abort_flag, kErrMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)stage * STAGE_BYTES);
                    const uint64_t adesc = sdesc_k_sw128(a_addr);
                    const uint64_t bdesc = sdesc_k_sw128(a_addr + A_TILE);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        // +32 bytes along K inside the swizzled 128-byte row = +2 in the address field
                        const uint32_t acc = (MODE == kModeBlock) ? (k > 0) : (kc > k0 || k > 0);
                        tc_mma(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, acc);
                    }
                    tc_commit(empty_bar(stage));
                    if (MODE == kModeBlock) tc_commit(accf_bar(it & 1u));
                }
                if (ok && MODE != kModeBlock) tc_commit(accf_bar(lt & 1u));
            }
            // all MMAs issued by this thread complete before TMEM is freed
            tc_commit(drain_bar);
            wait_bar_drain(drain_bar, 0u);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- epilogue ----
        const int sp = warp & 3;                 // TMEM lane quarter this warp may access
        const int ch = (warp - 2) >> 2;          // column half of the tile
        const int row_in_tile = sp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(sp * 32) << 16;
        uint32_t it = 0, lt = 0;
        bool ok = true;
        for (int tile = t_first; ok && tile < num_tiles; tile += t_step, ++lt) {
            const int m_blk = tile % num_m, n_blk = tile / num_m;
            const int m = m_blk * BM + row_in_tile;
            // SPLIT: rows of this tile to stage (the rest lie beyond M)
            const bool stage_row = SPLIT && row_in_tile < M - m_blk * BM;
            const int n_base = n_blk * BN + ch * 128;
            if (MODE != kModeBlock) {
                const uint32_t ab = lt & 1u, use = lt >> 1;
                float rs;
                if (MODE == kModeRow) rs = (m < M) ? sa[m] : 0.0f;
                else rs = __fmul_rn(sa[0], sb[0]);
                // column scales (lane j: column n_base + 32c + j), fetched before the wait
                float cbs[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int col = n_base + c * 32 + lane;
                    cbs[c] = (MODE == kModeRow && col < N) ? sb[col] : 0.0f;
                }
                bool w = true;
                if (lane == 0) w = wait_bar(accf_bar(ab), use & 1u, abort_flag, kErrEpilogue);
                w = __shfl_sync(0xFFFFFFFFu, w, 0);
                if (!w) break;
                tc_fence_after();
                // two 32-column chunks per TMEM round trip; the accumulator buffer is
                // released once its last columns are in registers
                uint8_t *ebuf = smem + EPI_OFF + (size_t)(warp - 2) * kEpiBufBytes;
                const int64_t row0 = (int64_t)m_blk * BM + sp * 32;
#pragma unroll
                for (int c2 = 0; c2 < 4; c2 += 2) {
                    uint32_t r[64];
                    tmem_ld32_async(tmem + lane_base + ab * BN + ch * 128 + c2 * 32, r);
                    tmem_ld32_async(tmem + lane_base + ab * BN + ch * 128 + c2 * 32 + 32, r + 32);
                    tmem_wait64(r);
                    if (c2 == 2) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acce_bar(ab));
                    }
                    uint32_t pk[32];
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = c2 + cc;
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[cc * 32 + j]);
                        if constexpr (SPLIT) {   // raw K-part partial to the stage; scaled after the sum
                            if (stage_row) {
                                float4 *dst = reinterpret_cast<float4 *>(stage + row_in_tile * kStagePitch + ch * 128 + c * 32);
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                            }
                            continue;
                        }
                        if (MODE == kModeRow) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v[j] * (rs * __shfl_sync(0xFFFFFFFFu, cbs[c], j));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v[j] * rs;
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[cc * 16 + j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    }
                    if constexpr (!SPLIT) store_rows_coalesced(ebuf, pk, lane, D, ldd, row0, M, n_base + c2 * 32, N);
                }
            } else {
                float acc[128];
#pragma unroll
                for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
                const int nkb_b = nk;                     // K blocks per row of sb
                const int nb = n_base / 128;              // this half's 128-row block of B
                const bool nb_ok = n_base < N;
                float a_next = (m < M) ? sa[(int64_t)k0 * M + m] : 0.0f;
                float b_next = nb_ok ? sb[(int64_t)nb * nkb_b + k0] : 0.0f;
                for (int kc = k0; kc < k1; ++kc, ++it) {
                    const uint32_t pb = it & 1u, use = it >> 1;
                    const float sc = __fmul_rn(a_next, b_next);
                    bool w = true;
                    if (lane == 0) w = wait_bar(accf_bar(pb), use & 1u, abort_flag, kErrEpilogue);
                    w = __shfl_sync(0xFFFFFFFFu, w, 0);
                    if (!w) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float v[32];
                        tmem_ld32(tmem + lane_base + pb * BN + ch * 128 + c * 32, v);
                        if (c == 3) {   // the partial buffer is free once the last slice is in registers
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(acce_bar(pb));
                            if (kc + 1 < k1) {   // next block's scales, after the release (see the pair kernel)
                                a_next = (m < M) ? sa[(int64_t)(kc + 1) * M + m] : 0.0f;
                                b_next = nb_ok ? sb[(int64_t)nb * nkb_b + kc + 1] : 0.0f;
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) acc[c * 32 + j] = fmaf(v[j], sc, acc[c * 32 + j]);
                    }
                }
                if (!ok) break;
                if constexpr (SPLIT) {   // this K part's promoted sum to the stage
                    if (stage_row) {
                        float4 *dst = reinterpret_cast<float4 *>(stage + row_in_tile * kStagePitch + ch * 128);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
                    }
                    continue;
                }
                uint8_t *ebuf = smem + EPI_OFF + (size_t)(warp - 2) * kEpiBufBytes;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(acc[h2 * 64 + 2 * j], acc[h2 * 64 + 2 * j + 1]);
                    store_rows_coalesced(ebuf, pk, lane, D, ldd, (int64_t)m_blk * BM + sp * 32, M, n_base + h2 * 64, N);
                }
            }
        }
    }

    if constexpr (SPLIT) {
        // Every thread of the cluster takes both barriers, on the error paths
        // too (a CTA's waits are all bounded, so each one gets here).
        __syncwarp();
        cluster_sync_all();   // every CTA has staged its K part
        if (warp >= 2)
            split_reduce_store<MODE>(stage, S, q, (int)threadIdx.x - 64, t_first % num_m, t_first / num_m, M, N, sa,
                                     sb, D, ldd);
        __syncwarp();         // the barrier below is warp-aligned
        cluster_sync_all();   // no CTA leaves while a peer may still read its stage
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------ 2-SM variant ----
// A CTA pair (cluster of 2) computes a 256 x BN tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA TMA-loads its own 128 rows of
// A and its own BN/2 rows of B (no multicast), the even CTA ("leader")
// issues the MMAs, which read both CTAs' shared memory and write each CTA's
// 128 accumulator rows into its own TMEM.  Per CTA and K chunk this moves
// 16 KiB + BN/2 x 128 B instead of 16 KiB + 32 KiB, so 6 (BN = 256) or 8
// (BN = 128) stages fit in shared memory and hide more TMA latency.
//   * The leader's full barrier counts both CTAs' bytes (the peer's TMA
//     signals it through its cluster address);
//   * tcgen05.commit multicasts to the same barrier in both CTAs (stage
//     free, accumulator / partial ready);
//   * both CTAs' epilogue warps release a TMEM buffer by arriving on the
//     leader's barrier (count 2 x 8 warps).
// Tensor and row scales only: the block-scaled GEMM on CTA pairs is the
// kernel in gemm_block.cu.
template <int MODE, int BN, bool GROUPED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(sm2::THREADS, 1)
k_gemm_fp8_2sm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
               int K, uint32_t idesc, const float *__restrict__ sa, const float *__restrict__ sb,
               __nv_bfloat16 *__restrict__ D, int64_t ldd, int full_tiles, int split_units,
               float *__restrict__ ws, uint32_t *__restrict__ flags, uint32_t epoch,
               const int64_t *__restrict__ goff, int G) {
    using C = sm2::Cfg<BN>;
    constexpr int STG = C::STAGES, NBUF = C::NBUF;
    constexpr int HALF = BN / 2;             // columns per epilogue warp
    static_assert(BN == 256, "the pair kernel runs 256 x 256 tiles");
    static_assert(MODE != kModeBlock, "block scales on CTA pairs: gemm_block.cu");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)STG * C::STAGE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBARS);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = (rank == 0);
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (M + 255) / 256;
    const int nk = (K + BK - 1) / BK;
    // Work items of this pair: whole tiles pair, pair + npairs, ... below
    // full_tiles, then (pair < split_units) one half of a split tail tile:
    // tile full_tiles + pair / 2, K blocks [0, nk/2) for the even pair and
    // [nk/2, nk) for the odd one.  With no split, full_tiles = every tile.
    // Grouped GEMM (MoE experts): group e owns rows [goff[e], goff[e+1]) of A
    // and D and rows [e*N, (e+1)*N) of B; its tiles follow group e-1's, m
    // fastest.  The tile count comes from one scan of the offsets.
    const int num_n = (N + BN - 1) / BN;
    int total_tiles = full_tiles;
    if constexpr (GROUPED) {
        pdl_wait();   // the group offsets may come from the previous kernel
        total_tiles = 0;
        for (int e = 0; e < G; ++e) total_tiles += (int)((goff[e + 1] - goff[e] + 255) / 256) * num_n;
    }
    const int n_full = (pair < total_tiles) ? (total_tiles - 1 - pair) / npairs + 1 : 0;
    const int n_items = n_full + (pair < split_units ? 1 : 0);
    struct Item {
        int tile, k0, k1, half, m_blk, n_blk, e;
        int64_t row0, row_end;   // rows of A / D this item's tile may write
    };
    auto item = [&](int i) -> Item {
        if constexpr (GROUPED) {
            int t = pair + i * npairs, e = 0;
            int64_t r0 = goff[0], r1 = goff[1];
            int mt = (int)((r1 - r0 + 255) / 256);
            while (t >= mt * num_n) {   // empty groups own no tiles and are skipped
                t -= mt * num_n;
                ++e;
                r0 = r1;
                r1 = goff[e + 1];
                mt = (int)((r1 - r0 + 255) / 256);
            }
            return Item{pair + i * npairs, 0, nk, -1, t % mt, t / mt, e, r0, r1};
        } else {
            // the first K half of a split tile runs before this pair's whole
            // tiles and the second half after them, so the second half finds
            // the first one's partial already published
            const int h = pair & 1, kh = nk / 2, ts = full_tiles + pair / 2;
            const bool first_half_first = pair < split_units && h == 0;
            const int j = first_half_first ? i - 1 : i;
            if (j >= 0 && j < n_full) {
                const int t = pair + j * npairs;
                return Item{t, 0, nk, -1, t % num_m, t / num_m, 0, 0, (int64_t)M};
            }
            return Item{ts, h ? kh : 0, h ? nk : kh, h, ts % num_m, ts / num_m, 0, 0, (int64_t)M};
        }
    };

    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STG + s]); };
    auto accf_bar = [&](int b) { return smem_u32(&bars[2 * STG + b]); };
    auto acce_bar = [&](int b) { return smem_u32(&bars[2 * STG + NBUF + b]); };
    const uint32_t drain_bar = smem_u32(&bars[2 * STG + 2 * NBUF]);
    const uint32_t part_bar = smem_u32(&bars[2 * STG + 2 * NBUF + 1]);

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
        mbar_init(part_bar, sm2::EPI);
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
                const Item w = item(i);
                const int a_row = (int)(w.row0 + w.m_blk * 256 + (int)rank * 128);
                const int b_row = w.e * N + w.n_blk * BN + (int)rank * HALF;
                for (int kc = w.k0; kc < w.k1; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(empty_bar(stage), (round & 1u) ^ 1u, abort_flag, kErrProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(full_bar(stage), 0);
                    if (leader) mbar_expect_tx(full_bar(stage), 2 * C::STAGE);
                    const uint32_t a_dst = smem_u32(smem + (size_t)stage * C::STAGE);
                    tma_load_2d_pair(a_dst, &tmA, full_leader, kc * BK, a_row);
                    tma_load_2d_pair(a_dst + A_TILE, &tmB, full_leader, kc * BK, b_row);
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
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_items; ++i, ++lt) {
                const Item w = item(i);
                const uint32_t ab = lt % NBUF, use = lt / NBUF;
                if (!wait_bar(acce_bar(ab), (use & 1u) ^ 1u, abort_flag, kErrMma)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * BN;
                for (int kc = w.k0; kc < w.k1; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(full_bar(stage), round & 1u, abort_flag, kErrMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)stage * C::STAGE);
                    const uint64_t adesc = sdesc_k_sw128(a_addr);
                    const uint64_t bdesc = sdesc_k_sw128(a_addr + A_TILE);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        tc_mma_pair(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kc > w.k0 || k > 0) ? 1u : 0u);
                    tc_commit_pair_both(empty_bar(stage));
                }
                if (ok) tc_commit_pair_both(accf_bar(lt % NBUF));
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
        uint32_t lt = 0;
        bool ok = true;
        for (int i = 0; ok && i < n_items; ++i, ++lt) {
            const Item wi = item(i);
            const int n_blk = wi.n_blk;
            const int64_t m = wi.row0 + wi.m_blk * 256 + (int)rank * 128 + sp * 32 + lane;
            const bool m_ok = m < wi.row_end;
            const int n_base = n_blk * BN + ch * HALF;
            const float *sbe = sb + (int64_t)wi.e * N;   // group e's column scales (ROW)
            {
                const uint32_t ab = lt % NBUF, use = lt / NBUF;
                float rs;
                if (MODE == kModeRow) rs = m_ok ? sa[m] : 0.0f;
                else rs = __fmul_rn(sa[wi.e], sb[wi.e]);
                // this warp's column scales (lane j holds column n_base + 32c + j),
                // fetched while the accumulator is still being computed
                float cbs[HALF / 32];
#pragma unroll
                for (int c = 0; c < HALF / 32; ++c) {
                    const int col = n_base + c * 32 + lane;
                    cbs[c] = (MODE == kModeRow && col < N) ? sbe[col] : 0.0f;
                }
                bool w = true;
                if (lane == 0) w = wait_bar(accf_bar(ab), use & 1u, abort_flag, kErrEpilogue);
                w = __shfl_sync(0xFFFFFFFFu, w, 0);
                if (!w) break;
                tc_fence_after();
                // split tail tile: this CTA's 128 x 256 partial in the workspace
                float *part = nullptr;
                uint32_t *flag = nullptr;
                if (wi.half >= 0) {
                    const int slot = wi.tile - full_tiles;
                    part = ws + ((size_t)slot * 2 + rank) * sm2::kSplitPartialFloats + (sp * 32 + lane);
                    flag = flags + slot * 2 + rank;
                    if (wi.half == 1) {   // wait for the first half's partial
                        bool f = true;
                        if (lane == 0) f = wait_flag(flag, epoch, abort_flag);
                        f = __shfl_sync(0xFFFFFFFFu, f, 0);
                        if (!f) break;
                        (void)ld_acquire_u32(flag);   // acquire on every lane
                    }
                }
                // two 32-column chunks per TMEM round trip (unrolled: the scale
                // array is indexed with constants only); the accumulator buffer is
                // released as soon as its last columns are in registers
                uint8_t *ebuf = smem + C::EPI_OFF + (size_t)(warp - 4) * kEpiBufBytes;
                const int64_t row0 = wi.row0 + wi.m_blk * 256 + (int)rank * 128 + sp * 32;
#pragma unroll
                for (int c2 = 0; c2 < HALF / 32; c2 += 2) {
                    uint32_t r[64];
                    tmem_ld32_async(tmem + lane_base + ab * BN + ch * HALF + c2 * 32, r);
                    tmem_ld32_async(tmem + lane_base + ab * BN + ch * HALF + c2 * 32 + 32, r + 32);
                    tmem_wait64(r);
                    if (c2 + 2 == HALF / 32) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar(ab), 0));
                    }
                    uint32_t pk[32];
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = c2 + cc;
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[cc * 32 + j]);
                        if (wi.half == 0) {   // first half: store the raw fp32 partial, no output
                            float *pc = part + (size_t)(ch * HALF + c * 32) * 128;
#pragma unroll
                            for (int j = 0; j < 32; ++j) pc[(size_t)j * 128] = v[j];
                            continue;
                        }
                        if (wi.half == 1) {   // second half: add the first half's partial (fixed order)
                            const float *pc = part + (size_t)(ch * HALF + c * 32) * 128;
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v[j] + pc[(size_t)j * 128];
                        }
                        if (MODE == kModeRow) {
                            const float cb = cbs[c];
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v[j] * (rs * __shfl_sync(0xFFFFFFFFu, cb, j));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = v[j] * rs;
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[cc * 16 + j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    }
                    if (wi.half != 0)
                        store_rows_coalesced(ebuf, pk, lane, D, ldd, row0, wi.row_end, n_base + c2 * 32, N);
                }
                if (wi.half == 0) {   // publish: every epilogue warp's stores, then the flag
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(part_bar);
                    if (warp == 4 && lane == 0) {
                        if (wait_bar(part_bar, 0u, abort_flag, kErrSplit)) st_release_u32(flag, epoch);
                    }
                } else if (wi.half == 1) {
                    // consumed: once every epilogue warp has seen the flag and read its
                    // share, clear it, so the workspace leaves this launch as it came
                    // (a replayed CUDA graph reuses the epoch it was captured with)
                    __syncwarp();
                    if (lane == 0) mbar_arrive(part_bar);
                    if (warp == 4 && lane == 0) {
                        if (wait_bar(part_bar, 0u, abort_flag, kErrSplit)) st_release_u32(flag, 0u);
                    }
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

// Per device: the 1-SM kernels' shared-memory opt-in done, and how many
// split-K clusters of each size fit at once (0 = not asked yet, -1 = none).
template <int MODE>
struct OneSmState {
    std::mutex mu;
    bool attr_done[64] = {};
    int cap[64][kMaxSplit + 1] = {};
};
template <int MODE>
OneSmState<MODE> &one_sm_state() {
    static OneSmState<MODE> st;
    return st;
}

template <int MODE>
cudaError_t one_sm_prepare(int dev) {
    OneSmState<MODE> &g = one_sm_state<MODE>();
    std::lock_guard<std::mutex> lk(g.mu);
    if (g.attr_done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_fp8<MODE, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_gemm_fp8<MODE, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e == cudaSuccess) g.attr_done[dev] = true;
    return e;
}

template <int MODE>
int split_cluster_capacity(int dev, int S) {
    OneSmState<MODE> &g = one_sm_state<MODE>();
    std::lock_guard<std::mutex> lk(g.mu);
    if (g.cap[dev][S] != 0) return g.cap[dev][S];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S * 16);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = S;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_gemm_fp8<MODE, true>, &cfg) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        n = -1;
    }
    g.cap[dev][S] = n;
    return n;
}

// K parts per tile for the 1-SM kernel.  A problem of fewer tiles than half
// the SMs leaves most tensor cores idle, so each tile is shared by a cluster
// of S CTAs: the largest S (at most 8, with at least two K blocks per part)
// for which every cluster is resident at once.  1 = no split.
template <int MODE>
int one_sm_split(int dev, int sms, int tiles, int nk) {
    if (tiles * 2 > sms) return 1;
    for (int S = std::min(kMaxSplit, nk / 2); S >= 2; --S)
        if (tiles * S <= sms && split_cluster_capacity<MODE>(dev, S) >= tiles) return S;
    return 1;
}

// Problems of any M whose 128 x 256 tiles fill at most a quarter of the SMs,
// with at least 8 K blocks, run on the 1-SM kernel with each tile shared by a
// cluster of S CTAs: one_sm_split takes the largest S from min(8, nk / 2)
// down to 2 whose clusters are all resident at once (for M <= 128 the split
// also applies up to half the SMs).  Measured (L2 flushed)
// against the pair kernel: 256 x 4096 x 4096 19.5 us (pair 22.5),
// 256 x 4096 x 16384 29.7 us (pair with its workspace split 41.0).
inline bool one_sm_cluster_split(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    return tiles * 4 <= sms && (K + BK - 1) / BK >= 8;
}

template <int MODE>
cudaError_t launch_gemm(cudaStream_t st, int sms, const CUtensorMap &ta, const CUtensorMap &tb, int M, int N, int K,
                        uint32_t idesc, const float *sa, const float *sb, void *D, int64_t ldd) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if ((e = one_sm_prepare<MODE>(dev)) != cudaSuccess) return e;
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int S = one_sm_split<MODE>(dev, sms, tiles, (K + BK - 1) / BK);
    if (S > 1)
        return pdl_launch_cluster(k_gemm_fp8<MODE, true>, dim3(tiles * S), dim3(THREADS), SMEM_BYTES, st, (unsigned)S,
                                  ta, tb, M, N, K, idesc, sa, sb, static_cast<__nv_bfloat16 *>(D), ldd);
    const int grid = std::max(1, std::min(tiles, sms));
    return pdl_launch(k_gemm_fp8<MODE, false>, dim3(grid), dim3(THREADS), SMEM_BYTES, st, ta, tb, M, N, K, idesc, sa,
                      sb, static_cast<__nv_bfloat16 *>(D), ldd);
}

// Pairs of the 2-SM kernel that fit on the device at once (cached per device).
template <int MODE, int BN, bool GROUPED = false>
int pair_capacity() {
    static int cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(k_gemm_fp8_2sm<MODE, BN, GROUPED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sm2::Cfg<BN>::SMEM) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(sm2::THREADS);
    cfg.dynamicSmemBytes = sm2::Cfg<BN>::SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_gemm_fp8_2sm<MODE, BN, GROUPED>, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

// Split-K plan for a grid of `cap` CTA pairs.  The r tiles of the last wave
// (all tiles, when they fit in half the pairs) are computed as two K halves
// on two pairs, the first half handing its fp32 partial to the second
// through the workspace.  With several waves the first halves run first and
// the second halves last, so no pair waits for a partial; measured on
// 4096 x 4096 tiles (L2 flushed, us): K = 8192 103.2 unsplit, 97.2 split;
// K = 4096 59.4 either way (the half-empty last wave already runs faster
// than a full one; with the halves run side by side it was 63.5).
// The fp32 hand-off through global memory costs several microseconds, so a
// pair split pays only for long K: measured on 16 tiles of 256 x 256, K =
// 4096 (32 K blocks) ran 22.5 us unsplit and 24.6 split, K = 16384 53.2 and
// 41.0.  Shorter-K problems with few tiles take the cluster split of the
// 1-SM kernel instead (one_sm_cluster_split below) or run unsplit.
constexpr int kPairSplitMinKBlocks = 64;
struct SplitPlan { int full_tiles, units; size_t bytes; };
SplitPlan split_plan(int64_t M, int64_t N, int64_t K, int cap) {
    const int tiles = (int)(((M + 255) / 256) * ((N + 255) / 256));
    const int nk = (int)((K + BK - 1) / BK);
    const int r = cap > 0 ? tiles % cap : 0;
    // r tiles in the last wave, split in K halves over 2r <= cap pairs; with
    // several waves the first halves run before each pair's whole tiles and
    // the second halves after them
    if (cap <= 0 || r == 0 || 2 * r > cap || nk < kPairSplitMinKBlocks) return SplitPlan{tiles, 0, 0};
    const size_t flags_off = (size_t)r * 2 * sm2::kSplitPartialFloats * sizeof(float);
    return SplitPlan{tiles - r, 2 * r, flags_off + (((size_t)r * 2 * sizeof(uint32_t) + 255) & ~(size_t)255)};
}

template <int MODE, int BN>
cudaError_t launch_gemm_2sm(cudaStream_t st, const CUtensorMap &ta, const CUtensorMap &tb, int M, int N, int K,
                            uint32_t idesc, const float *sa, const float *sb, void *D, int64_t ldd, int pairs_cap,
                            const SplitPlan &plan, void *ws, uint32_t epoch) {
    const int tiles = ((M + 255) / 256) * ((N + BN - 1) / BN);
    // with a split, full_tiles is a whole number of waves of pairs_cap pairs
    // (or zero, when the split halves are all the work)
    const int pairs = plan.units ? (plan.full_tiles > 0 ? pairs_cap : plan.units) : std::max(1, std::min(tiles, pairs_cap));
    float *part = static_cast<float *>(ws);
    uint32_t *flags = plan.units ? reinterpret_cast<uint32_t *>(static_cast<char *>(ws) +
                                                                (size_t)(plan.units / 2) * 2 * sm2::kSplitPartialFloats * sizeof(float))
                                 : nullptr;
    return pdl_launch(k_gemm_fp8_2sm<MODE, BN, false>, dim3(2 * pairs), dim3(sm2::THREADS), sm2::Cfg<BN>::SMEM, st,
                      ta, tb, M, N, K, idesc, sa, sb, static_cast<__nv_bfloat16 *>(D), ldd,
                      plan.units ? plan.full_tiles : tiles, plan.units, part, flags, epoch,
                      static_cast<const int64_t *>(nullptr), 0);
}

// Grouped launch: a persistent grid of every pair that fits; each pair
// derives its tiles from the group offsets on the device.
template <int MODE>
cudaError_t launch_gemm_grouped(cudaStream_t st, const CUtensorMap &ta, const CUtensorMap &tb, int64_t total_M,
                                int N, int K, uint32_t idesc, const float *sa, const float *sb, void *D, int64_t ldd,
                                const int64_t *goff, int G, int pairs_cap) {
    return pdl_launch(k_gemm_fp8_2sm<MODE, 256, true>, dim3(2 * pairs_cap), dim3(sm2::THREADS), sm2::Cfg<256>::SMEM,
                      st, ta, tb, (int)total_M, N, K, idesc, sa, sb, static_cast<__nv_bfloat16 *>(D), ldd, 0, 0,
                      static_cast<float *>(nullptr), static_cast<uint32_t *>(nullptr), 0u, goff, G);
}

uint32_t make_idesc(fp8_format fa, fp8_format fb, int mma_m, int mma_n) {
    // fp32 accumulator, A/B formats, K-major A and B, N >> 3, M >> 4
    return (1u << 4) | ((uint32_t)fa << 7) | ((uint32_t)fb << 10) | ((uint32_t)(mma_n >> 3) << 17) |
           ((uint32_t)(mma_m >> 4) << 24);
}

}  // namespace

using namespace fp8q_host;

// The block-scaled GEMM on CTA pairs lives in gemm_block.cu.
fp8_status fp8q_gemm_block_pair(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int64_t M,
                                int64_t N, int64_t K, const float *sa, const float *sb, void *D_bf16, int64_t ldd,
                                fp8_format qfmt, uint8_t *qo, float *qsinv, uint32_t *counts, cudaStream_t s);

namespace {
std::atomic<uint32_t> g_split_epoch[64];   // per device; a split launch publishes with a fresh value
}

extern "C" fp8_status fp8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp8_scale_mode mode, size_t *bytes) {
    if (!bytes) return FP8_ERR_INVALID_ARG;
    if (mode != FP8_SCALE_TENSOR && mode != FP8_SCALE_ROW && mode != FP8_SCALE_BLOCK) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8_ERR_SHAPE;
    *bytes = 0;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (mode == FP8_SCALE_BLOCK || M <= BM || N == 0 || K == 0 || one_sm_cluster_split(M, N, K, sms)) return FP8_OK;
    const int cap = (mode == FP8_SCALE_TENSOR) ? pair_capacity<kModeTensor, 256>() : pair_capacity<kModeRow, 256>();
    if (cap <= 0) return FP8_ERR_CUDA;
    *bytes = split_plan(M, N, K, cap).bytes;
    return FP8_OK;
}

extern "C" fp8_status fp8_gemm_scaled(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int64_t M,
                                      int64_t N, int64_t K, fp8_scale_mode mode, const float *a_scale_inv,
                                      const float *b_scale_inv, void *D_bf16, int64_t ldd, void *workspace,
                                      size_t workspace_bytes, void *stream) {
    if ((fa != FP8_E4M3 && fa != FP8_E5M2) || (fb != FP8_E4M3 && fb != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
    if (mode != FP8_SCALE_TENSOR && mode != FP8_SCALE_ROW && mode != FP8_SCALE_BLOCK) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || ldd < N) return FP8_ERR_SHAPE;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP8_ERR_SHAPE;
    if (K % 16) return FP8_ERR_SHAPE;
    if (N % 8 || ldd % 8) return FP8_ERR_ALIGNMENT;
    if (M == 0 || N == 0) {
        int sms;
        return check_device(&sms);
    }
    if (!D_bf16) return FP8_ERR_INVALID_ARG;
    if (K > 0 && (!A || !B || !a_scale_inv || !b_scale_inv)) return FP8_ERR_INVALID_ARG;
    if (!aligned16(D_bf16) || (A && !aligned16(A)) || (B && !aligned16(B))) return FP8_ERR_ALIGNMENT;
    if (workspace && !aligned16(workspace)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (K == 0) {
        return cudaMemset2DAsync(D_bf16, (size_t)ldd * 2, 0, (size_t)N * 2, (size_t)M, s) == cudaSuccess ? FP8_OK
                                                                                                       : FP8_ERR_CUDA;
    }
    // M > 128: a CTA pair per 256-row tile (2-SM MMA), unless the problem has
    // so few tiles that the cluster split-K of the 1-SM kernel applies;
    // otherwise one CTA per 128-row tile.
    if (M > BM && !one_sm_cluster_split(M, N, K, sms)) {
        if (mode == FP8_SCALE_BLOCK)
            return fp8q_gemm_block_pair(A, fa, B, fb, M, N, K, a_scale_inv, b_scale_inv, D_bf16, ldd, FP8_E4M3,
                                        nullptr, nullptr, nullptr, s);
        CUtensorMap ta, tb;
        if (!make_map(&ta, A, K, M, 128) || !make_map(&tb, B, K, N, 128)) return FP8_ERR_CUDA;
        const uint32_t idesc = make_idesc(fa, fb, 256, 256);
        cudaError_t e = cudaErrorUnknown;
        int cap;
        const int dev_cap = (mode == FP8_SCALE_TENSOR) ? pair_capacity<kModeTensor, 256>() : pair_capacity<kModeRow, 256>();
        if (dev_cap <= 0) return FP8_ERR_CUDA;
        SplitPlan plan{(int)(((M + 255) / 256) * ((N + 255) / 256)), 0, 0};
        uint32_t epoch = 0;
        if (workspace) {
            const SplitPlan sp = split_plan(M, N, K, dev_cap);
            if (sp.units > 0 && workspace_bytes >= sp.bytes) {
                int dev = 0;
                if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
                plan = sp;
                epoch = ++g_split_epoch[dev];
                if (epoch == 0) epoch = ++g_split_epoch[dev];   // 0 is what a fresh workspace holds
            }
        }
        if (mode == FP8_SCALE_TENSOR) {
            if ((cap = pair_capacity<kModeTensor, 256>()) > 0)
                e = launch_gemm_2sm<kModeTensor, 256>(s, ta, tb, (int)M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd, cap, plan, workspace, epoch);
        } else {
            if ((cap = pair_capacity<kModeRow, 256>()) > 0)
                e = launch_gemm_2sm<kModeRow, 256>(s, ta, tb, (int)M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd, cap, plan, workspace, epoch);
        }
        return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
    }
    CUtensorMap ta, tb;
    if (!make_map(&ta, A, K, M, BM) || !make_map(&tb, B, K, N, BN)) return FP8_ERR_CUDA;
    const uint32_t idesc = make_idesc(fa, fb, BM, BN);
    cudaError_t e;
    if (mode == FP8_SCALE_TENSOR)
        e = launch_gemm<kModeTensor>(s, sms, ta, tb, (int)M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd);
    else if (mode == FP8_SCALE_ROW)
        e = launch_gemm<kModeRow>(s, sms, ta, tb, (int)M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd);
    else
        e = launch_gemm<kModeBlock>(s, sms, ta, tb, (int)M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd);
    return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// Block-scaled GEMM whose output is requantized with 1 x 128 blocks for the
// next GEMM (the MLP chain: H = up(X) in bf16, requantized for the down
// projection).  With M > 128 and K > 0 one launch: the pair kernel's epilogue
// rounds each output to bf16 and quantizes its 128-column blocks in
// registers.  Otherwise the GEMM into D_bf16, then fp8_quantize_blockwise on
// it.  Either way the codes and scales equal fp8_quantize_blockwise(D).
extern "C" fp8_status fp8_gemm_block_requant(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                             int64_t M, int64_t N, int64_t K, const float *a_scale_inv,
                                             const float *b_scale_inv, void *D_bf16, int64_t ldd, fp8_format fo,
                                             uint8_t *q, float *q_scale_inv, uint32_t *counts, void *stream) {
    if ((fa != FP8_E4M3 && fa != FP8_E5M2) || (fb != FP8_E4M3 && fb != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
    if (fo != FP8_E4M3 && fo != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8_ERR_SHAPE;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP8_ERR_SHAPE;
    if (K % 16 || N % 16) return FP8_ERR_SHAPE;
    if (D_bf16 && ldd < N) return FP8_ERR_SHAPE;
    if (D_bf16 && (ldd % 8 || !aligned16(D_bf16))) return FP8_ERR_ALIGNMENT;
    const bool fused = M > BM && K > 0;
    if (M > 0 && N > 0) {
        if (!q || !q_scale_inv || (!fused && !D_bf16)) return FP8_ERR_INVALID_ARG;
        if (K > 0 && (!A || !B || !a_scale_inv || !b_scale_inv)) return FP8_ERR_INVALID_ARG;
    }
    if ((q && !aligned16(q)) || (A && !aligned16(A)) || (B && !aligned16(B))) return FP8_ERR_ALIGNMENT;
    if (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (M == 0 || N == 0) return FP8_OK;
    if (fused)
        return fp8q_gemm_block_pair(A, fa, B, fb, M, N, K, a_scale_inv, b_scale_inv, D_bf16, ldd, fo, q,
                                    q_scale_inv, counts, as_stream(stream));
    st = fp8_gemm_scaled(A, fa, B, fb, M, N, K, FP8_SCALE_BLOCK, a_scale_inv, b_scale_inv, D_bf16, ldd, nullptr, 0,
                         stream);
    if (st != FP8_OK) return st;
    return fp8_quantize_blockwise(D_bf16, M, N, ldd, fo, 1, q, q_scale_inv, counts, stream);
}

// The E8M0, the block-scaled pair and the bf16 weight-gradient GEMMs keep
// their own error words (gemm_mx.cu, gemm_block.cu, gemm_bf16.cu).
fp8_status fp8q_mx_device_error(uint32_t *out, int clear);
fp8_status fp8q_wgrad_device_error(uint32_t *out, int clear);
fp8_status fp8q_block_device_error(uint32_t *out, int clear);

extern "C" fp8_status fp8_device_error(uint32_t *host_out, int clear) {
    if (!host_out) return FP8_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return FP8_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
    uint32_t w = 0, g = 0;
    fp8_status st = fp8q_mx_device_error(&w, clear);
    if (st != FP8_OK) return st;
    st = fp8q_wgrad_device_error(&g, clear);
    if (st != FP8_OK) return st;
    uint32_t b = 0;
    st = fp8q_block_device_error(&b, clear);
    if (st != FP8_OK) return st;
    *host_out = v | w | g | b;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z)) != cudaSuccess) return FP8_ERR_CUDA;
    }
    return FP8_OK;
}

// ------------------------------------------------------------- grouped GEMM --
extern "C" fp8_status fp8_gemm_grouped(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int G,
                                       const int64_t *group_offsets, int64_t total_M, int64_t N, int64_t K,
                                       fp8_scale_mode mode, const float *a_scale_inv, const float *b_scale_inv,
                                       void *D_bf16, int64_t ldd, void *stream) {
    if ((fa != FP8_E4M3 && fa != FP8_E5M2) || (fb != FP8_E4M3 && fb != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
    if (mode != FP8_SCALE_TENSOR && mode != FP8_SCALE_ROW) return FP8_ERR_INVALID_ARG;
    if (G < 0 || total_M < 0 || N < 0 || K < 0 || ldd < N) return FP8_ERR_SHAPE;
    if (total_M >= (1 << 30) || (int64_t)G * N >= (1 << 30) || K > (1 << 30)) return FP8_ERR_SHAPE;
    if (K % 16) return FP8_ERR_SHAPE;
    if (N % 8 || ldd % 8) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (G == 0 || total_M == 0 || N == 0) return FP8_OK;
    if (!group_offsets || !D_bf16) return FP8_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(group_offsets) & 7u) return FP8_ERR_ALIGNMENT;
    cudaStream_t s = as_stream(stream);
    if (K == 0)
        return cudaMemset2DAsync(D_bf16, (size_t)ldd * 2, 0, (size_t)N * 2, (size_t)total_M, s) == cudaSuccess
                   ? FP8_OK : FP8_ERR_CUDA;
    if (!A || !B || !a_scale_inv || !b_scale_inv) return FP8_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D_bf16)) return FP8_ERR_ALIGNMENT;
    CUtensorMap ta, tb;
    if (!make_map(&ta, A, K, total_M, 128) || !make_map(&tb, B, K, (int64_t)G * N, 128)) return FP8_ERR_CUDA;
    const uint32_t idesc = make_idesc(fa, fb, 256, 256);
    cudaError_t e = cudaErrorUnknown;
    int cap;
    if (mode == FP8_SCALE_TENSOR) {
        if ((cap = pair_capacity<kModeTensor, 256, true>()) > 0)
            e = launch_gemm_grouped<kModeTensor>(s, ta, tb, total_M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd, group_offsets, G, cap);
    } else {
        if ((cap = pair_capacity<kModeRow, 256, true>()) > 0)
            e = launch_gemm_grouped<kModeRow>(s, ta, tb, total_M, (int)N, (int)K, idesc, a_scale_inv, b_scale_inv, D_bf16, ldd, group_offsets, G, cap);
    }
    return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// ---------------------------------------------- entry point without allocation --
// Some callers cannot allocate device memory at the point where they run the
// GEMM: code inside a framework that owns every device byte through its own
// caching allocator, or latency-critical paths where cudaMalloc's implicit
// device synchronisation is not acceptable.  fp8_gemm_scaled_noalloc gives
// them the split-K schedule without a caller workspace: the scratch lives in
// this file-scope array, which every GPU that loads the library holds until
// the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)10 << 20;   // 10 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64];   // device address of g_noalloc_scratch, per device
}

// One-time set-up per device (with that device current): look up the
// array's device address.  The array needs no clearing: a __device__ array
// without an initializer is zero when the module loads, and the split-K
// schedule leaves its hand-off flags at zero after every call.
static fp8_status noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return FP8_ERR_CUDA;
    if (dev >= 64) return FP8_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress((void **)&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return FP8_ERR_CUDA;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return FP8_OK;
}

extern "C" fp8_status fp8_gemm_scaled_noalloc(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                              int64_t M, int64_t N, int64_t K, fp8_scale_mode mode,
                                              const float *a_scale_inv, const float *b_scale_inv, void *D_bf16,
                                              int64_t ldd, void *stream) {
    size_t need = 0;
    fp8_status st = fp8_gemm_workspace_size(M, N, K, mode, &need);
    if (st != FP8_OK) return st;
    if (need > kNoAllocScratchBytes) return FP8_ERR_SHAPE;   // the split needs more than the built-in scratch
    void *scratch = nullptr;
    if (need > 0) {
        st = noalloc_scratch(&scratch);
        if (st != FP8_OK) return st;
    }
    return fp8_gemm_scaled(A, fa, B, fb, M, N, K, mode, a_scale_inv, b_scale_inv, D_bf16, ldd, scratch, need, stream);
}
