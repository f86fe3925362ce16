// gemm_mx.cu -- FP8 GEMM with power-of-two block scales applied by the
// tensor core (tcgen05.mma.kind::mxf8f6f4.block_scale with E8M0 factors).
//
// Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-block
// scales: 1x128 activation blocks and 128x128 weight blocks);
// "FP8训练与QAT量化感知训练：…用Soup把大模型微调提速2倍", section
// "FP8 三种缩放配方怎么选" (power-of-two scales); "H100 FP8加速实测：新一代计算
// 架构的飞跃" (FP8 multiply-accumulate on the tensor cores).
//
// Every mbarrier wait is bounded (about one second, see tc.cuh); on expiry
// the kernel records a bit in this file's device error word, stops issuing,
// drains its copies and MMAs, frees TMEM and returns.
#include <algorithm>
#include <mutex>

#include "tc.cuh"

using namespace fp8q;
using fp8q_host::pdl_launch;

namespace {

// ----------------------------------------- hardware block scales (E8M0) ----
// Power-of-two block scales applied inside the tensor core:
// tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale multiplies every
// 32-wide K slice of A's row m by 2^(sfa - 127) and of B's row n by
// 2^(sfb - 127) before accumulating, so the fp32 accumulator already holds
// sum_kb dA[m, kb] * dB[n, kb] * sum_{k in kb} A[m, k] B[n, k] and the
// epilogue only rounds to bf16 -- no per-128-K promotion.
//
// The E8M0 factors come as images in the MMA's scale-factor layout (see the
// quantizer): one byte per row and 128-wide K block, four K blocks per 32-bit
// word, 512 bytes per 128 rows and group of four K blocks.  Every fourth
// stage, each CTA of the pair TMA-loads its own 128 rows' SFA entry (512 B)
// and the SFB entries of all 256 tile columns (1 KiB; both CTAs need all
// columns, since each CTA's accumulator rows span the whole tile width) next
// to its A and B tiles; the leader copies them into TMEM with
// tcgen05.cp.cta_group::2.32x128b.warpx4 (32 lanes x 16 bytes broadcast to the
// four lane quarters: TMEM lane m % 32 (+ 32 q), column m / 32 holds row m's
// word) ahead of that stage's MMAs, and the MMAs of K block kb select byte
// kb % 4 of each word.  Copies and MMAs run in issue order, so a copy never
// overwrites factors an earlier MMA still reads.  One copy per four K blocks
// instead of one per block: the copies cost ~11 % of the GEMM at one per block.
// The SF columns sit after a single 256-column accumulator (TMEM has 512
// columns), so the epilogue drains the whole accumulator into registers and
// releases it before converting and storing (measured: the drain costs ~1 %).
namespace mx {
constexpr int SFA_BYTES = 512;                    // 128 rows x 4 bytes
constexpr int SFB_BYTES = 1024;                   // 256 columns x 4 bytes
constexpr int AB_STAGE = A_TILE + 128 * BK;       // this CTA's 128 rows of A and of B
constexpr int SF_STAGE = SFA_BYTES + SFB_BYTES;
constexpr int STAGES = 6;
constexpr int NBARS = 2 * STAGES + 3;             // full, empty, acc full, acc empty, drain
// after the pipeline and the barriers: one store_rows_coalesced buffer per epilogue warp
constexpr size_t EPI_OFF = ((size_t)STAGES * (AB_STAGE + SF_STAGE) + NBARS * 8 + 16 + 15) & ~(size_t)15;
constexpr size_t SMEM = 1024 + EPI_OFF + (size_t)sm2::EPI * kEpiBufBytes;
constexpr uint32_t SFA_COL = 256, SFB_COL = 260;  // TMEM columns after the accumulator
static_assert(SMEM <= 232448, "shared memory per block");
}  // namespace mx

// Shared-memory descriptor of a 32-row x 16-byte block without swizzle
// (8-row core matrices 128 bytes apart): the source of a 32x128b tcgen05.cp.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);    // start address (16-byte units)
    d |= (uint64_t)(128u >> 4) << 32;           // stride byte offset: 8 rows x 16 B
    d |= (uint64_t)1u << 46;                    // descriptor version for sm_100
    return d;                                   // layout type 0: no swizzle
}
__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_pair_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa, uint32_t sfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
        : "memory");
}

// QFMT < 0: D = bf16(sum).  QFMT = FP8_E4M3 / FP8_E5M2: the epilogue also
// requantizes its output with 1 x 128 blocks and power-of-two scales, as
// fp8_quantize_blockwise_e8m0 would quantize D: each thread holds one row of
// one 128-column block; D (optional) gets the bf16 values, qo [M, N] the
// codes, qsf the E8M0 image of the next GEMM's A operand (rows past M in the
// last 128-row group: e = 127), counts the non-finite / saturated counts.
template <int QFMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(sm2::THREADS, 1)
k_gemm_mx_2sm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB, int M, int N,
              int K, uint32_t idesc, __nv_bfloat16 *__restrict__ D, int64_t ldd, uint8_t *__restrict__ qo,
              uint8_t *__restrict__ qsf, uint32_t *__restrict__ counts) {
    constexpr int STG = mx::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sf_smem = smem + (size_t)STG * mx::AB_STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sf_smem + (size_t)STG * mx::SF_STAGE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + mx::NBARS);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = (rank == 0);
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (M + 255) / 256, num_n = (N + 255) / 256;
    const int tiles = num_m * num_n;
    const int mt = (M + 127) / 128, nt = (N + 127) / 128;   // 128-row entries per K block of each image
    const int nk = (K + BK - 1) / BK;
    const int n_items = (pair < tiles) ? (tiles - 1 - pair) / npairs + 1 : 0;

    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STG + s]); };
    const uint32_t accf_bar = smem_u32(&bars[2 * STG]);
    const uint32_t acce_bar = smem_u32(&bars[2 * STG + 1]);
    const uint32_t drain_bar = smem_u32(&bars[2 * STG + 2]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(accf_bar, 1);
        mbar_init(acce_bar, 2 * sm2::EPI);
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSB)) : "memory");
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
                const int m_blk = t % num_m, n_blk = t / num_m;
                const int a_row = m_blk * 256 + (int)rank * 128;
                const int b_row = n_blk * 256 + (int)rank * 128;
                const int sa_ent = m_blk * 2 + (int)rank, sb_ent = n_blk * 2;
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(empty_bar(stage), (round & 1u) ^ 1u, abort_flag, kErrProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(full_bar(stage), 0);
                    const bool sf = (kc & 3) == 0;   // first K block of a group of four
                    if (leader) mbar_expect_tx(full_bar(stage), 2 * (mx::AB_STAGE + (sf ? mx::SF_STAGE : 0)));
                    const uint32_t a_dst = smem_u32(smem + (size_t)stage * mx::AB_STAGE);
                    tma_load_2d_pair(a_dst, &tmA, full_leader, kc * BK, a_row);
                    tma_load_2d_pair(a_dst + A_TILE, &tmB, full_leader, kc * BK, b_row);
                    if (sf) {   // image rows of 16 bytes: 32 per 128-row entry
                        const uint32_t sf_dst = smem_u32(sf_smem + (size_t)stage * mx::SF_STAGE);
                        const int g = kc >> 2;
                        tma_load_2d_pair(sf_dst, &tmSA, full_leader, 0, (g * mt + sa_ent) * 32);
                        tma_load_2d_pair(sf_dst + mx::SFA_BYTES, &tmSB, full_leader, 0, (g * nt + sb_ent) * 32);
                    }
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
            const uint32_t sfa_t = tmem + mx::SFA_COL, sfb_t = tmem + mx::SFB_COL;
            for (int i = 0; ok && i < n_items; ++i) {
                if (!wait_bar(acce_bar, ((uint32_t)i & 1u) ^ 1u, abort_flag, kErrMma)) break;
                tc_fence_after();
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(full_bar(stage), round & 1u, abort_flag, kErrMma)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)stage * mx::AB_STAGE);
                    const uint32_t sf_addr = smem_u32(sf_smem + (size_t)stage * mx::SF_STAGE);
                    if ((kc & 3) == 0) {
                        tc_cp_sf_pair(sfa_t, sdesc_sf(sf_addr));
                        tc_cp_sf_pair(sfb_t, sdesc_sf(sf_addr + mx::SFA_BYTES));
                        tc_cp_sf_pair(sfb_t + 4, sdesc_sf(sf_addr + mx::SFA_BYTES + 512));
                    }
                    const uint64_t adesc = sdesc_k_sw128(a_addr);
                    const uint64_t bdesc = sdesc_k_sw128(a_addr + A_TILE);
                    // scale-factor byte kc % 4 of each 32-bit TMEM word for all
                    // four 32-wide slices of this K block
                    const uint32_t id = idesc | ((uint32_t)(kc & 3) << 4) | ((uint32_t)(kc & 3) << 29);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        tc_mma_pair_mx(tmem, adesc + 2u * k, bdesc + 2u * k, id, sfa_t, sfb_t,
                                       (kc > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_both(empty_bar(stage));
                }
                if (ok) tc_commit_pair_both(accf_bar);
            }
            tc_commit_pair_self(drain_bar);
            wait_bar_drain(drain_bar, 0u);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // --------------------------------------------------- epilogue ----
        const int sp = warp & 3;
        const int ch = (warp - 4) >> 2;
        const uint32_t src = tmem + ((uint32_t)(sp * 32) << 16) + ch * 128;
        uint32_t nf_q = 0, sat_q = 0;   // requantization counters
        for (int i = 0; i < n_items; ++i) {
            const int t = pair + i * npairs;
            const int m_blk = t % num_m, n_blk = t / num_m;
            const int64_t m = (int64_t)m_blk * 256 + (int)rank * 128 + sp * 32 + lane;
            const int n_base = n_blk * 256 + ch * 128;
            bool w = true;
            if (lane == 0) w = wait_bar(accf_bar, (uint32_t)i & 1u, abort_flag, kErrEpilogue);
            w = __shfl_sync(0xFFFFFFFFu, w, 0);
            if (!w) break;
            tc_fence_after();
            // the whole 128-column slice of this warp, then hand TMEM back
            uint32_t r0[64], r1[64];
            tmem_ld32_async(src, r0);
            tmem_ld32_async(src + 32, r0 + 32);
            tmem_ld32_async(src + 64, r1);
            tmem_ld32_async(src + 96, r1 + 32);
            tmem_wait64(r0);
            tmem_wait64(r1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar, 0));
            uint8_t *ebuf = smem + mx::EPI_OFF + (size_t)(warp - 4) * kEpiBufBytes;
            if constexpr (QFMT < 0) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const uint32_t *r = h2 ? r1 : r0;
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                    store_rows_coalesced(ebuf, pk, lane, D, ldd, m - lane, M, n_base + h2 * 64, N);
                }
            } else {
                constexpr float fm = fmax_of<QFMT>();
                uint32_t hb[2][32];   // the row's 128 outputs in bf16, RNE: the values the codes come from
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    hb[0][j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
                    hb[1][j] = pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
                }
                if (D != nullptr) {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) store_rows_coalesced(ebuf, hb[h2], lane, D, ldd, m - lane, M, n_base + h2 * 64, N);
                }
                // amax over the finite values of the block's columns below N (N % 16 == 0)
                const int nvalid = N - n_base;
                uint32_t m2 = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 32; ++j) m2 = amax_fast_word(m2, (h * 64 + 2 * j < nvalid) ? hb[h][j] : 0u);
                uint32_t mx16 = amax_fast_final(m2);
                const bool nonfin = mx16 == 0xFFFFFFFFu;
                if (nonfin) {
                    uint32_t bad = 0;
                    mx16 = 0;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (h * 64 + 2 * j < nvalid) mx16 = amax_exact_word(mx16, hb[h][j], bad);
                }
                const float amax = bf16bits_to_float(mx16);
                const float sc = pow2_scale_from_amax(amax, fm);
                const bool row_ok = m < M;
                const int64_t rt = ((int64_t)M + 127) / 128;
                if (nvalid > 0 && m < rt * 128)   // rows past M in the last 128-row group: factor 1
                    qsf[e8m0_offset(n_base / 128, rt, m)] = row_ok ? e8m0_of_scale(sc) : (uint8_t)127;
                if (counts != nullptr && row_ok && may_saturate(nonfin, amax, sc, fm)) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (h * 64 + 2 * j >= nvalid) continue;
                            const uint32_t w = hb[h][j];
                            nf_q += ((w & 0x7F80u) == 0x7F80u) + ((w & 0x7F800000u) == 0x7F800000u);
                            sat_q += (fabsf(__fmul_rn(bf_lo(w), sc)) > fm) + (fabsf(__fmul_rn(bf_hi(w), sc)) > fm);
                        }
                }
                uint32_t qw[32];   // 128 codes, four per word, column order
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t w0 = hb[j >> 4][2 * (j & 15)], w1 = hb[j >> 4][2 * (j & 15) + 1];
                    const uint32_t c0 = cvt2<QFMT>(__fmul_rn(bf_lo(w0), sc), __fmul_rn(bf_hi(w0), sc));
                    const uint32_t c1 = cvt2<QFMT>(__fmul_rn(bf_lo(w1), sc), __fmul_rn(bf_hi(w1), sc));
                    qw[j] = c0 | (c1 << 16);
                }
                store_rows_coalesced(ebuf, qw, lane, qo, (int64_t)N, m - lane, (int64_t)M, n_base, N);
            }
        }
        if constexpr (QFMT >= 0) {
            if (counts != nullptr) flush_counts(counts, nf_q, sat_q);
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

// 2-D map over an E8M0 scale image viewed as rows of 16 bytes, box 16 x
// box_rows, no swizzle (the 32x128b tcgen05.cp source layout).
bool make_sf_map(CUtensorMap *map, const void *base, int64_t rows16, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {16, (cuuint64_t)rows16};
    cuuint64_t strides[1] = {16};
    cuuint32_t box[2] = {16, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pairs of the E8M0 kernel that fit on the device at once (cached per device
// and variant).
template <int QFMT>
int mx_pair_capacity() {
    static int cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(k_gemm_mx_2sm<QFMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mx::SMEM) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(sm2::THREADS);
    cfg.dynamicSmemBytes = mx::SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_gemm_mx_2sm<QFMT>, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

// Instruction descriptor of kind::mxf8f6f4 with E8M0 scale factors: A/B
// formats, K-major A and B, N >> 3, scale type E8M0 (bit 23), M >> 4; the
// scale-factor byte selectors (bits 4-5 for B, 29-30 for A) are set per MMA.
uint32_t make_idesc_mx(fp8_format fa, fp8_format fb, int mma_m, int mma_n) {
    return ((uint32_t)fa << 7) | ((uint32_t)fb << 10) | ((uint32_t)(mma_n >> 3) << 17) | (1u << 23) |
           ((uint32_t)(mma_m >> 4) << 24);
}

template <int QFMT>
fp8_status launch_mx_q(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa, const CUtensorMap &tsb,
                       int64_t M, int64_t N, int64_t K, uint32_t idesc, void *D_bf16, int64_t ldd, uint8_t *qo,
                       uint8_t *qsf, uint32_t *counts, cudaStream_t s) {
    const int cap = mx_pair_capacity<QFMT>();
    if (cap <= 0) return FP8_ERR_CUDA;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, cap));
    return pdl_launch(k_gemm_mx_2sm<QFMT>, dim3(2 * pairs), dim3(sm2::THREADS), mx::SMEM, s, ta, tb, tsa, tsb,
                      (int)M, (int)N, (int)K, idesc, static_cast<__nv_bfloat16 *>(D_bf16), ldd, qo, qsf,
                      counts) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_CUDA;
}

// Maps and launch; qo == NULL: bf16 output only.
fp8_status launch_mx(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int64_t M, int64_t N,
                     int64_t K, const uint8_t *a_sf, const uint8_t *b_sf, void *D_bf16, int64_t ldd, fp8_format fo,
                     uint8_t *qo, uint8_t *qsf, uint32_t *counts, cudaStream_t s) {
    const int64_t ng = (K + 4 * BK - 1) / (4 * BK);   // groups of four K blocks in the images
    CUtensorMap ta, tb, tsa, tsb;
    if (!make_map(&ta, A, K, M, 128) || !make_map(&tb, B, K, N, 128)) return FP8_ERR_CUDA;
    if (!make_sf_map(&tsa, a_sf, ng * ((M + 127) / 128) * 32, 32) ||
        !make_sf_map(&tsb, b_sf, ng * ((N + 127) / 128) * 32, 64))
        return FP8_ERR_CUDA;
    const uint32_t idesc = make_idesc_mx(fa, fb, 256, 256);
    if (qo == nullptr) return launch_mx_q<-1>(ta, tb, tsa, tsb, M, N, K, idesc, D_bf16, ldd, nullptr, nullptr, nullptr, s);
    if (fo == FP8_E4M3) return launch_mx_q<FP8_E4M3>(ta, tb, tsa, tsb, M, N, K, idesc, D_bf16, ldd, qo, qsf, counts, s);
    return launch_mx_q<FP8_E5M2>(ta, tb, tsa, tsb, M, N, K, idesc, D_bf16, ldd, qo, qsf, counts, s);
}

}  // namespace

using namespace fp8q_host;

extern "C" fp8_status fp8_gemm_block_e8m0(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                          int64_t M, int64_t N, int64_t K, const uint8_t *a_sf, const uint8_t *b_sf,
                                          void *D_bf16, int64_t ldd, void *stream) {
    if ((fa != FP8_E4M3 && fa != FP8_E5M2) || (fb != FP8_E4M3 && fb != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || ldd < N) return FP8_ERR_SHAPE;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP8_ERR_SHAPE;
    if (K % 16) return FP8_ERR_SHAPE;
    if (N % 8 || ldd % 8) return FP8_ERR_ALIGNMENT;
    const int64_t ng = (K + 4 * BK - 1) / (4 * BK);   // groups of four K blocks in the images
    // image rows of 16 bytes must stay addressable by a 32-bit TMA coordinate
    if (ng * ((M + 127) / 128) * 32 >= (1ll << 31) || ng * ((N + 127) / 128) * 32 >= (1ll << 31)) return FP8_ERR_SHAPE;
    int sms;
    if (M == 0 || N == 0) return check_device(&sms);
    if (!D_bf16) return FP8_ERR_INVALID_ARG;
    if (K > 0 && (!A || !B || !a_sf || !b_sf)) return FP8_ERR_INVALID_ARG;
    if (!aligned16(D_bf16) || (A && !aligned16(A)) || (B && !aligned16(B)) || (a_sf && !aligned16(a_sf)) ||
        (b_sf && !aligned16(b_sf)))
        return FP8_ERR_ALIGNMENT;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (K == 0)
        return cudaMemset2DAsync(D_bf16, (size_t)ldd * 2, 0, (size_t)N * 2, (size_t)M, s) == cudaSuccess ? FP8_OK
                                                                                                       : FP8_ERR_CUDA;
    return launch_mx(A, fa, B, fb, M, N, K, a_sf, b_sf, D_bf16, ldd, FP8_E4M3, nullptr, nullptr, nullptr, s);
}

// The E8M0 GEMM with its output requantized 1 x 128 (power-of-two scales)
// in the epilogue; see include/fp8q.h.
extern "C" fp8_status fp8_gemm_block_e8m0_requant(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb,
                                                  int64_t M, int64_t N, int64_t K, const uint8_t *a_sf,
                                                  const uint8_t *b_sf, void *D_bf16, int64_t ldd, fp8_format fo,
                                                  uint8_t *q, uint8_t *q_sf, uint32_t *counts, void *stream) {
    if ((fa != FP8_E4M3 && fa != FP8_E5M2) || (fb != FP8_E4M3 && fb != FP8_E5M2)) return FP8_ERR_INVALID_ARG;
    if (fo != FP8_E4M3 && fo != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8_ERR_SHAPE;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP8_ERR_SHAPE;
    if (K % 16 || N % 16) return FP8_ERR_SHAPE;
    if (D_bf16 && ldd < N) return FP8_ERR_SHAPE;
    if (D_bf16 && (ldd % 8 || !aligned16(D_bf16))) return FP8_ERR_ALIGNMENT;
    const int64_t ng = (K + 4 * BK - 1) / (4 * BK);
    if (ng * ((M + 127) / 128) * 32 >= (1ll << 31) || ng * ((N + 127) / 128) * 32 >= (1ll << 31)) return FP8_ERR_SHAPE;
    if (M > 0 && N > 0) {
        if (!q || !q_sf) return FP8_ERR_INVALID_ARG;
        if (K > 0 && (!A || !B || !a_sf || !b_sf)) return FP8_ERR_INVALID_ARG;
    }
    if ((q && !aligned16(q)) || (A && !aligned16(A)) || (B && !aligned16(B)) || (a_sf && !aligned16(a_sf)) ||
        (b_sf && !aligned16(b_sf)))
        return FP8_ERR_ALIGNMENT;
    if (counts && (reinterpret_cast<uintptr_t>(counts) & 3u)) return FP8_ERR_ALIGNMENT;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    if (M == 0 || N == 0) return FP8_OK;
    cudaStream_t s = as_stream(stream);
    if (K == 0) {   // D = 0: codes 0, every block's factor 1 (e = 127)
        const size_t img = (size_t)((N + 511) / 512) * (size_t)((M + 127) / 128) * 512;
        if (D_bf16 && cudaMemset2DAsync(D_bf16, (size_t)ldd * 2, 0, (size_t)N * 2, (size_t)M, s) != cudaSuccess)
            return FP8_ERR_CUDA;
        if (cudaMemsetAsync(q, 0, (size_t)M * N, s) != cudaSuccess || cudaMemsetAsync(q_sf, 127, img, s) != cudaSuccess)
            return FP8_ERR_CUDA;
        return FP8_OK;
    }
    return launch_mx(A, fa, B, fb, M, N, K, a_sf, b_sf, D_bf16, ldd, fo, q, q_sf, counts, s);
}

// This file's device error word (read and optionally cleared by
// fp8_device_error together with the other GEMM file's).
fp8_status fp8q_mx_device_error(uint32_t *out, int clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
    *out = v;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z)) != cudaSuccess) return FP8_ERR_CUDA;
    }
    return FP8_OK;
}
