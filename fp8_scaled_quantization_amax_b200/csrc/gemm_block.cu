// gemm_block.cu -- FP8 GEMM with full fp32 per-block scales (1x128 blocks of
// A, 128x128 blocks of B), promoted per 128-wide K block on the CTA pairs.
//
// Sources: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3 (per-block
// scales: the tensor is cut into small blocks, each with its own scale),
// §5.3 (a fixed summation order per output, so results do not change run to
// run); "H100 FP8加速实测：新一代计算架构的飞跃" (the multiply-accumulate runs
// on the 8-bit floats in the tensor cores).
//
//   D[m, n] = bf16( sum_kb sa[kb, m] * sb[n / 128, kb] * sum_{k in kb} A[m, k] B[n, k] )
//
// The scales change every 128 elements of K, so no single epilogue scale
// exists: each K block's product is accumulated alone in tensor memory and
// the epilogue warps add it, scaled, into an fp32 register accumulator.
// What bounds this loop on sm_100a (measured with clock stamps):
//   * a CTA-pair MMA instruction (M = 256, K = 32) occupies the tensor core
//     ~190 cycles in a TMA-fed loop whether N is 128 or 256, so each K block
//     is issued as four N = 256 MMAs (splitting N doubles the MMA time);
//   * an mbarrier signal takes ~200 cycles from arrive to the waiter's
//     wake-up and a tcgen05.commit ~400 cycles from the MMAs' completion.
// Two 256-column TMEM buffers alternate by K-block parity: the MMAs of block
// kb + 1 run while block kb is read out, and the buffer goes back to the MMA
// as soon as the epilogue warps hold their columns in registers (before the
// second half of the FMAs).
// Layout per CTA of the pair (M = 256 rows per tile, 128 per CTA):
//   warp 0      TMA producer: per stage this CTA's 128 rows of A (16 KiB) and
//               its 128 rows of the tile's 256 rows of B (16 KiB);
//   warp 1      TMEM allocator; in the even CTA the MMA issuer;
//   warps 2-3   release warps of the two buffers: they return a partial
//               buffer to the MMA issuer once all eight epilogue warps
//               have read it (named barrier), so the epilogue warps never
//               stall on the mbarrier arrive (~200 cycles when it completes
//               a phase someone waits on);
//   warps 4-11  epilogue: warp w promotes TMEM lane quarter w % 4 (32 rows)
//               and column half g = (w - 4) / 4 (tile columns g * 128 .. +
//               127, one 128-row block of B, so one B scale) -- two 64-column
//               round trips, fp32 FMAs two columns per instruction
//               (fma.rn.f32x2: each column its own fma, one rounding per
//               term); then bf16 RNE and coalesced stores.
// Summation order per output is fixed (K blocks in order, each block's
// partial from the tensor core, then one FMA), so results are bit-identical
// run to run.  Every mbarrier wait is bounded (about one second, see tc.cuh);
// on expiry the kernel records a bit in this file's device error word, stops
// issuing, drains its copies and MMAs, frees TMEM and returns.
#include <algorithm>
#include <mutex>

#include "tc.cuh"

using namespace fp8q;
using fp8q_host::pdl_launch;

namespace {

namespace blk {
constexpr int STAGES = 6;
constexpr int B_TILE = 128 * BK;                // this CTA's 128 rows of B (16 KiB)
constexpr int STAGE = A_TILE + B_TILE;          // 32 KiB per stage and CTA
constexpr int NBUF = 2;                         // 256-column TMEM partial buffers
constexpr int NBARS = 2 * STAGES + 2 * NBUF + 1;   // full, empty, partial full / free, drain
constexpr size_t EPI_OFF = ((size_t)STAGES * STAGE + NBARS * 8 + 16 + 15) & ~(size_t)15;
constexpr size_t SMEM = 1024 + EPI_OFF + (size_t)sm2::EPI * kEpiBufBytes;
constexpr int PF = 1;                           // scale prefetch distance in K blocks
static_assert(SMEM <= 232448, "shared memory per block");
// Named barriers 1-2: the eight epilogue warps hand K block kb's finished
// reads to the release warp of buffer kb % 2 (warp 2 + kb % 2) through
// barrier 1 + kb % 2 (8 x 32 arriving threads + the 32 of the release warp).
constexpr int kReleaseThreads = 9 * 32;
}  // namespace blk

// 32 lanes x 64 consecutive fp32 columns in one load; valid after tmem_wait64.
__device__ __forceinline__ void tmem_ld64_async(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}
__device__ __forceinline__ void named_arrive(int id, int threads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// QFMT < 0: D = bf16(promoted sum).  QFMT = FP8_E4M3 / FP8_E5M2: the
// epilogue also requantizes its output with 1 x 128 blocks, as the 1x128
// block quantizer would quantize D (H of an MLP, requantized for the next
// GEMM): each thread holds one row of one 128-column block, so the block's
// amax, scale and cast happen in registers; D (optional) gets the bf16 values
// the codes were cast from, qo [M, N] the codes, qsinv [ceil(N / 128), M]
// the block scales' inverses, counts the non-finite / saturated counts.
template <int QFMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(sm2::THREADS, 1)
k_gemm_block_2sm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                 int K, uint32_t idesc, const float *__restrict__ sa, const float *__restrict__ sb,
                 __nv_bfloat16 *__restrict__ D, int64_t ldd, uint8_t *__restrict__ qo, float *__restrict__ qsinv,
                 uint32_t *__restrict__ counts) {
    constexpr int STG = blk::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)STG * blk::STAGE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + blk::NBARS);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = (rank == 0);
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (M + 255) / 256, num_n = (N + 255) / 256;
    const int tiles = num_m * num_n;
    const int nk = (K + BK - 1) / BK;
    const int n_items = (pair < tiles) ? (tiles - 1 - pair) / npairs + 1 : 0;

    auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_u32(&bars[STG + s]); };
    auto accf_bar = [&](int q) { return smem_u32(&bars[2 * STG + q]); };
    auto acce_bar = [&](int q) { return smem_u32(&bars[2 * STG + blk::NBUF + q]); };
    const uint32_t drain_bar = smem_u32(&bars[2 * STG + 2 * blk::NBUF]);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int q = 0; q < blk::NBUF; ++q) {
            mbar_init(accf_bar(q), 1);
            mbar_init(acce_bar(q), 2);   // both CTAs' release warps of that half
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

    // Each role branch resizes its own warpgroup's registers (the epilogue
    // holds a 128-wide fp32 accumulator row per thread); the launch pool is
    // checked on the host.
    if (warp == 0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(sm2::REGS_LOW));
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
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(empty_bar(stage), (round & 1u) ^ 1u, abort_flag, kErrProducer)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_leader = mapa_shared(full_bar(stage), 0);
                    if (leader) mbar_expect_tx(full_bar(stage), 2 * blk::STAGE);
                    const uint32_t a_dst = smem_u32(smem + (size_t)stage * blk::STAGE);
                    tma_load_2d_pair(a_dst, &tmA, full_leader, kc * BK, a_row);
                    tma_load_2d_pair(a_dst + A_TILE, &tmB, full_leader, kc * BK, b_row);
                    last_round[stage] = (int)round;
                }
            }
            if (leader && (!ok || *abort_flag)) {   // copies in flight must land before the CTA exits
                for (int s = 0; s < STG; ++s)
                    if (last_round[s] >= 0) wait_bar_drain(full_bar(s), (uint32_t)last_round[s] & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(sm2::REGS_LOW));
        // ------------------------------------- MMA issuer (leader only) --
        if (leader && lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int i = 0; ok && i < n_items; ++i) {
                for (int kc = 0; kc < nk; ++kc, ++it) {
                    const int stage = it % STG;
                    const uint32_t round = it / STG;
                    if (!wait_bar(full_bar(stage), round & 1u, abort_flag, kErrMma)) { ok = false; break; }
                    const uint32_t a_addr = smem_u32(smem + (size_t)stage * blk::STAGE);
                    const uint64_t adesc = sdesc_k_sw128(a_addr);
                    const uint64_t bdesc = sdesc_k_sw128(a_addr + A_TILE);
                    const int q = (int)(it & 1u);
                    if (!wait_bar(acce_bar(q), ((it >> 1) & 1u) ^ 1u, abort_flag, kErrMma)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)   // +32 bytes along K = +2 in the address field
                        tc_mma_pair(tmem + q * 256, adesc + 2u * k, bdesc + 2u * k, idesc, k > 0 ? 1u : 0u);
                    tc_commit_pair_both(accf_bar(q));
                    tc_commit_pair_both(empty_bar(stage));
                }
            }
            // all MMAs issued by this thread complete before TMEM is freed
            tc_commit_pair_self(drain_bar);
            wait_bar_drain(drain_bar, 0u);
        }
        __syncwarp();
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(sm2::REGS_LOW));
        // ---------------------------------------- release warp of buffer h --
        // An mbarrier arrive that completes a phase a thread is waiting on
        // stalls the arriving thread ~200 cycles; this warp takes that stall
        // off the epilogue warps, which only arrive on a named barrier.  Every
        // epilogue warp arrives once per K block on every path (the error path
        // included), so each bar.sync here returns.
        const int h = warp - 2;
        const uint32_t release_to = leader ? 0u : mapa_shared(acce_bar(0), 0);
        const uint32_t total = (uint32_t)n_items * (uint32_t)nk;
        for (uint32_t it = (uint32_t)h; it < total; it += 2) {
            named_sync(1 + h, blk::kReleaseThreads);
            if (lane == 0) {
                if (leader) mbar_arrive(acce_bar(h));
                else mbar_arrive_cluster(release_to + (uint32_t)(h * 8));
            }
            __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(sm2::REGS_HIGH));
        // --------------------------------------------------- epilogue ----
        const int sp = warp & 3;
        const int g = (warp - 4) >> 2;                  // column half: tile columns g * 128 .. + 127
        const uint32_t tsrc = tmem + ((uint32_t)(sp * 32) << 16) + (uint32_t)(g * 128);   // this warp's lanes and columns
        uint32_t nf_q = 0, sat_q = 0;   // requantization counters
        uint32_t it = 0;
        bool ok = true;
        for (int i = 0; ok && i < n_items; ++i) {
            const int t = pair + i * npairs;
            const int m_blk = t % num_m, n_blk = t / num_m;
            const int64_t row0 = (int64_t)m_blk * 256 + (int)rank * 128 + sp * 32;
            // Scale loads are unconditional, from addresses clamped into the
            // arrays: rows past M and columns past N are never stored, so their
            // scales do not matter, and a load whose value is selected at once
            // would stall the warp until it lands.
            const int nbn = (N + 127) / 128;
            const float *sap = sa + min(row0 + lane, (int64_t)M - 1);          // + kc * M: block kc
            const float *sbp = sb + (int64_t)min(n_blk * 2 + g, nbn - 1) * nk;  // [kc]
            float acc[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
            // Scales run PF K blocks ahead in PF register sets (the K loop is
            // unrolled by PF, so no register copy waits on a load).
            float as_[blk::PF], bs_[blk::PF];
#pragma unroll
            for (int p = 0; p < blk::PF; ++p) {
                const int64_t kb = min(p, nk - 1);
                as_[p] = sap[kb * M];
                bs_[p] = sbp[kb];
            }
            // One K block: wait for the partial, read this warp's 128 columns
            // in two round trips, hand the buffer back, promote.  A failed wait
            // (the kernel is aborting) only clears ok_tile: the tile runs to
            // its end on whatever TMEM holds, so the hot loop has no early
            // exit and every named-barrier arrival happens; its stores are
            // skipped.
            bool ok_tile = true;
            auto promote = [&](int kc, float &as, float &bs) {
                const float sc = __fmul_rn(as, bs);
                if (kc + blk::PF < nk) {   // block kc + PF's scales
                    as = sap[(int64_t)(kc + blk::PF) * M];
                    bs = sbp[kc + blk::PF];
                }
                const int q = (int)(it & 1u);
                bool w = true;
                if (lane == 0) w = wait_bar(accf_bar(q), (it >> 1) & 1u, abort_flag, kErrEpilogue);
                ok_tile = __shfl_sync(0xFFFFFFFFu, w, 0) && ok_tile;
                tc_fence_after();
                uint32_t r[64];
                tmem_ld64_async(tsrc + q * 256, r);
                tmem_wait64(r);
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    const float2 o = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), make_float2(sc, sc),
                                                make_float2(acc[j], acc[j + 1]));
                    acc[j] = o.x;
                    acc[j + 1] = o.y;
                }
                tmem_ld64_async(tsrc + q * 256 + 64, r);
                tmem_wait64(r);
                // the partial is in registers: the release warp hands the buffer back to the MMA
                tc_fence_before();
                named_arrive(1 + q, blk::kReleaseThreads);
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    const float2 o = __ffma2_rn(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), make_float2(sc, sc),
                                                make_float2(acc[64 + j], acc[64 + j + 1]));
                    acc[64 + j] = o.x;
                    acc[64 + j + 1] = o.y;
                }
                ++it;
            };
            for (int kc = 0; kc < nk; kc += blk::PF) {
#pragma unroll
                for (int p = 0; p < blk::PF; ++p)
                    if (kc + p < nk) promote(kc + p, as_[p], bs_[p]);
            }
            if (!ok_tile) {   // aborting: the release warps still expect one arrival per K block
                ok = false;
                for (const uint32_t total = (uint32_t)n_items * (uint32_t)nk; it < total; ++it)
                    named_arrive(1 + (int)(it & 1u), blk::kReleaseThreads);
                break;
            }
            uint8_t *ebuf = smem + blk::EPI_OFF + (size_t)(warp - 4) * kEpiBufBytes;
            const int colb = n_blk * 256 + g * 128;   // this warp's 128 columns: one 1 x 128 block
            if constexpr (QFMT < 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(acc[h * 64 + 2 * j], acc[h * 64 + 2 * j + 1]);
                    store_rows_coalesced(ebuf, pk, lane, D, ldd, row0, (int64_t)M, colb + h * 64, N);
                }
            } else {
                constexpr float fm = fmax_of<QFMT>();
                uint32_t hb[2][32];   // the row's 128 outputs in bf16, RNE: the values the codes come from
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 32; ++j) hb[h][j] = pack_bf16x2(acc[h * 64 + 2 * j], acc[h * 64 + 2 * j + 1]);
                if (D != nullptr) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) store_rows_coalesced(ebuf, hb[h], lane, D, ldd, row0, (int64_t)M, colb + h * 64, N);
                }
                // amax over the finite values of the block's columns below N (N % 16 == 0)
                const int nvalid = N - colb;
                uint32_t m2 = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 32; ++j) m2 = amax_fast_word(m2, (h * 64 + 2 * j < nvalid) ? hb[h][j] : 0u);
                uint32_t m = amax_fast_final(m2);
                const bool nonfin = m == 0xFFFFFFFFu;
                if (nonfin) {
                    uint32_t bad = 0;
                    m = 0;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (h * 64 + 2 * j < nvalid) m = amax_exact_word(m, hb[h][j], bad);
                }
                const float amax = bf16bits_to_float(m);
                const float s = scale_from_amax(amax, fm);
                const bool row_ok = row0 + lane < M;
                if (row_ok && nvalid > 0) qsinv[(int64_t)(colb / 128) * M + row0 + lane] = __fdiv_rn(1.0f, s);
                if (counts != nullptr && row_ok && may_saturate(nonfin, amax, s, fm)) {
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (h * 64 + 2 * j >= nvalid) continue;
                            const uint32_t w = hb[h][j];
                            nf_q += ((w & 0x7F80u) == 0x7F80u) + ((w & 0x7F800000u) == 0x7F800000u);
                            sat_q += (fabsf(__fmul_rn(bf_lo(w), s)) > fm) + (fabsf(__fmul_rn(bf_hi(w), s)) > fm);
                        }
                }
                uint32_t qw[32];   // 128 codes, four per word, column order
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const uint32_t w0 = hb[j >> 4][2 * (j & 15)], w1 = hb[j >> 4][2 * (j & 15) + 1];
                    const uint32_t c0 = cvt2<QFMT>(__fmul_rn(bf_lo(w0), s), __fmul_rn(bf_hi(w0), s));
                    const uint32_t c1 = cvt2<QFMT>(__fmul_rn(bf_lo(w1), s), __fmul_rn(bf_hi(w1), s));
                    qw[j] = c0 | (c1 << 16);
                }
                store_rows_coalesced(ebuf, qw, lane, qo, (int64_t)N, row0, (int64_t)M, colb, N);
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

// Pairs of the block-scaled kernel that fit on the device at once (cached per
// device and variant); 0 when the kernel cannot be launched as the register
// split needs.
template <int QFMT>
int block_pair_capacity() {
    static int cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(k_gemm_block_2sm<QFMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)blk::SMEM) !=
        cudaSuccess)
        return 0;
    cudaFuncAttributes fa;   // the setmaxnreg split assumes this launch register count
    if (cudaFuncGetAttributes(&fa, k_gemm_block_2sm<QFMT>) != cudaSuccess || fa.numRegs != sm2::REGS_LAUNCH) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(sm2::THREADS);
    cfg.dynamicSmemBytes = blk::SMEM;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)k_gemm_block_2sm<QFMT>, &cfg) != cudaSuccess) return 0;
    cache[dev] = n;
    return n;
}

template <int QFMT>
fp8_status launch_block_pair(const CUtensorMap &ta, const CUtensorMap &tb, int64_t M, int64_t N, int64_t K,
                             uint32_t idesc, const float *sa, const float *sb, void *D_bf16, int64_t ldd, uint8_t *qo,
                             float *qsinv, uint32_t *counts, cudaStream_t s) {
    const int cap = block_pair_capacity<QFMT>();
    if (cap <= 0) return FP8_ERR_CUDA;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, cap));
    return pdl_launch(k_gemm_block_2sm<QFMT>, dim3(2 * pairs), dim3(sm2::THREADS), blk::SMEM, s, ta, tb, (int)M,
                      (int)N, (int)K, idesc, sa, sb, static_cast<__nv_bfloat16 *>(D_bf16), ldd, qo, qsinv,
                      counts) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_CUDA;
}

}  // namespace

using namespace fp8q_host;

// The block-scaled GEMM on CTA pairs (M > 128 rows); arguments validated by
// the entry points.  qo == NULL: D only.  qo != NULL: the output is also
// requantized with 1 x 128 blocks of format qfmt (D may then be NULL).
// Returns FP8_ERR_CUDA when a map cannot be encoded or the launch fails.
fp8_status fp8q_gemm_block_pair(const uint8_t *A, fp8_format fa, const uint8_t *B, fp8_format fb, int64_t M,
                                int64_t N, int64_t K, const float *sa, const float *sb, void *D_bf16, int64_t ldd,
                                fp8_format qfmt, uint8_t *qo, float *qsinv, uint32_t *counts, cudaStream_t s) {
    CUtensorMap ta, tb;
    if (!make_map(&ta, A, K, M, 128) || !make_map(&tb, B, K, N, 128)) return FP8_ERR_CUDA;
    // fp32 accumulator, A/B formats, K-major A and B, N = 256 (>> 3), M = 256 (>> 4)
    const uint32_t idesc = (1u << 4) | ((uint32_t)fa << 7) | ((uint32_t)fb << 10) | ((uint32_t)(256 >> 3) << 17) |
                           ((uint32_t)(256 >> 4) << 24);
    if (qo == nullptr)
        return launch_block_pair<-1>(ta, tb, M, N, K, idesc, sa, sb, D_bf16, ldd, nullptr, nullptr, nullptr, s);
    if (qfmt == FP8_E4M3)
        return launch_block_pair<FP8_E4M3>(ta, tb, M, N, K, idesc, sa, sb, D_bf16, ldd, qo, qsinv, counts, s);
    return launch_block_pair<FP8_E5M2>(ta, tb, M, N, K, idesc, sa, sb, D_bf16, ldd, qo, qsinv, counts, s);
}

// This file's device error word (read and optionally cleared by
// fp8_device_error together with the other GEMM files').
fp8_status fp8q_block_device_error(uint32_t *out, int clear) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
    *out = v;
    if (clear) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z)) != cudaSuccess) return FP8_ERR_CUDA;
    }
    return FP8_OK;
}
