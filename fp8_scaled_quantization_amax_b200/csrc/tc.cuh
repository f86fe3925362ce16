// tc.cuh -- shared pieces of the tcgen05 GEMM kernels: tile constants, the
// PTX wrappers (mbarriers with bounded waits, TMA, tcgen05 MMA / TMEM / commit,
// shared-memory descriptors), CTA-pair helpers, and the host-side tensor-map
// encoding.  Everything sits in an anonymous namespace, so every translation
// unit that includes it gets its own copy -- including its own device error
// word g_gemm_error, which that unit's host code reads back.
#pragma once

#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace {

using namespace fp8q;

constexpr int BM = 128;                 // tile rows (TMEM lanes)
constexpr int BK = 128;                 // K chunk: one 128-byte swizzle row of FP8
constexpr int A_TILE = BM * BK;         // 16 KiB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kTimeoutNs = 1000000000ull;

enum : uint32_t { kErrProducer = 1u, kErrMma = 2u, kErrEpilogue = 4u, kErrDrain = 8u, kErrSplit = 16u };

__device__ unsigned int g_gemm_error;

// ------------------------------------------------------------- PTX glue --
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Local arrive used to release a TMEM buffer (relaxed for the same reason as
// mbar_arrive_cluster below: the guarded TMEM loads have completed).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait for the phase of `bar` with the given parity.  Gives up when
// the CTA's abort flag is raised or after kTimeoutNs (then it raises the flag
// and records `code` in the device error word).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t *abort_flag,
                                      uint32_t code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                atomicOr(&g_gemm_error, code);
                *abort_flag = 1u;
                return false;
            }
        }
    }
}
// Bounded wait that ignores the abort flag (used to drain work in flight).
__device__ __forceinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kTimeoutNs) {
            atomicOr(&g_gemm_error, kErrDrain);
            return false;
        }
    }
    return true;
}
// Split-K hand-off flag: the first-half pair publishes its partial with a
// release store of the launch's epoch; the second-half pair polls with
// acquire loads (bounded, like every wait in this file).
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ bool wait_flag(const uint32_t *p, uint32_t epoch, volatile uint32_t *abort_flag) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (ld_acquire_u32(p) == epoch) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                atomicOr(&g_gemm_error, kErrSplit);
                *abort_flag = 1u;
                return false;
            }
        }
        __nanosleep(32);
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// 32 lanes x 32 consecutive fp32 columns: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// 32 lanes x 32 columns, issued without waiting: the registers are only
// valid after tmem_wait64() on the array that contains them.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// One wait for all loads in flight; the 64 registers are named read-write so
// no use of them can move above the wait.
__device__ __forceinline__ void tmem_wait64(uint32_t (&r)[64]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31]), "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]),
                   "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]), "+r"(r[40]), "+r"(r[41]), "+r"(r[42]),
                   "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]), "+r"(r[48]), "+r"(r[49]),
                   "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]), "+r"(r[56]),
                   "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
                 :
                 : "memory");
}

// Packed fp32 pair arithmetic (sm_100): two IEEE round-to-nearest FMAs per
// instruction, which halves the issue cost of the block-scale promotion.
__device__ __forceinline__ uint64_t pack_f32x2(uint32_t lo, uint32_t hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart (the layout TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B and a 128-byte inner box).
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);    // start address (16-byte units)
    d |= (uint64_t)1u << 16;                    // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024u >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                    // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                    // layout: SWIZZLE_128B
    return d;
}

// Coalesced epilogue stores.  After tcgen05.ld a lane holds one output row,
// so storing straight from registers makes every 16-byte store instruction
// touch 32 rows (32 cache lines).  Instead a warp passes 128 bytes of each of
// its 32 rows (64 bf16 or 32 fp32 columns, pk[] = the lane's row) through a
// 16-row shared buffer in two passes: each lane of the half-warp writes its
// row, then every lane reads 16 bytes, so that one global store instruction
// writes 4 rows x 128 contiguous bytes (4 lines).  The 144-byte row pitch
// keeps both shared accesses free of bank conflicts.  ACC (fp32 only) adds
// the values already in D.  Warp-collective: all 32 lanes call it together.
constexpr int kEpiRowPitch = 144;
constexpr int kEpiBufBytes = 16 * kEpiRowPitch;   // per epilogue warp
template <typename T, bool ACC = false>
__device__ __forceinline__ void store_rows_coalesced(uint8_t *buf, const uint32_t (&pk)[32], int lane,
                                                     T *__restrict__ D, int64_t ldd, int64_t row0, int64_t row_end,
                                                     int col0, int N) {
    constexpr int kPer16 = 16 / (int)sizeof(T);   // columns per 16 bytes
    static_assert(!ACC || sizeof(T) == 4, "accumulation is for fp32 outputs");
    const uint32_t sb = smem_u32(buf);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if ((lane >> 4) == h) {
            const uint32_t dst = sb + (uint32_t)(lane & 15) * kEpiRowPitch;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16u * j), "r"(pk[4 * j]),
                             "r"(pk[4 * j + 1]), "r"(pk[4 * j + 2]), "r"(pk[4 * j + 3])
                             : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int rl = it * 4 + (lane >> 3), ck = lane & 7;
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(sb + (uint32_t)(rl * kEpiRowPitch + ck * 16))
                         : "memory");
            const int64_t row = row0 + h * 16 + rl;
            const int col = col0 + ck * kPer16;
            if (row < row_end && col < N) {
                uint4 *dst = reinterpret_cast<uint4 *>(D + row * ldd + col);
                if constexpr (ACC) {
                    const float4 p = *reinterpret_cast<const float4 *>(dst);
                    v.x = __float_as_uint(p.x + __uint_as_float(v.x));
                    v.y = __float_as_uint(p.y + __uint_as_float(v.y));
                    v.z = __float_as_uint(p.z + __uint_as_float(v.z));
                    v.w = __float_as_uint(p.w + __uint_as_float(v.w));
                }
                *dst = v;
            }
        }
        __syncwarp();   // the next pass overwrites the buffer
    }
}

namespace sm2 {
constexpr int EPI = 8;                 // epilogue warps 4..11 (warpgroups 1 and 2)
constexpr int THREADS = 12 * 32;       // warpgroup 0: producer (warp 0), MMA (warp 1), two idle warps
// The block-scaled pair kernel moves registers from warpgroup 0 to the
// epilogue warpgroups, which hold a 128-wide fp32 accumulator row per thread.  The split must
// not exceed the launch pool: 128 * 56 + 256 * 224 = 64512 = 384 * 168,
// so the kernel must launch at exactly 168 registers per thread (checked on
// the host before the first launch).
constexpr int REGS_LAUNCH = 168, REGS_LOW = 56, REGS_HIGH = 224;
static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= THREADS * REGS_LAUNCH, "register split exceeds the launch pool");
template <int BN>
struct Cfg {
    static constexpr int B_HALF = (BN / 2) * BK;
    static constexpr int STAGE = A_TILE + B_HALF;
    static constexpr int STAGES = (BN == 256) ? 6 : 8;
    static constexpr int NBUF = 512 / BN;
    static constexpr int NBARS = 2 * STAGES + 2 * NBUF + 2;   // + drain, + split partial written
    // epilogue store buffers (store_rows_coalesced), one per epilogue warp, 16-byte aligned
    static constexpr size_t EPI_OFF = ((size_t)STAGES * STAGE + NBARS * 8 + 16 + 15) & ~(size_t)15;
    static constexpr size_t SMEM = 1024 + EPI_OFF + (size_t)EPI * kEpiBufBytes;
};
// Split-K tail workspace: per split tile, per CTA of the pair, a 128 x 256
// fp32 partial stored column-major (row index fastest, so a warp's lanes write
// consecutive words), then one flag word per (tile, CTA).
constexpr size_t kSplitPartialFloats = 128 * 256;
}  // namespace sm2

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// 16-byte load from the shared memory of a CTA of this cluster (address from mapa_shared)
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Release of a TMEM buffer to the leader's MMA thread.  Relaxed: the TMEM
// loads it guards have already completed (tcgen05.wait::ld) and are ordered
// by tcgen05.fence::before_thread_sync; a release fence here would also wait
// for unrelated global loads and stores in flight (measured as the dominant
// "membar" stall of the block-scaled epilogue).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, uint32_t bar_cluster, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// arrive on the barrier at this shared offset in both CTAs of the pair
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)0x3)
        : "memory");
}
__device__ __forceinline__ void tc_commit_pair_self(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// ---------------------------------------------------------------- host ----
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over a [rows, K] FP8 matrix (row pitch K bytes), box 128 x box_rows,
// 128-byte swizzle; out-of-range boxes read zeros.
bool make_map(CUtensorMap *map, const void *base, int64_t K, int64_t rows, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
