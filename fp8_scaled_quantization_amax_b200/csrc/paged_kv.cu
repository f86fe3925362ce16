// paged_kv.cu -- paged FP8 KV cache: write new tokens into fixed-size blocks,
// read sequences back through their block tables.
//
// Sources: "ms-swift全链路能力解析：训练、推理、评测、量化与部署一体化解决方案" (vLLM's KV
// cache cut into fixed-size blocks handed out on demand) and
// "DeepL押注FP8：大模型训练与推理统一精度实战解析" §3.1 (K and V stored in
// FP8 halve the cache, dequantized when attention reads them).  Reading taken
// here: tokens arrive a few at a time, so each (token, head) row of Dh
// elements carries its own scale s = fmax / amax(row), stored as 1/s beside
// the codes.
//
// Layout: cache [num_blocks, block_size, H, Dh] FP8 = [num_slots, H, Dh] with
// slot = block * block_size + offset, so one token's H*Dh codes are
// contiguous; scale_cache [num_slots, H] fp32.
//
// Write: a CTA takes kTok tokens; thread c owns elements [8c, 8c + 8) of every
// one of them (one 16-byte load per token, all kTok in flight together).  A
// head spans G = Dh/8 consecutive threads: for head sizes 64, 128 and 256
// its amax is an unrolled shuffle reduction inside the group, otherwise a
// shared-memory max.  The kTok x H scales are then computed once each, by one thread per
// (token, head) -- the correctly rounded divisions are the costliest step of
// the kernel, and issuing them per 8-element chunk made it issue-bound --
// and read back from shared memory for the cast.  The codes leave as one
// 8-byte store per thread and token.
#include "common.cuh"

using namespace fp8q;

namespace {

constexpr int kTok = 4;
constexpr int kMaxRowElems = 8192;          // H * Dh per token
constexpr int kMaxThreads = kMaxRowElems / 8;

// G = Dh / 8 threads per head.  GS = G when G is 8, 16 or 32 (head sizes 64,
// 128, 256: the group reduction is an unrolled shuffle and the head index a
// shift), GS = 0 otherwise (a shared-memory max, runtime division).
// Dynamic shared memory: kTok * H uint32 head amax + kTok * H fp32 scales.
template <int FMT, int GS>
__global__ void __launch_bounds__(kMaxThreads)
k_paged_write(const uint4 *__restrict__ x, const int64_t *__restrict__ slot_mapping, int64_t T, int H,
              int G_rt, int64_t num_slots, uint2 *__restrict__ cache, float *__restrict__ scale_cache) {
    constexpr bool SHFL = GS > 0;
    const int G = SHFL ? GS : G_rt;
    constexpr float fm = fmax_of<FMT>();
    extern __shared__ uint32_t sm_paged[];
    uint32_t *head_amax = sm_paged;                                   // [kTok][H]
    float *head_scale = reinterpret_cast<float *>(sm_paged + kTok * H);   // [kTok][H]
    const int C = H * G;                                 // 8-element chunks per token
    const int c = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * kTok;
    int64_t slot[kTok];
    uint4 v[kTok];
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
        const int64_t t = t0 + k;
        // the row is read whether or not the token is padding, so the loads
        // of x do not wait for the slot ids
        slot[k] = t < T ? slot_mapping[t] : -1;
        v[k] = (t < T && c < C) ? ld_stream(x + t * C + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kTok; ++k)
        if (slot[k] >= num_slots) slot[k] = -1;          // outside the cache: padding
    if constexpr (!SHFL) {
        for (int i = threadIdx.x; i < kTok * H; i += blockDim.x) head_amax[i] = 0u;
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
        uint32_t m = amax_fast_final(amax_fast8(0u, v[k]));
        if (m == 0xFFFFFFFFu) {   // a NaN or Inf among the eight: the exact, skipping form
            uint32_t bad = 0;
            m = amax_exact8(0u, v[k], bad);
        }
        if constexpr (SHFL) {
#pragma unroll
            for (int o = GS >> 1; o > 0; o >>= 1) {
                const uint32_t w = __shfl_xor_sync(0xFFFFFFFFu, m, o);
                m = w > m ? w : m;
            }
            if (c < C && (c & (GS - 1)) == 0) head_amax[k * H + c / GS] = m;
        } else if (c < C) {
            atomicMax(&head_amax[k * H + c / G], m);
        }
    }
    __syncthreads();
    // one thread per (token, head): the scale, and 1/s into the cache
    for (int i = threadIdx.x; i < kTok * H; i += blockDim.x) {
        const int k = i / H, h = i - k * H;
        const float s = scale_from_amax(bf16bits_to_float(head_amax[i]), fm);
        head_scale[i] = s;
        const int64_t t = t0 + k;
        if (t < T) {
            const int64_t sl = slot_mapping[t];
            if (sl >= 0 && sl < num_slots) scale_cache[sl * H + h] = __fdiv_rn(1.0f, s);
        }
    }
    __syncthreads();
    if (c >= C) return;
    const int h = c / G;
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
        if (slot[k] < 0) continue;
        cache[slot[k] * C + c] = cast8<FMT>(v[k], head_scale[k * H + h]);
    }
}

// Eight FP8 codes -> eight bf16, each bf16_RNE(fp32(code) * d).
template <int FMT>
__device__ __forceinline__ uint4 dequant8(uint2 q, float d) {
    const uint32_t w[2] = {q.x, q.y};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float2 lo = fp8x2_to_float2<FMT>((uint16_t)(w[i] & 0xFFFFu));
        const float2 hi = fp8x2_to_float2<FMT>((uint16_t)(w[i] >> 16));
        o[2 * i] = pack_bf16x2(__fmul_rn(lo.x, d), __fmul_rn(lo.y, d));
        o[2 * i + 1] = pack_bf16x2(__fmul_rn(hi.x, d), __fmul_rn(hi.y, d));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int FMT>
__global__ void __launch_bounds__(kMaxThreads)
k_paged_gather(const uint2 *__restrict__ cache, const float *__restrict__ scale_cache,
               const int32_t *__restrict__ block_table, const int32_t *__restrict__ seq_lens, int64_t max_blocks,
               int H, int G, int64_t block_size, int64_t num_blocks, int64_t S_out, uint4 *__restrict__ out) {
    const int C = H * G;
    const int c = threadIdx.x;
    if (c >= C) return;
    const int64_t b = blockIdx.y;
    const int64_t t0 = (int64_t)blockIdx.x * kTok;
    const int64_t len = seq_lens[b];
    const int h = c / G;
    int64_t slot[kTok];
    uint2 q[kTok];
    float d[kTok];
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
        const int64_t t = t0 + k;
        int64_t blk = -1;
        if (t < S_out && t < len && t / block_size < max_blocks) blk = block_table[b * max_blocks + t / block_size];
        slot[k] = (blk >= 0 && blk < num_blocks) ? blk * block_size + t % block_size : -1;
        q[k] = slot[k] >= 0 ? ld_stream_u2(cache + slot[k] * C + c) : make_uint2(0, 0);
        d[k] = slot[k] >= 0 ? scale_cache[slot[k] * H + h] : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kTok; ++k) {
        const int64_t t = t0 + k;
        if (t >= S_out) break;
        out[(b * S_out + t) * C + c] = slot[k] >= 0 ? dequant8<FMT>(q[k], d[k]) : make_uint4(0, 0, 0, 0);
    }
}

}  // namespace

using namespace fp8q_host;

static fp8_status paged_shape(int64_t H, int64_t Dh) {
    if (H < 1 || Dh < 8 || Dh % 8 || H * Dh > kMaxRowElems) return FP8_ERR_SHAPE;
    return FP8_OK;
}

static int paged_threads(int64_t H, int64_t Dh) { return (int)(((H * Dh / 8) + 31) / 32 * 32); }

extern "C" fp8_status fp8_paged_kv_write(const void *kv_bf16, const int64_t *slot_mapping, int64_t T, int64_t H,
                                         int64_t Dh, int64_t num_slots, fp8_format fmt, uint8_t *cache,
                                         float *scale_cache, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (T < 0 || num_slots < 0) return FP8_ERR_SHAPE;
    fp8_status st = paged_shape(H, Dh);
    if (st != FP8_OK) return st;
    if (T == 0) return FP8_OK;
    if (!kv_bf16 || !slot_mapping || !cache || !scale_cache) return FP8_ERR_INVALID_ARG;
    if (!aligned16(kv_bf16) || !aligned16(cache)) return FP8_ERR_ALIGNMENT;
    if ((T + kTok - 1) / kTok > 0x7FFFFFFFll) return FP8_ERR_SHAPE;
    int sms;
    st = check_device(&sms);
    if (st != FP8_OK) return st;
    const int G = (int)(Dh / 8);
    const dim3 grid((unsigned)((T + kTok - 1) / kTok));
    const int thr = paged_threads(H, Dh);
    cudaStream_t s = as_stream(stream);
    const uint4 *x = (const uint4 *)kv_bf16;
    uint2 *q = (uint2 *)cache;
    const size_t sm = (size_t)kTok * H * 8;   // <= 32 KiB (H <= 1024)
#define FP8Q_PAGED_WRITE(F, GS) \
    k_paged_write<F, GS><<<grid, thr, sm, s>>>(x, slot_mapping, T, (int)H, G, num_slots, q, scale_cache)
    if (fmt == FP8_E4M3) {
        if (G == 16) FP8Q_PAGED_WRITE(FP8_E4M3, 16);
        else if (G == 8) FP8Q_PAGED_WRITE(FP8_E4M3, 8);
        else if (G == 32) FP8Q_PAGED_WRITE(FP8_E4M3, 32);
        else FP8Q_PAGED_WRITE(FP8_E4M3, 0);
    } else {
        if (G == 16) FP8Q_PAGED_WRITE(FP8_E5M2, 16);
        else if (G == 8) FP8Q_PAGED_WRITE(FP8_E5M2, 8);
        else if (G == 32) FP8Q_PAGED_WRITE(FP8_E5M2, 32);
        else FP8Q_PAGED_WRITE(FP8_E5M2, 0);
    }
#undef FP8Q_PAGED_WRITE
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" fp8_status fp8_paged_kv_gather(const uint8_t *cache, const float *scale_cache,
                                          const int32_t *block_table, const int32_t *seq_lens, int64_t B,
                                          int64_t max_blocks, int64_t H, int64_t Dh, int64_t block_size,
                                          int64_t num_blocks, int64_t S_out, fp8_format fmt, void *out_bf16,
                                          void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (B < 0 || max_blocks < 0 || block_size < 1 || num_blocks < 0 || S_out < 0) return FP8_ERR_SHAPE;
    fp8_status st = paged_shape(H, Dh);
    if (st != FP8_OK) return st;
    if (B == 0 || S_out == 0) return FP8_OK;
    if (B > 65535 || (S_out + kTok - 1) / kTok > 0x7FFFFFFFll) return FP8_ERR_SHAPE;
    if (!seq_lens || !out_bf16 || (max_blocks > 0 && !block_table)) return FP8_ERR_INVALID_ARG;
    if (num_blocks > 0 && (!cache || !scale_cache)) return FP8_ERR_INVALID_ARG;
    if (!aligned16(out_bf16) || (cache && !aligned16(cache))) return FP8_ERR_ALIGNMENT;
    int sms;
    st = check_device(&sms);
    if (st != FP8_OK) return st;
    const int G = (int)(Dh / 8);
    const dim3 grid((unsigned)((S_out + kTok - 1) / kTok), (unsigned)B);
    const int thr = paged_threads(H, Dh);
    cudaStream_t s = as_stream(stream);
    const uint2 *q = (const uint2 *)cache;
    uint4 *o = (uint4 *)out_bf16;
    if (fmt == FP8_E4M3)
        k_paged_gather<FP8_E4M3><<<grid, thr, 0, s>>>(q, scale_cache, block_table, seq_lens, max_blocks, (int)H, G,
                                                      block_size, num_blocks, S_out, o);
    else
        k_paged_gather<FP8_E5M2><<<grid, thr, 0, s>>>(q, scale_cache, block_table, seq_lens, max_blocks, (int)H, G,
                                                      block_size, num_blocks, S_out, o);
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
