// history.cu -- delayed-scaling amax-history update.
//
// Source: "DeepL押注FP8：大模型训练与推理统一精度实战解析" §2.3: delayed scaling
// predicts the current step's scale from the statistics of the previous steps,
// so no step waits on its own amax; when the current statistic deviates from
// the history beyond a threshold the scale is recomputed (§5.1: E5M2 overflow
// is the failure this guards against).  Reading taken here: the window
// statistic is the max over the ring, and the threshold is saturation, i.e.
// amax_t * s_t > fmax.
//
// One warp: the ring (<= 1024 entries) is reduced with a warp max; the whole
// update stays on the device, so a training step never syncs the host.
#include "common.cuh"

using namespace fp8q;

namespace {

template <int FMT>
__global__ void __launch_bounds__(32)
k_history(float *__restrict__ history, int32_t *__restrict__ pos, int len, const float *__restrict__ amax_cur,
          float *__restrict__ scale, float *__restrict__ scale_inv, uint32_t *__restrict__ saturated) {
    constexpr float fm = fmax_of<FMT>();
    const float a = *amax_cur;
    const float s_t = *scale;
    int p = *pos;
    if (p < 0 || p >= len) p = 0;   // a corrupted position restarts the ring
    __syncwarp();
    if (threadIdx.x == 0) history[p] = a;
    __syncwarp();
    uint32_t m = 0;   // non-negative floats compare as unsigned integers
    for (int i = threadIdx.x; i < len; i += 32) {
        const float h = history[i];
        const uint32_t b = h > 0.0f ? __float_as_uint(h) : 0u;
        m = b > m ? b : m;
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (threadIdx.x == 0) {
        *saturated = (__fmul_rn(a, s_t) > fm) ? 1u : 0u;
        *pos = (p + 1) % len;
        const float s = scale_from_amax(__uint_as_float(m), fm);
        *scale = s;
        *scale_inv = __fdiv_rn(1.0f, s);
    }
}

}  // namespace

using namespace fp8q_host;

extern "C" fp8_status fp8_amax_history_update(float *history, int32_t *pos, int len, const float *amax_cur,
                                              fp8_format fmt, float *scale, float *scale_inv,
                                              uint32_t *saturated, void *stream) {
    if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
    if (!history || !pos || !amax_cur || !scale || !scale_inv || !saturated) return FP8_ERR_INVALID_ARG;
    if (len < 1 || len > 1024) return FP8_ERR_SHAPE;
    int sms;
    fp8_status st = check_device(&sms);
    if (st != FP8_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (fmt == FP8_E4M3) k_history<FP8_E4M3><<<1, 32, 0, s>>>(history, pos, len, amax_cur, scale, scale_inv, saturated);
    else k_history<FP8_E5M2><<<1, 32, 0, s>>>(history, pos, len, amax_cur, scale, scale_inv, saturated);
    return cudaPeekAtLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}
