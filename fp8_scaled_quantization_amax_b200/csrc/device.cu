// device.cu -- device check and status strings shared by every entry point.
#include <mutex>

#include "common.cuh"

namespace fp8q_host {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_state[kMaxDevices];   // 0 unknown, 1 supported, 2 unsupported
int g_sms[kMaxDevices];
}  // namespace

fp8_status check_device(int *sm_count) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return FP8_ERR_CUDA;
    if (dev >= kMaxDevices) return FP8_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_state[dev] == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FP8_ERR_CUDA;
        g_state[dev] = (major == 10 && minor == 0) ? 1 : 2;
        g_sms[dev] = sms;
    }
    if (g_state[dev] != 1) return FP8_ERR_UNSUPPORTED_DEVICE;
    if (sm_count) *sm_count = g_sms[dev];
    return FP8_OK;
}

}  // namespace fp8q_host

extern "C" const char *fp8_status_string(fp8_status s) {
    switch (s) {
        case FP8_OK: return "FP8_OK";
        case FP8_ERR_INVALID_ARG: return "FP8_ERR_INVALID_ARG: null pointer or bad enum value";
        case FP8_ERR_SHAPE: return "FP8_ERR_SHAPE: negative or unsupported extent";
        case FP8_ERR_ALIGNMENT: return "FP8_ERR_ALIGNMENT: pointer or leading dimension not aligned";
        case FP8_ERR_UNSUPPORTED_DEVICE: return "FP8_ERR_UNSUPPORTED_DEVICE: needs compute capability 10.0 (sm_100a)";
        case FP8_ERR_CUDA: return "FP8_ERR_CUDA: a CUDA runtime call failed";
    }
    return "FP8_ERR_UNKNOWN";
}
