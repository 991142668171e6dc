// peak_probe.cu -- FP32 FMA throughput probe, the denominator of the fp32 path's roofline.
//
// The fp32 path of the library runs every step of the attention on the CUDA cores (no tensor
// cores, no TF32), so its kernels are bounded by the FP32 FMA rate of the GPU. The vendor's
// nominal rate assumes the maximum clock; this kernel measures the rate the GPU actually
// delivers: every thread runs kChains independent FMA chains (enough to cover the FMA latency
// with several warps per scheduler), so the only limit is the FMA pipe's issue rate.
// Not part of the method: a measurement helper for benchmarks.
#include "../../include/rsa.h"
#include "rsa_internal.h"

namespace {

constexpr int kChains = 16;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(256) ffma_probe_kernel(float *out, int iters, float mul, float add) {
    float x[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) x[k] = static_cast<float>(threadIdx.x) * 1e-3f + k;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
#pragma unroll
            for (int k = 0; k < kChains; ++k) x[k] = fmaf(x[k], mul, add);
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += x[k];
    // a store the compiler cannot prove dead, taken (almost) never
    if (s == 1234.5f) out[blockIdx.x] = s;
}

}  // namespace

extern "C" long long rsa_probe_ffma_flops_per_thread(int iters) {
    return 2LL * kChains * kUnroll * static_cast<long long>(iters);
}

extern "C" rsa_status_t rsa_probe_ffma(void *out, int blocks, int iters, void *stream) {
    if (!out || blocks <= 0 || iters <= 0) return RSA_ERR_INVALID_ARG;
    ffma_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<float *>(out), iters, 0.999999f, 1e-7f);
    return cudaGetLastError() == cudaSuccess ? RSA_OK : RSA_ERR_CUDA;
}
