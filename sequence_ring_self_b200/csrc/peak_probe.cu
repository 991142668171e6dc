// peak_probe.cu -- throughput probes: the FP32 FMA rate (the denominator of the fp32 path's
// roofline) and HBM read-only and write-only streaming rates (context for the slab kernels,
// whose traffic is almost all writes (scores) or almost all reads (softmax/PV)).
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

// Streaming over a buffer far larger than L2: every thread moves four independent 16-byte
// vectors per iteration (grid-stride), so many requests are in flight per SM. Read: the loaded
// words are folded into one value, stored only in a case that never occurs. Write: a pattern
// derived from the address.
constexpr int kVec = 4;

__global__ void __launch_bounds__(256) hbm_read_kernel(const uint4 *buf, size_t n, uint32_t *out) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    uint32_t acc = 0;
    size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + (kVec - 1) * stride < n; i += kVec * stride) {
        uint4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) v[u] = __ldcs(buf + i + u * stride);
#pragma unroll
        for (int u = 0; u < kVec; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n; i += stride) {
        const uint4 v = __ldcs(buf + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == 0x9e3779b9u) out[blockIdx.x] = acc;
}

__global__ void __launch_bounds__(256) hbm_write_kernel(uint4 *buf, size_t n) {
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + (kVec - 1) * stride < n; i += kVec * stride) {
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const uint32_t w = static_cast<uint32_t>(i + u * stride);
            buf[i + u * stride] = make_uint4(w, w + 1u, w + 2u, w + 3u);
        }
    }
    for (; i < n; i += stride) {
        const uint32_t w = static_cast<uint32_t>(i);
        buf[i] = make_uint4(w, w + 1u, w + 2u, w + 3u);
    }
}

}  // namespace

extern "C" rsa_status_t rsa_probe_hbm(void *buf, size_t bytes, int write, int blocks, void *out,
                                      void *stream) {
    if (!buf || bytes == 0 || bytes % 16 != 0 || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 ||
        blocks <= 0 || (write != 0 && write != 1) || (!write && !out))
        return RSA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t n = bytes / 16;
    if (write)
        hbm_write_kernel<<<blocks, 256, 0, st>>>(static_cast<uint4 *>(buf), n);
    else
        hbm_read_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4 *>(buf), n,
                                                static_cast<uint32_t *>(out));
    return cudaGetLastError() == cudaSuccess ? RSA_OK : RSA_ERR_CUDA;
}

extern "C" long long rsa_probe_ffma_flops_per_thread(int iters) {
    return 2LL * kChains * kUnroll * static_cast<long long>(iters);
}

extern "C" rsa_status_t rsa_probe_ffma(void *out, int blocks, int iters, void *stream) {
    if (!out || blocks <= 0 || iters <= 0) return RSA_ERR_INVALID_ARG;
    ffma_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<float *>(out), iters, 0.999999f, 1e-7f);
    return cudaGetLastError() == cudaSuccess ? RSA_OK : RSA_ERR_CUDA;
}
