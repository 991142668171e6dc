// rsa_noalloc.cu -- rsa_forward for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc: code that runs under another runtime's
// memory manager (a framework or serving process that owns the whole device pool and forbids
// outside allocations), and latency-critical paths where a cudaMalloc / cudaFree could
// synchronise the device or fragment memory after start-up. rsa_forward needs a workspace;
// this variant takes it from a fixed scratch array that lives in the library's own device
// memory instead, so the caller passes only the inputs and outputs.
//
// The scratch array is a file-scope __device__ array of RSA_NOALLOC_SCRATCH_BYTES: every
// GPU that loads the library holds it until the process exits. Host code cannot use the
// array's name as a device address (on the host it names a stand-in), so the device address
// is looked up with cudaGetSymbolAddress once per device, with that device current, on the
// first call made on it.
#include <mutex>

#include "../../include/rsa.h"
#include "rsa_internal.h"

namespace {

constexpr size_t kScratchBytes = RSA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mutex;
void *g_scratch[kMaxDevices];  // device address of g_noalloc_scratch, per device

rsa_status_t scratch_of_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return rsa::record_cuda_failure("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return RSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return rsa::record_cuda_failure("cudaGetSymbolAddress(scratch)", e);
        if (!p) return RSA_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return RSA_OK;
}

}  // namespace

extern "C" rsa_status_t rsa_forward_noalloc(const void *Q, const void *K, const void *V, void *O,
                                            float *lse, int B, int H, int L, int d, int N,
                                            int causal, rsa_dtype_t dt, void *stream) {
    // the checks rsa_forward makes, in its order, so that both report the same code
    rsa_status_t st;
    if (!rsa::check_args(B, H, L, d, N, dt, &st)) return st;
    if (!Q || !K || !V || !O || !lse) return RSA_ERR_INVALID_ARG;
    for (const void *p : {static_cast<const void *>(Q), K, V, static_cast<const void *>(O),
                          static_cast<const void *>(lse)})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return RSA_ERR_INVALID_ARG;
    // the largest plan that fits the scratch
    const size_t need = rsa_workspace_size(B, H, L, d, N, causal, dt, 0, kScratchBytes);
    if (need > kScratchBytes) return RSA_ERR_WORKSPACE;  // even the smallest plan does not fit
    // an sm_100 device (and its context on this thread) before the scratch lookup
    st = rsa::check_device();
    if (st != RSA_OK) return st;
    void *scratch = nullptr;
    st = scratch_of_current_device(&scratch);
    if (st != RSA_OK) return st;
    return rsa_forward(Q, K, V, O, lse, B, H, L, d, N, causal, dt, scratch, kScratchBytes, stream);
}
