// rsa_internal.h -- shared declarations between the C-ABI front end and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/rsa.h"

namespace rsa {

// ---- checks shared by the entry points (rsa_abi.cu) --------------------------------------
// Argument checks of every forward/backward entry point: sizes, divisibility, supported head
// dimension and dtype. On failure returns false and sets *why.
bool check_args(int B, int H, int L, int d, int N, rsa_dtype_t dt, rsa_status_t *why);
// Binds the current device's primary context on the calling thread and checks once per device
// that it is an sm_100 GPU (RSA_ERR_UNSUPPORTED otherwise); configures the kernels.
rsa_status_t check_device();
// Records which CUDA call failed (read back by rsa_last_error) and returns RSA_ERR_CUDA.
rsa_status_t record_cuda_failure(const char *what, cudaError_t e);

// Launch with programmatic stream serialisation: the kernel may start (and run its prologue)
// while the previous kernel in the stream finishes; it calls pdl_wait() before touching memory
// the previous kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// One group of the slab schedule: heads [bh0, bh0 + nh) and, inside each of them, the query
// rows [r0, r0 + R). The group's score slab lives in the workspace as [nh][R][Lp].
struct Group {
    int bh0, nh;
    int r0, R;
    int first_of_head;  // row-range groups: this group starts a head
    int last_of_head;   // row-range groups: this group ends a head
};

// Arguments every slab kernel shares.
struct SlabArgs {
    int L, Lp, N, c, causal, d;
    int bh0, nh, r0, R;
    float scale;
    int nRT;     // 128-row tiles per head in the group
    int nCT;     // column tiles per head (kernel-specific width)
    int ntiles;  // tiles in the launch (before causal skipping)
    int mode;    // kernel-specific (see each kernel)
    int nStat;      // forward: per-row softmax partials (one per 128 key columns)
    float2 *stats;  // forward: [nh][R][nStat] (max, sum of 2^(s - max)) in base-2 units
    int *status; // device status word
    // Views of a sequence-parallel rank (the defaults, in brackets, give the whole problem):
    int qrow0;   // first query row held: Q, O, dO, dQ and lse are stored at row i - qrow0 [0]
    int Lq;      // rows per head of that storage [L]
    int Lpq;     // rows per head of the backward's row statistics (padded to 64) [Lp]
    int kcol0;   // key window [kcol0, kend) of ring pass 1 and of the key-major backward [0]
    int kend;    // [L]
    int wlen;    // keys per window of the softmax partials' layout [L]
    int stat0;   // first softmax-partial slot of this window [0]
};

// ---- bf16 tensor-core kernels (kernels_tc.cu) -------------------------------------------
// Each returns a cudaError_t of its launch.
cudaError_t launch_qk_slab(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mS,
                           const SlabArgs &a, int num_sms, cudaStream_t st);
// Row softmax and ring pass 2: P = 2^(S - m) / l from the fp32 slab (mS: 32 x 128 boxes,
// 128-byte swizzle) and the partials in a.stats, O = P V (mV: 64 x 64 boxes; mO: [BH][L][d]
// bf16, 32 x 32 boxes, 64-byte swizzle, store); writes lse of the group's rows.
cudaError_t launch_pv_softmax(const CUtensorMap &mS, const CUtensorMap &mV, const CUtensorMap &mO,
                              float *lse, const SlabArgs &a, int num_sms, cudaStream_t st);
// Key-major backward: recompute P^T, dP^T -> dS^T in TMEM, and dV = P^T dO, dK = scale dS^T Q
// accumulated in TMEM over the group's query blocks.
// mStat: the padded row statistics [2][BH][Lp] fp32 (lse * log2(e), then D), box 64 x 1 x 1.
// mdK/mdV: [BH][L][d] bf16, 32 x 32 boxes, 64-byte swizzle (store).
cudaError_t launch_bwd_keys(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mQ,
                            const CUtensorMap &mdO, const CUtensorMap &mStat,
                            const CUtensorMap &mdK, const CUtensorMap &mdV, const SlabArgs &a,
                            int num_sms, cudaStream_t st);
// Row-major backward: recompute S, dP -> dS in TMEM per 128-query tile and dQ = scale dS K;
// forms D_i = dO_i . O_i and writes lse_i log2(e) and D_i to lse2_out / d_out ([BH][Lp] each,
// zero past L) for launch_bwd_keys, which must run after it.
// mQ/mdO/mO: 64 x 128 boxes; mK/mV: 64 x 128 boxes for d = 64, 64 x 64 for d = 128 (the key
// block of a step); mdQ: [BH][L][d] bf16, 32 x 32 boxes, 64-byte swizzle (store);
// lse: [BH][L] fp32 from the forward pass.
cudaError_t launch_bwd_rows(const CUtensorMap &mQ, const CUtensorMap &mdO, const CUtensorMap &mO,
                            const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mdQ,
                            const float *lse, float *lse2_out, float *d_out, const SlabArgs &a,
                            int num_sms, cudaStream_t st);
// Slab-free two-pass forward (kernels_fwd.cu), whole problem in one launch each, units of
// 128 query rows: pass 1 writes lse; pass 2 recomputes S, forms P on the chip and writes O.
// mQ: 64 x 128 boxes; mK/mV: 64 x KN boxes (KN = 128 keys for d = 64, 64 for d = 128);
// mO: as for launch_pv_softmax.
cudaError_t launch_fwd_stats(const CUtensorMap &mQ, const CUtensorMap &mK, float *lse,
                             const SlabArgs &a, int num_sms, cudaStream_t st);
cudaError_t launch_fwd_pv(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                          const CUtensorMap &mO, const float *lse, const SlabArgs &a, int num_sms,
                          cudaStream_t st);
cudaError_t fwd_kernels_configure();
cudaError_t tc_kernels_configure();  // opt-in shared memory sizes (once per device)
cudaError_t bwd_kernels_configure();

// ---- the block's linear layers (kernels_linear.cu) ----------------------------------------
// Y = act(X W^T + b) + R on M rows. X is read as (x_kin, M, K / x_kin) and Y written as
// (y_kin, M, N / y_kin) bf16 tensors (a plain row-major matrix has x_kin = K / y_kin = N).
struct LinArgs {
    int M, N, K;
    int x_kin, y_kin;
    int gelu;
    const float *bias;           // [N] or null
    const __nv_bfloat16 *res;    // [M][N] row-major or null
    int ntiles, nNT;             // (M / 128) x ceil(N / 256) tiles; nNT = ceil(N / 256)
    int *status;
};
cudaError_t launch_linear(const CUtensorMap &mX, const CUtensorMap &mW, const CUtensorMap &mY,
                          const LinArgs &a, int num_sms, cudaStream_t st);
cudaError_t linear_kernels_configure();

// ---- CUDA-core kernels (kernels_simt.cu) -----------------------------------------------
// Row softmax of the group's fp32 slab, in place: P written as bf16 (p_bf16 = 1) into the
// first half of each fp32 row, or as fp32 over S (p_bf16 = 0). Writes lse. Natural-unit
// scores, statistics computed here (the fp32 path).
cudaError_t launch_slab_softmax(float *slab, float *lse, const SlabArgs &a, int p_bf16,
                                cudaStream_t st);
// D_i = dO_i . O_i (and lse2 = lse * log2(e) when lse2 != NULL) for all rows of all heads,
// written in rows padded to Lp with zeros past L.
cudaError_t launch_rowdot(const void *dO, const void *O, const float *lse, float *Dp,
                          float *lse2, long long BH, int L, int Lp, int d, int bf16,
                          cudaStream_t st);
// fp32 path (every step in fp32 FMA).
cudaError_t launch_f32_qk_slab(const float *Q, const float *K, float *S, const SlabArgs &a,
                               cudaStream_t st);
cudaError_t launch_f32_ring_rows(const float *A, const float *Bm, float *out, const SlabArgs &a,
                                 cudaStream_t st);
cudaError_t launch_f32_bwd_slab(const float *Q, const float *K, const float *dO, const float *V,
                                const float *lse, const float *Dvec, float *P, float *dS,
                                const SlabArgs &a, cudaStream_t st);
cudaError_t launch_f32_ring_keys(const float *A, const float *Bm, float *out, float alpha,
                                 int accumulate, const SlabArgs &a, cudaStream_t st);

}  // namespace rsa
