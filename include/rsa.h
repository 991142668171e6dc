/*
 * rsa.h -- C ABI of the Ring Self-Attention (RSA) library for NVIDIA B200 (sm_100a).
 *
 * What the library computes. "Sequence Parallelism: Making 4D Parallelism Possible" (Li, Xue
 * et al., 2021; review page, Abstract and "Proposed method") splits a sequence of length L into
 * N chunks and computes self-attention by passing attention embeddings around a ring of
 * devices (Ring Self-Attention). The pages give no formula; this library computes exact
 * softmax attention on the ring schedule, per (batch b, head h):
 *
 *   chunk n holds query rows [n*c, (n+1)*c), c = L/N;
 *   ring pass 1:  S_n[:, block m] = Q_n K_m^T / sqrt(d),  m = (n + s) mod N,  s = 0..N-1
 *   row softmax over the whole key length: P = exp(S - m_i) / l_i,  lse_i = m_i + ln l_i
 *   ring pass 2:  O_n = sum_s P_n[:, block m] V_m
 *
 * and the backward pass (dQ, dK, dV) on the same schedule. On one GPU the ring's ranks are
 * chunks resident in one HBM and a ring step is an order of tiles inside the kernels; the
 * result does not depend on N beyond floating-point rounding.
 *
 * Conventions shared by every call:
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are contiguous [B, H, L, d] (d fastest) in device
 *     memory, in the element type `dt` (RSA_BF16: bfloat16; RSA_F32: float). lse is fp32
 *     [B, H, L]. Base pointers must be 16-byte aligned.
 *   - scale = 1/sqrt(d) is fixed. causal != 0 keeps keys j <= i only (the diagonal is kept).
 *     No dropout, bias or padding mask.
 *   - Supported: B, H, L >= 1, N >= 1 with L % N == 0; bf16 with d in {64, 128}; fp32 with
 *     d in {32, 64}; L <= 2^22 and B * H * ceil(L / 128) < 2^30. L need not be a multiple of
 *     any tile size.
 *   - Arithmetic: bf16 inputs with fp32 accumulation and fp32 softmax statistics; P and dS
 *     are rounded to bf16 before their GEMMs; outputs are rounded to nearest-even into `dt`.
 *     The fp32 path computes every step in fp32 on the CUDA cores (no TF32).
 *   - Ownership: the caller owns every buffer, including `workspace`. The library never
 *     allocates or frees device memory at run time and never synchronises `stream` (a
 *     cudaStream_t; NULL means the legacy default stream). Work is enqueued on `stream` in
 *     order. The one piece of device memory the library holds itself is the fixed scratch
 *     array of rsa_forward_noalloc (see there), a static part of the library's device code.
 *   - Device: calls run on the calling thread's current CUDA device. Every pointer passed and
 *     `stream` must belong to that device; make it current (cudaSetDevice) first.
 *   - Errors: arguments are checked before anything is launched; a failed check returns an
 *     error code and enqueues nothing. Nothing throws across this interface.
 */
#ifndef RSA_H_
#define RSA_H_

#include <stddef.h>

#if defined(__GNUC__)
#define RSA_API __attribute__((visibility("default")))
#else
#define RSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RSA_OK = 0,
    RSA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, L % N != 0 */
    RSA_ERR_UNSUPPORTED = 2, /* head dim, dtype or size outside the supported set, no sm_100 GPU */
    RSA_ERR_WORKSPACE = 3,   /* workspace smaller than the minimum plan needs */
    RSA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    RSA_ERR_TIMEOUT = 5      /* a kernel's bounded wait ran out (reported afterwards) */
} rsa_status_t;

typedef enum { RSA_F32 = 0, RSA_BF16 = 1 } rsa_dtype_t;

/*
 * Bytes of device workspace a call needs.
 *
 * The score slab (the c x L block of scores of every chunk, i.e. L x L per head) is
 * processed in groups, one after the other in the same workspace: a group is a set of whole
 * heads, or, when a head does not fit, the same range of rows (a multiple of 128) of one or
 * several heads. On the bf16 forward the groups are rectangles of heads x 128-row tiles chosen
 * to fill whole rounds of the GPU's SMs: the softmax / ring-pass-2 kernel runs one unit
 * (head, 128-row tile) per CTA, so a group takes ceil(units / resident CTAs) rounds and the
 * plan takes the rectangles with the fewest rounds in total.
 * `budget_bytes` caps the workspace: the returned size is that of the plan chosen within the
 * budget (or of the smallest plan, one 128-row range of one head, if nothing fits).
 * budget_bytes == 0 asks for the default plan (at most 4 GiB).
 * for_backward selects the backward call's needs: on the bf16 path the backward keeps no
 * slab (every score tile is recomputed on the chip) and needs only the padded per-row
 * statistics, 8 * B * H * roundup(L, 64) bytes, whatever the budget; the fp32 path keeps fp32
 * P and dS slabs, grouped as above, plus the same statistics.
 * Returns 0 if the arguments are invalid or unsupported.
 */
RSA_API size_t rsa_workspace_size(int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                          int for_backward, size_t budget_bytes);

/*
 * Forward pass (ring pass 1, row softmax, ring pass 2).
 * In:  Q, K, V  [B,H,L,d] device, dtype dt.
 * Out: O [B,H,L,d] device, dtype dt; lse [B,H,L] fp32 device (the softmax statistics the
 *      backward pass needs; must not be NULL).
 * workspace: device, >= rsa_workspace_size(..., for_backward = 0, ...) for the plan wanted;
 *      the plan is the largest one that fits ws_bytes. 256-byte aligned.
 */
RSA_API rsa_status_t rsa_forward(const void *Q, const void *K, const void *V, void *O, float *lse,
                         int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * Slab-free forward: the same result as rsa_forward for bf16 (up to the rounding of P), without
 * a score slab. Pass 1 visits the ring's key blocks for every 128-row tile and keeps only each
 * row's running max and sum of exponentials (lse); pass 2 recomputes the score tiles on the
 * chip, forms P = exp(S - lse) there and accumulates O = P V. The recomputation follows the
 * pages' recomputation in the backward pass (second page, gradient checkpointing), applied to
 * the forward's two ring passes; the pages themselves keep the scores between the passes.
 * In:  Q, K, V [B,H,L,d] device bf16 (RSA_BF16 only; RSA_F32 gives RSA_ERR_UNSUPPORTED).
 * Out: O [B,H,L,d] bf16, lse [B,H,L] fp32 (as rsa_forward's, usable by rsa_backward).
 * No workspace: nothing but the inputs and outputs lives in device memory.
 */
RSA_API rsa_status_t rsa_forward_recompute(const void *Q, const void *K, const void *V, void *O,
                                           float *lse, int B, int H, int L, int d, int N,
                                           int causal, rsa_dtype_t dt, void *stream);

/*
 * Backward pass on the same ring schedule: recomputes P from Q, K and lse, forms
 * dP = dO V^T and dS = P * (dP - D) with D_i = dO_i . O_i, then
 * dV_m = sum_n P_n[:, block m]^T dO_n, dK_m = scale sum_n dS_n[:, block m]^T Q_n and
 * dQ_n = scale sum_s dS_n[:, block m] K_m. On the bf16 path the key-major sums (dV, dK) and
 * the query-major sum (dQ) run as two kernels that each recompute the score tiles they need.
 * In:  Q, K, V, O, dO [B,H,L,d] device dtype dt; lse [B,H,L] fp32 from rsa_forward.
 * Out: dQ, dK, dV [B,H,L,d] device dtype dt.
 * workspace: device, >= rsa_workspace_size(..., for_backward = 1, ...), 256-byte aligned.
 */
RSA_API rsa_status_t rsa_backward(const void *Q, const void *K, const void *V, const void *O,
                          const void *dO, const float *lse, void *dQ, void *dK, void *dV,
                          int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                          void *workspace, size_t ws_bytes, void *stream);

/* Human-readable name of a status code (static string). */
RSA_API const char *rsa_status_string(rsa_status_t status);

/*
 * What the most recent RSA_ERR_CUDA returned on the calling thread came from: the CUDA or
 * driver call that failed, its error name and code, and for a tensor-map encoding the shape
 * it was given. Thread-local storage owned by the library, valid until the thread's next
 * failing call; an empty string if there was none. Not part of the paper's method: a
 * diagnostic of this library.
 */
RSA_API const char *rsa_last_error(void);

/*
 * Status reported by kernels since the last call of this function on the current device:
 * RSA_OK, or RSA_ERR_TIMEOUT if a bounded wait inside a kernel gave up (that kernel then
 * returned early and its outputs are invalid). Synchronises `stream` and clears the status.
 */
RSA_API rsa_status_t rsa_last_device_status(void *stream);

/*
 * Posts `code` (RSA_OK or RSA_ERR_TIMEOUT) into the current device's status word from a
 * one-thread kernel on `stream`, exactly as a kernel whose bounded wait gave up records its
 * failure. A failure-injection hook for testing the reporting path (rsa_last_device_status
 * must then return the code and clear it) without making any wait run out. Not part of the
 * paper's method. RSA_ERR_INVALID_ARG for any other code.
 */
RSA_API rsa_status_t rsa_debug_report_status(int code, void *stream);

/*
 * The plan a call with these arguments and ws_bytes would use, for inspection:
 * out[0] = number of groups, out[1] = heads per group, out[2] = rows per group,
 * out[3] = padded row length of the slab (elements), out[4] = bytes the plan uses.
 * Returns RSA_ERR_WORKSPACE if ws_bytes is below the minimum plan.
 */
RSA_API rsa_status_t rsa_plan_describe(int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                               int for_backward, size_t ws_bytes, long long out[5]);

/*
 * Per-kernel timing, for benchmarks. While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on the launch's stream (an extra ~1 us per launch);
 * rsa_profile_read() waits for those events, adds their elapsed times per kernel kind into
 * ms[kind] and the launch counts into launches[kind] (arrays of rsa_profile_kinds() entries,
 * caller-owned, host memory), and forgets them. Events come from a pool owned by the
 * library. Enabling or disabling drops unread records. Not for use during stream capture.
 * Returns RSA_ERR_CUDA if an event call fails.
 */
RSA_API rsa_status_t rsa_profile_enable(int on);
RSA_API int rsa_profile_kinds(void);
RSA_API const char *rsa_profile_kind_name(int kind); /* NULL if out of range */
RSA_API rsa_status_t rsa_profile_read(double *ms, long long *launches);

/*
 * FP32 FMA throughput probe (a benchmark helper, not part of the method): the denominator of
 * the fp32 path's roofline, which runs on the CUDA cores. Launches `blocks` blocks of 256
 * threads on `stream`; every thread performs rsa_probe_ffma_flops_per_thread(iters) flops of
 * independent FMA chains. The caller times the launch (CUDA events on `stream`) and divides.
 * out: device buffer of at least `blocks` floats (written only in a case that never occurs,
 * so that the compiler keeps the work). Returns RSA_ERR_INVALID_ARG for a NULL buffer or
 * non-positive counts, RSA_ERR_CUDA if the launch fails.
 */
RSA_API rsa_status_t rsa_probe_ffma(void *out, int blocks, int iters, void *stream);
RSA_API long long rsa_probe_ffma_flops_per_thread(int iters);

/*
 * HBM streaming probe (a benchmark helper, not part of the method): context for the slab
 * kernels, whose traffic is almost all writes (the scores) or almost all reads (softmax/PV).
 * Launches `blocks` blocks of 256 threads on `stream` that read (write = 0) or write
 * (write = 1) every byte of `buf` once, in 16-byte vectors, four independent ones per thread
 * and iteration. The caller times the launch (CUDA events on `stream`) and divides `bytes` by
 * the time; `bytes` should be far above the L2 size (126 MB) so that the rate is HBM's.
 * buf: device buffer of `bytes` bytes, 16-byte aligned, bytes a positive multiple of 16; the
 * write probe fills it with a pattern (word k of 16-byte vector i holds i + k, modulo 2^32).
 * out: device buffer of at least `blocks` 32-bit words for the read probe (written only in a
 * case that never occurs, so that the compiler keeps the loads); may be NULL for the write
 * probe. Returns RSA_ERR_INVALID_ARG for a NULL or misaligned buffer, a size that is not a
 * positive multiple of 16, non-positive blocks, write not 0 or 1, or a read probe without
 * `out`; RSA_ERR_CUDA if the launch fails.
 */
RSA_API rsa_status_t rsa_probe_hbm(void *buf, size_t bytes, int write, int blocks, void *out,
                                   void *stream);

/* Size of the scratch array rsa_forward_noalloc works in: 32 MiB of device memory per GPU
 * that loads the library, held until the process exits. */
#define RSA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * rsa_forward for callers that cannot allocate device memory. No counterpart on the pages:
 * it exists for callers that may not call cudaMalloc, such as code running under another
 * runtime that owns the device memory pool, or latency-critical paths where an allocation
 * could synchronise the device. It computes exactly what rsa_forward computes (same
 * arguments, same outputs) but takes its workspace from a fixed scratch array of
 * RSA_NOALLOC_SCRATCH_BYTES inside the library, so the caller passes only inputs and outputs;
 * the slab is processed in as many groups as that scratch requires. It allocates nothing and
 * calls no allocating routine.
 * - Problems whose smallest plan does not fit the scratch (rows longer than about 64,000
 *   keys) are rejected with RSA_ERR_WORKSPACE before anything is launched.
 * - The scratch array is part of the library's device code, so it occupies device memory
 *   once the code module holding it is loaded on a device: under CUDA's default lazy module
 *   loading that happens at the first rsa_forward_noalloc call on the device (whose address
 *   lookup loads the module), with CUDA_MODULE_LOADING=EAGER when the library's context is
 *   created. It stays until the process exits.
 * - The first call on a device looks up the scratch array's device address on that device,
 *   after the same argument and device checks rsa_forward makes (so both entry points return
 *   the same codes for the same arguments); make that first call before any stream capture
 *   on the device.
 * - Every call on a device uses the same scratch array, and it keeps the last call's
 *   contents (nothing in it needs to start cleared: each call writes every byte it reads).
 *   Calls whose work overlaps on the GPU (for example on two streams without ordering
 *   between them) race on the scratch and give wrong results; order them on one stream or
 *   with events.
 */
RSA_API rsa_status_t rsa_forward_noalloc(const void *Q, const void *K, const void *V, void *O,
                                         float *lse, int B, int H, int L, int d, int N,
                                         int causal, rsa_dtype_t dt, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RSA_H_ */
