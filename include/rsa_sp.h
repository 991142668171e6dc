/*
 * rsa_sp.h -- the per-rank steps of sequence-parallel Ring Self-Attention across GPUs.
 *
 * "Sequence Parallelism: Making 4D Parallelism Possible" (Li, Xue et al., 2021; review page,
 * Abstract and "Proposed method", points 1-3 and 6) splits the sequence into chunks, one per
 * device, and runs self-attention as a ring: each device keeps its chunk's queries and passes
 * the key and value chunks to its neighbour, so that after P - 1 steps every device has seen
 * every chunk; the backward pass runs on the same ring, the partial key and value gradients
 * travelling with it. The companion review of "Maximizing Parallelism in Distributed Training
 * for Huge Neural Networks" (3-D tensor parallelism; its proposed-method list) names the
 * overlap of computation with communication as the way such rings hide their transfers.
 *
 * These entry points are the computation of one rank; the exchange (NCCL send/receive over
 * NVLink) and its overlap belong to the caller (the package's ring module). Rank r of P holds
 * the queries, keys and values of rows [r c, (r + 1) c), c = L / P, and, for the keys and
 * values, a full-length buffer Kfull / Vfull [B, H, L, d] into which the ring delivers the
 * other ranks' chunks (chunk m = rows [m c, (m + 1) c) of every head; each (b, h) slice of a
 * chunk is contiguous, so the ring moves it without a copy). One ring step on rank r:
 *
 *   forward, step s, key chunk m = (r + s) mod P present in Kfull:
 *       rsa_sp_scores          S_r[:, chunk m] = Q_r K_m^T / sqrt(d) (+ the window's softmax
 *                              partials) into the rank's score slab (ring pass 1)
 *   once every value chunk is in Vfull:
 *       rsa_sp_softmax_pv      row softmax over the whole key length, O_r = sum over the ring
 *                              of P_r[:, chunk m] V_m (ring pass 2), lse_r
 *   backward (Kfull, Vfull kept from the forward):
 *       rsa_sp_backward_rows   dQ_r (every key chunk), and the rows' statistics
 *       rsa_sp_backward_keys   this rank's contribution to dK_m, dV_m for one chunk m
 *       rsa_sp_accumulate      the travelling fp32 accumulator += that contribution
 *
 * Conventions (as in rsa.h unless stated): bf16 only (RSA_BF16), d in {64, 128}; L % P == 0
 * and c = L / P a multiple of 128; 0 <= rank, m < P. Local tensors Q, O, dO, dQ, dK/dV parts
 * are contiguous [B, H, c, d] bf16; lse is fp32 [B, H, c]; Kfull, Vfull are [B, H, L, d] bf16.
 * Pointers 16-byte aligned, workspace 256-byte aligned. The workspace of one rank (from
 * rsa_sp_workspace_size) holds its score slab [B H][c][L] fp32 with the softmax partials
 * (forward) or its rows' statistics (backward); the slab is the method's c x L block of
 * scores per head, so this workspace is what sequence parallelism distributes. Errors as in
 * rsa.h; causal steps whose whole window is masked (m > rank) launch nothing and return
 * RSA_OK (their contributions are zero: pass NULL to rsa_sp_accumulate for them).
 */
#ifndef RSA_SP_H_
#define RSA_SP_H_

#include "rsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Workspace bytes of one rank: forward (for_backward = 0): B H c L 4 bytes of scores plus
 * B H c (P * 2 * ceil(c / 256)) * 8 bytes of softmax partials; backward: 2 B H c 4 bytes of
 * row statistics. 0 for invalid or unsupported arguments. */
RSA_API size_t rsa_sp_workspace_size(int B, int H, int L, int d, int P, int causal,
                                     int for_backward);

/* Ring pass 1, one step: scores of this rank's rows against key chunk m (rows [m c, (m+1) c)
 * of Kfull) into the slab, with their per-row softmax partials. */
RSA_API rsa_status_t rsa_sp_scores(const void *Q, const void *Kfull, int B, int H, int L, int d,
                                   int P, int rank, int m, int causal, void *workspace,
                                   size_t ws_bytes, void *stream);

/* Row softmax over the full key length and ring pass 2 on this rank's rows, after every
 * rsa_sp_scores step of the forward has run: O [B,H,c,d], lse [B,H,c]; Vfull complete. */
RSA_API rsa_status_t rsa_sp_softmax_pv(const void *Vfull, void *O, float *lse, int B, int H,
                                       int L, int d, int P, int rank, int causal,
                                       void *workspace, size_t ws_bytes, void *stream);

/* dQ of this rank's rows over every key chunk (S and dP recomputed from Q, Kfull, Vfull and
 * lse), and the rows' statistics (lse log2 e, D = dO . O) that rsa_sp_backward_keys reads,
 * written into the backward workspace. */
RSA_API rsa_status_t rsa_sp_backward_rows(const void *Q, const void *Kfull, const void *Vfull,
                                          const void *O, const void *dO, const float *lse,
                                          void *dQ, int B, int H, int L, int d, int P, int rank,
                                          int causal, void *workspace, size_t ws_bytes,
                                          void *stream);

/* This rank's rows' contribution to the gradients of key chunk m: dK_part = scale sum_i
 * dS_im Q_i, dV_part = sum_i P_im dO_i over the rank's rows i, bf16 [B,H,c,d]. Runs after
 * rsa_sp_backward_rows on the same workspace. */
RSA_API rsa_status_t rsa_sp_backward_keys(const void *Q, const void *Kfull, const void *Vfull,
                                          const void *dO, void *dK_part, void *dV_part, int B,
                                          int H, int L, int d, int P, int rank, int m,
                                          int causal, void *workspace, size_t ws_bytes,
                                          void *stream);

/* The travelling accumulator of the backward ring: acc[i] = (first ? 0 : acc[i]) + part[i]
 * for n elements (acc fp32, part bf16; part == NULL adds zero); when out != NULL, also
 * out[i] = acc[i] rounded to bf16 (the last step). */
RSA_API rsa_status_t rsa_sp_accumulate(float *acc, const void *part, void *out, long long n,
                                       int first, void *stream);

/*
 * The block's linear layers on a rank's rows (the rest of the block needs no exchange under
 * sequence parallelism: review page, Abstract). On M rows:
 *
 *   Y[m][n] = act( sum_k X[m][k] W[n][k] + bias[n] ) + R[m][n]
 *
 * act = exact GELU (x Phi(x)) when gelu != 0, else the identity. bf16 operands, fp32
 * accumulation on the tensor cores, bf16 output rounded to nearest-even.
 * X: bf16, the row-major [M][K] matrix stored as [K / x_kin][M][x_kin] (x_kin = K: a plain
 *    row-major X; x_kin = d: the [H][M][d] output of attention, read as [M][H d]).
 * W: bf16 [N][K] row-major (out x in). bias: fp32 [N] or NULL. R: bf16 [M][N] or NULL
 *    (residual; only with y_kin == N).
 * Y: bf16, the [M][N] result stored as [N / y_kin][M][y_kin] (y_kin = N: plain; y_kin = d: the
 *    query/key/value projection written straight into [3 H][M][d] for attention).
 * Supported: M % 128 == 0, N % 64 == 0, K % 64 == 0, x_kin % 64 == 0 dividing K, y_kin % 32 ==
 * 0 dividing N; RSA_ERR_UNSUPPORTED otherwise. Pointers 16-byte aligned. Errors as in rsa.h.
 */
RSA_API rsa_status_t rsa_linear(const void *X, const void *W, const float *bias, const void *R,
                                void *Y, int M, int N, int K, int x_kin, int y_kin, int gelu,
                                void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RSA_SP_H_ */
