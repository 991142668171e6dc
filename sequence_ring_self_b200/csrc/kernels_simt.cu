// kernels_simt.cu -- CUDA-core kernels of Ring Self-Attention.
//
//  * slab_softmax: the row softmax over the full key length that sits between the two ring
//    passes of the fp32 path ("Sequence Parallelism: Making 4D Parallelism Possible", review
//    page, "Proposed method": attention is computed chunk by chunk with the keys passed
//    around the ring). Each row of the fp32 score slab is read once with 16-byte loads and
//    held in registers; max and sum use warp shuffles (plus shared memory across the row's
//    warps). P is written in place over the scores. (The bf16 path forms P inside its ring
//    pass 2 kernel instead.)
//  * rowdot: D_i = dO_i . O_i for the fp32 backward pass.
//  * f32_*: the fp32 path, every step in fp32 FMA on the CUDA cores (no TF32), on the same
//    slab layout and ring order as the tensor-core path.
#include <cuda_bf16.h>

#include "rsa_internal.h"
#include "sm100_ptx.cuh"

namespace rsa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Causal rows read and write the slab up to the end of their 128-row tile's diagonal block
// (what the ring-pass-2 GEMM reads); other rows the whole padded row.
__device__ __forceinline__ int live_end(const SlabArgs &a, int i) {
    return a.causal ? min(a.Lp, (i / 128) * 128 + 128) : a.Lp;
}

// One row per 32*WPR threads; each thread holds EPT values (EPT/4 float4 loads).
template <int EPT, bool P_BF16>
__global__ void __launch_bounds__(1024)
    slab_softmax_kernel(float *__restrict__ slab, float *__restrict__ lse, const SlabArgs a,
                        int wpr) {
    pdl_wait();
    pdl_trigger();
    __shared__ float red_max[32];
    __shared__ float red_sum[32];
    const int tpr = 32 * wpr;
    const int rows_per_cta = blockDim.x / tpr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = threadIdx.x / tpr;          // row group inside the CTA
    const int tr = threadIdx.x - grp * tpr;     // thread inside the row
    const long long rid = static_cast<long long>(blockIdx.x) * rows_per_cta + grp;
    const long long nrows = static_cast<long long>(a.nh) * a.R;
    const bool active = rid < nrows;
    int h = 0, il = 0, i = 0, end = 0;
    if (active) {
        h = static_cast<int>(rid / a.R);
        il = static_cast<int>(rid - static_cast<long long>(h) * a.R);
        i = a.r0 + il;
        end = live_end(a, i);
    }
    float *row = slab + (static_cast<size_t>(h) * a.R + il) * a.Lp;

    float v[EPT];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < EPT / 4; ++u) {
        const int f = tr + tpr * u;
        float4 x = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (active && 4 * f < end) x = reinterpret_cast<const float4 *>(row)[f];
        v[4 * u] = x.x;
        v[4 * u + 1] = x.y;
        v[4 * u + 2] = x.z;
        v[4 * u + 3] = x.w;
        m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
    }
    m = warp_max(m);
    if (wpr > 1) {
        if (lane == 0) red_max[warp] = m;
        __syncthreads();
        m = -INFINITY;
        for (int w = 0; w < wpr; ++w) m = fmaxf(m, red_max[grp * wpr + w]);
    }
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
        float x;
        if (P_BF16)
            x = v[e] == -INFINITY ? 0.f : exp2f((v[e] - m) * kLog2e);
        else
            x = v[e] == -INFINITY ? 0.f : expf(v[e] - m);
        v[e] = x;
        s += x;
    }
    s = warp_sum(s);
    if (wpr > 1) {
        if (lane == 0) red_sum[warp] = s;
        __syncthreads();
        s = 0.f;
        for (int w = 0; w < wpr; ++w) s += red_sum[grp * wpr + w];
    } else {
        __syncwarp();
    }
    if (!active) return;
    const float inv = 1.f / s;
    if (tr == 0) lse[static_cast<size_t>(a.bh0 + h) * a.L + i] = m + logf(s);
#pragma unroll
    for (int u = 0; u < EPT / 4; ++u) {
        const int f = tr + tpr * u;
        if (4 * f >= end) continue;
        const float p0 = v[4 * u] * inv, p1 = v[4 * u + 1] * inv;
        const float p2 = v[4 * u + 2] * inv, p3 = v[4 * u + 3] * inv;
        if (P_BF16) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(p0, p1);
            __nv_bfloat162 hi = __floats2bfloat162_rn(p2, p3);
            uint2 w;
            w.x = *reinterpret_cast<uint32_t *>(&lo);
            w.y = *reinterpret_cast<uint32_t *>(&hi);
            reinterpret_cast<uint2 *>(row)[f] = w;
        } else {
            reinterpret_cast<float4 *>(row)[f] = make_float4(p0, p1, p2, p3);
        }
    }
}

// Row statistics for the backward pass, in rows padded to Lp (zeros past L):
//   D[bh][i] = dO_i . O_i  and, if lse2 is given, lse2[bh][i] = lse[bh][i] * log2(e).
// The flattened [rows][D] inputs are read as 16-byte vectors: vector t holds elements
// [8t, 8t + 8) (bf16) or [4t, 4t + 4) (fp32), so TPR = D / (elements per vector) consecutive
// threads share a row and reduce with shuffles. Warps stride in lockstep.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    rowdot_kernel(const uint4 *__restrict__ dO, const uint4 *__restrict__ O,
                  const float *__restrict__ lse, float *__restrict__ Dp, float *__restrict__ lse2,
                  long long BH, int L, int Lp) {
    pdl_wait();
    pdl_trigger();
    constexpr int EPV = BF16 ? 8 : 4;
    constexpr int TPR = D / EPV;
    constexpr int U = 4;  // vectors in flight per thread
    const long long rows = BH * L;
    const long long total = rows * TPR;
    const int lane = threadIdx.x & 31;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long t0 = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
         t0 < total; t0 += U * stride) {
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long t = t0 + u * stride + lane;
            if (t < total) {
                a[u] = dO[t];
                b[u] = O[t];
            } else {
                a[u] = make_uint4(0, 0, 0, 0);
                b[u] = a[u];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long t = t0 + u * stride + lane;
            float s = 0.f;
            if (BF16) {
                const __nv_bfloat162 *x = reinterpret_cast<const __nv_bfloat162 *>(&a[u]);
                const __nv_bfloat162 *y = reinterpret_cast<const __nv_bfloat162 *>(&b[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 p = __bfloat1622float2(x[e]), w = __bfloat1622float2(y[e]);
                    s = fmaf(p.x, w.x, s);
                    s = fmaf(p.y, w.y, s);
                }
            } else {
                const float *x = reinterpret_cast<const float *>(&a[u]);
                const float *y = reinterpret_cast<const float *>(&b[u]);
#pragma unroll
                for (int e = 0; e < 4; ++e) s = fmaf(x[e], y[e], s);
            }
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (t < total && (lane % TPR) == 0) {
                const long long r = t / TPR;
                const long long bh = r / L;
                const long long out = bh * Lp + (r - bh * L);
                Dp[out] = s;
                if (lse2) lse2[out] = lse[r] * kLog2e;
            }
        }
    }
    // padding rows [L, Lp) of every head
    const int pad = Lp - L;
    if (pad > 0) {
        for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
             t < BH * pad; t += stride) {
            const long long bh = t / pad;
            const long long out = bh * Lp + L + (t - bh * pad);
            Dp[out] = 0.f;
            if (lse2) lse2[out] = 0.f;
        }
    }
}

// ------------------------------------------------------------------------- fp32 path
// 64 x 64 output tiles, 256 threads in a 16 x 16 grid, 4 x 4 outputs per thread.

// S[h][i - r0][j] = scale * Q_i . K_j, -inf where masked; causal rows stop at the end of their
// 128-row tile's diagonal block (the columns the softmax reads).
template <int D>
__global__ void __launch_bounds__(256)
    f32_qk_slab_kernel(const float *__restrict__ Q, const float *__restrict__ K,
                       float *__restrict__ S, const SlabArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ float qs[64][D + 1];
    __shared__ float ks[64][D + 1];
    const int h = blockIdx.z;
    const int i0 = a.r0 + blockIdx.y * 64;  // head-relative
    const int j0 = blockIdx.x * 64;
    if (a.causal && j0 >= min(a.Lp, (i0 / 128) * 128 + 128)) return;
    const int bh = a.bh0 + h;
    const float *Qh = Q + static_cast<size_t>(bh) * a.L * D;
    const float *Kh = K + static_cast<size_t>(bh) * a.L * D;
    for (int x = threadIdx.x; x < 64 * D; x += 256) {
        const int r = x / D, k = x - r * D;
        const int iq = i0 + r, jk = j0 + r;
        qs[r][k] = (iq < a.L && iq < a.r0 + a.R) ? Qh[static_cast<size_t>(iq) * D + k] : 0.f;
        ks[r][k] = jk < a.L ? Kh[static_cast<size_t>(jk) * D + k] : 0.f;
    }
    __syncthreads();
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    float acc[4][4] = {};
#pragma unroll 8
    for (int k = 0; k < D; ++k) {
        float qa[4], kb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) qa[u] = qs[ty * 4 + u][k], kb[u] = ks[tx + 16 * u][k];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(qa[u], kb[w], acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= a.r0 + a.R) continue;
        float *srow = S + (static_cast<size_t>(h) * a.R + (i - a.r0)) * a.Lp;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int j = j0 + tx + 16 * w;
            if (j >= a.Lp) continue;
            const bool live = j < a.L && !(a.causal && j > i);
            srow[j] = live ? acc[u][w] * a.scale : -INFINITY;
        }
    }
}

// out[bh][i][:] = scale * sum_j A[h][i - r0][j] B[bh][j][:], k-blocks of 64 keys in ring order.
template <int D>
__global__ void __launch_bounds__(256)
    f32_ring_rows_kernel(const float *__restrict__ A, const float *__restrict__ Bm,
                         float *__restrict__ out, const SlabArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ float as[64][65];
    __shared__ float bs[64][D + 1];
    const int h = blockIdx.y;
    const int bh = a.bh0 + h;
    const int i0 = a.r0 + blockIdx.x * 64;
    const int end = a.causal ? min(a.Lp, (i0 / 128) * 128 + 128) : a.Lp;
    const int nkb = (end + 63) / 64;
    const int first = min(((i0 / a.c) * a.c) / 64, nkb - 1);
    const float *Bh = Bm + static_cast<size_t>(bh) * a.L * D;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    constexpr int CW = D / 16;
    float acc[4][CW] = {};
    for (int s = 0; s < nkb; ++s) {
        int kb = first + s;
        if (kb >= nkb) kb -= nkb;
        const int k0 = kb * 64;
        __syncthreads();
        for (int x = threadIdx.x; x < 64 * 64; x += 256) {
            const int r = x / 64, cidx = x - r * 64;
            const int i = i0 + r, j = k0 + cidx;
            as[r][cidx] = (i < a.r0 + a.R && j < end)
                              ? A[(static_cast<size_t>(h) * a.R + (i - a.r0)) * a.Lp + j]
                              : 0.f;
        }
        for (int x = threadIdx.x; x < 64 * D; x += 256) {
            const int r = x / D, k = x - r * D;
            const int j = k0 + r;
            bs[r][k] = j < a.L ? Bh[static_cast<size_t>(j) * D + k] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 64; ++kk) {
            float av[4], bv[CW];
#pragma unroll
            for (int u = 0; u < 4; ++u) av[u] = as[ty * 4 + u][kk];
#pragma unroll
            for (int w = 0; w < CW; ++w) bv[w] = bs[kk][tx + 16 * w];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < CW; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= a.r0 + a.R) continue;
#pragma unroll
        for (int w = 0; w < CW; ++w)
            out[(static_cast<size_t>(bh) * a.L + i) * D + tx + 16 * w] = acc[u][w] * a.scale;
    }
}

// P = exp(scale Q_i.K_j - lse_i), dS = P (dO_i.V_j - D_i); both fp32 slabs.
template <int D>
__global__ void __launch_bounds__(256)
    f32_bwd_slab_kernel(const float *__restrict__ Q, const float *__restrict__ K,
                        const float *__restrict__ dO, const float *__restrict__ V,
                        const float *__restrict__ lse, const float *__restrict__ Dvec,
                        float *__restrict__ P, float *__restrict__ dS, const SlabArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ float xs[64][D + 1];
    __shared__ float ys[64][D + 1];
    const int h = blockIdx.z;
    const int i0 = a.r0 + blockIdx.y * 64;
    const int j0 = blockIdx.x * 64;
    if (a.causal && j0 >= min(a.Lp, (i0 / 128) * 128 + 128)) return;
    const int bh = a.bh0 + h;
    const size_t hoff = static_cast<size_t>(bh) * a.L * D;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    float sacc[4][4] = {}, pacc[4][4] = {};
    for (int pass = 0; pass < 2; ++pass) {
        const float *X = pass == 0 ? Q : dO;
        const float *Y = pass == 0 ? K : V;
        __syncthreads();
        for (int x = threadIdx.x; x < 64 * D; x += 256) {
            const int r = x / D, k = x - r * D;
            const int iq = i0 + r, jk = j0 + r;
            xs[r][k] = (iq < a.L && iq < a.r0 + a.R) ? X[hoff + static_cast<size_t>(iq) * D + k] : 0.f;
            ys[r][k] = jk < a.L ? Y[hoff + static_cast<size_t>(jk) * D + k] : 0.f;
        }
        __syncthreads();
        float(*acc)[4] = pass == 0 ? sacc : pacc;
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            float xa[4], yb[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) xa[u] = xs[ty * 4 + u][k], yb[u] = ys[tx + 16 * u][k];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(xa[u], yb[w], acc[u][w]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty * 4 + u;
        if (i >= a.r0 + a.R) continue;
        const float l = lse[static_cast<size_t>(bh) * a.L + i];
        const float Di = Dvec[static_cast<size_t>(bh) * a.Lp + i];
        const size_t roff = (static_cast<size_t>(h) * a.R + (i - a.r0)) * a.Lp;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int j = j0 + tx + 16 * w;
            if (j >= a.Lp) continue;
            const bool live = j < a.L && !(a.causal && j > i);
            const float p = live ? expf(sacc[u][w] * a.scale - l) : 0.f;
            P[roff + j] = p;
            dS[roff + j] = p * (pacc[u][w] - Di);
        }
    }
}

// out[bh][j][:] (+)= alpha * sum_i A[h][i - r0][j] B[bh][i][:] over the group's rows
// (key-major ring: query blocks visited from the key tile's own chunk).
template <int D>
__global__ void __launch_bounds__(256)
    f32_ring_keys_kernel(const float *__restrict__ A, const float *__restrict__ Bm,
                         float *__restrict__ out, float alpha, int accumulate, const SlabArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ float as[64][65];
    __shared__ float bs[64][D + 1];
    const int h = blockIdx.y;
    const int bh = a.bh0 + h;
    const int j0 = blockIdx.x * 64;
    const int nqb = (a.R + 63) / 64;
    int lo = 0;
    if (a.causal) lo = max(0, (j0 - a.r0) / 64);
    const int cnt = nqb - lo;
    int first = 0;
    if (cnt > 0) first = min(max(((j0 / a.c) * a.c - a.r0) / 64, lo), nqb - 1) - lo;
    const float *Bh = Bm + static_cast<size_t>(bh) * a.L * D;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    constexpr int CW = D / 16;
    float acc[4][CW] = {};
    for (int s = 0; s < cnt; ++s) {
        int qb = first + s;
        if (qb >= cnt) qb -= cnt;
        qb += lo;
        const int il0 = qb * 64;  // group-relative
        __syncthreads();
        for (int x = threadIdx.x; x < 64 * 64; x += 256) {
            const int r = x / 64, cidx = x - r * 64;  // r: query, cidx: key
            const int il = il0 + r, j = j0 + cidx;
            // causal rows only hold the slab up to their tile's diagonal block
            const int i = a.r0 + il;
            const bool ok = il < a.R && j < min(a.L, a.causal ? (i / 128) * 128 + 128 : a.L);
            as[cidx][r] = ok ? A[(static_cast<size_t>(h) * a.R + il) * a.Lp + j] : 0.f;
        }
        for (int x = threadIdx.x; x < 64 * D; x += 256) {
            const int r = x / D, k = x - r * D;
            const int il = il0 + r;
            bs[r][k] = il < a.R ? Bh[static_cast<size_t>(a.r0 + il) * D + k] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 64; ++kk) {
            float av[4], bv[CW];
#pragma unroll
            for (int u = 0; u < 4; ++u) av[u] = as[ty * 4 + u][kk];
#pragma unroll
            for (int w = 0; w < CW; ++w) bv[w] = bs[kk][tx + 16 * w];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < CW; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int j = j0 + ty * 4 + u;
        if (j >= a.L) continue;
#pragma unroll
        for (int w = 0; w < CW; ++w) {
            float *o = out + (static_cast<size_t>(bh) * a.L + j) * D + tx + 16 * w;
            const float v = acc[u][w] * alpha;
            *o = accumulate ? *o + v : v;
        }
    }
}

}  // namespace

cudaError_t launch_slab_softmax(float *slab, float *lse, const SlabArgs &a, int p_bf16,
                                cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    const int EPT = a.Lp > 16384 ? 32 : 16;
    int wpr = (a.Lp + 32 * EPT - 1) / (32 * EPT);
    if (wpr > 32) return cudaErrorInvalidValue;
    const int threads = wpr >= 8 ? 32 * wpr : 256;
    const int rows_per_cta = threads / (32 * wpr);
    const long long nrows = static_cast<long long>(a.nh) * a.R;
    const long long grid = (nrows + rows_per_cta - 1) / rows_per_cta;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (EPT == 16) {
        if (p_bf16)
            e = launch_pdl(slab_softmax_kernel<16, true>, dim3((unsigned)grid), dim3(threads), 0, st, slab, lse, a, wpr);
        else
            e = launch_pdl(slab_softmax_kernel<16, false>, dim3((unsigned)grid), dim3(threads), 0, st, slab, lse, a, wpr);
    } else {
        if (p_bf16)
            e = launch_pdl(slab_softmax_kernel<32, true>, dim3((unsigned)grid), dim3(threads), 0, st, slab, lse, a, wpr);
        else
            e = launch_pdl(slab_softmax_kernel<32, false>, dim3((unsigned)grid), dim3(threads), 0, st, slab, lse, a, wpr);
    }
    return e;
}

cudaError_t launch_rowdot(const void *dO, const void *O, const float *lse, float *Dp,
                          float *lse2, long long BH, int L, int Lp, int d, int bf16,
                          cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    const long long vectors = BH * L * d / (bf16 ? 8 : 4);
    long long grid = (vectors + 255) / 256;
    if (grid > 148 * 8) grid = 148 * 8;  // a full SM of threads each; up to 4 vectors per thread
    if (grid < 1) grid = 1;
    const unsigned g = static_cast<unsigned>(grid);
    auto *a = static_cast<const uint4 *>(dO);
    auto *b = static_cast<const uint4 *>(O);
    if (bf16) {
        if (d == 64) e = launch_pdl(rowdot_kernel<64, true>, dim3(g), dim3(256), 0, st, a, b, lse, Dp, lse2, BH, L, Lp);
        else e = launch_pdl(rowdot_kernel<128, true>, dim3(g), dim3(256), 0, st, a, b, lse, Dp, lse2, BH, L, Lp);
    } else {
        if (d == 32) e = launch_pdl(rowdot_kernel<32, false>, dim3(g), dim3(256), 0, st, a, b, lse, Dp, lse2, BH, L, Lp);
        else e = launch_pdl(rowdot_kernel<64, false>, dim3(g), dim3(256), 0, st, a, b, lse, Dp, lse2, BH, L, Lp);
    }
    return e;
}

cudaError_t launch_f32_qk_slab(const float *Q, const float *K, float *S, const SlabArgs &a,
                               cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    dim3 grid((a.Lp + 63) / 64, (a.R + 63) / 64, a.nh);
    if (a.d == 32) e = launch_pdl(f32_qk_slab_kernel<32>, dim3(grid), dim3(256), 0, st, Q, K, S, a);
    else e = launch_pdl(f32_qk_slab_kernel<64>, dim3(grid), dim3(256), 0, st, Q, K, S, a);
    return e;
}

cudaError_t launch_f32_ring_rows(const float *A, const float *Bm, float *out, const SlabArgs &a,
                                 cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    dim3 grid((a.R + 63) / 64, a.nh);
    if (a.d == 32) e = launch_pdl(f32_ring_rows_kernel<32>, dim3(grid), dim3(256), 0, st, A, Bm, out, a);
    else e = launch_pdl(f32_ring_rows_kernel<64>, dim3(grid), dim3(256), 0, st, A, Bm, out, a);
    return e;
}

cudaError_t launch_f32_bwd_slab(const float *Q, const float *K, const float *dO, const float *V,
                                const float *lse, const float *Dvec, float *P, float *dS,
                                const SlabArgs &a, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    dim3 grid((a.Lp + 63) / 64, (a.R + 63) / 64, a.nh);
    if (a.d == 32) e = launch_pdl(f32_bwd_slab_kernel<32>, dim3(grid), dim3(256), 0, st, Q, K, dO, V, lse, Dvec, P, dS, a);
    else e = launch_pdl(f32_bwd_slab_kernel<64>, dim3(grid), dim3(256), 0, st, Q, K, dO, V, lse, Dvec, P, dS, a);
    return e;
}

cudaError_t launch_f32_ring_keys(const float *A, const float *Bm, float *out, float alpha,
                                 int accumulate, const SlabArgs &a, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    dim3 grid((a.L + 63) / 64, a.nh);
    if (a.d == 32) e = launch_pdl(f32_ring_keys_kernel<32>, dim3(grid), dim3(256), 0, st, A, Bm, out, alpha, accumulate, a);
    else e = launch_pdl(f32_ring_keys_kernel<64>, dim3(grid), dim3(256), 0, st, A, Bm, out, alpha, accumulate, a);
    return e;
}

}  // namespace rsa
