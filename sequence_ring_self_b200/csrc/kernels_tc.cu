// kernels_tc.cu -- bf16 tensor-core kernels of Ring Self-Attention for sm_100a.
//
// The method ("Sequence Parallelism: Making 4D Parallelism Possible", review page, Abstract and
// "Proposed method"): the sequence is cut into N chunks of c = L/N rows; chunk n builds its
// c x L score slab by visiting key chunk m = (n + s) mod N at ring step s, takes the row
// softmax over the whole slab, and accumulates O_n = sum_s P_n[:, block m] V_m on a second
// ring pass; the backward pass runs the same schedule. On one GPU a ring step is an order
// of tiles: each kernel below visits the key (or query) blocks of a tile starting at the
// block of its own chunk and wrapping around, which is the ring rotation.
//
// Two kernels here (the backward's key-major kernel is in kernels_bwd.cu), persistent and
// warp-specialised (192 threads = 6 warps):
//   warp 0 lane 0 : TMA producer (global -> shared, 128-byte swizzle, mbarrier pipeline)
//   warp 1        : allocates TMEM; lane 0 issues tcgen05.mma into a double-buffered
//                   TMEM accumulator and commits to mbarriers
//   warps 2..5    : epilogue; warp w reads TMEM lanes 32*(w%4)..+31 (one tile row each)
//
//   qk_slab    (ring pass 1)      S = scale * Q K^T, masked, fp32 slab      A, B K-major
//   ring_rows  (ring pass 2, dQ)  out = scale * A B over the slab's keys      B MN-major
#include "tc_common.cuh"

namespace rsa {
namespace {

constexpr int kThreads = 192;
using namespace tc;

// ======================================================================================
// qk_slab: S[h][i - r0][j] = log2(e) * scale * Q_i . K_j  (fp32 scores in base-2 units;
// -inf where j >= L or causal j > i), and per row and 128-column half tile the softmax
// partials (max_j S, sum_j 2^(S - max)) for the streaming softmax.
// Tile = 128 query rows x 256 keys; K-loop over d in blocks of 64 (one 128-byte swizzle row).
// 320 threads: producer, MMA, and 8 epilogue warps (2 per TMEM lane quarter, 128 columns each).
// ======================================================================================
template <int D>
struct QkCfg {
    static constexpr int BM = 128, BN = 256;
    static constexpr int KB = D / 64;
    static constexpr int A_BYTES = BM * 64 * 2;
    static constexpr int B_BYTES = BN * 64 * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 3;
    static constexpr int EPI_BYTES = 8 * 2 * 4096;  // per epilogue warp: 2 x (32 rows x 128 B)
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + (int)sizeof(Ctl);
    static constexpr uint32_t TMEM_COLS = 512;
};

struct QkTile {
    int h, i0, ct;
};

// Tiles are (head, 128-row tile, 256-column tile); causal tiles right of the diagonal are
// skipped. The column tiles of a row tile start at the block holding its own chunk's keys.
__device__ __forceinline__ bool qk_decode(const SlabArgs &a, int t, QkTile &tl) {
    const int per_head = a.nRT * a.nCT;
    tl.h = t / per_head;
    const int rem = t - tl.h * per_head;
    const int rt = rem / a.nCT;
    const int cti = rem - rt * a.nCT;
    tl.i0 = a.r0 + rt * 128;
    int live = a.nCT;
    if (a.causal) live = min(a.nCT, (min(a.L, tl.i0 + 128) + 255) / 256);
    if (cti >= live) return false;
    const int n = tl.i0 / a.c;
    const int first = min((n * a.c) / 256, live - 1);
    tl.ct = ring_block(first, cti, live);
    return true;
}

constexpr int kQkThreads = 320;

__device__ __forceinline__ void softmax_combine(float &m, float &l, float m2, float l2) {
    const float nm = fmaxf(m, m2);
    if (nm == -INFINITY) return;
    l = l * fast_exp2(m - nm) + l2 * fast_exp2(m2 - nm);
    m = nm;
}

template <int D>
__global__ void __launch_bounds__(kQkThreads, 1)
    qk_slab_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                   const __grid_constant__ CUtensorMap mS, const SlabArgs a) {
    using C = QkCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    uint8_t *stages = smem;
    uint8_t *epi = smem + C::STAGES * C::STAGE_BYTES;
    Ctl *ctl = reinterpret_cast<Ctl *>(epi + C::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        init_ctl(ctl, C::STAGES, 8);
        prefetch_tmap(&mQ);
        prefetch_tmap(&mK);
        prefetch_tmap(&mS);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    // everything above (barriers, TMEM, descriptor prefetch) overlaps the previous kernel
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            Pipe p{0, 0};
            bool issued[C::STAGES];
            uint32_t ipar[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                QkTile tl;
                if (!qk_decode(a, t, tl)) continue;
                for (int kb = 0; kb < C::KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    tma_load_3d(sa, &mQ, bar, kb * 64, tl.i0, a.bh0 + tl.h);
                    tma_load_3d(sa + C::A_BYTES, &mK, bar, kb * 64, tl.ct * C::BN, a.bh0 + tl.h);
                    issued[p.stage] = true;
                    ipar[p.stage] = p.phase;
                    pipe_next(p, C::STAGES);
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) drain_wait(&ctl->full[s], ipar[s]);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            Pipe p{0, 0};
            int acc = 0;
            uint32_t aph = 0;
            const uint32_t idesc = idesc_bf16_f32(128, C::BN, 0, 0);
            constexpr uint64_t KM = sdesc_const(16, 1024);
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                QkTile tl;
                if (!qk_decode(a, t, tl)) continue;
                if (!mbar_wait(&ctl->tempty[acc], aph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t dcol = tmem + acc * C::BN;
                for (int kb = 0; kb < C::KB; ++kb) {
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(stages + p.stage * C::STAGE_BYTES);
                    const uint64_t da = sdesc(KM, sa), db = sdesc(KM, sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(dcol, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    tc_commit(&ctl->empty[p.stage]);
                    pipe_next(p, C::STAGES);
                }
                if (!ok) break;
                tc_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        const int ew = warp - 2, q = warp & 3, hf = ew >> 2;
        uint8_t *ebuf = epi + ew * 8192;
        const float sl2 = a.scale * kLog2e;
        int acc = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            QkTile tl;
            if (!qk_decode(a, t, tl)) continue;
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const int i = tl.i0 + 32 * q + lane;
            const int i_min = tl.i0 + 32 * q;  // smallest row of this warp
            float run_m = -INFINITY, run_l = 0.f;
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                const int col = hf * 128 + cc * 32;
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * C::BN + col, r);
                tmem_ld_wait();
                const int j0 = tl.ct * C::BN + col;
                float v[32];
                float cm = -INFINITY;
                if (j0 + 32 <= a.L && (!a.causal || j0 + 31 <= i_min)) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        v[e] = __uint_as_float(r[e]) * sl2;
                        cm = fmaxf(cm, v[e]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = j0 + e;
                        const bool live = j < a.L && !(a.causal && j > i);
                        v[e] = live ? __uint_as_float(r[e]) * sl2 : -INFINITY;
                        cm = fmaxf(cm, v[e]);
                    }
                }
                if (cm != -INFINITY) {
                    float cs = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e) cs += fast_exp2(v[e] - cm);
                    softmax_combine(run_m, run_l, cm, cs);
                }
                uint8_t *buf = ebuf + (cc & 1) * 4096;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4)
                    *reinterpret_cast<float4 *>(buf + sw128_offset(lane, e4)) =
                        make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&mS, buf, j0, tl.i0 - a.r0 + 32 * q, tl.h);
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            if (i < a.r0 + a.R)
                a.stats[(static_cast<size_t>(tl.h) * a.R + (i - a.r0)) * a.nStat + 2 * tl.ct + hf] =
                    make_float2(run_m, run_l);
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (threadIdx.x == 0 && ctl->abort) atomicExch(a.status, 5);
}

// ======================================================================================
// ring_rows: out[bh][i][:] = scale * sum_j P(i, j) * V[bh][j][:]   (bf16 out; ring pass 2)
// P is the row-major bf16 slab P[h][i - r0][j], read K-major in 128 x 64 boxes. V ([L][D])
// is the MN-major operand, read in 64-row boxes 64 columns wide. K-loop over 64-key blocks
// in ring order starting at the tile's own chunk; causal tiles stop at their diagonal block.
// ======================================================================================
template <int D>
struct RowsCfg {
    static constexpr int A_BYTES = 128 * 64 * 2;
    static constexpr int B_BYTES = 64 * D * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = D == 64 ? 6 : 5;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + (int)sizeof(Ctl);
    static constexpr uint32_t TMEM_COLS = D == 64 ? 128 : 256;
};

struct RowsTile {
    int h, i0, nkb, first;
};

// Tiles are (128-row tile, head), longest causal tiles first.
__device__ __forceinline__ void rows_decode(const SlabArgs &a, int t, RowsTile &tl) {
    const int rt = a.nRT - 1 - t / a.nh;
    tl.h = t - (t / a.nh) * a.nh;
    tl.i0 = a.r0 + rt * 128;
    const int live_end = a.causal ? min(a.L, tl.i0 + 128) : a.L;
    tl.nkb = (live_end + 63) / 64;
    const int n = tl.i0 / a.c;
    tl.first = min((n * a.c) / 64, tl.nkb - 1);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    ring_rows_kernel(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB,
                     __nv_bfloat16 *__restrict__ out, const SlabArgs a) {
    using C = RowsCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    uint8_t *stages = smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + C::STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        init_ctl(ctl, C::STAGES, 4);
        prefetch_tmap(&mA);
        prefetch_tmap(&mB);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    // everything above (barriers, TMEM, descriptor prefetch) overlaps the previous kernel
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            Pipe p{0, 0};
            bool issued[C::STAGES];
            uint32_t ipar[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                RowsTile tl;
                rows_decode(a, t, tl);
                for (int s = 0; s < tl.nkb; ++s) {
                    const int kb = ring_block(tl.first, s, tl.nkb);
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    tma_load_3d(sa, &mA, bar, kb * 64, tl.i0 - a.r0, tl.h);
#pragma unroll
                    for (int dp = 0; dp < D / 64; ++dp)
                        tma_load_3d(sa + C::A_BYTES + dp * 8192, &mB, bar, dp * 64, kb * 64,
                                    a.bh0 + tl.h);
                    issued[p.stage] = true;
                    ipar[p.stage] = p.phase;
                    pipe_next(p, C::STAGES);
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) drain_wait(&ctl->full[s], ipar[s]);
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            Pipe p{0, 0};
            int acc = 0;
            uint32_t aph = 0;
            const uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
            constexpr uint64_t DA = sdesc_const(16, 1024);    // K-major P
            constexpr uint64_t DB = sdesc_const(8192, 1024);  // MN-major V
            constexpr uint32_t KSTEP_A = 2;  // 16 K-elements in 16-byte units
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                RowsTile tl;
                rows_decode(a, t, tl);
                if (!mbar_wait(&ctl->tempty[acc], aph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t dcol = tmem + acc * D;
                for (int s = 0; s < tl.nkb; ++s) {
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(stages + p.stage * C::STAGE_BYTES);
                    const uint64_t da = sdesc(DA, sa), db = sdesc(DB, sa + C::A_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(dcol, da + KSTEP_A * k, db + 128 * k, idesc, (s | k) != 0 ? 1u : 0u);
                    tc_commit(&ctl->empty[p.stage]);
                    pipe_next(p, C::STAGES);
                }
                if (!ok) break;
                tc_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        int acc = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            RowsTile tl;
            rows_decode(a, t, tl);
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const int i = tl.i0 + 32 * q + lane;
            const bool row_ok = i < a.r0 + a.R;
            __nv_bfloat16 *orow = out + (static_cast<size_t>(a.bh0 + tl.h) * a.L + i) * D;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * D + cc * 32, r);
                tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            w[u] = pack_bf16x2(__uint_as_float(r[8 * g + 2 * u]) * a.scale,
                                               __uint_as_float(r[8 * g + 2 * u + 1]) * a.scale);
                        st_global_v4(orow + cc * 32 + 8 * g, w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (threadIdx.x == 0 && ctl->abort) atomicExch(a.status, 5);
}

}  // namespace

int tc::grid_for(int ntiles, int num_sms) {
    return ntiles < num_sms ? (ntiles > 0 ? ntiles : 1) : num_sms;
}

cudaError_t tc_kernels_configure() {
    cudaError_t e;
#define RSA_SMEM(kern, bytes)                                                                  \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);        \
    if (e != cudaSuccess) return e;
    RSA_SMEM(qk_slab_kernel<64>, QkCfg<64>::SMEM)
    RSA_SMEM(qk_slab_kernel<128>, QkCfg<128>::SMEM)
    RSA_SMEM(ring_rows_kernel<64>, RowsCfg<64>::SMEM)
    RSA_SMEM(ring_rows_kernel<128>, RowsCfg<128>::SMEM)
#undef RSA_SMEM
    return cudaSuccess;
}

cudaError_t launch_qk_slab(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mS,
                           const SlabArgs &a, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    const int grid = tc::grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        e = launch_pdl(qk_slab_kernel<64>, dim3(grid), dim3(kQkThreads), QkCfg<64>::SMEM, st, mQ, mK, mS, a);
    else
        e = launch_pdl(qk_slab_kernel<128>, dim3(grid), dim3(kQkThreads), QkCfg<128>::SMEM, st, mQ, mK, mS, a);
    return e;
}

cudaError_t launch_ring_rows(const CUtensorMap &mA, const CUtensorMap &mB, void *out,
                             const SlabArgs &a, int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    auto *o = static_cast<__nv_bfloat16 *>(out);
    if (a.d == 64)
        return launch_pdl(ring_rows_kernel<64>, dim3(grid), dim3(kThreads), RowsCfg<64>::SMEM,
                          st, mA, mB, o, a);
    return launch_pdl(ring_rows_kernel<128>, dim3(grid), dim3(kThreads), RowsCfg<128>::SMEM, st,
                      mA, mB, o, a);
}

}  // namespace rsa
