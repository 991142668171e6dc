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
// Four kernels, all persistent and warp-specialised (192 threads = 6 warps):
//   warp 0 lane 0 : TMA producer (global -> shared, 128-byte swizzle, mbarrier pipeline)
//   warp 1        : allocates TMEM; lane 0 issues tcgen05.mma into a double-buffered
//                   TMEM accumulator and commits to mbarriers
//   warps 2..5    : epilogue; warp w reads TMEM lanes 32*(w%4)..+31 (one tile row each)
//
//   qk_slab    (ring pass 1)   S = scale * Q K^T, masked, fp32 slab        A,B K-major
//   ring_rows  (ring pass 2 / dQ) out = scale * A B, A bf16 slab rows       A K-major, B MN-major
//   bwd_slab   (recompute + dP) P = exp(scale QK^T - lse), dS = P (dO V^T - D) as bf16 slabs
//   ring_keys  (dV, dK)        dV = P^T dO, dK = scale dS^T Q over query blocks  A,B MN-major
#include "rsa_internal.h"
#include "sm100_ptx.cuh"

namespace rsa {
namespace {

constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr float kLog2e = 1.4426950408889634f;

struct Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct Pipe {
    int stage;
    uint32_t phase;
};

__device__ __forceinline__ void pipe_next(Pipe &p, int stages) {
    if (++p.stage == stages) {
        p.stage = 0;
        p.phase ^= 1u;
    }
}

__device__ __forceinline__ uint8_t *align_1024(uint8_t *p) {
    const uint32_t a = smem_addr(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Bounded wait that ignores the abort flag (used to drain work already in flight).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    int dummy = 0;
    mbar_wait(bar, parity, &dummy);
}

// Warp-uniform wait: lane 0 polls, the verdict is broadcast, the warp re-converges.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

__device__ __forceinline__ void init_ctl(Ctl *ctl, int stages, int tempty_count) {
    for (int s = 0; s < stages; ++s) {
        mbar_init(&ctl->full[s], 1);
        mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
        mbar_init(&ctl->tfull[a], 1);
        mbar_init(&ctl->tempty[a], tempty_count);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
}

// Ring rotation of `count` blocks starting at `first`: step t visits (first + t) mod count.
__device__ __forceinline__ int ring_block(int first, int t, int count) {
    int b = first + t;
    return b >= count ? b - count : b;
}

// Store 8 packed bf16 values (16 bytes) to global memory.
__device__ __forceinline__ void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// ======================================================================================
// qk_slab: S[h][i - r0][j] = scale * Q_i . K_j   (fp32; -inf where j >= L or causal j > i)
// Tile = 128 query rows x 256 keys; K-loop over d in blocks of 64 (one 128-byte swizzle row).
// ======================================================================================
template <int D>
struct QkCfg {
    static constexpr int BM = 128, BN = 256;
    static constexpr int KB = D / 64;
    static constexpr int A_BYTES = BM * 64 * 2;
    static constexpr int B_BYTES = BN * 64 * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 3;
    static constexpr int EPI_BYTES = 4 * 2 * 4096;  // per epilogue warp: 2 x (32 rows x 128 B)
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
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
        init_ctl(ctl, C::STAGES, 4);
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
                    const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(dcol, smem_desc_sw128(sa + 32 * k, 16, 1024),
                                    smem_desc_sw128(sb + 32 * k, 16, 1024), idesc,
                                    (kb | k) != 0 ? 1u : 0u);
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
        const int ew = warp - 2, q = warp & 3;
        uint8_t *ebuf = epi + ew * 8192;
        int acc = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            QkTile tl;
            if (!qk_decode(a, t, tl)) continue;
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const int i = tl.i0 + 32 * q + lane;
#pragma unroll 1
            for (int cc = 0; cc < C::BN / 32; ++cc) {
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * C::BN + cc * 32, r);
                tmem_ld_wait();
                uint8_t *buf = ebuf + (cc & 1) * 4096;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                const int j0 = tl.ct * C::BN + cc * 32;
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = j0 + 4 * e4 + u;
                        const bool live = j < a.L && !(a.causal && j > i);
                        v[u] = live ? __uint_as_float(r[4 * e4 + u]) * a.scale : -INFINITY;
                    }
                    *reinterpret_cast<float4 *>(buf + sw128_offset(lane, e4)) =
                        make_float4(v[0], v[1], v[2], v[3]);
                }
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
// ring_rows: out[bh][i][:] = scale * sum_j A[h][i - r0][j] * B[bh][j][:]   (bf16 out)
// A is a bf16 slab (P or dS), read K-major in 128 x 64 boxes; B ([L][D], V or K) is the
// MN-major operand, read in 64-row boxes 64 columns wide. K-loop over 64-key blocks in
// ring order starting at the tile's own chunk; causal tiles stop at their diagonal block.
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
                    const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(dcol, smem_desc_sw128(sa + 32 * k, 16, 1024),
                                    smem_desc_sw128(sb + 2048 * k, 8192, 1024), idesc,
                                    (s | k) != 0 ? 1u : 0u);
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

// ======================================================================================
// bwd_slab: for a 128 x 128 tile of the slab,
//   S  = Q_i K_j^T,  dP = dO_i V_j^T  (two TMEM accumulators)
//   P  = exp(scale S - lse_i)  (0 where j >= L or causal j > i),  dS = P (dP - D_i)
// P and dS are written as bf16 slabs with TMA stores.
// ======================================================================================
template <int D>
struct BwdCfg {
    static constexpr int BN = 128;
    static constexpr int KB = D / 64;
    static constexpr int T_BYTES = 128 * 64 * 2;  // one 128 x 64 bf16 box
    static constexpr int STAGE_BYTES = 4 * T_BYTES;
    static constexpr int STAGES = 2;
    static constexpr int EPI_BYTES = 4 * 4 * 4096;  // per warp: {P, dS} x 2 buffers
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + (int)sizeof(Ctl);
    static constexpr uint32_t TMEM_COLS = 512;
};

struct BwdTile {
    int h, i0, ct;
};

__device__ __forceinline__ bool bwd_decode(const SlabArgs &a, int t, BwdTile &tl) {
    const int per_head = a.nRT * a.nCT;
    tl.h = t / per_head;
    const int rem = t - tl.h * per_head;
    const int rt = rem / a.nCT;
    const int cti = rem - rt * a.nCT;
    tl.i0 = a.r0 + rt * 128;
    int live = a.nCT;
    if (a.causal) live = min(a.nCT, (min(a.L, tl.i0 + 128) + 127) / 128);
    if (cti >= live) return false;
    const int n = tl.i0 / a.c;
    const int first = min((n * a.c) / 128, live - 1);
    tl.ct = ring_block(first, cti, live);
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_slab_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                    const __grid_constant__ CUtensorMap mdO, const __grid_constant__ CUtensorMap mV,
                    const __grid_constant__ CUtensorMap mP, const __grid_constant__ CUtensorMap mdS,
                    const float *__restrict__ lse, const float *__restrict__ Dvec,
                    const SlabArgs a) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    uint8_t *stages = smem;
    uint8_t *epi = smem + C::STAGES * C::STAGE_BYTES;
    Ctl *ctl = reinterpret_cast<Ctl *>(epi + C::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        init_ctl(ctl, C::STAGES, 4);
        prefetch_tmap(&mQ);
        prefetch_tmap(&mK);
        prefetch_tmap(&mdO);
        prefetch_tmap(&mV);
        prefetch_tmap(&mP);
        prefetch_tmap(&mdS);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            Pipe p{0, 0};
            bool issued[C::STAGES];
            uint32_t ipar[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BwdTile tl;
                if (!bwd_decode(a, t, tl)) continue;
                const int bh = a.bh0 + tl.h;
                for (int kb = 0; kb < C::KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *s0 = stages + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    tma_load_3d(s0, &mQ, bar, kb * 64, tl.i0, bh);
                    tma_load_3d(s0 + C::T_BYTES, &mK, bar, kb * 64, tl.ct * C::BN, bh);
                    tma_load_3d(s0 + 2 * C::T_BYTES, &mdO, bar, kb * 64, tl.i0, bh);
                    tma_load_3d(s0 + 3 * C::T_BYTES, &mV, bar, kb * 64, tl.ct * C::BN, bh);
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
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BwdTile tl;
                if (!bwd_decode(a, t, tl)) continue;
                if (!mbar_wait(&ctl->tempty[acc], aph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t d_s = tmem + acc * 256;
                const uint32_t d_dp = d_s + 128;
                for (int kb = 0; kb < C::KB; ++kb) {
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s0 = smem_addr(stages + p.stage * C::STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t en = (kb | k) != 0 ? 1u : 0u;
                        tc_mma_bf16(d_s, smem_desc_sw128(s0 + 32 * k, 16, 1024),
                                    smem_desc_sw128(s0 + C::T_BYTES + 32 * k, 16, 1024), idesc,
                                    en);
                        tc_mma_bf16(d_dp, smem_desc_sw128(s0 + 2 * C::T_BYTES + 32 * k, 16, 1024),
                                    smem_desc_sw128(s0 + 3 * C::T_BYTES + 32 * k, 16, 1024),
                                    idesc, en);
                    }
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
        const int ew = warp - 2, q = warp & 3;
        uint8_t *ebuf = epi + ew * 16384;  // [buffer b][P | dS] x 4 KB
        int acc = 0;
        uint32_t aph = 0;
        const float sl2 = a.scale * kLog2e;
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            BwdTile tl;
            if (!bwd_decode(a, t, tl)) continue;
            const int i = tl.i0 + 32 * q + lane;
            const size_t row = static_cast<size_t>(a.bh0 + tl.h) * a.L + i;
            const float lse2 = i < a.L ? lse[row] * kLog2e : 0.f;
            const float Di = i < a.L ? Dvec[row] : 0.f;
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const uint32_t tl_s = tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * 256;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint8_t *bp = ebuf + half * 8192;
                uint8_t *bds = bp + 4096;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
#pragma unroll 1
                for (int sub = 0; sub < 2; ++sub) {
                    const int col = half * 64 + sub * 32;
                    uint32_t rs[32], rd[32];
                    tmem_ld32(tl_s + col, rs);
                    tmem_ld32(tl_s + 128 + col, rd);
                    tmem_ld_wait();
                    const int j0 = tl.ct * C::BN + col;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint32_t wp[4], wd[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            float pv[2], dv[2];
#pragma unroll
                            for (int z = 0; z < 2; ++z) {
                                const int e = 8 * g + 2 * u + z;
                                const int j = j0 + e;
                                const bool live = j < a.L && !(a.causal && j > i);
                                const float p =
                                    live ? exp2f(__uint_as_float(rs[e]) * sl2 - lse2) : 0.f;
                                pv[z] = p;
                                dv[z] = p * (__uint_as_float(rd[e]) - Di);
                            }
                            wp[u] = pack_bf16x2(pv[0], pv[1]);
                            wd[u] = pack_bf16x2(dv[0], dv[1]);
                        }
                        const uint32_t off = sw128_offset(lane, sub * 4 + g);
                        *reinterpret_cast<uint4 *>(bp + off) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
                        *reinterpret_cast<uint4 *>(bds + off) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int jc = tl.ct * C::BN + half * 64;
                    const int ir = tl.i0 - a.r0 + 32 * q;
                    tma_store_3d(&mP, bp, jc, ir, tl.h);
                    tma_store_3d(&mdS, bds, jc, ir, tl.h);
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
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
// ring_keys: for a tile of 128 keys j (key-major ring),
//   dV_j = sum_i P[i][j] dO_i,   dK_j = scale sum_i dS[i][j] Q_i
// over the group's query rows, in 64-row blocks starting at the key tile's own chunk.
// A operands (P^T, dS^T) are MN-major reads of the row-major slabs; B operands (dO, Q) are
// MN-major [rows][D] boxes. mode 0: write bf16 outputs; 1: add into fp32 accumulators;
// 2: accumulators + this group -> bf16 outputs.
// ======================================================================================
template <int D>
struct KeysCfg {
    static constexpr int A_BYTES = 2 * 64 * 64 * 2;  // 128 keys x 64 queries
    static constexpr int B_BYTES = 64 * D * 2;       // 64 queries x D
    static constexpr int STAGE_BYTES = 2 * (A_BYTES + B_BYTES);
    static constexpr int STAGES = 3;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + (int)sizeof(Ctl);
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256 : 512;
};

struct KeysTile {
    int h, j0, lo, nqb, first;
};

// Tiles are (128-key tile, head), longest causal tiles (smallest keys) first. Returns false
// when no query row of the group can see the tile's keys.
__device__ __forceinline__ bool keys_decode(const SlabArgs &a, int t, KeysTile &tl) {
    const int kt = t / a.nh;
    tl.h = t - kt * a.nh;
    tl.j0 = kt * 128;
    const int nqb = (a.R + 63) / 64;
    int lo = 0;
    if (a.causal) lo = max(0, (tl.j0 - a.r0) / 64);
    if (lo >= nqb) return false;
    tl.lo = lo;
    tl.nqb = nqb;
    const int m = tl.j0 / a.c;
    const int want = (m * a.c - a.r0) / 64;
    tl.first = min(max(want, lo), nqb - 1) - lo;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    ring_keys_kernel(const __grid_constant__ CUtensorMap mPt, const __grid_constant__ CUtensorMap mdO,
                     const __grid_constant__ CUtensorMap mdSt, const __grid_constant__ CUtensorMap mQ,
                     __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV,
                     float *__restrict__ acc_dK, float *__restrict__ acc_dV, const SlabArgs a) {
    using C = KeysCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    uint8_t *stages = smem;
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + C::STAGES * C::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // stage layout: [P^T 16 KB][dO B_BYTES][dS^T 16 KB][Q B_BYTES]
    constexpr int OFF_DO = C::A_BYTES;
    constexpr int OFF_DS = C::A_BYTES + C::B_BYTES;
    constexpr int OFF_Q = 2 * C::A_BYTES + C::B_BYTES;

    if (threadIdx.x == 0) {
        init_ctl(ctl, C::STAGES, 4);
        prefetch_tmap(&mPt);
        prefetch_tmap(&mdO);
        prefetch_tmap(&mdSt);
        prefetch_tmap(&mQ);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            Pipe p{0, 0};
            bool issued[C::STAGES];
            uint32_t ipar[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                KeysTile tl;
                if (!keys_decode(a, t, tl)) continue;
                const int bh = a.bh0 + tl.h;
                const int cnt = tl.nqb - tl.lo;
                for (int s = 0; s < cnt; ++s) {
                    const int qb = tl.lo + ring_block(tl.first, s, cnt);
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *s0 = stages + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    const int irow = qb * 64;  // group-relative query row
                    tma_load_3d(s0, &mPt, bar, tl.j0, irow, tl.h);
                    tma_load_3d(s0 + 8192, &mPt, bar, tl.j0 + 64, irow, tl.h);
                    tma_load_3d(s0 + OFF_DS, &mdSt, bar, tl.j0, irow, tl.h);
                    tma_load_3d(s0 + OFF_DS + 8192, &mdSt, bar, tl.j0 + 64, irow, tl.h);
#pragma unroll
                    for (int dp = 0; dp < D / 64; ++dp) {
                        tma_load_3d(s0 + OFF_DO + dp * 8192, &mdO, bar, dp * 64, a.r0 + irow, bh);
                        tma_load_3d(s0 + OFF_Q + dp * 8192, &mQ, bar, dp * 64, a.r0 + irow, bh);
                    }
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
            const uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                KeysTile tl;
                if (!keys_decode(a, t, tl)) continue;
                if (!mbar_wait(&ctl->tempty[acc], aph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t d_v = tmem + acc * (2 * D);
                const uint32_t d_k = d_v + D;
                const int cnt = tl.nqb - tl.lo;
                for (int s = 0; s < cnt; ++s) {
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t s0 = smem_addr(stages + p.stage * C::STAGE_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t en = (s | k) != 0 ? 1u : 0u;
                        tc_mma_bf16(d_v, smem_desc_sw128(s0 + 2048 * k, 8192, 1024),
                                    smem_desc_sw128(s0 + OFF_DO + 2048 * k, 8192, 1024), idesc, en);
                        tc_mma_bf16(d_k, smem_desc_sw128(s0 + OFF_DS + 2048 * k, 8192, 1024),
                                    smem_desc_sw128(s0 + OFF_Q + 2048 * k, 8192, 1024), idesc, en);
                    }
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
            KeysTile tl;
            if (!keys_decode(a, t, tl)) continue;
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const int j = tl.j0 + 32 * q + lane;
            const bool ok = j < a.L;
            const size_t orow = (static_cast<size_t>(a.bh0 + tl.h) * a.L + j) * D;
            const size_t arow = static_cast<size_t>(j) * D;  // accumulators hold one head
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
                const float mul = which ? a.scale : 1.f;
                __nv_bfloat16 *o = which ? dK : dV;
                float *accp = which ? acc_dK : acc_dV;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t r[32];
                    tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * (2 * D) +
                                  which * D + cc * 32,
                              r);
                    tmem_ld_wait();
                    if (!ok) continue;
                    float v[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) * mul;
                    if (a.mode != 0) {
                        float4 *ap = reinterpret_cast<float4 *>(accp + arow + cc * 32);
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            const float4 x = ap[g];
                            v[4 * g] += x.x;
                            v[4 * g + 1] += x.y;
                            v[4 * g + 2] += x.z;
                            v[4 * g + 3] += x.w;
                        }
                        if (a.mode == 1) {
#pragma unroll
                            for (int g = 0; g < 8; ++g)
                                ap[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                            continue;
                        }
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        st_global_v4(o + orow + cc * 32 + 8 * g, pack_bf16x2(v[8 * g], v[8 * g + 1]),
                                     pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                     pack_bf16x2(v[8 * g + 4], v[8 * g + 5]),
                                     pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
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

int grid_for(int ntiles, int num_sms) { return ntiles < num_sms ? (ntiles > 0 ? ntiles : 1) : num_sms; }

}  // namespace

cudaError_t tc_kernels_configure() {
    cudaError_t e;
#define RSA_SMEM(kern, bytes)                                                                  \
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);        \
    if (e != cudaSuccess) return e;
    RSA_SMEM(qk_slab_kernel<64>, QkCfg<64>::SMEM)
    RSA_SMEM(qk_slab_kernel<128>, QkCfg<128>::SMEM)
    RSA_SMEM(ring_rows_kernel<64>, RowsCfg<64>::SMEM)
    RSA_SMEM(ring_rows_kernel<128>, RowsCfg<128>::SMEM)
    RSA_SMEM(bwd_slab_kernel<64>, BwdCfg<64>::SMEM)
    RSA_SMEM(bwd_slab_kernel<128>, BwdCfg<128>::SMEM)
    RSA_SMEM(ring_keys_kernel<64>, KeysCfg<64>::SMEM)
    RSA_SMEM(ring_keys_kernel<128>, KeysCfg<128>::SMEM)
#undef RSA_SMEM
    return cudaSuccess;
}

cudaError_t launch_qk_slab(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mS,
                           const SlabArgs &a, int num_sms, cudaStream_t st) {
    const int grid = grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        qk_slab_kernel<64><<<grid, kThreads, QkCfg<64>::SMEM, st>>>(mQ, mK, mS, a);
    else
        qk_slab_kernel<128><<<grid, kThreads, QkCfg<128>::SMEM, st>>>(mQ, mK, mS, a);
    return cudaGetLastError();
}

cudaError_t launch_ring_rows(const CUtensorMap &mA, const CUtensorMap &mB, void *out,
                             const SlabArgs &a, int num_sms, cudaStream_t st) {
    const int grid = grid_for(a.ntiles, num_sms);
    auto *o = static_cast<__nv_bfloat16 *>(out);
    if (a.d == 64)
        ring_rows_kernel<64><<<grid, kThreads, RowsCfg<64>::SMEM, st>>>(mA, mB, o, a);
    else
        ring_rows_kernel<128><<<grid, kThreads, RowsCfg<128>::SMEM, st>>>(mA, mB, o, a);
    return cudaGetLastError();
}

cudaError_t launch_bwd_slab(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mdO,
                            const CUtensorMap &mV, const CUtensorMap &mP, const CUtensorMap &mdS,
                            const float *lse, const float *Dvec, const SlabArgs &a, int num_sms,
                            cudaStream_t st) {
    const int grid = grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        bwd_slab_kernel<64><<<grid, kThreads, BwdCfg<64>::SMEM, st>>>(mQ, mK, mdO, mV, mP, mdS,
                                                                      lse, Dvec, a);
    else
        bwd_slab_kernel<128><<<grid, kThreads, BwdCfg<128>::SMEM, st>>>(mQ, mK, mdO, mV, mP, mdS,
                                                                        lse, Dvec, a);
    return cudaGetLastError();
}

cudaError_t launch_ring_keys(const CUtensorMap &mPt, const CUtensorMap &mdO,
                             const CUtensorMap &mdSt, const CUtensorMap &mQ, void *dK, void *dV,
                             float *acc_dK, float *acc_dV, const SlabArgs &a, int num_sms,
                             cudaStream_t st) {
    const int grid = grid_for(a.ntiles, num_sms);
    auto *k = static_cast<__nv_bfloat16 *>(dK);
    auto *v = static_cast<__nv_bfloat16 *>(dV);
    if (a.d == 64)
        ring_keys_kernel<64><<<grid, kThreads, KeysCfg<64>::SMEM, st>>>(mPt, mdO, mdSt, mQ, k, v,
                                                                        acc_dK, acc_dV, a);
    else
        ring_keys_kernel<128><<<grid, kThreads, KeysCfg<128>::SMEM, st>>>(mPt, mdO, mdSt, mQ, k, v,
                                                                          acc_dK, acc_dV, a);
    return cudaGetLastError();
}

}  // namespace rsa
