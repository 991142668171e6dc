// kernels_bwd.cu -- the backward pass of Ring Self-Attention on the key-major ring (sm_100a).
//
// "Sequence Parallelism: Making 4D Parallelism Possible" (review page, "Proposed method")
// runs the backward pass on the same ring as the forward. Seen from key chunk m, the ring
// brings every query chunk n = (m - s) mod N in turn; this kernel takes that view for a tile
// of 128 keys (K_m, V_m resident in shared memory) and visits the group's query rows in
// 64-row blocks, starting at the block of its own chunk and wrapping around:
//
//   S^T  = K_m Q_n^T,   dP^T = V_m dO_n^T                   (tcgen05, TMEM accumulators)
//   P^T  = exp(scale S^T - lse_n),  dS^T = P^T (dP^T - D_n)   (epilogue warps, fp32 -> bf16)
//   dV_m += P^T dO_n,   dK_m += scale dS^T Q_n               (tcgen05, A operand in TMEM)
//
// P never leaves the chip: it is recomputed from lse (the forward's fp32 row statistics), in
// the manner of recomputation in the backward pass. The epilogue writes P^T and dS^T as bf16
// pairs back into the TMEM columns it has just read S^T and dP^T from, and the dV/dK MMAs take
// their A operand from there. dS^T also goes to the key-major dS^T slab (plain 16-byte stores,
// 64 contiguous bytes per key row) for the dQ ring GEMM, which reads it as an MN-major operand.
//
// Roles (320 threads): warp 0 lane 0 issues TMA loads (K/V per key tile, Q/dO and the rows'
// statistics per step); warp 1 owns TMEM and lane 0 issues tcgen05.mma; warps 2..9 are the
// epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (keys) and query columns 32*((w-2)/4)..+31.
// The S^T/dP^T accumulators are double-buffered and the MMA warp issues step t's S^T/dP^T
// before step t-1's dV/dK, so the tensor core works on one step while the epilogue works on
// the previous one. MMAs of one thread execute in issue order, so step t's dV/dK MMAs read
// P^T/dS^T of buffer b before step t+2's S^T/dP^T MMAs overwrite it.
#include "tc_common.cuh"

namespace rsa {
namespace {

using namespace tc;

constexpr int kBkThreads = 320;
constexpr int kEpiWarps = 8;

template <int D>
struct BkCfg {
    static constexpr int QB = 64;                        // query rows per step
    static constexpr int KV_BYTES = 128 * D * 2;         // resident [128 keys][D] tile
    static constexpr int KV_SLOTS = 2;
    static constexpr int QT_BYTES = QB * D * 2;          // [64 queries][D] tile
    static constexpr int STAT_OFF = 2 * QT_BYTES;        // then lse*log2(e) [64] and D [64]
    static constexpr int STAGE_BYTES = 2 * QT_BYTES + 1024;
    static constexpr int STAGES = D == 64 ? 5 : 2;
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_STAGE = OFF_KV + KV_SLOTS * 2 * KV_BYTES;
    static constexpr int OFF_CTL = OFF_STAGE + STAGES * STAGE_BYTES;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: S^T[b] at 128 b, dP^T[b] at 128 b + 64, dV at 256, dK at 256 + D.
    // P^T / dS^T of step t (bf16 pairs) overwrite S^T[b] / dP^T[b]: queries 32h..32h+31 of
    // step t occupy columns 32h .. 32h + 15 of the buffer.
};

struct BkCtl {
    uint64_t full[8], empty[8];      // Q/dO stages
    uint64_t kvfull[2], kvempty[2];  // resident K/V slots
    uint64_t sfull[2];               // S^T/dP^T of buffer b computed
    uint64_t pready[2];              // P^T/dS^T of buffer b written to TMEM
    uint64_t accfull, accempty;      // dV/dK accumulators
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
constexpr int bk_smem() {
    return 1024 + BkCfg<D>::OFF_CTL + static_cast<int>(sizeof(BkCtl));
}

struct BkTile {
    int h, j0, lo, cnt, first;
};

// Work unit t = (128-key tile, head), longest causal tiles (smallest keys) first. The query
// blocks of the group that can see the keys are lo .. lo + cnt - 1; the ring starts at the
// block holding the keys' own chunk.
__device__ __forceinline__ bool bk_decode(const SlabArgs &a, int t, BkTile &tl) {
    const int kt = t / a.nh;
    tl.h = t - kt * a.nh;
    tl.j0 = kt * 128;
    const int nqb = (a.R + 63) / 64;
    int lo = 0;
    if (a.causal) lo = max(0, (tl.j0 - a.r0) / 64);
    if (lo >= nqb) return false;
    tl.lo = lo;
    tl.cnt = nqb - lo;
    const int m = tl.j0 / a.c;
    const int want = (m * a.c - a.r0) / 64;
    tl.first = min(max(want, lo), nqb - 1) - lo;
    return true;
}

// P^T = 2^(S^T * scale * log2(e) - lse * log2(e)) and dS^T = P^T (dP^T - D) for one thread's
// 32 query columns, packed to bf16 pairs. MASK zeroes the entries with key j >= L, query
// i >= the group's end, or (causal) j > i.
template <bool MASK>
__device__ __forceinline__ void epi_compute(const uint32_t (&rs)[32], const uint32_t (&rd)[32],
                                            const float *stat, float sl2, int j, int ic, int L,
                                            int r_end, int causal, uint32_t (&wp)[16],
                                            uint32_t (&wd)[16]) {
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
        const float4 l4 = reinterpret_cast<const float4 *>(stat)[e4];
        const float4 d4 = reinterpret_cast<const float4 *>(stat + 64)[e4];
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        float pv[4], sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = 4 * e4 + u;
            float p = fast_exp2(fmaf(__uint_as_float(rs[e]), sl2, -lv[u]));
            if (MASK) {
                const int i = ic + e;
                p = (j >= L || i >= r_end || (causal && j > i)) ? 0.f : p;
            }
            pv[u] = p;
            sv[u] = p * (__uint_as_float(rd[e]) - dv[u]);
        }
        wp[2 * e4] = pack_bf16x2(pv[0], pv[1]);
        wp[2 * e4 + 1] = pack_bf16x2(pv[2], pv[3]);
        wd[2 * e4] = pack_bf16x2(sv[0], sv[1]);
        wd[2 * e4 + 1] = pack_bf16x2(sv[2], sv[3]);
    }
}

__device__ __forceinline__ int bk_block(const BkTile &tl, int s) {
    return tl.lo + ring_block(tl.first, s, tl.cnt);
}

template <int D>
__global__ void __launch_bounds__(kBkThreads, 1)
    bwd_keys_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                    const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mdO,
                    const __grid_constant__ CUtensorMap mStat, __nv_bfloat16 *__restrict__ dSt,
                    __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV,
                    float *__restrict__ acc_dK, float *__restrict__ acc_dV, const SlabArgs a) {
    using C = BkCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    BkCtl *ctl = reinterpret_cast<BkCtl *>(smem + C::OFF_CTL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int s = 0; s < C::KV_SLOTS; ++s) {
            mbar_init(&ctl->kvfull[s], 1);
            mbar_init(&ctl->kvempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->sfull[b], 1);
            mbar_init(&ctl->pready[b], kEpiWarps);
        }
        mbar_init(&ctl->accfull, 1);
        mbar_init(&ctl->accempty, kEpiWarps);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mK);
        prefetch_tmap(&mV);
        prefetch_tmap(&mQ);
        prefetch_tmap(&mdO);
        prefetch_tmap(&mStat);
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
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            Pipe p{0, 0}, kv{0, 0};
            bool issued[C::STAGES], kissued[C::KV_SLOTS];
            uint32_t ipar[C::STAGES], kpar[C::KV_SLOTS];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            for (int s = 0; s < C::KV_SLOTS; ++s) kissued[s] = false, kpar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BkTile tl;
                if (!bk_decode(a, t, tl)) continue;
                const int bh = a.bh0 + tl.h;
                if (!mbar_wait(&ctl->kvempty[kv.stage], kv.phase ^ 1u, &ctl->abort)) break;
                {
                    uint8_t *ks = smem + C::OFF_KV + kv.stage * 2 * C::KV_BYTES;
                    uint64_t *bar = &ctl->kvfull[kv.stage];
                    mbar_arrive_expect_tx(bar, 2 * C::KV_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb) {
                        tma_load_3d(ks + kb * 16384, &mK, bar, kb * 64, tl.j0, bh);
                        tma_load_3d(ks + C::KV_BYTES + kb * 16384, &mV, bar, kb * 64, tl.j0, bh);
                    }
                    kissued[kv.stage] = true;
                    kpar[kv.stage] = kv.phase;
                    pipe_next(kv, C::KV_SLOTS);
                }
                for (int s = 0; s < tl.cnt; ++s) {
                    const int row = a.r0 + bk_block(tl, s) * 64;
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + C::OFF_STAGE + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, 2 * C::QT_BYTES + 512);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb) {
                        tma_load_3d(st + kb * 8192, &mQ, bar, kb * 64, row, bh);
                        tma_load_3d(st + C::QT_BYTES + kb * 8192, &mdO, bar, kb * 64, row, bh);
                    }
                    tma_load_3d(st + C::STAT_OFF, &mStat, bar, row, bh, 0);        // lse * log2(e)
                    tma_load_3d(st + C::STAT_OFF + 256, &mStat, bar, row, bh, 1);  // D
                    issued[p.stage] = true;
                    ipar[p.stage] = p.phase;
                    pipe_next(p, C::STAGES);
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) drain_wait(&ctl->full[s], ipar[s]);
            for (int s = 0; s < C::KV_SLOTS; ++s)
                if (kissued[s]) drain_wait(&ctl->kvfull[s], kpar[s]);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint64_t KM = sdesc_const(16, 1024);    // K-major, 128-byte swizzle
            constexpr uint64_t MN = sdesc_const(8192, 1024);  // MN-major, 64-wide blocks 8 KB apart
            const uint32_t id_s = idesc_bf16_f32(128, C::QB, 0, 0);  // S^T, dP^T
            const uint32_t id_g = idesc_bf16_f32(128, D, 0, 1);      // dV, dK (A in TMEM)
            const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + D;
            Pipe p{0, 0}, kv{0, 0};
            uint32_t gstep = 0, acc_ph = 0;
            bool ok = true;
            // dV/dK work of the previous step, issued after the next step's S^T/dP^T
            bool pend = false, pend_first = false;
            int pend_stage = 0;
            uint32_t pend_b = 0, pend_ph = 0;
            auto grad = [&](void) -> bool {
                if (!mbar_wait(&ctl->pready[pend_b], pend_ph, &ctl->abort)) return false;
                if (pend_first && !mbar_wait(&ctl->accempty, acc_ph ^ 1u, &ctl->abort)) return false;
                tc_fence_after();
                const uint32_t st = smem_addr(smem + C::OFF_STAGE + pend_stage * C::STAGE_BYTES);
                const uint64_t d_do = sdesc(MN, st + C::QT_BYTES), d_q = sdesc(MN, st);
                const uint32_t t_p = tmem + 128 * pend_b, t_ds = t_p + 64;
#pragma unroll
                for (int k = 0; k < C::QB / 16; ++k) {
                    const uint32_t en = (pend_first && k == 0) ? 0u : 1u;
                    const uint32_t col = (k >> 1) * 32 + (k & 1) * 8;  // 16 queries per MMA
                    tc_mma_bf16_ts(t_dv, t_p + col, d_do + 128 * k, id_g, en);
                    tc_mma_bf16_ts(t_dk, t_ds + col, d_q + 128 * k, id_g, en);
                }
                tc_commit(&ctl->empty[pend_stage]);
                pend = false;
                return true;
            };
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BkTile tl;
                if (!bk_decode(a, t, tl)) continue;
                if (!mbar_wait(&ctl->kvfull[kv.stage], kv.phase, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t ks = smem_addr(smem + C::OFF_KV + kv.stage * 2 * C::KV_BYTES);
                const uint32_t vs = ks + C::KV_BYTES;
                const uint64_t d_k = sdesc(KM, ks), d_v = sdesc(KM, vs);
                for (int s = 0; s < tl.cnt; ++s) {
                    const uint32_t b = gstep & 1u;
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    // buffer b was last read by the dV/dK MMAs of step gstep - 2, issued
                    // before these (in-order execution)
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + C::OFF_STAGE + p.stage * C::STAGE_BYTES);
                    const uint32_t t_s = tmem + 128 * b, t_p = t_s + 64;
                    const uint64_t d_q = sdesc(KM, st), d_do = sdesc(KM, st + C::QT_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t en = (kb | k) != 0 ? 1u : 0u;
                            const uint32_t ko = kb * 1024 + 2 * k, qo = kb * 512 + 2 * k;
                            tc_mma_bf16(t_s, d_k + ko, d_q + qo, id_s, en);
                            tc_mma_bf16(t_p, d_v + ko, d_do + qo, id_s, en);
                        }
                    tc_commit(&ctl->sfull[b]);
                    if (s == tl.cnt - 1) tc_commit(&ctl->kvempty[kv.stage]);
                    if (pend && !grad()) {
                        ok = false;
                        break;
                    }
                    pend = true;
                    pend_first = s == 0;
                    pend_stage = p.stage;
                    pend_b = b;
                    pend_ph = (gstep >> 1) & 1u;
                    pipe_next(p, C::STAGES);
                    ++gstep;
                }
                if (!ok) break;
                if (pend && !grad()) break;
                tc_commit(&ctl->accfull);
                acc_ph ^= 1u;
                pipe_next(kv, C::KV_SLOTS);
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 2, q = warp & 3, hf = ew >> 2;
        const float sl2 = a.scale * kLog2e;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        uint32_t gstep = 0, acc_ph = 0;
        Pipe ps{0, 0};  // the Q/dO stage of the current step (same order as the producer's)
        bool ok = true;
        for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
            BkTile tl;
            if (!bk_decode(a, t, tl)) continue;
            const int bh = a.bh0 + tl.h;
            const int j = tl.j0 + 32 * q + lane;  // this thread's key
            for (int s = 0; s < tl.cnt; ++s) {
                const uint32_t b = gstep & 1u, bph = (gstep >> 1) & 1u;
                const int i0 = a.r0 + bk_block(tl, s) * 64;
                const int ic = i0 + 32 * hf;  // first query column of this warp
                const int r_end = a.r0 + a.R;
                if (!warp_wait(&ctl->sfull[b], bph, &ctl->abort) ||
                    !warp_wait(&ctl->full[ps.stage], ps.phase, &ctl->abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_s = tmem + lane_base + 128 * b + 32 * hf;
                uint32_t rs[32], rd[32];
                tmem_ld32(t_s, rs);
                tmem_ld32(t_s + 64, rd);
                tmem_ld_wait();
                const bool masked = (a.causal && ic < tl.j0 + 128) || tl.j0 + 128 > a.L ||
                                    ic + 32 > r_end;
                // row statistics of this warp's 32 queries, loaded with the step's Q/dO stage
                const float *stat = reinterpret_cast<const float *>(
                    smem + C::OFF_STAGE + ps.stage * C::STAGE_BYTES + C::STAT_OFF) + 32 * hf;
                uint32_t wp[16], wd[16];
                if (!masked)
                    epi_compute<false>(rs, rd, stat, sl2, 0, 0, 0, 0, 0, wp, wd);
                else
                    epi_compute<true>(rs, rd, stat, sl2, j, ic, a.L, r_end, a.causal, wp, wd);
                // P^T and dS^T over the columns just read, as the dV/dK MMAs' A operands
                tmem_st16(t_s, wp);
                tmem_st16(t_s + 64, wd);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->pready[b]);
                // dS^T row j, queries [ic, ic + 32) of the key-major slab (64 contiguous bytes)
                if (j < a.L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        dSt + (static_cast<size_t>(tl.h) * a.L + j) * a.dst_pitch + (ic - a.r0));
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        dst[g] = make_uint4(wd[4 * g], wd[4 * g + 1], wd[4 * g + 2], wd[4 * g + 3]);
                }
                ++gstep;
                pipe_next(ps, C::STAGES);
            }
            if (!ok) break;
            // dV_m and dK_m of this key tile
            if (!warp_wait(&ctl->accfull, acc_ph, &ctl->abort)) break;
            tc_fence_after();
            const bool key_ok = j < a.L;
            const size_t orow = (static_cast<size_t>(bh) * a.L + (key_ok ? j : 0)) * D;
            const size_t arow = static_cast<size_t>(key_ok ? j : 0) * D;  // one head per group
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
                const float mul = which ? a.scale : 1.f;
                __nv_bfloat16 *o = which ? dK : dV;
                float *accp = which ? acc_dK : acc_dV;
#pragma unroll 1
                for (int cc = 0; cc < D / 64; ++cc) {
                    const int col = hf * (D / 2) + cc * 32;
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + 256 + which * D + col, r);
                    tmem_ld_wait();
                    if (!key_ok) continue;
                    float v[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) * mul;
                    if (a.mode != 0) {
                        float4 *ap = reinterpret_cast<float4 *>(accp + arow + col);
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
                    uint4 *op = reinterpret_cast<uint4 *>(o + orow + col);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        op[g] = make_uint4(pack_bf16x2(v[8 * g], v[8 * g + 1]),
                                           pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                           pack_bf16x2(v[8 * g + 4], v[8 * g + 5]),
                                           pack_bf16x2(v[8 * g + 6], v[8 * g + 7]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty);
            acc_ph ^= 1u;
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

cudaError_t bwd_kernels_configure() {
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bk_smem<64>());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(bwd_keys_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                bk_smem<128>());
}

cudaError_t launch_bwd_keys(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mQ,
                            const CUtensorMap &mdO, const CUtensorMap &mStat, void *dSt, void *dK,
                            void *dV, float *acc_dK, float *acc_dV, const SlabArgs &a, int num_sms,
                            cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    const int grid = tc::grid_for(a.ntiles, num_sms);
    auto *k = static_cast<__nv_bfloat16 *>(dK);
    auto *v = static_cast<__nv_bfloat16 *>(dV);
    auto *ds = static_cast<__nv_bfloat16 *>(dSt);
    if (a.d == 64)
        e = launch_pdl(bwd_keys_kernel<64>, dim3(grid), dim3(kBkThreads), bk_smem<64>(), st, mK, mV, mQ, mdO, mStat, ds, k, v, acc_dK, acc_dV, a);
    else
        e = launch_pdl(bwd_keys_kernel<128>, dim3(grid), dim3(kBkThreads), bk_smem<128>(), st, mK, mV, mQ, mdO, mStat, ds, k, v, acc_dK, acc_dV, a);
    return e;
}

}  // namespace rsa
