// kernels_fwd.cu -- the slab-free two-pass forward of Ring Self-Attention (sm_100a).
//
// Ring Self-Attention ("Sequence Parallelism: Making 4D Parallelism Possible", review page,
// "Proposed method") computes each chunk's scores against every key chunk in ring order,
// takes the softmax over the whole key length, and accumulates P V on a second ring pass.
// The slab forward (kernels_tc.cu) keeps the scores of a chunk in HBM between the passes; this
// variant recomputes them instead, so no score ever leaves the chip:
//
//   pass 1 (fwd_stats):   per query row, m = max_j s_ij and l = sum_j 2^(s_ij - m) over the
//                         ring's key blocks (s in base-2 units), lse = ln 2 (m + log2 l)
//   pass 2 (fwd_pv):      S again, P = 2^(s - lse log2(e)) in TMEM, O += P V
//
// Both passes take the query-major ring view of the backward's dQ kernel: a unit is a tile of
// 128 queries (Q copied into TMEM once with tcgen05.cp, the A operand of S = Q K^T), visiting
// key blocks of KN keys from the block of its own chunk and wrapping around. Roles (320
// threads): warp 0 lane 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 2..9 epilogue
// (TMEM lanes 32*(w%4)..+31 are its rows; keys KN/2*((w-2)/4)..+KN/2 of each block).
#include "tc_common.cuh"

namespace rsa {
namespace {

using namespace tc;

constexpr int kFwThreads = 320;
constexpr int kFwEpiWarps = 8;

template <int D>
struct FwCfg {
    static constexpr int KN = D == 64 ? 128 : 64;        // keys per step
    static constexpr int QT_BYTES = 128 * D * 2;         // [128 queries][D] tile
    static constexpr int KB_BYTES = KN * D * 2;          // [KN keys][D] block
    static constexpr int KCHUNK = KN * 128;              // one 64-column box of a block
    static constexpr uint32_t TMEM_COLS = 512;
};

struct FwUnit {
    int h, i0, cnt, first;
};

// Unit t = (128-query tile, head), longest causal tiles first; key blocks 0 .. cnt - 1 in
// ring order from the block holding the first key of the tile's own chunk.
__device__ __forceinline__ void fw_decode(const SlabArgs &a, int t, int kn, FwUnit &u) {
    const int k = t / a.nh;
    u.h = t - k * a.nh;
    const int nqt = (a.L + 127) / 128;
    const int qt = a.causal ? nqt - 1 - k : k;
    u.i0 = qt * 128;
    const int end = a.causal ? min(a.L, u.i0 + 128) : a.L;
    u.cnt = (end + kn - 1) / kn;
    const int n = u.i0 / a.c;
    u.first = min((n * a.c) / kn, u.cnt - 1);
}

__device__ __forceinline__ void fw_combine(float &m, float &l, float m2, float l2) {
    const float nm = fmaxf(m, m2);
    if (nm == -INFINITY) return;
    l = l * fast_exp2(m - nm) + l2 * fast_exp2(m2 - nm);
    m = nm;
}

// 16-byte chunk g of row r in a [32 rows][64 bytes] staging tile, 64-byte swizzle.
__device__ __forceinline__ uint32_t fw_sw64(uint32_t row, uint32_t g) {
    return row * 64u + ((g ^ ((row >> 1) & 3u)) << 4);
}

// ====================================================================== pass 1: row statistics

template <int D>
struct StCfg : FwCfg<D> {
    using B = FwCfg<D>;
    static constexpr int STAGES = 6;                      // K blocks
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGE = B::QT_BYTES;
    static constexpr int OFF_PART = OFF_STAGE + STAGES * B::KB_BYTES;  // [2][2][2][128] fp32
    static constexpr int OFF_CTL = OFF_PART + 4096;
    // TMEM: S[b] at KN b, Q (bf16 pairs, D / 2 columns) at 2 KN
    static constexpr uint32_t T_Q = 2 * B::KN;
};

struct StCtl {
    uint64_t full[8], empty[8];  // K blocks
    uint64_t qfull, qempty;      // the unit's Q tile
    uint64_t sfull[2], sfree[2]; // S[b] computed / loaded by every epilogue warp
    uint64_t dpair[4];           // both warps of rows 32q .. 32q + 31 posted their partials
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
constexpr int st_smem() {
    return 1024 + StCfg<D>::OFF_CTL + static_cast<int>(sizeof(StCtl));
}

template <int D>
__global__ void __launch_bounds__(kFwThreads, 1)
    fwd_stats_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                     float *__restrict__ lse, const SlabArgs a) {
    using C = StCfg<D>;
    constexpr int KN = C::KN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    StCtl *ctl = reinterpret_cast<StCtl *>(smem + C::OFF_CTL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->qfull, 1);
        mbar_init(&ctl->qempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->sfull[b], 1);
            mbar_init(&ctl->sfree[b], kFwEpiWarps);
        }
        for (int w = 0; w < 4; ++w) mbar_init(&ctl->dpair[w], 2);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mQ);
        prefetch_tmap(&mK);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            Pipe p{0, 0};
            uint32_t qph = 0;
            bool issued[C::STAGES], qissued = false;
            uint32_t ipar[C::STAGES], qpar = 0;
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                FwUnit u;
                fw_decode(a, t, KN, u);
                const int bh = a.bh0 + u.h;
                if (!mbar_wait(&ctl->qempty, qph ^ 1u, &ctl->abort)) break;
                mbar_arrive_expect_tx(&ctl->qfull, C::QT_BYTES);
#pragma unroll
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_3d(smem + C::OFF_Q + kb * 16384, &mQ, &ctl->qfull, kb * 64, u.i0, bh);
                qissued = true;
                qpar = qph;
                qph ^= 1u;
                for (int s = 0; s < u.cnt; ++s) {
                    const int j0 = ring_block(u.first, s, u.cnt) * KN;
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + C::OFF_STAGE + p.stage * C::KB_BYTES;
                    mbar_arrive_expect_tx(&ctl->full[p.stage], C::KB_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_3d(st + kb * C::KCHUNK, &mK, &ctl->full[p.stage], kb * 64, j0, bh);
                    issued[p.stage] = true;
                    ipar[p.stage] = p.phase;
                    pipe_next(p, C::STAGES);
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) drain_wait(&ctl->full[s], ipar[s]);
            if (qissued) drain_wait(&ctl->qfull, qpar);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint64_t KM = sdesc_const(16, 1024);  // K-major, 128-byte swizzle
            const uint32_t id_s = idesc_bf16_f32(128, KN, 0, 0);
            Pipe p{0, 0};
            uint32_t gstep = 0, qph = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                FwUnit u;
                fw_decode(a, t, KN, u);
                if (!mbar_wait(&ctl->qfull, qph, &ctl->abort)) break;
                qph ^= 1u;
                tc_fence_after();
                {
                    // Q -> TMEM (after the previous unit's S MMAs, in issue order)
                    const uint64_t d_q = sdesc(KM, smem_addr(smem + C::OFF_Q));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_cp_128x256b(tmem + C::T_Q + 8 * k, d_q + (k >> 2) * 1024 + 2 * (k & 3));
                    tc_commit(&ctl->qempty);
                }
                for (int s = 0; s < u.cnt; ++s) {
                    const uint32_t b = gstep & 1u;
                    // S[b] was loaded by every epilogue warp two steps ago
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort) ||
                        (gstep >= 2 && !mbar_wait(&ctl->sfree[b], ((gstep >> 1) & 1u) ^ 1u, &ctl->abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t d_k = sdesc(KM, smem_addr(smem + C::OFF_STAGE + p.stage * C::KB_BYTES));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ko = (k >> 2) * (C::KCHUNK >> 4) + 2 * (k & 3);
                        tc_mma_bf16_ts(tmem + KN * b, tmem + C::T_Q + 8 * k, d_k + ko, id_s, k ? 1u : 0u);
                    }
                    tc_commit(&ctl->sfull[b]);
                    tc_commit(&ctl->empty[p.stage]);
                    pipe_next(p, C::STAGES);
                    ++gstep;
                }
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        constexpr int NCH = KN / 64;  // 32-key chunks per warp and step
        const int ew = warp - 2, q = warp & 3, hf = ew >> 2;
        const float sl2 = a.scale * kLog2e;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        float *part = reinterpret_cast<float *>(smem + C::OFF_PART);
        uint32_t gstep = 0, unit = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x, ++unit) {
            FwUnit u;
            fw_decode(a, t, KN, u);
            const int bh = a.bh0 + u.h;
            const int rt = 32 * q + lane;    // this thread's row of the tile
            const int iw = u.i0 + 32 * q;   // this warp's first row
            const int i = iw + lane;         // this thread's row
            float m = -INFINITY, l = 0.f;    // over this warp's half of every key block
            for (int s = 0; s < u.cnt; ++s) {
                const uint32_t b = gstep & 1u;
                const int jw = ring_block(u.first, s, u.cnt) * KN + hf * (KN / 2);  // first key
                if (!warp_wait(&ctl->sfull[b], (gstep >> 1) & 1u, &ctl->abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[NCH][32];
#pragma unroll
                for (int c = 0; c < NCH; ++c)
                    tmem_ld32(tmem + lane_base + KN * b + hf * (KN / 2) + 32 * c, r[c]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->sfree[b]);
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int jc = jw + 32 * c;
                    const bool masked = jc + 32 > a.L || (a.causal && jc + 31 > iw);
                    float v[32], cm = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = jc + e;
                        const bool live = !masked || (j < a.L && !(a.causal && j > i));
                        v[e] = live ? __uint_as_float(r[c][e]) * sl2 : -INFINITY;
                        cm = fmaxf(cm, v[e]);
                    }
                    if (cm != -INFINITY) {
                        float cs = 0.f;
#pragma unroll
                        for (int e = 0; e < 32; ++e) cs += fast_exp2(v[e] - cm);
                        fw_combine(m, l, cm, cs);
                    }
                }
                ++gstep;
            }
            if (!ok) break;
            // join the two halves of each row, then lse = ln 2 (m + log2 l)
            float *pb = part + (unit & 1u) * 512;
            pb[hf * 256 + rt] = m;
            pb[hf * 256 + 128 + rt] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->dpair[q]);
            if (!warp_wait(&ctl->dpair[q], unit & 1u, &ctl->abort)) break;
            fw_combine(m, l, pb[(hf ^ 1) * 256 + rt], pb[(hf ^ 1) * 256 + 128 + rt]);
            if (hf == 0 && i < a.L)
                lse[static_cast<size_t>(bh) * a.L + i] = (m + __log2f(l)) * 0.6931471805599453f;
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

// ====================================================================== pass 2: O = P V

template <int D>
struct PrCfg : FwCfg<D> {
    using B = FwCfg<D>;
    static constexpr int STAGE_BYTES = 2 * B::KB_BYTES;  // K block, V block
    static constexpr int STAGES = 4;
    static constexpr int OUT_BUFS = D == 64 ? 2 : 1;     // 2 KB staging buffers per warp
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGE = B::QT_BYTES;
    static constexpr int OFF_OUT = OFF_STAGE + STAGES * STAGE_BYTES;
    static constexpr int OFF_CTL = OFF_OUT + kFwEpiWarps * OUT_BUFS * 2048;
    // TMEM: S[b] at KN b (P of the step as bf16 pairs over its first columns: keys 32g..32g+31
    // of the block in columns 32g .. 32g + 15), O at 2 KN, Q at 2 KN + D
    static constexpr uint32_t T_O = 2 * B::KN, T_Q = T_O + D;
    static_assert(T_Q + D / 2 <= B::TMEM_COLS, "TMEM columns");
};

struct PrCtl {
    uint64_t full[8], empty[8];  // K/V blocks
    uint64_t qfull, qempty;      // the unit's Q tile
    uint64_t sfull[2];           // S[b] computed
    uint64_t pready[2];          // P of buffer b written to TMEM
    uint64_t accfull, accempty;  // O accumulator
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
constexpr int pr_smem() {
    return 1024 + PrCfg<D>::OFF_CTL + static_cast<int>(sizeof(PrCtl));
}

template <int D>
__global__ void __launch_bounds__(kFwThreads, 1)
    fwd_pv_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                  const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mO,
                  const float *__restrict__ lse, const SlabArgs a) {
    using C = PrCfg<D>;
    constexpr int KN = C::KN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    PrCtl *ctl = reinterpret_cast<PrCtl *>(smem + C::OFF_CTL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->qfull, 1);
        mbar_init(&ctl->qempty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->sfull[b], 1);
            mbar_init(&ctl->pready[b], kFwEpiWarps);
        }
        mbar_init(&ctl->accfull, 1);
        mbar_init(&ctl->accempty, kFwEpiWarps);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mQ);
        prefetch_tmap(&mK);
        prefetch_tmap(&mV);
        prefetch_tmap(&mO);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            Pipe p{0, 0};
            uint32_t qph = 0;
            bool issued[C::STAGES], qissued = false;
            uint32_t ipar[C::STAGES], qpar = 0;
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                FwUnit u;
                fw_decode(a, t, KN, u);
                const int bh = a.bh0 + u.h;
                if (!mbar_wait(&ctl->qempty, qph ^ 1u, &ctl->abort)) break;
                mbar_arrive_expect_tx(&ctl->qfull, C::QT_BYTES);
#pragma unroll
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_3d(smem + C::OFF_Q + kb * 16384, &mQ, &ctl->qfull, kb * 64, u.i0, bh);
                qissued = true;
                qpar = qph;
                qph ^= 1u;
                for (int s = 0; s < u.cnt; ++s) {
                    const int j0 = ring_block(u.first, s, u.cnt) * KN;
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + C::OFF_STAGE + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb) {
                        tma_load_3d(st + kb * C::KCHUNK, &mK, bar, kb * 64, j0, bh);
                        tma_load_3d(st + C::KB_BYTES + kb * C::KCHUNK, &mV, bar, kb * 64, j0, bh);
                    }
                    issued[p.stage] = true;
                    ipar[p.stage] = p.phase;
                    pipe_next(p, C::STAGES);
                }
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) drain_wait(&ctl->full[s], ipar[s]);
            if (qissued) drain_wait(&ctl->qfull, qpar);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint64_t KM = sdesc_const(16, 1024);          // K-major, 128-byte swizzle
            constexpr uint64_t MN = sdesc_const(C::KCHUNK, 1024);   // V: MN-major, 64-wide boxes
            const uint32_t id_s = idesc_bf16_f32(128, KN, 0, 0);    // S
            const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);     // O (A = P in TMEM)
            Pipe p{0, 0};
            uint32_t gstep = 0, acc_ph = 0, qph = 0;
            bool ok = true;
            bool pend = false, pend_first = false;
            int pend_stage = 0;
            uint32_t pend_b = 0, pend_ph = 0;
            auto pv = [&](void) -> bool {
                if (!mbar_wait(&ctl->pready[pend_b], pend_ph, &ctl->abort)) return false;
                if (pend_first && !mbar_wait(&ctl->accempty, acc_ph ^ 1u, &ctl->abort)) return false;
                tc_fence_after();
                const uint64_t d_v = sdesc(MN, smem_addr(smem + C::OFF_STAGE + pend_stage * C::STAGE_BYTES +
                                                          C::KB_BYTES));
#pragma unroll
                for (int k = 0; k < KN / 16; ++k) {
                    const uint32_t en = (pend_first && k == 0) ? 0u : 1u;
                    const uint32_t col = (k >> 1) * 32 + (k & 1) * 8;  // 16 keys per MMA
                    tc_mma_bf16_ts(tmem + C::T_O, tmem + KN * pend_b + col, d_v + 128 * k, id_o, en);
                }
                tc_commit(&ctl->empty[pend_stage]);
                pend = false;
                return true;
            };
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                FwUnit u;
                fw_decode(a, t, KN, u);
                if (!mbar_wait(&ctl->qfull, qph, &ctl->abort)) break;
                qph ^= 1u;
                tc_fence_after();
                {
                    // Q -> TMEM (after the previous unit's S MMAs, in issue order)
                    const uint64_t d_q = sdesc(KM, smem_addr(smem + C::OFF_Q));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_cp_128x256b(tmem + C::T_Q + 8 * k, d_q + (k >> 2) * 1024 + 2 * (k & 3));
                    tc_commit(&ctl->qempty);
                }
                for (int s = 0; s < u.cnt; ++s) {
                    const uint32_t b = gstep & 1u;
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // S[b]: its last reader was the PV MMAs of step gstep - 2, issued earlier
                    const uint64_t d_k = sdesc(KM, smem_addr(smem + C::OFF_STAGE + p.stage * C::STAGE_BYTES));
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ko = (k >> 2) * (C::KCHUNK >> 4) + 2 * (k & 3);
                        tc_mma_bf16_ts(tmem + KN * b, tmem + C::T_Q + 8 * k, d_k + ko, id_s, k ? 1u : 0u);
                    }
                    tc_commit(&ctl->sfull[b]);
                    if (pend && !pv()) {
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
                if (pend && !pv()) break;
                tc_commit(&ctl->accfull);
                acc_ph ^= 1u;
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        constexpr int NCH = KN / 64;  // 32-key chunks per warp and step
        const int ew = warp - 2, q = warp & 3, hf = ew >> 2;
        const float sl2 = a.scale * kLog2e;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        uint8_t *obase = smem + C::OFF_OUT + ew * C::OUT_BUFS * 2048;
        uint32_t gstep = 0, acc_ph = 0;
        int obuf = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
            FwUnit u;
            fw_decode(a, t, KN, u);
            const int bh = a.bh0 + u.h;
            const int iw = u.i0 + 32 * q;  // this warp's first row
            const int i = iw + lane;        // this thread's row
            const float lse2 = i < a.L ? lse[static_cast<size_t>(bh) * a.L + i] * kLog2e : 0.f;
            const float2 sl = make_float2(sl2, sl2), nl = make_float2(-lse2, -lse2);
            for (int s = 0; s < u.cnt; ++s) {
                const uint32_t b = gstep & 1u, bph = (gstep >> 1) & 1u;
                const int jw = ring_block(u.first, s, u.cnt) * KN + hf * (KN / 2);  // first key
                if (!warp_wait(&ctl->sfull[b], bph, &ctl->abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_s = tmem + lane_base + KN * b + hf * (KN / 2);
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    uint32_t r[32], w[16];
                    tmem_ld32(t_s + 32 * c, r);
                    tmem_ld_wait();
                    const int jc = jw + 32 * c;
                    if (jc + 32 <= a.L && !(a.causal && jc + 31 > iw)) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 x = ffma2(make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])),
                                                   sl, nl);
                            w[e >> 1] = pack_bf16x2(fast_exp2(x.x), fast_exp2(x.y));
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float pr[2];
#pragma unroll
                            for (int v = 0; v < 2; ++v) {
                                const int j = jc + e + v;
                                const float p = fast_exp2(fmaf(__uint_as_float(r[e + v]), sl2, -lse2));
                                pr[v] = (j >= a.L || (a.causal && j > i)) ? 0.f : p;
                            }
                            w[e >> 1] = pack_bf16x2(pr[0], pr[1]);
                        }
                    }
                    // P over the S columns just read, as the PV MMAs' A operand
                    tmem_st16(t_s + 32 * c, w);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->pready[b]);
                ++gstep;
            }
            if (!ok) break;
            // O of this query tile, bf16, through the staging buffer
            if (!warp_wait(&ctl->accfull, acc_ph, &ctl->abort)) break;
            acc_ph ^= 1u;
            tc_fence_after();
            uint32_t r[D / 64][32];
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc)
                tmem_ld32(tmem + lane_base + C::T_O + hf * (D / 2) + 32 * cc, r[cc]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty);
            if (iw >= a.L) continue;  // the whole 32-row box lies past the sequence
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                uint8_t *buf = obase + obuf * 2048;
                obuf = obuf + 1 == C::OUT_BUFS ? 0 : obuf + 1;
                if (lane == 0) bulk_wait_read<C::OUT_BUFS - 1>();
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t v[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        v[x] = pack_bf16x2(__uint_as_float(r[cc][8 * g + 2 * x]),
                                           __uint_as_float(r[cc][8 * g + 2 * x + 1]));
                    *reinterpret_cast<uint4 *>(buf + fw_sw64(lane, g)) = make_uint4(v[0], v[1], v[2], v[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&mO, buf, hf * (D / 2) + 32 * cc, iw, bh);
                    bulk_commit();
                }
            }
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

}  // namespace

cudaError_t fwd_kernels_configure() {
    const cudaFuncAttribute smem = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(fwd_stats_kernel<64>, smem, st_smem<64>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fwd_stats_kernel<128>, smem, st_smem<128>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fwd_pv_kernel<64>, smem, pr_smem<64>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fwd_pv_kernel<128>, smem, pr_smem<128>());
    return e;
}

cudaError_t launch_fwd_stats(const CUtensorMap &mQ, const CUtensorMap &mK, float *lse,
                             const SlabArgs &a, int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        return launch_pdl(fwd_stats_kernel<64>, dim3(grid), dim3(kFwThreads), st_smem<64>(), st,
                          mQ, mK, lse, a);
    return launch_pdl(fwd_stats_kernel<128>, dim3(grid), dim3(kFwThreads), st_smem<128>(), st, mQ,
                      mK, lse, a);
}

cudaError_t launch_fwd_pv(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                          const CUtensorMap &mO, const float *lse, const SlabArgs &a, int num_sms,
                          cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        return launch_pdl(fwd_pv_kernel<64>, dim3(grid), dim3(kFwThreads), pr_smem<64>(), st, mQ,
                          mK, mV, mO, lse, a);
    return launch_pdl(fwd_pv_kernel<128>, dim3(grid), dim3(kFwThreads), pr_smem<128>(), st, mQ,
                      mK, mV, mO, lse, a);
}

}  // namespace rsa
