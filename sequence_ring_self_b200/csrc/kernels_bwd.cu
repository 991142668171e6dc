// kernels_bwd.cu -- the backward pass of Ring Self-Attention on the key-major ring (sm_100a).
//
// "Sequence Parallelism: Making 4D Parallelism Possible" (review page, "Proposed method")
// runs the backward pass on the same ring as the forward. Seen from key chunk m, the ring
// brings every query chunk n = (m - s) mod N in turn; this kernel takes that view for a tile
// of 128 keys (K_m, V_m resident on the chip: in TMEM for d = 64, in shared memory for
// d = 128) and visits the query rows in 64-row blocks, starting at the block of its own chunk
// and wrapping around:
//
//   S^T  = K_m Q_n^T,   dP^T = V_m dO_n^T                   (tcgen05, TMEM accumulators)
//   P^T  = exp(scale S^T - lse_n),  dS^T = P^T (dP^T - D_n)   (epilogue warps, fp32 -> bf16)
//   dV_m += P^T dO_n,   dK_m += scale dS^T Q_n               (tcgen05, A operand in TMEM)
//
// P never leaves the chip: it is recomputed from lse (the forward's fp32 row statistics), in
// the manner of recomputation in the backward pass. The epilogue writes P^T and dS^T as bf16
// pairs back into the TMEM columns it has just read S^T and dP^T from, and the dV/dK MMAs take
// their A operand from there. dQ comes from the row-major companion kernel below, which
// recomputes S, P, dP and dS for its query rows, so no dS slab is ever written; it runs first
// and also writes the rows' statistics (lse log2(e) and D_i = dO_i . O_i) this kernel reads.
//
// Roles (320 threads): warp 0 lane 0 issues TMA loads (K/V per key tile, Q/dO and the rows'
// statistics per step); warp 1 owns TMEM and lane 0 issues tcgen05.mma; warps 2..9 are the
// epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (keys) and query columns 32*((w-2)/4)..+31.
// The S^T/dP^T accumulators are double-buffered and the MMA warp issues a step's S^T/dP^T
// two steps ahead of its dV/dK, so the tensor core works on one step while the epilogue works
// on another. MMAs of one thread
// execute in issue order, so step t's dV/dK MMAs read P^T/dS^T of buffer b before step t+2's
// S^T/dP^T MMAs overwrite it.
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
    // d = 128: one K/V slot (the next unit's K/V load waits for the unit's last S^T/dP^T
    // MMAs, once per 128-key unit) buys four Q/dO stages: a stage is held from its S^T/dP^T
    // MMAs to its dV/dK MMAs, about a step and a half, so with two stages the producer could
    // not load step t + 2 before step t's dV/dK MMAs had finished and the MMA thread waited
    // for the load (measured: about a third of every step)
    static constexpr int KV_SLOTS = D == 64 ? 2 : 1;
    static constexpr int QT_BYTES = QB * D * 2;          // [64 queries][D] tile
    static constexpr int STAT_OFF = 2 * QT_BYTES;        // then lse*log2(e) [64] and D [64]
    static constexpr int STAGE_BYTES = 2 * QT_BYTES + 1024;
    static constexpr int STAGES = D == 64 ? 5 : 4;
    static constexpr int OUT_BUFS = D == 64 ? 2 : 1;     // 2 KB staging buffers per warp
    static constexpr int OFF_KV = 0;
    static constexpr int OFF_STAGE = OFF_KV + KV_SLOTS * 2 * KV_BYTES;
    static constexpr int OFF_OUT = OFF_STAGE + STAGES * STAGE_BYTES;
    static constexpr int OFF_CTL = OFF_OUT + kEpiWarps * OUT_BUFS * 2048;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: S^T[b] at 128 b, dP^T[b] at 128 b + 64, dV at 256, dK at 256 + D.
    // P^T / dS^T of step t (bf16 pairs) overwrite S^T[b] / dP^T[b]: queries 32h..32h+31 of
    // step t occupy columns 32h .. 32h + 15 of the buffer.
    // For d = 64 the unit's K and V tiles are also copied into TMEM (bf16 pairs, 32 columns
    // each, at T_K and T_V) and the S^T / dP^T MMAs take their A operand from there, which
    // halves their shared-memory traffic; for d = 128 the columns are all taken.
    static constexpr bool KV_TMEM = D == 64;
    static constexpr uint32_t T_K = 256 + 2 * D, T_V = T_K + D / 2;
    static_assert(!KV_TMEM || T_V + D / 2 <= TMEM_COLS, "TMEM columns");
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
    tl.j0 = a.kcol0 + kt * 128;
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
    if (!MASK) {
        // packed pairs: the exponent, dP - D and the product each one instruction per pair
        const float2 sl = make_float2(sl2, sl2);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
            const float4 l4 = reinterpret_cast<const float4 *>(stat)[e4];
            const float4 d4 = reinterpret_cast<const float4 *>(stat + 64)[e4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int e = 4 * e4 + 2 * h;
                const float2 nl = h ? make_float2(-l4.z, -l4.w) : make_float2(-l4.x, -l4.y);
                const float2 dv = h ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
                const float2 x = ffma2(make_float2(__uint_as_float(rs[e]), __uint_as_float(rs[e + 1])),
                                       sl, nl);
                const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                const float2 g = fsub2(make_float2(__uint_as_float(rd[e]), __uint_as_float(rd[e + 1])),
                                       dv);
                const float2 ds = fmul2(p, g);
                wp[e >> 1] = pack_bf16x2(p.x, p.y);
                wd[e >> 1] = pack_bf16x2(ds.x, ds.y);
            }
        }
    } else {
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
}

// 16-byte chunk g of row r in a [32 rows][64 bytes] staging tile, 64-byte swizzle (the
// chunk index is XORed with bits 7..8 of the row's byte offset).
__device__ __forceinline__ uint32_t sw64_offset(uint32_t row, uint32_t g) {
    return row * 64u + ((g ^ ((row >> 1) & 3u)) << 4);
}

__device__ __forceinline__ int bk_block(const BkTile &tl, int s) {
    return tl.lo + ring_block(tl.first, s, tl.cnt);
}

template <int D>
__global__ void __launch_bounds__(kBkThreads, 1)
    bwd_keys_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                    const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mdO,
                    const __grid_constant__ CUtensorMap mStat, const __grid_constant__ CUtensorMap mdK,
                    const __grid_constant__ CUtensorMap mdV, const SlabArgs a) {
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
        prefetch_tmap(&mdK);
        prefetch_tmap(&mdV);
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
                        tma_load_3d(st + kb * 8192, &mQ, bar, kb * 64, row - a.qrow0, bh);
                        tma_load_3d(st + C::QT_BYTES + kb * 8192, &mdO, bar, kb * 64, row - a.qrow0, bh);
                    }
                    tma_load_3d(st + C::STAT_OFF, &mStat, bar, row - a.qrow0, bh, 0);        // lse * log2(e)
                    tma_load_3d(st + C::STAT_OFF + 256, &mStat, bar, row - a.qrow0, bh, 1);  // D
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
            // S^T/dP^T run two steps ahead of dV/dK. Every barrier poll of this thread waits
            // for the MMAs it has in flight (the pipe then idles until the next issue), so the
            // loop polls once per step: pready(g), which the epilogue posts only once the Q/dO
            // stage of step g + 2 has landed too. d = 64: the unit's K and V are copied into
            // TMEM and the S^T/dP^T MMAs take A from there; d = 128: A comes from the unit's
            // K/V slot in shared memory, released after the unit's last S^T/dP^T MMAs.
            constexpr uint64_t KM = sdesc_const(16, 1024);
            constexpr uint64_t MN = sdesc_const(8192, 1024);
            const uint32_t id_s = idesc_bf16_f32(128, C::QB, 0, 0);
            const uint32_t id_g = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + D;
            struct Cursor {
                int t, s;
                BkTile tl;
                Pipe p;
            };
            auto seek = [&](Cursor &c) -> bool {  // first unit at or after c.t with work
                for (; c.t < a.ntiles; c.t += gridDim.x)
                    if (bk_decode(a, c.t, c.tl)) {
                        c.s = 0;
                        return true;
                    }
                return false;
            };
            auto advance = [&](Cursor &c) -> bool {
                pipe_next(c.p, C::STAGES);
                if (++c.s < c.tl.cnt) return true;
                c.t += gridDim.x;
                return seek(c);
            };
            Cursor is{static_cast<int>(blockIdx.x), 0, {}, {0, 0}};
            Cursor gr = is;
            bool has_is = seek(is), has_gr = seek(gr);
            Pipe kv{0, 0};
            uint32_t kslot = 0;  // d = 128: the K/V slot of the unit under `is`
            uint32_t gi = 0, gg = 0, acc_ph = 0;
            auto issue_s = [&]() -> bool {  // S^T, dP^T of the step under `is`, buffer gi & 1
                if (is.s == 0) {
                    if (!mbar_wait(&ctl->kvfull[kv.stage], kv.phase, &ctl->abort)) return false;
                    tc_fence_after();
                    if (C::KV_TMEM) {
                        // K, V -> TMEM (after every earlier S^T/dP^T MMA, in issue order)
                        const uint32_t ks = smem_addr(smem + C::OFF_KV + kv.stage * 2 * C::KV_BYTES);
                        const uint64_t d_k = sdesc(KM, ks), d_v = sdesc(KM, ks + C::KV_BYTES);
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            tc_cp_128x256b(tmem + C::T_K + 8 * k, d_k + 2 * k);
                            tc_cp_128x256b(tmem + C::T_V + 8 * k, d_v + 2 * k);
                        }
                        tc_commit(&ctl->kvempty[kv.stage]);
                        pipe_next(kv, C::KV_SLOTS);
                    } else {
                        kslot = kv.stage;
                    }
                }
                // the first two stages are not vouched for by a pready
                if (gi < 2 && !mbar_wait(&ctl->full[is.p.stage], is.p.phase, &ctl->abort))
                    return false;
                tc_fence_after();
                const uint32_t st = smem_addr(smem + C::OFF_STAGE + is.p.stage * C::STAGE_BYTES);
                const uint64_t d_q = sdesc(KM, st), d_do = sdesc(KM, st + C::QT_BYTES);
                const uint32_t t_s = tmem + 128 * (gi & 1u), t_p = t_s + 64;
                if (C::KV_TMEM) {
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        tc_mma_bf16_ts(t_s, tmem + C::T_K + 8 * k, d_q + 2 * k, id_s, k ? 1u : 0u);
                        tc_mma_bf16_ts(t_p, tmem + C::T_V + 8 * k, d_do + 2 * k, id_s, k ? 1u : 0u);
                    }
                } else {
                    const uint32_t ks = smem_addr(smem + C::OFF_KV + kslot * 2 * C::KV_BYTES);
                    const uint64_t d_k = sdesc(KM, ks), d_v = sdesc(KM, ks + C::KV_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t en = (kb | k) != 0 ? 1u : 0u;
                            const uint32_t ko = kb * 1024 + 2 * k, qo = kb * 512 + 2 * k;
                            tc_mma_bf16(t_s, d_k + ko, d_q + qo, id_s, en);
                            tc_mma_bf16(t_p, d_v + ko, d_do + qo, id_s, en);
                        }
                }
                tc_commit(&ctl->sfull[gi & 1u]);
                if (!C::KV_TMEM && is.s == is.tl.cnt - 1) {
                    tc_commit(&ctl->kvempty[kv.stage]);  // the unit's last reader of its K/V
                    pipe_next(kv, C::KV_SLOTS);
                }
                ++gi;
                has_is = advance(is);
                return true;
            };
            bool ok = true;
            if (has_is) ok = issue_s();
            if (ok && has_is) ok = issue_s();
            while (ok && has_gr) {
                const uint32_t b = gg & 1u;
                if (!mbar_wait(&ctl->pready[b], (gg >> 1) & 1u, &ctl->abort)) break;
                const bool first = gr.s == 0, last = gr.s == gr.tl.cnt - 1;
                if (first && !mbar_wait(&ctl->accempty, acc_ph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t st = smem_addr(smem + C::OFF_STAGE + gr.p.stage * C::STAGE_BYTES);
                const uint64_t d_do = sdesc(MN, st + C::QT_BYTES), d_q = sdesc(MN, st);
                const uint32_t t_p = tmem + 128 * b, t_ds = t_p + 64;
#pragma unroll
                for (int k = 0; k < C::QB / 16; ++k) {
                    const uint32_t en = (first && k == 0) ? 0u : 1u;
                    const uint32_t col = (k >> 1) * 32 + (k & 1) * 8;  // 16 queries per MMA
                    tc_mma_bf16_ts(t_dv, t_p + col, d_do + 128 * k, id_g, en);
                    tc_mma_bf16_ts(t_dk, t_ds + col, d_q + 128 * k, id_g, en);
                }
                tc_commit(&ctl->empty[gr.p.stage]);
                if (last) {
                    tc_commit(&ctl->accfull);
                    acc_ph ^= 1u;
                }
                ++gg;
                has_gr = advance(gr);
                if (has_is) ok = issue_s();
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
        uint8_t *obase = smem + C::OFF_OUT + ew * C::OUT_BUFS * 2048;
        int obuf = 0;
        uint32_t gstep = 0, acc_ph = 0;
        Pipe ps{0, 0};  // the Q/dO stage of the current step (same order as the producer's)
        bool ok = true;
        uint32_t total = 0;  // steps of this CTA (pready(g) vouches for stage g + 2)
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            BkTile tl;
            if (bk_decode(a, t, tl)) total += tl.cnt;
        }
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
                const bool masked = (a.causal && ic < tl.j0 + 128) || tl.j0 + 128 > a.kend ||
                                    ic + 32 > r_end;
                // row statistics of this warp's 32 queries, loaded with the step's Q/dO stage
                const float *stat = reinterpret_cast<const float *>(
                    smem + C::OFF_STAGE + ps.stage * C::STAGE_BYTES + C::STAT_OFF) + 32 * hf;
                uint32_t wp[16], wd[16];
                if (!masked)
                    epi_compute<false>(rs, rd, stat, sl2, 0, 0, 0, 0, 0, wp, wd);
                else
                    epi_compute<true>(rs, rd, stat, sl2, j, ic, a.kend, r_end, a.causal, wp, wd);
                // P^T and dS^T over the columns just read, as the dV/dK MMAs' A operands
                tmem_st16(t_s, wp);
                tmem_st16(t_s + 64, wd);
                tmem_st_wait();
                tc_fence_before();
                if (gstep + 2 < total) {
                    Pipe p2 = ps;
                    pipe_next(p2, C::STAGES);
                    pipe_next(p2, C::STAGES);
                    if (!warp_wait(&ctl->full[p2.stage], p2.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->pready[b]);
                ++gstep;
                pipe_next(ps, C::STAGES);
            }
            if (!ok) break;
            // dV_m and dK_m of this key tile (scale dS^T Q for dK), bf16 through the staging
            // buffer: warp (q, hf) stores keys j0 + 32q .. +31, columns hf*D/2 .. +D/2
            if (!warp_wait(&ctl->accfull, acc_ph, &ctl->abort)) break;
            tc_fence_after();
            const int jw = tl.j0 + 32 * q;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
                const float mul = which ? a.scale : 1.f;
#pragma unroll 1
                for (int cc = 0; cc < D / 64; ++cc) {
                    const int col = hf * (D / 2) + cc * 32;
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_base + 256 + which * D + col, r);
                    tmem_ld_wait();
                    if (jw >= a.kend) continue;  // the whole 32-row box lies past the key window
                    uint8_t *buf = obase + obuf * 2048;
                    obuf = obuf + 1 == C::OUT_BUFS ? 0 : obuf + 1;
                    if (lane == 0) bulk_wait_read<C::OUT_BUFS - 1>();
                    __syncwarp();
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint32_t w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            w[u] = pack_bf16x2(__uint_as_float(r[8 * g + 2 * u]) * mul,
                                               __uint_as_float(r[8 * g + 2 * u + 1]) * mul);
                        *reinterpret_cast<uint4 *>(buf + sw64_offset(lane, g)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(which ? &mdK : &mdV, buf, col, jw - a.kcol0, bh);
                        bulk_commit();
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty);
            acc_ph ^= 1u;
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


// ====================================================================== dQ on the query ring
//
// The row-major half of the backward pass. Seen from query chunk n the ring brings key
// chunk m = (n + s) mod N at step s; this kernel takes that view for a tile of 128 queries
// (Q_n, dO_n and their row statistics resident in shared memory) and visits the keys in
// blocks of KN keys, starting at the block of its own chunk and wrapping around:
//
//   S  = Q_n K_m^T,   dP = dO_n V_m^T                       (tcgen05, TMEM accumulators)
//   dS = exp(scale S - lse_n) (dP - D_n)                     (epilogue warps, fp32 -> bf16)
//   dQ_n += scale dS K_m                                      (tcgen05, A operand in TMEM)
//
// S and dP are recomputed instead of read back from the key-major kernel: the extra MMA work
// costs less than a dS slab round trip through HBM. Each thread of the epilogue owns one query
// row, so its statistics lse_i and D_i are two registers. D_i = dO_i . O_i is formed here, from
// the O tile loaded with Q and dO, and written out (with lse_i log2(e)) for the key-major
// kernel, which runs next.
//
// Roles (320 threads) as in the key-major kernel: warp 0 lane 0 issues TMA loads, warp 1
// owns TMEM and lane 0 issues tcgen05.mma, warps 2..9 are the epilogue (TMEM lanes
// 32*(w%4)..+31 are its query rows; it takes keys KN/2*((w-2)/4) .. +KN/2 of each block).
// S is double-buffered, dP single-buffered: the epilogue loads dP first and releases it
// (dpfree) before it works on S, so the next block's dP MMAs wait only for that load. (A
// schedule with dP double-buffered at d = 128, S/dP two steps ahead and one poll per step was
// measured slower: with three K/V stages the epilogue's wait for the stage two steps ahead put
// a load latency on every step.)
// Each poll of a barrier by the MMA thread stalls the tensor pipe for about a hundred cycles,
// so blocks are as wide as TMEM allows (KN = 128 keys for d = 64). Q and dO are copied into
// TMEM once per unit (tcgen05.cp) and the S and dP MMAs take them from there: with both
// operands in shared memory a 128 x 128 x 16 MMA reads 8 KB per 64 cycles, all the shared
// memory bandwidth there is, and the K/V loads of later blocks would slow it down.
// dQ leaves TMEM through a per-warp swizzled staging buffer and TMA stores.

constexpr int kBrThreads = 320;

template <int D>
struct BrCfg {
    static constexpr int KN = D == 64 ? 128 : 64;        // keys per step
    static constexpr int QT_BYTES = 128 * D * 2;         // [128 queries][D] tile
    static constexpr int SLOT_BYTES = 3 * QT_BYTES;      // Q, dO, O tiles of the unit
    // one slot: it is free again once Q and dO are in TMEM and D is formed, early in a unit
    static constexpr int Q_SLOTS = 1;
    static constexpr int KB_BYTES = KN * D * 2;          // [KN keys][D] block
    static constexpr int KCHUNK = KN * 128;              // one 64-column box of a block
    static constexpr int STAGE_BYTES = 2 * KB_BYTES;     // K block, V block
    static constexpr int STAGES = D == 64 ? 4 : 3;
    static constexpr int OUT_BUFS = D == 64 ? 2 : 1;     // 2 KB staging buffers per warp
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGE = OFF_Q + Q_SLOTS * SLOT_BYTES;
    static constexpr int OFF_OUT = OFF_STAGE + STAGES * STAGE_BYTES;
    static constexpr int OFF_PART = OFF_OUT + kEpiWarps * OUT_BUFS * 2048;  // [2][2][128] fp32
    static constexpr int OFF_CTL = OFF_PART + 2048;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: S[b] at KN b, dP at 2 KN, dQ at 3 KN, then the unit's Q and dO as bf16
    // pairs (the A operands of the S and dP MMAs, D / 2 columns each). dS of a step (bf16
    // pairs) overwrites S[b]: keys 32g .. 32g + 31 of the block occupy columns 32g .. 32g + 15.
    static constexpr uint32_t T_DP = 2 * KN, T_DQ = 3 * KN, T_Q = T_DQ + D, T_DO = T_Q + D / 2;
    static_assert(T_DO + D / 2 <= TMEM_COLS, "TMEM columns");
};

struct BrCtl {
    uint64_t full[8], empty[8];    // K/V block stages
    uint64_t qfull[2], qempty[2];  // resident Q/dO/O slots
    uint64_t sfull[2];             // S[b] and dP computed
    uint64_t dpfree;               // dP loaded by every epilogue warp
    uint64_t pready[2];            // dS of buffer b written to TMEM
    uint64_t accfull, accempty;    // dQ accumulator
    uint64_t dpair[4];             // both warps of rows 32q .. 32q + 31 posted their D partials
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
constexpr int br_smem() {
    return 1024 + BrCfg<D>::OFF_CTL + static_cast<int>(sizeof(BrCtl));
}

struct BrTile {
    int h, i0, cnt, first;
};

// Work unit t = (128-query tile, head), longest causal tiles (largest queries) first. The
// key blocks (kn keys each) the tile can see are 0 .. cnt - 1; the ring starts at the block
// holding the first key of the tile's own chunk.
__device__ __forceinline__ void br_decode(const SlabArgs &a, int t, int kn, BrTile &tl) {
    const int u = t / a.nh;
    tl.h = t - u * a.nh;
    const int nqt = (a.R + 127) / 128;
    const int qt = a.causal ? nqt - 1 - u : u;
    tl.i0 = a.r0 + qt * 128;
    const int end = a.causal ? min(a.L, tl.i0 + 128) : a.L;
    tl.cnt = (end + kn - 1) / kn;
    const int n = tl.i0 / a.c;
    tl.first = min((n * a.c) / kn, tl.cnt - 1);
}

// dS = 2^(S * scale * log2(e) - lse * log2(e)) (dP - D) for 32 keys of one query row, packed
// to bf16 pairs. MASK zeroes keys j >= L and (causal) j > i.
template <bool MASK>
__device__ __forceinline__ void br_compute(const uint32_t (&rs)[32], const uint32_t *rd, float sl2,
                                           float lse2, float Di, int j0, int i, int L, int causal,
                                           uint32_t (&wd)[16]) {
    if (!MASK) {
        // packed pairs: the exponent, dP - D and the product each one instruction per pair
        const float2 sl = make_float2(sl2, sl2), nl = make_float2(-lse2, -lse2);
        const float2 dd = make_float2(Di, Di);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float2 x = ffma2(make_float2(__uint_as_float(rs[e]), __uint_as_float(rs[e + 1])),
                                   sl, nl);
            const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            const float2 g = fsub2(make_float2(__uint_as_float(rd[e]), __uint_as_float(rd[e + 1])), dd);
            const float2 ds = fmul2(p, g);
            wd[e >> 1] = pack_bf16x2(ds.x, ds.y);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            float v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float p = fast_exp2(fmaf(__uint_as_float(rs[e + u]), sl2, -lse2));
                if (MASK) {
                    const int j = j0 + e + u;
                    p = (j >= L || (causal && j > i)) ? 0.f : p;
                }
                v[u] = p * (__uint_as_float(rd[e + u]) - Di);
            }
            wd[e >> 1] = pack_bf16x2(v[0], v[1]);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kBrThreads, 1)
    bwd_rows_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mdO,
                    const __grid_constant__ CUtensorMap mO, const __grid_constant__ CUtensorMap mK,
                    const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mdQ,
                    const float *__restrict__ lse, float *__restrict__ lse2_out,
                    float *__restrict__ d_out, const SlabArgs a) {
    using C = BrCfg<D>;
    constexpr int KN = C::KN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    BrCtl *ctl = reinterpret_cast<BrCtl *>(smem + C::OFF_CTL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int s = 0; s < C::Q_SLOTS; ++s) {
            mbar_init(&ctl->qfull[s], 1);
            // released by the copies of Q and dO into TMEM and by every epilogue warp once
            // it has formed its rows' D from the dO and O tiles
            mbar_init(&ctl->qempty[s], 1 + kEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->sfull[b], 1);
            mbar_init(&ctl->pready[b], kEpiWarps);
        }
        mbar_init(&ctl->dpfree, kEpiWarps);
        for (int w = 0; w < 4; ++w) mbar_init(&ctl->dpair[w], 2);
        mbar_init(&ctl->accfull, 1);
        mbar_init(&ctl->accempty, kEpiWarps);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mQ);
        prefetch_tmap(&mdO);
        prefetch_tmap(&mO);
        prefetch_tmap(&mK);
        prefetch_tmap(&mV);
        prefetch_tmap(&mdQ);
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
            Pipe p{0, 0}, qs{0, 0};
            bool issued[C::STAGES], qissued[C::Q_SLOTS];
            uint32_t ipar[C::STAGES], qpar[C::Q_SLOTS];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            for (int s = 0; s < C::Q_SLOTS; ++s) qissued[s] = false, qpar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BrTile tl;
                br_decode(a, t, KN, tl);
                const int bh = a.bh0 + tl.h;
                if (!mbar_wait(&ctl->qempty[qs.stage], qs.phase ^ 1u, &ctl->abort)) break;
                {
                    uint8_t *slot = smem + C::OFF_Q + qs.stage * C::SLOT_BYTES;
                    uint64_t *bar = &ctl->qfull[qs.stage];
                    mbar_arrive_expect_tx(bar, C::SLOT_BYTES);
#pragma unroll
                    for (int kb = 0; kb < D / 64; ++kb) {
                        tma_load_3d(slot + kb * 16384, &mQ, bar, kb * 64, tl.i0 - a.qrow0, bh);
                        tma_load_3d(slot + C::QT_BYTES + kb * 16384, &mdO, bar, kb * 64,
                                    tl.i0 - a.qrow0, bh);
                        tma_load_3d(slot + 2 * C::QT_BYTES + kb * 16384, &mO, bar, kb * 64,
                                    tl.i0 - a.qrow0, bh);
                    }
                    qissued[qs.stage] = true;
                    qpar[qs.stage] = qs.phase;
                    pipe_next(qs, C::Q_SLOTS);
                }
                for (int s = 0; s < tl.cnt; ++s) {
                    const int j0 = ring_block(tl.first, s, tl.cnt) * KN;
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
            for (int s = 0; s < C::Q_SLOTS; ++s)
                if (qissued[s]) drain_wait(&ctl->qfull[s], qpar[s]);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint64_t KM = sdesc_const(16, 1024);          // K-major, 128-byte swizzle
            constexpr uint64_t MN = sdesc_const(C::KCHUNK, 1024);   // MN-major, 64-wide boxes
            const uint32_t id_s = idesc_bf16_f32(128, KN, 0, 0);    // S, dP
            const uint32_t id_g = idesc_bf16_f32(128, D, 0, 1);     // dQ (A in TMEM)
            const uint32_t t_dp = tmem + C::T_DP, t_dq = tmem + C::T_DQ;
            Pipe p{0, 0}, qs{0, 0};
            uint32_t gstep = 0, acc_ph = 0;
            bool ok = true;
            bool pend = false, pend_first = false;
            int pend_stage = 0;
            uint32_t pend_b = 0, pend_ph = 0;
            auto grad = [&](void) -> bool {
                if (!mbar_wait(&ctl->pready[pend_b], pend_ph, &ctl->abort)) return false;
                if (pend_first && !mbar_wait(&ctl->accempty, acc_ph ^ 1u, &ctl->abort)) return false;
                tc_fence_after();
                const uint32_t st = smem_addr(smem + C::OFF_STAGE + pend_stage * C::STAGE_BYTES);
                const uint64_t d_k = sdesc(MN, st);
                const uint32_t t_ds = tmem + KN * pend_b;
#pragma unroll
                for (int k = 0; k < KN / 16; ++k) {
                    const uint32_t en = (pend_first && k == 0) ? 0u : 1u;
                    const uint32_t col = (k >> 1) * 32 + (k & 1) * 8;  // 16 keys per MMA
                    tc_mma_bf16_ts(t_dq, t_ds + col, d_k + 128 * k, id_g, en);
                }
                tc_commit(&ctl->empty[pend_stage]);
                pend = false;
                return true;
            };
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                BrTile tl;
                br_decode(a, t, KN, tl);
                if (!mbar_wait(&ctl->qfull[qs.stage], qs.phase, &ctl->abort)) break;
                tc_fence_after();
                {
                    // Q, dO -> TMEM (after the previous unit's S/dP MMAs, in issue order)
                    const uint32_t slot = smem_addr(smem + C::OFF_Q + qs.stage * C::SLOT_BYTES);
                    const uint64_t d_q = sdesc(KM, slot), d_do = sdesc(KM, slot + C::QT_BYTES);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t o = (k >> 2) * 1024 + 2 * (k & 3);
                        tc_cp_128x256b(tmem + C::T_Q + 8 * k, d_q + o);
                        tc_cp_128x256b(tmem + C::T_DO + 8 * k, d_do + o);
                    }
                    tc_commit(&ctl->qempty[qs.stage]);
                }
                for (int s = 0; s < tl.cnt; ++s) {
                    const uint32_t b = gstep & 1u;
                    if (!mbar_wait(&ctl->full[p.stage], p.phase, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + C::OFF_STAGE + p.stage * C::STAGE_BYTES);
                    const uint32_t t_s = tmem + KN * b;
                    const uint64_t d_k = sdesc(KM, st), d_v = sdesc(KM, st + C::KB_BYTES);
                    // S[b]: its last reader was the dQ MMAs of step gstep - 2, issued earlier
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ko = (k >> 2) * (C::KCHUNK >> 4) + 2 * (k & 3);
                        tc_mma_bf16_ts(t_s, tmem + C::T_Q + 8 * k, d_k + ko, id_s, k ? 1u : 0u);
                    }
                    // dP: every epilogue warp has loaded the previous step's dP
                    if (gstep > 0 && !mbar_wait(&ctl->dpfree, (gstep - 1) & 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t ko = (k >> 2) * (C::KCHUNK >> 4) + 2 * (k & 3);
                        tc_mma_bf16_ts(t_dp, tmem + C::T_DO + 8 * k, d_v + ko, id_s, k ? 1u : 0u);
                    }
                    tc_commit(&ctl->sfull[b]);
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
                pipe_next(qs, C::Q_SLOTS);
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
        float *part = reinterpret_cast<float *>(smem + C::OFF_PART);
        uint32_t gstep = 0, acc_ph = 0, unit = 0;
        int obuf = 0;
        Pipe qs{0, 0};
        bool ok = true;
        for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x, ++unit) {
            BrTile tl;
            br_decode(a, t, KN, tl);
            const int bh = a.bh0 + tl.h;
            const int rt = 32 * q + lane;    // this thread's row of the tile
            const int iw = tl.i0 + 32 * q;  // this warp's first query row
            const int i = iw + lane;         // this thread's query row
            const float lse_i =
                i < a.r0 + a.R ? lse[static_cast<size_t>(bh) * a.Lq + (i - a.qrow0)] : 0.f;
            if (!warp_wait(&ctl->qfull[qs.stage], qs.phase, &ctl->abort)) break;
            // D_i = dO_i . O_i: this warp's half of the columns, then the other half's partial
            // through shared memory (rows past L are zero-filled, so their D is 0)
            const uint8_t *slot = smem + C::OFF_Q + qs.stage * C::SLOT_BYTES;
            float dpart = 0.f;
#pragma unroll
            for (int g = hf * (D / 16); g < (hf + 1) * (D / 16); ++g) {
                const uint32_t off = (g >> 3) * 16384 + sw128_offset(rt, g & 7);
                const uint4 x = *reinterpret_cast<const uint4 *>(slot + C::QT_BYTES + off);
                const uint4 y = *reinterpret_cast<const uint4 *>(slot + 2 * C::QT_BYTES + off);
                const __nv_bfloat162 *xb = reinterpret_cast<const __nv_bfloat162 *>(&x);
                const __nv_bfloat162 *yb = reinterpret_cast<const __nv_bfloat162 *>(&y);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 u = __bfloat1622float2(xb[e]), w = __bfloat1622float2(yb[e]);
                    dpart = fmaf(u.x, w.x, dpart);
                    dpart = fmaf(u.y, w.y, dpart);
                }
            }
            float *pb = part + (unit & 1u) * 256;
            pb[hf * 128 + rt] = dpart;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->dpair[q]);
            if (!warp_wait(&ctl->dpair[q], unit & 1u, &ctl->abort)) break;
            const float Di = dpart + pb[(hf ^ 1) * 128 + rt];
            const float lse2 = lse_i * kLog2e;
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->qempty[qs.stage]);
            pipe_next(qs, C::Q_SLOTS);
            // the rows' statistics for the key-major kernel, padded with zeros to Lp
            if (hf == 0 && i - a.qrow0 < a.Lpq) {
                lse2_out[static_cast<size_t>(bh) * a.Lpq + (i - a.qrow0)] = lse2;
                d_out[static_cast<size_t>(bh) * a.Lpq + (i - a.qrow0)] = Di;
            }
            for (int s = 0; s < tl.cnt; ++s) {
                const uint32_t b = gstep & 1u, bph = (gstep >> 1) & 1u;
                const int jw = ring_block(tl.first, s, tl.cnt) * KN + hf * (KN / 2);  // first key
                if (!warp_wait(&ctl->sfull[b], bph, &ctl->abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_s = tmem + lane_base + KN * b + hf * (KN / 2);
                uint32_t rd[NCH][32], rs[32];
#pragma unroll
                for (int c = 0; c < NCH; ++c) tmem_ld32(tmem + lane_base + C::T_DP + hf * (KN / 2) + 32 * c, rd[c]);
                tmem_ld32(t_s, rs);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->dpfree);
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    if (c > 0) {
                        tmem_ld32(t_s + 32 * c, rs);
                        tmem_ld_wait();
                    }
                    const int jc = jw + 32 * c;
                    uint32_t wd[16];
                    if (jc + 32 <= a.L && !(a.causal && jc + 31 > iw))
                        br_compute<false>(rs, rd[c], sl2, lse2, Di, 0, 0, 0, 0, wd);
                    else
                        br_compute<true>(rs, rd[c], sl2, lse2, Di, jc, i, a.L, a.causal, wd);
                    // dS over the S columns just read, as the dQ MMAs' A operand
                    tmem_st16(t_s + 32 * c, wd);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->pready[b]);
                ++gstep;
            }
            if (!ok) break;
            // dQ of this query tile: scale * accumulator, bf16, through the staging buffer
            if (!warp_wait(&ctl->accfull, acc_ph, &ctl->abort)) break;
            acc_ph ^= 1u;
            tc_fence_after();
            uint32_t r[D / 64][32];
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc)
                tmem_ld32(tmem + lane_base + C::T_DQ + hf * (D / 2) + 32 * cc, r[cc]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty);
            if (iw >= a.r0 + a.R) continue;  // the whole 32-row box lies past the rows held
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                uint8_t *buf = obase + obuf * 2048;
                obuf = obuf + 1 == C::OUT_BUFS ? 0 : obuf + 1;
                if (lane == 0) bulk_wait_read<C::OUT_BUFS - 1>();
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        w[u] = pack_bf16x2(__uint_as_float(r[cc][8 * g + 2 * u]) * a.scale,
                                           __uint_as_float(r[cc][8 * g + 2 * u + 1]) * a.scale);
                    *reinterpret_cast<uint4 *>(buf + sw64_offset(lane, g)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&mdQ, buf, hf * (D / 2) + 32 * cc, iw - a.qrow0, bh);
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

cudaError_t bwd_kernels_configure() {
    const cudaFuncAttribute smem = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<64>, smem, bk_smem<64>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_keys_kernel<128>, smem, bk_smem<128>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_rows_kernel<64>, smem, br_smem<64>());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(bwd_rows_kernel<128>, smem, br_smem<128>());
    return e;
}

cudaError_t launch_bwd_keys(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mQ,
                            const CUtensorMap &mdO, const CUtensorMap &mStat,
                            const CUtensorMap &mdK, const CUtensorMap &mdV, const SlabArgs &a,
                            int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        return launch_pdl(bwd_keys_kernel<64>, dim3(grid), dim3(kBkThreads), bk_smem<64>(), st,
                          mK, mV, mQ, mdO, mStat, mdK, mdV, a);
    return launch_pdl(bwd_keys_kernel<128>, dim3(grid), dim3(kBkThreads), bk_smem<128>(), st, mK,
                      mV, mQ, mdO, mStat, mdK, mdV, a);
}

cudaError_t launch_bwd_rows(const CUtensorMap &mQ, const CUtensorMap &mdO, const CUtensorMap &mO,
                            const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mdQ,
                            const float *lse, float *lse2_out, float *d_out, const SlabArgs &a,
                            int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    if (a.d == 64)
        return launch_pdl(bwd_rows_kernel<64>, dim3(grid), dim3(kBrThreads), br_smem<64>(), st,
                          mQ, mdO, mO, mK, mV, mdQ, lse, lse2_out, d_out, a);
    return launch_pdl(bwd_rows_kernel<128>, dim3(grid), dim3(kBrThreads), br_smem<128>(), st, mQ,
                      mdO, mO, mK, mV, mdQ, lse, lse2_out, d_out, a);
}

}  // namespace rsa
