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
// The forward's two kernels (the backward's are in kernels_bwd.cu), persistent and
// warp-specialised (320 threads = 10 warps):
//   warp 0 lane 0 : TMA producer (global -> shared, 128-byte swizzle, mbarrier pipeline)
//   warp 1        : allocates TMEM; lane 0 issues tcgen05.mma and commits to mbarriers
//   warps 2..9    : epilogue; warp w reads TMEM lanes 32*(w%4)..+31 (one tile row each)
//
//   qk_slab     (ring pass 1)      S = scale * Q K^T, masked, fp32 slab + softmax partials
//   pv_softmax  (softmax, pass 2)  P = softmax(S) formed on the chip, O = P V
#include "tc_common.cuh"

namespace rsa {
namespace {

using namespace tc;

// ======================================================================================
// qk_slab: S = log2(e) * scale * Q_i . K_j for row i, key j (fp32 scores in base-2 units;
// -inf where j >= L or causal j > i), and per row and 128-column half tile the softmax
// partials (max_j S, sum_j 2^(S - max)) that pv_softmax combines into each row's statistics.
// Tile = 128 query rows x 256 keys; K-loop over d in blocks of 64 (one 128-byte swizzle row).
// Slab layout: per (head, 128-row tile) of the group, the key chunks of 32 one after the other,
// each a contiguous [128 rows][32 keys] block (16 KB), so that ring pass 2 streams whole 16 KB
// blocks from HBM instead of 128-byte row pieces a slab row apart.
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

// Tiles are (head, 128-row tile, 256-column tile of the key window [kcol0, kend)); causal
// tiles right of the diagonal are skipped. The column tiles of a row tile start at the block
// holding its own chunk's keys.
__device__ __forceinline__ bool qk_decode(const SlabArgs &a, int t, QkTile &tl) {
    const int per_head = a.nRT * a.nCT;
    tl.h = t / per_head;
    const int rem = t - tl.h * per_head;
    const int rt = rem / a.nCT;
    const int cti = rem - rt * a.nCT;
    tl.i0 = a.r0 + rt * 128;
    int live = a.nCT;
    if (a.causal) live = min(a.nCT, (min(a.kend, tl.i0 + 128) - a.kcol0 + 255) / 256);
    if (cti >= live) return false;
    const int n = tl.i0 / a.c;
    const int first = min(max((n * a.c - a.kcol0) / 256, 0), live - 1);
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
                    tma_load_3d(sa, &mQ, bar, kb * 64, tl.i0 - a.qrow0, a.bh0 + tl.h);
                    tma_load_3d(sa + C::A_BYTES, &mK, bar, kb * 64, a.kcol0 + tl.ct * C::BN,
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
                const int j0 = a.kcol0 + tl.ct * C::BN + col;
                float v[32];
                float cm = -INFINITY;
                if (j0 + 32 <= a.kend && (!a.causal || j0 + 31 <= i_min)) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        v[e] = __uint_as_float(r[e]) * sl2;
                        cm = fmaxf(cm, v[e]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = j0 + e;
                        const bool live = j < a.kend && !(a.causal && j > i);
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
                    // slab tile (head, row tile) holds [key chunk of 32][128 rows][32 keys]
                    tma_store_4d(&mS, buf, 0, 32 * q, (j0 - a.kcol0) >> 5,
                                 tl.h * a.nRT + ((tl.i0 - a.r0) >> 7));
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            if (i < a.r0 + a.R)
                a.stats[(static_cast<size_t>(tl.h) * a.R + (i - a.r0)) * a.nStat + a.stat0 + 2 * tl.ct + hf] =
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
// pv_softmax: the row softmax and ring pass 2 in one kernel.
//   P[i][j] = 2^(S[i][j] - m_i - log2 l_i),   O_i = sum over the ring of P[i][block m] V_m
// where (m_i, l_i) combine the per-row partials that qk_slab left (max and sum of 2^(s - max)
// per 128 key columns), and lse_i = ln 2 (m_i + log2 l_i) is written for the backward pass.
// Work unit: (128-row tile, head), longest causal tiles first; the key blocks (64 keys) of a
// unit are visited in ring order from the block of the tile's own chunk. Per step the
// producer loads the fp32 score block (two 32-column boxes, 128 rows) and the V block; the
// epilogue warps turn the scores into bf16 P in TMEM (key k of the block in column k / 2 of
// the buffer, two keys per column) and the MMA thread accumulates O += P V with P as the TMEM
// operand. P never goes back to HBM: the slab is read once, in fp32.
// Roles: warp 0 lane 0 TMA producer, warp 1 TMEM owner and MMA issuer, then EW epilogue warps:
// warp w reads TMEM lanes 32*(w%4)..+31 (its rows) and takes KS = 256 / EW keys of each block
// (slice (w-2)/4). 8 epilogue warps (32 keys each); d = 64: two CTAs per SM (2 stages, 97 KB of
// shared memory and 256 TMEM columns apiece); d = 128: one CTA per SM with 4 stages. (16
// epilogue warps of 16 keys at d = 128 were measured slower: twice the barrier hand-offs per
// block for the same work.)
// ======================================================================================
template <int D>
struct PvCfg {
    static constexpr int EW = 8;                      // epilogue warps
    static constexpr int THREADS = 64 + 32 * EW;
    static constexpr int KS = 256 / EW;               // keys of a block per epilogue warp
    static constexpr int OCOLS = D / (EW / 4);        // O columns stored per epilogue warp
    static constexpr int S_BYTES = 128 * 64 * 4;      // [128 rows][64 keys] fp32, two 16 KB boxes
    static constexpr int V_BYTES = 64 * D * 2;        // [64 keys][D] bf16
    static constexpr int STAGE_BYTES = S_BYTES + V_BYTES;
    static constexpr int CTAS = D == 64 ? 2 : 1;
    static constexpr int STAGES = D == 64 ? 2 : 4;
    static constexpr int OFF_OUT = STAGES * STAGE_BYTES;  // 2 KB staging buffer per warp
    static constexpr int OFF_CTL = OFF_OUT + EW * 2048;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t T_O = 64;            // P[b] at 32 b (bf16 pairs), O at 64
    static_assert(T_O + D <= TMEM_COLS, "TMEM columns");
    static_assert(OCOLS % 32 == 0 && KS % 16 == 0, "epilogue slices");
};

struct PvCtl {
    uint64_t full[8], empty[8];  // score / V stages
    uint64_t pready[2];          // P of buffer b written to TMEM
    uint64_t pfree[2];           // the MMAs that read P of buffer b are done
    uint64_t accfull, accempty;  // O accumulator
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <int D>
constexpr int pv_smem() {
    return 1024 + PvCfg<D>::OFF_CTL + static_cast<int>(sizeof(PvCtl));
}

struct PvTile {
    int h, i0, nkb, first;
};

// Units are (128-row tile, head), longest causal tiles first.
__device__ __forceinline__ void pv_decode(const SlabArgs &a, int t, PvTile &tl) {
    const int rt = a.nRT - 1 - t / a.nh;
    tl.h = t - (t / a.nh) * a.nh;
    tl.i0 = a.r0 + rt * 128;
    const int live_end = a.causal ? min(a.L, tl.i0 + 128) : a.L;
    tl.nkb = (live_end + 63) / 64;
    const int n = tl.i0 / a.c;
    tl.first = min((n * a.c) / 64, tl.nkb - 1);
}

// 16-byte chunk g of row r in a [32 rows][64 bytes] staging tile, 64-byte swizzle.
__device__ __forceinline__ uint32_t pv_sw64(uint32_t row, uint32_t g) {
    return row * 64u + ((g ^ ((row >> 1) & 3u)) << 4);
}

// P = 2^(s - ml) for the KS scores of one row (16-byte chunks c0 .. c0 + KS/4 - 1 of the row in
// a 128-byte-swizzled [128 rows][32 keys] fp32 box), as bf16 pairs
template <int KS>
__device__ __forceinline__ void pv_probs(const uint8_t *box, uint32_t row, uint32_t c0, float ml,
                                         uint32_t (&w)[KS / 2]) {
    const float2 m2 = make_float2(ml, ml);
#pragma unroll
    for (int c = 0; c < KS / 4; ++c) {
        const float4 x = *reinterpret_cast<const float4 *>(box + sw128_offset(row, c0 + c));
        const float2 lo = fsub2(make_float2(x.x, x.y), m2);
        const float2 hi = fsub2(make_float2(x.z, x.w), m2);
        w[2 * c] = pack_bf16x2(fast_exp2(lo.x), fast_exp2(lo.y));
        w[2 * c + 1] = pack_bf16x2(fast_exp2(hi.x), fast_exp2(hi.y));
    }
}

template <int D>
__global__ void __launch_bounds__(PvCfg<D>::THREADS, PvCfg<D>::CTAS)
    pv_softmax_kernel(const __grid_constant__ CUtensorMap mS, const __grid_constant__ CUtensorMap mV,
                      const __grid_constant__ CUtensorMap mO, float *__restrict__ lse,
                      const SlabArgs a) {
    using C = PvCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    PvCtl *ctl = reinterpret_cast<PvCtl *>(smem + C::OFF_CTL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->pready[b], C::EW);
            mbar_init(&ctl->pfree[b], 1);
        }
        mbar_init(&ctl->accfull, 1);
        mbar_init(&ctl->accempty, C::EW);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        prefetch_tmap(&mS);
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
            bool issued[C::STAGES];
            uint32_t ipar[C::STAGES];
            for (int s = 0; s < C::STAGES; ++s) issued[s] = false, ipar[s] = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                PvTile tl;
                pv_decode(a, t, tl);
                for (int s = 0; s < tl.nkb; ++s) {
                    const int j0 = ring_block(tl.first, s, tl.nkb) * 64;
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    const int tile = tl.h * a.nRT + ((tl.i0 - a.r0) >> 7);
                    tma_load_4d(st, &mS, bar, 0, 0, j0 >> 5, tile);
                    tma_load_4d(st + 16384, &mS, bar, 0, 0, (j0 >> 5) + 1, tile);
#pragma unroll
                    for (int dp = 0; dp < D / 64; ++dp)
                        tma_load_3d(st + C::S_BYTES + dp * 8192, &mV, bar, dp * 64, j0,
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
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint64_t MN = sdesc_const(8192, 1024);  // V: MN-major, 64-wide blocks
            const uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t t_o = tmem + C::T_O;
            Pipe p{0, 0};
            uint32_t gstep = 0, acc_ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                PvTile tl;
                pv_decode(a, t, tl);
                for (int s = 0; s < tl.nkb; ++s) {
                    const uint32_t b = gstep & 1u;
                    if (!mbar_wait(&ctl->pready[b], (gstep >> 1) & 1u, &ctl->abort) ||
                        (s == 0 && !mbar_wait(&ctl->accempty, acc_ph ^ 1u, &ctl->abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dv = sdesc(MN, smem_addr(smem + p.stage * C::STAGE_BYTES + C::S_BYTES));
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // 16 keys per MMA, P columns 8k .. 8k + 7
                        tc_mma_bf16_ts(t_o, tmem + 32 * b + 8 * k, dv + 128 * k, idesc,
                                       (s | k) != 0 ? 1u : 0u);
                    tc_commit(&ctl->empty[p.stage]);
                    tc_commit(&ctl->pfree[b]);
                    pipe_next(p, C::STAGES);
                    ++gstep;
                }
                if (!ok) break;
                tc_commit(&ctl->accfull);
                acc_ph ^= 1u;
            }
            tc_commit(&ctl->drain);
            drain_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 2, q = warp & 3, ks = ew >> 2;  // ks: this warp's key slice
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        uint8_t *obuf = smem + C::OFF_OUT + ew * 2048;
        // the slice's keys in the score block: box (ks * KS) / 32, 16-byte chunks from c0
        const int kbox = (ks * C::KS) / 32;
        const uint32_t c0 = ((ks * C::KS) % 32) / 4;
        uint32_t gstep = 0, acc_ph = 0;
        Pipe p{0, 0};
        bool ok = true;
        for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
            PvTile tl;
            pv_decode(a, t, tl);
            const int bh = a.bh0 + tl.h;
            const int iw = tl.i0 + 32 * q;  // this warp's first row
            const int i = iw + lane;         // this thread's row
            // the row's softmax statistics from the slab GEMM's partials
            float ml = 0.f;
            if (i < a.r0 + a.R) {
                // causal: the partials of the windows up to the one holding the tile's last
                // live key (each window holds 2 * ceil(wlen / 256) slots)
                int nlive = a.nStat;
                if (a.causal) {
                    const int end = min(a.L, (i / 128) * 128 + 128);
                    const int wl = (end - 1) / a.wlen;
                    nlive = wl * 2 * ((a.wlen + 255) / 256) + 2 * ((end - wl * a.wlen + 255) / 256);
                }
                const float2 *st = a.stats + (static_cast<size_t>(tl.h) * a.R + (i - a.r0)) * a.nStat;
                float m = -INFINITY, l = 0.f;
                for (int k = 0; k < nlive; ++k) {
                    const float2 x = st[k];
                    softmax_combine(m, l, x.x, x.y);
                }
                ml = m + __log2f(l);
                if (ks == 0)
                    lse[static_cast<size_t>(bh) * a.Lq + (i - a.qrow0)] = ml * 0.6931471805599453f;
            }
            for (int s = 0; s < tl.nkb; ++s) {
                const uint32_t b = gstep & 1u, bph = (gstep >> 1) & 1u;
                // scores of this step landed; P[b] is no longer read by the MMAs of step - 2
                if (!warp_wait(&ctl->full[p.stage], p.phase, &ctl->abort) ||
                    !warp_wait(&ctl->pfree[b], bph ^ 1u, &ctl->abort)) {
                    ok = false;
                    break;
                }
                const uint8_t *box = smem + p.stage * C::STAGE_BYTES + kbox * 16384;
                uint32_t w[C::KS / 2];
                pv_probs<C::KS>(box, 32 * q + lane, c0, ml, w);
                tc_fence_after();
                const uint32_t tcol = tmem + lane_base + 32 * b + (ks * C::KS) / 2;
                if constexpr (C::KS == 32)
                    tmem_st16(tcol, w);
                else
                    tmem_st8(tcol, w);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->pready[b]);
                pipe_next(p, C::STAGES);
                ++gstep;
            }
            if (!ok) break;
            // O of this tile, bf16, through the staging buffer: OCOLS columns per warp
            if (!warp_wait(&ctl->accfull, acc_ph, &ctl->abort)) break;
            acc_ph ^= 1u;
            tc_fence_after();
            uint32_t r[C::OCOLS / 32][32];
#pragma unroll
            for (int cc = 0; cc < C::OCOLS / 32; ++cc)
                tmem_ld32(tmem + lane_base + C::T_O + ks * C::OCOLS + 32 * cc, r[cc]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty);
            if (iw >= a.r0 + a.R) continue;  // the whole 32-row box lies past the group's rows
#pragma unroll
            for (int cc = 0; cc < C::OCOLS / 32; ++cc) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = pack_bf16x2(__uint_as_float(r[cc][8 * g + 2 * u]),
                                           __uint_as_float(r[cc][8 * g + 2 * u + 1]));
                    *reinterpret_cast<uint4 *>(obuf + pv_sw64(lane, g)) = make_uint4(v[0], v[1], v[2], v[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&mO, obuf, ks * C::OCOLS + 32 * cc, iw - a.qrow0, bh);
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
    RSA_SMEM(pv_softmax_kernel<64>, pv_smem<64>())
    RSA_SMEM(pv_softmax_kernel<128>, pv_smem<128>())
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

cudaError_t launch_pv_softmax(const CUtensorMap &mS, const CUtensorMap &mV, const CUtensorMap &mO,
                              float *lse, const SlabArgs &a, int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms * (a.d == 64 ? PvCfg<64>::CTAS : PvCfg<128>::CTAS));
    if (a.d == 64)
        return launch_pdl(pv_softmax_kernel<64>, dim3(grid), dim3(PvCfg<64>::THREADS), pv_smem<64>(),
                          st, mS, mV, mO, lse, a);
    return launch_pdl(pv_softmax_kernel<128>, dim3(grid), dim3(PvCfg<128>::THREADS), pv_smem<128>(),
                      st, mS, mV, mO, lse, a);
}

}  // namespace rsa
