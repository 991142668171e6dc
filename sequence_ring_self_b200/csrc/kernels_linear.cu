// kernels_linear.cu -- the linear layers of the Transformer block on a chunk of rows (sm_100a).
//
// Sequence parallelism ("Sequence Parallelism: Making 4D Parallelism Possible", review page,
// Abstract) splits the whole block by the sequence: self-attention exchanges key and value
// chunks around the ring, and the block's linear layers work on their own chunk's rows with
// no exchange. Each of them is
//
//   Y[m][n] = act( sum_k X[m][k] W[n][k] + b[n] ) + R[m][n]       (act: identity or GELU)
//
// a dense contraction on the tensor cores: tiles of 128 rows x 256 columns accumulated in
// TMEM over K in blocks of 64, operands staged by TMA in 128-byte-swizzled shared memory, and
// the bias, the exact GELU (x Phi(x), with erf) and the residual applied on the way out of
// TMEM. The operand and output tensor maps also split or merge heads: a [H][M][d] tensor is
// read as the row-major [M][H d] matrix it stands for (k -> (k mod d, row, k / d)), and the
// query/key/value projection writes [3H][M][d] (n -> (n mod d, row, n / d)), so attention reads
// its operands and writes its output without any copy.
//
// Persistent and warp-specialised (320 threads): warp 0 lane 0 TMA producer, warp 1 TMEM owner
// and MMA issuer (lane 0), warps 2..9 epilogue (warp w reads TMEM lanes 32*(w%4)..+31, its rows,
// and columns 128*((w-2)/4) .. +127 of the tile in four 32-column chunks).
#include "tc_common.cuh"

namespace rsa {
namespace {

using namespace tc;

constexpr int kLinThreads = 320;

struct LinCfg {
    static constexpr int BM = 128, BN = 256, BK = 64;
    static constexpr int A_BYTES = BM * BK * 2;   // 16 KB
    static constexpr int B_BYTES = BN * BK * 2;   // 32 KB
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int EPI_BYTES = 8 * 2 * 2048;  // per epilogue warp: 2 x (32 rows x 64 B)
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + (int)sizeof(Ctl);
    static constexpr uint32_t TMEM_COLS = 512;    // two 256-column accumulators
};

// 16-byte chunk g of row r in a [32 rows][64 bytes] staging tile, 64-byte swizzle.
__device__ __forceinline__ uint32_t lin_sw64(uint32_t row, uint32_t g) {
    return row * 64u + ((g ^ ((row >> 1) & 3u)) << 4);
}

__device__ __forceinline__ float gelu_exact(float x) {
    return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

__global__ void __launch_bounds__(kLinThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mW,
                  const __grid_constant__ CUtensorMap mY, const LinArgs a) {
    using C = LinCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1024(smem_raw);
    uint8_t *stages = smem;
    uint8_t *epi = smem + C::STAGES * C::STAGE_BYTES;
    Ctl *ctl = reinterpret_cast<Ctl *>(epi + C::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = a.K / C::BK;

    if (threadIdx.x == 0) {
        init_ctl(ctl, C::STAGES, 8);
        prefetch_tmap(&mX);
        prefetch_tmap(&mW);
        prefetch_tmap(&mY);
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
                const int m0 = (t / a.nNT) * C::BM, n0 = (t % a.nNT) * C::BN;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&ctl->empty[p.stage], p.phase ^ 1u, &ctl->abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + p.stage * C::STAGE_BYTES;
                    uint64_t *bar = &ctl->full[p.stage];
                    mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
                    const int k0 = kb * C::BK;
                    tma_load_3d(sa, &mX, bar, k0 % a.x_kin, m0, k0 / a.x_kin);
                    tma_load_3d(sa + C::A_BYTES, &mW, bar, k0, n0, 0);
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
            Pipe p{0, 0};
            int acc = 0;
            uint32_t aph = 0;
            const uint32_t idesc = idesc_bf16_f32(C::BM, C::BN, 0, 0);
            constexpr uint64_t KM = sdesc_const(16, 1024);
            bool ok = true;
            for (int t = blockIdx.x; ok && t < a.ntiles; t += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[acc], aph ^ 1u, &ctl->abort)) break;
                tc_fence_after();
                const uint32_t dcol = tmem + acc * C::BN;
                for (int kb = 0; kb < nkb; ++kb) {
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
        // ------------------------------------------------------------------ epilogue
        const int ew = warp - 2, q = warp & 3, hf = ew >> 2;
        uint8_t *ebuf = epi + ew * 4096;
        int acc = 0, sb = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
            const int m0 = (t / a.nNT) * C::BM, n0 = (t % a.nNT) * C::BN;
            if (!warp_wait(&ctl->tfull[acc], aph, &ctl->abort)) break;
            tc_fence_after();
            const int m = m0 + 32 * q + lane;  // this thread's row
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
                const int col = hf * 128 + cc * 32;
                const int n = n0 + col;  // first column of this chunk
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + acc * C::BN + col, r);
                tmem_ld_wait();
                if (n >= a.N) continue;  // past the last column (N is a multiple of 64)
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
                if (a.bias) {
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 b4 = reinterpret_cast<const float4 *>(a.bias + n)[e4];
                        v[4 * e4] += b4.x, v[4 * e4 + 1] += b4.y, v[4 * e4 + 2] += b4.z, v[4 * e4 + 3] += b4.w;
                    }
                }
                if (a.gelu) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = gelu_exact(v[e]);
                }
                if (a.res) {
                    const uint4 *rp = reinterpret_cast<const uint4 *>(a.res + static_cast<size_t>(m) * a.N + n);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint4 x = rp[g];
                        const __nv_bfloat162 *xb = reinterpret_cast<const __nv_bfloat162 *>(&x);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 f = __bfloat1622float2(xb[u]);
                            v[8 * g + 2 * u] += f.x;
                            v[8 * g + 2 * u + 1] += f.y;
                        }
                    }
                }
                uint8_t *buf = ebuf + sb * 2048;
                sb ^= 1;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) w[u] = pack_bf16x2(v[8 * g + 2 * u], v[8 * g + 2 * u + 1]);
                    *reinterpret_cast<uint4 *>(buf + lin_sw64(lane, g)) = make_uint4(w[0], w[1], w[2], w[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&mY, buf, n % a.y_kin, m0 + 32 * q, n / a.y_kin);
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

}  // namespace

cudaError_t linear_kernels_configure() {
    return cudaFuncSetAttribute(linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                LinCfg::SMEM);
}

cudaError_t launch_linear(const CUtensorMap &mX, const CUtensorMap &mW, const CUtensorMap &mY,
                          const LinArgs &a, int num_sms, cudaStream_t st) {
    const int grid = tc::grid_for(a.ntiles, num_sms);
    return launch_pdl(linear_kernel, dim3(grid), dim3(kLinThreads), LinCfg::SMEM, st, mX, mW, mY, a);
}

}  // namespace rsa
