// rsa_abi.cu -- C ABI of the Ring Self-Attention library: argument checks, the slab-group
// planner, TMA descriptor set-up and the per-group kernel schedule.
//
// Ring Self-Attention ("Sequence Parallelism: Making 4D Parallelism Possible", review page,
// Abstract and "Proposed method") cuts the sequence into N chunks and lets each chunk see
// every key chunk in ring order. Here all chunks live in one GPU's HBM; the score slabs of
// the chunks (c x L each, L x L per head) are produced, normalised and consumed group by
// group so that the workspace stays within a budget. A group is a set of whole heads, or a
// range of rows (a multiple of 128) of one head when a whole head does not fit.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <math.h>
#include <mutex>
#include <stdio.h>
#include <string.h>
#include <vector>

#include "../../include/rsa.h"
#include "../../include/rsa_sp.h"
#include "rsa_internal.h"

namespace rsa {
__device__ int g_status_word;  // RSA_OK or RSA_ERR_TIMEOUT, set by kernels
}

namespace {

using rsa::Group;
using rsa::SlabArgs;

constexpr size_t kAlign = 256;
constexpr size_t kDefaultBudget = size_t(4) << 30;
constexpr int kMaxDevices = 64;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// What the last RSA_ERR_CUDA of the calling thread came from (see rsa_last_error).
thread_local char g_err[320];

rsa_status_t cuda_fail(const char *what, int code, const char *name) {
    snprintf(g_err, sizeof(g_err), "%s failed: %s (%d)", what, name ? name : "?", code);
    return RSA_ERR_CUDA;
}

rsa_status_t cuda_fail(const char *what, cudaError_t e) {
    return cuda_fail(what, static_cast<int>(e), cudaGetErrorName(e));
}

struct Plan {
    int B, H, L, d, N, causal, bwd;
    rsa_dtype_t dt;
    long long BH;
    int Lp, c;
    int whole;     // every group holds whole heads (R == L)
    long long Gh;  // heads per group
    int R;         // rows per group (a multiple of 128, or L)
    long long gt;  // row groups per head: ceil(L / R)
    long long ngroups;
    size_t row_bytes;   // slab bytes per row (all slabs of the pass)
    size_t slab_bytes;  // slab region
    size_t off_D, total;
};

bool args_ok(int B, int H, int L, int d, int N, rsa_dtype_t dt, rsa_status_t *why) {
    if (B <= 0 || H <= 0 || L <= 0 || N <= 0 || d <= 0 || L % N != 0) {
        *why = RSA_ERR_INVALID_ARG;
        return false;
    }
    // work units (B*H heads x 128-row tiles) are counted in 32-bit ints by the kernels
    const long long BH = static_cast<long long>(B) * H;
    if (L > (1 << 22) || BH > 0x7fffffffLL || BH * ((L + 127) / 128) > 0x3fffffffLL) {
        *why = RSA_ERR_UNSUPPORTED;
        return false;
    }
    if (dt == RSA_BF16) {
        if (d != 64 && d != 128) {
            *why = RSA_ERR_UNSUPPORTED;
            return false;
        }
    } else if (dt == RSA_F32) {
        if (d != 32 && d != 64) {
            *why = RSA_ERR_UNSUPPORTED;
            return false;
        }
    } else {
        *why = RSA_ERR_UNSUPPORTED;
        return false;
    }
    return true;
}

// The softmax / ring-pass-2 kernel runs a slab group's (head, 128-row tile) units on one CTA
// each, all units of a group alike in length (each streams its rows' scores), so a group takes
// about ceil(units / slots) rounds of one unit's time, slots being the CTAs the kernel keeps
// resident: 148 SMs (B200) times its CTAs per SM (2 at d = 64, 1 at d = 128). One CTA
// streams at a small share of HBM's bandwidth (measured about 40 GB/s), so a round with few
// units leaves HBM idle: a group is costed in whole rounds.
constexpr long long kSms = 148;
long long pv_slots(int d) { return kSms * (d == 64 ? 2 : 1); }

// bf16 forward: groups are rectangles of Gh heads x R rows (R = rt * 128, or L). Among the
// rectangles that fit the budget, take the one whose groups take the fewest rounds in total,
// then the fewest groups. Head counts are enumerated by their distinct balanced values.
void plan_rect(Plan &p, size_t budget) {
    const long long nRT = (p.L + 127) / 128;
    const size_t tile_bytes = size_t(128) * p.row_bytes;  // one 128-row tile of one head
    const size_t head_bytes = size_t(nRT) * tile_bytes;   // the slab stores whole 128-row tiles
    const long long fit_tiles = static_cast<long long>(budget / tile_bytes);
    const long long fit_heads = static_cast<long long>(budget / head_bytes);
    long long best_cost = -1, best_groups = 0, best_nh = 1, best_rt = 1;
    const long long slots = pv_slots(p.d);
    auto rounds = [slots](long long u) { return (u + slots - 1) / slots; };
    // the plan's total rounds for nh heads x rt tiles per group (the last row group of a head
    // takes the remaining tiles; `balance` first spreads the tiles evenly over the row groups)
    auto consider = [&](long long nh, long long rt, bool balance) {
        const long long ngh = (p.BH + nh - 1) / nh, last_h = p.BH - (ngh - 1) * nh;
        long long ngt = (nRT + rt - 1) / rt;
        const long long rt2 = balance ? (nRT + ngt - 1) / ngt : rt;
        ngt = (nRT + rt2 - 1) / rt2;
        const long long last_t = nRT - (ngt - 1) * rt2;
        const long long cost = (ngh - 1) * (ngt - 1) * rounds(nh * rt2) + (ngh - 1) * rounds(nh * last_t) +
                               (ngt - 1) * rounds(last_h * rt2) + rounds(last_h * last_t);
        const long long groups = ngh * ngt;
        if (best_cost < 0 || cost < best_cost || (cost == best_cost && groups < best_groups)) {
            best_cost = cost;
            best_groups = groups;
            best_nh = nh;
            best_rt = rt2;
        }
    };
    for (long long gh = 1; gh <= p.BH;) {
        const long long nh = (p.BH + gh - 1) / gh;  // heads per group with gh head groups
        long long rt_max = 0;
        if (fit_heads >= nh)
            rt_max = nRT;
        else if (fit_tiles >= nh)
            rt_max = fit_tiles / nh;
        if (rt_max > 0) {
            consider(nh, rt_max, true);
            // tile counts that make a group a whole number of rounds
            for (long long k = 1; k <= 64; ++k) {
                const long long rt = k * slots / nh;
                if (rt < 1) continue;
                if (rt >= rt_max) break;
                consider(nh, rt, false);
                consider(nh, rt, true);
            }
        }
        if (nh == 1) break;
        gh = (p.BH + nh - 2) / (nh - 1);  // the next head-group count with fewer heads per group
    }
    // nothing fits: the smallest plan (one 128-row tile of one head)
    p.Gh = best_nh;
    p.R = best_rt * 128 >= p.L ? p.L : static_cast<int>(best_rt * 128);
    p.whole = p.R == p.L;
    p.gt = (p.L + p.R - 1) / p.R;
    p.ngroups = ((p.BH + p.Gh - 1) / p.Gh) * p.gt;
    // whole 128-row tiles: the scores (4 Lp bytes a row) first, then the partials
    const size_t rows = size_t(p.Gh) * ((p.R + 127) / 128) * 128;
    p.slab_bytes = align_up(rows * p.Lp * 4, kAlign) + align_up(rows * (p.row_bytes - p.Lp * 4), kAlign);
    p.off_D = p.slab_bytes;
    p.total = p.off_D;
}

// Largest plan whose workspace fits `budget` (the smallest plan if none does).
Plan make_plan(int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt, int bwd,
               size_t budget) {
    Plan p{};
    p.B = B, p.H = H, p.L = L, p.d = d, p.N = N, p.causal = causal ? 1 : 0, p.bwd = bwd ? 1 : 0;
    p.dt = dt;
    p.BH = static_cast<long long>(B) * H;
    p.Lp = (L + 63) / 64 * 64;
    p.c = L / N;
    p.gt = 1;
    // backward: padded row statistics D and lse * log2(e), [2][BH][Lp] fp32
    const size_t fixed = bwd ? align_up(size_t(2) * p.BH * p.Lp * 4, kAlign) : 0;
    if (bwd && dt == RSA_BF16) {
        // the bf16 backward recomputes every score tile on the chip: no slab, one group
        p.whole = 1;
        p.Gh = p.BH;
        p.R = L;
        p.ngroups = 1;
        p.row_bytes = 0;
        p.slab_bytes = 0;
        p.off_D = 0;
        p.total = fixed;
        return p;
    }
    // forward: fp32 scores (4 B per score; the fp32 path writes P over them); backward (fp32
    // path): fp32 P and dS (8 B)
    p.row_bytes = bwd ? size_t(8) * p.Lp : size_t(4) * p.Lp;
    if (!bwd && dt == RSA_BF16) {
        // plus the per-row softmax partials, one float2 per 128 columns
        p.row_bytes += size_t(8) * 2 * ((p.Lp + 255) / 256);
        plan_rect(p, budget);
        return p;
    }
    const size_t head_bytes = align_up(size_t(L) * p.row_bytes, kAlign);
    if (budget >= fixed + head_bytes) {
        p.whole = 1;
        long long gh = static_cast<long long>((budget - fixed) / head_bytes);
        p.Gh = gh < p.BH ? gh : p.BH;
        p.R = L;
        p.ngroups = (p.BH + p.Gh - 1) / p.Gh;
        p.slab_bytes = align_up(size_t(p.Gh) * L * p.row_bytes, kAlign);
        p.off_D = p.slab_bytes;
        p.total = p.off_D + fixed;
    } else {
        p.whole = 0;
        p.Gh = 1;
        size_t avail = budget > fixed ? budget - fixed : 0;
        long long r = static_cast<long long>(avail / p.row_bytes) / 128 * 128;
        if (r < 128) r = 128;
        if (r >= L) r = L;  // only when L <= 128: a whole head is the minimum plan
        if (r == L) {
            p.whole = 1;
            p.R = L;
            p.ngroups = p.BH;
            p.slab_bytes = head_bytes;
            p.off_D = p.slab_bytes;
            p.total = p.off_D + fixed;
            return p;
        }
        p.R = static_cast<int>(r);
        p.gt = (L + p.R - 1) / p.R;
        p.ngroups = p.BH * p.gt;
        p.slab_bytes = align_up(size_t(p.R) * p.row_bytes, kAlign);
        p.off_D = p.slab_bytes;
        p.total = p.off_D + fixed;
    }
    return p;
}

// Group g of a plan: head group g / gt, row group g % gt.
Group group_of(const Plan &p, long long g) {
    Group G{};
    const long long hg = g / p.gt, rg = g - hg * p.gt;
    G.bh0 = static_cast<int>(hg * p.Gh);
    const long long nh = p.BH - hg * p.Gh;
    G.nh = static_cast<int>(nh < p.Gh ? nh : p.Gh);
    G.r0 = static_cast<int>(rg * p.R);
    G.R = p.L - G.r0 < p.R ? p.L - G.r0 : p.R;
    G.first_of_head = G.r0 == 0;
    G.last_of_head = G.r0 + G.R == p.L;
    return G;
}

// ---------------------------------------------------------------- per-device state

struct DeviceState {
    bool ready;
    int sms;
    int *status;
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

rsa_status_t device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return RSA_ERR_UNSUPPORTED;
    // make the device's primary context current on this thread: the tensor maps are encoded
    // through the driver API, which needs one, possibly before any launch of this thread
    e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_fail("cudaSetDevice", e);
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &s = g_dev[dev];
    if (!s.ready) {
        int major = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
        if (major != 10) return RSA_ERR_UNSUPPORTED;
        e = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
        if ((e = rsa::tc_kernels_configure()) != cudaSuccess ||
            (e = rsa::bwd_kernels_configure()) != cudaSuccess ||
            (e = rsa::fwd_kernels_configure()) != cudaSuccess ||
            (e = rsa::linear_kernels_configure()) != cudaSuccess)
            return cuda_fail("cudaFuncSetAttribute", e);
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, rsa::g_status_word);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress", e);
        s.status = static_cast<int *>(ptr);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || !fn)
                return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0, nullptr);
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        s.ready = true;
    }
    *out = &s;
    return RSA_OK;
}

// ---------------------------------------------------------------- per-kernel timing

enum Kind {
    K_QK_SLAB, K_SOFTMAX, K_PV, K_ROWDOT, K_BWD_KEYS, K_BWD_ROWS,
    K_F32_QK, K_F32_PV, K_F32_BWD, K_F32_KEYS, K_F32_DQ, K_FWD_STATS, K_FWD_PV, K_SP_ACC, K_LINEAR, K_COUNT
};
const char *kKindNames[K_COUNT] = {
    "qk_slab", "slab_softmax", "pv_softmax", "rowdot", "bwd_keys", "bwd_rows",
    "f32_qk_slab", "f32_pv_ring_rows", "f32_bwd_slab", "f32_ring_keys", "f32_dq_ring_rows",
    "fwd_stats", "fwd_pv", "sp_accumulate", "linear"};

struct ProfRec {
    int kind;
    cudaEvent_t a, b;
};
std::mutex g_prof_mutex;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t pool_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

void drop_records() {
    for (auto &r : g_prof) {
        g_pool.push_back(r.a);
        g_pool.push_back(r.b);
    }
    g_prof.clear();
}

// Launch helper: brackets the launch with events when profiling is on.
template <class F>
rsa_status_t timed(int kind, cudaStream_t s, F &&launch) {
    cudaEvent_t a = nullptr, b = nullptr;
    if (g_prof_on) {
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        a = pool_event();
        b = pool_event();
        if (!a || !b) return cuda_fail("cudaEventCreate", 0, nullptr);
        const cudaError_t e = cudaEventRecord(a, s);
        if (e != cudaSuccess) return cuda_fail("cudaEventRecord", e);
    }
    const cudaError_t e = launch();
    if (e != cudaSuccess) return cuda_fail(kKindNames[kind], e);
    if (a) {
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        const cudaError_t e2 = cudaEventRecord(b, s);
        if (e2 != cudaSuccess) return cuda_fail("cudaEventRecord", e2);
        g_prof.push_back({kind, a, b});
    }
    return RSA_OK;
}

#define RSA_LAUNCH(kind, expr)                                                   \
    do {                                                                         \
        rsa_status_t st_ = timed(kind, s, [&]() -> cudaError_t { return (expr); }); \
        if (st_ != RSA_OK) return st_;                                           \
    } while (0)

// 3-D tiled tensor map (128-byte swizzle unless told otherwise), zero fill out of bounds.
bool map3d(CUtensorMap *m, CUtensorMapDataType type, const void *base, uint64_t d0, uint64_t d1,
           uint64_t d2, uint64_t pitch1, uint64_t pitch2, uint32_t box0, uint32_t box1,
           CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {pitch1, pitch2};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, type, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_err, sizeof(g_err),
                 "cuTensorMapEncodeTiled failed (%d): base %p dims %llu x %llu x %llu box %u x %u",
                 static_cast<int>(r), base, static_cast<unsigned long long>(d0),
                 static_cast<unsigned long long>(d1), static_cast<unsigned long long>(d2), box0,
                 box1);
        return false;
    }
    return true;
}

// The fp32 score slab of `tiles` (head, 128-row tile) units whose key chunks of 32 are
// contiguous [128 rows][32 keys] blocks, `chunks` of them per unit and `unit_chunks` between
// units: a 4-D tensor (32 keys, 128 rows, chunks, tiles), 128-byte swizzle, box (32, box_rows).
bool map_slab(CUtensorMap *m, void *base, uint64_t chunks, uint64_t unit_chunks, uint64_t tiles,
              uint32_t box_rows) {
    cuuint64_t dims[4] = {32, 128, chunks, tiles};
    cuuint64_t strides[3] = {128, 16384, unit_chunks * 16384};
    cuuint32_t box[4] = {32, box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_err, sizeof(g_err),
                 "cuTensorMapEncodeTiled failed (%d): slab base %p chunks %llu of %llu tiles %llu",
                 static_cast<int>(r), base, static_cast<unsigned long long>(chunks),
                 static_cast<unsigned long long>(unit_chunks), static_cast<unsigned long long>(tiles));
        return false;
    }
    return true;
}

// Input tensor [BH][L][d] bf16, box of 64 columns x `rows` rows.
bool map_input(CUtensorMap *m, const void *base, const Plan &p, uint32_t rows) {
    return map3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, p.d, p.L, p.BH, uint64_t(p.d) * 2,
                 uint64_t(p.L) * p.d * 2, 64, rows);
}

// Output tensor [BH][L][d] bf16 written by TMA stores of 32 x 32 boxes (64-byte swizzle).
bool map_output(CUtensorMap *m, void *base, const Plan &p) {
    return map3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, p.d, p.L, p.BH, uint64_t(p.d) * 2,
                 uint64_t(p.L) * p.d * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

SlabArgs slab_args(const Plan &p, const Group &G, int *status) {
    SlabArgs a{};
    a.L = p.L, a.Lp = p.Lp, a.N = p.N, a.c = p.c, a.causal = p.causal, a.d = p.d;
    a.bh0 = G.bh0, a.nh = G.nh, a.r0 = G.r0, a.R = G.R;
    a.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(p.d)));
    a.nRT = (G.R + 127) / 128;
    a.status = status;
    a.qrow0 = 0, a.Lq = p.L, a.Lpq = p.Lp;
    a.kcol0 = 0, a.kend = p.L, a.wlen = p.L, a.stat0 = 0;
    return a;
}

#define RSA_TRY(expr)                                          \
    do {                                                       \
        const cudaError_t e_ = (expr);                         \
        if (e_ != cudaSuccess) return cuda_fail(#expr, e_);    \
    } while (0)

rsa_status_t check_common(const Plan &p, void *ws, size_t ws_bytes) {
    if (p.total > ws_bytes) return RSA_ERR_WORKSPACE;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return RSA_ERR_INVALID_ARG;
    return RSA_OK;
}


// ---------------------------------------------------------------- sequence-parallel layout

// One rank's share of the sequence-parallel ring: rows [rank c, (rank + 1) c) of every head.
struct SpLayout {
    long long BH;
    int c, Lp, nCT, nStat;
    size_t slab_bytes, part_bytes, fwd_total, bwd_total;
};

bool sp_args_ok(int B, int H, int L, int d, int P, int rank, int m, rsa_status_t *why) {
    if (!args_ok(B, H, L, d, P, RSA_BF16, why)) return false;
    if (rank < 0 || rank >= P || m < 0 || m >= P) {
        *why = RSA_ERR_INVALID_ARG;
        return false;
    }
    // whole 128-row tiles per rank; key chunks aligned with the kernels' 64/128-key blocks
    if ((L / P) % 128 != 0) {
        *why = RSA_ERR_UNSUPPORTED;
        return false;
    }
    return true;
}

SpLayout sp_layout(int B, int H, int L, int P) {
    SpLayout y{};
    y.BH = static_cast<long long>(B) * H;
    y.c = L / P;
    y.Lp = L;  // a multiple of 128
    y.nCT = (y.c + 255) / 256;
    y.nStat = P * 2 * y.nCT;
    y.slab_bytes = align_up(size_t(y.BH) * y.c * y.Lp * 4, kAlign);
    y.part_bytes = align_up(size_t(y.BH) * y.c * y.nStat * 8, kAlign);
    y.fwd_total = y.slab_bytes + y.part_bytes;
    y.bwd_total = align_up(size_t(2) * y.BH * y.c * 4, kAlign);
    return y;
}

SlabArgs sp_slab_args(const SpLayout &y, int L, int d, int P, int rank, int causal, int *status) {
    SlabArgs a{};
    a.L = L, a.Lp = y.Lp, a.N = P, a.c = y.c, a.causal = causal ? 1 : 0, a.d = d;
    a.bh0 = 0, a.nh = static_cast<int>(y.BH), a.r0 = rank * y.c, a.R = y.c;
    a.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(d)));
    a.nRT = y.c / 128;
    a.status = status;
    a.qrow0 = rank * y.c, a.Lq = y.c, a.Lpq = y.c;
    a.kcol0 = 0, a.kend = L, a.wlen = y.c, a.stat0 = 0;
    a.nCT = y.nCT, a.nStat = y.nStat;
    return a;
}

// bf16 [BH][rows][d] tensor, boxes of 64 columns x box_rows rows (128-byte swizzle)
bool map_rows(CUtensorMap *m, const void *base, long long BH, int rows, int d, uint32_t box_rows) {
    return map3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d, rows, BH, uint64_t(d) * 2,
                 uint64_t(rows) * d * 2, 64, box_rows);
}

// bf16 [BH][rows][d] output written by 32 x 32 TMA stores (64-byte swizzle)
bool map_rows_out(CUtensorMap *m, void *base, long long BH, int rows, int d) {
    return map3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d, rows, BH, uint64_t(d) * 2,
                 uint64_t(rows) * d * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

bool ws_ok(const void *ws) { return ws && (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) == 0; }

// The travelling accumulator of the backward ring (rsa_sp_accumulate): 8 elements per thread
// where the tail allows, one otherwise.
__global__ void sp_accumulate_kernel(float *__restrict__ acc, const __nv_bfloat16 *__restrict__ part,
                                     __nv_bfloat16 *__restrict__ out, long long n, int first) {
    const long long nv = n / 8;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < nv; v += stride) {
        float x[8];
        if (first) {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = 0.f;
        } else {
            const float4 a0 = reinterpret_cast<const float4 *>(acc)[2 * v];
            const float4 a1 = reinterpret_cast<const float4 *>(acc)[2 * v + 1];
            x[0] = a0.x, x[1] = a0.y, x[2] = a0.z, x[3] = a0.w;
            x[4] = a1.x, x[5] = a1.y, x[6] = a1.z, x[7] = a1.w;
        }
        if (part) {
            const uint4 p = reinterpret_cast<const uint4 *>(part)[v];
            const __nv_bfloat162 *pb = reinterpret_cast<const __nv_bfloat162 *>(&p);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(pb[e]);
                x[2 * e] += f.x;
                x[2 * e + 1] += f.y;
            }
        }
        reinterpret_cast<float4 *>(acc)[2 * v] = make_float4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<float4 *>(acc)[2 * v + 1] = make_float4(x[4], x[5], x[6], x[7]);
        if (out) {
            uint4 o;
            uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
                ow[e] = *reinterpret_cast<uint32_t *>(&b);
            }
            reinterpret_cast<uint4 *>(out)[v] = o;
        }
    }
    for (long long i = nv * 8 + blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n; i += stride) {
        float x = first ? 0.f : acc[i];
        if (part) x += __bfloat162float(part[i]);
        acc[i] = x;
        if (out) out[i] = __float2bfloat16_rn(x);
    }
}

}  // namespace

bool rsa::check_args(int B, int H, int L, int d, int N, rsa_dtype_t dt, rsa_status_t *why) {
    return args_ok(B, H, L, d, N, dt, why);
}

rsa_status_t rsa::check_device() {
    DeviceState *s = nullptr;
    return device_state(&s);
}

rsa_status_t rsa::record_cuda_failure(const char *what, cudaError_t e) { return cuda_fail(what, e); }

namespace {
// Writes `code` into the device status word from the GPU, as a kernel whose bounded wait gave
// up does (see rsa_debug_report_status).
__global__ void report_status_kernel(int *word, int code) { atomicExch(word, code); }
}  // namespace

extern "C" {

rsa_status_t rsa_debug_report_status(int code, void *stream) {
    if (code != RSA_OK && code != RSA_ERR_TIMEOUT) return RSA_ERR_INVALID_ARG;
    DeviceState *s = nullptr;
    const rsa_status_t st = device_state(&s);
    if (st != RSA_OK) return st;
    report_status_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(s->status, code);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? RSA_OK : cuda_fail("report_status_kernel", e);
}

const char *rsa_status_string(rsa_status_t s) {
    switch (s) {
        case RSA_OK: return "RSA_OK";
        case RSA_ERR_INVALID_ARG: return "RSA_ERR_INVALID_ARG";
        case RSA_ERR_UNSUPPORTED: return "RSA_ERR_UNSUPPORTED";
        case RSA_ERR_WORKSPACE: return "RSA_ERR_WORKSPACE";
        case RSA_ERR_CUDA: return "RSA_ERR_CUDA";
        case RSA_ERR_TIMEOUT: return "RSA_ERR_TIMEOUT";
    }
    return "RSA_ERR_UNKNOWN";
}

size_t rsa_workspace_size(int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                          int for_backward, size_t budget_bytes) {
    rsa_status_t why;
    if (!args_ok(B, H, L, d, N, dt, &why)) return 0;
    const Plan p = make_plan(B, H, L, d, N, causal, dt, for_backward,
                             budget_bytes ? budget_bytes : kDefaultBudget);
    return p.total;
}

rsa_status_t rsa_plan_describe(int B, int H, int L, int d, int N, int causal, rsa_dtype_t dt,
                               int for_backward, size_t ws_bytes, long long out[5]) {
    rsa_status_t why;
    if (!out) return RSA_ERR_INVALID_ARG;
    if (!args_ok(B, H, L, d, N, dt, &why)) return why;
    const Plan p = make_plan(B, H, L, d, N, causal, dt, for_backward, ws_bytes);
    out[0] = p.ngroups;
    out[1] = p.Gh;
    out[2] = p.R;
    out[3] = p.Lp;
    out[4] = static_cast<long long>(p.total);
    return p.total > ws_bytes ? RSA_ERR_WORKSPACE : RSA_OK;
}

const char *rsa_last_error(void) { return g_err; }

rsa_status_t rsa_profile_enable(int on) {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    drop_records();
    g_prof_on = on != 0;
    return RSA_OK;
}

int rsa_profile_kinds(void) { return K_COUNT; }

const char *rsa_profile_kind_name(int kind) {
    return kind >= 0 && kind < K_COUNT ? kKindNames[kind] : nullptr;
}

rsa_status_t rsa_profile_read(double *ms, long long *launches) {
    if (!ms || !launches) return RSA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    rsa_status_t st = RSA_OK;
    for (auto &r : g_prof) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
            st = RSA_ERR_CUDA;
            continue;
        }
        ms[r.kind] += t;
        launches[r.kind] += 1;
    }
    drop_records();
    return st;
}

rsa_status_t rsa_last_device_status(void *stream) {
    DeviceState *s = nullptr;
    rsa_status_t st = device_state(&s);
    if (st != RSA_OK) return st;
    RSA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int v = 0;
    RSA_TRY(cudaMemcpy(&v, s->status, sizeof(int), cudaMemcpyDeviceToHost));
    const int zero = 0;
    RSA_TRY(cudaMemcpy(s->status, &zero, sizeof(int), cudaMemcpyHostToDevice));
    return static_cast<rsa_status_t>(v);
}

rsa_status_t rsa_forward(const void *Q, const void *K, const void *V, void *O, float *lse, int B,
                         int H, int L, int d, int N, int causal, rsa_dtype_t dt, void *workspace,
                         size_t ws_bytes, void *stream) {
    rsa_status_t why;
    if (!args_ok(B, H, L, d, N, dt, &why)) return why;
    if (!Q || !K || !V || !O || !lse) return RSA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(lse))
        return RSA_ERR_INVALID_ARG;
    const Plan p = make_plan(B, H, L, d, N, causal, dt, 0, ws_bytes);
    rsa_status_t st = check_common(p, workspace, ws_bytes);
    if (st != RSA_OK) return st;
    DeviceState *dev = nullptr;
    st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *slab = static_cast<float *>(workspace);

    if (dt == RSA_F32) {
        for (long long g = 0; g < p.ngroups; ++g) {
            const Group G = group_of(p, g);
            SlabArgs a = slab_args(p, G, dev->status);
            RSA_LAUNCH(K_F32_QK, rsa::launch_f32_qk_slab(static_cast<const float *>(Q),
                                            static_cast<const float *>(K), slab, a, s));
            RSA_LAUNCH(K_SOFTMAX, rsa::launch_slab_softmax(slab, lse, a, 0, s));
            a.scale = 1.f;
            RSA_LAUNCH(K_F32_PV, rsa::launch_f32_ring_rows(slab, static_cast<const float *>(V),
                                              static_cast<float *>(O), a, s));
        }
        return RSA_OK;
    }

    CUtensorMap mQ, mK, mV, mO;
    if (!map_input(&mQ, Q, p, 128) || !map_input(&mK, K, p, 256) || !map_input(&mV, V, p, 64) ||
        !map_output(&mO, O, p))
        return RSA_ERR_CUDA;
    for (long long g = 0; g < p.ngroups; ++g) {
        const Group G = group_of(p, g);
        SlabArgs a = slab_args(p, G, dev->status);
        // the slab: per (head, 128-row tile) unit, Lp / 32 contiguous [128 rows][32 keys] blocks
        const uint64_t chunks = uint64_t(p.Lp) / 32, tiles = uint64_t(G.nh) * a.nRT;
        a.nCT = (p.Lp + 255) / 256;
        a.nStat = 2 * a.nCT;
        a.stats = reinterpret_cast<float2 *>(reinterpret_cast<uint8_t *>(slab) +
                                             align_up(tiles * chunks * 16384, kAlign));
        CUtensorMap mS, mSld;
        if (!map_slab(&mS, slab, chunks, chunks, tiles, 32) ||
            !map_slab(&mSld, slab, chunks, chunks, tiles, 128))
            return RSA_ERR_CUDA;
        // ring pass 1: score slab and per-row softmax partials
        a.ntiles = G.nh * a.nRT * a.nCT;
        RSA_LAUNCH(K_QK_SLAB, rsa::launch_qk_slab(mQ, mK, mS, a, dev->sms, s));
        // row softmax over the full key length and ring pass 2, O = P V
        a.ntiles = G.nh * a.nRT;
        RSA_LAUNCH(K_PV, rsa::launch_pv_softmax(mSld, mV, mO, lse, a, dev->sms, s));
    }
    return RSA_OK;
}

rsa_status_t rsa_forward_recompute(const void *Q, const void *K, const void *V, void *O,
                                   float *lse, int B, int H, int L, int d, int N, int causal,
                                   rsa_dtype_t dt, void *stream) {
    rsa_status_t why;
    if (!args_ok(B, H, L, d, N, dt, &why)) return why;
    if (dt != RSA_BF16) return RSA_ERR_UNSUPPORTED;
    if (!Q || !K || !V || !O || !lse) return RSA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(lse))
        return RSA_ERR_INVALID_ARG;
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // one group of every head and row: nothing but Q, K, V, O and lse lives in HBM
    const Plan p = make_plan(B, H, L, d, N, causal, dt, 1, 0);
    const uint32_t kn = d == 64 ? 128 : 64;  // keys per step
    CUtensorMap mQ, mK, mV, mO;
    if (!map_input(&mQ, Q, p, 128) || !map_input(&mK, K, p, kn) || !map_input(&mV, V, p, kn) ||
        !map_output(&mO, O, p))
        return RSA_ERR_CUDA;
    SlabArgs a = slab_args(p, group_of(p, 0), dev->status);
    a.ntiles = static_cast<int>(p.BH) * ((L + 127) / 128);
    // pass 1: per-row max and sum over the ring -> lse
    RSA_LAUNCH(K_FWD_STATS, rsa::launch_fwd_stats(mQ, mK, lse, a, dev->sms, s));
    // pass 2: S again, P = 2^(S log2(e) scale - lse log2(e)) on the chip, O = P V
    RSA_LAUNCH(K_FWD_PV, rsa::launch_fwd_pv(mQ, mK, mV, mO, lse, a, dev->sms, s));
    return RSA_OK;
}

rsa_status_t rsa_backward(const void *Q, const void *K, const void *V, const void *O,
                          const void *dO, const float *lse, void *dQ, void *dK, void *dV, int B,
                          int H, int L, int d, int N, int causal, rsa_dtype_t dt, void *workspace,
                          size_t ws_bytes, void *stream) {
    rsa_status_t why;
    if (!args_ok(B, H, L, d, N, dt, &why)) return why;
    const void *ptrs[] = {Q, K, V, O, dO, lse, dQ, dK, dV};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return RSA_ERR_INVALID_ARG;
    const Plan p = make_plan(B, H, L, d, N, causal, dt, 1, ws_bytes);
    rsa_status_t st = check_common(p, workspace, ws_bytes);
    if (st != RSA_OK) return st;
    DeviceState *dev = nullptr;
    st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // row statistics [2][BH][Lp]: lse * log2(e), then D
    float *lse2 = reinterpret_cast<float *>(ws + p.off_D);
    float *Dvec = lse2 + size_t(p.BH) * p.Lp;
    const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(d)));

    if (dt == RSA_F32) {
        // D_i = dO_i . O_i, in rows padded to Lp
        RSA_LAUNCH(K_ROWDOT, rsa::launch_rowdot(dO, O, lse, Dvec, nullptr, p.BH, L, p.Lp, d, 0, s));
    }

    if (dt == RSA_F32) {
        for (long long g = 0; g < p.ngroups; ++g) {
            const Group G = group_of(p, g);
            SlabArgs a = slab_args(p, G, dev->status);
            float *P = reinterpret_cast<float *>(ws);
            float *dS = P + size_t(G.nh) * G.R * p.Lp;
            const float *q = static_cast<const float *>(Q), *k = static_cast<const float *>(K);
            RSA_LAUNCH(K_F32_BWD, rsa::launch_f32_bwd_slab(q, k, static_cast<const float *>(dO),
                                             static_cast<const float *>(V), lse, Dvec, P, dS, a, s));
            const int accum = G.first_of_head ? 0 : 1;
            RSA_LAUNCH(K_F32_KEYS, rsa::launch_f32_ring_keys(P, static_cast<const float *>(dO),
                                              static_cast<float *>(dV), 1.f, accum, a, s));
            RSA_LAUNCH(K_F32_KEYS, rsa::launch_f32_ring_keys(dS, q, static_cast<float *>(dK), scale, accum, a, s));
            a.scale = scale;
            RSA_LAUNCH(K_F32_DQ, rsa::launch_f32_ring_rows(dS, k, static_cast<float *>(dQ), a, s));
        }
        return RSA_OK;
    }

    // Two kernels over the whole problem (one group): the query-major ring gives dQ (and the
    // rows' D and lse * log2(e)), then the key-major ring gives dK and dV; both recompute S and
    // dP tile by tile from Q, K, V, dO and the row statistics, so nothing but the statistics
    // goes through HBM.
    CUtensorMap mK128, mV128, mQ64, mdO64, mStat64, mQ128, mdO128, mO128, mK64, mV64;
    CUtensorMap mdQ, mdK, mdV;
    const uint64_t stat_pitch = uint64_t(p.Lp) * 4;
    if (!map_input(&mK128, K, p, 128) || !map_input(&mV128, V, p, 128) ||
        !map_input(&mQ64, Q, p, 64) || !map_input(&mdO64, dO, p, 64) ||
        !map_input(&mQ128, Q, p, 128) || !map_input(&mdO128, dO, p, 128) ||
        !map_input(&mO128, O, p, 128) || !map_input(&mK64, K, p, 64) ||
        !map_input(&mV64, V, p, 64) ||
        !map3d(&mStat64, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lse2, p.Lp, p.BH, 2, stat_pitch,
               stat_pitch * p.BH, 64, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map_output(&mdQ, dQ, p) || !map_output(&mdK, dK, p) || !map_output(&mdV, dV, p))
        return RSA_ERR_CUDA;
    const Group G = group_of(p, 0);
    SlabArgs a = slab_args(p, G, dev->status);
    a.mode = 0;
    a.ntiles = G.nh * ((L + 127) / 128);
    // query-major ring: S, dP -> dS in TMEM; dQ_n = scale * sum_m dS_nm K_m
    // (blocks of 128 keys for d = 64, of 64 keys for d = 128)
    const CUtensorMap &mKr = d == 64 ? mK128 : mK64, &mVr = d == 64 ? mV128 : mV64;
    RSA_LAUNCH(K_BWD_ROWS, rsa::launch_bwd_rows(mQ128, mdO128, mO128, mKr, mVr, mdQ, lse, lse2,
                                                Dvec, a, dev->sms, s));
    // key-major ring: P^T, dP^T -> dS^T in TMEM; dV_m, dK_m over all query blocks
    RSA_LAUNCH(K_BWD_KEYS, rsa::launch_bwd_keys(mK128, mV128, mQ64, mdO64, mStat64, mdK, mdV, a,
                                                dev->sms, s));
    return RSA_OK;
}

// ---------------------------------------------------------------- sequence-parallel steps

size_t rsa_sp_workspace_size(int B, int H, int L, int d, int P, int causal, int for_backward) {
    (void)causal;
    rsa_status_t why;
    if (!sp_args_ok(B, H, L, d, P, 0, 0, &why)) return 0;
    const SpLayout y = sp_layout(B, H, L, P);
    return for_backward ? y.bwd_total : y.fwd_total;
}

rsa_status_t rsa_sp_scores(const void *Q, const void *Kfull, int B, int H, int L, int d, int P,
                           int rank, int m, int causal, void *workspace, size_t ws_bytes,
                           void *stream) {
    rsa_status_t why;
    if (!sp_args_ok(B, H, L, d, P, rank, m, &why)) return why;
    if (!Q || !Kfull || !aligned16(Q) || !aligned16(Kfull) || !ws_ok(workspace))
        return RSA_ERR_INVALID_ARG;
    const SpLayout y = sp_layout(B, H, L, P);
    if (ws_bytes < y.fwd_total) return RSA_ERR_WORKSPACE;
    if (causal && m > rank) return RSA_OK;  // the whole window lies right of the diagonal
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    SlabArgs a = sp_slab_args(y, L, d, P, rank, causal, dev->status);
    a.kcol0 = m * y.c, a.kend = (m + 1) * y.c, a.stat0 = m * 2 * y.nCT;
    a.stats = reinterpret_cast<float2 *>(ws + y.slab_bytes);
    a.ntiles = a.nh * a.nRT * a.nCT;
    // the slab window of chunk m: key chunks [m c / 32, (m + 1) c / 32) of every (head, row
    // tile) unit of the rank's scores; the map's extent clips the stores of a tile that reaches
    // past the window
    const uint64_t chunks = uint64_t(y.Lp) / 32, tiles = uint64_t(y.BH) * (y.c / 128);
    CUtensorMap mQ, mK, mS;
    if (!map_rows(&mQ, Q, y.BH, y.c, d, 128) || !map_rows(&mK, Kfull, y.BH, L, d, 256) ||
        !map_slab(&mS, ws + size_t(m) * (y.c / 32) * 16384, y.c / 32, chunks, tiles, 32))
        return RSA_ERR_CUDA;
    RSA_LAUNCH(K_QK_SLAB, rsa::launch_qk_slab(mQ, mK, mS, a, dev->sms, s));
    return RSA_OK;
}

rsa_status_t rsa_sp_softmax_pv(const void *Vfull, void *O, float *lse, int B, int H, int L, int d,
                               int P, int rank, int causal, void *workspace, size_t ws_bytes,
                               void *stream) {
    rsa_status_t why;
    if (!sp_args_ok(B, H, L, d, P, rank, 0, &why)) return why;
    if (!Vfull || !O || !lse || !aligned16(Vfull) || !aligned16(O) || !aligned16(lse) ||
        !ws_ok(workspace))
        return RSA_ERR_INVALID_ARG;
    const SpLayout y = sp_layout(B, H, L, P);
    if (ws_bytes < y.fwd_total) return RSA_ERR_WORKSPACE;
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    SlabArgs a = sp_slab_args(y, L, d, P, rank, causal, dev->status);
    a.stats = reinterpret_cast<float2 *>(ws + y.slab_bytes);
    a.ntiles = a.nh * a.nRT;
    const uint64_t chunks = uint64_t(y.Lp) / 32, tiles = uint64_t(y.BH) * (y.c / 128);
    CUtensorMap mS, mV, mO;
    if (!map_slab(&mS, ws, chunks, chunks, tiles, 128) || !map_rows(&mV, Vfull, y.BH, L, d, 64) ||
        !map_rows_out(&mO, O, y.BH, y.c, d))
        return RSA_ERR_CUDA;
    RSA_LAUNCH(K_PV, rsa::launch_pv_softmax(mS, mV, mO, lse, a, dev->sms, s));
    return RSA_OK;
}

rsa_status_t rsa_sp_backward_rows(const void *Q, const void *Kfull, const void *Vfull,
                                  const void *O, const void *dO, const float *lse, void *dQ,
                                  int B, int H, int L, int d, int P, int rank, int causal,
                                  void *workspace, size_t ws_bytes, void *stream) {
    rsa_status_t why;
    if (!sp_args_ok(B, H, L, d, P, rank, 0, &why)) return why;
    const void *ptrs[] = {Q, Kfull, Vfull, O, dO, lse, dQ};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return RSA_ERR_INVALID_ARG;
    if (!ws_ok(workspace)) return RSA_ERR_INVALID_ARG;
    const SpLayout y = sp_layout(B, H, L, P);
    if (ws_bytes < y.bwd_total) return RSA_ERR_WORKSPACE;
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *lse2 = static_cast<float *>(workspace);
    float *Dvec = lse2 + size_t(y.BH) * y.c;
    SlabArgs a = sp_slab_args(y, L, d, P, rank, causal, dev->status);
    a.ntiles = a.nh * a.nRT;
    const uint32_t kn = d == 64 ? 128 : 64;  // keys per step of the query-major kernel
    CUtensorMap mQ, mdO, mO, mK, mV, mdQ;
    if (!map_rows(&mQ, Q, y.BH, y.c, d, 128) || !map_rows(&mdO, dO, y.BH, y.c, d, 128) ||
        !map_rows(&mO, O, y.BH, y.c, d, 128) || !map_rows(&mK, Kfull, y.BH, L, d, kn) ||
        !map_rows(&mV, Vfull, y.BH, L, d, kn) || !map_rows_out(&mdQ, dQ, y.BH, y.c, d))
        return RSA_ERR_CUDA;
    RSA_LAUNCH(K_BWD_ROWS, rsa::launch_bwd_rows(mQ, mdO, mO, mK, mV, mdQ, lse, lse2, Dvec, a,
                                                dev->sms, s));
    return RSA_OK;
}

rsa_status_t rsa_sp_backward_keys(const void *Q, const void *Kfull, const void *Vfull,
                                  const void *dO, void *dK_part, void *dV_part, int B, int H,
                                  int L, int d, int P, int rank, int m, int causal,
                                  void *workspace, size_t ws_bytes, void *stream) {
    rsa_status_t why;
    if (!sp_args_ok(B, H, L, d, P, rank, m, &why)) return why;
    const void *ptrs[] = {Q, Kfull, Vfull, dO, dK_part, dV_part};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return RSA_ERR_INVALID_ARG;
    if (!ws_ok(workspace)) return RSA_ERR_INVALID_ARG;
    const SpLayout y = sp_layout(B, H, L, P);
    if (ws_bytes < y.bwd_total) return RSA_ERR_WORKSPACE;
    if (causal && m > rank) return RSA_OK;  // no row of this rank sees a key of chunk m
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *lse2 = static_cast<float *>(workspace);
    SlabArgs a = sp_slab_args(y, L, d, P, rank, causal, dev->status);
    a.kcol0 = m * y.c, a.kend = (m + 1) * y.c;
    a.ntiles = a.nh * (y.c / 128);
    a.mode = 0;
    const uint64_t stat_pitch = uint64_t(y.c) * 4;
    CUtensorMap mK, mV, mQ, mdO, mStat, mdK, mdV;
    if (!map_rows(&mK, Kfull, y.BH, L, d, 128) || !map_rows(&mV, Vfull, y.BH, L, d, 128) ||
        !map_rows(&mQ, Q, y.BH, y.c, d, 64) || !map_rows(&mdO, dO, y.BH, y.c, d, 64) ||
        !map3d(&mStat, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lse2, y.c, y.BH, 2, stat_pitch,
               stat_pitch * y.BH, 64, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !map_rows_out(&mdK, dK_part, y.BH, y.c, d) || !map_rows_out(&mdV, dV_part, y.BH, y.c, d))
        return RSA_ERR_CUDA;
    RSA_LAUNCH(K_BWD_KEYS, rsa::launch_bwd_keys(mK, mV, mQ, mdO, mStat, mdK, mdV, a, dev->sms, s));
    return RSA_OK;
}

rsa_status_t rsa_sp_accumulate(float *acc, const void *part, void *out, long long n, int first,
                               void *stream) {
    if (!acc || n < 0 || !aligned16(acc) || (part && !aligned16(part)) || (out && !aligned16(out)))
        return RSA_ERR_INVALID_ARG;
    if (n == 0) return RSA_OK;
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long work = (n + 7) / 8;
    long long blocks = (work + 255) / 256;
    const long long cap = static_cast<long long>(dev->sms) * 8;
    if (blocks > cap) blocks = cap;
    RSA_LAUNCH(K_SP_ACC, (sp_accumulate_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
                              acc, static_cast<const __nv_bfloat16 *>(part),
                              static_cast<__nv_bfloat16 *>(out), n, first ? 1 : 0),
                          cudaGetLastError()));
    return RSA_OK;
}

rsa_status_t rsa_linear(const void *X, const void *W, const float *bias, const void *R, void *Y,
                        int M, int N, int K, int x_kin, int y_kin, int gelu, void *stream) {
    if (!X || !W || !Y || !aligned16(X) || !aligned16(W) || !aligned16(Y) ||
        (bias && !aligned16(bias)) || (R && !aligned16(R)))
        return RSA_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || x_kin <= 0 || y_kin <= 0) return RSA_ERR_INVALID_ARG;
    if (M % 128 != 0 || N % 64 != 0 || K % 64 != 0 || x_kin % 64 != 0 || K % x_kin != 0 ||
        y_kin % 32 != 0 || N % y_kin != 0 || (R && y_kin != N))
        return RSA_ERR_UNSUPPORTED;
    if (static_cast<long long>(M / 128) * ((N + 255) / 256) > 0x3fffffffLL) return RSA_ERR_UNSUPPORTED;
    DeviceState *dev = nullptr;
    rsa_status_t st = device_state(&dev);
    if (st != RSA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap mX, mW, mY;
    if (!map3d(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, x_kin, M, K / x_kin, uint64_t(x_kin) * 2,
               uint64_t(M) * x_kin * 2, 64, 128) ||
        !map3d(&mW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, K, N, 1, uint64_t(K) * 2,
               uint64_t(N) * K * 2, 64, 256) ||
        !map3d(&mY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, y_kin, M, N / y_kin, uint64_t(y_kin) * 2,
               uint64_t(M) * y_kin * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return RSA_ERR_CUDA;
    rsa::LinArgs a{};
    a.M = M, a.N = N, a.K = K, a.x_kin = x_kin, a.y_kin = y_kin, a.gelu = gelu ? 1 : 0;
    a.bias = bias;
    a.res = static_cast<const __nv_bfloat16 *>(R);
    a.nNT = (N + 255) / 256;
    a.ntiles = (M / 128) * a.nNT;
    a.status = dev->status;
    RSA_LAUNCH(K_LINEAR, rsa::launch_linear(mX, mW, mY, a, dev->sms, s));
    return RSA_OK;
}

}  // extern "C"
