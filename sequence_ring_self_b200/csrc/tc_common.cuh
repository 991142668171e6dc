// tc_common.cuh -- pieces shared by the tensor-core kernels: the per-CTA control block
// (mbarriers, TMEM base, abort flag), pipeline counters and small warp-level helpers.
#pragma once

#include "rsa_internal.h"
#include "sm100_ptx.cuh"

namespace rsa {
namespace tc {

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



// 2^x on the MUFU unit (ex2.approx.ftz: relative error about 2^-22, flushes denormals).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100): one instruction computes both lanes of a float2.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

int grid_for(int ntiles, int num_sms);

}  // namespace tc
}  // namespace rsa
