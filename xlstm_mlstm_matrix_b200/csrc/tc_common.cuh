// Device helpers shared by the tcgen05 kernels: bounded mbarrier waits that
// report a timeout in the status block, bf16 packing, and the in-place scaling
// of a 128B-swizzled V stage by per-token weights.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"

namespace xlstm {
namespace {

using namespace sm100;

constexpr uint64_t kTimeoutNs = 1000000000ull;   // 1 s per wait

struct Shared {
    volatile int *abort_flag;
    int32_t *status;
};

__device__ __forceinline__ void record_timeout(const Shared &sh, int where) {
    *sh.abort_flag = 1;
    if (sh.status && atomicCAS(&sh.status[kStatusCode], 0, (int32_t)XLSTM_ERR_TIMEOUT) == 0)
        sh.status[kStatusWhere] = where;
}

// Single-thread bounded wait; gives up on timeout or when another role aborted.
// Only the first test is inlined at the call sites; the waiting loop exists once.
__device__ __noinline__ bool wait1_slow(const Shared &sh, uint64_t *bar, uint32_t parity, int where) {
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        // suspended in hardware (no issue slots) until the phase completes or 20 us pass
        if (mbar_try_wait_suspend(bar, parity, 20000)) return true;
        if (*sh.abort_flag) return false;
        if (global_timer_ns() - t0 > kTimeoutNs) {
            record_timeout(sh, where);
            return false;
        }
    }
}
__device__ __forceinline__ bool wait1(const Shared &sh, uint64_t *bar, uint32_t parity, int where) {
    return mbar_try_wait(bar, parity) || wait1_slow(sh, bar, parity, where);
}
// Whole-warp bounded wait: every lane agrees on the outcome.
__device__ __forceinline__ bool waitw(const Shared &sh, uint64_t *bar, uint32_t parity, int where) {
    return __all_sync(0xffffffffu, wait1(sh, bar, parity, where));
}
// Teardown wait: bounded, ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kTimeoutNs) return;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}


// V <- w V in place: the 16L 16-byte chunks of an L-token x 128-value stage (two
// 64-value boxes of L rows of 128 B), chunk e in row (token) (e mod 8L) / 8;
// 128 threads, L/8 chunks each.  The 128B swizzle permutes chunks within a row,
// so the token of a chunk does not depend on it.
// All loads are issued before any store: the stores go to the same buffer, so
// interleaving them would serialise every load behind the previous store.
template <int L = 64>
__device__ __forceinline__ void scale_v_rows(uint8_t *Vs, const float *w, int t128) {
    constexpr int N = L / 8;
    uint4 u[N];
    float ws[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int e = t128 + 128 * i;
        u[i] = *reinterpret_cast<const uint4 *>(Vs + 16 * e);
        ws[i] = w[(e & (8 * L - 1)) >> 3];
    }
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const float2 w2 = make_float2(ws[i], ws[i]);
        const float2 a = __fmul2_rn(bf16x2_to_float2(u[i].x), w2), b = __fmul2_rn(bf16x2_to_float2(u[i].y), w2);
        const float2 c = __fmul2_rn(bf16x2_to_float2(u[i].z), w2), d = __fmul2_rn(bf16x2_to_float2(u[i].w), w2);
        u[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y), pack_bf16x2(c.x, c.y), pack_bf16x2(d.x, d.y));
    }
#pragma unroll
    for (int i = 0; i < N; ++i) *reinterpret_cast<uint4 *>(Vs + 16 * (t128 + 128 * i)) = u[i];
}

}  // namespace
}  // namespace xlstm
