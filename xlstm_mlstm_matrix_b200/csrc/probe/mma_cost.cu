// Microbenchmark of tcgen05.mma issue cost on sm_100a (one thread issuing
// back-to-back MMAs on zero operands; clock64 around the sequence, completion
// observed through tcgen05.commit).  Measurement tooling, not part of the
// library: built as its own shared object and driven by bench.py --probe mma.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../sm100.cuh"

using namespace xlstm::sm100;

namespace {

constexpr int kThreads = 128;
constexpr int kSmemA = 32768, kSmemB = 65536, kSmemBg = 16384;

struct ProbeArgs {
    int form;          // 0: A and B in shared memory (ss); 1: A in tensor memory (ts)
    int M, N;          // instruction shape (K = 16)
    int a_mn, b_mn;    // MN-major operand layouts (shared-memory operands only)
    int nmma;          // MMAs in the timed sequence
    int nacc;          // accumulators cycled through (1, 2 or 4)
    int commit_every;  // 0: one commit at the end; k: a commit after every k MMAs
    int issue;         // 0: lane 0 of warp 0 alone; 1: warp 0 converged, elect.sync picks the issuing lane;
                       // 2: lane 0 of warps 0 and 1, each to its own accumulator, half the MMAs each;
                       // 3: like 0 with a fully unrolled, compile-time issue sequence;
                       // 4: a rolled loop over 16 K steps (descriptor + step offset, accumulate = step > 0);
                       // 5: like 3 with one unrelated integer instruction between MMAs;
                       // 6: like 3 with descriptors from a runtime base (offsets added at run time);
                       // 7: groups of 4 unrolled MMAs inside a rolled loop
    int rt_base;       // runtime zero added to the descriptors in mode 6
    int bg;            // background load on warps 1-3 while the MMAs run: 0 none, 1 tensor-memory loads,
                       // 2 tensor-memory stores, 3 shared-memory loads, 4 shared-memory stores
};

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t.reg .b32 R;\n\telect.sync R|P1, 0xffffffff;\n\tselp.b32 %0, 1, 0, P1;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ bool wait_bounded(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > 1000000000ull) return false;
    return true;
}

__global__ void __launch_bounds__(kThreads, 1) mma_cost_kernel(ProbeArgs a, long long *cycles, int *ok) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *As = sm, *Bs = sm + kSmemA;
    uint8_t *Bg = sm + kSmemA + kSmemB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSmemA + kSmemB + kSmemBg);
    uint32_t *slot = reinterpret_cast<uint32_t *>(bar + 6);
    volatile int *stop = reinterpret_cast<volatile int *>(bar + 7);
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < (kSmemA + kSmemB + kSmemBg) / 16; i += kThreads)
        reinterpret_cast<uint4 *>(sm)[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        *stop = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *slot;
    {   // zero the tensor-memory A operand region (columns 448..479), every lane quarter
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = 0.f;
        tmem_st32(tm + ((uint32_t)(32 * warp) << 16) + 448, z);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t idesc = make_idesc(a.M, a.N, kFmtBF16, kFmtBF16, a.a_mn, a.b_mn);
    const uint64_t da = a.a_mn ? smem_desc_sw128(smem_u32(As), 8192, 1024) : smem_desc_sw128(smem_u32(As), 16, 1024);
    const uint64_t db = a.b_mn ? smem_desc_sw128(smem_u32(Bs), 8192, 1024) : smem_desc_sw128(smem_u32(Bs), 16, 1024);
    const bool issuer = (a.issue == 1) ? (warp == 0) : (a.issue == 2 ? (warp < 2 && (tid & 31) == 0) : tid == 0);
    if (tid == 0) {   // warm-up
        for (int i = 0; i < 8; ++i) mma_f16_ss(tm, da, db, idesc, i > 0);
        tc_commit(&bar[0]);
        ok[blockIdx.x] = wait_bounded(&bar[0], 0) ? 1 : 0;
    }
    __syncthreads();
    tc_fence_after();
    long long t0 = 0;
    if (issuer) {
        t0 = clock64();
        if (a.issue == 3) {
#pragma unroll 1
            for (int r = 0; r < a.nmma / 16; ++r) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint64_t o = (uint64_t)((j & 3) * 32 >> 4);
                    mma_f16_ss(tm, da + o, db + o, idesc, 1);
                }
            }
        } else if (a.issue == 9) {
#pragma unroll 1
            for (int r = 0; r < a.nmma / 16; ++r) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint64_t o = (uint64_t)((j & 3) * 32 >> 4);
                    mma_f16_ts(tm, tm + 448 + 8 * (j & 3), db + o, idesc, 1);
                }
            }
        } else if (a.issue == 8) {   // no MMA: hold the background running for about 60k cycles
            const long long ts0 = clock64();
            while (clock64() - ts0 < 60000) {
            }
        } else if (a.issue == 4) {
#pragma unroll 1
            for (int r = 0; r < a.nmma / 16; ++r) {
#pragma unroll 1
                for (int ks = 0; ks < 16; ++ks) {
                    const uint64_t o = (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4) & 0x1FF;
                    mma_f16_ss(tm, da + (uint64_t)((ks & 3) * 2), db + (uint64_t)((ks & 3) * 2) + (o & 0), idesc, ks > 0 || r > 0);
                }
            }
        } else if (a.issue == 5) {
            uint32_t x = (uint32_t)a.rt_base;
#pragma unroll 1
            for (int r = 0; r < a.nmma / 16; ++r) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint64_t o = (uint64_t)((j & 3) * 32 >> 4);
                    mma_f16_ss(tm, da + o, db + o, idesc, 1);
                    asm volatile("add.u32 %0, %0, 1;" : "+r"(x));
                }
            }
            if (x == 0x7fffffff) ok[blockIdx.x] = 2;
        } else if (a.issue == 6) {
#pragma unroll 1
            for (int r = 0; r < a.nmma / 16; ++r) {
                const uint64_t ra = da + (uint64_t)(a.rt_base + r * 0), rb = db + (uint64_t)(a.rt_base + r * 0);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const uint64_t o = (uint64_t)((j & 3) * 32 >> 4);
                    mma_f16_ss(tm, ra + o, rb + o, idesc, 1);
                }
            }
        } else if (a.issue == 7) {
#pragma unroll 1
            for (int r = 0; r < a.nmma / 4; ++r) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint64_t o = (uint64_t)(j * 32 >> 4);
                    mma_f16_ss(tm, da + o, db + o, idesc, 1);
                }
            }
        } else {
            const int n = a.issue == 2 ? a.nmma / 2 : a.nmma;
            const uint32_t dbase = tm + (a.issue == 2 ? (uint32_t)warp * a.N : 0u);
            for (int i = 0; i < n; ++i) {
                const uint32_t d = dbase + (uint32_t)(i % a.nacc) * a.N;
                const int ks = i & 3;
                const uint64_t oa = a.a_mn ? (uint64_t)(ks * 2048 >> 4) : (uint64_t)(ks * 32 >> 4);
                const uint64_t ob = a.b_mn ? (uint64_t)(ks * 2048 >> 4) : (uint64_t)(ks * 32 >> 4);
                const bool me = a.issue == 1 ? elect_one() : true;
                if (me) {
                    if (a.form == 1)
                        mma_f16_ts(d, tm + 448 + 8 * ks, db + ob, idesc, 1);
                    else
                        mma_f16_ss(d, da + oa, db + ob, idesc, 1);
                    if (a.commit_every && (i + 1) % a.commit_every == 0) tc_commit(&bar[1]);
                }
                if (a.issue == 1) __syncwarp();
            }
        }
    }
    if (a.bg && warp >= 1 && !issuer) {   // background traffic until the MMAs are done (bounded)
        const uint32_t lb = (uint32_t)(32 * warp) << 16;
        float r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0.f;
        uint4 acc = make_uint4(0, 0, 0, 0);
        long long it = 0;
        const long long tb0 = clock64();
        for (; it < 4000000 && !*stop; ++it) {
            if (a.bg == 1) {
                tmem_ld32(tm + lb + 320, r);
                tmem_wait_ld();
            } else if (a.bg == 2) {
                tmem_st32(tm + lb + 320, r);
                tmem_wait_st();
            } else if (a.bg == 3) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t addr = smem_u32(Bg) + 16u * (uint32_t)(((int)it * 8 + i) * 32 % 1024 + (tid & 31));
                    uint32_t x0, x1, x2, x3;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3) : "r"(addr));
                    acc.x ^= x0 ^ x1 ^ x2 ^ x3;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     smem_u32(Bg) + 16u * (uint32_t)(((int)it * 8 + i + warp) * 32 % 1024 + (tid & 31))),
                                 "r"(acc.x), "r"(acc.y), "r"(acc.z), "r"(acc.w)
                                 : "memory");
            }
        }
        if (warp == 1 && (tid & 31) == 0) {
            cycles[gridDim.x + blockIdx.x] = it;
            cycles[2 * gridDim.x + blockIdx.x] = clock64() - tb0;
        }
        if (a.bg == 1 && r[0] == 12345.f) ok[blockIdx.x] = 3;
        if (acc.x == 0xdeadbeef) ok[blockIdx.x] = 3;
    }
    // one commit per issuing thread onto barrier 0 (count = issuers), then wait
    if (issuer && (a.issue != 1 || (tid & 31) == 0)) tc_commit(&bar[2 + (a.issue == 2 ? warp : 0)]);
    if (issuer && (tid & 31) == 0) {
        const bool good = wait_bounded(&bar[2 + (a.issue == 2 ? warp : 0)], 0);
        const long long t1 = clock64();
        if (warp == 0) cycles[blockIdx.x] = a.issue == 8 ? 0 : t1 - t0;
        if (!good) ok[blockIdx.x] = 0;
        *stop = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int mma_probe_run(int form, int M, int N, int a_mn, int b_mn, int nmma, int nacc, int commit_every,
                             int issue, int ctas, long long *cycles_host) {
    const int bg = issue / 16;
    issue %= 16;
    if (issue < 0 || issue > 9 || bg > 4 || (bg && issue != 3 && issue != 8 && issue != 9) ||
        (issue == 8 && !bg) || (issue == 2 && (2 * nacc * N + 64 > 512 || nmma % 2)) ||
        (issue >= 3 && ((form && issue != 9) || (!form && issue == 9) || nmma % 16 || a_mn || b_mn)))
        return -1;
    issue += 16 * bg;
    if (M != 64 && M != 128) return -1;
    if (N < 16 || N > 256 || N % 16) return -1;
    if (nacc < 1 || nacc * N + 64 > 512 || (form == 1 && (M != 128 || a_mn))) return -1;
    if (ctas < 1 || ctas > 1024 || nmma < 1) return -1;
    ProbeArgs a{form, M, N, a_mn, b_mn, nmma, nacc, commit_every, issue % 16, 0, issue / 16};
    long long *dc = nullptr;
    int *dok = nullptr;
    if (cudaMalloc(&dc, 3 * ctas * sizeof(long long)) != cudaSuccess) return -2;
    cudaMemset(dc, 0, 3 * ctas * sizeof(long long));
    if (cudaMalloc(&dok, ctas * sizeof(int)) != cudaSuccess) { cudaFree(dc); return -2; }
    const int smem = kSmemA + kSmemB + kSmemBg + 64 + 1024;
    cudaFuncSetAttribute(mma_cost_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    mma_cost_kernel<<<ctas, kThreads, smem>>>(a, dc, dok);
    int rc = cudaDeviceSynchronize() == cudaSuccess ? 0 : -3;
    int *okh = new int[ctas];
    if (rc == 0 && cudaMemcpy(cycles_host, dc, 3 * ctas * sizeof(long long), cudaMemcpyDeviceToHost) != cudaSuccess)
        rc = -3;
    if (rc == 0 && cudaMemcpy(okh, dok, ctas * sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) rc = -3;
    for (int i = 0; rc == 0 && i < ctas; ++i)
        if (!okh[i]) rc = -4;
    delete[] okh;
    cudaFree(dc);
    cudaFree(dok);
    return rc;
}
