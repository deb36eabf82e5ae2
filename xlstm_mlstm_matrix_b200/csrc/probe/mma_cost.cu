// Microbenchmark of tcgen05.mma issue cost on sm_100a (one thread issuing
// back-to-back MMAs on zero operands; clock64 around the sequence, completion
// observed through tcgen05.commit).  Measurement tooling, not part of the
// library: built as its own shared object and driven by bench.py --probe mma.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../sm100.cuh"

using namespace xlstm::sm100;

namespace {

constexpr int kThreads = 384;
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
    int bg;            // background load while the MMAs run: 0 none, 1 tensor-memory loads,
                       // 2 tensor-memory stores, 3 shared-memory loads, 4 shared-memory stores
    int nbg;           // background warps: 3 (warps 1-3) or 11 (warps 1-11)
    int random;        // operands: 0 zeros, 1 pseudo-random bf16 in (-1, 1)
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

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) mma_cost_kernel(ProbeArgs a, long long *cycles, int *ok,
                                                               const uint8_t *gsrc) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *As = sm, *Bs = sm + kSmemA;
    uint8_t *Bg = sm + kSmemA + kSmemB;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + kSmemA + kSmemB + kSmemBg);
    uint32_t *slot = reinterpret_cast<uint32_t *>(bar + 6);
    volatile int *stop = reinterpret_cast<volatile int *>(bar + 7);
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < (kSmemA + kSmemB + kSmemBg) / 4; i += kThreads) {
        uint32_t w = 0;
        if (a.random) {   // two bf16 values of magnitude below 1 from an integer hash of the index
            uint32_t h = (uint32_t)i * 2654435761u;
            h ^= h >> 15; h *= 2246822519u; h ^= h >> 13;
            w = (h & 0x807F807Fu) | 0x3E003E00u;
        }
        reinterpret_cast<uint32_t *>(sm)[i] = w;
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        mbar_init(&bar[4], 1);
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
    if (warp < 4) {   // the tensor-memory A operand region (columns 448..479), every lane quarter
        float z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = a.random ? __uint_as_float(0x3E003E00u | ((tid * 37 + i * 11) & 0x007F007Fu)) : 0.f;
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
        } else if (a.issue == 10 || a.issue == 11) {
            // the per-chunk MMA program of the d_qk = 256 chunkwise kernel (S 16 at M=64; readout 8 ss +
            // 16 ts + 8 ss at M=128 N=64; intra 4 at N=64; update 4 at N=256; six commits), 32 chunks;
            // 10: rolled K loops as in the kernel, 11: fully unrolled groups
            const uint32_t idS = make_idesc(64, 64, kFmtBF16, kFmtBF16, 0, 0);
            const uint32_t idR = make_idesc(128, 64, kFmtBF16, kFmtBF16, 0, 0);
            const uint32_t idPV = make_idesc(128, 64, kFmtBF16, kFmtBF16, 1, 0);
            const uint32_t idU = make_idesc(128, 256, kFmtBF16, kFmtBF16, 1, 1);
            const uint64_t dq = smem_desc_sw128(smem_u32(Bs), 16, 1024), dk = smem_desc_sw128(smem_u32(Bs) + 32768, 16, 1024);
            const uint64_t dclo = smem_desc_sw128(smem_u32(As), 16, 1024);
            const uint64_t dvmn = smem_desc_sw128(smem_u32(As), 8192, 1024), dkmn = smem_desc_sw128(smem_u32(Bs), 8192, 1024);
            const uint32_t TS = 256, TH = 320, TC = 0, TCHI = 384;
#define KSTEP(ks) (uint64_t)((((ks) >> 2) * 8192 + ((ks) & 3) * 32) >> 4)
#define CSTEP(ks) (uint64_t)((((ks) >> 2) * 16384 + ((ks) & 3) * 32) >> 4)
            for (int c = 0; c < a.nmma / 56; ++c) {
                if (a.issue == 10) {
#pragma unroll 1
                    for (int ks = 0; ks < 16; ++ks) mma_f16_ss(tm + TS, dq + KSTEP(ks & 7), dk + KSTEP(ks & 7), idS, ks > 0);
                    tc_commit(&bar[1]);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) mma_f16_ss(tm + TH, dclo + CSTEP(kk & 3), dq + KSTEP(kk), idR, kk > 0);
                    tc_commit(&bar[1]);
#pragma unroll 1
                    for (int ks = 0; ks < 16; ++ks) mma_f16_ts(tm + TH, tm + TCHI + 4 * (ks & 7), dq + KSTEP(ks & 7), idR, 1);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) mma_f16_ss(tm + TH, dclo + CSTEP(kk & 3), dq + KSTEP(kk), idR, 1);
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks) mma_f16_ss(tm + TH, dvmn + (uint64_t)(ks * 2048 >> 4), dq + (uint64_t)(ks * 32 >> 4), idPV, 1);
                    tc_commit(&bar[1]);
                    tc_commit(&bar[1]);
#pragma unroll 1
                    for (int ks = 0; ks < 4; ++ks) mma_f16_ss(tm + TC, dvmn + (uint64_t)(ks * 2048 >> 4), dkmn + (uint64_t)(ks * 2048 >> 4), idU, 1);
                    tc_commit(&bar[1]);
                    tc_commit(&bar[1]);
                } else {
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) mma_f16_ss(tm + TS, dq + KSTEP(ks & 7), dk + KSTEP(ks & 7), idS, ks > 0);
                    tc_commit(&bar[1]);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_f16_ss(tm + TH, dclo + CSTEP(kk & 3), dq + KSTEP(kk), idR, kk > 0);
                    tc_commit(&bar[1]);
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) mma_f16_ts(tm + TH, tm + TCHI + 4 * (ks & 7), dq + KSTEP(ks & 7), idR, 1);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) mma_f16_ss(tm + TH, dclo + CSTEP(kk & 3), dq + KSTEP(kk), idR, 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) mma_f16_ss(tm + TH, dvmn + (uint64_t)(ks * 2048 >> 4), dq + (uint64_t)(ks * 32 >> 4), idPV, 1);
                    tc_commit(&bar[1]);
                    tc_commit(&bar[1]);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) mma_f16_ss(tm + TC, dvmn + (uint64_t)(ks * 2048 >> 4), dkmn + (uint64_t)(ks * 2048 >> 4), idU, 1);
                    tc_commit(&bar[1]);
                    tc_commit(&bar[1]);
                }
            }
#undef KSTEP
#undef CSTEP
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
    if (a.bg == 6 && warp == 1 && (tid & 31) == 0) {   // TMA-style bulk copies into shared memory
        long long it = 0;
        const long long tb0 = clock64();
        bool good = true;
        for (; it < 200000 && !*stop && good; ++it) {
            mbar_arrive_expect_tx(&bar[4], (uint32_t)kSmemBg);
            bulk_load(smem_u32(Bg), gsrc + (size_t)(it & 63) * kSmemBg, (uint32_t)kSmemBg, &bar[4]);
            good = wait_bounded(&bar[4], (uint32_t)(it & 1));
        }
        cycles[gridDim.x + blockIdx.x] = it;
        cycles[2 * gridDim.x + blockIdx.x] = clock64() - tb0;
        if (!good) ok[blockIdx.x] = 0;
    }
    if (a.bg && a.bg != 6 && warp >= 1 && warp <= a.nbg && !issuer) {   // background traffic until the MMAs are done (bounded)
        const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
        float r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0.f;
        uint4 acc = make_uint4(0, 0, 0, 0);
        long long it = 0;
        const long long tb0 = clock64();
        for (; it < 4000000 && !*stop; ++it) {
            if (a.bg == 1) {
                tmem_ld32(tm + lb + 320 + 32 * (warp >> 2), r);
                tmem_wait_ld();
            } else if (a.bg == 2) {
                tmem_st32(tm + lb + 320 + 32 * (warp >> 2), r);
                tmem_wait_st();
            } else if (a.bg == 5) {   // arithmetic only: dependent fused multiply-adds
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = fmaf(r[i], 1.0001f, 0.5f);
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
        if ((a.bg == 1 || a.bg == 5) && r[0] == 12345.f) ok[blockIdx.x] = 3;
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
    // issue = pattern + 16 * background kind + 128 * (11 background warps) + 256 * (random operands)
    const int random = (issue >> 8) & 1, many = (issue >> 7) & 1;
    issue &= 127;
    const int bg = issue / 16;
    issue %= 16;
    if (issue < 0 || issue > 11 || bg > 6 || (bg && issue != 3 && issue != 8 && issue != 9 && issue < 10) ||
        (issue == 8 && !bg) || (issue == 2 && (2 * nacc * N + 64 > 512 || nmma % 2)) ||
        (issue >= 3 && issue < 10 && ((form && issue != 9) || (!form && issue == 9) || nmma % 16 || a_mn || b_mn)) ||
        (issue >= 10 && (nmma % 56 || form || M != 128 || N != 64)))
        return -1;
    issue += 16 * bg;
    if (M != 64 && M != 128) return -1;
    if (N < 16 || N > 256 || N % 16) return -1;
    if (nacc < 1 || nacc * N + 64 > 512 || (form == 1 && (M != 128 || a_mn))) return -1;
    if (ctas < 1 || ctas > 1024 || nmma < 1) return -1;
    ProbeArgs a{form, M, N, a_mn, b_mn, nmma, nacc, commit_every, issue % 16, 0, issue / 16, many ? 11 : 3, random};
    long long *dc = nullptr;
    int *dok = nullptr;
    if (cudaMalloc(&dc, 3 * ctas * sizeof(long long)) != cudaSuccess) return -2;
    cudaMemset(dc, 0, 3 * ctas * sizeof(long long));
    if (cudaMalloc(&dok, ctas * sizeof(int)) != cudaSuccess) { cudaFree(dc); return -2; }
    const int smem = kSmemA + kSmemB + kSmemBg + 64 + 1024;
    cudaFuncSetAttribute(mma_cost_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    uint8_t *gsrc = nullptr;
    if (cudaMalloc(&gsrc, 64 * kSmemBg) != cudaSuccess) { cudaFree(dc); cudaFree(dok); return -2; }
    cudaMemset(gsrc, 0, 64 * kSmemBg);
    mma_cost_kernel<<<ctas, kThreads, smem>>>(a, dc, dok, gsrc);
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
    cudaFree(gsrc);
    return rc;
}
