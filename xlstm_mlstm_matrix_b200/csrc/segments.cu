// Segment-parallel chunkwise forward, for long sequences with too few heads to
// fill the GPU.
//
// The mLSTM recurrence (xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3, with the
// stabilizer of the "sLSTM" section) maps the state entering a stretch of tokens
// to the state leaving it by an affine map whose coefficients depend only on the
// stretch's own tokens.  A sequence cut into segments therefore runs in three
// launches:
//  1. summary (tensor cores), for every segment but the last, from a zero state:
//     with F_t = sum_{r<=t} f~_r counted from the segment start, u_t = i~_t - F_t,
//     F = F_last and u* = max_t u_t,
//        C_seg = sum_t e^{u_t - u*} v_t k_t^T,   n_seg = sum_t e^{u_t - u*} k_t,
//     the stabilized state the segment alone leaves, in the gauge m_seg = F + u*
//     (the unrolled rule m_t = max(f~_t + m_{t-1}, i~_t) started from -inf);
//  2. combine (CUDA cores): entry state of segment g+1 from that of g,
//        m' = max(F + m, m_seg),
//        C' = e^{F + m - m'} C + e^{m_seg - m'} C_seg    (n likewise);
//     every coefficient is <= 1;
//  3. the chunkwise kernel runs all segments at once, each from its entry state;
//     the last one writes the final state.
// Steps 1 and 2 read k, v and the gates once more and pass d_v x d_qk floats per
// segment through the workspace; the sequential chain per block becomes nseg
// times shorter.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "tma_host.cuh"

namespace xlstm {
namespace {

using namespace sm100;

constexpr int kL = 64;            // chunk length (tokens)
constexpr int kDvs = 128;         // value rows per block
constexpr int kSumThreads = 256;
constexpr int kRing = 4;          // weight-ring slots (even: each slot has one producer warp)
static_assert(kSegChunk == 64, "segment plan in 64-token chunks");
constexpr int kMinSegChunks = 8;  // shortest segment worth a summary
constexpr int kMaxSegChunks = 1024;   // longest segment (its per-chunk F offsets sit in shared memory)
constexpr int kCombineThreads = 256;

template <int DQK>
struct SumCfg {
    static constexpr int NKB = DQK / 64;          // 64-column boxes of k
    static constexpr int K_BYTES = NKB * 8192;
    static constexpr int V_BYTES = 2 * 8192;      // 128 value columns
    // k / v stages in flight: as many as ~190 KB hold (the copies are the bound)
    static constexpr int STAGES = DQK == 256 ? 4 : (DQK == 128 ? 6 : 8);
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_W = OFF_V + STAGES * V_BYTES;    // kRing x 64 weights
    static constexpr int OFF_RED = OFF_W + kRing * kL * 4;    // F_seg and u* (doubles)
    static constexpr int OFF_F = OFF_RED + 16;                // per-chunk F at the chunk's start (doubles)
    static constexpr int OFF_UM = OFF_F + kMaxSegChunks * 8;  // per-chunk max_t (i_t - F_t), F from the chunk's start
    static constexpr int OFF_BAR = OFF_UM + kMaxSegChunks * 8;
    // barriers: KV_FULL, KV_EMPTY, VS per stage; W_FULL, W_EMPTY per ring slot; DONE, DRAIN
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = STAGES, B_VS = 2 * STAGES, B_W_FULL = 3 * STAGES,
                         B_W_EMPTY = B_W_FULL + kRing, B_DONE = B_W_EMPTY + kRing, B_DRAIN = B_DONE + 1,
                         NBARS = B_DRAIN + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;         // + alignment slack
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Where a wait of the summary kernel gave up (status block; the chunkwise
// kernel's codes are below 40).
enum : int32_t { kWhereSumKvEmpty = 41, kWhereSumVs, kWhereSumWEmpty, kWhereSumKv, kWhereSumW, kWhereSumDone };

struct SumParams {
    int T, dv, nslices, nsum, seg_chunks, BH;   // nsum = nseg - 1 summaries per sequence
    const float *ig, *fg;
    float *segC, *segN;   // [nsum][BH][d_v][d_qk], [nsum][BH][d_qk]
    double *segS;         // [nsum][BH][2]: F, m_seg
    int32_t *status;
};

// Inclusive prefix sum over the 64 tokens of a chunk held two per lane (a, b):
// returns the sum before token a (within the chunk) and the chunk total.
__device__ __forceinline__ void chunk_scan(double fa, double fb, double &excl, double &total) {
    double incl = fa + fb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if ((threadIdx.x & 31) >= o) incl += y;
    }
    excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if ((threadIdx.x & 31) == 0) excl = 0.0;
    total = __shfl_sync(0xffffffffu, incl, 31);
}

// Per segment: its state from a zero start (C_seg, n_seg) and the scalars F, m_seg.
// Block = (sequence, segment, 128 value rows); warps: 0 TMA, 1 MMA (owns TMEM),
// 2-3 weights, 4-7 w V in place, n_seg and the read-out of C_seg.
template <int DQK>
__global__ void __launch_bounds__(kSumThreads, 1)
    seg_summary_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const SumParams p) {
    using C = SumCfg<DQK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    Shared sh{reinterpret_cast<volatile int *>(sm + C::OFF_MISC + 4), p.status};
    float *wring = reinterpret_cast<float *>(sm + C::OFF_W);
    double *red = reinterpret_cast<double *>(sm + C::OFF_RED);
    double *chunkF = reinterpret_cast<double *>(sm + C::OFF_F);   // F before chunk c, from its run's start

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x % p.nslices;
    const int g = (blockIdx.x / p.nslices) % p.nsum;
    const int bh = blockIdx.x / (p.nslices * p.nsum);
    const int v0 = slice * kDvs;
    const int NC = p.seg_chunks;   // a summarised segment is never the last: all its chunks are full
    const int t_base = kL * NC * g;
    const float *ig = p.ig + (size_t)bh * p.T + t_base, *fg = p.fg + (size_t)bh * p.T + t_base;

    if (tid == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&bar[C::B_KV_FULL + i], 1);
            mbar_init(&bar[C::B_KV_EMPTY + i], 2);   // the update MMAs and the n_seg sum read k
            mbar_init(&bar[C::B_VS + i], 1);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&bar[C::B_W_FULL + i], 1);
            mbar_init(&bar[C::B_W_EMPTY + i], 1);
        }
        mbar_init(&bar[C::B_DONE], 1);
        mbar_init(&bar[C::B_DRAIN], 1);
        *sh.abort_flag = 0;
        fence_mbar_init();
        // the first stages load while the gates are scanned
        for (int c = 0; c < C::STAGES && c < NC; ++c) {
            mbar_arrive_expect_tx(&bar[C::B_KV_FULL + c], C::K_BYTES + C::V_BYTES);
            for (int b = 0; b < C::NKB; ++b)
                tma_load_3d(sm + C::OFF_K + c * C::K_BYTES + b * 8192, &tmk, &bar[C::B_KV_FULL + c], 64 * b,
                            t_base + kL * c, bh);
            for (int b = 0; b < 2; ++b)
                tma_load_3d(sm + C::OFF_V + c * C::V_BYTES + b * 8192, &tmv, &bar[C::B_KV_FULL + c], v0 + 64 * b,
                            t_base + kL * c, bh);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, DQK);
        tmem_relinquish();
    }
    // F and u* of the segment.  Pass 1: warp w takes chunks w, w + 8, ... in groups of
    // eight, every gate load of a group issued before its first scan (one memory
    // round trip per group, not per chunk): per chunk the total of f~ and
    // max_t (i~_t - F_t) with F counted from the chunk's start.  Pass 2 (warp 0):
    // the chunk totals scanned into F at each chunk's start, F_seg, and
    // u* = max over chunks of (that maximum - F at the chunk's start).
    double *umc = reinterpret_cast<double *>(sm + C::OFF_UM);
    for (int c0 = warp; c0 < NC; c0 += 64) {
        float fa[8], fb[8], ia[8], ib[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = c0 + 8 * j;
            if (c < NC) {
                const int t = kL * c + 2 * lane;
                fa[j] = fg[t]; fb[j] = fg[t + 1]; ia[j] = ig[t]; ib[j] = ig[t + 1];
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = c0 + 8 * j;
            if (c < NC) {   // warp-uniform
                double excl, total;
                chunk_scan(fa[j], fb[j], excl, total);
                const double Fa = excl + fa[j], Fb = Fa + fb[j];
                double um = fmax((double)ia[j] - Fa, (double)ib[j] - Fb);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) um = fmax(um, __shfl_xor_sync(0xffffffffu, um, o));
                if (lane == 0) { chunkF[c] = total; umc[c] = um; }
            }
        }
    }
    __syncthreads();
    if (warp == 0) {   // chunk totals -> F at each chunk's start; lane l scans a contiguous run
        const int per = (NC + 31) / 32, c0 = lane * per, c1 = min(NC, c0 + per);
        double run = 0.0;
        for (int c = c0; c < c1; ++c) run += chunkF[c];
        double incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        double f = incl - run, um = -INFINITY;
        for (int c = c0; c < c1; ++c) {
            const double tot = chunkF[c];
            chunkF[c] = f;
            um = fmax(um, umc[c] - f);
            f += tot;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) um = fmax(um, __shfl_xor_sync(0xffffffffu, um, o));
        if (lane == 31) { red[0] = incl; red[1] = um; }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const double Fseg = red[0], ustar = red[1];

    if (warp == 0) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int c = 0; c < C::STAGES && c < NC; ++c) issued[c] = 1;   // issued before the gate scan
            for (int c = C::STAGES; c < NC; ++c) {
                const int s = c % C::STAGES;
                if (!wait1(sh, &bar[C::B_KV_EMPTY + s], ((c / C::STAGES) - 1) & 1, kWhereSumKvEmpty)) break;
                mbar_arrive_expect_tx(&bar[C::B_KV_FULL + s], C::K_BYTES + C::V_BYTES);
                uint8_t *Ks = sm + C::OFF_K + s * C::K_BYTES;
                uint8_t *Vs = sm + C::OFF_V + s * C::V_BYTES;
                for (int b = 0; b < C::NKB; ++b)
                    tma_load_3d(Ks + b * 8192, &tmk, &bar[C::B_KV_FULL + s], 64 * b, t_base + kL * c, bh);
                // a box past d_v (the upper half of a 64-row last slice) is zero-filled by the copy
                for (int b = 0; b < 2; ++b)
                    tma_load_3d(Vs + b * 8192, &tmv, &bar[C::B_KV_FULL + s], v0 + 64 * b, t_base + kL * c, bh);
                ++issued[s];
            }
            for (int s = 0; s < C::STAGES; ++s)   // every issued copy lands before shared memory is released
                if (issued[s]) drain_wait(&bar[C::B_KV_FULL + s], (issued[s] - 1) & 1);
        }
    } else if (warp == 1) {
        // ===================== MMA issuer: C_seg += (w V)^T K =====================
        if (lane == 0) {
            const uint32_t idU = make_idesc(128, DQK, kFmtBF16, kFmtBF16, 1, 1);
            bool issued = false;
            for (int c = 0; c < NC; ++c) {
                const int s = c % C::STAGES;
                if (!wait1(sh, &bar[C::B_VS + s], (c / C::STAGES) & 1, kWhereSumVs)) break;
                tc_fence_after();
                const uint64_t dv_mn = smem_desc_sw128(smem_u32(sm + C::OFF_V + s * C::V_BYTES), 8192, 1024);
                const uint64_t dk_mn = smem_desc_sw128(smem_u32(sm + C::OFF_K + s * C::K_BYTES), 8192, 1024);
#pragma unroll 1
                for (int ks = 0; ks < kL / 16; ++ks)
                    mma_f16_ss(tm, dv_mn + (uint32_t)(ks * 2048 >> 4), dk_mn + (uint32_t)(ks * 2048 >> 4), idU,
                               (c > 0 || ks > 0) ? 1u : 0u);
                issued = true;
                tc_commit(&bar[C::B_KV_EMPTY + s]);
            }
            if (issued) {   // C_seg complete, and nothing in flight when tensor memory is freed
                tc_commit(&bar[C::B_DONE]);
                tc_commit(&bar[C::B_DRAIN]);
                drain_wait(&bar[C::B_DRAIN], 0);
            }
        }
    } else if (warp == 2 || warp == 3) {
        // ===================== weights w_t = e^{u_t - u*} =====================
        // Warp 2 takes the even chunks, warp 3 the odd ones (a ring slot always has
        // the same producer); F at a chunk's start comes from the first pass.  The
        // gates of a warp's next chunk are loaded while it processes the current one
        // (scalar loads: a sequence's gates start at an arbitrary float offset).
        int c = warp - 2;
        float fan = 0.f, fbn = 0.f, ian = 0.f, ibn = 0.f;
        if (c < NC) {
            const int t = kL * c + 2 * lane;
            fan = fg[t]; fbn = fg[t + 1]; ian = ig[t]; ibn = ig[t + 1];
        }
        for (; c < NC; c += 2) {
            const int slot = c % kRing;
            const double fa = fan, fb = fbn, ia = ian, ib = ibn;
            if (c + 2 < NC) {
                const int t = kL * (c + 2) + 2 * lane;
                fan = fg[t]; fbn = fg[t + 1]; ian = ig[t]; ibn = ig[t + 1];
            }
            const double F0 = chunkF[c];
            if (c >= kRing && !waitw(sh, &bar[C::B_W_EMPTY + slot], ((c / kRing) - 1) & 1, kWhereSumWEmpty)) break;
            double excl, total;
            chunk_scan(fa, fb, excl, total);
            const double Fa = F0 + excl + fa, Fb = Fa + fb;
            float *w = wring + slot * kL;
            w[2 * lane] = expf((float)(ia - Fa - ustar));
            w[2 * lane + 1] = expf((float)(ib - Fb - ustar));
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[C::B_W_FULL + slot]);
        }
        if (warp == 2 && lane == 0 && slice == 0) {
            double *sc = p.segS + ((size_t)g * p.BH + bh) * 2;
            sc[0] = Fseg;
            sc[1] = Fseg + ustar;
        }
    } else {
        // ===================== w V in place, n_seg; read-out of C_seg =====================
        // n_seg (the first value slice only): thread t128 sums 8 consecutive columns
        // (column group cg, one 16-byte k chunk per token) over the tokens of its token
        // group tg; the TG partial sums of a column are added once, at the end.
        constexpr int NCG = DQK / 8, TG = 128 / NCG, TPT = kL / TG;   // column groups, token groups, tokens each
        const int t128 = tid - 128;
        const int cg = t128 % NCG, tg = t128 / NCG;
        float nacc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) nacc[i] = 0.f;
        bool alive = true;
        for (int c = 0; c < NC; ++c) {
            const int s = c % C::STAGES, slot = c % kRing;
            alive = alive && waitw(sh, &bar[C::B_KV_FULL + s], (c / C::STAGES) & 1, kWhereSumKv) &&
                    waitw(sh, &bar[C::B_W_FULL + slot], (c / kRing) & 1, kWhereSumW);
            const float *w = wring + slot * kL;
            if (alive) {
                scale_v_rows(sm + C::OFF_V + s * C::V_BYTES, w, t128);
                fence_proxy_async_smem();   // the MMA (async proxy) reads what these stores wrote
            }
            // unconditional: every warp of the group takes every barrier, even after
            // another warp of it gave up
            named_barrier(1, 128);
            if (t128 == 0 && alive) mbar_arrive(&bar[C::B_VS + s]);
            if (alive && slice == 0) {
                const uint8_t *kb = sm + C::OFF_K + s * C::K_BYTES + (cg >> 3) * 8192;
                uint4 u[TPT];
#pragma unroll
                for (int i = 0; i < TPT; ++i) u[i] = *reinterpret_cast<const uint4 *>(kb + sw128_offset(TPT * tg + i, cg & 7));
#pragma unroll
                for (int i = 0; i < TPT; ++i) {
                    float x[8];
                    unpack_bf16x8(u[i], x);
                    const float wt = w[TPT * tg + i];
#pragma unroll
                    for (int e = 0; e < 8; ++e) nacc[e] = fmaf(wt, x[e], nacc[e]);
                }
            }
            named_barrier(1, 128);
            if (t128 == 0 && alive) {
                mbar_arrive(&bar[C::B_W_EMPTY + slot]);
                mbar_arrive(&bar[C::B_KV_EMPTY + s]);
            }
        }
        alive = alive && waitw(sh, &bar[C::B_DONE], 0, kWhereSumDone);
        // every k stage has been read (all updates are complete): the first one holds
        // the TG x d_qk partial sums of n_seg
        float *part = reinterpret_cast<float *>(sm + C::OFF_K);
        if (alive && slice == 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) part[tg * DQK + 8 * cg + e] = nacc[e];
        }
        named_barrier(1, 128);
        if (alive && slice == 0) {
            for (int j = t128; j < DQK; j += 128) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < TG; ++i) acc += part[i * DQK + j];
                p.segN[((size_t)g * p.BH + bh) * DQK + j] = acc;
            }
        }
        const int v = v0 + t128;
        if (alive && v < p.dv) {   // warp-uniform: d_v is a multiple of 64
            tc_fence_after();
            const uint32_t lane_base = (uint32_t)(32 * (warp - 4)) << 16;
            float *dst = p.segC + (((size_t)g * p.BH + bh) * p.dv + v) * DQK;
            float r[32];
#pragma unroll 1
            for (int i = 0; i < DQK / 32; ++i) {
                tmem_ld32(tm + lane_base + 32 * i, r);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4 *>(dst + 32 * i + x) = make_float4(r[x], r[x + 1], r[x + 2], r[x + 3]);
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, DQK);
    }
}

struct CombineParams {
    int BH, dv, dqk, nsum;
    const float *C0, *n0, *m0;   // caller's initial state (null: zero state, m = 0)
    float *segC, *segN, *segM;   // summaries in, entry states of segments 1..nsum out (in place)
    const double *segS;
    float *C1, *n1, *m1;         // non-null: only the state after the last summary is written, here,
                                 // and the summaries are left as they are
};

// Entry states, in place over the summaries: slot g becomes the state entering
// segment g+1.  One thread per 4 consecutive floats of (C, n) of one sequence;
// every thread runs the scalar chain of gauges itself, in float64.  The loads of
// a batch of segments are issued before any of them is combined, so that the
// chain waits on one memory round trip per batch, not per segment.
__global__ void __launch_bounds__(kCombineThreads) seg_combine_kernel(const CombineParams p) {
    constexpr int kBatch = 8;
    const int bh = blockIdx.y;
    const int nC4 = p.dv * p.dqk / 4, n4 = nC4 + p.dqk / 4;
    const int e4 = blockIdx.x * kCombineThreads + threadIdx.x;
    if (e4 >= n4) return;
    const bool isC = e4 < nC4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (isC && p.C0) x = reinterpret_cast<const float4 *>(p.C0 + (size_t)bh * p.dv * p.dqk)[e4];
    if (!isC && p.n0) x = reinterpret_cast<const float4 *>(p.n0 + (size_t)bh * p.dqk)[e4 - nC4];
    double m = p.m0 ? (double)p.m0[bh] : 0.0;
    auto slot = [&](int g) {
        return isC ? reinterpret_cast<float4 *>(p.segC + ((size_t)g * p.BH + bh) * p.dv * p.dqk) + e4
                   : reinterpret_cast<float4 *>(p.segN + ((size_t)g * p.BH + bh) * p.dqk) + (e4 - nC4);
    };
    for (int g0 = 0; g0 < p.nsum; g0 += kBatch) {
        float4 y[kBatch];
        double F[kBatch], ms[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (g0 + j < p.nsum) {
                const size_t k = ((size_t)(g0 + j) * p.BH + bh) * 2;
                y[j] = *slot(g0 + j);
                F[j] = p.segS[k];
                ms[j] = p.segS[k + 1];
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (g0 + j < p.nsum) {
                // the new gauge, rounded to the fp32 m the chunkwise kernel reads, so that
                // the state handed on is exactly in the gauge it is labelled with
                const double mp = (double)(float)fmax(F[j] + m, ms[j]);
                const float a = (float)exp(F[j] + m - mp), b = (float)exp(ms[j] - mp);
                x = make_float4(fmaf(a, x.x, b * y[j].x), fmaf(a, x.y, b * y[j].y), fmaf(a, x.z, b * y[j].z),
                                fmaf(a, x.w, b * y[j].w));
                if (!p.C1) {
                    *slot(g0 + j) = x;
                    if (e4 == 0) p.segM[(size_t)(g0 + j) * p.BH + bh] = (float)mp;
                }
                m = mp;
            }
        }
    }
    if (p.C1) {
        if (isC)
            reinterpret_cast<float4 *>(p.C1 + (size_t)bh * p.dv * p.dqk)[e4] = x;
        else if (p.n1)
            reinterpret_cast<float4 *>(p.n1 + (size_t)bh * p.dqk)[e4 - nC4] = x;
        if (e4 == 0 && p.m1) p.m1[bh] = (float)m;
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }


template <int DQK>
cudaError_t launch_summaries_dqk(const FwdArgs &a, const SegPlan &sp, cudaStream_t s) {
    using C = SumCfg<DQK>;
    const int BH = a.B * a.H;
    CUtensorMap tk, tv;
    if (!make_tmap_3d_bf16(&tk, a.k, DQK, a.T, BH, 64, 64) || !make_tmap_3d_bf16(&tv, a.v, a.dv, a.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    char *ws = static_cast<char *>(a.seg_ws);
    SumParams p;
    p.T = a.T; p.dv = a.dv; p.nslices = (a.dv + kDvs - 1) / kDvs; p.nsum = sp.nseg - 1;
    p.seg_chunks = sp.seg_chunks; p.BH = BH; p.ig = a.ig; p.fg = a.fg;
    p.segC = reinterpret_cast<float *>(ws + sp.off_C);
    p.segN = reinterpret_cast<float *>(ws + sp.off_N);
    p.segS = reinterpret_cast<double *>(ws + sp.off_S);
    p.status = a.status;
    auto kern = seg_summary_kernel<DQK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<BH * p.nsum * p.nslices, kSumThreads, C::SMEM, s>>>(tk, tv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    CombineParams q;
    q.BH = BH; q.dv = a.dv; q.dqk = DQK; q.nsum = p.nsum;
    q.C0 = a.C0; q.n0 = a.n0; q.m0 = a.m0;
    q.segC = p.segC; q.segN = p.segN; q.segM = reinterpret_cast<float *>(ws + sp.off_M); q.segS = p.segS;
    q.C1 = q.n1 = q.m1 = nullptr;
    const int n4 = (a.dv * DQK + DQK) / 4;
    seg_combine_kernel<<<dim3((n4 + kCombineThreads - 1) / kCombineThreads, BH), kCombineThreads, 0, s>>>(q);
    return cudaGetLastError();
}

template <int DQK>
cudaError_t launch_summary_whole(const FwdArgs &a, float *C_seg, float *n_seg, double *F_m, cudaStream_t s) {
    using C = SumCfg<DQK>;
    const int BH = a.B * a.H;
    CUtensorMap tk, tv;
    if (!make_tmap_3d_bf16(&tk, a.k, DQK, a.T, BH, 64, 64) || !make_tmap_3d_bf16(&tv, a.v, a.dv, a.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    SumParams p;
    p.T = a.T; p.dv = a.dv; p.nslices = (a.dv + kDvs - 1) / kDvs; p.nsum = 1;
    p.seg_chunks = a.T / kL; p.BH = BH; p.ig = a.ig; p.fg = a.fg;
    p.segC = C_seg; p.segN = n_seg; p.segS = F_m; p.status = a.status;
    auto kern = seg_summary_kernel<DQK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<BH * p.nslices, kSumThreads, C::SMEM, s>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

bool summary_supported(const FwdArgs &a) {
    FwdArgs b = a;
    b.chunk = kL;   // a summary does not depend on the chunk length of the forward pass
    return chunkwise_tc_supported(b) && a.T > 0 && a.T % kL == 0 && a.T / kL <= kMaxSegChunks;
}

cudaError_t launch_summary(const FwdArgs &a, float *C_seg, float *n_seg, double *F_m, cudaStream_t s) {
    switch (a.dqk) {
        case 64: return launch_summary_whole<64>(a, C_seg, n_seg, F_m, s);
        case 128: return launch_summary_whole<128>(a, C_seg, n_seg, F_m, s);
        case 256: return launch_summary_whole<256>(a, C_seg, n_seg, F_m, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_combine(int BH, int dv, int dqk, int nsum, const float *C0, const float *n0, const float *m0,
                           const float *segC, const float *segN, const double *segS, float *C1, float *n1, float *m1,
                           cudaStream_t s) {
    CombineParams q;
    q.BH = BH; q.dv = dv; q.dqk = dqk; q.nsum = nsum;
    q.C0 = C0; q.n0 = n0; q.m0 = m0;
    q.segC = const_cast<float *>(segC); q.segN = const_cast<float *>(segN); q.segM = nullptr; q.segS = segS;
    q.C1 = C1; q.n1 = n1; q.m1 = m1;
    const int n4 = (dv * dqk + dqk) / 4;
    seg_combine_kernel<<<dim3((n4 + kCombineThreads - 1) / kCombineThreads, BH), kCombineThreads, 0, s>>>(q);
    return cudaGetLastError();
}

int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0, v = 0;
        n = (cudaGetDevice(&dev) == cudaSuccess &&
             cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
                ? v
                : 148;
    }
    return n;
}

SegPlan segment_plan(const FwdArgs &a) {
    SegPlan sp;
    sp.nseg = 1;
    if (!chunkwise_tc_shape_ok(a)) return sp;
    const long long BH = (long long)a.B * a.H;
    const long long blocks = BH * ((a.dv + kDvs - 1) / kDvs);
    const int NC = (a.T + kL - 1) / kL;
    const long long fit = sm_count() / blocks;   // segments per sequence that still fit one wave
    int G = (int)std::min<long long>(fit, NC / kMinSegChunks);
    if (G < 2) return sp;
    G = std::max(G, (NC + kMaxSegChunks - 1) / kMaxSegChunks);   // no segment longer than kMaxSegChunks
    sp.seg_chunks = (NC + G - 1) / G;
    const int per = a.chunk / kL;   // segments hold whole chunks of the forward pass
    sp.seg_chunks = (sp.seg_chunks + per - 1) / per * per;
    G = (NC + sp.seg_chunks - 1) / sp.seg_chunks;
    if (G < 2) return sp;
    sp.nseg = G;
    const size_t nsum = (size_t)(G - 1) * BH;
    sp.off_S = 0;
    sp.off_M = align256(sp.off_S + nsum * 2 * sizeof(double));
    sp.off_N = align256(sp.off_M + nsum * sizeof(float));
    sp.off_C = align256(sp.off_N + nsum * a.dqk * sizeof(float));
    sp.bytes = align256(sp.off_C + nsum * (size_t)a.dv * a.dqk * sizeof(float));
    return sp;
}

cudaError_t launch_segment_entry_states(const FwdArgs &a, const SegPlan &sp, cudaStream_t s) {
    switch (a.dqk) {
        case 64: return launch_summaries_dqk<64>(a, sp, s);
        case 128: return launch_summaries_dqk<128>(a, sp, s);
        case 256: return launch_summaries_dqk<256>(a, sp, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xlstm
