// Chunkwise mLSTM forward on sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// The math (xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3 with the "sLSTM"
// stabilizer), evaluated per chunk of L = 64 tokens.  With the chunk-local
// cumulative log forget gate F_t = sum_{r<=t} f~_r, u_s = i~_s - F_s and the
// running maximum mu_t = max(m, max_{s<=t} u_s), the stabilizer is exactly
// m_t = F_t + mu_t, and
//   h~_t = [e^{b-mu_t} C_acc q_t + sum_{s<=t} e^{u_s-mu_t} (q_t.k_s) v_s]
//          / max(|e^{b-mu_t} n_acc.q_t + sum_{s<=t} e^{u_s-mu_t} q_t.k_s|, e^{-m_t})
// (q already multiplied by qk_scale).  (C_acc, n_acc) is the state in a lazily
// moved gauge, C~ = e^{b-m} C_acc with b <= m.  The update is
//   C_acc <- e^{b-b'} C_acc + sum_s e^{u_s-b'} v_s k_s^T
// with b' = b (weights <= e^{kRescale}) unless the stabilizer ran more than
// kRescale past b; then b' = mu_L and C_acc is rescaled once in tensor memory.
// Every exponent is <= 0 except those bounded update weights.  The gate scan
// runs in float64 (one warp, 64 tokens per chunk): with strong forgetting F_t
// reaches 1e5 and more inside one chunk, where m_t = F_t + mu_t and the
// pairwise exponents u_s - mu_t would otherwise cancel catastrophically in
// fp32; the pairwise exponents are handed on as float hi/lo pairs.
//
// Block = one (batch, head) and a 128-row slice of d_v; it walks the chunks in
// order with C_acc (128 x d_qk fp32) resident in tensor memory.  Per chunk:
//   S       = Q K^T                           kind::f16 M=64  N=64 K=d_qk
//   H_inter = (C_hi + C_lo) Q^T               kind::f16 M=128 N=64 K=d_qk, A in TMEM
//   H_intra = V^T (P_hi + P_lo)^T             kind::f16 M=128 N=64 K=64
//   C_acc  += (w V)^T K                       kind::f16 M=128 N=d_qk K=64
// C_hi = bf16(C_acc), C_lo = bf16(C_acc - C_hi) (a 16-bit split, ~2^-17
// relative) are written each chunk by the CUDA-core warps; the same split is
// used for P_ts = scale S_ts e^{u_s-mu_t} [s<=t].  A single bf16 or tf32 copy
// of either loses up to 2^-9 / 2^-11 per element, which rows whose readout
// cancels amplify past a 2e-2 tolerance.  q itself is bf16 and exact, so the
// readout multiplies the raw q tile; e^{b-mu_t} scale is applied per token in
// the epilogue:  h~[t][v] = (a_t H_inter[v][t] + H_intra[v][t]) / den_t.
//
// Warp roles: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2 gate scan,
// 3 normaliser n_acc, 4-7 state split, P, epilogue.  Every wait is bounded: a
// wait that gives up records XLSTM_ERR_TIMEOUT in the status block, each role
// drains what it has in flight, tensor memory is freed and the kernel returns.
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace xlstm {
namespace {

using namespace sm100;

constexpr int kL = 64;              // chunk length
constexpr int kDvs = 128;           // rows of C per block
constexpr int kThreads = 256;
constexpr int kNG = 4;              // gate-ring slots
constexpr double kRescale = 20.0;   // gauge drift allowed before C_acc is rescaled
constexpr double kLog2e = 1.4426950408889634;
constexpr uint64_t kTimeoutNs = 1000000000ull;   // 1 s per wait

// Where a wait gave up (reported in the status block).
enum : int32_t {
    kWhereTmaKvEmpty = 1, kWhereTmaQEmpty, kWhereMmaKvFull, kWhereMmaQFull, kWhereMmaSEmpty,
    kWhereMmaOps, kWhereMmaHEmpty, kWhereMmaUpd, kWhereGateEmpty, kWhereNormGate, kWhereNormKv,
    kWhereNormFree, kWhereCwGate, kWhereCwQ, kWhereCwN, kWhereCwS, kWhereCwH, kWhereCwFinal,
    kWhereCwUpd, kWhereMmaConv
};

// Test hook: make the gate warp withhold one hand-off so that its consumers time out.
int g_fault_next = 0;

}  // namespace
void set_chunkwise_tc_fault(int mode) { g_fault_next = mode; }
namespace {

template <int DQK>
struct Cfg {
    static constexpr bool BIG = DQK == 256;            // TMEM is full: C_lo in smem, S shares H_intra
    static constexpr int NKB = DQK / 64;               // 64-column boxes of q and k
    static constexpr int QST = BIG ? 1 : 2;            // q stages
    static constexpr int Q_BYTES = NKB * 8192;
    static constexpr int K_BYTES = NKB * 8192;
    static constexpr int V_BYTES = 2 * 8192;           // 128 value columns
    static constexpr int P_BYTES = 2 * 8192;           // P_hi, P_lo
    static constexpr int CLO_BYTES = BIG ? NKB * 16384 : 0;   // 128 rows x d_qk bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QST * Q_BYTES;
    static constexpr int OFF_V = OFF_K + 2 * K_BYTES;
    static constexpr int OFF_P = OFF_V + 2 * V_BYTES;
    static constexpr int OFF_CLO = OFF_P + P_BYTES;
    // gate ring: per slot UH, UL, MH, ML, A, W, LOWER [64] + 8 chunk scalars
    static constexpr int G_FLOATS = 7 * kL + 8;
    static constexpr int OFF_G = OFF_CLO + CLO_BYTES;
    static constexpr int OFF_N = OFF_G + kNG * G_FLOATS * 4;   // n_acc double buffer
    static constexpr int OFF_SC = OFF_N + 2 * DQK * 4;          // nq, rsum, inv_den [64]
    static constexpr int OFF_BAR = OFF_SC + 3 * kL * 4;
    static constexpr int NBARS = 32;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;          // + alignment slack
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_C = 0;
    static constexpr uint32_t TM_CHI = DQK;
    static constexpr uint32_t TM_CLO = DQK + DQK / 2;          // unused when BIG
    static constexpr uint32_t TM_HI = BIG ? DQK + DQK / 2 : 2 * DQK;
    static constexpr uint32_t TM_HA = TM_HI + 64;
    static constexpr uint32_t TM_S = BIG ? TM_HA : TM_HA + 64;
    static_assert(TM_S + 64 <= TMEM_COLS, "tensor memory budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Gate-ring slot field offsets (floats).
enum : int {
    kGUh = 0, kGUl = kL, kGMh = 2 * kL, kGMl = 3 * kL, kGA = 4 * kL, kGW = 5 * kL, kGLower = 6 * kL,
    kGScal = 7 * kL
};
// Chunk scalars inside a slot.
enum : int { kSRho = 0, kSRescale = 1, kSMEnd = 2, kSGsc = 3 };

// Barrier indices.
enum : int {
    B_KV_FULL = 0, B_KV_EMPTY = 2, B_Q_FULL = 4, B_Q_EMPTY = 6, B_G_FULL = 8, B_G_EMPTY = B_G_FULL + kNG,
    B_S_FULL = B_G_EMPTY + kNG, B_S_EMPTY, B_OPS, B_CONV, B_H_FULL, B_H_EMPTY, B_UPD_READY, B_UPD_DONE,
    B_N_READY, B_N_FREE = B_N_READY + 2, B_DRAIN = B_N_FREE + 2, B_COUNT
};
static_assert(B_COUNT <= 32, "barrier space");

struct TcParams {
    int T, dv, nslices;
    float scale;
    const float *ig, *fg, *C0, *n0, *m0;
    float *h, *C1, *n1, *m1;
    int32_t *status;
    int fault;
};

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
__device__ __forceinline__ bool wait1(const Shared &sh, uint64_t *bar, uint32_t parity, int where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*sh.abort_flag) return false;
        if (global_timer_ns() - t0 > kTimeoutNs) {
            record_timeout(sh, where);
            return false;
        }
    }
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

// x -> (hi, lo) float pair with hi + lo = x to ~2^-48; -inf -> (-inf, 0).
__device__ __forceinline__ void split_double(double x, float &hi, float &lo) {
    hi = (float)x;
    lo = isfinite(hi) ? (float)(x - (double)hi) : 0.f;
}

template <int DQK>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const TcParams p) {
    using C = Cfg<DQK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    Shared sh{reinterpret_cast<volatile int *>(sm + C::OFF_MISC + 4), p.status};
    float *gring = reinterpret_cast<float *>(sm + C::OFF_G);
    float *nbuf = reinterpret_cast<float *>(sm + C::OFF_N);
    float *nq_s = reinterpret_cast<float *>(sm + C::OFF_SC);
    float *rs_s = nq_s + kL;
    float *inv_s = rs_s + kL;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / p.nslices;
    const int slice = blockIdx.x % p.nslices;
    const int v0 = slice * kDvs;
    const int T = p.T;
    const int NC = (T + kL - 1) / kL;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[B_KV_FULL + i], 1); mbar_init(&bar[B_KV_EMPTY + i], 2);
            mbar_init(&bar[B_Q_FULL + i], 1); mbar_init(&bar[B_Q_EMPTY + i], 2);
            mbar_init(&bar[B_N_READY + i], 1); mbar_init(&bar[B_N_FREE + i], 1);
        }
        for (int i = 0; i < kNG; ++i) { mbar_init(&bar[B_G_FULL + i], 1); mbar_init(&bar[B_G_EMPTY + i], 2); }
        mbar_init(&bar[B_S_FULL], 1); mbar_init(&bar[B_S_EMPTY], 1); mbar_init(&bar[B_OPS], 1);
        mbar_init(&bar[B_CONV], 1); mbar_init(&bar[B_H_FULL], 1); mbar_init(&bar[B_H_EMPTY], 1);
        mbar_init(&bar[B_UPD_READY], 1); mbar_init(&bar[B_UPD_DONE], 1); mbar_init(&bar[B_DRAIN], 1);
        *sh.abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    uint8_t *Ps = sm + C::OFF_P;

    if (warp == 0) {
        // ===================== TMA producer =====================
        if (lane == 0) {
            int kv_issued[2] = {0, 0}, q_issued[2] = {0, 0};
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1, qs = c % C::QST;
                if (c >= 2 && !wait1(sh, &bar[B_KV_EMPTY + s], ((c >> 1) - 1) & 1, kWhereTmaKvEmpty)) break;
                mbar_arrive_expect_tx(&bar[B_KV_FULL + s], C::K_BYTES + C::V_BYTES);
                uint8_t *Ks = sm + C::OFF_K + s * C::K_BYTES;
                uint8_t *Vs = sm + C::OFF_V + s * C::V_BYTES;
                for (int b = 0; b < C::NKB; ++b) tma_load_3d(Ks + b * 8192, &tmk, &bar[B_KV_FULL + s], 64 * b, kL * c, bh);
                for (int b = 0; b < 2; ++b) tma_load_3d(Vs + b * 8192, &tmv, &bar[B_KV_FULL + s], v0 + 64 * b, kL * c, bh);
                ++kv_issued[s];
                if (c >= C::QST && !wait1(sh, &bar[B_Q_EMPTY + qs], ((c / C::QST) - 1) & 1, kWhereTmaQEmpty)) break;
                mbar_arrive_expect_tx(&bar[B_Q_FULL + qs], C::Q_BYTES);
                uint8_t *Qs = sm + C::OFF_Q + qs * C::Q_BYTES;
                for (int b = 0; b < C::NKB; ++b) tma_load_3d(Qs + b * 8192, &tmq, &bar[B_Q_FULL + qs], 64 * b, kL * c, bh);
                ++q_issued[qs];
            }
            // drain: every issued copy must land before shared memory is released
            for (int s = 0; s < 2; ++s) {
                if (kv_issued[s]) drain_wait(&bar[B_KV_FULL + s], (kv_issued[s] - 1) & 1);
                if (q_issued[s]) drain_wait(&bar[B_Q_FULL + s], (q_issued[s] - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            const uint32_t idS = make_idesc(64, 64, kFmtBF16, kFmtBF16, 0, 0);
            const uint32_t idR = make_idesc(128, 64, kFmtBF16, kFmtBF16, 0, 0);
            const uint32_t idPV = make_idesc(128, 64, kFmtBF16, kFmtBF16, 1, 0);
            const uint32_t idU = make_idesc(128, DQK, kFmtBF16, kFmtBF16, 1, 1);
            const uint32_t p_addr = smem_u32(Ps), clo_addr = smem_u32(sm + C::OFF_CLO);
            bool issued = false;
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1, qs = c % C::QST;
                const uint32_t q_addr = smem_u32(sm + C::OFF_Q + qs * C::Q_BYTES);
                const uint32_t k_addr = smem_u32(sm + C::OFF_K + s * C::K_BYTES);
                const uint32_t v_addr = smem_u32(sm + C::OFF_V + s * C::V_BYTES);
                if (!wait1(sh, &bar[B_KV_FULL + s], (c >> 1) & 1, kWhereMmaKvFull)) break;
                if (!wait1(sh, &bar[B_Q_FULL + qs], (c / C::QST) & 1, kWhereMmaQFull)) break;
                if (c >= 1 && !wait1(sh, &bar[B_S_EMPTY], (c - 1) & 1, kWhereMmaSEmpty)) break;
                if (C::BIG && c >= 1 && !wait1(sh, &bar[B_H_EMPTY], (c - 1) & 1, kWhereMmaHEmpty)) break;
                tc_fence_after();
                // S = Q K^T
#pragma unroll
                for (int ks = 0; ks < DQK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_f16_ss(tm + C::TM_S, smem_desc_sw128(q_addr + off, 16, 1024),
                               smem_desc_sw128(k_addr + off, 16, 1024), idS, ks > 0);
                }
                issued = true;
                tc_commit(&bar[B_S_FULL]);
                if (!wait1(sh, &bar[B_CONV], c & 1, kWhereMmaConv)) break;
                if (!wait1(sh, &bar[B_OPS], c & 1, kWhereMmaOps)) break;
                if (!C::BIG && c >= 1 && !wait1(sh, &bar[B_H_EMPTY], (c - 1) & 1, kWhereMmaHEmpty)) break;
                tc_fence_after();
                // H_inter = C_hi Q^T + C_lo Q^T
#pragma unroll
                for (int ks = 0; ks < DQK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    mma_f16_ts(tm + C::TM_HI, tm + C::TM_CHI + 8 * ks, smem_desc_sw128(q_addr + off, 16, 1024),
                               idR, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < DQK / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    if (C::BIG)
                        mma_f16_ss(tm + C::TM_HI, smem_desc_sw128(clo_addr + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                                   smem_desc_sw128(q_addr + off, 16, 1024), idR, 1);
                    else
                        mma_f16_ts(tm + C::TM_HI, tm + C::TM_CLO + 8 * ks, smem_desc_sw128(q_addr + off, 16, 1024),
                                   idR, 1);
                }
                // H_intra = V^T P_hi^T + V^T P_lo^T
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < kL / 16; ++ks)
                        mma_f16_ss(tm + C::TM_HA, smem_desc_sw128(v_addr + ks * 2048, 8192, 1024),
                                   smem_desc_sw128(p_addr + part * 8192 + ks * 32, 16, 1024), idPV,
                                   (part | ks) != 0);
                tc_commit(&bar[B_H_FULL]);
                tc_commit(&bar[B_Q_EMPTY + qs]);
                if (!wait1(sh, &bar[B_UPD_READY], c & 1, kWhereMmaUpd)) break;
                tc_fence_after();
                // C_acc += (w V)^T K
#pragma unroll
                for (int ks = 0; ks < kL / 16; ++ks)
                    mma_f16_ss(tm + C::TM_C, smem_desc_sw128(v_addr + ks * 2048, 8192, 1024),
                               smem_desc_sw128(k_addr + ks * 2048, 8192, 1024), idU, 1);
                tc_commit(&bar[B_UPD_DONE]);
                tc_commit(&bar[B_KV_EMPTY + s]);
            }
            if (issued) {   // drain: all issued MMAs complete before tensor memory is freed
                tc_commit(&bar[B_DRAIN]);
                drain_wait(&bar[B_DRAIN], 0);
            }
        }
    } else if (warp == 2) {
        // ===================== gate scan (float64) =====================
        double m = p.m0 ? (double)p.m0[bh] : 0.0;
        double b = m;
        const float *ig = p.ig + (size_t)bh * T, *fg = p.fg + (size_t)bh * T;
        for (int c = 0; c < NC; ++c) {
            const int slot = c % kNG;
            if (c >= kNG && !waitw(sh, &bar[B_G_EMPTY + slot], ((c / kNG) - 1) & 1, kWhereGateEmpty)) break;
            const int t0 = kL * c, len = min(kL, T - t0);
            const int ta = 2 * lane, tb = 2 * lane + 1;
            const double ia = ta < len ? (double)ig[t0 + ta] : -INFINITY, fa = ta < len ? (double)fg[t0 + ta] : 0.0;
            const double ib = tb < len ? (double)ig[t0 + tb] : -INFINITY, fb = tb < len ? (double)fg[t0 + tb] : 0.0;
            // inclusive prefix sum of f over the chunk
            const double pair = fa + fb;
            double incl = pair;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            double excl = __shfl_up_sync(0xffffffffu, incl, 1);
            if (lane == 0) excl = 0.0;
            const double Fa = excl + fa, Fb = Fa + fb;
            const double ua = ia - Fa, ub = ib - Fb;
            // running max of u, seeded with m
            double run = fmax(ua, ub);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run = fmax(run, y);
            }
            double before = __shfl_up_sync(0xffffffffu, run, 1);
            if (lane == 0) before = -INFINITY;
            const double mua = fmax(fmax(m, before), ua), mub = fmax(mua, ub);
            const double muL = __shfl_sync(0xffffffffu, mub, 31);
            const double FL = __shfl_sync(0xffffffffu, Fb, 31);
            const bool rescale = muL - b > kRescale;
            const double bnew = rescale ? muL : b;
            float *g = gring + slot * C::G_FLOATS;
            split_double(ua * kLog2e, g[kGUh + ta], g[kGUl + ta]);
            split_double(ub * kLog2e, g[kGUh + tb], g[kGUl + tb]);
            split_double(mua * kLog2e, g[kGMh + ta], g[kGMl + ta]);
            split_double(mub * kLog2e, g[kGMh + tb], g[kGMl + tb]);
            g[kGA + ta] = p.scale * expf((float)(b - mua));
            g[kGA + tb] = p.scale * expf((float)(b - mub));
            g[kGW + ta] = expf((float)(ua - bnew));
            g[kGW + tb] = expf((float)(ub - bnew));
            g[kGLower + ta] = expf((float)(-(Fa + mua)));
            g[kGLower + tb] = expf((float)(-(Fb + mub)));
            const float rho = expf((float)(b - bnew));
            m = FL + muL;
            b = bnew + FL;
            if (lane == 0) {
                g[kGScal + kSRho] = rho;
                g[kGScal + kSRescale] = rescale ? 1.f : 0.f;
                g[kGScal + kSMEnd] = (float)m;
                g[kGScal + kSGsc] = expf((float)(b - m));   // final-state gauge factor e^{b-m}
            }
            __syncwarp();
            if (lane == 0 && !(p.fault == 1 && c == 1)) mbar_arrive(&bar[B_G_FULL + slot]);
        }
    } else if (warp == 3) {
        // ===================== normaliser n_acc =====================
        constexpr int NPL = DQK / 32;             // columns per lane
        const int j0 = lane * NPL;
        float nacc[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) nacc[i] = p.n0 ? p.n0[(size_t)bh * DQK + j0 + i] : 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) nbuf[j0 + i] = nacc[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_N_READY]);
        float gsc = 1.f;
        bool alive = true;
        for (int c = 0; c < NC && alive; ++c) {
            const int slot = c % kNG, s = c & 1;
            alive = waitw(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereNormGate) &&
                    waitw(sh, &bar[B_KV_FULL + s], (c >> 1) & 1, kWhereNormKv);
            if (!alive) break;
            const float *g = gring + slot * C::G_FLOATS;
            const float rho = g[kGScal + kSRho];
            gsc = g[kGScal + kSGsc];
#pragma unroll
            for (int i = 0; i < NPL; ++i) nacc[i] *= rho;
            const uint8_t *Ks = sm + C::OFF_K + s * C::K_BYTES;
            const uint32_t box = j0 >> 6, chunk = (j0 & 63) >> 3, within = (j0 & 7) * 2;
            for (int t = 0; t < kL; ++t) {
                const float w = g[kGW + t];
                const uint8_t *src = Ks + box * 8192 + sw128_offset(t, chunk) + within;
                if (NPL == 8) {
                    float x[8];
                    unpack_bf16x8(*reinterpret_cast<const uint4 *>(src), x);
#pragma unroll
                    for (int i = 0; i < 8; ++i) nacc[i % NPL] = fmaf(w, x[i], nacc[i % NPL]);
                } else if (NPL == 4) {
                    const uint2 u = *reinterpret_cast<const uint2 *>(src);
                    const float x[4] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y)};
#pragma unroll
                    for (int i = 0; i < 4; ++i) nacc[i % NPL] = fmaf(w, x[i], nacc[i % NPL]);
                } else {
                    const uint32_t u = *reinterpret_cast<const uint32_t *>(src);
                    const float x[2] = {bf_lo(u), bf_hi(u)};
#pragma unroll
                    for (int i = 0; i < 2; ++i) nacc[i % NPL] = fmaf(w, x[i], nacc[i % NPL]);
                }
            }
            const int nb = (c + 1) & 1;
            if (c >= 1 && !waitw(sh, &bar[B_N_FREE + nb], ((c - 1) >> 1) & 1, kWhereNormFree)) { alive = false; break; }
#pragma unroll
            for (int i = 0; i < NPL; ++i) nbuf[nb * DQK + j0 + i] = nacc[i];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar[B_N_READY + nb]);
                mbar_arrive(&bar[B_KV_EMPTY + s]);
                mbar_arrive(&bar[B_G_EMPTY + slot]);
            }
        }
        if (alive && slice == 0 && p.n1) {
#pragma unroll
            for (int i = 0; i < NPL; ++i) p.n1[(size_t)bh * DQK + j0 + i] = nacc[i] * gsc;
        }
    } else {
        // ===================== state split, P, epilogue (warps 4-7) =====================
        const int ct = tid - 128;            // 0..127: TMEM lane / C row of this block
        const int wq = warp - 4;             // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const int v = v0 + ct;
        float *hout = p.h + (size_t)bh * T * p.dv + v;
        uint8_t *clo_s = sm + C::OFF_CLO;
        // initial state into tensor memory: C_acc = C0 (b = m = m0) or zero
        {
            float r[32];
            const float *src = p.C0 ? p.C0 + ((size_t)bh * p.dv + v) * DQK : nullptr;
#pragma unroll 1
            for (int i = 0; i < DQK / 32; ++i) {
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = src ? src[32 * i + x] : 0.f;
                tmem_st32(tm + lane_base + C::TM_C + 32 * i, r);
            }
            tmem_wait_st();
        }
        bool alive = true;
        float m_end = p.m0 ? p.m0[bh] : 0.f, gsc = 1.f;
        const int trow = ct >> 1, half = ct & 1;     // nq pass: row and half of d_qk
        for (int c = 0; c < NC; ++c) {
            const int slot = c % kNG, s = c & 1, qs = c % C::QST;
            const float *g = gring + slot * C::G_FLOATS;
            // --- split the state at chunk start into C_hi + C_lo (bf16 pair)
            if (c >= 1) alive = alive && waitw(sh, &bar[B_UPD_DONE], (c - 1) & 1, kWhereCwUpd);
            if (alive) {
                tc_fence_after();
                float r[32];
#pragma unroll 1
                for (int i = 0; i < DQK / 32; ++i) {
                    tmem_ld32(tm + lane_base + C::TM_C + 32 * i, r);
                    tmem_wait_ld();
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        hi[x] = pack_bf16x2(r[2 * x], r[2 * x + 1]);
                        lo[x] = pack_bf16x2(r[2 * x] - bf_lo(hi[x]), r[2 * x + 1] - bf_hi(hi[x]));
                    }
                    tmem_st16(tm + lane_base + C::TM_CHI + 16 * i, hi);
                    if (C::BIG) {
                        // K-major 128B-swizzled [128 rows][d_qk] bf16 tile, row ct
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int j = 32 * i + 8 * q4;
                            *reinterpret_cast<uint4 *>(clo_s + (j >> 6) * 16384 + sw128_offset(ct, (j & 63) >> 3)) =
                                make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
                        }
                    } else {
                        tmem_st16(tm + lane_base + C::TM_CLO + 16 * i, lo);
                    }
                }
                tmem_wait_st();
                if (C::BIG) fence_proxy_async_smem();
                tc_fence_before();
            }
            named_barrier(1, 128);
            if (ct == 0 && alive) mbar_arrive(&bar[B_CONV]);
            // --- nq_t = a_t (n_acc . q_t) in fp32
            alive = alive && waitw(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereCwGate);
            alive = alive && waitw(sh, &bar[B_Q_FULL + qs], (c / C::QST) & 1, kWhereCwQ);
            alive = alive && waitw(sh, &bar[B_N_READY + (c & 1)], (c >> 1) & 1, kWhereCwN);
            if (alive) {
                const uint8_t *Qs = sm + C::OFF_Q + qs * C::Q_BYTES;
                const float *nn = nbuf + (c & 1) * DQK;
                float nq = 0.f;
#pragma unroll 4
                for (int gi = 0; gi < DQK / 16; ++gi) {
                    const int j = half * (DQK / 2) + 8 * gi;
                    const uint4 u = *reinterpret_cast<const uint4 *>(Qs + (j >> 6) * 8192 + sw128_offset(trow, (j & 63) >> 3));
                    float x[8];
                    unpack_bf16x8(u, x);
                    const float4 n0 = *reinterpret_cast<const float4 *>(nn + j);
                    const float4 n1 = *reinterpret_cast<const float4 *>(nn + j + 4);
                    nq = fmaf(x[0], n0.x, nq); nq = fmaf(x[1], n0.y, nq);
                    nq = fmaf(x[2], n0.z, nq); nq = fmaf(x[3], n0.w, nq);
                    nq = fmaf(x[4], n1.x, nq); nq = fmaf(x[5], n1.y, nq);
                    nq = fmaf(x[6], n1.z, nq); nq = fmaf(x[7], n1.w, nq);
                }
                nq += __shfl_xor_sync(0xffffffffu, nq, 1);
                if (half == 0) nq_s[trow] = g[kGA + trow] * nq;
            }
            named_barrier(1, 128);
            if (ct == 0 && alive) {
                mbar_arrive(&bar[B_Q_EMPTY + qs]);
                mbar_arrive(&bar[B_N_FREE + (c & 1)]);
            }
            // --- P = scale S e^{u_s - mu_t} on s <= t as a bf16 hi/lo pair
            alive = alive && waitw(sh, &bar[B_S_FULL], c & 1, kWhereCwS);
            if (alive) {
                tc_fence_after();
                float r0[32], r1[32];
                tmem_ld32(tm + lane_base + C::TM_S, r0);
                tmem_ld32(tm + lane_base + C::TM_S + 32, r1);
                tmem_wait_ld();
                if (lane < 16) {
                    const int t = 16 * wq + lane;
                    const float mh = g[kGMh + t], ml = g[kGMl + t];
                    float rs = 0.f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int s0 = 8 * ch + 2 * i;
                            const float sa = (s0 < 32) ? r0[s0] : r1[s0 - 32];
                            const float sb = (s0 + 1 < 32) ? r0[s0 + 1] : r1[s0 - 31];
                            const float ea = (g[kGUh + s0] - mh) + (g[kGUl + s0] - ml);
                            const float eb = (g[kGUh + s0 + 1] - mh) + (g[kGUl + s0 + 1] - ml);
                            const float pa = (s0 <= t) ? p.scale * sa * exp2f(ea) : 0.f;
                            const float pb = (s0 + 1 <= t) ? p.scale * sb * exp2f(eb) : 0.f;
                            hi[i] = pack_bf16x2(pa, pb);
                            lo[i] = pack_bf16x2(pa - bf_lo(hi[i]), pb - bf_hi(hi[i]));
                            rs += pa + pb;
                        }
                        *reinterpret_cast<uint4 *>(Ps + sw128_offset(t, ch)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4 *>(Ps + 8192 + sw128_offset(t, ch)) =
                            make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                    rs_s[t] = rs;
                }
                tc_fence_before();
                fence_proxy_async_smem();
            }
            named_barrier(1, 128);
            if (ct == 0 && alive) {
                mbar_arrive(&bar[B_S_EMPTY]);
                mbar_arrive(&bar[B_OPS]);
            }
            if (alive && ct < kL)
                inv_s[ct] = 1.f / fmaxf(fabsf(nq_s[ct] + rs_s[ct]), g[kGLower + ct]);
            // --- after the readout: gauge move of C_acc, then V <- w V in place
            alive = alive && waitw(sh, &bar[B_H_FULL], c & 1, kWhereCwH);
            if (alive) {
                tc_fence_after();
                if (g[kGScal + kSRescale] != 0.f) {   // C_acc *= e^{b - b'}
                    const float rho = g[kGScal + kSRho];
                    float r[32];
#pragma unroll 1
                    for (int i = 0; i < DQK / 32; ++i) {
                        tmem_ld32(tm + lane_base + C::TM_C + 32 * i, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) r[x] *= rho;
                        tmem_st32(tm + lane_base + C::TM_C + 32 * i, r);
                    }
                    tmem_wait_st();
                }
                uint8_t *Vs = sm + C::OFF_V + s * C::V_BYTES;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = ct + 128 * i;              // 16-byte chunk index in the stage
                    const float w = g[kGW + ((e & 511) >> 3)];   // rows are tokens
                    uint4 *ptr = reinterpret_cast<uint4 *>(Vs + 16 * e);
                    float x[8];
                    unpack_bf16x8(*ptr, x);
                    *ptr = make_uint4(pack_bf16x2(w * x[0], w * x[1]), pack_bf16x2(w * x[2], w * x[3]),
                                      pack_bf16x2(w * x[4], w * x[5]), pack_bf16x2(w * x[6], w * x[7]));
                }
                fence_proxy_async_smem();
                tc_fence_before();
            }
            named_barrier(1, 128);
            if (ct == 0 && alive) mbar_arrive(&bar[B_UPD_READY]);
            // --- epilogue: h~[t][v] = (a_t H_inter[v][t] + H_intra[v][t]) / den_t
            if (alive) {
                const int len = min(kL, T - kL * c);
                float *hc = hout + (size_t)kL * c * p.dv;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float ri[32], ra[32];
                    tmem_ld32(tm + lane_base + C::TM_HI + 32 * hh, ri);
                    tmem_ld32(tm + lane_base + C::TM_HA + 32 * hh, ra);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int t = 32 * hh + x;
                        const float hv = fmaf(g[kGA + t], ri[x], ra[x]) * inv_s[t];
                        if (t < len) hc[(size_t)t * p.dv] = hv;
                    }
                }
                m_end = g[kGScal + kSMEnd];
                gsc = g[kGScal + kSGsc];
                tc_fence_before();
            }
            named_barrier(1, 128);
            if (ct == 0 && alive) {
                mbar_arrive(&bar[B_H_EMPTY]);
                mbar_arrive(&bar[B_G_EMPTY + slot]);
            }
        }
        // final state: C~ = e^{b - m} C_acc
        alive = alive && waitw(sh, &bar[B_UPD_DONE], (NC - 1) & 1, kWhereCwFinal);
        if (alive) {
            tc_fence_after();
            if (p.C1) {
                float r[32];
                float *dst = p.C1 + ((size_t)bh * p.dv + v) * DQK;
#pragma unroll 1
                for (int i = 0; i < DQK / 32; ++i) {
                    tmem_ld32(tm + lane_base + C::TM_C + 32 * i, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; x += 4)
                        *reinterpret_cast<float4 *>(dst + 32 * i + x) =
                            make_float4(r[x] * gsc, r[x + 1] * gsc, r[x + 2] * gsc, r[x + 3] * gsc);
                }
            }
            if (slice == 0 && ct == 0 && p.m1) p.m1[bh] = m_end;
        }
        tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, C::TMEM_COLS);
    }
}

template <int DQK>
cudaError_t launch_dqk(const FwdArgs &a, cudaStream_t s, int fault) {
    using C = Cfg<DQK>;
    const int BH = a.B * a.H;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_3d_bf16(&tq, a.q, DQK, a.T, BH, 64, 64) || !make_tmap_3d_bf16(&tk, a.k, DQK, a.T, BH, 64, 64) ||
        !make_tmap_3d_bf16(&tv, a.v, a.dv, a.T, BH, 64, 64))
        return cudaErrorInvalidValue;
    TcParams p;
    p.T = a.T; p.dv = a.dv; p.nslices = a.dv / kDvs; p.scale = a.scale;
    p.ig = a.ig; p.fg = a.fg; p.C0 = a.C0; p.n0 = a.n0; p.m0 = a.m0;
    p.h = a.h; p.C1 = a.C1; p.n1 = a.n1; p.m1 = a.m1; p.status = a.status; p.fault = fault;
    auto kern = chunk_tc_kernel<DQK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<BH * p.nslices, kThreads, C::SMEM, s>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

bool chunkwise_tc_supported(const FwdArgs &a) {
    if (a.dtype != XLSTM_BF16 || a.chunk != kL || a.T < 1) return false;
    if (a.dv % kDvs != 0) return false;
    if (a.dqk != 64 && a.dqk != 128 && a.dqk != 256) return false;
    return encode_tiled_fn() != nullptr;
}

cudaError_t launch_chunkwise_tc(const FwdArgs &a, cudaStream_t s) {
    const int fault = g_fault_next;
    g_fault_next = 0;
    switch (a.dqk) {
        case 64: return launch_dqk<64>(a, s, fault);
        case 128: return launch_dqk<128>(a, s, fault);
        case 256: return launch_dqk<256>(a, s, fault);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xlstm
