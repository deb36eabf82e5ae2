// Chunkwise mLSTM forward on sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// The math (xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3 with the "sLSTM"
// stabilizer), evaluated per chunk of L = 64 tokens, or L = 128 for d_qk <= 128.  With the chunk-local
// cumulative log forget gate F_t = sum_{r<=t} f~_r, u_s = i~_s - F_s and the
// running maximum mu_t = max(m, max_{s<=t} u_s), the stabilizer is exactly
// m_t = F_t + mu_t, and (q already multiplied by qk_scale)
//   h~_t = [e^{b-mu_t} C_acc q_t + sum_{s<=t} e^{u_s-mu_t} (q_t.k_s) v_s]
//          / max(|e^{b-mu_t} n_acc.q_t + sum_{s<=t} e^{u_s-mu_t} q_t.k_s|, e^{-m_t}).
// (C_acc, n_acc) is the state in a lazily moved gauge: C~ = e^{b-m} C_acc, b <= m.
//
// Each chunk picks a reference r (>= b) and weights w_s = e^{u_s-r}:
//   fast chunk (the stabilizer rises by at most kGrowth inside the chunk):
//     r = b if mu_L - b <= kRescale, else mu_L - kRescale (the state is then
//     rescaled by rho = e^{b-r} as it is split).  Because e^{u_s-mu_t} =
//     w_s e^{r-mu_t}, one accumulator holds the whole numerator,
//        H = (rho C_acc) Q^T + (w V)^T (mask S)^T,    h~_t = a_t H_t / den_t,
//     with a_t = scale e^{r-mu_t} <= scale e^{kGrowth-kRescale}, w_s <= e^{kRescale}:
//     no per-element exponentials and no overflow.
//   exact chunk (the stabilizer jumps by more, e.g. a forget gate near zero):
//     r = mu_L, P_ts = scale S_ts e^{u_s-mu_t} element by element (every
//     exponent <= 0), the intra part kept in its own accumulator.
// The update is C_acc <- rho C_acc + (w V)^T K, b <- r + F_L.  The gate scan runs
// in float64 (one warp): inside a chunk F_t can reach 1e5 (strong forgetting),
// where m_t = F_t + mu_t and u_s - mu_t would cancel in fp32; pairwise
// exponents are handed on as float hi/lo pairs.
//
// Block = one (batch, head) and 128 value rows; C_acc (128 x d_qk fp32) lives in
// tensor memory for the whole sequence.  Per chunk, on the tensor cores:
//   S   = Q K^T                          kind::f16 M=L   N=L  K=d_qk (M = 64 or 128)
//   H   = (C_hi + C_lo) Q^T              kind::f16 M=128 N=L  K=d_qk (C_hi from TMEM)
//   H  += (w V)^T P^T                    kind::f16 M=128 N=L  K=L
//   C_acc += (w V)^T K                   kind::f16 M=128 N=d_qk K=L
// C_hi = bf16(C), C_lo = bf16(C - C_hi) give ~2^-17 relative operands: a single
// bf16 or tf32 copy of the state loses 2^-9 / 2^-11 per element, which rows whose
// readout cancels against the rest of the state amplify past 2e-2.  The intra
// weights P are one bf16 copy (rounded to nearest): every P_ts multiplies a single
// value vector, so its 2^-9 error stays relative to that term (at most 8e-3 of a
// row in the stress cases, against 2e-2).  q is bf16 and exact, so the raw q tile
// is the readout operand.  For d_qk = 256 tensor
// memory is full (C_acc 256 + C_hi 128 + H 64 + S 64 columns) and C_lo goes
// through a 32 KB shared half-buffer, refilled while the first half is read.
// With L = 128 (d_qk <= 128) the chunk's S and H take 128 columns each (for
// d_qk = 128: C_acc 128 + C_hi 64 + C_lo 64 + H 128 + S 128 = all 512), every
// chunk issues about 3/8 fewer MMAs per token and splits the state half as
// often; V then has one shared-memory stage (the two-stage q and k tiles and the
// 32 KB P tile fill the rest), loaded once the previous chunk's update is done.
//
// Warps: 0 TMA producer (and L2 prefetch two chunks ahead), 1 MMA issuer (owns
// TMEM), 2 gate scan, 3 normaliser (warps 0 and 3 swap roles at L = 128 and at
// d_qk = 256),
// 4-7 state group (the first columns of the state split, n.q, epilogue), 8-11
// token group (w V, the other columns of the state split, P).
// Every wait is bounded: one that gives up records XLSTM_ERR_TIMEOUT in the
// status block; each role drains what it has in flight, TMEM is freed, return.
#include <math.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "tma_host.cuh"

#include <mutex>

namespace xlstm {
namespace {

using namespace sm100;

constexpr int kDvs = 128;           // value rows per block

constexpr int kThreads = 384;
constexpr int kNG = 4;              // gate-ring slots
constexpr double kRescale = 20.0;   // gauge drift allowed before the state is rescaled
constexpr double kGrowth = 90.0;    // stabilizer rise inside a chunk handled by the fast path
constexpr double kLog2e = 1.4426950408889634;

// Where a wait gave up (reported in the status block).
enum : int32_t {
    kWhereTmaKvEmpty = 1, kWhereTmaQEmpty, kWhereMmaKvFull, kWhereMmaQFull, kWhereMmaSEmpty, kWhereMmaGate,
    kWhereMmaConv, kWhereMmaOps, kWhereMmaVt, kWhereMmaHEmpty, kWhereMmaClo, kWhereGateEmpty, kWhereNormGate,
    kWhereNormKv, kWhereNormFree, kWhereStUpd, kWhereStGate, kWhereStClo, kWhereStOps, kWhereStH, kWhereStFinal,
    kWhereTkH, kWhereTkGate, kWhereTkKv, kWhereTkQ, kWhereTkN, kWhereTkS, kWhereTkUpd, kWhereTkClo, kWhereTkConv,
    kWhereStQ, kWhereStN
};

// Test hook: make the gate warp withhold one hand-off so that its consumers time out.
int g_fault_next = 0;


}  // namespace
void set_chunkwise_tc_fault(int mode) { g_fault_next = mode; }
namespace {

template <int DQK, int L>
struct Cfg {
    static_assert(L == 64 || (L == 128 && DQK <= 128), "chunk length");
    static constexpr int kL = L;
    static constexpr bool BIG = DQK == 256;
    // 32-column blocks of the state split done by the state group; the token group
    // does the rest.  The state group comes to the split from the previous chunk's
    // epilogue, the token group straight from the update, so it takes the larger part.
    static constexpr int SPLIT_ST = BIG ? 2 : (DQK == 128 ? 1 : 0);
    static constexpr int NKB = DQK / 64;               // 64-column boxes of q and k
    static constexpr int BOX = L * 128;                // bytes of one 64-column box of an L-row tile
    static constexpr int Q_BYTES = NKB * BOX;
    static constexpr int K_BYTES = NKB * BOX;
    static constexpr int V_BYTES = 2 * BOX;            // 128 value columns
    static constexpr int VST = L == 64 ? 2 : 1;        // V stages
    static constexpr int P_BYTES = L * L * 2;          // P, bf16: L/64 boxes of L rows
    static constexpr int CLO_BYTES = BIG ? 2 * 16384 : 0;     // half of C_lo: 128 rows x 128 cols bf16
    static constexpr int OFF_Q = 0;                    // two stages each
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + 2 * K_BYTES;
    static constexpr int OFF_P = OFF_V + VST * V_BYTES;
    static constexpr int OFF_CLO = OFF_P + P_BYTES;
    // gate ring: per slot UH, UL, MH, ML, AH, AN, W, LOWER [L] + 8 chunk scalars
    static constexpr int G_UH = 0, G_UL = L, G_MH = 2 * L, G_ML = 3 * L, G_AH = 4 * L, G_AN = 5 * L, G_W = 6 * L,
                         G_LOWER = 7 * L, G_SCAL = 8 * L;
    static constexpr int G_FLOATS = 8 * L + 8;
    static constexpr int OFF_G = OFF_CLO + CLO_BYTES;
    // n_acc double buffer; the upper half of the columns sits 16 bytes further on so
    // that the two threads of a token (one per half) read from different banks
    static constexpr int NBUF = DQK + 4;
    static constexpr int OFF_N = OFF_G + kNG * G_FLOATS * 4;
    static constexpr int OFF_SC = OFF_N + 2 * NBUF * 4;         // nq, rsum, inv, coef [2][L] each
    static constexpr int OFF_BAR = OFF_SC + 8 * L * 4;
    static constexpr int NBARS = 48;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;          // + alignment slack
    static constexpr uint32_t TM_C = 0;
    static constexpr uint32_t TM_CHI = DQK;
    static constexpr uint32_t TM_CLO = DQK + DQK / 2;          // unused when BIG
    static constexpr uint32_t TM_H = BIG ? DQK + DQK / 2 : 2 * DQK;
    static constexpr uint32_t TM_S = TM_H + L;                 // S, or the intra part of an exact chunk
    // tensor-memory columns allocated (a power of two): 256 when the state, its readout
    // copy and one chunk's S and H fit (d_qk = 64, L = 64), and then two blocks share an SM
    static constexpr uint32_t TMEM_COLS = TM_S + L <= 256 ? 256 : 512;
    static_assert(TM_S + L <= TMEM_COLS, "tensor memory budget");
    // blocks per SM: two when tensor memory, shared memory (228 KB per SM, 1 KB of it
    // reserved per block) and 80 registers a thread allow; the kernel's launch bounds
    static constexpr int CTAS = TMEM_COLS == 256 && 2 * (SMEM + 1024) <= 233472 ? 2 : 1;
    static_assert(SMEM <= 232448, "shared memory budget");
};

// Chunk scalars at G_SCAL of a gate-ring slot.
enum : int { kSRho = 0, kSRescale = 1, kSExact = 2, kSMEnd = 3, kSGsc = 4 };

// Barriers.
enum : int {
    B_K_FULL = 0, B_K_EMPTY = 2, B_V_FULL = 4, B_V_EMPTY = 6, B_Q_FULL = 8, B_Q_EMPTY = 10, B_G_FULL = 12,
    B_G_EMPTY = B_G_FULL + kNG,
    // B_VT: w V is in place for a fast chunk (token group); B_VT_EXACT: the gauge
    // move and w V of an exact chunk are done (state group).  Two producers on one
    // barrier could complete two phases before the MMA warp waits for the first.
    // B_OPS (P and the row sums of chunk c) and, with two V stages, B_VT come in pairs
    // indexed by the chunk's parity: the phase for chunk c+2 cannot complete before
    // each consumer has waited for chunk c's (it needs a later hand-off of that
    // consumer: the epilogue of c, or the update of c), where one barrier's phase for
    // c+1 could.
    B_S_FULL = B_G_EMPTY + kNG, B_S_EMPTY, B_OPS, B_VT = B_OPS + 2, B_VT_EXACT = B_VT + 2, B_CONV0, B_CONV1,
    B_CLO_FREE, B_H_FULL, B_H_EMPTY,
    B_UPD_DONE, B_N_READY, B_N_FREE = B_N_READY + 2, B_DRAIN = B_N_FREE + 2, B_COUNT
};
static_assert(B_COUNT <= 48, "barrier space");

struct TcParams {
    int T, dv, nslices;
    int nseg, seg_len, BH;      // the sequence in nseg segments of seg_len tokens (nseg = 1: whole)
    float scale;
    const float *ig, *fg, *C0, *n0, *m0;
    const float *segC, *segN, *segM;   // entry states of segments 1 .. nseg-1
    float *h, *C1, *n1, *m1;
    int32_t *status;
    int fault;
    int block0;   // index of this launch's first block in the whole grid (a split launch)
};

// Entry state of segment seg of sequence bh: the caller's (or none: zero state,
// m = 0) for the first segment, the combined summaries of the earlier segments
// for the others.  Pointers to the (bh) row: C [d_v][d_qk], n [d_qk], m scalar.
template <int DQK>
__device__ __forceinline__ const float *entry_C(const TcParams &p, int bh, int seg) {
    if (seg == 0) return p.C0 ? p.C0 + (size_t)bh * p.dv * DQK : nullptr;
    return p.segC + ((size_t)(seg - 1) * p.BH + bh) * p.dv * DQK;
}
template <int DQK>
__device__ __forceinline__ const float *entry_n(const TcParams &p, int bh, int seg) {
    if (seg == 0) return p.n0 ? p.n0 + (size_t)bh * DQK : nullptr;
    return p.segN + ((size_t)(seg - 1) * p.BH + bh) * DQK;
}
__device__ __forceinline__ const float *entry_m(const TcParams &p, int bh, int seg) {
    if (seg == 0) return p.m0 ? p.m0 + bh : nullptr;
    return p.segM + (size_t)(seg - 1) * p.BH + bh;
}

// (x0, x1) -> bf16 pairs hi = trunc(x), lo = round(x - hi): |x - hi - lo| <= 2^-16 |x|.
// The high half is a plain truncation (two masks and a byte permute) so that
// only the residual needs a rounding conversion.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const uint32_t a = __float_as_uint(x0), b = __float_as_uint(x1);
    hi = __byte_perm(a, b, 0x7632);
    const float2 r = __fadd2_rn(make_float2(x0, x1), make_float2(__uint_as_float((a & 0xFFFF0000u) ^ 0x80000000u),
                                                                __uint_as_float((b & 0xFFFF0000u) ^ 0x80000000u)));
    lo = pack_bf16x2(r.x, r.y);
}
// Descriptor offset (16-byte units) of K-step ks in a K-major 128B-swizzled tile of
// 64-column boxes BOX bytes apart (q, k and P tiles: L rows of 128 B; the C_lo
// tile: 128 rows).
template <int BOX>
__device__ __forceinline__ uint32_t kstep(int ks) { return (uint32_t)(((ks >> 2) * BOX + (ks & 3) * 32) >> 4); }

// Padded index of column j in an n buffer.
template <int DQK>
__device__ __forceinline__ int nidx(int j) { return j + (j >= DQK / 2 ? 4 : 0); }

// x -> (hi, lo) float pair with hi + lo = x to ~2^-48; -inf -> (-inf, 0).
__device__ __forceinline__ void split_double(double x, float &hi, float &lo) {
    hi = (float)x;
    lo = isfinite(hi) ? (float)(x - (double)hi) : 0.f;
}

// 32 consecutive floats of a shared array into registers (broadcast loads).
__device__ __forceinline__ void load32(const float *src, float (&d)[32]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float4 x = reinterpret_cast<const float4 *>(src)[i];
        d[4 * i] = x.x; d[4 * i + 1] = x.y; d[4 * i + 2] = x.z; d[4 * i + 3] = x.w;
    }
}

// One 32-column block [32 i, 32 i + 32) of this thread's C_acc row: optional
// gauge move (C_acc *= rho, written back), then the split C = C_hi + C_lo.
// lo_mode: 0 C_hi and C_lo to TMEM; 1 C_hi to TMEM, C_lo to the shared tile at
// local column jlo; 2 C_hi only; 3 C_lo only (shared tile, no gauge move).
template <class C>
__device__ __forceinline__ void split_state_block(float (&r)[32], uint32_t tm, uint32_t lane_base, int i, bool mv,
                                                  float rho, int lo_mode, uint8_t *clo_s, int row, int jlo) {
    if (mv) {
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
            const float2 y = __fmul2_rn(make_float2(r[x], r[x + 1]), make_float2(rho, rho));
            r[x] = y.x; r[x + 1] = y.y;
        }
        tmem_st32(tm + lane_base + C::TM_C + 32 * i, r);
    }
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) split_bf16x2(r[2 * x], r[2 * x + 1], hi[x], lo[x]);
    if (lo_mode != 3) tmem_st16(tm + lane_base + C::TM_CHI + 16 * i, hi);
    if (lo_mode == 0) {
        tmem_st16(tm + lane_base + C::TM_CLO + 16 * i, lo);
    } else if (lo_mode == 1 || lo_mode == 3) {   // K-major 128B-swizzled [128 rows][128 cols] bf16 half tile
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const int j = jlo + 8 * q4;
            *reinterpret_cast<uint4 *>(clo_s + (j >> 6) * 16384 + sw128_offset(row, (j & 63) >> 3)) =
                make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
        }
    }
}

// ---- exact-chunk paths (rare: the stabilizer jumps inside the chunk), kept out of
// line so that the per-chunk code of the fast path stays compact in the
// instruction cache.

// C_acc *= rho over this thread's row (gauge move to r = mu_L), then V <- w V.
template <class C>
__device__ __noinline__ void exact_gauge_move_and_scale_v(uint32_t tm, uint32_t lane_base, float rho, uint8_t *Vs,
                                                          const float *w, int t128) {
    float r[32];
#pragma unroll 1
    for (int i = 0; i < C::NKB * 2; ++i) {
        tmem_ld32(tm + lane_base + C::TM_C + 32 * i, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) r[x] *= rho;
        tmem_st32(tm + lane_base + C::TM_C + 32 * i, r);
    }
    tmem_wait_st();
    scale_v_rows<C::kL>(Vs, w, t128);
}

// Epilogue of an exact chunk: h~ = coef_t H + inv_t intra, each 32-token group.
template <class C>
__device__ __noinline__ void exact_epilogue(uint32_t tm, uint32_t lane_base, const float *coef, const float *inv,
                                            float *hc, size_t dv, int len) {
#pragma unroll 1
    for (int hh = 0; hh < C::kL / 32; ++hh) {
        float rh[32], ra[32], cf[32];
        tmem_ld32(tm + lane_base + C::TM_H + 32 * hh, rh);
        tmem_ld32(tm + lane_base + C::TM_S + 32 * hh, ra);
        load32(coef + 32 * hh, cf);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) rh[x] *= cf[x];
        load32(inv + 32 * hh, cf);
#pragma unroll
        for (int x = 0; x < 32; ++x) rh[x] = fmaf(ra[x], cf[x], rh[x]);
        float *hrow = hc + (size_t)32 * hh * dv;
        const int n = min(32, len - 32 * hh);
#pragma unroll 1
        for (int x = 0; x < n; ++x) hrow[(size_t)x * dv] = rh[x];
    }
}

// Epilogue of a chunk stored as bf16 h~ (the output stage's bf16 h; the output
// gate, if any, is applied by a separate pass): the fast and the exact chunk
// forms; the kernel calls it for exact chunks and stores fast ones inline.  Out
// of line, like the fp32 exact epilogue.  Element (t, v) of the chunk is at
// h + t * dv.
template <class C>
__device__ __noinline__ void bf16_epilogue(uint32_t tm, uint32_t lane_base, const float *coef, const float *inv,
                                           bool exact, __nv_bfloat16 *h, size_t dv, int len) {
#pragma unroll 1
    for (int hh = 0; hh < C::kL / 32; ++hh) {
        float rh[32], cf[32];
        tmem_ld32(tm + lane_base + C::TM_H + 32 * hh, rh);
        load32(coef + 32 * hh, cf);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) rh[x] *= cf[x];
        if (exact) {
            float ra[32];
            tmem_ld32(tm + lane_base + C::TM_S + 32 * hh, ra);
            load32(inv + 32 * hh, cf);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) rh[x] = fmaf(ra[x], cf[x], rh[x]);
        }
        const int n = min(32, len - 32 * hh);
        __nv_bfloat16 *hrow = h + (size_t)32 * hh * dv;
#pragma unroll
        for (int x = 0; x < 32; ++x)
            if (x < n) hrow[(size_t)x * dv] = __float2bfloat16_rn(rh[x]);
    }
}

// 2^e for e <= 0 with the hardware's approximate exponential (relative error far
// below the 2^-16 of the bf16 hi/lo operands it feeds; 2^e below 2^-126 flushes to 0).
__device__ __forceinline__ float ex2_approx(float e) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(e));
    return y;
}

// P row of one thread (bf16, K-major 128B-swizzled) and the row sum, L = 64.
__device__ __forceinline__ void store_p_row(const float (&r0)[32], uint8_t *Ps, float *rs, float rsum, int t,
                                            int lane) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pk[i] = pack_bf16x2(r0[8 * ch + 2 * i], r0[8 * ch + 2 * i + 1]);
        const int chunk = 4 * (lane >> 4) + ch;
        *reinterpret_cast<uint4 *>(Ps + sw128_offset(t, chunk)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    rsum += __shfl_xor_sync(0xffffffffu, rsum, 16);
    if (lane < 16) rs[t] = rsum;
}

// Columns [32 j, 32 j + 32) of P row t, L = 128: two 64-column boxes of 128 rows.
__device__ __forceinline__ void store_p_cols128(const float (&r0)[32], uint8_t *Ps, int t, int j) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pk[i] = pack_bf16x2(r0[8 * ch + 2 * i], r0[8 * ch + 2 * i + 1]);
        const int c16 = 4 * j + ch;   // 16-byte chunk of the row, 0..15
        *reinterpret_cast<uint4 *>(Ps + (c16 >> 3) * 16384 + sw128_offset(t, c16 & 7)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

// P of a fast chunk from S: the causal mask, and the row sum of mask(S) w times AH_t.
// L = 64 (M = 64): token row 16 wq + (l & 15) in lane l & 15 of each quarter; lanes
// l and l + 16 take columns [0, 32) and [32, 64) of that row.  L = 128 (M = 128):
// lane = token row; a warp's rows [32 wq, 32 wq + 32) need column groups 0..wq
// only, the groups above the diagonal are stored as zeros without a load.
template <class C>
__device__ __forceinline__ void p_pass(uint32_t s_tmem, const float *g, uint8_t *Ps, float *rs, int wq, int lane) {
    if (C::kL == 64) {
        float r0[32];
        tmem_ld16x2_32(s_tmem, r0);
        tmem_wait_ld();
        const int t = 16 * wq + (lane & 15);
        const int s0 = 32 * (lane >> 4);
        float ww[32];
        load32(g + C::G_W + s0, ww);
        float2 r2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            r0[i] = (s0 + i <= t) ? r0[i] : 0.f;
            r0[i + 1] = (s0 + i + 1 <= t) ? r0[i + 1] : 0.f;
            r2 = __ffma2_rn(make_float2(r0[i], r0[i + 1]), make_float2(ww[i], ww[i + 1]), r2);
        }
        store_p_row(r0, Ps, rs, g[C::G_AH + t] * (r2.x + r2.y), t, lane);
    } else {
        const int t = 32 * wq + lane;
        float2 r2 = make_float2(0.f, 0.f);
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
            float r0[32];
            if (j <= wq) {
                tmem_ld32(s_tmem + 32 * j, r0);
                float ww[32];
                load32(g + C::G_W + 32 * j, ww);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    r0[i] = (32 * j + i <= t) ? r0[i] : 0.f;
                    r0[i + 1] = (32 * j + i + 1 <= t) ? r0[i + 1] : 0.f;
                    r2 = __ffma2_rn(make_float2(r0[i], r0[i + 1]), make_float2(ww[i], ww[i + 1]), r2);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r0[i] = 0.f;
            }
            store_p_cols128(r0, Ps, t, j);
        }
        rs[t] = g[C::G_AH + t] * (r2.x + r2.y);
    }
}

// Exact chunk: P_ts = scale S_ts e^{u_s - mu_t} for s <= t (every exponent <= 0,
// from the float hi/lo pairs) and the plain row sums.  Same layouts as p_pass.
template <class C>
__device__ __noinline__ void exact_p_pass(uint32_t s_tmem, const float *g, uint8_t *Ps, float *rs, float scale,
                                          int wq, int lane) {
    if (C::kL == 64) {
        float r0[32];
        tmem_ld16x2_32(s_tmem, r0);
        tmem_wait_ld();
        const int t = 16 * wq + (lane & 15);
        const int s0 = 32 * (lane >> 4);
        const float mh = g[C::G_MH + t], ml = g[C::G_ML + t];
        float rsum = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float e = (g[C::G_UH + s0 + i] - mh) + (g[C::G_UL + s0 + i] - ml);
            r0[i] = (s0 + i <= t) ? scale * r0[i] * ex2_approx(e) : 0.f;
            rsum += r0[i];
        }
        store_p_row(r0, Ps, rs, rsum, t, lane);
    } else {
        const int t = 32 * wq + lane;
        const float mh = g[C::G_MH + t], ml = g[C::G_ML + t];
        float rsum = 0.f;
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
            float r0[32];
            if (j <= wq) {
                tmem_ld32(s_tmem + 32 * j, r0);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int sidx = 32 * j + i;
                    const float e = (g[C::G_UH + sidx] - mh) + (g[C::G_UL + sidx] - ml);
                    r0[i] = (sidx <= t) ? scale * r0[i] * ex2_approx(e) : 0.f;
                    rsum += r0[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) r0[i] = 0.f;
            }
            store_p_cols128(r0, Ps, t, j);
        }
        rs[t] = rsum;
    }
}

// n.q_t of one chunk in fp32 (thread st of the state group); stores AN_t (n_acc . q_t).
// L = 64: two threads per token (st >> 1), each over half of d_qk, the halves joined
// by a lane shuffle.  L = 128: one thread per token over all of d_qk.
template <class C>
__device__ __forceinline__ void nq_pass(const uint8_t *Qs, const float *nbuf_s, const float *g, float *nq, int st) {
    constexpr int DQK = C::NKB * 64;
    constexpr int NH = C::kL == 64 ? 2 : 1;    // threads per token
    constexpr int CPT = DQK / 8 / NH;          // 16-byte q chunks per thread
    const int trow = NH == 2 ? st >> 1 : st, half = NH == 2 ? st & 1 : 0;
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 1
    for (int g0 = 0; g0 < CPT; g0 += 4) {
        uint4 u[4];
        float4 na[4], nb[4];
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            // the upper-half thread walks its chunks rotated by 4 so that the
            // pair of a token hits distinct banks
            const int ci = half ? (g0 + k4 + 4) % CPT : g0 + k4;
            const int jc = half * (DQK / 2) + 8 * ci;
            u[k4] = *reinterpret_cast<const uint4 *>(Qs + (jc >> 6) * C::BOX + sw128_offset(trow, (jc & 63) >> 3));
            const float *np = nbuf_s + nidx<DQK>(jc);
            na[k4] = *reinterpret_cast<const float4 *>(np);
            nb[k4] = *reinterpret_cast<const float4 *>(np + 4);
        }
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            acc[k4] = __ffma2_rn(bf16x2_to_float2(u[k4].x), make_float2(na[k4].x, na[k4].y), acc[k4]);
            acc[k4] = __ffma2_rn(bf16x2_to_float2(u[k4].y), make_float2(na[k4].z, na[k4].w), acc[k4]);
            acc[k4] = __ffma2_rn(bf16x2_to_float2(u[k4].z), make_float2(nb[k4].x, nb[k4].y), acc[k4]);
            acc[k4] = __ffma2_rn(bf16x2_to_float2(u[k4].w), make_float2(nb[k4].z, nb[k4].w), acc[k4]);
        }
    }
    float v = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
    if (NH == 2) v += __shfl_xor_sync(0xffffffffu, v, 1);
    if (half == 0) nq[trow] = g[C::G_AN + trow] * v;
}

// Blocks [i0, i1) of this thread's C_acc row through split_state_block, with the
// next block's tensor-memory load in flight while a block is split.
template <class C>
__device__ __forceinline__ void split_range(uint32_t tm, uint32_t lane_base, int i0, int i1, bool mv, float rho,
                                            int lo_mode, uint8_t *clo_s, int row, int jlo0) {
    float ra[32], rb[32];
    tmem_ld32(tm + lane_base + C::TM_C + 32 * i0, ra);
#pragma unroll 1
    for (int i = i0; i < i1; i += 2) {
        tmem_wait_ld();
        if (i + 1 < i1) tmem_ld32(tm + lane_base + C::TM_C + 32 * (i + 1), rb);
        split_state_block<C>(ra, tm, lane_base, i, mv, rho, lo_mode, clo_s, row, jlo0 + 32 * (i - i0));
        if (i + 1 < i1) {
            tmem_wait_ld();
            if (i + 2 < i1) tmem_ld32(tm + lane_base + C::TM_C + 32 * (i + 2), ra);
            split_state_block<C>(rb, tm, lane_base, i + 1, mv, rho, lo_mode, clo_s, row, jlo0 + 32 * (i + 1 - i0));
        }
    }
}

// BF16H: h~ is stored as bf16 (the output stage's bf16 h); the plain
// instantiation keeps the fp32 store path alone.
template <int DQK, int L, bool BF16H>
__global__ void __launch_bounds__(kThreads, Cfg<DQK, L>::CTAS)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const TcParams p) {
    using C = Cfg<DQK, L>;
    constexpr int kL = L;
    // The normaliser runs on warp 0 (SMSP 0) and the TMA producer on warp 3 where that
    // measured faster: at L = 128 the P pass of rows 96-127 (four column groups, warp 11)
    // shares SMSP 3 with warp 3; at d_qk = 256 the normaliser is the longest of the
    // single-warp roles.  Otherwise the other way round.
    constexpr bool kSwap = L == 128 || DQK == 256;
    constexpr int kWarpTma = kSwap ? 3 : 0, kWarpNorm = kSwap ? 0 : 3;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::OFF_MISC);
    Shared sh{reinterpret_cast<volatile int *>(sm + C::OFF_MISC + 4), p.status};
    float *gring = reinterpret_cast<float *>(sm + C::OFF_G);
    float *nbuf = reinterpret_cast<float *>(sm + C::OFF_N);
    float *nq_s = reinterpret_cast<float *>(sm + C::OFF_SC);   // [2][L]
    float *rs_s = nq_s + 2 * kL;                               // [2][L]
    float *inv_s = rs_s + 2 * kL;                              // [2][L] 1/den_t
    float *coef_s = inv_s + 2 * kL;                            // [2][L] AH_t/den_t

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int blk = (int)blockIdx.x + p.block0;
    const int slice = blk % p.nslices;
    const int seg = (blk / p.nslices) % p.nseg;
    const int bh = blk / (p.nslices * p.nseg);
    const int v0 = slice * kDvs;
    const int t_base = p.seg_len * seg;                    // first token of this block's segment
    const int T = min(p.T - t_base, p.seg_len);            // tokens in the segment
    const int NC = (T + kL - 1) / kL;
    const bool last_seg = seg == p.nseg - 1;               // the final state is written by the last segment

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[B_K_FULL + i], 1); mbar_init(&bar[B_K_EMPTY + i], 2);   // MMA update + normaliser
            mbar_init(&bar[B_V_FULL + i], 1); mbar_init(&bar[B_V_EMPTY + i], 1);   // MMA update
            mbar_init(&bar[B_Q_FULL + i], 1); mbar_init(&bar[B_Q_EMPTY + i], 2);
            mbar_init(&bar[B_N_READY + i], 1); mbar_init(&bar[B_N_FREE + i], 1);
        }
        for (int i = 0; i < kNG; ++i) { mbar_init(&bar[B_G_FULL + i], 1); mbar_init(&bar[B_G_EMPTY + i], 3); }
        const int ones[] = {B_S_FULL, B_S_EMPTY, B_OPS, B_OPS + 1, B_VT, B_VT + 1, B_VT_EXACT, B_CONV1, B_CLO_FREE,
                            B_H_FULL, B_H_EMPTY, B_UPD_DONE, B_DRAIN};
        mbar_init(&bar[B_CONV0], 2);   // both compute groups split half of the state
        for (int b : ones) mbar_init(&bar[b], 1);
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

    if (warp == kWarpTma) {
        // ===================== TMA producer =====================
        // Order per chunk: k, q, then v.  With one V stage (L = 128) the v copy waits
        // for the previous chunk's update, and k and q of the chunk must not queue
        // behind that wait: the chunk's S needs them first.
        if (lane == 0) {
            int k_issued[2] = {0, 0}, q_issued[2] = {0, 0}, v_issued[2] = {0, 0};
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1, sv = C::VST == 2 ? s : 0;
                if (c + 2 < NC) {   // chunk c+2 into L2 now, so that its stage load hits L2 later
                    for (int b = 0; b < C::NKB; ++b) {
                        tma_prefetch_l2_3d(&tmk, 64 * b, t_base + kL * (c + 2), bh);
                        tma_prefetch_l2_3d(&tmq, 64 * b, t_base + kL * (c + 2), bh);
                    }
                    for (int b = 0; b < 2; ++b)
                        if (v0 + 64 * b < p.dv) tma_prefetch_l2_3d(&tmv, v0 + 64 * b, t_base + kL * (c + 2), bh);
                }
                if (c >= 2 && !wait1(sh, &bar[B_K_EMPTY + s], ((c >> 1) - 1) & 1, kWhereTmaKvEmpty)) break;
                mbar_arrive_expect_tx(&bar[B_K_FULL + s], C::K_BYTES);
                uint8_t *Ks = sm + C::OFF_K + s * C::K_BYTES;
                for (int b = 0; b < C::NKB; ++b)
                    tma_load_3d(Ks + b * C::BOX, &tmk, &bar[B_K_FULL + s], 64 * b, t_base + kL * c, bh);
                ++k_issued[s];
                if (c >= 2 && !wait1(sh, &bar[B_Q_EMPTY + s], ((c >> 1) - 1) & 1, kWhereTmaQEmpty)) break;
                mbar_arrive_expect_tx(&bar[B_Q_FULL + s], C::Q_BYTES);
                uint8_t *Qs = sm + C::OFF_Q + s * C::Q_BYTES;
                for (int b = 0; b < C::NKB; ++b)
                    tma_load_3d(Qs + b * C::BOX, &tmq, &bar[B_Q_FULL + s], 64 * b, t_base + kL * c, bh);
                ++q_issued[s];
                // two V stages: the k stage's release (the same commit after the update of
                // chunk c-2) already covers this stage; one stage: wait for chunk c-1's update
                if (C::VST == 1 && c >= 1 && !wait1(sh, &bar[B_V_EMPTY], (c - 1) & 1, kWhereTmaKvEmpty)) break;
                mbar_arrive_expect_tx(&bar[B_V_FULL + sv], C::V_BYTES);
                uint8_t *Vs = sm + C::OFF_V + sv * C::V_BYTES;
                // a box past d_v (the upper half of a 64-row last slice) is zero-filled by the copy
                for (int b = 0; b < 2; ++b)
                    tma_load_3d(Vs + b * C::BOX, &tmv, &bar[B_V_FULL + sv], v0 + 64 * b, t_base + kL * c, bh);
                ++v_issued[sv];
            }
            // drain: every issued copy must land before shared memory is released
            for (int s = 0; s < 2; ++s) {
                if (k_issued[s]) drain_wait(&bar[B_K_FULL + s], (k_issued[s] - 1) & 1);
                if (q_issued[s]) drain_wait(&bar[B_Q_FULL + s], (q_issued[s] - 1) & 1);
                if (v_issued[s]) drain_wait(&bar[B_V_FULL + s], (v_issued[s] - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        if (lane == 0) {
            const uint32_t idS = make_idesc(kL, kL, kFmtBF16, kFmtBF16, 0, 0);   // M = N = L
            const uint32_t idR = make_idesc(128, kL, kFmtBF16, kFmtBF16, 0, 0);
            const uint32_t idPV = make_idesc(128, kL, kFmtBF16, kFmtBF16, 1, 0);
            const uint32_t idU = make_idesc(128, DQK, kFmtBF16, kFmtBF16, 1, 1);
            const uint32_t p_addr = smem_u32(Ps), clo_addr = smem_u32(sm + C::OFF_CLO);
            bool issued = false, prev_exact = false;
            int nfast = 0, nexact = 0;   // phases of B_VT (one V stage) and B_VT_EXACT consumed
            for (int c = 0; c < NC; ++c) {
                const int s = c & 1, slot = c % kNG, sv = C::VST == 2 ? s : 0;
                const uint32_t vph = C::VST == 2 ? (c >> 1) & 1 : c & 1;   // phase of V_FULL
                const uint32_t q_addr = smem_u32(sm + C::OFF_Q + s * C::Q_BYTES);
                const uint32_t k_addr = smem_u32(sm + C::OFF_K + s * C::K_BYTES);
                const uint32_t v_addr = smem_u32(sm + C::OFF_V + sv * C::V_BYTES);
                if (!wait1(sh, &bar[B_K_FULL + s], (c >> 1) & 1, kWhereMmaKvFull)) break;
                if (!wait1(sh, &bar[B_Q_FULL + s], (c >> 1) & 1, kWhereMmaQFull)) break;
                if (c >= 1 && !wait1(sh, &bar[B_S_EMPTY], (c - 1) & 1, kWhereMmaSEmpty)) break;
                if (c >= 1 && prev_exact && !wait1(sh, &bar[B_H_EMPTY], (c - 1) & 1, kWhereMmaHEmpty)) break;
                tc_fence_after();
                // Descriptors are built once per chunk and advanced by K-step offsets (in
                // 16-byte units; shared addresses stay below 2^18, so the address field of
                // a descriptor never carries).  The issue loops stay rolled: unrolled issue
                // makes the MMAs faster but the compute warps slower, and the layer with them.
                const uint64_t dq = smem_desc_sw128(q_addr, 16, 1024), dk = smem_desc_sw128(k_addr, 16, 1024);
                const uint64_t dv_mn = smem_desc_sw128(v_addr, C::BOX, 1024);
                const uint64_t dk_mn = smem_desc_sw128(k_addr, C::BOX, 1024);
                // S = Q K^T
#pragma unroll 1
                for (int ks = 0; ks < DQK / 16; ++ks)
                    mma_f16_ss(tm + C::TM_S, dq + kstep<C::BOX>(ks), dk + kstep<C::BOX>(ks), idS, ks > 0);
                issued = true;
                tc_commit(&bar[B_S_FULL]);
                if (!wait1(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereMmaGate)) break;
                const bool exact = gring[slot * C::G_FLOATS + C::G_SCAL + kSExact] != 0.f;
                if (!wait1(sh, &bar[B_CONV0], c & 1, kWhereMmaConv)) break;
                // Two V stages: w V(c) is waited here, before the readout, on the barrier of
                // c's parity, which the token group completes once per chunk (exact chunks
                // included, unscaled); it scales V(c+1) during the readout and V(c+2) only
                // after this chunk's update.  One V stage: V(c+1) cannot land before this
                // chunk's update, so the wait moves to the intra part.
                if (C::VST == 2 && !exact && !wait1(sh, &bar[B_VT + (c & 1)], (c >> 1) & 1, kWhereMmaVt)) break;
                if (c >= 1 && !prev_exact && !wait1(sh, &bar[B_H_EMPTY], (c - 1) & 1, kWhereMmaHEmpty)) break;
                tc_fence_after();
                // H = C_hi Q^T + C_lo Q^T
                if (C::BIG) {
                    // C_lo of the lower half first (its shared tile is complete at conv0), then
                    // release the tile, so that the token group refills it with the upper half
                    // while the C_hi MMAs run
                    const uint64_t dclo = smem_desc_sw128(clo_addr, 16, 1024);   // [2 boxes][128 rows][128 B]
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16_ss(tm + C::TM_H, dclo + kstep<16384>(kk), dq + kstep<C::BOX>(kk), idR, kk > 0);
                    tc_commit(&bar[B_CLO_FREE]);
#pragma unroll 1
                    for (int ks = 0; ks < DQK / 16; ++ks)
                        mma_f16_ts(tm + C::TM_H, tm + C::TM_CHI + 8 * ks, dq + kstep<C::BOX>(ks), idR, 1);
                    if (!wait1(sh, &bar[B_CONV1], c & 1, kWhereMmaClo)) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16_ss(tm + C::TM_H, dclo + kstep<16384>(kk), dq + kstep<C::BOX>(8 + kk), idR, 1);
                } else {
#pragma unroll 1
                    for (int ks = 0; ks < DQK / 16; ++ks)
                        mma_f16_ts(tm + C::TM_H, tm + C::TM_CHI + 8 * ks, dq + kstep<C::BOX>(ks), idR, ks > 0);
#pragma unroll 1
                    for (int ks = 0; ks < DQK / 16; ++ks)
                        mma_f16_ts(tm + C::TM_H, tm + C::TM_CLO + 8 * ks, dq + kstep<C::BOX>(ks), idR, 1);
                }
                // intra part: fast chunks accumulate (w V)^T (mask S)^T onto H; exact
                // chunks put V^T P^T into the S columns
                // P(c) is needed only from here: the C Q^T MMAs above overlap its computation
                // (P(c+2) needs S(c+2), issued after this chunk)
                if (!wait1(sh, &bar[B_OPS + (c & 1)], (c >> 1) & 1, kWhereMmaOps)) break;
                if (!wait1(sh, &bar[B_V_FULL + sv], vph, kWhereMmaKvFull)) break;
                if (C::VST == 1 && !exact && !wait1(sh, &bar[B_VT], (nfast++) & 1, kWhereMmaVt)) break;
                tc_fence_after();
                {
                    const uint64_t dp = smem_desc_sw128(p_addr, 16, 1024);
                    const uint32_t dst = exact ? tm + C::TM_S : tm + C::TM_H;
#pragma unroll 1
                    for (int ks = 0; ks < kL / 16; ++ks)   // K = 16 tokens each
                        mma_f16_ss(dst, dv_mn + (uint32_t)(ks * 2048 >> 4), dp + kstep<C::BOX>(ks), idPV,
                                   exact ? (uint32_t)(ks != 0) : 1u);
                }
                tc_commit(&bar[B_H_FULL]);
                tc_commit(&bar[B_Q_EMPTY + s]);
                if (exact) {
                    if (!wait1(sh, &bar[B_VT_EXACT], (nexact++) & 1, kWhereMmaVt)) break;
                    tc_fence_after();
                }
                // C_acc += (w V)^T K
#pragma unroll 1
                for (int ks = 0; ks < kL / 16; ++ks)
                    mma_f16_ss(tm + C::TM_C, dv_mn + (uint32_t)(ks * 2048 >> 4), dk_mn + (uint32_t)(ks * 2048 >> 4),
                               idU, 1);
                tc_commit(&bar[B_UPD_DONE]);
                tc_commit(&bar[B_K_EMPTY + s]);   // with two V stages this also frees V(c)'s stage
                if (C::VST == 1) tc_commit(&bar[B_V_EMPTY]);
                prev_exact = exact;
            }
            if (issued) {   // drain: all issued MMAs complete before tensor memory is freed
                tc_commit(&bar[B_DRAIN]);
                drain_wait(&bar[B_DRAIN], 0);
            }
        }
    } else if (warp == 2) {
        // ===================== gate scan (float64) =====================
        const float *m0 = entry_m(p, bh, seg);
        double m = m0 ? (double)*m0 : 0.0;
        double b = m;
        const float *ig = p.ig + (size_t)bh * p.T + t_base, *fg = p.fg + (size_t)bh * p.T + t_base;
        for (int c = 0; c < NC; ++c) {
            const int slot = c % kNG;
            if (c >= kNG && !waitw(sh, &bar[B_G_EMPTY + slot], ((c / kNG) - 1) & 1, kWhereGateEmpty)) break;
            const int t0 = kL * c, len = min(kL, T - t0);
            constexpr int TPL = kL / 32;   // consecutive tokens per lane
            double iv[TPL], F[TPL], u[TPL], mu[TPL];
            double incl = 0.0;
#pragma unroll
            for (int j = 0; j < TPL; ++j) {
                const int t = TPL * lane + j;
                iv[j] = t < len ? (double)ig[t0 + t] : -INFINITY;
                F[j] = t < len ? (double)fg[t0 + t] : 0.0;   // f~ for now, F after the scan
                incl = j ? incl + F[j] : F[j];
            }
            // inclusive prefix sum of f over the chunk
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            double excl = __shfl_up_sync(0xffffffffu, incl, 1);
            if (lane == 0) excl = 0.0;
#pragma unroll
            for (int j = 0; j < TPL; ++j) {
                F[j] = (j ? F[j - 1] : excl) + F[j];
                u[j] = iv[j] - F[j];
            }
            // running max of u, seeded with m
            double run = u[0];
#pragma unroll
            for (int j = 1; j < TPL; ++j) run = fmax(run, u[j]);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run = fmax(run, y);
            }
            double before = __shfl_up_sync(0xffffffffu, run, 1);
            if (lane == 0) before = -INFINITY;
#pragma unroll
            for (int j = 0; j < TPL; ++j) mu[j] = fmax(j ? mu[j - 1] : fmax(m, before), u[j]);
            const double muL = __shfl_sync(0xffffffffu, mu[TPL - 1], 31);
            const double mu0 = __shfl_sync(0xffffffffu, mu[0], 0);
            const double FL = __shfl_sync(0xffffffffu, F[TPL - 1], 31);
            const bool exact = muL - mu0 > kGrowth;
            const double r = exact ? muL : (muL - b <= kRescale ? b : muL - kRescale);
            float *g = gring + slot * C::G_FLOATS;
            const double aref = exact ? b : r;   // reference of the H coefficient
#pragma unroll
            for (int j = 0; j < TPL; ++j) {
                const int t = TPL * lane + j;
                split_double(u[j] * kLog2e, g[C::G_UH + t], g[C::G_UL + t]);
                split_double(mu[j] * kLog2e, g[C::G_MH + t], g[C::G_ML + t]);
                g[C::G_AH + t] = p.scale * expf((float)(aref - mu[j]));
                g[C::G_AN + t] = p.scale * expf((float)(b - mu[j]));
                g[C::G_W + t] = expf((float)(u[j] - r));
                g[C::G_LOWER + t] = expf((float)(-(F[j] + mu[j])));
            }
            const float rho = expf((float)(b - r));
            const bool rescale = r != b;
            m = FL + muL;
            b = r + FL;
            if (lane == 0) {
                g[C::G_SCAL + kSRho] = rho;
                g[C::G_SCAL + kSRescale] = rescale ? 1.f : 0.f;
                g[C::G_SCAL + kSExact] = exact ? 1.f : 0.f;
                g[C::G_SCAL + kSMEnd] = (float)m;
                g[C::G_SCAL + kSGsc] = expf((float)(b - m));   // final-state gauge factor e^{b-m}
            }
            __syncwarp();
            if (lane == 0 && !(p.fault == 1 && c == 1)) mbar_arrive(&bar[B_G_FULL + slot]);
        }
    } else if (warp == kWarpNorm) {
        // ===================== normaliser n_acc =====================
        constexpr int NPL = DQK / 32;             // columns per lane
        const int j0 = lane * NPL;
        float nacc[NPL];
        const float *n0 = entry_n<DQK>(p, bh, seg);
#pragma unroll
        for (int i = 0; i < NPL; ++i) nacc[i] = n0 ? n0[j0 + i] : 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) nbuf[nidx<DQK>(j0 + i)] = nacc[i];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_N_READY]);
        float gsc = 1.f;
        bool alive = true;
        for (int c = 0; c < NC && alive; ++c) {
            const int slot = c % kNG, s = c & 1;
            alive = waitw(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereNormGate) &&
                    waitw(sh, &bar[B_K_FULL + s], (c >> 1) & 1, kWhereNormKv);
            if (!alive) break;
            const float *g = gring + slot * C::G_FLOATS;
            const float rho = g[C::G_SCAL + kSRho];
            gsc = g[C::G_SCAL + kSGsc];
#pragma unroll
            for (int i = 0; i < NPL; ++i) nacc[i] *= rho;
            const uint8_t *Ks = sm + C::OFF_K + s * C::K_BYTES;
            const uint32_t box = j0 >> 6, chunk = (j0 & 63) >> 3, within = (j0 & 7) * 2;
#pragma unroll 4
            for (int t = 0; t < kL; ++t) {
                const float w = g[C::G_W + t];
                const uint8_t *src = Ks + box * C::BOX + sw128_offset(t, chunk) + within;
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
            for (int i = 0; i < NPL; ++i) nbuf[nb * C::NBUF + nidx<DQK>(j0 + i)] = nacc[i];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar[B_N_READY + nb]);
                mbar_arrive(&bar[B_K_EMPTY + s]);
                mbar_arrive(&bar[B_G_EMPTY + slot]);
            }
        }
        if (alive && slice == 0 && last_seg && p.n1) {
#pragma unroll
            for (int i = 0; i < NPL; ++i) p.n1[(size_t)bh * DQK + j0 + i] = nacc[i] * gsc;
        }
    } else if (warp < 8) {
        // ===================== state group (warps 4-7) =====================
        const int st = tid - 128;            // 0..127: TMEM lane / value row of this block
        const int wq = warp - 4;             // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const int v = v0 + st;
        const bool vok = v < p.dv;       // rows past d_v (a 64-row last slice) are computed on zeros and not stored
        float *hout = p.h + ((size_t)bh * p.T + t_base) * p.dv + v;
        uint8_t *clo_s = sm + C::OFF_CLO;
        {   // initial state: C_acc = C0 (gauge b = m = m0) or zero
            float r[32];
            const float *C0 = entry_C<DQK>(p, bh, seg);
            const float *src = C0 && vok ? C0 + (size_t)v * DQK : nullptr;
#pragma unroll 1
            for (int i = 0; i < DQK / 32; ++i) {
#pragma unroll
                for (int x = 0; x < 32; ++x) r[x] = src ? src[32 * i + x] : 0.f;
                tmem_st32(tm + lane_base + C::TM_C + 32 * i, r);
            }
            tmem_wait_st();
        }
        named_barrier(3, 256);   // C_acc is initialised before either group splits it
        bool alive = true;
        const float *m0 = entry_m(p, bh, seg);
        float m_end = m0 ? *m0 : 0.f, gsc = 1.f;
        for (int c = 0; c < NC; ++c) {
            const int slot = c % kNG, s = c & 1, sb = c & 1;
            const float *g = gring + slot * C::G_FLOATS;
            if (c >= 1) alive = alive && waitw(sh, &bar[B_UPD_DONE], (c - 1) & 1, kWhereStUpd);
            alive = alive && waitw(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereStGate);
            const bool exact = alive && g[C::G_SCAL + kSExact] != 0.f;
            // --- first columns of the state split (C_lo of it: TMEM, or the shared tile)
            if (alive) {
                tc_fence_after();
                const bool mv = !exact && g[C::G_SCAL + kSRescale] != 0.f;
                const float rho = g[C::G_SCAL + kSRho];
                // columns [0, 32 SPLIT_ST); the token group splits the rest
                if (C::SPLIT_ST > 0)
                    split_range<C>(tm, lane_base, 0, C::SPLIT_ST, mv, rho, C::BIG ? 1 : 0, clo_s, st, 0);
                tmem_wait_st();
                if (C::BIG) fence_proxy_async_smem();
                tc_fence_before();
            }
            named_barrier(1, 128);
            if (st == 0 && alive) mbar_arrive(&bar[B_CONV0]);
            // --- n.q_t of this chunk (coefficient AN_t = scale e^{b - mu_t}); the state group
            //     waits for the readout anyway, so it takes this off the token group
            alive = alive && waitw(sh, &bar[B_Q_FULL + s], (c >> 1) & 1, kWhereStQ);
            alive = alive && waitw(sh, &bar[B_N_READY + s], (c >> 1) & 1, kWhereStN);
            if (alive) nq_pass<C>(sm + C::OFF_Q + s * C::Q_BYTES, nbuf + s * C::NBUF, g, nq_s + sb * kL, st);
            named_barrier(1, 128);
            if (st == 0 && alive) {
                mbar_arrive(&bar[B_Q_EMPTY + s]);
                mbar_arrive(&bar[B_N_FREE + s]);
            }
            // --- denominators, once the token group has published the row sums (P(c+2),
            //     the next phase of this barrier, needs S(c+2), which the MMA warp issues
            //     only after the readout of c+1 has waited for this chunk's epilogue)
            alive = alive && waitw(sh, &bar[B_OPS + (c & 1)], (c >> 1) & 1, kWhereStOps);
            if (alive && st < kL) {
                const float inv = 1.f / fmaxf(fabsf(nq_s[sb * kL + st] + rs_s[sb * kL + st]), g[C::G_LOWER + st]);
                inv_s[sb * kL + st] = inv;
                coef_s[sb * kL + st] = g[C::G_AH + st] * inv;
            }
            named_barrier(1, 128);
            alive = alive && waitw(sh, &bar[B_H_FULL], c & 1, kWhereStH);
            if (alive) {
                tc_fence_after();
                if (exact) {   // exact chunk: gauge move to r = mu_L, then V <- w V
                    exact_gauge_move_and_scale_v<C>(tm, lane_base, g[C::G_SCAL + kSRho],
                                                    sm + C::OFF_V + (C::VST == 2 ? s : 0) * C::V_BYTES, g + C::G_W,
                                                    st);
                    fence_proxy_async_smem();
                    tc_fence_before();
                }
            }
            named_barrier(1, 128);   // unconditional: every warp of the group takes every barrier
            if (st == 0 && alive && exact) mbar_arrive(&bar[B_VT_EXACT]);
            // --- epilogue: h~[t][v] = (AH_t H[v][t] (+ intra[v][t])) / den_t
            if (alive) {
                const int len = min(kL, T - kL * c);
                float *hc = hout + (size_t)kL * c * p.dv;
                if (exact && vok) {
                    if (BF16H)
                        bf16_epilogue<C>(tm, lane_base, coef_s + sb * kL, inv_s + sb * kL, true,
                                         static_cast<__nv_bfloat16 *>(static_cast<void *>(p.h)) +
                                             ((size_t)bh * p.T + t_base + kL * c) * p.dv + v,
                                         p.dv, len);
                    else
                        exact_epilogue<C>(tm, lane_base, coef_s + sb * kL, inv_s + sb * kL, hc, p.dv, len);
                } else if (vok && BF16H) {   // fast chunk, h~ stored as bf16
                    __nv_bfloat16 *hb = static_cast<__nv_bfloat16 *>(static_cast<void *>(p.h)) +
                                        ((size_t)bh * p.T + t_base + kL * c) * p.dv + v;
#pragma unroll 1
                    for (int hh = 0; hh < kL / 32; ++hh) {
                        float rh[32], cf[32];
                        tmem_ld32(tm + lane_base + C::TM_H + 32 * hh, rh);
                        load32(coef_s + sb * kL + 32 * hh, cf);
                        tmem_wait_ld();
                        __nv_bfloat16 *hrow = hb + (size_t)32 * hh * p.dv;
                        const int n = min(32, len - 32 * hh);
                        if (n == 32) {
#pragma unroll
                            for (int x = 0; x < 32; ++x) hrow[(size_t)x * p.dv] = __float2bfloat16_rn(rh[x] * cf[x]);
                        } else {   // the last, partial chunk of a sequence
#pragma unroll
                            for (int x = 0; x < 32; ++x)
                                if (x < n) hrow[(size_t)x * p.dv] = __float2bfloat16_rn(rh[x] * cf[x]);
                        }
                    }
                } else if (vok) {
#pragma unroll 1
                    for (int hh = 0; hh < kL / 32; ++hh) {
                        float rh[32], cf[32];
                        tmem_ld32(tm + lane_base + C::TM_H + 32 * hh, rh);
                        load32(coef_s + sb * kL + 32 * hh, cf);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) rh[x] *= cf[x];
                        float *hrow = hc + (size_t)32 * hh * p.dv;
                        const int n = min(32, len - 32 * hh);
                        if (n == 32) {
#pragma unroll
                            for (int x = 0; x < 32; ++x) hrow[(size_t)x * p.dv] = rh[x];
                        } else {   // the last, partial chunk of a sequence
#pragma unroll
                            for (int x = 0; x < 32; ++x)
                                if (x < n) hrow[(size_t)x * p.dv] = rh[x];
                        }
                    }
                }
                m_end = g[C::G_SCAL + kSMEnd];
                gsc = g[C::G_SCAL + kSGsc];
                tc_fence_before();
            }
            named_barrier(1, 128);
            if (st == 0 && alive) {
                mbar_arrive(&bar[B_H_EMPTY]);
                mbar_arrive(&bar[B_G_EMPTY + slot]);
            }
        }
        // final state: C~ = e^{b - m} C_acc
        alive = alive && waitw(sh, &bar[B_UPD_DONE], (NC - 1) & 1, kWhereStFinal);
        if (alive) {
            tc_fence_after();
            if (p.C1 && vok && last_seg) {
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
            if (slice == 0 && st == 0 && last_seg && p.m1) p.m1[bh] = m_end;
        }
        tc_fence_before();
    } else {
        // ===================== token group (warps 8-11) =====================
        const int tk = tid - 256;            // 0..127
        const int wq = warp - 8;             // TMEM lane quarter
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        uint8_t *clo_s = sm + C::OFF_CLO;
        bool alive = true;
        // Chunk c in the loop body below.  With two V stages the body ends with the
        // operand of chunk c+1 that needs neither its split nor the P tile: V(c+1) <-
        // w V(c+1) (fast chunks), which overlaps the readout MMAs of chunk c instead
        // of following them.  With one V stage V(c) lands only after the update of
        // chunk c-1, and is scaled after the P pass of chunk c.
        for (int c = -1; c < NC; ++c) {
          if (c >= 0) {
            const int slot = c % kNG, sb = c & 1;
            const float *g = gring + slot * C::G_FLOATS;
            alive = alive && waitw(sh, &bar[B_G_FULL + slot], (c / kNG) & 1, kWhereTkGate);
            const bool exact = alive && g[C::G_SCAL + kSExact] != 0.f;
            // --- the other columns of the state split (for d_qk = 256, the C_lo of columns
            //     128-255 waits for the shared tile)
            if (c >= 1) alive = alive && waitw(sh, &bar[B_UPD_DONE], (c - 1) & 1, kWhereTkUpd);
            if (alive) {
                tc_fence_after();
                const bool mv = !exact && g[C::G_SCAL + kSRescale] != 0.f;
                const float rho = g[C::G_SCAL + kSRho];
                if (C::BIG) {   // columns 64-127 with their C_lo (shared tile), then C_hi of 128-255
                    split_range<C>(tm, lane_base, 2, 4, mv, rho, 1, clo_s, tk, 64);
                    split_range<C>(tm, lane_base, 4, 8, mv, rho, 2, clo_s, tk, 0);
                } else {
                    split_range<C>(tm, lane_base, C::SPLIT_ST, DQK / 32, mv, rho, 0, clo_s, tk, 0);
                }
                tmem_wait_st();
                tc_fence_before();
            }
            named_barrier(2, 128);
            if (tk == 0 && alive) mbar_arrive(&bar[B_CONV0]);
            // the P tile is free once PV(c-1) completed
            if (c >= 1) alive = alive && waitw(sh, &bar[B_H_FULL], (c - 1) & 1, kWhereTkH);
            // --- P from S
            alive = alive && waitw(sh, &bar[B_S_FULL], c & 1, kWhereTkS);
            if (alive) {
                tc_fence_after();
                if (exact)
                    exact_p_pass<C>(tm + lane_base + C::TM_S, g, Ps, rs_s + sb * kL, p.scale, wq, lane);
                else
                    p_pass<C>(tm + lane_base + C::TM_S, g, Ps, rs_s + sb * kL, wq, lane);
                tc_fence_before();
                fence_proxy_async_smem();
            }
            named_barrier(2, 128);
            if (tk == 0 && alive) {
                mbar_arrive(&bar[B_S_EMPTY]);
                mbar_arrive(&bar[B_OPS + (c & 1)]);
                if (C::VST == 2) mbar_arrive(&bar[B_G_EMPTY + slot]);
            }
            if (C::VST == 1) {   // --- fast chunk: V(c) <- w V(c) in place, before the intra product
                // An exact chunk's V is not touched here, and not waited for either: nothing
                // would hold V(c+1) back until this wait (the MMA warp's update, which frees
                // the stage, waits only for the state group then), so its phase could be
                // overtaken.  A later wait for a fast chunk's V stays exact: V(c') has landed
                // by then up to c'-1 (S(c') follows the update of c'-1) and not beyond c'.
                if (!exact) alive = alive && waitw(sh, &bar[B_V_FULL], c & 1, kWhereTkKv);
                if (alive && !exact) {
                    scale_v_rows<kL>(sm + C::OFF_V, g + C::G_W, tk);
                    fence_proxy_async_smem();
                }
                named_barrier(2, 128);   // unconditional: every warp of the group takes every barrier
                if (tk == 0 && alive) {
                    if (!exact) mbar_arrive(&bar[B_VT]);
                    mbar_arrive(&bar[B_G_EMPTY + slot]);
                }
            }
            if (C::BIG) {   // second half of C_lo once the MMA has consumed the first
                alive = alive && waitw(sh, &bar[B_CLO_FREE], c & 1, kWhereTkClo);
                if (alive) {
                    tc_fence_after();
                    split_range<C>(tm, lane_base, DQK / 64, DQK / 32, false, 1.f, 3, clo_s, tk, 0);
                    fence_proxy_async_smem();
                    tc_fence_before();
                }
                named_barrier(2, 128);
                if (tk == 0 && alive) mbar_arrive(&bar[B_CONV1]);
            }
          }
            if (C::VST == 2 && c + 1 < NC) {
                const int j = c + 1, sj = j & 1, slot_j = j % kNG;
                const float *gj = gring + slot_j * C::G_FLOATS;
                // the MMA warp waits for w V(c) right after the split of chunk c; V(c+1) is
                // scaled after that split (its barrier is the other one of the pair)
                if (c >= 0) alive = alive && waitw(sh, &bar[B_CONV0], c & 1, kWhereTkConv);
                alive = alive && waitw(sh, &bar[B_G_FULL + slot_j], (j / kNG) & 1, kWhereTkGate);
                const bool ex = alive && gj[C::G_SCAL + kSExact] != 0.f;
                // --- fast chunk: V <- w V in place, before the intra product
                alive = alive && waitw(sh, &bar[B_V_FULL + sj], (j >> 1) & 1, kWhereTkKv);
                if (alive && !ex) {
                    scale_v_rows<kL>(sm + C::OFF_V + sj * C::V_BYTES, gj + C::G_W, tk);
                    fence_proxy_async_smem();
                }
                named_barrier(2, 128);   // unconditional: every warp of the group takes every barrier
                if (tk == 0 && alive) mbar_arrive(&bar[B_VT + (j & 1)]);
            }
            if (c == -1) named_barrier(3, 256);   // C_acc is initialised before either group splits it
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tm, C::TMEM_COLS);
    }
}

// Blocks of the first launch when a grid of nblk one-per-SM blocks ends in a partial
// wave: every block before that wave, rounded down to whole sequences (per_seq blocks
// each, so that their h~ is one contiguous range).  0: no split (one wave or less,
// whole waves, not one sequence before the last wave, or more than four blocks' h~
// for each SM the last wave leaves idle: their gate would outlast that wave).
int overlap_split(int nblk, int per_seq) {
    const int nsm = sm_count();
    if (nsm <= 0 || nblk <= nsm || nblk % nsm == 0) return 0;
    const int first = (nblk - nblk % nsm) / per_seq * per_seq;
    const int idle = nsm - (nblk - first);
    return first >= per_seq && idle >= 1 && first <= 4 * idle ? first : 0;
}

// The second stream of a split launch and its two events, one set per device, made on
// first use and kept; the mutex keeps the record / wait sequence of one call from
// interleaving with another's.
struct OverlapStreams {
    std::mutex mu;
    cudaStream_t side = nullptr;
    cudaEvent_t first = nullptr, gated = nullptr;
    bool ok = false;
};
OverlapStreams *overlap_streams() {
    constexpr int kMaxDev = 64;
    static OverlapStreams sets[kMaxDev];
    static std::once_flag once[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    OverlapStreams &o = sets[dev];
    std::call_once(once[dev], [&o] {
        o.ok = cudaStreamCreateWithFlags(&o.side, cudaStreamNonBlocking) == cudaSuccess &&
               cudaEventCreateWithFlags(&o.first, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&o.gated, cudaEventDisableTiming) == cudaSuccess;
    });
    return o.ok ? &o : nullptr;
}

template <int DQK, int L>
cudaError_t launch_dqk(const FwdArgs &a, cudaStream_t s, int fault) {
    using C = Cfg<DQK, L>;
    const int BH = a.B * a.H;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_3d_bf16(&tq, a.q, DQK, a.T, BH, 64, L) || !make_tmap_3d_bf16(&tk, a.k, DQK, a.T, BH, 64, L) ||
        !make_tmap_3d_bf16(&tv, a.v, a.dv, a.T, BH, 64, L))
        return cudaErrorInvalidValue;
    TcParams p;
    p.T = a.T; p.dv = a.dv; p.nslices = (a.dv + kDvs - 1) / kDvs; p.scale = a.scale;
    p.ig = a.ig; p.fg = a.fg; p.C0 = a.C0; p.n0 = a.n0; p.m0 = a.m0;
    p.h = a.h; p.C1 = a.C1; p.n1 = a.n1; p.m1 = a.m1; p.status = a.status; p.fault = fault;
    p.BH = BH; p.nseg = 1; p.seg_len = a.T;
    p.segC = p.segN = p.segM = nullptr;
    cudaError_t e;
    if (a.seg_ws) {   // entry states of the segments first, on the same stream
        const SegPlan sp = segment_plan(a);
        if (sp.nseg > 1) {
            if ((e = launch_segment_entry_states(a, sp, s)) != cudaSuccess) return e;
            const char *ws = static_cast<const char *>(a.seg_ws);
            p.nseg = sp.nseg; p.seg_len = sp.seg_chunks * kSegChunk;   // a multiple of L (segment_plan)
            p.segC = reinterpret_cast<const float *>(ws + sp.off_C);
            p.segN = reinterpret_cast<const float *>(ws + sp.off_N);
            p.segM = reinterpret_cast<const float *>(ws + sp.off_M);
        }
    }
    auto kern = a.out.h_bf16 ? chunk_tc_kernel<DQK, L, true> : chunk_tc_kernel<DQK, L, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e == cudaSuccess && C::CTAS > 1)   // room for both blocks' shared memory
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int nblk = BH * p.nseg * p.nslices, per_seq = p.nseg * p.nslices;
    const int split = a.out.o && C::CTAS == 1 ? overlap_split(nblk, per_seq) : 0;
    OverlapStreams *ov = split ? overlap_streams() : nullptr;
    p.block0 = 0;
    if (!ov) {
        kern<<<nblk, kThreads, C::SMEM, s>>>(tq, tk, tv, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // the output gate as one streaming pass over h~ in place
        if (a.out.o) return launch_output_gate(a.out, a.h, (size_t)BH * a.T * a.dv, s);
        return cudaSuccess;
    }
    // The output gate of the blocks before the last, partial wave runs on the SMs that
    // wave leaves idle: blocks [0, split), then the rest, on the caller's stream; a
    // second stream waits for the first blocks and gates their h~ with one block on
    // each idle SM, blocks that no block of the rest can share (whichever of the two
    // launches is placed first, the rest find their SMs); the caller's stream waits
    // for that gate and gates the rest's h~.
    std::lock_guard<std::mutex> lock(ov->mu);
    const size_t nA = (size_t)(split / per_seq) * a.T * a.dv, nAll = (size_t)BH * a.T * a.dv;
    kern<<<split, kThreads, C::SMEM, s>>>(tq, tk, tv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ov->first, s)) != cudaSuccess) return e;
    p.block0 = split;
    kern<<<nblk - split, kThreads, C::SMEM, s>>>(tq, tk, tv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(ov->side, ov->first, 0)) != cudaSuccess) return e;
    if ((e = launch_output_gate_on_sms(a.out, a.h, nA, ov->side, sm_count() - (nblk - split))) != cudaSuccess)
        return e;
    if ((e = cudaEventRecord(ov->gated, ov->side)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(s, ov->gated, 0)) != cudaSuccess) return e;
    const size_t hb = a.out.h_bf16 ? 2 : 4, ob = a.out.o_bf16 ? 2 : 4;
    OutStage rest = a.out;
    rest.o = static_cast<const char *>(a.out.o) + nA * ob;
    return launch_output_gate(rest, reinterpret_cast<char *>(a.h) + nA * hb, nAll - nA, s);
}

}  // namespace

bool chunkwise_tc_shape_ok(const FwdArgs &a) {
    if (a.dtype != XLSTM_BF16 || a.T < 1) return false;
    if (a.dv % 64 != 0) return false;   // whole 64-row boxes; a last slice may hold 64 rows of 128
    if (a.dqk != 64 && a.dqk != 128 && a.dqk != 256) return false;
    // tensor memory holds the state, its readout copy and one chunk's S and H:
    // L = 128 leaves no room for them at d_qk = 256
    return a.chunk == 64 || (a.chunk == 128 && a.dqk <= 128);
}

bool chunkwise_tc_supported(const FwdArgs &a) { return chunkwise_tc_shape_ok(a) && encode_tiled_fn() != nullptr; }

cudaError_t launch_chunkwise_tc(const FwdArgs &a, cudaStream_t s) {
    const int fault = g_fault_next;
    g_fault_next = 0;
    if (a.chunk == 128) {
        switch (a.dqk) {
            case 64: return launch_dqk<64, 128>(a, s, fault);
            case 128: return launch_dqk<128, 128>(a, s, fault);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (a.dqk) {
        case 64: return launch_dqk<64, 64>(a, s, fault);
        case 128: return launch_dqk<128, 64>(a, s, fault);
        case 256: return launch_dqk<256, 64>(a, s, fault);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace xlstm
