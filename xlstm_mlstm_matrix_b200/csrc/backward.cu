// Backward pass of the mLSTM forward (vector-Jacobian product), chunkwise.
//
// What is differentiated: the readout of the xLSTM page's "mLSTM (matrix LSTM)"
// section, eq. 3 with the true states of eq. 1-2 (h_t = C_t q_t / max(|n_t^T q_t|,
// 1), f_t = e^{f~_t}, i_t = e^{i~_t}); the stabilizer of the "sLSTM" section only
// stores those states, so the gauge m is a constant of the derivative.  Every
// quantity is the true one rescaled by e^{m_t}, so no factor exceeds 1.
//
// Per (batch, head) the sequence is cut into chunks of L = 64 tokens:
//  1. states (CUDA cores, per value slice, sequential in t): the stored state at
//     the entry of every chunk, and per token the stabilizer m_t, s~_t = n~_t . q_t
//     and the slice's share of dh_t . h~_t;
//  2. adjoints (CUDA cores, per value slice, sequential backwards in t): the
//     adjoint of the state at the exit of every chunk,
//        dC~ <- f'_t (dC~ + (dh_t / den~_t) q_t^T),   dn~ <- f'_t (dn~ + ds~_t q_t),
//     with ds~_t = -(dh_t . h~_t / den~_t) sign(s~_t) where |s~_t| > e^{-m_t}, else 0;
//     it ends as the gradient of the initial state;
//  3. chunk gradients (CUDA cores, every (b, h, chunk) at once): with F_t the
//     chunk-local cumulative f~, u_s = i~_s - F_s, entry gauge m_0,
//        W_ts = e^{u_s + F_t - m_t} (s <= t),  a_t = e^{F_t + m_0 - m_t},
//        z_t = e^{u_t + F_L - m_L},  DN_t = dh_t / den~_t,
//        M_ts = W_ts (DN_t . v_s + ds~_t),  E_ts = W_ts (q_t . k_s),
//     dq = scale (diag(a) (DN C~_0 + ds~ n~_0^T) + M K),
//     dk = M^T Q + diag(z) (V dC~_ex + 1 dn~_ex^T),   di~_t = k_t . dk_t,
//     dv = E^T DN + diag(z) K dC~_ex^T,
//     df~_r = sum of the log-weight gradients of every pair the decay from r
//             belongs to: intra pairs (s < r <= t, M_ts (q_t . k_s)), entry pairs
//             (t >= r), exit pairs (s < r) and the entry-to-exit pair.
// The states kernel also forms each value slice's share of dh_t . h~_t from the
// state it holds (fp32, so the forward's own rounding of h~ does not enter); a
// small kernel sums the shares, which every value slice of steps 2 and 3 needs.
#include <math.h>

#include "common.cuh"

namespace xlstm {
namespace {

constexpr int kL = 64;
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRpw = 4;                 // rows per warp (sequential kernels)
constexpr int kRows = kWarps * kRpw;    // value rows per block
constexpr int kTok = 16;                // tokens staged per barrier

struct BwdLayout {
    size_t off_C, off_dC, off_n, off_dn, off_m0, off_mt, off_st, off_gt, off_gp, off_dm, bytes;
};

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

BwdLayout bwd_layout(int BH, int T, int dqk, int dv) {
    BwdLayout l;
    const size_t NC = (size_t)(T + kL - 1) / kL, slices = (size_t)(dv + kRows - 1) / kRows;
    l.off_C = 256;
    l.off_dC = al256(l.off_C + NC * BH * (size_t)dv * dqk * 4);
    l.off_n = al256(l.off_dC + NC * BH * (size_t)dv * dqk * 4);
    l.off_dn = al256(l.off_n + NC * BH * (size_t)dqk * 4);
    l.off_m0 = al256(l.off_dn + NC * BH * (size_t)dqk * 4);
    l.off_mt = al256(l.off_m0 + NC * BH * 8);
    l.off_st = al256(l.off_mt + (size_t)BH * T * 8);
    l.off_gt = al256(l.off_st + (size_t)BH * T * 4);
    l.off_gp = al256(l.off_gt + (size_t)BH * T * 4);
    l.off_dm = al256(l.off_gp + slices * BH * (size_t)T * 4);
    l.bytes = al256(l.off_dm + slices * BH * 4);
    return l;
}

struct BwdP {
    int B, H, T, dqk, dv, slices, NC;
    float scale;
    const void *q, *k, *v;
    const float *ig, *fg, *C0, *n0, *m0, *dh, *dCT, *dnT;
    float *dq, *dk, *dv_, *di, *df, *dC0, *dn0, *dm0;
    float *wC, *wdC, *wn, *wdn, *wst, *wgt, *wgp, *wdm;
    double *wm0, *wmt;
};

// ---- 1. states at chunk entries, m_t and s~_t per token -----------------------------
// Layout as the recurrent forward: warp w holds rows [w*kRpw, (w+1)*kRpw) of the
// block's slice in registers, lane l columns l, l+32, ...; each warp keeps n~.
template <typename Tin, int MAXC>
__global__ void __launch_bounds__(kThreads) bwd_states_kernel(BwdP p) {
    extern __shared__ float sm[];
    const int dqk = p.dqk, dv = p.dv;
    float *sq = sm;                          // [kTok][dqk] scaled q
    float *sk = sq + kTok * dqk;             // [kTok][dqk]
    float *sv = sk + kTok * dqk;             // [kTok][kRows]
    float *sdh = sv + kTok * kRows;          // [kTok][kRows] dh of the block's rows
    float *sg = sdh + kTok * kRows;          // [kTok][2] (i~, f~)
    float *sgw = sg + 2 * kTok;              // [kTok][kWarps] per-warp shares of dh . h~
    // per-lane parts of n~ . q and of the warp's share of dh . (C~ q), [kWarps][kTok][33]: summed
    // once per staged block of tokens (they do not feed the recurrence)
    float *rs = sgw + kTok * kWarps;
    float *rn = rs + kWarps * kTok * 33;
    double *smt = reinterpret_cast<double *>(rn + kWarps * kTok * 33);   // [kTok] m_t
    float *sfi = reinterpret_cast<float *>(smt + kTok);                 // [kTok][2] (f'_t, i'_t)
    const int bh = blockIdx.x / p.slices, slice = blockIdx.x % p.slices, row0 = slice * kRows;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Tin *q = static_cast<const Tin *>(p.q) + (size_t)bh * p.T * dqk;
    const Tin *k = static_cast<const Tin *>(p.k) + (size_t)bh * p.T * dqk;
    const Tin *v = static_cast<const Tin *>(p.v) + (size_t)bh * p.T * dv;
    const float *dh = p.dh + (size_t)bh * p.T * dv;
    const float *ig = p.ig + (size_t)bh * p.T, *fg = p.fg + (size_t)bh * p.T;
    float C[kRpw][MAXC], n[MAXC];
    double m = p.m0 ? (double)p.m0[bh] : 0.0;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int j = lane + 32 * c;
        n[c] = (p.n0 && j < dqk) ? p.n0[(size_t)bh * dqk + j] : 0.f;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) {
            const int row = row0 + warp * kRpw + r;
            C[r][c] = (p.C0 && j < dqk && row < dv) ? p.C0[((size_t)bh * dv + row) * dqk + j] : 0.f;
        }
    }
    for (int t0 = 0; t0 < p.T; t0 += kTok) {
        const int nt = min(kTok, p.T - t0);
        __syncthreads();
        for (int e = tid; e < nt * dqk; e += kThreads) {
            sq[e] = p.scale * to_f32(q[(size_t)t0 * dqk + e]);
            sk[e] = to_f32(k[(size_t)t0 * dqk + e]);
        }
        for (int e = tid; e < nt * kRows; e += kThreads) {
            const int tt = e / kRows, r = e % kRows;
            const bool ok = row0 + r < dv;
            sv[e] = ok ? to_f32(v[(size_t)(t0 + tt) * dv + row0 + r]) : 0.f;
            sdh[e] = ok ? dh[(size_t)(t0 + tt) * dv + row0 + r] : 0.f;
        }
        if (tid < nt) {
            sg[2 * tid] = ig[t0 + tid];
            sg[2 * tid + 1] = fg[t0 + tid];
        }
        __syncthreads();
        // the staged tokens' gates once per block: the stabilizer chain (float64) on one
        // thread, f' and i' on one thread per token
        if (tid == 0) {
            double mm = m;
            for (int tt = 0; tt < nt; ++tt) {
                mm = fmax((double)sg[2 * tt + 1] + mm, (double)sg[2 * tt]);
                smt[tt] = mm;
            }
        }
        __syncthreads();
        if (tid < nt) {
            const double mp = tid ? smt[tid - 1] : m, it = sg[2 * tid], ft = sg[2 * tid + 1], mn = smt[tid];
            sfi[2 * tid] = expf((float)(ft + mp - mn));
            sfi[2 * tid + 1] = expf((float)(it - mn));
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const int t = t0 + tt;
            if (t % kL == 0) {   // the stored state entering chunk t / L
                const size_t ci = (size_t)(t / kL) * (p.B * p.H) + bh;
#pragma unroll
                for (int c = 0; c < MAXC; ++c) {
                    const int j = lane + 32 * c;
                    if (j >= dqk) continue;
#pragma unroll
                    for (int r = 0; r < kRpw; ++r) {
                        const int row = row0 + warp * kRpw + r;
                        if (row < dv) p.wC[(ci * dv + row) * dqk + j] = C[r][c];
                    }
                    if (slice == 0 && warp == 0) p.wn[ci * dqk + j] = n[c];
                }
                if (slice == 0 && tid == 0) p.wm0[ci] = m;
            }
            const double m_new = smt[tt];
            const float fp = sfi[2 * tt], ip = sfi[2 * tt + 1];
            const float *qt = sq + tt * dqk, *kt = sk + tt * dqk;
            float s = 0.f, num = 0.f;   // n~ . q and this lane's share of sum_r dh_r (C~ q)_r
#pragma unroll
            for (int c = 0; c < MAXC; ++c) {
                const int j = lane + 32 * c;
                const float kv = (j < dqk) ? kt[j] : 0.f, qv = (j < dqk) ? qt[j] : 0.f;
                n[c] = fmaf(fp, n[c], ip * kv);
                s = fmaf(n[c], qv, s);
                float cq = 0.f;
#pragma unroll
                for (int r = 0; r < kRpw; ++r) {
                    C[r][c] = fmaf(fp, C[r][c], ip * sv[tt * kRows + warp * kRpw + r] * kv);
                    cq = fmaf(sdh[tt * kRows + warp * kRpw + r], C[r][c], cq);
                }
                num = fmaf(cq, qv, num);
            }
            rs[(warp * kTok + tt) * 33 + lane] = s;
            rn[(warp * kTok + tt) * 33 + lane] = num;
            m = m_new;
        }
        __syncthreads();
        if (lane < nt) {   // token tt = lane: the lane sums, the readout's denominator, this warp's share
            const int tt = lane, t = t0 + tt;
            // pairwise, in the order of a butterfly reduction over the 32 lanes
            float a[32], b[32];
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                a[l] = rs[(warp * kTok + tt) * 33 + l];
                b[l] = rn[(warp * kTok + tt) * 33 + l];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int l = 0; l < o; ++l) {
                    a[l] += a[l + o];
                    b[l] += b[l + o];
                }
            const float s = a[0], num = b[0];
            const double mt = smt[tt];
            const float lower = expf((float)(-mt));
            const float den = fabsf(s) > lower ? fabsf(s) : lower;
            sgw[tt * kWarps + warp] = num / den;
            if (slice == 0 && warp == 0) {
                p.wmt[(size_t)bh * p.T + t] = mt;
                p.wst[(size_t)bh * p.T + t] = s;
            }
        }
        __syncthreads();
        if (tid < nt) {   // this slice's share of dh_t . h~_t
            float g = 0.f;
            for (int w = 0; w < kWarps; ++w) g += sgw[tid * kWarps + w];
            p.wgp[((size_t)slice * (p.B * p.H) + bh) * p.T + t0 + tid] = g;
        }
    }
}

// ---- dh . h~ per token: the value slices' shares summed in order ---------------------------
__global__ void __launch_bounds__(kThreads) bwd_gsum_kernel(const float *gp, float *g, size_t n, int slices) {
    const size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= n) return;
    float s = 0.f;
    for (int sl = 0; sl < slices; ++sl) s += gp[(size_t)sl * n + i];
    g[i] = s;
}

// The readout's derivative factors of token t: den~_t and ds~_t.
__device__ __forceinline__ void readout_factors(float s, double m, float g, float &den, float &ds) {
    const float lower = expf((float)(-m));
    const bool clamp = !(fabsf(s) > lower);
    den = clamp ? lower : fabsf(s);
    ds = clamp ? 0.f : -(g / den) * (s > 0.f ? 1.f : -1.f);
}

// ---- 2. adjoints at chunk exits, backwards in t -----------------------------------------
// Three blocks per SM up to d_qk = 256 (the register cap leaves those forms unspilled).
template <typename Tin, int MAXC>
__global__ void __launch_bounds__(kThreads, MAXC <= 8 ? 3 : 1) bwd_adjoint_kernel(BwdP p) {
    extern __shared__ float sm[];
    const int dqk = p.dqk, dv = p.dv;
    float *sq = sm;                          // [kTok][dqk] scaled q
    float *sdh = sq + kTok * dqk;            // [kTok][kRows] dh_t / den~_t
    float *ssc = sdh + kTok * kRows;         // [kTok][3] (ds~_t, f'_t, den~_t)
    const int bh = blockIdx.x / p.slices, slice = blockIdx.x % p.slices, row0 = slice * kRows;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Tin *q = static_cast<const Tin *>(p.q) + (size_t)bh * p.T * dqk;
    const float *fg = p.fg + (size_t)bh * p.T;
    const double *mt = p.wmt + (size_t)bh * p.T;
    const float *st = p.wst + (size_t)bh * p.T, *gt = p.wgt + (size_t)bh * p.T;
    const float *dh = p.dh + (size_t)bh * p.T * dv;
    float D[kRpw][MAXC], dn[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int j = lane + 32 * c;
        dn[c] = (p.dnT && j < dqk) ? p.dnT[(size_t)bh * dqk + j] : 0.f;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) {
            const int row = row0 + warp * kRpw + r;
            D[r][c] = (p.dCT && j < dqk && row < dv) ? p.dCT[((size_t)bh * dv + row) * dqk + j] : 0.f;
        }
    }
    const double m_init = p.m0 ? (double)p.m0[bh] : 0.0;
    const int nblk = (p.T + kTok - 1) / kTok;
    for (int b = nblk - 1; b >= 0; --b) {
        const int t0 = b * kTok, nt = min(kTok, p.T - t0);
        __syncthreads();
        for (int e = tid; e < nt * dqk; e += kThreads) sq[e] = p.scale * to_f32(q[(size_t)t0 * dqk + e]);
        if (tid < nt) {
            const int t = t0 + tid;
            float den, ds;
            readout_factors(st[t], mt[t], gt[t], den, ds);
            const double mp = t > 0 ? mt[t - 1] : m_init;
            ssc[3 * tid] = ds;
            ssc[3 * tid + 1] = expf((float)((double)fg[t] + mp - mt[t]));
            ssc[3 * tid + 2] = den;
        }
        __syncthreads();
        // dh / den~ of the block's rows
        for (int e = tid; e < nt * kRows; e += kThreads) {
            const int tt = e / kRows, r = e % kRows, t = t0 + tt;
            sdh[e] = (row0 + r < dv) ? dh[(size_t)t * dv + row0 + r] / ssc[3 * tt + 2] : 0.f;
        }
        __syncthreads();
        for (int tt = nt - 1; tt >= 0; --tt) {
            const int t = t0 + tt;
            if (t == p.T - 1 || (t + 1) % kL == 0) {   // the adjoint at the exit of chunk t / L
                const size_t ci = (size_t)(t / kL) * (p.B * p.H) + bh;
#pragma unroll
                for (int c = 0; c < MAXC; ++c) {
                    const int j = lane + 32 * c;
                    if (j >= dqk) continue;
#pragma unroll
                    for (int r = 0; r < kRpw; ++r) {
                        const int row = row0 + warp * kRpw + r;
                        if (row < dv) p.wdC[(ci * dv + row) * dqk + j] = D[r][c];
                    }
                    if (slice == 0 && warp == 0) p.wdn[ci * dqk + j] = dn[c];
                }
            }
            const float ds = ssc[3 * tt], fp = ssc[3 * tt + 1];
            const float *qt = sq + tt * dqk;
#pragma unroll
            for (int c = 0; c < MAXC; ++c) {
                const int j = lane + 32 * c;
                const float qv = (j < dqk) ? qt[j] : 0.f;
                dn[c] = fp * fmaf(ds, qv, dn[c]);
#pragma unroll
                for (int r = 0; r < kRpw; ++r) D[r][c] = fp * fmaf(sdh[tt * kRows + warp * kRpw + r], qv, D[r][c]);
            }
        }
    }
    // the gradient of the initial state, and this slice's share of dm0
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int j = lane + 32 * c;
        if (j >= dqk) continue;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) {
            const int row = row0 + warp * kRpw + r;
            if (row >= dv) continue;
            const size_t e = ((size_t)bh * dv + row) * dqk + j;
            if (p.dC0) p.dC0[e] = D[r][c];
            if (p.C0) part = fmaf(D[r][c], p.C0[e], part);
        }
        if (slice == 0 && warp == 0) {
            if (p.dn0) p.dn0[(size_t)bh * dqk + j] = dn[c];
            if (p.n0) part = fmaf(dn[c], p.n0[(size_t)bh * dqk + j], part);
        }
    }
    part = warp_sum(part);
    __shared__ float red[kWarps];
    if (lane == 0) red[warp] = part;
    __syncthreads();
    if (tid == 0) {
        float s = 0.f;
        for (int w = 0; w < kWarps; ++w) s += red[w];
        p.wdm[(size_t)slice * (p.B * p.H) + bh] = s;
    }
}

__global__ void bwd_dm0_kernel(const float *part, float *dm0, int BH, int slices) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    float s = 0.f;
    for (int i = 0; i < slices; ++i) s += part[(size_t)i * BH + bh];
    dm0[bh] = s;
}

// ---- 3. gradients of every chunk, all chunks at once ------------------------------------
constexpr int kLd = kL + 1;   // padded row of the L x L matrices
constexpr int kAs = 68;       // row of a 32 x 64 operand tile: 16-byte aligned, rows 4 banks apart

// The block's 64 x 64 product tile, 4 x 4 outputs per thread (rows 4 ty + i, columns
// 4 tx + j; ty = tid / 16, tx = tid % 16): acc += A^T B over the 32 rows k of the
// K-major tiles As[k][row] and Bs[k][col].  Two 16-byte shared loads per 16 FMAs.
__device__ __forceinline__ void tile_fma(const float *As, const float *Bs, float (&acc)[4][4], int ty, int tx) {
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(As + k * kAs + 4 * ty);
        const float4 b = *reinterpret_cast<const float4 *>(Bs + k * kAs + 4 * tx);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}
__device__ __forceinline__ void zero48(float (&acc)[4][8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
}
__device__ __forceinline__ void zero44(float (&acc)[4][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
}
// One thread's 8 elements (e = tid + 256 i) of a 32 x 64 operand tile, fetched into
// registers so that the next tile's global loads overlap the current tile's FMAs.
//   TOKT: element (kk = e % 32, t = e / 32) = get(t, k0 + kk)   (token-major source, transposed)
//   rows: element (kk = e / 64, c = e % 64) = get(k0 + kk, c0 + c)
// Zero outside t < L, k0 + kk < nk, c0 + c < nc.
template <bool TOKT, class G>
__device__ __forceinline__ void fetch8(G get, int k0, int nk, int c0, int nc, int L, float (&r)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = threadIdx.x + kThreads * i;
        if (TOKT) {
            const int t = e >> 5, kk = e & 31;
            r[i] = (t < L && k0 + kk < nk) ? get(t, k0 + kk) : 0.f;
        } else {
            const int kk = e >> 6, c = e & 63;
            r[i] = (k0 + kk < nk && c0 + c < nc) ? get(k0 + kk, c0 + c) : 0.f;
        }
    }
}
template <bool TOKT>
__device__ __forceinline__ void put8(float *dst, const float (&r)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = threadIdx.x + kThreads * i;
        dst[TOKT ? (e & 31) * kAs + (e >> 5) : (e >> 6) * kAs + (e & 63)] = r[i];
    }
}

// 64 x 128 product tile, 4 x 8 outputs per thread: rows 4 ty + i, columns 4 tx + j and
// 64 + 4 tx + j (two groups of four, so each 16-byte load of a quarter-warp is contiguous).
// B is a K-major 32 x 128 tile with rows kBs floats apart.
constexpr int kBs = 132;
__device__ __forceinline__ void tile_fma_w(const float *As, const float *Bs, float (&acc)[4][8], int ty, int tx) {
#pragma unroll 4
    for (int k = 0; k < 32; ++k) {
        const float4 a = *reinterpret_cast<const float4 *>(As + k * kAs + 4 * ty);
        const float4 b0 = *reinterpret_cast<const float4 *>(Bs + k * kBs + 4 * tx);
        const float4 b1 = *reinterpret_cast<const float4 *>(Bs + k * kBs + 64 + 4 * tx);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
}
// One thread's 16 elements (e = tid + 256 i) of a 32 x 128 row-major operand tile:
// element (kk = e / 128, c = e % 128) = get(k0 + kk, c0 + c), zero outside k0 + kk < nk, c0 + c < nc.
template <class G>
__device__ __forceinline__ void fetch16(G get, int k0, int nk, int c0, int nc, float (&r)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kThreads * i, kk = e >> 7, c = e & 127;
        r[i] = (k0 + kk < nk && c0 + c < nc) ? get(k0 + kk, c0 + c) : 0.f;
    }
}
__device__ __forceinline__ void put16(float *dst, const float (&r)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kThreads * i;
        dst[(e >> 7) * kBs + (e & 127)] = r[i];
    }
}

// Sum over the 16 threads (tx) that share a row group: lanes l and l ^ 1, 2, 4, 8.
__device__ __forceinline__ float sum16(float x) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <typename Tin>
__device__ __forceinline__ float ld_in(const Tin *p, size_t i) { return to_f32(p[i]); }

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 2) bwd_chunk_kernel(BwdP p) {
    extern __shared__ float sm[];
    float *Mm = sm;                     // [kL][kLd] M_ts
    float *Em = Mm + kL * kLd;          // [kL][kLd] E_ts
    float *Gm = Em + kL * kLd;          // [kL][kLd] S, then G_ts
    float *As = Gm + kL * kLd;          // [32][kAs] K-major operand tiles of the products
    float *Bs = As + 32 * kAs;          // [32][kBs] (64-wide tiles use the first kAs-strided rows)
    float *sa = Bs + 32 * kBs, *sz = sa + kL, *sden = sz + kL, *sds = sden + kL;
    float *sG0 = sds + kL, *sGx = sG0 + kL, *sdi = sGx + kL, *sdfi = sdi + kL, *red = sdfi + kL;
    double *su = reinterpret_cast<double *>(red + 2 * kWarps);   // [kL] u_s
    double *sFm = su + kL;                                       // [kL] F_t - m_t

    const int dqk = p.dqk, dv = p.dv, BH = p.B * p.H;
    const int c = blockIdx.x % p.NC, bh = blockIdx.x / p.NC;
    const int t0 = c * kL, L = min(kL, p.T - t0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t ci = (size_t)c * BH + bh;
    const Tin *q = static_cast<const Tin *>(p.q) + ((size_t)bh * p.T + t0) * dqk;
    const Tin *k = static_cast<const Tin *>(p.k) + ((size_t)bh * p.T + t0) * dqk;
    const Tin *v = static_cast<const Tin *>(p.v) + ((size_t)bh * p.T + t0) * dv;
    const float *dh = p.dh + ((size_t)bh * p.T + t0) * dv;
    const float *C0 = p.wC + ci * dv * dqk, *n0 = p.wn + ci * dqk;
    const float *Dx = p.wdC + ci * dv * dqk, *dnx = p.wdn + ci * dqk;

    // ---- per-token scalars (float64 gate arithmetic, as in the forward)
    if (warp == 0) {
        const double m0 = p.wm0[ci];
        const double *mt = p.wmt + (size_t)bh * p.T + t0;
        double F = 0.0;
        // sequential over 32-token halves: lane l holds tokens l and l + 32
        double fl[2] = {0.0, 0.0}, il[2] = {0.0, 0.0};
        for (int h2 = 0; h2 < 2; ++h2) {
            const int t = lane + 32 * h2;
            fl[h2] = t < L ? (double)p.fg[(size_t)bh * p.T + t0 + t] : 0.0;
            il[h2] = t < L ? (double)p.ig[(size_t)bh * p.T + t0 + t] : 0.0;
        }
        double Ft[2];
        for (int h2 = 0; h2 < 2; ++h2) {
            double incl = fl[h2];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            Ft[h2] = F + incl;
            F += __shfl_sync(0xffffffffu, incl, 31);
        }
        const double FL = __shfl_sync(0xffffffffu, (L - 1) < 32 ? Ft[0] : Ft[1], (L - 1) & 31);
        const double mL = mt[L - 1];
        for (int h2 = 0; h2 < 2; ++h2) {
            const int t = lane + 32 * h2;
            if (t < L) {
                const double m = mt[t];
                const double u = il[h2] - Ft[h2];
                su[t] = u;
                sFm[t] = Ft[h2] - m;
                sa[t] = expf((float)(Ft[h2] + m0 - m));
                sz[t] = expf((float)(u + FL - mL));
                float den, ds;
                readout_factors(p.wst[(size_t)bh * p.T + t0 + t], m, p.wgt[(size_t)bh * p.T + t0 + t], den, ds);
                sden[t] = den;
                sds[t] = ds;
            } else {
                su[t] = 0.0; sFm[t] = -INFINITY; sa[t] = 0.f; sz[t] = 0.f; sden[t] = 1.f; sds[t] = 0.f;
            }
            sG0[t] = 0.f; sGx[t] = 0.f; sdi[t] = 0.f;
        }
        if (lane == 0) red[kWarps] = expf((float)(FL + m0 - mL));   // a_L': entry state carried to the exit
    }
    __syncthreads();

    const int ty = tid >> 4, tx = tid & 15;   // the 4 x 4 output block of this thread
    // acc += A^T B over K in 32-deep tiles, the next tile's loads in flight during the
    // current tile's FMAs.  A[k][t] = ga(t, k) (token-major, k < na); B[k][s] = gb(s, k)
    // (product_tt, token-major, k < nb) or B[k][c] = gb(k, c0 + c) (product_tr, k < nb,
    // c0 + c < ncb).  Zero past the chunk's L tokens.
    auto product_tt = [&](auto ga, int na, auto gb, int nb, int K, float (&acc)[4][4]) {
        float ra[8], rb[8];
        fetch8<true>(ga, 0, na, 0, 0, L, ra);
        fetch8<true>(gb, 0, nb, 0, 0, L, rb);
        for (int k0 = 0; k0 < K; k0 += 32) {
            __syncthreads();
            put8<true>(As, ra);
            put8<true>(Bs, rb);
            __syncthreads();
            if (k0 + 32 < K) {
                fetch8<true>(ga, k0 + 32, na, 0, 0, L, ra);
                fetch8<true>(gb, k0 + 32, nb, 0, 0, L, rb);
            }
            tile_fma(As, Bs, acc, ty, tx);
        }
    };
    // 64 x 128 output tiles (B row-major, 128 columns from c0)
    auto product_trw = [&](auto ga, int na, auto gb, int nb, int c0, int ncb, int K, float (&acc)[4][8]) {
        float ra[8], rb[16];
        fetch8<true>(ga, 0, na, 0, 0, L, ra);
        fetch16(gb, 0, nb, c0, ncb, rb);
        for (int k0 = 0; k0 < K; k0 += 32) {
            __syncthreads();
            put8<true>(As, ra);
            put16(Bs, rb);
            __syncthreads();
            if (k0 + 32 < K) {
                fetch8<true>(ga, k0 + 32, na, 0, 0, L, ra);
                fetch16(gb, k0 + 32, nb, c0, ncb, rb);
            }
            tile_fma_w(As, Bs, acc, ty, tx);
        }
    };
    auto product_tr = [&](auto ga, int na, auto gb, int nb, int c0, int ncb, int K, float (&acc)[4][4]) {
        float ra[8], rb[8];
        fetch8<true>(ga, 0, na, 0, 0, L, ra);
        fetch8<false>(gb, 0, nb, c0, ncb, L, rb);
        for (int k0 = 0; k0 < K; k0 += 32) {
            __syncthreads();
            put8<true>(As, ra);
            put8<false>(Bs, rb);
            __syncthreads();
            if (k0 + 32 < K) {
                fetch8<true>(ga, k0 + 32, na, 0, 0, L, ra);
                fetch8<false>(gb, k0 + 32, nb, c0, ncb, L, rb);
            }
            tile_fma(As, Bs, acc, ty, tx);
        }
    };
    const auto Q = [&](int t, int j) { return p.scale * ld_in(q, (size_t)t * dqk + j); };
    const auto Kf = [&](int t, int j) { return ld_in(k, (size_t)t * dqk + j); };
    const auto Vf = [&](int t, int r) { return ld_in(v, (size_t)t * dv + r); };
    const auto DN = [&](int t, int r) { return dh[(size_t)t * dv + r] / sden[t]; };
    const auto Mf = [&](int t, int s) { return Mm[t * kLd + s]; };
    const auto MT = [&](int t, int s) { return Mm[s * kLd + t]; };
    const auto ET = [&](int t, int s) { return Em[s * kLd + t]; };

    // ---- S = Q K^T and P = DN V^T (64 x 64), then M, E and the intra pairs' G
    {
        float accS[4][4], accP[4][4];
        zero44(accS);
        zero44(accP);
        product_tt(Q, dqk, Kf, dqk, dqk, accS);
        product_tt(DN, dv, Vf, dv, dv, accP);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * ty + i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int s2 = 4 * tx + j;
                const float w = (s2 <= t && t < L) ? expf((float)(su[s2] + sFm[t])) : 0.f;
                const float Mv = w * (accP[i][j] + sds[t]);
                Mm[t * kLd + s2] = Mv;
                Em[t * kLd + s2] = w * accS[i][j];
                Gm[t * kLd + s2] = (s2 < t) ? Mv * accS[i][j] : 0.f;
            }
        }
    }
    __syncthreads();
    // intra pairs' share of df~_r: sum over t >= r, s < r of G_ts
    if (tid < kL) {
        const int r = tid;
        float acc = 0.f;
        for (int t = r; t < L; ++t)
            for (int s = 0; s < r; ++s) acc += Gm[t * kLd + s];
        sdfi[r] = acc;
    }
    // ---- dq = scale (diag(a) (DN C~_0 + ds~ n~_0^T) + M K); G_t0 = a_t q_t . (DN C~_0 + ds~ n~_0)_t
    const auto C0f = [&](int r, int j) { return C0[(size_t)r * dqk + j]; };
    const auto Dxf = [&](int r, int j) { return Dx[(size_t)r * dqk + j]; };
    for (int j0 = 0; j0 < dqk; j0 += 128) {
        float acc[4][8], intra[4][8];
        zero48(acc);
        zero48(intra);
        product_trw(DN, dv, C0f, dv, j0, dqk, dv, acc);
        product_trw(Mf, kL, Kf, L, j0, dqk, kL, intra);   // M K (M is zero above the diagonal and past L)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * ty + i;
            float g0 = 0.f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = j0 + 64 * (jj >> 2) + 4 * tx + (jj & 3);
                if (t < L && j < dqk) {
                    const float A1 = sa[t] * (acc[i][jj] + sds[t] * n0[j]);
                    p.dq[((size_t)bh * p.T + t0 + t) * dqk + j] = p.scale * (A1 + intra[i][jj]);
                    g0 = fmaf(Q(t, j), A1, g0);
                }
            }
            g0 = sum16(g0);
            if (tx == 0) sG0[t] += g0;
        }
    }
    // ---- dk = M^T Q + diag(z) (V dC~_ex + 1 dn~_ex^T); di~ = k . dk; G_s,ex = k_s . (exit part)
    for (int j0 = 0; j0 < dqk; j0 += 128) {
        float acc[4][8], intra[4][8];
        zero48(acc);
        zero48(intra);
        product_trw(Vf, dv, Dxf, dv, j0, dqk, dv, acc);
        product_trw(MT, kL, Q, L, j0, dqk, kL, intra);   // M^T Q
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * ty + i;
            float di = 0.f, gx = 0.f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = j0 + 64 * (jj >> 2) + 4 * tx + (jj & 3);
                if (t < L && j < dqk) {
                    const float ex = sz[t] * (acc[i][jj] + dnx[j]);
                    const float dkv = intra[i][jj] + ex;
                    p.dk[((size_t)bh * p.T + t0 + t) * dqk + j] = dkv;
                    const float kv = Kf(t, j);
                    di = fmaf(kv, dkv, di);
                    gx = fmaf(kv, ex, gx);
                }
            }
            di = sum16(di);
            gx = sum16(gx);
            if (tx == 0) {
                sdi[t] += di;
                sGx[t] += gx;
            }
        }
    }
    // ---- dv = E^T DN + diag(z) K dC~_ex^T
    const auto DxT = [&](int j, int r) { return Dx[(size_t)r * dqk + j]; };
    for (int r0 = 0; r0 < dv; r0 += 128) {
        float ex[4][8], intra[4][8];
        zero48(ex);
        zero48(intra);
        product_trw(Kf, dqk, DxT, dqk, r0, dv, dqk, ex);
        product_trw(ET, kL, DN, L, r0, dv, kL, intra);   // E^T DN
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = 4 * ty + i;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int r = r0 + 64 * (jj >> 2) + 4 * tx + (jj & 3);
                if (t < L && r < dv) p.dv_[((size_t)bh * p.T + t0 + t) * dv + r] = intra[i][jj] + sz[t] * ex[i][jj];
            }
        }
    }
    __syncthreads();
    // ---- the entry state carried to the exit: G_0,ex = a_L' (<dC~_ex, C~_0> + <dn~_ex, n~_0>)
    {
        float part = 0.f;
        for (size_t e = tid; e < (size_t)dv * dqk; e += kThreads) part = fmaf(Dx[e], C0[e], part);
        for (int j = tid; j < dqk; j += kThreads) part = fmaf(dnx[j], n0[j], part);
        part = warp_sum(part);
        __syncthreads();
        if (lane == 0) red[warp] = part;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < kWarps; ++w) s += red[w];
            red[kWarps + 1] = red[kWarps] * s;
        }
        __syncthreads();
    }
    // ---- df~_r and di~_r
    if (tid < L) {
        const int r = tid;
        float acc = sdfi[r] + red[kWarps + 1];
        for (int t = r; t < L; ++t) acc += sG0[t];
        for (int s = 0; s < r; ++s) acc += sGx[s];
        p.df[(size_t)bh * p.T + t0 + r] = acc;
        p.di[(size_t)bh * p.T + t0 + r] = sdi[r];
    }
}

size_t chunk_smem_bytes() {
    return (size_t)(3 * kL * kLd + 32 * kAs + 32 * kBs + 9 * kL + 2 * kWarps) * sizeof(float) + 2 * kL * sizeof(double) +
           16;
}

template <typename Tin>
cudaError_t launch_bwd_typed(BwdP p, cudaStream_t s) {
    const int maxc = (p.dqk + 31) / 32;
    const size_t smem_seq = (size_t)(2 * kTok * p.dqk + 2 * kTok * kRows + 2 * kTok + kTok * kWarps +
                                     2 * kWarps * kTok * 33 + 2 * kTok) * sizeof(float) + kTok * sizeof(double) + 16;
    const dim3 gseq(p.B * p.H * p.slices);
    cudaError_t e;
#define XLSTM_BWD_SEQ(MC)                                                                              \
    if (maxc <= MC) {                                                                                  \
        auto k1 = bwd_states_kernel<Tin, MC>;                                                          \
        auto k2 = bwd_adjoint_kernel<Tin, MC>;                                                         \
        if ((e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_seq)) \
            != cudaSuccess) return e;                                                                  \
        if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_seq)) \
            != cudaSuccess) return e;                                                                  \
        if (p.T > 0) {                                                                                 \
            k1<<<gseq, kThreads, smem_seq, s>>>(p);                                                    \
            if ((e = cudaGetLastError()) != cudaSuccess) return e;                                     \
            const size_t rows = (size_t)p.B * p.H * p.T;                                               \
            bwd_gsum_kernel<<<(unsigned)((rows + kThreads - 1) / kThreads), kThreads, 0, s>>>(p.wgp, p.wgt, rows, p.slices); \
            if ((e = cudaGetLastError()) != cudaSuccess) return e;                                     \
        }                                                                                              \
        k2<<<gseq, kThreads, smem_seq, s>>>(p);                                                        \
        if ((e = cudaGetLastError()) != cudaSuccess) return e;                                         \
    } else
    XLSTM_BWD_SEQ(1) XLSTM_BWD_SEQ(2) XLSTM_BWD_SEQ(4) XLSTM_BWD_SEQ(8) XLSTM_BWD_SEQ(16) return cudaErrorInvalidValue;
#undef XLSTM_BWD_SEQ
    if (p.dm0) {
        const int BH = p.B * p.H;
        bwd_dm0_kernel<<<(BH + 255) / 256, 256, 0, s>>>(p.wdm, p.dm0, BH, p.slices);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.NC == 0) return cudaSuccess;
    const size_t smem3 = chunk_smem_bytes();
    auto k3 = bwd_chunk_kernel<Tin>;
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3)) != cudaSuccess)
        return e;
    k3<<<p.B * p.H * p.NC, kThreads, smem3, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t backward_workspace_bytes(int BH, int T, int dqk, int dv) { return bwd_layout(BH, T, dqk, dv).bytes; }

cudaError_t launch_backward(const BwdArgs &a, cudaStream_t s) {
    const int BH = a.B * a.H;
    const BwdLayout l = bwd_layout(BH, a.T, a.dqk, a.dv);
    char *ws = static_cast<char *>(a.workspace);
    BwdP p;
    p.B = a.B; p.H = a.H; p.T = a.T; p.dqk = a.dqk; p.dv = a.dv;
    p.slices = (a.dv + kRows - 1) / kRows;
    p.NC = (a.T + kL - 1) / kL;
    p.scale = a.scale;
    p.q = a.q; p.k = a.k; p.v = a.v; p.ig = a.ig; p.fg = a.fg;
    p.C0 = a.C0; p.n0 = a.n0; p.m0 = a.m0; p.dh = a.dh; p.dCT = a.dCT; p.dnT = a.dnT;
    p.dq = a.dq; p.dk = a.dk; p.dv_ = a.dv_; p.di = a.di; p.df = a.df; p.dC0 = a.dC0; p.dn0 = a.dn0; p.dm0 = a.dm0;
    p.wC = reinterpret_cast<float *>(ws + l.off_C);
    p.wdC = reinterpret_cast<float *>(ws + l.off_dC);
    p.wn = reinterpret_cast<float *>(ws + l.off_n);
    p.wdn = reinterpret_cast<float *>(ws + l.off_dn);
    p.wm0 = reinterpret_cast<double *>(ws + l.off_m0);
    p.wmt = reinterpret_cast<double *>(ws + l.off_mt);
    p.wst = reinterpret_cast<float *>(ws + l.off_st);
    p.wgt = reinterpret_cast<float *>(ws + l.off_gt);
    p.wgp = reinterpret_cast<float *>(ws + l.off_gp);
    p.wdm = reinterpret_cast<float *>(ws + l.off_dm);
    return a.dtype == XLSTM_BF16 ? launch_bwd_typed<__nv_bfloat16>(p, s) : launch_bwd_typed<float>(p, s);
}

}  // namespace xlstm
