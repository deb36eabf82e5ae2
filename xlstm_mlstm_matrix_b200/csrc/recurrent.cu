// Recurrent mLSTM forward: the per-token recurrence with the state on chip.
//
// This is the O(1)-state, O(T)-time form of the xLSTM page ("xLSTM 블록 구성":
// constant memory and linear time at inference), i.e. the page's
// forward_recurrent listing applied token after token, without projections
// and output gate, with the stabilized readout max(|n~^T q|, e^{-m}).
//
// A block owns kRows rows of C~ for one (batch, head): warp w holds rows
// [w*kRpw, (w+1)*kRpw) in registers, lane l holds columns l, l+32, ... of each.
// The normaliser n~ is spread over the block, thread i holding columns i, i+256,
// ...: per token each thread stores its part of n~^T q, and the staged tokens'
// sums and denominators are formed once per staged block, when the outputs are
// written, so no block barrier sits on the per-token path.
// Inputs for kTok tokens are staged in shared memory per barrier; the outputs
// of those tokens are staged too and written back as contiguous rows.
#include "common.cuh"

namespace xlstm {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRpw = 4;                 // rows per warp
constexpr int kRows = kWarps * kRpw;    // rows per block
constexpr int kTok = 16;                // tokens staged per barrier

struct RecP {
    int B, H, T, dqk, dv, slices;
    float scale;
    const void *q, *k, *v;
    const float *ig, *fg, *C0, *n0, *m0;
    float *h, *C1, *n1, *m1;
};

template <typename Tin, int MAXC>
__global__ void __launch_bounds__(kThreads) recurrent_kernel(RecP p) {
    extern __shared__ float sm[];
    const int dqk = p.dqk, dv = p.dv;
    float *sq = sm;                          // [kTok][dqk] scaled q
    float *sk = sq + kTok * dqk;             // [kTok][dqk]
    float *sv = sk + kTok * dqk;             // [kTok][kRows]
    float *sg = sv + kTok * kRows;           // [kTok][4] (f', i', e^{-m_t}, m_t) of each staged token
    float *sh = sg + 4 * kTok;               // [kTok][kRows] outputs (before the denominator)
    float *snq = sh + kTok * kRows;          // [kTok][kThreads] parts of n~^T q
    float *sden = snq + kTok * kThreads;     // [kTok] 1 / max(|n~^T q|, e^{-m_t})

    const int bh = blockIdx.x / p.slices;
    const int slice = blockIdx.x % p.slices;
    const int row0 = slice * kRows;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const Tin *q = static_cast<const Tin *>(p.q) + (size_t)bh * p.T * dqk;
    const Tin *k = static_cast<const Tin *>(p.k) + (size_t)bh * p.T * dqk;
    const Tin *v = static_cast<const Tin *>(p.v) + (size_t)bh * p.T * dv;
    const float *ig = p.ig + (size_t)bh * p.T;
    const float *fg = p.fg + (size_t)bh * p.T;

    constexpr int NJ = (MAXC * 32 + kThreads - 1) / kThreads;   // normaliser columns per thread
    float C[kRpw][MAXC];
    float n[NJ];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < NJ; ++i) {
        const int j = tid + kThreads * i;
        n[i] = (p.n0 && j < dqk) ? p.n0[(size_t)bh * dqk + j] : 0.f;
    }
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int j = lane + 32 * c;
#pragma unroll
        for (int r = 0; r < kRpw; ++r) {
            const int row = row0 + warp * kRpw + r;
            C[r][c] = (p.C0 && j < dqk && row < dv) ? p.C0[((size_t)bh * dv + row) * dqk + j] : 0.f;
        }
    }
    if (p.m0) m = p.m0[bh];

    for (int t0 = 0; t0 < p.T; t0 += kTok) {
        const int nt = min(kTok, p.T - t0);
        __syncthreads();   // previous block's outputs have been written out
        for (int e = tid; e < nt * dqk; e += kThreads) {
            sq[e] = p.scale * to_f32(q[(size_t)t0 * dqk + e]);
            sk[e] = to_f32(k[(size_t)t0 * dqk + e]);
        }
        for (int e = tid; e < nt * kRows; e += kThreads) {
            const int tt = e / kRows, r = e % kRows;
            sv[e] = (row0 + r < dv) ? to_f32(v[(size_t)(t0 + tt) * dv + row0 + r]) : 0.f;
        }
        if (tid < nt) {   // the gates of the staged tokens, once per block: the stabilizer chain
            sg[4 * tid] = fg[t0 + tid];   // on one thread, the exponentials on one thread per token
            sg[4 * tid + 1] = ig[t0 + tid];
        }
        __syncthreads();
        if (tid == 0) {
            float mm = m;
            for (int tt = 0; tt < nt; ++tt) {
                const float a = sg[4 * tt] + mm;
                mm = (a > sg[4 * tt + 1]) ? a : sg[4 * tt + 1];
                sg[4 * tt + 3] = mm;
            }
        }
        __syncthreads();
        if (tid < nt) {
            const float mp = tid ? sg[4 * (tid - 1) + 3] : m, f = sg[4 * tid], i = sg[4 * tid + 1];
            float m_new, fp, ip;
            stabilized_gates(f, i, mp, m_new, fp, ip);
            sg[4 * tid] = fp;
            sg[4 * tid + 1] = ip;
            sg[4 * tid + 2] = expf(-m_new);
        }
        __syncthreads();

        for (int tt = 0; tt < nt; ++tt) {
            const float fp = sg[4 * tt], ip = sg[4 * tt + 1], m_new = sg[4 * tt + 3];
            const float *qt = sq + tt * dqk, *kt = sk + tt * dqk;
            float qv[MAXC], kv[MAXC];
#pragma unroll
            for (int c = 0; c < MAXC; ++c) {
                const int j = lane + 32 * c;
                qv[c] = (j < dqk) ? qt[j] : 0.f;
                kv[c] = (j < dqk) ? kt[j] : 0.f;
            }
            float nq = 0.f;   // this thread's part of n~^T q
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
                const int j = tid + kThreads * i;
                if (j < dqk) {
                    n[i] = fp * n[i] + ip * kt[j];
                    nq += n[i] * qt[j];
                }
            }
            snq[tt * kThreads + tid] = nq;
            float acc[kRpw];
#pragma unroll
            for (int r = 0; r < kRpw; ++r) {
                const float a = ip * sv[tt * kRows + warp * kRpw + r];
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < MAXC; ++c) {
                    C[r][c] = fmaf(fp, C[r][c], a * kv[c]);
                    s += C[r][c] * qv[c];
                }
                acc[r] = s;
            }
            // the warp's four row sums at once: lanes trade half of their values at each
            // of the first two steps (xor 16, then 8), then sum one value (xor 4, 2, 1);
            // lane 8 r ends with row r
            static_assert(kRpw == 4, "four rows per warp");
            const bool b4 = lane & 16, b3 = lane & 8;
            float s0 = b4 ? acc[2] : acc[0], s1 = b4 ? acc[3] : acc[1];
            s0 += __shfl_xor_sync(0xffffffffu, b4 ? acc[0] : acc[2], 16);
            s1 += __shfl_xor_sync(0xffffffffu, b4 ? acc[1] : acc[3], 16);
            float rsum = b3 ? s1 : s0;
            rsum += __shfl_xor_sync(0xffffffffu, b3 ? s0 : s1, 8);
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) rsum += __shfl_xor_sync(0xffffffffu, rsum, o);
            if ((lane & 7) == 0) sh[tt * kRows + warp * kRpw + (lane >> 3)] = rsum;
            m = m_new;
        }
        __syncthreads();
        {   // n~^T q of each staged token: 16 threads per token, 16 parts each, then a 16-lane sum
            const int tt = tid >> 4, part = tid & 15;
            float x = 0.f;
            if (tt < nt) {
#pragma unroll
                for (int i = 0; i < kThreads / 16; ++i) x += snq[tt * kThreads + part + 16 * i];
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            if (part == 0 && tt < nt) sden[tt] = 1.f / fmaxf(fabsf(x), sg[4 * tt + 2]);
        }
        __syncthreads();
        float *h = p.h + ((size_t)bh * p.T + t0) * dv + row0;
        for (int e = tid; e < nt * kRows; e += kThreads) {
            const int tt = e / kRows, r = e % kRows;
            if (row0 + r < dv) h[(size_t)tt * dv + r] = sh[e] * sden[tt];
        }
    }

    // Final state.
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        const int j = lane + 32 * c;
        if (j >= dqk) continue;
        if (p.C1) {
#pragma unroll
            for (int r = 0; r < kRpw; ++r) {
                const int row = row0 + warp * kRpw + r;
                if (row < dv) p.C1[((size_t)bh * dv + row) * dqk + j] = C[r][c];
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NJ; ++i) {
        const int j = tid + kThreads * i;
        if (p.n1 && slice == 0 && j < dqk) p.n1[(size_t)bh * dqk + j] = n[i];
    }
    if (p.m1 && slice == 0 && tid == 0) p.m1[bh] = m;
}

template <typename Tin>
cudaError_t launch_typed(const RecP &p, int dqk, cudaStream_t s) {
    const int slices = p.slices;
    dim3 grid(p.B * p.H * slices);
    const size_t smem = (size_t)(2 * kTok * dqk + 2 * kTok * kRows + 4 * kTok + kTok * kThreads + kTok) * sizeof(float);
    const int maxc = (dqk + 31) / 32;
#define XLSTM_REC_CASE(MC)                                                                   \
    if (maxc <= MC) {                                                                        \
        auto kern = recurrent_kernel<Tin, MC>;                                               \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);  \
        kern<<<grid, kThreads, smem, s>>>(p);                                                \
        return cudaGetLastError();                                                           \
    }
    XLSTM_REC_CASE(1)
    XLSTM_REC_CASE(2)
    XLSTM_REC_CASE(4)
    XLSTM_REC_CASE(8)
    XLSTM_REC_CASE(16)
#undef XLSTM_REC_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent(const FwdArgs &a, cudaStream_t s) {
    RecP p;
    p.B = a.B; p.H = a.H; p.T = a.T; p.dqk = a.dqk; p.dv = a.dv;
    p.slices = (a.dv + kRows - 1) / kRows;
    p.scale = a.scale;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.ig = a.ig; p.fg = a.fg; p.C0 = a.C0; p.n0 = a.n0; p.m0 = a.m0;
    p.h = a.h; p.C1 = a.C1; p.n1 = a.n1; p.m1 = a.m1;
    return a.dtype == XLSTM_BF16 ? launch_typed<__nv_bfloat16>(p, a.dqk, s)
                                 : launch_typed<float>(p, a.dqk, s);
}

}  // namespace xlstm
