// Chunkwise-parallel mLSTM forward on fp32 CUDA cores.
//
// Used for fp32 inputs (where fp32 arithmetic is needed to meet a 1e-4
// relative tolerance) and for head sizes the tensor-core kernel does not
// take.  Same math as that kernel, evaluated per chunk of L tokens:
//
//   F_t = sum_{r<=t} f~_r,  u_s = i~_s - F_s,  mu_t = max(m0, max_{s<=t} u_s),
//   m_t = F_t + mu_t   (the unrolled stabilizer m_t = max(f~_t + m_{t-1}, i~_t)),
//   h~_t = [e^{m0-mu_t} C~0 q_t + sum_{s<=t} e^{u_s-mu_t} (q_t.k_s) v_s]
//          / max(|e^{m0-mu_t} n~0.q_t + sum_{s<=t} e^{u_s-mu_t} q_t.k_s|, e^{-m_t}),
//   C~_L = e^{m0-mu_L} C~0 + sum_s e^{u_s-mu_L} v_s k_s^T  (likewise n~), m <- m_L.
// Every exponent above is <= 0, so nothing overflows however large the gates.
// The gate scan runs in float64 and hands the pairwise exponents u_s - mu_t on
// as float hi/lo pairs: with strong forgetting F_t reaches 1e5 and more inside
// one chunk, where the fp32 difference would cancel catastrophically.
//
// A block owns kDvs rows of C~ for one (batch, head) and keeps them in shared
// memory for the whole sequence; q and k are streamed through in kKt-wide
// column tiles.
#include "common.cuh"

namespace xlstm {
namespace {

constexpr int kThreads = 256;
constexpr int kDvs = 32;   // rows of C~ per block
constexpr int kKt = 32;    // d_qk tile

struct ChunkP {
    int B, H, T, dqk, dv, L, slices;
    float scale;
    const void *q, *k, *v;
    const float *ig, *fg, *C0, *n0, *m0;
    float *h, *C1, *n1, *m1;
    OutStage out;
};

template <typename Tin, int L>
__global__ void __launch_bounds__(kThreads) chunk_simt_kernel(ChunkP p) {
    extern __shared__ double smd[];
    double *mst = smd;                       // carried stabilizer m (float64)
    float *sm = reinterpret_cast<float *>(smd + 2);
    const int dqk = p.dqk, dv = p.dv;
    const int cst = dqk + 1;                 // padded row stride of C~
    float *Cs = sm;                          // [kDvs][dqk+1]
    float *ns = Cs + kDvs * cst;             // [dqk]
    float *Qt = ns + dqk;                    // [L][kKt+1]
    float *Kt = Qt + L * (kKt + 1);          // [L][kKt+1]
    float *Vs = Kt + L * (kKt + 1);          // [L][kDvs]
    float *Ps = Vs + L * kDvs;               // [L][L+1]
    float *sc = Ps + L * (L + 1);            // per-token scalars
    float *uh_s = sc, *ul_s = sc + L, *mh_s = sc + 2 * L, *ml_s = sc + 3 * L, *al_s = sc + 4 * L;
    float *lo_s = sc + 5 * L, *g_s = sc + 6 * L, *nq_s = sc + 7 * L, *r_s = sc + 8 * L;
    float *ig_s = sc + 9 * L, *fg_s = sc + 10 * L, *misc = sc + 11 * L;   // misc[0] = beta, misc[1] = m

    const int bh = blockIdx.x / p.slices;
    const int row0 = (blockIdx.x % p.slices) * kDvs;
    const int tid = threadIdx.x;
    const Tin *q = static_cast<const Tin *>(p.q) + (size_t)bh * p.T * dqk;
    const Tin *k = static_cast<const Tin *>(p.k) + (size_t)bh * p.T * dqk;
    const Tin *v = static_cast<const Tin *>(p.v) + (size_t)bh * p.T * dv;

    for (int e = tid; e < kDvs * dqk; e += kThreads) {
        const int r = e / dqk, j = e % dqk;
        Cs[r * cst + j] = (p.C0 && row0 + r < dv) ? p.C0[((size_t)bh * dv + row0 + r) * dqk + j] : 0.f;
    }
    for (int j = tid; j < dqk; j += kThreads) ns[j] = p.n0 ? p.n0[(size_t)bh * dqk + j] : 0.f;
    if (tid == 0) {
        mst[0] = p.m0 ? (double)p.m0[bh] : 0.0;
        misc[1] = (float)mst[0];
    }

    constexpr int kS = (L * L + kThreads - 1) / kThreads;     // S entries per thread
    constexpr int kH = (L * kDvs + kThreads - 1) / kThreads;  // h entries per thread

    for (int t0 = 0; t0 < p.T; t0 += L) {
        const int len = min(L, p.T - t0);
        __syncthreads();
        if (tid < L) {
            ig_s[tid] = tid < len ? p.ig[(size_t)bh * p.T + t0 + tid] : 0.f;
            fg_s[tid] = tid < len ? p.fg[(size_t)bh * p.T + t0 + tid] : 0.f;
        }
        __syncthreads();
        if (tid == 0) {   // gate scan (float64): cumulative log forget and running max
            const double m0 = mst[0];
            double F = 0.0, mu = m0;
            for (int t = 0; t < len; ++t) {
                F += (double)fg_s[t];
                const double u = (double)ig_s[t] - F;
                mu = fmax(mu, u);
                uh_s[t] = (float)u;
                ul_s[t] = isfinite(uh_s[t]) ? (float)(u - (double)uh_s[t]) : 0.f;
                mh_s[t] = (float)mu;
                ml_s[t] = (float)(mu - (double)mh_s[t]);
                al_s[t] = expf((float)(m0 - mu));
                lo_s[t] = expf((float)(-(F + mu)));
            }
            for (int t = 0; t < len; ++t)
                g_s[t] = expf((float)(((double)uh_s[t] + (double)ul_s[t]) - mu));
            for (int t = len; t < L; ++t) {
                uh_s[t] = 0.f; ul_s[t] = 0.f; mh_s[t] = 0.f; ml_s[t] = 0.f;
                al_s[t] = 0.f; lo_s[t] = 1.f; g_s[t] = 0.f;
            }
            misc[0] = expf((float)(m0 - mu));
            mst[0] = F + mu;
            misc[1] = (float)mst[0];
        }

        // S = Q K^T, H_inter = Q C~0^T, nq = Q n~0, over d_qk tiles.
        float S[kS], Hi[kH], nq = 0.f;
#pragma unroll
        for (int x = 0; x < kS; ++x) S[x] = 0.f;
#pragma unroll
        for (int x = 0; x < kH; ++x) Hi[x] = 0.f;
        for (int j0 = 0; j0 < dqk; j0 += kKt) {
            __syncthreads();
            for (int e = tid; e < L * kKt; e += kThreads) {
                const int t = e / kKt, j = e % kKt;
                const bool ok = t < len && j0 + j < dqk;
                Qt[t * (kKt + 1) + j] = ok ? p.scale * to_f32(q[(size_t)(t0 + t) * dqk + j0 + j]) : 0.f;
                Kt[t * (kKt + 1) + j] = ok ? to_f32(k[(size_t)(t0 + t) * dqk + j0 + j]) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int x = 0; x < kS; ++x) {
                const int e = tid + x * kThreads;
                if (e < L * L) {
                    const int t = e / L, s = e % L;
                    float a = 0.f;
#pragma unroll 8
                    for (int j = 0; j < kKt; ++j) a += Qt[t * (kKt + 1) + j] * Kt[s * (kKt + 1) + j];
                    S[x] += a;
                }
            }
#pragma unroll
            for (int x = 0; x < kH; ++x) {
                const int e = tid + x * kThreads;
                if (e < L * kDvs) {
                    const int t = e / kDvs, r = e % kDvs;
                    float a = 0.f;
                    const int jn = min(kKt, dqk - j0);
                    for (int j = 0; j < jn; ++j) a += Qt[t * (kKt + 1) + j] * Cs[r * cst + j0 + j];
                    Hi[x] += a;
                }
            }
            if (tid < L) {
                const int jn = min(kKt, dqk - j0);
                for (int j = 0; j < jn; ++j) nq += Qt[tid * (kKt + 1) + j] * ns[j0 + j];
            }
        }
        // P = S * e^{u_s - mu_t} on s <= t, and row sums.
#pragma unroll
        for (int x = 0; x < kS; ++x) {
            const int e = tid + x * kThreads;
            if (e < L * L) {
                const int t = e / L, s = e % L;
                const float e = (uh_s[s] - mh_s[t]) + (ul_s[s] - ml_s[t]);
                Ps[t * (L + 1) + s] = (s <= t && t < len) ? S[x] * expf(e) : 0.f;
            }
        }
        if (tid < L) nq_s[tid] = nq;
        for (int e = tid; e < L * kDvs; e += kThreads) {
            const int s = e / kDvs, r = e % kDvs;
            Vs[e] = (s < len && row0 + r < dv) ? to_f32(v[(size_t)(t0 + s) * dv + row0 + r]) : 0.f;
        }
        __syncthreads();
        if (tid < L) {
            float a = 0.f;
            for (int s = 0; s < L; ++s) a += Ps[tid * (L + 1) + s];
            r_s[tid] = a;
        }
        __syncthreads();
        // h = (alpha H_inter + P V) / max(|alpha nq + r|, e^{-m_t}).
#pragma unroll
        for (int x = 0; x < kH; ++x) {
            const int e = tid + x * kThreads;
            if (e < L * kDvs) {
                const int t = e / kDvs, r = e % kDvs;
                float a = 0.f;
                for (int s = 0; s <= t; ++s) a += Ps[t * (L + 1) + s] * Vs[s * kDvs + r];
                const float num = al_s[t] * Hi[x] + a;
                const float den = fmaxf(fabsf(al_s[t] * nq_s[t] + r_s[t]), lo_s[t]);
                if (t < len && row0 + r < dv) store_h(p.out, p.h, ((size_t)bh * p.T + t0 + t) * dv + row0 + r, num / den);
            }
        }
        __syncthreads();
        // Weighted values g_s v_s, then C~ <- beta C~ + (g V)^T K and n~ likewise.
        for (int e = tid; e < L * kDvs; e += kThreads) Vs[e] *= g_s[e / kDvs];
        const float beta = misc[0];
        for (int j0 = 0; j0 < dqk; j0 += kKt) {
            __syncthreads();
            for (int e = tid; e < L * kKt; e += kThreads) {
                const int t = e / kKt, j = e % kKt;
                Kt[t * (kKt + 1) + j] = (t < len && j0 + j < dqk) ? to_f32(k[(size_t)(t0 + t) * dqk + j0 + j]) : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < kDvs * kKt; e += kThreads) {
                const int r = e / kKt, j = e % kKt;
                if (j0 + j < dqk) {
                    float a = 0.f;
                    for (int s = 0; s < len; ++s) a += Vs[s * kDvs + r] * Kt[s * (kKt + 1) + j];
                    Cs[r * cst + j0 + j] = beta * Cs[r * cst + j0 + j] + a;
                }
            }
            if (tid < kKt && j0 + tid < dqk) {
                float a = 0.f;
                for (int s = 0; s < len; ++s) a += g_s[s] * Kt[s * (kKt + 1) + tid];
                ns[j0 + tid] = beta * ns[j0 + tid] + a;
            }
        }
    }
    __syncthreads();
    if (p.C1)
        for (int e = tid; e < kDvs * dqk; e += kThreads) {
            const int r = e / dqk, j = e % dqk;
            if (row0 + r < dv) p.C1[((size_t)bh * dv + row0 + r) * dqk + j] = Cs[r * cst + j];
        }
    if (p.n1 && row0 == 0)
        for (int j = tid; j < dqk; j += kThreads) p.n1[(size_t)bh * dqk + j] = ns[j];
    if (p.m1 && row0 == 0 && tid == 0) p.m1[bh] = misc[1];
}

template <typename Tin, int L>
cudaError_t launch_L(const ChunkP &p, cudaStream_t s) {
    const size_t smem = 2 * sizeof(double) + (size_t)(kDvs * (p.dqk + 1) + p.dqk + 2 * L * (kKt + 1) +
                                                      L * kDvs + L * (L + 1) + 11 * L + 2) * sizeof(float);
    auto kern = chunk_simt_kernel<Tin, L>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.B * p.H * p.slices, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_typed(const ChunkP &p, cudaStream_t s) {
    switch (p.L) {
        case 16: return launch_L<Tin, 16>(p, s);
        case 32: return launch_L<Tin, 32>(p, s);
        case 64: return launch_L<Tin, 64>(p, s);
        case 128: return launch_L<Tin, 128>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_chunkwise_simt(const FwdArgs &a, cudaStream_t s) {
    ChunkP p;
    p.B = a.B; p.H = a.H; p.T = a.T; p.dqk = a.dqk; p.dv = a.dv; p.L = a.chunk;
    p.slices = (a.dv + kDvs - 1) / kDvs;
    p.scale = a.scale;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.ig = a.ig; p.fg = a.fg; p.C0 = a.C0; p.n0 = a.n0; p.m0 = a.m0;
    p.h = a.h; p.C1 = a.C1; p.n1 = a.n1; p.m1 = a.m1;
    p.out = a.out;
    return a.dtype == XLSTM_BF16 ? launch_typed<__nv_bfloat16>(p, s) : launch_typed<float>(p, s);
}

}  // namespace xlstm
