// Single-step mLSTM decode kernel (memory-bound).
//
// One step of the recurrence (xLSTM page, "mLSTM (matrix LSTM)" eq. 1-3 with
// the "sLSTM" stabilizer), for every (batch, head) at once:
//   m' = max(f~ + m, i~); f' = e^{f~+m-m'}; i' = e^{i~-m'}
//   C' = f' C + i' v k^T;  n' = f' n + i' k;  h~ = C' q / max(|n'^T q|, e^{-m'})
//
// The state C (d_v x d_qk fp32 per head) dominates the traffic: it is read and
// written exactly once, as 128-bit streaming accesses.  A block owns a range of
// C rows of one head; lanes of a warp cover one row (or several short rows)
// with float4s, so every warp-wide access is a contiguous run.  The block
// first stages k and the scaled q in shared memory and computes n' and n'^T q
// itself (d_qk MACs, negligible), so no second pass is needed.
#include "common.cuh"

namespace xlstm {
namespace {

constexpr int kThreads = 256;
// Rows per lane in flight: with all columns of a row group loaded before use, two
// rows keep enough loads outstanding and leave room for more resident blocks than four
// (decode shape: 0.175 ms at two, 0.191 at four or eight, 0.226 at one).
constexpr int kUnroll = 2;

struct StepP {
    int BH, dqk, dv, rows_per_block;
    float scale;
    const void *q, *k, *v;
    const float *ig, *fg, *C, *n, *m;
    float *h, *C1, *n1, *m1;
};

// NC: float4 columns per lane per row (ceil(d_qk / 4 / lanes per row)); all of a row
// group's loads are issued before any of it is used.
template <typename Tin, int NC>
__global__ void __launch_bounds__(kThreads) step_kernel(StepP p) {
    extern __shared__ float4 smem4[];
    const int dqk = p.dqk, G = dqk >> 2;   // float4 per row
    float4 *qs4 = smem4;                   // scaled q
    float4 *ks4 = smem4 + G;               // k
    __shared__ float red[kThreads / 32];

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const Tin *q = static_cast<const Tin *>(p.q) + (size_t)bh * dqk;
    const Tin *k = static_cast<const Tin *>(p.k) + (size_t)bh * dqk;
    const Tin *v = static_cast<const Tin *>(p.v) + (size_t)bh * p.dv;

    float m_new, fp, ip;
    stabilized_gates(p.fg[bh], p.ig[bh], p.m[bh], m_new, fp, ip);

    float *qs = reinterpret_cast<float *>(qs4), *ks = reinterpret_cast<float *>(ks4);
    for (int j = tid; j < dqk; j += kThreads) {
        qs[j] = p.scale * to_f32(q[j]);
        ks[j] = to_f32(k[j]);
    }
    __syncthreads();

    // n' = f' n + i' k and its dot with q (every block; block 0 stores n').
    float part = 0.f;
    const float *nin = p.n + (size_t)bh * dqk;
    for (int j = tid; j < dqk; j += kThreads) {
        const float nn = fp * nin[j] + ip * ks[j];
        part += nn * qs[j];
        if (blockIdx.y == 0) p.n1[(size_t)bh * dqk + j] = nn;
    }
    part = warp_sum(part);
    if (lane == 0) red[warp] = part;
    __syncthreads();
    float nq = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) nq += red[w];
    const float den = fmaxf(fabsf(nq), expf(-m_new));
    const float inv_den = 1.f / den;

    // Lane layout over rows: LG lanes per row, RW rows per warp iteration.
    const int LG = (G <= 32 && (G & (G - 1)) == 0) ? G : 32;
    const int RW = 32 / LG;

    const int lrow = lane / LG, lcol = lane % LG;
    const int r_begin = blockIdx.y * p.rows_per_block;
    const int r_end = min(p.dv, r_begin + p.rows_per_block);
    const float4 *C4 = reinterpret_cast<const float4 *>(p.C) + (size_t)bh * p.dv * G;
    float4 *C14 = reinterpret_cast<float4 *>(p.C1) + (size_t)bh * p.dv * G;
    float *h = p.h + (size_t)bh * p.dv;
    const int warps = kThreads / 32;

    for (int r0 = r_begin + warp * RW * kUnroll; r0 < r_end; r0 += warps * RW * kUnroll) {
        float acc[kUnroll], vr[kUnroll];
        float4 cv[kUnroll][NC];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int r = r0 + u * RW + lrow;
            acc[u] = 0.f;
            vr[u] = r < r_end ? to_f32(v[r]) : 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int j4 = lcol + c * LG;
                cv[u][c] = (r < r_end && j4 < G) ? __ldcs(C4 + (size_t)r * G + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j4 = lcol + c * LG;
            if (j4 < G) {
                const float4 kv = ks4[j4], qv = qs4[j4];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int r = r0 + u * RW + lrow;
                    if (r < r_end) {
                        const float a = ip * vr[u];
                        float4 o;
                        o.x = fmaf(fp, cv[u][c].x, a * kv.x);
                        o.y = fmaf(fp, cv[u][c].y, a * kv.y);
                        o.z = fmaf(fp, cv[u][c].z, a * kv.z);
                        o.w = fmaf(fp, cv[u][c].w, a * kv.w);
                        __stcs(C14 + (size_t)r * G + j4, o);
                        acc[u] += o.x * qv.x + o.y * qv.y + o.z * qv.z + o.w * qv.w;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float s = acc[u];
            for (int o = LG >> 1; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const int r = r0 + u * RW + lrow;
            if (lcol == 0 && r < r_end) h[r] = s * inv_den;
        }
    }
    if (blockIdx.y == 0 && tid == 0) p.m1[bh] = m_new;
}

}  // namespace

cudaError_t launch_step(const FwdArgs &a, cudaStream_t s) {
    StepP p;
    p.BH = a.B * a.H;
    p.dqk = a.dqk;
    p.dv = a.dv;
    p.scale = a.scale;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.ig = a.ig; p.fg = a.fg; p.C = a.C0; p.n = a.n0; p.m = a.m0;
    p.h = a.h; p.C1 = a.C1; p.n1 = a.n1; p.m1 = a.m1;
    // In-place n/m updates are only race-free when one block owns a head.
    const bool inplace = (a.n1 == a.n0) || (a.m1 == a.m0);
    int blocks_per_head = 1;
    if (!inplace) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const long long target = 8LL * sms;
        while ((long long)p.BH * blocks_per_head < target && a.dv / (blocks_per_head * 2) >= 16)
            blocks_per_head *= 2;
    }
    p.rows_per_block = (a.dv + blocks_per_head - 1) / blocks_per_head;
    dim3 grid(p.BH, blocks_per_head);
    const size_t smem = 2 * (size_t)a.dqk * sizeof(float);
    const int G = a.dqk / 4, LG = (G <= 32 && (G & (G - 1)) == 0) ? G : 32, nc = (G + LG - 1) / LG;
#define XLSTM_STEP_LAUNCH(NCV)                                                          \
    if (nc == NCV) {                                                                    \
        if (a.dtype == XLSTM_BF16)                                                      \
            step_kernel<__nv_bfloat16, NCV><<<grid, kThreads, smem, s>>>(p);            \
        else                                                                            \
            step_kernel<float, NCV><<<grid, kThreads, smem, s>>>(p);                    \
        return cudaGetLastError();                                                      \
    }
    XLSTM_STEP_LAUNCH(1) XLSTM_STEP_LAUNCH(2) XLSTM_STEP_LAUNCH(3) XLSTM_STEP_LAUNCH(4)
#undef XLSTM_STEP_LAUNCH
    return cudaErrorInvalidValue;
}

}  // namespace xlstm
