// Output stage of the mLSTM readout (xLSTM page, "mLSTM (matrix LSTM)" eq. 3,
// and the o_t line of its listing): h = sigmoid(o~) h~, element by element, as
// one streaming pass over h~ in place after the tensor-core chunkwise kernel.
// Memory-bound: each element is read once from h~ and o~ and written once, with
// 16-byte vector accesses (d_v is a multiple of 16 and every pointer is 16-byte
// aligned, so 8-element groups never straddle a row or a boundary).
#include "common.cuh"

namespace xlstm {
namespace {

__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4 *>(p)), b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void store8(float *p, const float (&x)[8]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 v = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&v);
    }
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w[0], w[1], w[2], w[3]));
}

template <typename TH, typename TO>
__global__ void __launch_bounds__(256) output_gate_kernel(TH *h, const TO *o, size_t groups) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
        float hv[8], ov[8];
        load8(h + 8 * g, hv);
        load8(o + 8 * g, ov);
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i] = gate_h(hv[i], ov[i]);
        store8(h + 8 * g, hv);
    }
}

// Raw 8-element groups, held as loaded until every load of the thread is issued.
template <typename T> struct Raw8;
template <> struct Raw8<float> {
    float4 a, b;
    __device__ void load(const float *p) {
        a = __ldcs(reinterpret_cast<const float4 *>(p));
        b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    }
    __device__ void unpack(float (&x)[8]) const {
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
};
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ void load(const __nv_bfloat16 *p) { u = __ldcs(reinterpret_cast<const uint4 *>(p)); }
    __device__ void unpack(float (&x)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};

// The gate on a fixed set of SMs beside another kernel: one 1024-thread block per SM,
// each holding more than half of the SM's shared memory (unused) so that no second
// block, nor a block of a kernel that needs the whole SM, can share it.  Grid-strided,
// kGroups groups of 8 elements per thread in flight (two when h~ or o~ is fp32, to stay
// within the 64 registers a thread of a 1024-thread block has).
constexpr int kFenceThreads = 1024;
template <typename TH, typename TO>
__global__ void __launch_bounds__(kFenceThreads, 1) output_gate_fenced_kernel(TH *h, const TO *o, size_t groups) {
    constexpr int kGroups = sizeof(TH) == 2 && sizeof(TO) == 2 ? 4 : 2;
    const size_t step = (size_t)gridDim.x * kFenceThreads * kGroups;
    for (size_t g0 = (size_t)blockIdx.x * kFenceThreads * kGroups + threadIdx.x; g0 < groups; g0 += step) {
        Raw8<TH> hr[kGroups];
        Raw8<TO> orw[kGroups];
#pragma unroll
        for (int j = 0; j < kGroups; ++j) {
            const size_t g = g0 + (size_t)kFenceThreads * j;
            if (g < groups) {
                hr[j].load(h + 8 * g);
                orw[j].load(o + 8 * g);
            }
        }
#pragma unroll
        for (int j = 0; j < kGroups; ++j) {
            const size_t g = g0 + (size_t)kFenceThreads * j;
            if (g < groups) {
                float hv[8], ov[8];
                hr[j].unpack(hv);
                orw[j].unpack(ov);
#pragma unroll
                for (int i = 0; i < 8; ++i) hv[i] = gate_h(hv[i], ov[i]);
                store8(h + 8 * g, hv);
            }
        }
    }
}

template <typename TH, typename TO>
cudaError_t launch_fenced(void *h, const void *o, size_t n, cudaStream_t s, int nsm) {
    const size_t groups = n / 8;
    if (groups == 0) return cudaSuccess;
    int dev = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e != cudaSuccess) return e;
    const int smem = per_sm / 2 + 1024;
    auto k = output_gate_fenced_kernel<TH, TO>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    k<<<nsm, kFenceThreads, smem, s>>>(static_cast<TH *>(h), static_cast<const TO *>(o), groups);
    return cudaGetLastError();
}

template <typename TH, typename TO>
cudaError_t launch_typed(void *h, const void *o, size_t n, cudaStream_t s, int per_sm) {
    const size_t groups = n / 8;
    if (groups == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t want = (groups + 255) / 256;
    const size_t cap = (size_t)sms * per_sm;
    const int blocks = (int)(want < cap ? want : cap);
    output_gate_kernel<TH, TO><<<blocks, 256, 0, s>>>(static_cast<TH *>(h), static_cast<const TO *>(o), groups);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_output_gate(const OutStage &os, void *h, size_t n, cudaStream_t s) {
    if (!os.o || n % 8) return cudaErrorInvalidValue;
    if (os.h_bf16)
        return os.o_bf16 ? launch_typed<__nv_bfloat16, __nv_bfloat16>(h, os.o, n, s, 8)
                         : launch_typed<__nv_bfloat16, float>(h, os.o, n, s, 8);
    return os.o_bf16 ? launch_typed<float, __nv_bfloat16>(h, os.o, n, s, 8) : launch_typed<float, float>(h, os.o, n, s, 8);
}

cudaError_t launch_output_gate_on_sms(const OutStage &os, void *h, size_t n, cudaStream_t s, int nsm) {
    if (!os.o || n % 8 || nsm < 1) return cudaErrorInvalidValue;
    if (os.h_bf16)
        return os.o_bf16 ? launch_fenced<__nv_bfloat16, __nv_bfloat16>(h, os.o, n, s, nsm)
                         : launch_fenced<__nv_bfloat16, float>(h, os.o, n, s, nsm);
    return os.o_bf16 ? launch_fenced<float, __nv_bfloat16>(h, os.o, n, s, nsm)
                     : launch_fenced<float, float>(h, os.o, n, s, nsm);
}

}  // namespace xlstm
