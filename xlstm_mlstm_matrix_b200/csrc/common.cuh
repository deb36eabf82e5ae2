// Internal declarations shared by the kernels of the mLSTM library (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/xlstm_mlstm.h"

namespace xlstm {

// Output stage (xLSTM page, "mLSTM (matrix LSTM)" eq. 3 and the o_t line of its
// listing): h = sigmoid(o~) h~ when output-gate pre-activations are given, with
// h stored as fp32 or bf16.  The chunkwise kernels apply it in their epilogue.
struct OutStage {
    const void *o = nullptr;   // [B][H][T][d_v] pre-activations o~, or null (h = h~)
    int o_bf16 = 0, h_bf16 = 0;
};

// Everything one forward launch needs, already validated by the C ABI layer.
struct FwdArgs {
    int B, H, T, dqk, dv;
    int dtype;          // xlstm_dtype_t
    float scale;        // qk_scale
    int chunk;          // L (chunkwise only)
    const void *q, *k, *v;
    const float *ig, *fg;
    const float *C0, *n0, *m0;   // all null = zero state
    float *h, *C1, *n1, *m1;     // state outs may be null
    int32_t *status;             // device status block (4 x int32), may be null
    void *seg_ws;                // scratch for the segment-parallel chunkwise path (null: sequential)
    OutStage out;                // chunkwise only; h points to bf16 elements when out.h_bf16
};

// How a long sequence is cut into segments that run in parallel (nseg = 1: not
// cut), and where the segment summaries sit in the scratch (byte offsets).
// seg_chunks counts chunks of kSegChunk tokens, a multiple of the call's chunk length.
constexpr int kSegChunk = 64;
struct SegPlan {
    int nseg = 1, seg_chunks = 0;
    size_t off_S = 0, off_M = 0, off_N = 0, off_C = 0, bytes = 0;
};
SegPlan segment_plan(const FwdArgs &a);
// Summaries of segments 0 .. nseg-2 and the entry states of segments 1 .. nseg-1.
cudaError_t launch_segment_entry_states(const FwdArgs &a, const SegPlan &sp, cudaStream_t s);
// Summary of a whole sequence (T a multiple of 64, at most 65536 tokens): the state it
// leaves from a zero state with the stabilizer at -inf, and (F, m_seg) per (b, h).
bool summary_supported(const FwdArgs &a);
cudaError_t launch_summary(const FwdArgs &a, float *C_seg, float *n_seg, double *F_m, cudaStream_t s);
// The state after nsum summaries [nsum][B*H] chained onto (C0, n0, m0) (null: zero state).
cudaError_t launch_combine(int BH, int dv, int dqk, int nsum, const float *C0, const float *n0, const float *m0,
                           const float *segC, const float *segN, const double *segS, float *C1, float *n1, float *m1,
                           cudaStream_t s);

// Everything one backward launch needs (validated by the C ABI layer).
struct BwdArgs {
    int B, H, T, dqk, dv, dtype;
    float scale;
    const void *q, *k, *v;
    const float *ig, *fg, *C0, *n0, *m0;   // forward inputs (null state: zero, m = 0)
    const float *dh, *dCT, *dnT;           // upstream gradients (dCT, dnT may be null)
    float *dq, *dk, *dv_, *di, *df;        // gradients of the inputs (fp32)
    float *dC0, *dn0, *dm0;                // gradients of the initial state (each may be null)
    void *workspace;                       // backward_workspace_bytes(...)
};
size_t backward_workspace_bytes(int BH, int T, int dqk, int dv);
cudaError_t launch_backward(const BwdArgs &a, cudaStream_t s);

// Device status block layout (first 16 bytes of the workspace).
enum : int32_t { kStatusCode = 0, kStatusWhere = 1 };

cudaError_t launch_step(const FwdArgs &a, cudaStream_t s);
cudaError_t launch_recurrent(const FwdArgs &a, cudaStream_t s);
cudaError_t launch_chunkwise_simt(const FwdArgs &a, cudaStream_t s);
bool chunkwise_tc_shape_ok(const FwdArgs &a);     // shapes the tensor-core kernel takes
bool chunkwise_tc_supported(const FwdArgs &a);    // ... and the driver's TMA encoder is available
cudaError_t launch_chunkwise_tc(const FwdArgs &a, cudaStream_t s);
// h <- sigmoid(o~) h~ over n elements in place (h in the output stage's dtype).
int sm_count();   // SMs of the current device (first call's device; 148 if the query fails)
// The output gate over n elements of h~ in place (n a multiple of 8, 16-byte aligned
// pointers): a grid-strided streaming pass over every SM; _on_sms: on nsm SMs only,
// one block each that no other block shares, beside a kernel that holds the rest.
cudaError_t launch_output_gate(const OutStage &os, void *h, size_t n, cudaStream_t s);
cudaError_t launch_output_gate_on_sms(const OutStage &os, void *h, size_t n, cudaStream_t s, int nsm);
void set_chunkwise_tc_fault(int mode);   // test hook: applies to the next launch only

// ---- small device helpers ------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Element e of o~ (read-only path).
__device__ __forceinline__ float load_o(const OutStage &os, size_t e) {
    return os.o_bf16 ? __bfloat162float(__ldg(static_cast<const __nv_bfloat16 *>(os.o) + e))
                     : __ldg(static_cast<const float *>(os.o) + e);
}
// sigmoid(o~) h~, formed as h~ / (1 + e^{-o~}): o~ -> -inf gives a signed zero.
__device__ __forceinline__ float gate_h(float h_tilde, float o) { return h_tilde / (1.f + expf(-o)); }
__device__ __forceinline__ void put_h(const OutStage &os, void *h, size_t e, float val) {
    if (os.h_bf16)
        static_cast<__nv_bfloat16 *>(h)[e] = __float2bfloat16_rn(val);
    else
        static_cast<float *>(h)[e] = val;
}
// Element e of h (the same flat index into o~): h~ through the output stage.
__device__ __forceinline__ void store_h(const OutStage &os, void *h, size_t e, float h_tilde) {
    put_h(os, h, e, os.o ? gate_h(h_tilde, load_o(os, e)) : h_tilde);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Stabilized gates of one step: m' = max(f~ + m, i~), f' = e^{f~+m-m'}, i' = e^{i~-m'}.
__device__ __forceinline__ void stabilized_gates(float fg, float ig, float m, float &m_new,
                                                 float &fp, float &ip) {
    const float a = fg + m;
    m_new = (a > ig) ? a : ig;
    fp = expf(a - m_new);
    ip = expf(ig - m_new);
}

}  // namespace xlstm
