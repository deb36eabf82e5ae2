// Chunkwise forward for callers that cannot allocate device memory.
//
// xlstm_mlstm_fwd_chunkwise needs a small caller-provided workspace (its device
// status block).  Some callers have no way to provide one: a plug-in running
// inside a host framework that owns every device allocation and hands the
// plug-in no allocator, or code on a latency-critical path where calling
// cudaMalloc (which can synchronise the device and can fail) is not allowed.
// This entry point serves them: its scratch is a fixed array in the library's
// own device memory, so the call allocates nothing.
#include <mutex>

#include "common.cuh"

namespace {

// The library's scratch: one status block's worth, with room to spare.  Every
// GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = 4096;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per device.
// (In host code the array's name is only a host-side stand-in; a kernel given
// it would not reach the device array.)
xlstm_status_t scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return XLSTM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return XLSTM_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return XLSTM_OK;
}

}  // namespace

extern "C" xlstm_status_t xlstm_mlstm_fwd_chunkwise_noalloc(
    const xlstm_mlstm_desc_t *desc, const void *q, const void *k, const void *v, const float *i_pre,
    const float *f_pre, const float *C_in, const float *n_in, const float *m_in, float *h_out, float *C_out,
    float *n_out, float *m_out, cudaStream_t stream) {
    if (!desc) return XLSTM_ERR_INVALID_ARG;
    // problems whose scratch need exceeds the fixed array are refused
    if (xlstm_mlstm_workspace_size(desc) > kNoAllocScratchBytes) return XLSTM_ERR_WORKSPACE;
    void *scratch = nullptr;
    const xlstm_status_t st = scratch_address(&scratch);
    if (st != XLSTM_OK) return st;
    // The chunkwise call clears the status block (a stream-ordered memset)
    // before its kernel runs, so nothing from an earlier call leaks in.
    return xlstm_mlstm_fwd_chunkwise(desc, q, k, v, i_pre, f_pre, C_in, n_in, m_in, h_out, C_out, n_out,
                                     m_out, scratch, kNoAllocScratchBytes, stream);
}

extern "C" xlstm_status_t xlstm_mlstm_noalloc_status(int32_t *where, cudaStream_t stream) {
    void *scratch = nullptr;
    const xlstm_status_t st = scratch_address(&scratch);
    if (st != XLSTM_OK) return st;
    return xlstm_mlstm_workspace_status(scratch, where, stream);
}
