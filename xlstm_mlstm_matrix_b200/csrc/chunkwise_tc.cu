// Tensor-core (tcgen05) chunkwise kernel: not built yet.
#include "common.cuh"
namespace xlstm {
bool chunkwise_tc_supported(const FwdArgs &) { return false; }
cudaError_t launch_chunkwise_tc(const FwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace xlstm
