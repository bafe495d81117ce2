// placeholder until the tensor-core kernel lands
#include "h2o_internal.cuh"
namespace h2o {
bool attn_umma_supported(int, int) { return false; }
cudaError_t launch_attn_umma(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace h2o
