// Placeholder until the tcgen05 grouped GEMMs land.
#include "kernels.cuh"
namespace sre {
bool ffn_tc_supported(const FfnArgs&) { return false; }
cudaError_t launch_ffn_tc(const FfnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace sre
