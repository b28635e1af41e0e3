// Tensor-core decode kernel (tcgen05 / TMEM / TMA) -- not built yet.
#include "mlra_internal.cuh"

namespace mlra {
bool tc_supported(const mlra_config_t&) { return false; }
void tc_grid(const mlra_config_t&, int num_sms, int* n_groups, int* ctas_per_group) {
  *n_groups = 1;
  *ctas_per_group = num_sms;
}
cudaError_t launch_decode_tc(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mlra
