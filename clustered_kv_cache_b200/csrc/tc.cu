// Tensor-core kernels (tcgen05 + TMEM + TMA) of the bf16 / head_dim 128 hot path.
#include "tc.h"

namespace kvc {

// First error recorded by a bounded device-side wait (0 = none).
__device__ unsigned int g_device_error = 0;

cudaError_t tc_read_and_clear_error(unsigned int* value) {
  cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  const unsigned int zero = 0;
  return *value ? cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) : cudaSuccess;
}

bool tc_codec_supported(const kvc_layer_desc*, const kvc_predictor*) { return false; }
size_t tc_workspace(int, const kvc_layer_desc*, const kvc_predictor*, int64_t) { return 0; }
cudaError_t tc_codec_layer(const kvc_layer_desc*, const kvc_predictor*, bool, const void*, const void*, const void*,
                           const void*, const kvc_codes*, void*, void*, void*, size_t, cudaStream_t) {
  return cudaErrorNotSupported;
}
bool tc_attend_supported(const kvc_layer_desc*, const kvc_predictor*, int64_t) { return false; }
cudaError_t tc_attend(const kvc_layer_desc*, const kvc_predictor*, const void*, int64_t, const kvc_codes*, const void*,
                      const void*, const void*, const void*, int64_t, float, void*, void*, size_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kvc
