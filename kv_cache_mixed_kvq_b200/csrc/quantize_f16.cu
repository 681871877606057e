// Quantize-append instances for f16 inputs.
#include "quantize.cuh"

namespace kvq {
cudaError_t launch_quantize_f16(const QuantizeArgs& a, cudaStream_t stream) {
  return launch_quantize_typed<__half>(a, stream);
}
}  // namespace kvq
