// Quantize-append instances for f32 inputs.
#include "quantize.cuh"

namespace kvq {
cudaError_t launch_quantize_f32(const QuantizeArgs& a, cudaStream_t stream) {
  return launch_quantize_typed<float>(a, stream);
}
}  // namespace kvq
