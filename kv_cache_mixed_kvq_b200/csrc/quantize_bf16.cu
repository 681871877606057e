// Quantize-append instances for bf16 inputs.
#include "quantize.cuh"

namespace kvq {
cudaError_t launch_quantize_bf16(const QuantizeArgs& a, cudaStream_t stream) {
  return launch_quantize_typed<__nv_bfloat16>(a, stream);
}
}  // namespace kvq
