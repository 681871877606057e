// Quantize-append launcher: picks the instance for the input type.
#include "internal.h"

namespace kvq {
cudaError_t launch_quantize_bf16(const QuantizeArgs& a, cudaStream_t stream);
cudaError_t launch_quantize_f16(const QuantizeArgs& a, cudaStream_t stream);
cudaError_t launch_quantize_f32(const QuantizeArgs& a, cudaStream_t stream);

cudaError_t launch_quantize_append(const QuantizeArgs& a, cudaStream_t stream) {
  switch (a.in_dtype) {
    case KVQ_F32: return launch_quantize_f32(a, stream);
    case KVQ_BF16: return launch_quantize_bf16(a, stream);
    default: return launch_quantize_f16(a, stream);
  }
}
}  // namespace kvq
