// Decode kernel instances for the paged layout, keys at 8 bits and values
// at 8 bits.
#include "decode.cuh"

namespace kvq {
bool get_decode_kernel_k8v8_paged(int head_dim, int groups_k, int groups_v, int variant,
                                  DecodeKernel* out) {
  return get_decode_kernel_bits<8, 8, true>(head_dim, groups_k, groups_v, variant, out);
}
}  // namespace kvq
