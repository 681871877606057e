// Decode kernel instances for the paged layout, keys at 4 bits and values
// at 4 bits.
#include "decode.cuh"

namespace kvq {
bool get_decode_kernel_k4v4_paged(int head_dim, int groups_k, int groups_v, int variant,
                                  DecodeKernel* out) {
  return get_decode_kernel_bits<4, 4, true>(head_dim, groups_k, groups_v, variant, out);
}
}  // namespace kvq
