// Tensor-memory decode kernel instances for keys at 4 bits and values at 8 bits.
#include "decode_tc.cuh"

namespace kvq {
bool get_decode_tc_kernel_k4v8(int groups_k, int groups_v, int heads_per_cta,
                                 DecodeKernel* out) {
  return get_decode_tc_kernel_bits<4, 8>(groups_k, groups_v, heads_per_cta, out);
}
}  // namespace kvq
