// Tensor-memory decode kernel instances for keys at 8 bits and values at 4 bits.
#include "decode_tc.cuh"

namespace kvq {
bool get_decode_tc_kernel_k8v4(int groups_k, int groups_v, int heads_per_cta,
                                 DecodeKernel* out) {
  return get_decode_tc_kernel_bits<8, 4>(groups_k, groups_v, heads_per_cta, out);
}
}  // namespace kvq
