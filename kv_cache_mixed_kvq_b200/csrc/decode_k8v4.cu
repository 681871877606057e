// Decode kernel instances for keys at 8 bits and values at 4 bits.
#include "decode.cuh"

namespace kvq {
bool get_decode_kernel_k8v4_paged(int head_dim, int groups_k, int groups_v, int variant,
                                  DecodeKernel* out);

// variant bit 2: the paged layout's instances (decode_k8v4_paged.cu)
bool get_decode_kernel_k8v4(int head_dim, int groups_k, int groups_v, int variant,
                            DecodeKernel* out) {
  if (variant & 4) return get_decode_kernel_k8v4_paged(head_dim, groups_k, groups_v, variant & 3, out);
  return get_decode_kernel_bits<8, 4, false>(head_dim, groups_k, groups_v, variant, out);
}
}  // namespace kvq
