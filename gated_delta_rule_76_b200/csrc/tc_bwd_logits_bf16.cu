// Instantiations of the tensor-core chunk backward: gates given as logits, bf16 gradients.
#define GDN_TC_BWD_INSTANTIATE
#include "tc_bwd_launch.cuh"

namespace gdn {
template cudaError_t tc_grad_dispatch<true, __nv_bfloat16, __nv_bfloat16>(const CUtensorMap*,
                                                                     const tcbwd::grad::Params&, Flags, bool,
                                                                     bool, cudaStream_t);
template cudaError_t tc_grad_dispatch<true, __nv_bfloat16, float>(const CUtensorMap*,
                                                                     const tcbwd::grad::Params&, Flags, bool,
                                                                     bool, cudaStream_t);
}  // namespace gdn
