// Instantiations of the tensor-core chunk backward for gates given as logits.
#define GDN_TC_BWD_INSTANTIATE
#include "tc_bwd_launch.cuh"

namespace gdn {
template cudaError_t tc_bwd_dispatch<true>(const CUtensorMap*, const tcbwd::scan::Params&, const CUtensorMap*,
                                          const tcbwd::grad::Params&, Flags, bool, bool, cudaStream_t);
}  // namespace gdn
