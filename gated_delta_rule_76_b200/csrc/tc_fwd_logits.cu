// Instantiations of the tensor-core chunk forward for gates given as logits.
#define GDN_TC_FWD_INSTANTIATE
#include "tc_fwd_launch.cuh"

namespace gdn {
template cudaError_t tc_fwd_dispatch<true>(const CUtensorMap*, const tcfwd::Params&, Flags, bool, bool, cudaStream_t);
}  // namespace gdn
