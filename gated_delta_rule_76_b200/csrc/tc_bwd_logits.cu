// Instantiations of the tensor-core chunk backward: gates given as logits, fp32 gradients.
#define GDN_TC_BWD_INSTANTIATE
#define GDN_TC_BWD_SCAN
#include "tc_bwd_launch.cuh"

namespace gdn {
template cudaError_t tc_scan_dispatch<true>(const CUtensorMap*, const tcbwd::scan::Params&, Flags,
                                            bool, bool, cudaStream_t);
template cudaError_t tc_grad_dispatch<true, float, float>(const CUtensorMap*, const tcbwd::grad::Params&,
                                                     Flags, bool, bool, cudaStream_t);
}  // namespace gdn
