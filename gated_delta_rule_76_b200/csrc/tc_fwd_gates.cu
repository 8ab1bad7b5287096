// Instantiations of the tensor-core chunk forward for gates given as values.
#define GDN_TC_FWD_INSTANTIATE
#include "tc_fwd_launch.cuh"

namespace gdn {
template cudaError_t tc_fwd_dispatch<false>(const CUtensorMap*, const tcfwd::Params&, Flags, bool, bool, cudaStream_t);
}  // namespace gdn

#ifdef GDN_FWD_TRACE
// Profiling builds only: copy the phase timestamps of CTA 0 of the last forward to the host.
extern "C" __attribute__((visibility("default"))) int gdn_fwd_trace_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, gdn::tcfwd::g_fwd_trace, sizeof(unsigned long long) * 64 * 32);
}
#endif
