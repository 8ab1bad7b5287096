// Instantiations of the tensor-core chunk backward: gates given as values, fp32 gradients.
#define GDN_TC_BWD_INSTANTIATE
#define GDN_TC_BWD_SCAN
#include "tc_bwd_launch.cuh"

namespace gdn {
template cudaError_t tc_scan_dispatch<false>(const CUtensorMap*, const tcbwd::scan::Params&, Flags,
                                            bool, bool, cudaStream_t);
template cudaError_t tc_grad_dispatch<false, float, float>(const CUtensorMap*, const tcbwd::grad::Params&,
                                                     Flags, bool, bool, cudaStream_t);
}  // namespace gdn

#ifdef GDN_BWD_TRACE
// Profiling builds only: copy the phase timestamps of CTA 0 of the last gradient kernel to the host.
extern "C" __attribute__((visibility("default"))) int gdn_bwd_trace_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, gdn::tcbwd::g_bwd_trace, sizeof(unsigned long long) * 16 * 16);
}
// ... and those of CTA 0 of the last reverse scan.
extern "C" __attribute__((visibility("default"))) int gdn_scan_trace_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, gdn::tcbwd::g_scan_trace, sizeof(unsigned long long) * 64 * 32);
}
#endif
