// Launches of the tensor-core chunk backward's two kernels (reverse state-gradient scan, chunk-parallel
// gradients), with the dispatch over their instantiations: LG, gates given as logits; GT, the
// gradients' type (fp32, or bf16: the inputs' dtype); QT, that of dq and dk (fp32 when they are
// per-value-head partials summed afterwards).  Each (LG, GT) is compiled in its own translation
// unit (tc_bwd_{gates,logits}{,_bf16}.cu); tc_bwd.cu plans the workspace and builds the tensor maps
// and parameters.
#pragma once

#include <cuda.h>

#include "launch.h"
#include "tc_chunk_bwd.cuh"

namespace gdn {

template <bool LG>
cudaError_t tc_scan_dispatch(const CUtensorMap* ms, const tcbwd::scan::Params& sp, Flags f, bool split,
                             bool bf16_gates, cudaStream_t st);
template <bool LG, class GT, class QT>
cudaError_t tc_grad_dispatch(const CUtensorMap* mg, const tcbwd::grad::Params& gp, Flags f, bool split,
                             bool bf16_gates, cudaStream_t st);

#ifdef GDN_TC_BWD_INSTANTIATE
namespace {

template <bool APC, bool GPC, class TG, bool SPLIT, bool LG>
cudaError_t launch_scan(const CUtensorMap* m, const tcbwd::scan::Params& p, cudaStream_t st) {
    auto kernel = tcbwd::scan::chunk_bwd_scan_kernel<APC, GPC, TG, SPLIT, LG>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tcbwd::scan::kSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<p.pb.B * p.pb.Hv, tcbwd::scan::kThreads, tcbwd::scan::kSmemBytes, st>>>(m[0], m[1], m[2], m[3], m[4],
                                                                                    m[5], p);
    count_launch();
    return cudaGetLastError();
}

template <bool APC, bool GPC, class TG, bool SPLIT, bool LG, class GT, class QT>
cudaError_t launch_grad(const CUtensorMap* m, const tcbwd::grad::Params& p, cudaStream_t st) {
    auto kernel = tcbwd::grad::chunk_bwd_grad_kernel<APC, GPC, TG, SPLIT, LG, GT, QT>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tcbwd::grad::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long nch = (long)p.pb.B * p.pb.Hv * p.pb.NT;
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const long grid = nch < nsm ? nch : nsm;  // persistent: one CTA per SM walks the chunks
    kernel<<<(unsigned)grid, tcbwd::grad::kThreads, tcbwd::grad::kSmemBytes, st>>>(m[0], m[1], m[2], m[3], m[4],
                                                                                 m[5], m[6], m[7], m[8], m[9], p);
    count_launch();
    return cudaGetLastError();
}

}  // namespace

#ifdef GDN_TC_BWD_SCAN
template <bool LG>
cudaError_t tc_scan_dispatch(const CUtensorMap* ms, const tcbwd::scan::Params& sp, Flags f, bool split,
                             bool bf16_gates, cudaStream_t st) {
    if (split)
        return bf16_gates ? launch_scan<false, false, __nv_bfloat16, true, LG>(ms, sp, st)
                          : launch_scan<false, false, float, true, LG>(ms, sp, st);
    if (f.apc && f.gpc) return launch_scan<true, true, __nv_bfloat16, false, LG>(ms, sp, st);
    if (f.apc) return launch_scan<true, false, __nv_bfloat16, false, LG>(ms, sp, st);
    if (f.gpc) return launch_scan<false, true, __nv_bfloat16, false, LG>(ms, sp, st);
    if (bf16_gates) return launch_scan<false, false, __nv_bfloat16, false, LG>(ms, sp, st);
    return launch_scan<false, false, float, false, LG>(ms, sp, st);
}
#endif

// The layer core's split form returns fp32 gradients only.
template <bool LG, class GT, class QT>
cudaError_t tc_grad_dispatch(const CUtensorMap* m, const tcbwd::grad::Params& gp, Flags f, bool split,
                             bool bf16_gates, cudaStream_t st) {
    if constexpr (std::is_same<GT, float>::value) {
        if (split)
            return bf16_gates ? launch_grad<false, false, __nv_bfloat16, true, LG, GT, QT>(m, gp, st)
                              : launch_grad<false, false, float, true, LG, GT, QT>(m, gp, st);
    } else {
        if (split) return cudaErrorInvalidValue;
    }
    if (f.apc && f.gpc) return launch_grad<true, true, __nv_bfloat16, false, LG, GT, QT>(m, gp, st);
    if (f.apc) return launch_grad<true, false, __nv_bfloat16, false, LG, GT, QT>(m, gp, st);
    if (f.gpc) return launch_grad<false, true, __nv_bfloat16, false, LG, GT, QT>(m, gp, st);
    if (bf16_gates) return launch_grad<false, false, __nv_bfloat16, false, LG, GT, QT>(m, gp, st);
    return launch_grad<false, false, float, false, LG, GT, QT>(m, gp, st);
}
#endif  // GDN_TC_BWD_INSTANTIATE

}  // namespace gdn
