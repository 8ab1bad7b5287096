// Launch of the tensor-core chunk forward for one gate form (LG: gates given as logits), with the
// dispatch over the kernel's instantiations.  Each form is compiled in its own translation unit
// (tc_fwd_gates.cu, tc_fwd_logits.cu); tc_fwd.cu builds the tensor maps and parameters.
#pragma once

#include <cuda.h>

#include "launch.h"
#include "tc_chunk_fwd.cuh"

namespace gdn {

template <bool LG>
cudaError_t tc_fwd_dispatch(const CUtensorMap* maps, const tcfwd::Params& p, Flags f, bool split, bool bf16_gates,
                            cudaStream_t st);

#ifdef GDN_TC_FWD_INSTANTIATE
namespace {

template <bool APC, bool GPC, bool GATE, class TG, bool SPLIT, bool LG>
cudaError_t launch_tc(const CUtensorMap* maps, const tcfwd::Params& p, cudaStream_t st) {
    auto kernel = tcfwd::chunk_fwd_kernel<APC, GPC, GATE, TG, SPLIT, LG>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tcfwd::kSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<p.pb.B * p.pb.Hv, tcfwd::kThreads, tcfwd::kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                        maps[4], maps[5], maps[6], p);
    count_launch();
    return cudaGetLastError();
}

template <bool APC, bool GPC, class TG, bool LG>
cudaError_t launch_tc_g(bool gate, const CUtensorMap* maps, const tcfwd::Params& p, cudaStream_t st) {
    return gate ? launch_tc<APC, GPC, true, TG, false, LG>(maps, p, st)
                : launch_tc<APC, GPC, false, TG, false, LG>(maps, p, st);
}

}  // namespace

template <bool LG>
cudaError_t tc_fwd_dispatch(const CUtensorMap* maps, const tcfwd::Params& p, Flags f, bool split, bool bf16_gates,
                            cudaStream_t st) {
    const bool gate = f.gate;
    if (split) {
        // the layer core's form (scalar gates): with the swish output gate (its forward), or
        // without it (the raw o and the chunk states for its backward)
        if (gate)
            return bf16_gates ? launch_tc<false, false, true, __nv_bfloat16, true, LG>(maps, p, st)
                              : launch_tc<false, false, true, float, true, LG>(maps, p, st);
        return bf16_gates ? launch_tc<false, false, false, __nv_bfloat16, true, LG>(maps, p, st)
                          : launch_tc<false, false, false, float, true, LG>(maps, p, st);
    }
    if (f.apc && f.gpc) return launch_tc_g<true, true, __nv_bfloat16, LG>(gate, maps, p, st);
    if (f.apc) return launch_tc_g<true, false, __nv_bfloat16, LG>(gate, maps, p, st);
    if (f.gpc) return launch_tc_g<false, true, __nv_bfloat16, LG>(gate, maps, p, st);
    if (bf16_gates) return launch_tc_g<false, false, __nv_bfloat16, LG>(gate, maps, p, st);
    return launch_tc_g<false, false, float, LG>(gate, maps, p, st);
}
#endif  // GDN_TC_FWD_INSTANTIATE

}  // namespace gdn
