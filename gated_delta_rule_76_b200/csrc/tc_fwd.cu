// Host side of the tensor-core chunk forward: TMA descriptors, dispatch, launch.
#include <cuda.h>

#include <type_traits>

#include "launch.h"
#include "tc_chunk_fwd.cuh"

namespace gdn {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B, T, H, 128] bf16, boxes of 64 channels x 1 head x 64 tokens x 1 sequence, 128-byte swizzle.
// Tokens past T are zero-filled by the hardware.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || !base) return false;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool APC, bool GPC, bool GATE, class TG>
cudaError_t launch_tc(const CUtensorMap* maps, const tcfwd::Params& p, cudaStream_t st) {
    auto kernel = tcfwd::chunk_fwd_kernel<APC, GPC, GATE, TG>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tcfwd::kSmemBytes);
    if (e != cudaSuccess) return e;
    kernel<<<p.pb.B * p.pb.Hv, tcfwd::kThreads, tcfwd::kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                        maps[4], maps[5], p);
    count_launch();
    return cudaGetLastError();
}

template <bool APC, bool GPC, class TG>
cudaError_t launch_tc_g(bool gate, const CUtensorMap* maps, const tcfwd::Params& p, cudaStream_t st) {
    return gate ? launch_tc<APC, GPC, true, TG>(maps, p, st) : launch_tc<APC, GPC, false, TG>(maps, p, st);
}

}  // namespace

bool tc_fwd_eligible(const Problem& pb, bool bf16_inputs, bool bf16_gates, Flags f) {
    if (!bf16_inputs || pb.dk != 128 || pb.dv != 128 || pb.T < 1) return false;
    if ((f.apc || f.gpc) && !bf16_gates) return false;  // channel gates are loaded by TMA as bf16 tiles
    return encode_fn() != nullptr;
}

cudaError_t tc_chunk_fwd(const Problem& pb, const ChunkIO& io, Flags f, bool bf16_gates, int* err,
                         cudaStream_t st) {
    CUtensorMap maps[6];
    bool ok = make_map(&maps[0], io.q, pb.B, pb.T, pb.Hk) && make_map(&maps[1], io.k, pb.B, pb.T, pb.Hk) &&
              make_map(&maps[2], io.v, pb.B, pb.T, pb.Hv);
    // Unused maps are copies of a valid one (never dereferenced).
    maps[3] = maps[2];
    maps[4] = maps[2];
    maps[5] = maps[2];
    if (ok && f.apc) ok = make_map(&maps[3], io.alpha, pb.B, pb.T, pb.Hv);
    if (ok && f.gpc) ok = make_map(&maps[4], io.b, pb.B, pb.T, pb.Hv) && make_map(&maps[5], io.w, pb.B, pb.T, pb.Hv);
    if (!ok) return cudaErrorInvalidValue;
    tcfwd::Params p;
    p.pb = pb;
    p.alpha = io.alpha;
    p.b = io.b;
    p.z = io.z;
    p.h0 = io.h0;
    p.o = io.o;
    p.o_type = io.o_type == 1 ? 1 : 0;
    p.ht = io.ht;
    p.err = err;
    const bool gate = f.gate;
    if (f.apc && f.gpc) return launch_tc_g<true, true, __nv_bfloat16>(gate, maps, p, st);
    if (f.apc) return launch_tc_g<true, false, __nv_bfloat16>(gate, maps, p, st);
    if (f.gpc) return launch_tc_g<false, true, __nv_bfloat16>(gate, maps, p, st);
    if (bf16_gates) return launch_tc_g<false, false, __nv_bfloat16>(gate, maps, p, st);
    return launch_tc_g<false, false, float>(gate, maps, p, st);
}

}  // namespace gdn

#ifdef GDN_FWD_TRACE
// Profiling builds only: copy the phase timestamps of CTA 0 of the last forward to the host.
extern "C" __attribute__((visibility("default"))) int gdn_fwd_trace_read(unsigned long long* host) {
    return (int)cudaMemcpyFromSymbol(host, gdn::tcfwd::g_fwd_trace, sizeof(unsigned long long) * 64 * 32);
}
#endif
