// Templated launchers, instantiated once per (tensor dtype, gate dtype) in inst_*.cu.
#pragma once
#include <type_traits>

#include "launch.h"

namespace gdn {

template <class K, class... Args>
cudaError_t launch_kernel(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args... args) {
    if (grid.x == 0 || grid.y == 0 || grid.z == 0) return cudaSuccess;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    kernel<<<grid, block, smem, st>>>(args...);
    count_launch();
    return cudaGetLastError();
}

// dq or dk of the key heads from the per-value-head partials [B,T,Hv,dk] (gqa_reduce_kernel).
// out_bf16: the sums are written in bf16 (else fp32).
inline cudaError_t gqa_reduce(const Problem& pb, const float* part, void* out, bool out_bf16, cudaStream_t st) {
    const long rows = (long)pb.B * pb.T;
    const int blocks = (int)(rows < 148L * 8 ? rows : 148L * 8);
    const size_t smem = (size_t)(pb.Hv + pb.Hk + 1) * sizeof(int);
    if (out_bf16)
        return launch_kernel(gqa_reduce_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), smem, st, pb, part,
                             static_cast<__nv_bfloat16*>(out));
    return launch_kernel(gqa_reduce_kernel<float>, dim3(blocks), dim3(256), smem, st, pb, part,
                         static_cast<float*>(out));
}

#define GDN_TRY(expr)                         \
    do {                                      \
        cudaError_t e_ = (expr);              \
        if (e_ != cudaSuccess) return e_;     \
    } while (0)

template <class TIn, class TG, bool APC, bool GPC, int DK>
cudaError_t chunk_fwd_t(const Problem& pb, const ChunkIO& io, const ChunkWs& ws, bool gate,
                        bool save_states, bool write_out, cudaStream_t st) {
    const dim3 block(kSimtThreads);
    GDN_TRY(launch_kernel(chunk_prep_kernel<TIn, TG, APC, GPC, DK>, dim3(pb.NT, pb.Hv, pb.B),
                          block, chunk_prep_smem<DK>(), st, pb, io, ws, save_states ? 1 : 0));
    const dim3 sgrid(pb.dv / kDvTileFwd, pb.Hv, pb.B);
    if (gate)
        GDN_TRY(launch_kernel(chunk_scan_fwd_kernel<TIn, TG, GPC, DK, true>, sgrid, block,
                              chunk_scan_fwd_smem<DK>(), st, pb, io, ws, write_out ? 1 : 0,
                              save_states ? 1 : 0));
    else
        GDN_TRY(launch_kernel(chunk_scan_fwd_kernel<TIn, TG, GPC, DK, false>, sgrid, block,
                              chunk_scan_fwd_smem<DK>(), st, pb, io, ws, write_out ? 1 : 0,
                              save_states ? 1 : 0));
    // pairs whose decay left the factors' range (marked by prep): their outputs again, exactly
    if (!ws.flags || (!write_out && !io.ht)) return cudaSuccess;
    return seq_fwd(pb, io, Flags{APC, GPC, gate}, std::is_same<TIn, float>::value, std::is_same<TG, float>::value,
                   ws.flags, nullptr, st);
}

template <class TIn, class TG, bool APC, bool GPC, int DK>
cudaError_t chunk_bwd_t(const Problem& pb, const ChunkIO& io, const ChunkWs& ws, bool direct_qk,
                        bool paired, cudaStream_t st) {
    const dim3 block(kSimtThreads);
    if (!paired) GDN_TRY((chunk_fwd_t<TIn, TG, APC, GPC, DK>(pb, io, ws, false, true, false, st)));
    GDN_TRY(launch_kernel(chunk_scan_bwd_kernel<TIn, TG, GPC, DK>, dim3(pb.dv / kDvTile, pb.Hv, pb.B),
                          block, chunk_scan_bwd_smem<DK>(), st, pb, io, ws));
    GDN_TRY(launch_kernel(chunk_grad_kernel<TIn, TG, APC, GPC, DK, DK>, dim3(pb.NT, pb.Hv, pb.B),
                          block, chunk_grad_smem<DK, DK>(), st, pb, io, ws, direct_qk ? 1 : 0));
    // pairs whose decay left the factors' range (marked by prep): every gradient again, exactly;
    // the pair's slice of the chunk-state array holds its checkpoints
    if (ws.flags && ws.sbuf)
        GDN_TRY(seq_bwd(pb, io, Flags{APC, GPC, false}, std::is_same<TIn, float>::value, std::is_same<TG, float>::value,
                        ws.flags, direct_qk ? static_cast<float*>(io.dq) : ws.dq_v,
                        direct_qk ? static_cast<float*>(io.dk) : ws.dk_v, direct_qk, ws.S0,
                        (long)pb.NT * DK * DK, ws.sbuf, st));
    if (!direct_qk) {
        GDN_TRY(gqa_reduce(pb, (const float*)ws.dq_v, io.dq, false, st));
        GDN_TRY(gqa_reduce(pb, (const float*)ws.dk_v, io.dk, false, st));
    }
    return cudaSuccess;
}

// Runtime -> compile-time dispatch over (alpha per channel, gates per channel, head dim).
template <class TIn, class TG, class F>
cudaError_t dispatch_chunk(const Problem& pb, Flags f, F&& fn) {
#define GDN_CASE(APC, GPC, DK)                                                       \
    if (f.apc == APC && f.gpc == GPC && pb.dk == DK)                                 \
        return fn(std::integral_constant<bool, APC>{}, std::integral_constant<bool, GPC>{}, \
                  std::integral_constant<int, DK>{});
    GDN_CASE(true, true, 128) GDN_CASE(true, false, 128) GDN_CASE(false, true, 128)
    GDN_CASE(false, false, 128) GDN_CASE(true, true, 64) GDN_CASE(true, false, 64)
    GDN_CASE(false, true, 64) GDN_CASE(false, false, 64)
#undef GDN_CASE
    return cudaErrorInvalidValue;
}

template <class TIn, class TG>
cudaError_t chunk_fwd_impl(const Problem& pb, const ChunkIO& io, const ChunkWs& ws, Flags f,
                           cudaStream_t st) {
    return dispatch_chunk<TIn, TG>(pb, f, [&](auto apc, auto gpc, auto dk) {
        return chunk_fwd_t<TIn, TG, decltype(apc)::value, decltype(gpc)::value, decltype(dk)::value>(
            pb, io, ws, f.gate, f.paired, io.o != nullptr, st);
    });
}

template <class TIn, class TG>
cudaError_t chunk_bwd_impl(const Problem& pb, const ChunkIO& io, const ChunkWs& ws, Flags f,
                           bool direct_qk, cudaStream_t st) {
    return dispatch_chunk<TIn, TG>(pb, f, [&](auto apc, auto gpc, auto dk) {
        return chunk_bwd_t<TIn, TG, decltype(apc)::value, decltype(gpc)::value, decltype(dk)::value>(
            pb, io, ws, direct_qk, f.paired, st);
    });
}

template <class TIn, class TG>
cudaError_t decode_impl(const DecodeParams& p, Flags f, cudaStream_t st) {
    const bool conv = p.conv_state != nullptr, gate = p.z != nullptr;
    const dim3 grid(p.Hv, p.N), block(256);
#define GDN_DEC(APC, GPC, D, CONV, GATE)                                                         \
    if (f.apc == APC && f.gpc == GPC && p.dk == D && conv == CONV && gate == GATE)              \
        return launch_kernel(decode_step_kernel<TIn, TG, APC, GPC, D, D, CONV, GATE>, grid, block, 0, \
                             st, p);
#define GDN_DEC_D(APC, GPC, CONV, GATE) GDN_DEC(APC, GPC, 128, CONV, GATE) GDN_DEC(APC, GPC, 64, CONV, GATE)
#define GDN_DEC_G(CONV, GATE) GDN_DEC_D(true, true, CONV, GATE) GDN_DEC_D(true, false, CONV, GATE) \
    GDN_DEC_D(false, true, CONV, GATE) GDN_DEC_D(false, false, CONV, GATE)
    GDN_DEC_G(false, false) GDN_DEC_G(false, true) GDN_DEC_G(true, false) GDN_DEC_G(true, true)
#undef GDN_DEC_G
#undef GDN_DEC_D
#undef GDN_DEC
    return cudaErrorInvalidValue;
}

template <class TIn>
cudaError_t decode_conv_shift(const DecodeParams& p, cudaStream_t st) {
    const long total = (long)p.N * (2L * p.Hk * p.dk + (long)p.Hv * p.dv);
    const long blocks = (total + 255) / 256;
    return launch_kernel(conv_state_shift_kernel<TIn>, dim3(static_cast<unsigned>(blocks < 65535 ? blocks : 65535)),
                         dim3(256), 0, st, const_cast<void*>(p.conv_state), p.q, p.k, p.v, p.sq, p.sk,
                         p.sv, p.N, p.Hk, p.Hv, p.dk, p.dv);
}

template <class TIn>
cudaError_t conv_impl(const ConvParams& p, cudaStream_t st) {
    const dim3 grid((unsigned)((p.T + kConvTile - 1) / kConvTile), (unsigned)((2 * p.Hk + p.Hv + 3) / 4), (unsigned)p.B);
    if (p.d == 128 && p.q_lo)
        return launch_kernel(conv_silu_l2_kernel<TIn, __nv_bfloat16, 128, true>, grid, dim3(128), 0, st, p);
    if (p.d == 128) return launch_kernel(conv_silu_l2_kernel<TIn, float, 128>, grid, dim3(128), 0, st, p);
    if (p.d == 64) return launch_kernel(conv_silu_l2_kernel<TIn, float, 64>, grid, dim3(128), 0, st, p);
    return cudaErrorInvalidValue;
}

#define GDN_DEFINE_LAUNCHERS(NAME, TIN, TG)                                                      \
    cudaError_t NAME##_chunk_fwd(const Problem& pb, const ChunkIO& io, const ChunkWs& ws,         \
                                 Flags f, cudaStream_t st) {                                     \
        return chunk_fwd_impl<TIN, TG>(pb, io, ws, f, st);                                       \
    }                                                                                            \
    cudaError_t NAME##_chunk_bwd(const Problem& pb, const ChunkIO& io, const ChunkWs& ws,         \
                                 Flags f, bool direct_qk, cudaStream_t st) {                     \
        return chunk_bwd_impl<TIN, TG>(pb, io, ws, f, direct_qk, st);                            \
    }                                                                                            \
    cudaError_t NAME##_decode(const DecodeParams& p, Flags f, cudaStream_t st) {                 \
        GDN_TRY((decode_impl<TIN, TG>(p, f, st)));                                               \
        if (p.conv_state) return decode_conv_shift<TIN>(p, st);                                  \
        return cudaSuccess;                                                                      \
    }                                                                                            \
    cudaError_t NAME##_conv(const ConvParams& p, cudaStream_t st) { return conv_impl<TIN>(p, st); }

}  // namespace gdn
