// Host side of the exact sequential recurrence (seq.cuh): the pairs the chunk kernels marked in
// their flag array are recomputed token by token after the chunk kernels of the same call.
#include <type_traits>

#include "launch.h"
#include "seq.cuh"

namespace gdn {

namespace {

template <class T>
struct tag {
    using type = T;
};

template <class TIn, class TG, int D>
cudaError_t launch_seq_fwd(const seq::Params& p, cudaStream_t st) {
    auto kernel = seq::seq_fwd_kernel<TIn, TG, D>;
    const size_t smem = seq::seq_fwd_smem<D>();
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<p.pb.B * p.pb.Hv, 2 * D, smem, st>>>(p);
    count_launch();
    return cudaGetLastError();
}

template <class TIn, class TG, int D>
cudaError_t launch_seq_bwd(const seq::Params& p, cudaStream_t st) {
    auto kernel = seq::seq_bwd_kernel<TIn, TG, D>;
    const size_t smem = seq::seq_bwd_smem<D>();
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<p.pb.B * p.pb.Hv, seq::seq_bwd_threads<D>(), smem, st>>>(p);
    count_launch();
    return cudaGetLastError();
}

// Runtime (tensor dtype, gate dtype, head size) -> instantiation.
template <class F>
cudaError_t dispatch(bool tin_f32, bool tg_f32, int d, F&& fn) {
    using bf = __nv_bfloat16;
    if (d != 64 && d != 128) return cudaErrorInvalidValue;
    auto by_d = [&](auto tin, auto tg) {
        return d == 128 ? fn(tin, tg, std::integral_constant<int, 128>{}) : fn(tin, tg, std::integral_constant<int, 64>{});
    };
    if (tin_f32) return tg_f32 ? by_d(tag<float>{}, tag<float>{})
                               : by_d(tag<float>{}, tag<bf>{});
    return tg_f32 ? by_d(tag<bf>{}, tag<float>{})
                  : by_d(tag<bf>{}, tag<bf>{});
}

seq::Params common_params(const Problem& pb, const ChunkIO& io, Flags f, const int* flags) {
    seq::Params p{};
    p.pb = pb;
    p.q = io.q; p.k = io.k; p.v = io.v; p.alpha = io.alpha; p.b = io.b; p.w = io.w;
    p.q_lo = io.q_lo; p.k_lo = io.k_lo; p.v_lo = io.v_lo;
    p.apc = f.apc ? 1 : 0;
    p.gpc = f.gpc ? 1 : 0;
    p.flags = flags;
    p.h0 = io.h0;
    return p;
}

}  // namespace

size_t seq_sbuf_floats(const Problem& pb) { return (size_t)pb.B * pb.Hv * seq::kTB * pb.dk * pb.dv; }

cudaError_t seq_fwd(const Problem& pb, const ChunkIO& io, Flags f, bool tin_f32, bool tg_f32, const int* flags,
                    float* o_raw, cudaStream_t st) {
    seq::Params p = common_params(pb, io, f, flags);
    p.z = f.gate ? io.z : nullptr;
    p.z_bf16 = io.z_bf16;
    p.o = io.o;
    p.o_type = io.o_type;
    p.o_raw = f.gate ? o_raw : nullptr;
    p.norm_w = f.gate ? io.norm_w : nullptr;
    p.norm_w_f32 = io.norm_w_f32;
    p.norm_eps = io.norm_eps;
    p.ht = io.ht;
    return dispatch(tin_f32, tg_f32, pb.dk, [&](auto tin, auto tg, auto d) {
        return launch_seq_fwd<typename decltype(tin)::type, typename decltype(tg)::type, decltype(d)::value>(p, st);
    });
}

cudaError_t seq_bwd(const Problem& pb, const ChunkIO& io, Flags f, bool tin_f32, bool tg_f32, const int* flags,
                    void* dq, void* dk, bool direct, float* ck, long ck_stride, float* sbuf, cudaStream_t st) {
    seq::Params p = common_params(pb, io, f, flags);
    p.dout = io.dout;
    p.dout_lo = io.dout_lo;
    p.dht = io.dht;
    p.dq = dq;
    p.dk = dk;
    p.direct = direct ? 1 : 0;
    p.dv = io.dv;
    p.dalpha = io.dalpha;
    p.db = io.db;
    p.dw = io.dw;
    p.grad_bf16 = io.grad_type == 1 ? 1 : 0;
    p.gate_grad_bf16 = io.grad_type == 1 && !tg_f32 ? 1 : 0;
    p.dh0 = io.dh0;
    p.ck = ck;
    p.ck_stride = ck_stride;
    p.sbuf = sbuf;
    return dispatch(tin_f32, tg_f32, pb.dk, [&](auto tin, auto tg, auto d) {
        return launch_seq_bwd<typename decltype(tin)::type, typename decltype(tg)::type, decltype(d)::value>(p, st);
    });
}

}  // namespace gdn
