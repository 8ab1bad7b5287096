// Gates given as logits (Problem::gate_logits): the backward's gradients of the gates turned into
// gradients of their logits, and the gradient of alpha's per-head scale.
//   alpha = exp(-a_h softplus(x)):  d x = d alpha * alpha * (-a_h sigmoid(x)),
//                                   d a_h = sum over tokens (and channels) of d alpha * alpha * (-softplus(x))
//   g = sigmoid(x) (b, w, beta):     d x = d g * g (1 - g)
// (explainer «Architecture et versions hybrides», Figure 1 caption: alpha takes the Mamba-2
// parametrisation; zubnet.ai news item: two sigmoid gates).  The kernels of the recurrence apply the
// forward transforms where they read a gate; these two kernels run after a backward.
#include "launch.h"

namespace gdn {

namespace {

__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

template <class TG>
__device__ __forceinline__ float ldg_f(const TG* p, long i) { return to_f32(__ldg(p + i)); }
__device__ __forceinline__ float ld_f(const float* p, long i) { return p[i]; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p, long i) { return __bfloat162float(p[i]); }

// One block per value head: the sum over batch, tokens and channels, in a fixed order.  GT is the
// gradients' type (fp32, or bf16 for gradients returned in the inputs' dtype); the sums are fp32.
template <class TG, class GT>
__global__ void __launch_bounds__(256) alpha_scale_grad_kernel(const TG* __restrict__ xa, const GT* __restrict__ da,
                                                               const float* __restrict__ a_scale,
                                                               float* __restrict__ dscale, long rows, int Hv, int width) {
    __shared__ float red[256];
    const int hv = blockIdx.x;
    const float a = a_scale[hv];
    float s = 0.f;
    const long n = rows * width;  // rows = B * T (the head's elements)
    for (long i = threadIdx.x; i < n; i += blockDim.x) {
        const long row = i / width, c = i - row * width;
        const long e = (row * Hv + hv) * width + c;
        const float x = ldg_f(xa, e), sp = softplus_f(x);
        s = fmaf(ld_f(da, e) * expf(-a * sp), -sp, s);
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int m = 128; m > 0; m >>= 1) {
        if ((int)threadIdx.x < m) red[threadIdx.x] += red[threadIdx.x + m];
        __syncthreads();
    }
    if (threadIdx.x == 0) dscale[hv] = red[0];
}

// In place: d alpha -> d x_alpha (width = channels of alpha, 1 for a scalar decay).
template <class TG, class GT>
__global__ void __launch_bounds__(256) alpha_logit_grad_kernel(const TG* __restrict__ xa, GT* __restrict__ da,
                                                               const float* __restrict__ a_scale, long n, int Hv,
                                                               int width) {
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const int hv = (int)((i / width) % Hv);
        const float a = __ldg(a_scale + hv), x = ldg_f(xa, i);
        st_g(da + i, ld_f(da, i) * expf(-a * softplus_f(x)) * (-a * sigmoid_f(x)));
    }
}

// In place: d g -> d x for a sigmoid gate.
template <class TG, class GT>
__global__ void __launch_bounds__(256) sigmoid_logit_grad_kernel(const TG* __restrict__ xg, GT* __restrict__ dg,
                                                                 long n) {
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const float g = sigmoid_f(ldg_f(xg, i));
        st_g(dg + i, ld_f(dg, i) * g * (1.f - g));
    }
}

unsigned grid_for(long n) {
    const long b = (n + 255) / 256;
    return (unsigned)(b < 148L * 16 ? (b > 0 ? b : 1) : 148L * 16);
}

template <class TG, class GT>
cudaError_t logit_grads_t(const Problem& pb, Flags f, const void* xa, const void* xb, const void* xw, GT* dalpha,
                          GT* db, GT* dw, float* dscale, cudaStream_t st) {
    const long rows = (long)pb.B * pb.T;
    const int wa = f.apc ? pb.dk : 1, wb = f.gpc ? pb.dk : 1;
    const TG* a = static_cast<const TG*>(xa);
    if (dscale) {
        alpha_scale_grad_kernel<TG, GT><<<pb.Hv, 256, 0, st>>>(a, dalpha, pb.alpha_scale, dscale, rows, pb.Hv, wa);
        count_launch();
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const long na = rows * pb.Hv * wa, nb = rows * pb.Hv * wb, nw = rows * pb.Hv * pb.dv;
    alpha_logit_grad_kernel<TG, GT><<<grid_for(na), 256, 0, st>>>(a, dalpha, pb.alpha_scale, na, pb.Hv, wa);
    count_launch();
    sigmoid_logit_grad_kernel<TG, GT><<<grid_for(nb), 256, 0, st>>>(static_cast<const TG*>(xb), db, nb);
    count_launch();
    if (f.gpc) {
        sigmoid_logit_grad_kernel<TG, GT><<<grid_for(nw), 256, 0, st>>>(static_cast<const TG*>(xw), dw, nw);
        count_launch();
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t gate_logit_grads(const Problem& pb, Flags f, bool tg_f32, const void* x_alpha, const void* x_b,
                             const void* x_w, void* dalpha, void* db, void* dw, bool grad_bf16, float* dalpha_scale,
                             cudaStream_t st) {
    if (grad_bf16) {
        using G = __nv_bfloat16;
        auto* a = static_cast<G*>(dalpha);
        auto* b = static_cast<G*>(db);
        auto* w = static_cast<G*>(dw);
        return tg_f32 ? logit_grads_t<float, G>(pb, f, x_alpha, x_b, x_w, a, b, w, dalpha_scale, st)
                      : logit_grads_t<__nv_bfloat16, G>(pb, f, x_alpha, x_b, x_w, a, b, w, dalpha_scale, st);
    }
    auto* a = static_cast<float*>(dalpha);
    auto* b = static_cast<float*>(db);
    auto* w = static_cast<float*>(dw);
    return tg_f32 ? logit_grads_t<float, float>(pb, f, x_alpha, x_b, x_w, a, b, w, dalpha_scale, st)
                  : logit_grads_t<__nv_bfloat16, float>(pb, f, x_alpha, x_b, x_w, a, b, w, dalpha_scale, st);
}

}  // namespace gdn
