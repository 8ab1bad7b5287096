// Backward of the GQA layer core's elementwise parts: the swish(z) output gate, and the causal
// depthwise convolution (kernel 4, zero history) + SiLU + L2 norm in front of the recurrence
// (explainer «Architecture et versions hybrides», Figure 1 caption; mkdocs chapter «Gated
// DeltaNet», «La convolution causale», «La porte de sortie»).  The recurrence's own backward is
// the chunk backward; gdn_layer_core_bwd (gdn_api.cu) chains the pieces.
#include <cuda_runtime.h>

#include <type_traits>

#include "launch.cuh"

namespace gdn {

namespace {

__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }

// y = o * z * sigmoid(z):  do = dy * z * sigmoid(z),  dz = dy * o * (s + z s (1 - s)).
// With dout_lo (bf16 outputs only), do is stored as hi = bf16(do) and lo = bf16(do - hi).
template <class T, class TO>
__global__ void __launch_bounds__(256) swish_gate_bwd_kernel(const float* __restrict__ o, const T* __restrict__ z,
                                                             const T* __restrict__ dy, TO* __restrict__ dout,
                                                             TO* __restrict__ dout_lo, float* __restrict__ dz, long n) {
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const float zz = to_f32(z[i]), g = to_f32(dy[i]);
        const float s = sigmoid_fast(zz);
        const float d = g * zz * s;
        const TO hi = from_f32<TO>(d);
        dout[i] = hi;
        if (dout_lo) dout_lo[i] = from_f32<TO>(d - to_f32(hi));
        dz[i] = g * o[i] * (s + zz * s * (1.f - s));
    }
}

constexpr int kTile = 64;  // tokens per warp

// Grid (ceil(T / kTile), ceil((2 Hk + Hv) / 4), B), 4 warps a block; a warp takes one conv row
// (a q, k or v head) over one tile of tokens, lane l owning channels PER l .. PER l + PER - 1.
//   forward, recomputed:  u_t = sum_tap w[tap] x_{t-3+tap},  a_t = u_t sigmoid(u_t),
//                         out_t = a_t / sqrt(|a_t|^2 + eps) (q and k rows; v rows: out_t = a_t)
//   backward:             da = (g - out (out . g)) / n  (or g),  du = da (s + u s (1 - s)),
//                         dx_s = sum_tap w[tap] du_{s+3-tap},  dw[tap] += du_t x_{t-3+tap}.
// dx_s needs du at s .. s + 3, so the warp forms du over its tile and the three tokens after it,
// finishing each dx_s three tokens later; the weight gradient's per-tile partial sums go to
// wpart[b * ntile + tile][channel][tap] (reduced by dconv_reduce_kernel, no atomics).
template <class TIn, int D>
__global__ void __launch_bounds__(128) conv_silu_l2_bwd_kernel(const TIn* __restrict__ xq, const TIn* __restrict__ xk,
                                                               const TIn* __restrict__ xv, const TIn* __restrict__ conv_w,
                                                               const float* __restrict__ gq, const float* __restrict__ gk,
                                                               const float* __restrict__ gv, float* __restrict__ dxq,
                                                               float* __restrict__ dxk, float* __restrict__ dxv,
                                                               float* __restrict__ wpart, int T, int Hk, int Hv) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int hrow = blockIdx.y * 4 + (threadIdx.x >> 5);
    if (hrow >= 2 * Hk + Hv) return;
    const int b = blockIdx.z, tile = blockIdx.x, ntile = gridDim.x;
    const int ta = tile * kTile, tb = min(ta + kTile, T), te = min(tb + 3, T);
    const TIn* x;
    const float* g;
    float* dx;
    int H, h, ch0;
    bool norm;
    if (hrow < Hk) {
        x = xq; g = gq; dx = dxq; H = Hk; h = hrow; ch0 = h * D; norm = true;
    } else if (hrow < 2 * Hk) {
        x = xk; g = gk; dx = dxk; H = Hk; h = hrow - Hk; ch0 = Hk * D + h * D; norm = true;
    } else {
        x = xv; g = gv; dx = dxv; H = Hv; h = hrow - 2 * Hk; ch0 = 2 * Hk * D + h * D; norm = false;
    }
    const int c0 = PER * lane;
    const long stride = (long)H * D;
    const long base = (long)b * T * stride + (long)h * D + c0;
    float wt[PER][4];
#pragma unroll
    for (int i = 0; i < PER; ++i)
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) wt[i][tap] = to_f32(conv_w[(ch0 + c0 + i) * 4 + tap]);
    // xw[j]: input at t - 3 + j (j = 0..3 after loading x_t); acc[j]: dx of token t - 3 + j
    float xw[4][PER], acc[4][PER], dwp[PER][4];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xw[j][i] = 0.f;
            acc[j][i] = 0.f;
            dwp[i][j] = 0.f;
        }
    }
#pragma unroll
    for (int j = 1; j < 4; ++j) {
        const int tt = ta - 4 + j;  // tokens ta-3 .. ta-1 go to slots 1..3, shifted in below
        if (tt >= 0) {
#pragma unroll
            for (int i = 0; i < PER; ++i) xw[j][i] = to_f32(x[base + (long)tt * stride + i]);
        }
    }
    for (int t = ta; t < te; ++t) {
        // shift the windows: slot 0 drops token t - 4 (x) / finishes token t - 4 (dx)
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float fin = acc[0][i];
            if (t - 4 >= ta && t - 4 < tb) dx[base + (long)(t - 4) * stride + i] = fin;
            xw[0][i] = xw[1][i]; xw[1][i] = xw[2][i]; xw[2][i] = xw[3][i];
            xw[3][i] = to_f32(x[base + (long)t * stride + i]);
            acc[0][i] = acc[1][i]; acc[1][i] = acc[2][i]; acc[2][i] = acc[3][i]; acc[3][i] = 0.f;
        }
        float u[PER], s[PER], a[PER], gg[PER];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            float v = 0.f;
            v += wt[i][0] * xw[0][i];
            v += wt[i][1] * xw[1][i];
            v += wt[i][2] * xw[2][i];
            v += wt[i][3] * xw[3][i];
            u[i] = v;
            s[i] = sigmoid_fast(v);
            a[i] = v * s[i];
            ss += a[i] * a[i];
            gg[i] = g[base + (long)t * stride + i];
        }
        float da[PER];
        if (norm) {
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float rn = rsqrtf(ss + 1e-6f);
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) dot += a[i] * rn * gg[i];
#pragma unroll
            for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
#pragma unroll
            for (int i = 0; i < PER; ++i) da[i] = (gg[i] - a[i] * rn * dot) * rn;
        } else {
#pragma unroll
            for (int i = 0; i < PER; ++i) da[i] = gg[i];
        }
        const bool own = t < tb;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float du = da[i] * (s[i] + u[i] * s[i] * (1.f - s[i]));
            // dx_{t-3+tap} += w[tap] du_t  (slot tap holds token t - 3 + tap)
#pragma unroll
            for (int tap = 0; tap < 4; ++tap) acc[tap][i] += wt[i][tap] * du;
            if (own) {
#pragma unroll
                for (int tap = 0; tap < 4; ++tap) dwp[i][tap] += du * xw[tap][i];
            }
        }
    }
    // the window's last tokens te-4 .. te-1 (those inside the tile) are complete
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int tt = te - 4 + j;
        if (tt >= ta && tt < tb) {
#pragma unroll
            for (int i = 0; i < PER; ++i) dx[base + (long)tt * stride + i] = acc[j][i];
        }
    }
    const long cch = 2L * Hk * D + (long)Hv * D;
    float* wp = wpart + ((long)b * ntile + tile) * cch * 4;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        *reinterpret_cast<float4*>(wp + (ch0 + c0 + i) * 4) = make_float4(dwp[i][0], dwp[i][1], dwp[i][2], dwp[i][3]);
    }
}

__global__ void __launch_bounds__(256) accumulate_kernel(float4* __restrict__ dst, const float4* __restrict__ src,
                                                         float* __restrict__ dst1, const float* __restrict__ src1,
                                                         long n4, long n) {
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
        float4 a = dst[i];
        const float4 b = src[i];
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        dst[i] = a;
    }
    // what the float4 body leaves (n % 4 elements, or all of them when the pointers are unaligned)
    for (long t = 4 * n4 + (long)blockIdx.x * blockDim.x + threadIdx.x; t < n; t += (long)gridDim.x * blockDim.x)
        dst1[t] += src1[t];
}

// dconv_w[j] = sum over partials p of wpart[p][j]  (j = channel * 4 + tap), one thread per j.
__global__ void __launch_bounds__(256) dconv_reduce_kernel(const float* __restrict__ wpart, float* __restrict__ dw,
                                                           long nj, int np) {
    const long j = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= nj) return;
    float s = 0.f;
    for (int p = 0; p < np; ++p) s += wpart[(long)p * nj + j];
    dw[j] = s;
}

template <class TIn>
cudaError_t conv_bwd_t(const LayerBwdIO& io, cudaStream_t st) {
    const int ntile = (io.T + kTile - 1) / kTile;
    const dim3 grid((unsigned)ntile, (unsigned)((2 * io.Hk + io.Hv + 3) / 4), (unsigned)io.B);
    const TIn* xq = static_cast<const TIn*>(io.xq);
    const TIn* xk = static_cast<const TIn*>(io.xk);
    const TIn* xv = static_cast<const TIn*>(io.xv);
    const TIn* cw = static_cast<const TIn*>(io.conv_w);
    cudaError_t e;
    if (io.d == 128)
        e = launch_kernel(conv_silu_l2_bwd_kernel<TIn, 128>, grid, dim3(128), 0, st, xq, xk, xv, cw, io.gq, io.gk,
                          io.gv, io.dxq, io.dxk, io.dxv, io.wpart, io.T, io.Hk, io.Hv);
    else if (io.d == 64)
        e = launch_kernel(conv_silu_l2_bwd_kernel<TIn, 64>, grid, dim3(128), 0, st, xq, xk, xv, cw, io.gq, io.gk,
                          io.gv, io.dxq, io.dxk, io.dxv, io.wpart, io.T, io.Hk, io.Hv);
    else
        return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    const long nj = (2L * io.Hk * io.d + (long)io.Hv * io.d) * 4;
    return launch_kernel(dconv_reduce_kernel, dim3((unsigned)((nj + 255) / 256)), dim3(256), 0, st, (const float*)io.wpart,
                         io.dconv_w, nj, io.B * ntile);
}

template <class T>
cudaError_t gate_bwd_t(const LayerBwdIO& io, cudaStream_t st) {
    const long n = (long)io.B * io.T * io.Hv * io.d;
    const long blocks = (n + 255) / 256 < 148L * 32 ? (n + 255) / 256 : 148L * 32;
    if (io.dout16)
        return launch_kernel(swish_gate_bwd_kernel<T, __nv_bfloat16>, dim3((unsigned)blocks), dim3(256), 0, st,
                             (const float*)io.o, static_cast<const T*>(io.z), static_cast<const T*>(io.dy), io.dout16,
                             io.dout16_lo, io.dz, n);
    return launch_kernel(swish_gate_bwd_kernel<T, float>, dim3((unsigned)blocks), dim3(256), 0, st, (const float*)io.o,
                         static_cast<const T*>(io.z), static_cast<const T*>(io.dy), io.dout, (float*)nullptr, io.dz, n);
}

}  // namespace

size_t layer_bwd_wpart_floats(int B, int T, int Hk, int Hv, int d) {
    return (size_t)B * ((T + kTile - 1) / kTile) * (2 * (size_t)Hk * d + (size_t)Hv * d) * 4;
}

cudaError_t layer_gate_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st) {
    return bf16 ? gate_bwd_t<__nv_bfloat16>(io, st) : gate_bwd_t<float>(io, st);
}

cudaError_t layer_conv_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st) {
    return bf16 ? conv_bwd_t<__nv_bfloat16>(io, st) : conv_bwd_t<float>(io, st);
}

cudaError_t layer_accumulate(float* dst, const float* src, long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    // float4 body only when both pointers are 16-byte aligned
    const bool v4 = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15u) == 0;
    const long n4 = v4 ? n / 4 : 0;
    const long work = n4 > n - 4 * n4 ? n4 : n - 4 * n4;
    const long blocks = (work + 255) / 256 < 148L * 16 ? (work + 255) / 256 : 148L * 16;
    return launch_kernel(accumulate_kernel, dim3((unsigned)(blocks > 0 ? blocks : 1)), dim3(256), 0, st,
                         reinterpret_cast<float4*>(dst), reinterpret_cast<const float4*>(src), dst, src, n4, n);
}

}  // namespace gdn
