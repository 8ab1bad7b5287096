// The GQA layer core's parts around the recurrence: the output norm and swish(z) gate (forward for
// the CUDA-core form, whose chunk kernels split a row's columns over CTAs; the tensor-core forward
// fuses them in its epilogue), and the backward of the gate, the norm, and the causal depthwise
// convolution (kernel 4, zero history) + SiLU + L2 norm in front of the recurrence (explainer
// «Architecture et versions hybrides», Figure 1 caption; mkdocs chapter «Gated DeltaNet», «La
// convolution causale», «La porte de sortie», «Le décompte»).  The recurrence's own backward is the
// chunk backward; gdn_layer_core_bwd (gdn_api.cu) chains the pieces.
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

// ---- output norm + gate: one warp per (token, head) row of D values, lane l owns D/32 of them ------
// forward   y = n * wn * swish(z),  n = o * r,  r = (mean_j o_j^2 + eps)^(-1/2)
// backward  dn = dy * wn * swish(z),  dz = dy * n * wn * swish'(z),  dwn += dy * n * swish(z),
//           do = r * (dn - n * mean_j(dn * n))
constexpr int kNormBlocks = 148 * 8;  // 8 warps each: the backward's per-warp partials of dwn
constexpr int kNormWarps = kNormBlocks * 8;

__device__ __forceinline__ float warp_sum_all(float x) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}
__device__ __forceinline__ float norm_weight(const void* w, int f32, int c) {
    return f32 ? static_cast<const float*>(w)[c] : __bfloat162float(static_cast<const __nv_bfloat16*>(w)[c]);
}

template <class T, class TO, int D>
__global__ void __launch_bounds__(256) rmsnorm_gate_fwd_kernel(const float* __restrict__ o, const T* __restrict__ z,
                                                               const void* norm_w, int norm_w_f32, float eps,
                                                               TO* __restrict__ y, long rows) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    float wn[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) wn[i] = norm_weight(norm_w, norm_w_f32, PER * lane + i);
    for (long row = (long)blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += (long)gridDim.x * 8) {
        const long base = row * D + PER * lane;
        float ov[PER], ss = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            ov[i] = o[base + i];
            ss += ov[i] * ov[i];
        }
        const float r = rsqrtf(warp_sum_all(ss) * (1.f / D) + eps);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float zz = to_f32(z[base + i]);
            y[base + i] = from_f32<TO>(ov[i] * r * wn[i] * zz * sigmoid_fast(zz));
        }
    }
}

// With dout_lo (bf16 outputs only), do is stored as hi = bf16(do) and lo = bf16(do - hi).  npart
// receives each warp's partial sums of dwn ([kNormWarps][D]), reduced by sum_partials_kernel.
template <class T, class TO, int D>
__global__ void __launch_bounds__(256) rmsnorm_gate_bwd_kernel(const float* __restrict__ o, const T* __restrict__ z,
                                                               const T* __restrict__ dy, const void* norm_w,
                                                               int norm_w_f32, float eps, TO* __restrict__ dout,
                                                               TO* __restrict__ dout_lo, float* __restrict__ dz,
                                                               float* __restrict__ npart, long rows) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const long gw = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
    float wn[PER], dwn[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        wn[i] = norm_weight(norm_w, norm_w_f32, PER * lane + i);
        dwn[i] = 0.f;
    }
    for (long row = gw; row < rows; row += (long)gridDim.x * 8) {
        const long base = row * D + PER * lane;
        float n[PER], dn[PER], ss = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            n[i] = o[base + i];
            ss += n[i] * n[i];
        }
        const float r = rsqrtf(warp_sum_all(ss) * (1.f / D) + eps);
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            n[i] *= r;
            const float zz = to_f32(z[base + i]), g = to_f32(dy[base + i]);
            const float s = sigmoid_fast(zz), sw = zz * s;
            dn[i] = g * wn[i] * sw;
            dz[base + i] = g * n[i] * wn[i] * (s + zz * s * (1.f - s));
            dwn[i] = fmaf(g * n[i], sw, dwn[i]);
            m += dn[i] * n[i];
        }
        m = warp_sum_all(m) * (1.f / D);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const float d = r * (dn[i] - n[i] * m);
            const TO hi = from_f32<TO>(d);
            dout[base + i] = hi;
            if (dout_lo) dout_lo[base + i] = from_f32<TO>(d - to_f32(hi));
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) npart[gw * D + PER * lane + i] = dwn[i];
}

// out[j] = sum over partials p of part[p][j], one thread per j (a fixed order: deterministic).
__global__ void __launch_bounds__(256) sum_partials_kernel(const float* __restrict__ part, float* __restrict__ out,
                                                          long nj, int np) {
    const long j = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= nj) return;
    float s = 0.f;
    for (int p = 0; p < np; ++p) s += part[(long)p * nj + j];
    out[j] = s;
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

template <class T, int D>
cudaError_t norm_gate_bwd_t(const LayerBwdIO& io, cudaStream_t st) {
    const long rows = (long)io.B * io.T * io.Hv;
    const T* z = static_cast<const T*>(io.z);
    const T* dy = static_cast<const T*>(io.dy);
    cudaError_t e;
    if (io.dout16)
        e = launch_kernel(rmsnorm_gate_bwd_kernel<T, __nv_bfloat16, D>, dim3(kNormBlocks), dim3(256), 0, st,
                          (const float*)io.o, z, dy, io.norm_w, io.norm_w_f32, io.norm_eps, io.dout16, io.dout16_lo,
                          io.dz, io.npart, rows);
    else
        e = launch_kernel(rmsnorm_gate_bwd_kernel<T, float, D>, dim3(kNormBlocks), dim3(256), 0, st,
                          (const float*)io.o, z, dy, io.norm_w, io.norm_w_f32, io.norm_eps, io.dout, (float*)nullptr,
                          io.dz, io.npart, rows);
    if (e != cudaSuccess) return e;
    return launch_kernel(sum_partials_kernel, dim3((unsigned)((D + 255) / 256)), dim3(256), 0, st,
                         (const float*)io.npart, io.dnorm_w, (long)D, kNormWarps);
}

template <class T>
cudaError_t gate_bwd_t(const LayerBwdIO& io, cudaStream_t st) {
    if (io.norm_w) return io.d == 128 ? norm_gate_bwd_t<T, 128>(io, st) : norm_gate_bwd_t<T, 64>(io, st);
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

size_t layer_norm_partials_floats(int d) { return (size_t)kNormWarps * d; }

cudaError_t layer_norm_gate_fwd(const float* o, const void* z, const void* norm_w, int norm_w_f32, float eps,
                                void* y, int y_f32, bool bf16, long rows, int d, cudaStream_t st) {
    const long blocks = (rows + 7) / 8 < kNormBlocks ? (rows + 7) / 8 : kNormBlocks;
    const dim3 grid((unsigned)(blocks > 0 ? blocks : 1));
#define GDN_NG(T, TO, D)                                                                                   \
    return launch_kernel(rmsnorm_gate_fwd_kernel<T, TO, D>, grid, dim3(256), 0, st, o, static_cast<const T*>(z), \
                         norm_w, norm_w_f32, eps, static_cast<TO*>(y), rows)
    if (bf16) {
        if (d == 128) { if (y_f32) GDN_NG(__nv_bfloat16, float, 128); GDN_NG(__nv_bfloat16, __nv_bfloat16, 128); }
        if (y_f32) GDN_NG(__nv_bfloat16, float, 64);
        GDN_NG(__nv_bfloat16, __nv_bfloat16, 64);
    }
    if (d == 128) GDN_NG(float, float, 128);
    GDN_NG(float, float, 64);
#undef GDN_NG
}

size_t layer_bwd_wpart_floats(int B, int T, int Hk, int Hv, int d) {
    return (size_t)B * ((T + kTile - 1) / kTile) * (2 * (size_t)Hk * d + (size_t)Hv * d) * 4;
}

cudaError_t layer_gate_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st) {
    return bf16 ? gate_bwd_t<__nv_bfloat16>(io, st) : gate_bwd_t<float>(io, st);
}

cudaError_t layer_conv_bwd(const LayerBwdIO& io, bool bf16, cudaStream_t st) {
    return bf16 ? conv_bwd_t<__nv_bfloat16>(io, st) : conv_bwd_t<float>(io, st);
}

}  // namespace gdn
