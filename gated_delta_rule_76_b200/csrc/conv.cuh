// Layer-core prologue: causal depthwise convolution (kernel 4, no bias, zero history) + SiLU on
// the q, k, v projections, then L2 normalisation of every q and k head row
// (explainer «Architecture et versions hybrides», Figure 1 caption; mkdocs chapter «Gated
// DeltaNet», «La convolution causale»).  Rows of d = 128 or 64 channels; conv_w[ch][3] weights
// the current token, conv_w[ch][0] the token three back.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace gdn {

struct ConvParams {
    const void *xq, *xk, *xv, *conv_w;
    void *q, *k, *v;      // outputs [B,T,Hk,d], [B,T,Hk,d], [B,T,Hv,d] in TOut
    // Split outputs (TOut = bf16): the fp32 result x is stored as hi = bf16(x) in q, k, v and
    // lo = bf16(x - hi) here, for the tensor-core forward.
    void *q_lo, *k_lo, *v_lo;
    void* conv_state_out; // [B, Cch, 3] or null
    int B, T, Hk, Hv, d;
};

// PER consecutive channels <-> registers (vector loads and stores of 4 to 16 bytes).
template <int PER>
__device__ __forceinline__ void load_ch(const float* src, float (&x)[PER]) {
    if constexpr (PER == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        x[0] = v.x; x[1] = v.y;
    }
}
template <int PER>
__device__ __forceinline__ void load_ch(const __nv_bfloat16* src, float (&x)[PER]) {
    if constexpr (PER == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(src);
        x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
        x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    } else {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
        x[0] = __uint_as_float(v << 16); x[1] = __uint_as_float(v & 0xFFFF0000u);
    }
}
template <int PER>
__device__ __forceinline__ void store_ch(float* dst, const float (&y)[PER]) {
    if constexpr (PER == 4) *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
    else *reinterpret_cast<float2*>(dst) = make_float2(y[0], y[1]);
}
__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat16 a, __nv_bfloat16 b) {
    return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}
template <int PER>
__device__ __forceinline__ void store_ch(__nv_bfloat16* dst, const __nv_bfloat16 (&y)[PER]) {
    if constexpr (PER == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(bf16x2_bits(y[0], y[1]), bf16x2_bits(y[2], y[3]));
    else *reinterpret_cast<uint32_t*>(dst) = bf16x2_bits(y[0], y[1]);
}

constexpr int kConvTile = 64;  // tokens per warp

// Grid (ceil(T / kConvTile), ceil((2 Hk + Hv) / 4), B), 4 warps a block.  A warp takes one conv
// row (a q, k or v head) over one tile of tokens; lane l owns channels PER l .. PER l + PER - 1 and
// walks the tokens in order with the three previous inputs in registers, so each input is read
// once (plus a three-token lead-in per tile).  The L2 norm of a q / k row is a warp reduction.
template <class TIn, class TOut, int D, bool SPLIT = false>
__global__ void __launch_bounds__(128) conv_silu_l2_kernel(ConvParams p) {
    static_assert(!SPLIT || std::is_same<TOut, __nv_bfloat16>::value, "split outputs are bf16 pairs");
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const int hrow = blockIdx.y * 4 + (threadIdx.x >> 5);
    if (hrow >= 2 * p.Hk + p.Hv) return;
    const int b = blockIdx.z;
    const int ta = blockIdx.x * kConvTile, tb = min(ta + kConvTile, p.T);
    const TIn* x;
    TOut *out, *out_lo;
    int H, h, ch0;
    bool norm;
    if (hrow < p.Hk) {
        x = static_cast<const TIn*>(p.xq); out = static_cast<TOut*>(p.q); out_lo = static_cast<TOut*>(p.q_lo);
        H = p.Hk; h = hrow; ch0 = h * D; norm = true;
    } else if (hrow < 2 * p.Hk) {
        x = static_cast<const TIn*>(p.xk); out = static_cast<TOut*>(p.k); out_lo = static_cast<TOut*>(p.k_lo);
        H = p.Hk; h = hrow - p.Hk; ch0 = p.Hk * D + h * D; norm = true;
    } else {
        x = static_cast<const TIn*>(p.xv); out = static_cast<TOut*>(p.v); out_lo = static_cast<TOut*>(p.v_lo);
        H = p.Hv; h = hrow - 2 * p.Hk; ch0 = 2 * p.Hk * D + h * D; norm = false;
    }
    const int c0 = PER * lane;
    const long stride = (long)H * D;                        // elements between tokens
    const long base = (long)b * p.T * stride + (long)h * D + c0;
    const TIn* cw = static_cast<const TIn*>(p.conv_w);
    float wt[PER][4];
#pragma unroll
    for (int i = 0; i < PER; ++i)
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) wt[i][tap] = to_f32(cw[(ch0 + c0 + i) * 4 + tap]);
    // x3, x2, x1: inputs at t - 3, t - 2, t - 1 (zero before the sequence start)
    float x3[PER], x2[PER], x1[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) x3[i] = x2[i] = x1[i] = 0.f;
    if (ta >= 3) load_ch<PER>(x + base + (long)(ta - 3) * stride, x3);
    if (ta >= 2) load_ch<PER>(x + base + (long)(ta - 2) * stride, x2);
    if (ta >= 1) load_ch<PER>(x + base + (long)(ta - 1) * stride, x1);
#pragma unroll 4
    for (int t = ta; t < tb; ++t) {
        float x0[PER], y[PER];
        load_ch<PER>(x + base + (long)t * stride, x0);
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            float acc = 0.f;
            acc += wt[i][0] * x3[i];
            acc += wt[i][1] * x2[i];
            acc += wt[i][2] * x1[i];
            acc += wt[i][3] * x0[i];
            y[i] = acc * __fdividef(1.0f, 1.0f + __expf(-acc));  // SiLU (fast reciprocal: a few ulp)
            ss += y[i] * y[i];
        }
        float scale = 1.f;
        if (norm) {
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            scale = rsqrtf(ss + 1e-6f);
        }
        const long o = base + (long)t * stride;  // outputs share the inputs' [B,T,H,D] layout
        if constexpr (SPLIT) {
            __nv_bfloat16 hi[PER], lo[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const float r = y[i] * scale;
                hi[i] = __float2bfloat16_rn(r);
                lo[i] = __float2bfloat16_rn(r - __bfloat162float(hi[i]));
            }
            store_ch<PER>(out + o, hi);
            store_ch<PER>(out_lo + o, lo);
        } else {
            float r[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) r[i] = y[i] * scale;
            store_ch<PER>(out + o, r);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            x3[i] = x2[i];
            x2[i] = x1[i];
            x1[i] = x0[i];
        }
    }
    // The last three raw inputs of each channel (zero before the start), for a decode that
    // continues this sequence: the tile that ends the sequence holds them in its window.
    if (p.conv_state_out && tb == p.T) {
        const long cch = 2L * p.Hk * D + (long)p.Hv * D;
        TIn* cs = static_cast<TIn*>(p.conv_state_out);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            TIn* d = cs + ((long)b * cch + ch0 + c0 + i) * 3;
            d[0] = from_f32<TIn>(x3[i]);
            d[1] = from_f32<TIn>(x2[i]);
            d[2] = from_f32<TIn>(x1[i]);
        }
    }
}

}  // namespace gdn
