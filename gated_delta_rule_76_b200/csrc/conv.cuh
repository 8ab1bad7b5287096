// Layer-core prologue: causal depthwise convolution (kernel 4, no bias, zero history) + SiLU on
// the q, k, v projections, then L2 normalisation of every q and k head row
// (explainer «Architecture et versions hybrides», Figure 1 caption; mkdocs chapter «Gated
// DeltaNet», «La convolution causale»).  One warp per (token, head) row of d = 128 or 64
// channels; conv_w[ch][3] weights the current token, conv_w[ch][0] the token three back.
#pragma once
#include "common.cuh"

namespace gdn {

struct ConvParams {
    const void *xq, *xk, *xv, *conv_w;
    void *q, *k, *v;      // outputs [B,T,Hk,d], [B,T,Hk,d], [B,T,Hv,d] in TOut
    void* conv_state_out; // [B, Cch, 3] or null
    int B, T, Hk, Hv, d;
};

template <class TIn, class TOut, int D>
__global__ void __launch_bounds__(256) conv_silu_l2_kernel(ConvParams p) {
    constexpr int PER = D / 32;  // channels per lane
    const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int rows_per_tok = 2 * p.Hk + p.Hv;
    const long nrows = (long)p.B * p.T * rows_per_tok;
    if (warp >= nrows) return;
    const int hrow = (int)(warp % rows_per_tok);
    const long bt = warp / rows_per_tok;
    const int t = (int)(bt % p.T);
    const TIn* x;
    TOut* out;
    int H, h, ch0;
    bool norm;
    if (hrow < p.Hk) {
        x = static_cast<const TIn*>(p.xq); out = static_cast<TOut*>(p.q); H = p.Hk; h = hrow;
        ch0 = h * D; norm = true;
    } else if (hrow < 2 * p.Hk) {
        x = static_cast<const TIn*>(p.xk); out = static_cast<TOut*>(p.k); H = p.Hk; h = hrow - p.Hk;
        ch0 = p.Hk * D + h * D; norm = true;
    } else {
        x = static_cast<const TIn*>(p.xv); out = static_cast<TOut*>(p.v); H = p.Hv; h = hrow - 2 * p.Hk;
        ch0 = 2 * p.Hk * D + h * D; norm = false;
    }
    const TIn* cw = static_cast<const TIn*>(p.conv_w);
    float y[PER];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        float acc = 0.f;
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
            const int tt = t - 3 + tap;
            if (tt >= 0) acc += to_f32(cw[(ch0 + c) * 4 + tap]) * to_f32(x[((bt - t + tt) * H + h) * D + c]);
        }
        y[i] = acc / (1.0f + __expf(-acc));
        ss += y[i] * y[i];
    }
    float scale = 1.f;
    if (norm) {
#pragma unroll
        for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        scale = rsqrtf(ss + 1e-6f);
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) out[(bt * H + h) * D + lane + 32 * i] = from_f32<TOut>(y[i] * scale);
    // The last three raw inputs of each channel, for a decode that continues this sequence.
    if (p.conv_state_out && t == p.T - 1) {
        const long cch = 2L * p.Hk * D + (long)p.Hv * D;
        const long b = bt / p.T;
        TIn* cs = static_cast<TIn*>(p.conv_state_out);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int c = lane + 32 * i;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int tt = t - 2 + j;
                cs[(b * cch + ch0 + c) * 3 + j] =
                    tt >= 0 ? x[((bt - t + tt) * H + h) * D + c] : from_f32<TIn>(0.f);
            }
        }
    }
}

}  // namespace gdn
