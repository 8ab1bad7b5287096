// Shared device helpers of the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

constexpr int kChunk = 64;  // chunk length of the chunkwise form (64, as the pages' kernels use)

// ---- element conversion ------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Gradient stores: fp32, or bf16 when the gradients are returned in the inputs' dtype (rounded
// once, from the fp32 value).
__device__ __forceinline__ void st_g(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_g(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
// Four consecutive elements (16-byte aligned for fp32, 8-byte aligned for bf16).
__device__ __forceinline__ void st4_g(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void st4_g(__nv_bfloat16* p, float a, float b, float c, float d) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }

// ---- problem description passed to every kernel by value ---------------------------------
struct Problem {
    int B, T, Hk, Hv, dk, dv;
    int NT;         // number of chunks, ceil(T / 64)
    float scale;
    const int32_t* head_map;  // may be null: hv / (Hv / Hk)
    // Gates given as logits x (explainer «Architecture et versions hybrides», Figure 1 caption: alpha
    // takes the Mamba-2 parametrisation; zubnet.ai news item: two sigmoid gates):
    //   alpha = exp(-alpha_scale[hv] softplus(x)),  b, w, beta = sigmoid(x).
    // Every kernel applies the transform where it reads a gate, in fp32.
    int gate_logits;
    const float* alpha_scale;  // [Hv] fp32 (gate_logits only)

    // The transforms with the form chosen at compile time: kernels instantiated for logits (LG)
    // apply them, the others read the gates as stored.  No branch then sits between a gate's load
    // and its use (a branch on a loaded value waits for the load, which serialises the loads of an
    // unrolled loop).
    template <bool LG>
    __device__ __forceinline__ float alpha_t(int hv, float x) const {
        if constexpr (LG) {
            const float sp = fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));  // softplus(x)
            return expf(-__ldg(alpha_scale + hv) * sp);
        } else {
            return x;
        }
    }
    template <bool LG>
    __device__ __forceinline__ float sig_t(float x) const {
        if constexpr (LG) return 1.f / (1.f + expf(-x));
        else return x;
    }
    // Run-time forms, for the kernels not instantiated per form.
    __device__ __forceinline__ float alpha_of(int hv, float x) const {
        return gate_logits ? alpha_t<true>(hv, x) : x;
    }
    __device__ __forceinline__ float sig_of(float x) const { return gate_logits ? sig_t<true>(x) : x; }

    // An explicit map entry outside [0, Hk) breaks the interface's precondition; it is clamped
    // into range so that no kernel reads outside q or k (the result is then unspecified).
    __device__ __forceinline__ int key_head(int hv) const {
        if (!head_map) return hv / (Hv / Hk);
        const int h = __ldg(head_map + hv);
        return h < 0 ? 0 : (h >= Hk ? Hk - 1 : h);
    }
    // Element offsets of one token row in the token-major layouts.
    __device__ __forceinline__ long qk_row(int b, int t, int hk) const {
        return ((long)(b * T + t) * Hk + hk) * dk;
    }
    __device__ __forceinline__ long v_row(int b, int t, int hv) const {
        return ((long)(b * T + t) * Hv + hv) * dv;
    }
    __device__ __forceinline__ long gate_row(int b, int t, int hv, int width) const {
        return ((long)(b * T + t) * Hv + hv) * width;
    }
    __device__ __forceinline__ long state_off(int b, int hv) const {
        return ((long)b * Hv + hv) * dk * dv;
    }
};

// Scalar gate of token t0 + r of value head hv (one value per token), or `fill` for a row r >= L
// past the end of the sequence.  The load itself is unconditional, from the row clamped to the
// last token: a load under a branch is waited for where the branch ends, which would serialise
// the loads of an unrolled loop.
// KIND: 0 the value as stored, 1 a decay alpha, 2 a sigmoid gate; the transforms of gate logits
// are applied when LG is set.
template <int KIND = 0, bool LG = false, class TG>
__device__ __forceinline__ float gate_or(const TG* g, const Problem& pb, int b, int t0, int r, int L, int hv,
                                         float fill) {
    float x = to_f32(__ldg(g + pb.gate_row(b, t0 + (r < L ? r : L - 1), hv, 1)));
    if constexpr (KIND == 1) x = pb.alpha_t<LG>(hv, x);
    else if constexpr (KIND == 2) x = pb.sig_t<LG>(x);
    return r < L ? x : fill;
}

}  // namespace gdn
