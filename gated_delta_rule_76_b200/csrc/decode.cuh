// Single-token decode step: one CTA per (sequence, value head) streams the fp32 state
// [dk x dv] from HBM once, updates it in registers and writes it back once.
//
// Step (Gated DeltaNet-2 summary, «Règle Delta Portée-2»), column j of the state is independent
// of the other columns:
//   Sbar = Diag(alpha) S;  r_j = sum_i e_i Sbar_ij;  S_ij = Sbar_ij + k_i (zw_j - r_j);
//   o_j = scale * sum_i q_i S_ij          (e = b .* k, zw = w .* v)
// Thread layout: DV/4 column quads (16-byte vector loads of a row slice) x row groups; every
// row group is one warp or half a warp reading whole 256/512-byte row segments.
#pragma once
#include "common.cuh"

namespace gdn {

struct DecodeParams {
    const void* q; const void* k; const void* v;
    const void* alpha; const void* b; const void* w;
    float* state; void* o;
    int o_f32;  // o written in fp32 instead of TIn
    const int32_t* head_map;
    const void* conv_state; const void* conv_w; const void* z;
    // elements from one sequence's token to the next (Hk*dk, Hv*dv, ... when dense)
    long sq, sk, sv, sa, sb, sw, sz;
    int N, Hk, Hv, dk, dv;
    float scale;
    int gate_logits;           // gates as logits: alpha = exp(-alpha_scale[hv] softplus(x)), sigmoid b, w
    const float* alpha_scale;  // [Hv] fp32 (gate_logits only)
};

template <class TIn, class TG, bool APC, bool GPC, int DK, int DV, bool CONV, bool GATE>
__global__ void __launch_bounds__(256)
decode_step_kernel(DecodeParams p) {
    constexpr int NTH = 256;
    constexpr int CQ = DV / 4;          // column quads
    constexpr int RG = NTH / CQ;        // row groups
    constexpr int R = DK / RG;          // rows per thread
    static_assert(R >= 1 && DK % RG == 0, "bad decode tiling");

    __shared__ float qs[DK], ks[DK], es[DK], as_[DK], zs[DV];
    __shared__ float red[RG][DV];
    __shared__ float nrm[2];

    const int hv = blockIdx.x, n = blockIdx.y, tid = threadIdx.x;
    // a map entry outside [0, Hk) breaks the precondition: clamped, so no read leaves q or k
    const int hk = p.head_map ? min(max(__ldg(p.head_map + hv), 0), p.Hk - 1) : hv / (p.Hv / p.Hk);
    const TIn* q = static_cast<const TIn*>(p.q) + n * p.sq + hk * DK;
    const TIn* k = static_cast<const TIn*>(p.k) + n * p.sk + hk * DK;
    const TIn* v = static_cast<const TIn*>(p.v) + n * p.sv + hv * DV;
    const TG* al = static_cast<const TG*>(p.alpha) + n * p.sa + hv * (APC ? DK : 1);
    const TG* bg = static_cast<const TG*>(p.b) + n * p.sb + hv * (GPC ? DK : 1);
    const TG* wg = GPC ? static_cast<const TG*>(p.w) + n * p.sw + hv * DV : bg;

    // ---- gates: every load issued first, then (gates as logits) the transforms under one branch,
    // so that no load waits for another (a branch on a loaded value waits for the load) -----
    constexpr int NI = (DK + NTH - 1) / NTH, NJ = (DV + NTH - 1) / NTH;
    float ga[NI], gb[NI], gw[NJ];
#pragma unroll
    for (int u = 0; u < NI; ++u) {
        const int i = tid + u * NTH;
        ga[u] = i < DK ? to_f32(al[APC ? i : 0]) : 0.f;
        gb[u] = i < DK ? to_f32(bg[GPC ? i : 0]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < NJ; ++u) {
        const int j = tid + u * NTH;
        gw[u] = j < DV ? to_f32(wg[GPC ? j : 0]) : 0.f;
    }
    if (p.gate_logits) {  // alpha = exp(-alpha_scale[hv] softplus(x)); b, w = sigmoid(x)
        const float a_h = __ldg(p.alpha_scale + hv);
#pragma unroll
        for (int u = 0; u < NI; ++u) {
            ga[u] = expf(-a_h * (fmaxf(ga[u], 0.f) + log1pf(expf(-fabsf(ga[u])))));
            gb[u] = 1.f / (1.f + expf(-gb[u]));
        }
#pragma unroll
        for (int u = 0; u < NJ; ++u) gw[u] = 1.f / (1.f + expf(-gw[u]));
    }

    // ---- per-token vectors -------------------------------------------------------------
    if (CONV) {
        // Causal conv (kernel 4) over the 3 stored inputs and the new one, then SiLU.
        const int cch = 2 * p.Hk * DK + p.Hv * DV;
        const TIn* cs = static_cast<const TIn*>(p.conv_state) + (long)n * cch * 3;
        const TIn* cw = static_cast<const TIn*>(p.conv_w);
        auto conv = [&](int ch, float x) {
            float acc = to_f32(cw[ch * 4 + 3]) * x;
#pragma unroll
            for (int i = 0; i < 3; ++i) acc += to_f32(cw[ch * 4 + i]) * to_f32(cs[ch * 3 + i]);
            return acc / (1.0f + __expf(-acc));
        };
        for (int i = tid; i < DK; i += NTH) {
            qs[i] = conv(hk * DK + i, to_f32(q[i]));
            ks[i] = conv(p.Hk * DK + hk * DK + i, to_f32(k[i]));
        }
        for (int j = tid; j < DV; j += NTH) zs[j] = conv(2 * p.Hk * DK + hv * DV + j, to_f32(v[j]));
        __syncthreads();
        // L2 normalisation of q and k: x / sqrt(sum x^2 + 1e-6).
        if (tid < 64) {
            const float* src = tid < 32 ? qs : ks;
            float ss = 0.f;
            for (int i = tid & 31; i < DK; i += 32) ss += src[i] * src[i];
#pragma unroll
            for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if ((tid & 31) == 0) nrm[tid >> 5] = rsqrtf(ss + 1e-6f);
        }
        __syncthreads();
        for (int i = tid; i < DK; i += NTH) { qs[i] *= nrm[0]; ks[i] *= nrm[1]; }
        __syncthreads();
    } else {
        for (int i = tid; i < DK; i += NTH) { qs[i] = to_f32(q[i]); ks[i] = to_f32(k[i]); }
        for (int j = tid; j < DV; j += NTH) zs[j] = to_f32(v[j]);
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < NI; ++u) {
        const int i = tid + u * NTH;
        if (i < DK) {
            as_[i] = ga[u];
            es[i] = gb[u] * ks[i];
        }
    }
#pragma unroll
    for (int u = 0; u < NJ; ++u) {
        const int j = tid + u * NTH;
        if (j < DV) zs[j] *= gw[u];
    }
    __syncthreads();

    // ---- state read, decay, erase read-out ---------------------------------------------
    const int cq = tid % CQ, rg = tid / CQ;
    float4* S = reinterpret_cast<float4*>(p.state + ((long)n * p.Hv + hv) * DK * DV);
    float4 s[R];
#pragma unroll
    for (int i = 0; i < R; ++i) s[i] = S[(rg + i * RG) * CQ + cq];
    float4 racc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int r = rg + i * RG;
        const float a = as_[r], e = es[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        racc.x += e * s[i].x; racc.y += e * s[i].y; racc.z += e * s[i].z; racc.w += e * s[i].w;
    }
    reinterpret_cast<float4*>(&red[rg][0])[cq] = racc;
    __syncthreads();
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int g = 0; g < RG; ++g) {
        const float4 t = reinterpret_cast<const float4*>(&red[g][0])[cq];
        u.x += t.x; u.y += t.y; u.z += t.z; u.w += t.w;
    }
    u.x = zs[4 * cq + 0] - u.x; u.y = zs[4 * cq + 1] - u.y;
    u.z = zs[4 * cq + 2] - u.z; u.w = zs[4 * cq + 3] - u.w;
    __syncthreads();  // red is reused below

    // ---- write along k, read out with q, store --------------------------------------------
    float4 oacc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int r = rg + i * RG;
        const float kk = ks[r], qq = qs[r];
        s[i].x += kk * u.x; s[i].y += kk * u.y; s[i].z += kk * u.z; s[i].w += kk * u.w;
        oacc.x += qq * s[i].x; oacc.y += qq * s[i].y; oacc.z += qq * s[i].z; oacc.w += qq * s[i].w;
        S[r * CQ + cq] = s[i];
    }
    reinterpret_cast<float4*>(&red[rg][0])[cq] = oacc;
    __syncthreads();
    if (rg == 0) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g = 0; g < RG; ++g) {
            const float4 t = reinterpret_cast<const float4*>(&red[g][0])[cq];
            acc.x += t.x; acc.y += t.y; acc.z += t.z; acc.w += t.w;
        }
        float ov[4] = {acc.x * p.scale, acc.y * p.scale, acc.z * p.scale, acc.w * p.scale};
        TIn* o = static_cast<TIn*>(p.o) + ((long)n * p.Hv + hv) * DV + 4 * cq;
        if (GATE) {
            const TIn* zg = static_cast<const TIn*>(p.z) + n * p.sz + hv * DV + 4 * cq;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float zz = to_f32(zg[c]);
                ov[c] *= zz * sigmoidf_(zz);
            }
        }
        if (p.o_f32) {
            *reinterpret_cast<float4*>(static_cast<float*>(p.o) + ((long)n * p.Hv + hv) * DV + 4 * cq) =
                make_float4(ov[0], ov[1], ov[2], ov[3]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) o[c] = from_f32<TIn>(ov[c]);
        }
    }
}

// After the decode kernel: shift every channel's stored inputs and append the new raw input.
template <class TIn>
__global__ void conv_state_shift_kernel(void* conv_state, const void* q, const void* k,
                                        const void* v, long sq, long sk, long sv, int N, int Hk, int Hv, int dk,
                                        int dv) {
    const long cch = 2L * Hk * dk + (long)Hv * dv;
    const long total = (long)N * cch;
    for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total;
         idx += (long)gridDim.x * blockDim.x) {
        const long n = idx / cch, ch = idx % cch;
        TIn x;
        if (ch < (long)Hk * dk) x = static_cast<const TIn*>(q)[n * sq + ch];
        else if (ch < 2L * Hk * dk) x = static_cast<const TIn*>(k)[n * sk + ch - (long)Hk * dk];
        else x = static_cast<const TIn*>(v)[n * sv + ch - 2L * Hk * dk];
        TIn* cs = static_cast<TIn*>(conv_state) + idx * 3;
        cs[0] = cs[1];
        cs[1] = cs[2];
        cs[2] = x;
    }
}

}  // namespace gdn
