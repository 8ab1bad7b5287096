// Exact sequential recurrence on CUDA cores (fp32 state and arithmetic), one CTA per (sequence,
// value head): the path for pairs whose decay leaves the range of the chunk kernels.
//
// The chunk kernels carry the decay inside a chunk of 64 tokens as a ratio Gamma_r / Gamma_s of the
// running product Gamma of alpha (GDN-2 summary, «Entraînement Parallèle Efficace par Blocs»: the
// decay is absorbed into the erase and write factors).  When the product over a chunk falls below
// 2^-100 on some channel, 1/Gamma leaves the fp32 range and the factors overflow.  Every chunk
// kernel checks its chunk's product (decay_out_of_range) and marks the (sequence, head) pair in a
// flag array; the kernels here then recompute the marked pairs token by token from the update
// itself (GDN-2 summary, «Méthodologie» §1):
//     Sbar = Diag(alpha_t) S_{t-1},  r = Sbar^T e_t,  S_t = Sbar + k_t (z_t - r)^T,  o_t = scale S_t^T q_t
// with e = b .* k, z = w .* v, and overwrite the chunk kernels' results for those pairs.  No ratio
// of decays is ever formed, so any alpha in [0, 1] is exact to fp32 rounding.
//
// Forward (seq_fwd_kernel, 2*D threads): thread (j, h) owns value column j of the state and rows
// [h*D/2, h*D/2 + D/2); both reductions of a token (r and o, over the key rows) are in-thread sums
// plus one shuffle between the two halves, so the token loop has no CTA barrier.
// Backward (seq_bwd_kernel, D*D/32 threads): thread (rb, cb) owns an 8 x 4 tile of the state and of
// its gradient.  Sums over value columns (dq, dk, de, dalpha) are warp shuffles; sums over key rows
// (r, dz) go through shared memory.  The reverse sweep needs S_{t-1} and S_t at every token: a first
// forward pass stores the state entering every chunk (checkpoints), then each chunk is recomputed in
// sub-chunks of 16 tokens from its checkpoint, storing the 16 entering states, and swept in reverse.
//
// Inputs are staged 16 tokens at a time into shared memory as fp32 vectors (scalar gates broadcast),
// double-buffered between consecutive blocks.
#pragma once
#include "common.cuh"

namespace gdn {
namespace seq {

constexpr int kTB = 16;                                   // tokens per staged block (= sub-chunk)
constexpr float kMinChunkDecay = 7.888609052210118e-31f;  // 2^-100

// True when a chunk's decay product on one channel is below the range the chunk kernels' factors
// can carry (or is not a number).  The chunk kernels call it on every channel of every chunk.
__device__ __forceinline__ bool decay_out_of_range(float chunk_product) {
    return !(chunk_product >= kMinChunkDecay);
}

struct Params {
    Problem pb;
    const void *q, *k, *v, *alpha, *b, *w;  // the chunk kernels' inputs (TIn / TG)
    const void *q_lo, *k_lo, *v_lo;          // split inputs: bf16 lo halves (q = q + q_lo, ...), or NULL
    int apc, gpc;                            // alpha per channel; b, w per channel (else scalar beta)
    const int* flags;                        // [B*Hv]: only marked pairs run; NULL: every pair
    const float* h0;                         // [B,Hv,dk,dv] or NULL
    // forward
    const void* z;                           // swish output gate [B,T,Hv,dv], or NULL
    int z_bf16;                              // z stored as bf16 (else as TIn)
    void* o;                                 // [B,T,Hv,dv], or NULL
    int o_type;                              // 0: TIn, 1: fp32, 2: bf16
    float* o_raw;                            // with z: the output before the gate (fp32), or NULL
    const void* norm_w;                      // with z: the output norm's weights [dv] (bf16 unless
    int norm_w_f32;                          //   norm_w_f32), or NULL: no norm
    float norm_eps;
    float* ht;                               // [B,Hv,dk,dv] or NULL
    // backward
    const void* dout;                        // [B,T,Hv,dv] TIn
    const void* dout_lo;                     // bf16 lo half of dout (dout = dout + dout_lo), or NULL
    const float* dht;                        // [B,Hv,dk,dv] or NULL
    void *dq, *dk;                           // [B,T,Hk,dk] when direct, else [B,T,Hv,dk] per value head
    int direct;
    void *dv, *dalpha, *db, *dw;             // shapes of v, alpha, b (or beta), w
    int grad_bf16;                           // dv (and dq, dk when direct) in bf16
    int gate_grad_bf16;                      // dalpha, db, dw in bf16
    float* dh0;                              // may be NULL
    float* ck;                               // per pair ck_stride floats: states entering chunks 1..NT-1
    long ck_stride;
    float* sbuf;                             // per pair kTB states (floats kTB * dk * dv)
};

// One gradient element, fp32 or bf16.
__device__ __forceinline__ void put_g(void* p, long i, float v, bool bf) {
    if (bf) st_g(static_cast<__nv_bfloat16*>(p) + i, v);
    else st_g(static_cast<float*>(p) + i, v);
}

// ---- staging of one block of kTB tokens ---------------------------------------------------
// Vectors of a token, in the fp32 staging buffer [kTB][NVEC][D]: alpha, b, k, q, v, w, and the
// output gate z (forward) or the output gradient (backward) in the last slot.
enum Vec { V_A = 0, V_B, V_K, V_Q, V_V, V_W, V_X, NVEC };

template <class TIn, class TG, int D, int NTH>
struct Stager {
    static constexpr int CH = D / 4;                      // 4-element chunks of one vector
    static constexpr int NCHUNK = kTB * NVEC * CH;        // chunks of a block
    static constexpr int PER = (NCHUNK + NTH - 1) / NTH;  // chunks per thread
    static constexpr int BATCH = 4;                       // chunks loaded before they are stored

    __device__ __forceinline__ static float4 ld4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
    __device__ __forceinline__ static float4 ld4(const __nv_bfloat16* p) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
    }
    __device__ __forceinline__ static float ld1(const float* p) { return __ldg(p); }
    __device__ __forceinline__ static float ld1(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

    // Chunk c4 of vector v of token t, with the lo half of a split input added.
    __device__ __forceinline__ static float4 load_vec(const Params& p, int v, int b, int t, int hk, int hv, int c4,
                                                      bool bwd) {
        const Problem& pb = p.pb;
        const long qk = pb.qk_row(b, t, hk) + 4 * c4, vv = pb.v_row(b, t, hv) + 4 * c4;
        const long gc = pb.gate_row(b, t, hv, D) + 4 * c4;
        const __nv_bfloat16* lo = nullptr;
        long lo_off = 0;
        float4 x;
        switch (v) {
            case V_A: {
                float4 a = ld4(static_cast<const TG*>(p.alpha) + gc);
                a.x = pb.alpha_of(hv, a.x); a.y = pb.alpha_of(hv, a.y);
                a.z = pb.alpha_of(hv, a.z); a.w = pb.alpha_of(hv, a.w);
                return a;
            }
            case V_B:
            case V_W: {
                float4 g = ld4(static_cast<const TG*>(v == V_B ? p.b : p.w) + gc);
                g.x = pb.sig_of(g.x); g.y = pb.sig_of(g.y); g.z = pb.sig_of(g.z); g.w = pb.sig_of(g.w);
                return g;
            }
            case V_K: x = ld4(static_cast<const TIn*>(p.k) + qk); lo = static_cast<const __nv_bfloat16*>(p.k_lo); lo_off = qk; break;
            case V_Q: x = ld4(static_cast<const TIn*>(p.q) + qk); lo = static_cast<const __nv_bfloat16*>(p.q_lo); lo_off = qk; break;
            case V_V: x = ld4(static_cast<const TIn*>(p.v) + vv); lo = static_cast<const __nv_bfloat16*>(p.v_lo); lo_off = vv; break;
            default:
                if (bwd) {
                    x = ld4(static_cast<const TIn*>(p.dout) + vv);
                    lo = static_cast<const __nv_bfloat16*>(p.dout_lo);
                    lo_off = vv;
                    break;
                }
                if (p.z_bf16) return ld4(static_cast<const __nv_bfloat16*>(p.z) + vv);
                return ld4(static_cast<const TIn*>(p.z) + vv);
        }
        if (lo) {
            const float4 l = ld4(lo + lo_off);
            x.x += l.x; x.y += l.y; x.z += l.z; x.w += l.w;
        }
        return x;
    }
    __device__ __forceinline__ static bool active(const Params& p, int v, bool bwd) {
        if (v == V_A) return p.apc;
        if (v == V_B || v == V_W) return p.gpc;
        if (v == V_X) return bwd || p.z != nullptr;
        return true;
    }

    // Stage the block of tokens t0 .. t0 + kTB - 1 into buf [kTB][NVEC][D] (scal: [kTB][2]).  Tokens
    // past T get alpha = 1 and zeros elsewhere, which leaves the state unchanged; scalar gates are
    // broadcast over their vector.  Barriers inside (the buffer must not be in use).
    __device__ __forceinline__ static void stage(const Params& p, int b, int hk, int hv, int t0, float* buf,
                                                 float* scal, bool bwd) {
        const int tid = threadIdx.x;
        if (tid < kTB) {
            const bool in = t0 + tid < p.pb.T;
            const long g = p.pb.gate_row(b, in ? t0 + tid : 0, hv, 1);
            scal[2 * tid] = in && !p.apc ? p.pb.alpha_of(hv, ld1(static_cast<const TG*>(p.alpha) + g)) : 1.f;
            scal[2 * tid + 1] = in && !p.gpc ? p.pb.sig_of(ld1(static_cast<const TG*>(p.b) + g)) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int i0 = 0; i0 < PER; i0 += BATCH) {
            float4 x[BATCH];
#pragma unroll
            for (int i = i0; i < i0 + BATCH && i < PER; ++i) {
                const int id = tid + i * NTH;
                const int c4 = id % CH, v = (id / CH) % NVEC, tau = id / (CH * NVEC);
                x[i - i0] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (id < NCHUNK && t0 + tau < p.pb.T && active(p, v, bwd))
                    x[i - i0] = load_vec(p, v, b, t0 + tau, hk, hv, c4, bwd);
            }
#pragma unroll
            for (int i = i0; i < i0 + BATCH && i < PER; ++i) {
                const int id = tid + i * NTH;
                if (id >= NCHUNK) continue;
                const int c4 = id % CH, v = (id / CH) % NVEC, tau = id / (CH * NVEC);
                float4 y = x[i - i0];
                if (t0 + tau >= p.pb.T) {
                    const float f = v == V_A ? 1.f : 0.f;
                    y = make_float4(f, f, f, f);
                } else if (!active(p, v, bwd)) {
                    const float s = v == V_A ? scal[2 * tau] : (v == V_B || v == V_W) ? scal[2 * tau + 1] : 0.f;
                    y = make_float4(s, s, s, s);
                }
                *reinterpret_cast<float4*>(buf + (tau * NVEC + v) * D + 4 * c4) = y;
            }
        }
        __syncthreads();
    }
};

template <class TIn>
__device__ __forceinline__ void store_out(const Params& p, long off, float x) {
    if (p.o_type == 1) static_cast<float*>(p.o)[off] = x;
    else if (p.o_type == 2) static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(x);
    else static_cast<TIn*>(p.o)[off] = from_f32<TIn>(x);
}

// ------------------------------------------------------------------------------------------
// Forward: grid B*Hv, 2*D threads, dynamic shared memory seq_fwd_smem<D>().
// ------------------------------------------------------------------------------------------
template <int D>
constexpr size_t seq_fwd_smem() {
    return (size_t)2 * kTB * NVEC * D * sizeof(float) + 2 * kTB * 2 * sizeof(float) + 2 * 16 * sizeof(float);
}

template <class TIn, class TG, int D>
__global__ void __launch_bounds__(2 * D) seq_fwd_kernel(Params p) {
    constexpr int NTH = 2 * D, R = D / 2;
    extern __shared__ float4 smem_f4[];
    float* stage = reinterpret_cast<float*>(smem_f4);       // [2][kTB][NVEC][D]
    float* scal = stage + 2 * kTB * NVEC * D;               // [2][kTB][2]
    float* nred = scal + 2 * kTB * 2;                       // [2 token parities][NTH / 32 warps]
    const Problem& pb = p.pb;
    const int pair = blockIdx.x;
    if (p.flags && !p.flags[pair]) return;
    const int b = pair / pb.Hv, hv = pair % pb.Hv, hk = pb.key_head(hv);
    const int tid = threadIdx.x;
    const int h = (tid >> 4) & 1, j = (tid & 15) + 16 * (tid >> 5);
    const bool norm = p.z && p.norm_w;
    const float wn = !norm ? 1.f
                           : p.norm_w_f32 ? static_cast<const float*>(p.norm_w)[j]
                                          : __bfloat162float(static_cast<const __nv_bfloat16*>(p.norm_w)[j]);
    const int r0 = R * h;
    const long soff = pb.state_off(b, hv);

    float S[R];
#pragma unroll
    for (int i = 0; i < R; ++i) S[i] = p.h0 ? p.h0[soff + (long)(r0 + i) * D + j] : 0.f;

    using SG = Stager<TIn, TG, D, NTH>;
    const int nblk = (pb.T + kTB - 1) / kTB;
    for (int blk = 0; blk < nblk; ++blk) {
        const int t0 = blk * kTB;
        float* buf = stage + (blk & 1) * kTB * NVEC * D;
        SG::stage(p, b, hk, hv, t0, buf, scal + (blk & 1) * 2 * kTB, false);
        const int L = min(kTB, pb.T - t0);
        for (int tau = 0; tau < L; ++tau) {
            const int t = t0 + tau;
            const float* x = buf + tau * NVEC * D;
            // Sbar = Diag(alpha) S;  r_j = sum_c (b k)_c Sbar_cj
            float r = 0.f;
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 a = *reinterpret_cast<const float4*>(x + V_A * D + r0 + i);
                const float4 bb = *reinterpret_cast<const float4*>(x + V_B * D + r0 + i);
                const float4 kk = *reinterpret_cast<const float4*>(x + V_K * D + r0 + i);
                S[i] *= a.x; S[i + 1] *= a.y; S[i + 2] *= a.z; S[i + 3] *= a.w;
                r = fmaf(bb.x * kk.x, S[i], r);
                r = fmaf(bb.y * kk.y, S[i + 1], r);
                r = fmaf(bb.z * kk.z, S[i + 2], r);
                r = fmaf(bb.w * kk.w, S[i + 3], r);
            }
            r += __shfl_xor_sync(0xffffffffu, r, 16);
            const float u = x[V_W * D + j] * x[V_V * D + j] - r;
            // S += k (z - r)^T;  o_j = scale sum_c q_c S_cj
            float o = 0.f;
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 kk = *reinterpret_cast<const float4*>(x + V_K * D + r0 + i);
                const float4 qq = *reinterpret_cast<const float4*>(x + V_Q * D + r0 + i);
                S[i] = fmaf(kk.x, u, S[i]);
                S[i + 1] = fmaf(kk.y, u, S[i + 1]);
                S[i + 2] = fmaf(kk.z, u, S[i + 2]);
                S[i + 3] = fmaf(kk.w, u, S[i + 3]);
                o = fmaf(qq.x, S[i], o);
                o = fmaf(qq.y, S[i + 1], o);
                o = fmaf(qq.z, S[i + 2], o);
                o = fmaf(qq.w, S[i + 3], o);
            }
            o += __shfl_xor_sync(0xffffffffu, o, 16);
            float ov = pb.scale * o;
            float rs = 1.f;
            if (norm) {
                // the row's sum of squares over the D columns: 16 columns per warp (each held by the
                // two halves), then the warps' partials through shared memory (one barrier a token)
                float sq = ov * ov;
#pragma unroll
                for (int m = 1; m < 16; m <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, m);
                float* nr = nred + (t & 1) * 16;
                if ((tid & 31) == 0) nr[tid >> 5] = sq;
                __syncthreads();
                float tot = 0.f;
#pragma unroll
                for (int w8 = 0; w8 < NTH / 32; ++w8) tot += nr[w8];
                rs = rsqrtf(tot * (1.f / D) + p.norm_eps);
            }
            if (h == 0 && p.o) {
                const long off = pb.v_row(b, t, hv) + j;
                if (p.z) {
                    if (p.o_raw) p.o_raw[off] = ov;
                    const float zz = x[V_X * D + j];
                    ov *= rs * wn * zz * sigmoidf_(zz);
                }
                store_out<TIn>(p, off, ov);
            }
        }
    }
    if (p.ht) {
#pragma unroll
        for (int i = 0; i < R; ++i) p.ht[soff + (long)(r0 + i) * D + j] = S[i];
    }
}

// ------------------------------------------------------------------------------------------
// Backward: grid B*Hv, D*D/32 threads, dynamic shared memory seq_bwd_smem<D>().
// Thread (rb, cb): rows 8 rb .. 8 rb + 7, columns 4 cb .. 4 cb + 3.  A warp holds whole rows
// (D = 128: one row block, 32 column blocks; D = 64: two row blocks of 16 column blocks).
// ------------------------------------------------------------------------------------------
template <int D>
constexpr int seq_bwd_threads() { return D * D / 32; }
template <int D>
constexpr size_t seq_bwd_smem() {
    return (size_t)2 * kTB * NVEC * D * sizeof(float) + 2 * kTB * 2 * sizeof(float)  // staging
           + (size_t)(D / 8) * 2 * D * sizeof(float)                                  // row-block partials
           + (size_t)2 * D * sizeof(float) + 4 * sizeof(float);                       // column sums, scalars
}

// Reduce-scatter of 32 values over the W lanes of a lane group: afterwards lane l holds the sums of
// entries 32/W * (l % W) + i, i < 32/W, in x[0 ..].
template <int W>
__device__ __forceinline__ void reduce_scatter32(float (&x)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = W / 2, n = 32; o >= 1; o >>= 1) {
        const int half = n / 2;  // n: live values before this step (32 / (W / 2 / o))
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i < half) {
                const float send = upper ? x[i] : x[i + half];
                const float keep = upper ? x[i + half] : x[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        n = half;
    }
}

template <class TIn, class TG, int D>
__global__ void __launch_bounds__(D * D / 32) seq_bwd_kernel(Params p) {
    constexpr int NTH = D * D / 32, RB = D / 8, CB = D / 4, W = CB < 32 ? CB : 32;
    constexpr int NV_LANE = 32 / W;  // reduced values per lane after the reduce-scatter
    extern __shared__ float4 smem_f4[];
    float* stage = reinterpret_cast<float*>(smem_f4);        // [2][kTB][NVEC][D]
    float* scal = stage + 2 * kTB * NVEC * D;                // [2][kTB][2]
    float* red = scal + 2 * kTB * 2;                         // [RB][2][D]
    float* fin = red + RB * 2 * D;                           // [2][D]
    float* acc = fin + 2 * D;                                // scalar-gate sums of a token
    const Problem& pb = p.pb;
    const int pair = blockIdx.x;
    if (p.flags && !p.flags[pair]) return;
    const int b = pair / pb.Hv, hv = pair % pb.Hv, hk = pb.key_head(hv);
    const int tid = threadIdx.x, lane = tid & 31;
    const int cb = tid % CB, rb = tid / CB;
    const int c0 = 8 * rb, j0 = 4 * cb;
    const long soff = pb.state_off(b, hv);
    constexpr int DD = D * D;
    float* ck = p.ck + pair * p.ck_stride;
    float* sb = p.sbuf + (long)pair * kTB * DD;

    auto ld_state = [&](const float* src, float (&S)[8][4]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = *reinterpret_cast<const float4*>(src + (c0 + i) * D + j0);
            S[i][0] = v.x; S[i][1] = v.y; S[i][2] = v.z; S[i][3] = v.w;
        }
    };
    auto st_state = [&](float* dst, const float (&S)[8][4]) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *reinterpret_cast<float4*>(dst + (c0 + i) * D + j0) = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
    };
    auto init_state = [&](float (&S)[8][4]) {
        if (p.h0) ld_state(p.h0 + soff, S);
        else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int u = 0; u < 4; ++u) S[i][u] = 0.f;
        }
    };
    // Column sums over the key rows of two per-thread partials (4 columns each): through shared
    // memory, two barriers.
    auto col_sums = [&](const float (&pa)[4], const float (&pb2)[4], float (&sa)[4], float (&sb2)[4]) {
        *reinterpret_cast<float4*>(red + (rb * 2 + 0) * D + j0) = make_float4(pa[0], pa[1], pa[2], pa[3]);
        *reinterpret_cast<float4*>(red + (rb * 2 + 1) * D + j0) = make_float4(pb2[0], pb2[1], pb2[2], pb2[3]);
        __syncthreads();
        if (tid < 2 * D) {
            const int qn = tid / D, jj = tid % D;
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < RB; ++r) s += red[(r * 2 + qn) * D + jj];
            fin[qn * D + jj] = s;
        }
        __syncthreads();
        const float4 a = *reinterpret_cast<const float4*>(fin + j0);
        const float4 c = *reinterpret_cast<const float4*>(fin + D + j0);
        sa[0] = a.x; sa[1] = a.y; sa[2] = a.z; sa[3] = a.w;
        sb2[0] = c.x; sb2[1] = c.y; sb2[2] = c.z; sb2[3] = c.w;
    };
    // One forward token on the tile: S <- Diag(alpha) S + k (z - Sbar^T e)^T.
    auto fwd_step = [&](const float* x, float (&S)[8][4]) {
        float pr[4] = {0.f, 0.f, 0.f, 0.f}, zero[4] = {0.f, 0.f, 0.f, 0.f}, r[4], dummy[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a = x[V_A * D + c0 + i], e = x[V_B * D + c0 + i] * x[V_K * D + c0 + i];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                S[i][u] *= a;
                pr[u] = fmaf(e, S[i][u], pr[u]);
            }
        }
        col_sums(pr, zero, r, dummy);
#pragma unroll
        for (int u = 0; u < 4; ++u) r[u] = x[V_W * D + j0 + u] * x[V_V * D + j0 + u] - r[u];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float kk = x[V_K * D + c0 + i];
#pragma unroll
            for (int u = 0; u < 4; ++u) S[i][u] = fmaf(kk, r[u], S[i][u]);
        }
    };

    using SG = Stager<TIn, TG, D, NTH>;
    const int NT = pb.NT;
    if (tid < 4) acc[tid] = 0.f;
    float S[8][4], dS[8][4];

    // ---- 1. checkpoints: the state entering chunks 1 .. NT-1 ---------------------------------
    init_state(S);
    {
        const int last = NT > 1 ? (NT - 1) * (kChunk / kTB) : 0;  // blocks before the last chunk
        for (int blk = 0; blk < last; ++blk) {
            const int t0 = blk * kTB;
            float* buf = stage + (blk & 1) * kTB * NVEC * D;
            SG::stage(p, b, hk, hv, t0, buf, scal + (blk & 1) * 2 * kTB, true);
            for (int tau = 0; tau < kTB; ++tau) fwd_step(buf + tau * NVEC * D, S);
            if (((t0 + kTB) & (kChunk - 1)) == 0) st_state(ck + (long)((t0 + kTB) / kChunk - 1) * DD, S);
        }
    }
    __syncthreads();

    // ---- 2. reverse sweep, chunk by chunk, sub-chunk by sub-chunk -----------------------------
    if (p.dht) ld_state(p.dht + soff, dS);
    else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int u = 0; u < 4; ++u) dS[i][u] = 0.f;
    }
    int sched = 0;  // staging buffer parity
    for (int n = NT - 1; n >= 0; --n) {
        const int cs = n * kChunk, L = min(kChunk, pb.T - cs);
        for (int g = (L + kTB - 1) / kTB - 1; g >= 0; --g) {
            // forward from the chunk's checkpoint through sub-chunk g, storing its entering states
            if (n == 0) init_state(S);
            else ld_state(ck + (long)(n - 1) * DD, S);
            float* buf = stage;
            for (int bb = 0; bb <= g; ++bb) {
                buf = stage + (sched & 1) * kTB * NVEC * D;
                SG::stage(p, b, hk, hv, cs + bb * kTB, buf, scal + (sched & 1) * 2 * kTB, true);
                ++sched;
                for (int tau = 0; tau < kTB; ++tau) {
                    if (bb == g) st_state(sb + tau * DD, S);
                    fwd_step(buf + tau * NVEC * D, S);
                }
            }
            __syncthreads();  // the entering states are visible to every thread
            // reverse over the sub-chunk's tokens (S holds the state after its last token)
            const int t0 = cs + g * kTB, nt = min(kTB, pb.T - t0);
            for (int tau = nt - 1; tau >= 0; --tau) {
                const int t = t0 + tau;
                const float* x = buf + tau * NVEC * D;
                float Sp[8][4];
                ld_state(sb + tau * DD, Sp);
                float a[8], e[8], kk[8], qq[8], bg[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    a[i] = x[V_A * D + c0 + i];
                    bg[i] = x[V_B * D + c0 + i];
                    kk[i] = x[V_K * D + c0 + i];
                    qq[i] = x[V_Q * D + c0 + i];
                    e[i] = bg[i] * kk[i];
                }
                float dov[4], vv[4], ww[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    dov[u] = pb.scale * x[V_X * D + j0 + u];
                    vv[u] = x[V_V * D + j0 + u];
                    ww[u] = x[V_W * D + j0 + u];
                }
                // dq = scale S_t do (row sums, below); dS += scale q do^T; Sbar = Diag(alpha) S_{t-1}
                float red32[32];
                float pr[4] = {0.f, 0.f, 0.f, 0.f}, pz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float sq = 0.f;
                    const float ea = e[i] * a[i];  // r = Sbar^T e with Sbar = Diag(alpha) S_{t-1}
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        sq = fmaf(S[i][u], dov[u], sq);
                        dS[i][u] = fmaf(qq[i], dov[u], dS[i][u]);
                        pr[u] = fmaf(ea, Sp[i][u], pr[u]);
                        pz[u] = fmaf(dS[i][u], kk[i], pz[u]);
                    }
                    red32[i] = sq;
                }
                float r[4], dz[4];
                col_sums(pr, pz, r, dz);  // r = Sbar^T e, dz = dS^T k
                float dvw[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    dvw[u] = dz[u];
                    r[u] = ww[u] * vv[u] - r[u];  // u = z - r
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float sk = 0.f, se = 0.f, sa = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        sk = fmaf(dS[i][u], r[u], sk);                    // dk part: dS (z - r)
                        se = fmaf(Sp[i][u], dz[u], se);                   // S_{t-1} dz (de = -alpha * this)
                        const float dsb = fmaf(-e[i], dz[u], dS[i][u]);   // dSbar = dS - e dz^T
                        sa = fmaf(dsb, Sp[i][u], sa);                     // dalpha = sum_j dSbar S_{t-1}
                        dS[i][u] = a[i] * dsb;                            // gradient of S_{t-1}
                    }
                    red32[8 + i] = sk;
                    red32[16 + i] = -a[i] * se;
                    red32[24 + i] = sa;
                }
                reduce_scatter32<W>(red32);
                // lane l (W = 32) holds quantity l / 8 of row l % 8 (W = 16: two consecutive entries)
                // de of row i sits 8 entries after the dk part of row i: 8 / NV_LANE lanes further on
                float de_l[NV_LANE];
                const int de_src = (lane & ~(W - 1)) | (((lane % W) + 8 / NV_LANE) % W);
#pragma unroll
                for (int m = 0; m < NV_LANE; ++m) de_l[m] = __shfl_sync(0xffffffffu, red32[m], de_src);
                const long tok_qk = p.direct ? pb.qk_row(b, t, hk) : ((long)(b * pb.T + t) * pb.Hv + hv) * D;
#pragma unroll
                for (int m = 0; m < NV_LANE; ++m) {
                    const int idx = NV_LANE * (lane % W) + m, qn = idx / 8, i = idx % 8, c = c0 + i;
                    const float val = red32[m];
                    const bool qbf = p.grad_bf16 && p.direct;  // per-value-head partials stay fp32
                    if (qn == 0) put_g(p.dq, tok_qk + c, val, qbf);
                    else if (qn == 1) put_g(p.dk, tok_qk + c, val + bg[i] * de_l[m], qbf);
                    else if (qn == 2) {
                        if (p.gpc) put_g(p.db, pb.gate_row(b, t, hv, D) + c, kk[i] * val, p.gate_grad_bf16);
                        else atomicAdd(acc + 1, kk[i] * val);
                    } else {
                        if (p.apc) put_g(p.dalpha, pb.gate_row(b, t, hv, D) + c, val, p.gate_grad_bf16);
                        else atomicAdd(acc + 0, val);
                    }
                }
                if (rb == 0) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const long off = pb.v_row(b, t, hv) + j0 + u;
                        put_g(p.dv, off, ww[u] * dvw[u], p.grad_bf16);
                        if (p.gpc) put_g(p.dw, off, vv[u] * dvw[u], p.gate_grad_bf16);
                        else atomicAdd(acc + 1, vv[u] * dvw[u]);
                    }
                }
                // S_{t-1} is the next (earlier) token's S_t
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int u = 0; u < 4; ++u) S[i][u] = Sp[i][u];
                __syncthreads();
                if (tid == 0 && (!p.apc || !p.gpc)) {
                    const long g1 = pb.gate_row(b, t, hv, 1);
                    if (!p.apc) put_g(p.dalpha, g1, acc[0], p.gate_grad_bf16);
                    if (!p.gpc) put_g(p.db, g1, acc[1], p.gate_grad_bf16);
                    acc[0] = 0.f;
                    acc[1] = 0.f;
                }
            }
            __syncthreads();
        }
    }
    if (p.dh0) st_state(p.dh0 + soff, dS);
}

}  // namespace seq
}  // namespace gdn
