// Chunkwise forward and backward on CUDA cores in fp32 (used for fp32 inputs, any dk/dv in
// {64,128}, and as the general path).  Chunk length C = 64.
//
// Per chunk, with Gamma_r = prod_{i<=r} alpha_i (per key channel; the exponential of the
// cumulative log decay), gamma = Gamma_{C-1}, e = b.*k, z = w.*v (Gated DeltaNet-2 summary,
// «Entraînement Parallèle Efficace par Blocs»: the decay is absorbed into the erase and write
// factors and a lower-triangular system is solved):
//   Ehat = e.*Gamma, Qhat = q.*Gamma, Ktil = k./Gamma, Kbar = k.*gamma./Gamma
//   A = strict_lower(Ehat Ktil^T),  P = lower(Qhat Ktil^T),  T = (I + A)^-1
//   V' = T (Z - Ehat S0)                        (the write-side minus erase-side auxiliaries)
//   O  = scale (Qhat S0 + P V'),   S_end = Diag(gamma) S0 + Kbar^T V'
// Tokens past T in the last chunk are padded with k = q = e = z = 0 and alpha = 1, which
// leaves the state untouched, so the padded chunk gives the exact result.
//
// Kernels: chunk_prep (parallel over chunks: factors, A, P, T), chunk_scan_fwd (sequential
// over chunks, parallel over (b, hv, 32-column slices of dv): the state slice stays in shared
// memory), chunk_scan_bwd (reverse scan of the state gradient), chunk_grad (parallel over
// chunks: gradients of every input).
#pragma once
#include "block_gemm.cuh"
#include "common.cuh"
#include "seq.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
constexpr int kDvTile = 32;     // dv columns per backward scan CTA
constexpr int kDvTileFwd = 64;  // dv columns per forward scan CTA (4 x 4 register tiles)

// CTA-wide element loop over N = IT * kSimtThreads indices: every load of a thread is issued before
// any of its stores, so their latencies overlap (load(idx) -> float, store(idx, value)).
template <int N, class Load, class Store>
__device__ __forceinline__ void cta_load(Load load, Store store) {
    static_assert(N % kSimtThreads == 0, "N must be a multiple of the CTA size");
    constexpr int IT = N / kSimtThreads;
    float v[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) v[it] = load((int)threadIdx.x + it * kSimtThreads);
#pragma unroll
    for (int it = 0; it < IT; ++it) store((int)threadIdx.x + it * kSimtThreads, v[it]);
}

struct ChunkWs {
    float *T, *P, *Eh, *Qh, *Kb, *Kt, *Gm, *gam;  // per chunk factors
    float *S0, *dSC;                              // per chunk states / state gradients
    float *V, *Y, *dV, *dY;                       // per chunk [C][dv] intermediates (backward)
    float* dbw;                                   // [BH][NT][dv/32][C] scalar-beta partials
    float *dq_v, *dk_v;                           // [B,T,Hv,dk] per value head (GQA)
    int* flags;                                   // [B*Hv]: pairs outside the decay range (seq.cuh)
    float* sbuf;                                  // the sequential backward's states (seq.cuh)
};

struct ChunkIO {
    const void *q, *k, *v, *alpha, *b, *w, *z;
    // Tensor-core forward only: fp32 q, k, v given as bf16 pairs, q = q + q_lo etc. (NULL: plain)
    const void *q_lo, *k_lo, *v_lo;
    const float* h0;
    void* o;
    int o_type;  // 0: o in TIn, 1: fp32, 2: bf16
    int z_bf16;  // z stored as bf16 (else as TIn)
    // The layer's output norm before the gate (tensor-core forward and sequential kernels only):
    // weights [dv] (bf16 unless norm_w_f32), or NULL
    const void* norm_w;
    int norm_w_f32;
    float norm_eps;
    float* ht;
    const void* dout;
    const void* dout_lo;  // tensor-core backward only: dout as a bf16 hi/lo pair (dout = dout + dout_lo), or NULL
    const float* dht;
    void *dq, *dk, *dv, *dalpha, *db, *dw;
    int grad_type;  // 0: the gradients above in fp32; 1: in bf16 (tensor-core backward only)
    float* dh0;
};

__device__ __forceinline__ long chunk_index(const Problem& pb, int b, int hv, int n) {
    return ((long)b * pb.Hv + hv) * pb.NT + n;
}

// ------------------------------------------------------------------------------------------
// chunk_prep: grid (NT, Hv, B).
// ------------------------------------------------------------------------------------------
template <class TIn, class TG, bool APC, bool GPC, int DK>
__global__ void __launch_bounds__(kSimtThreads)
chunk_prep_kernel(Problem pb, ChunkIO io, ChunkWs ws, int save_bwd) {
    constexpr int C = kChunk, LD = DK + 1, LC = C + 1;
    extern __shared__ float smem[];
    float* Eh = smem;                 // [C][LD]
    float* Qh = Eh + C * LD;          // [C][LD]
    float* Kt = Qh + C * LD;          // [C][LD]
    float* scratch = Kt + C * LD;
    // A [C][LC] takes Eh's space once the first product has read it, T [C][LC] takes Qh's once the
    // second has (each product ends with a CTA barrier): two CTAs fit on an SM.
    float* A = Eh;
    float* Tm = Qh;

    const int n = blockIdx.x, hv = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int hk = pb.key_head(hv);
    const int t0 = n * C, L = min(C, pb.T - t0);
    const long ci = chunk_index(pb, b, hv, n);
    const TIn* q = static_cast<const TIn*>(io.q);
    const TIn* k = static_cast<const TIn*>(io.k);
    const TG* al = static_cast<const TG*>(io.alpha);
    const TG* bg = static_cast<const TG*>(io.b);

    // Cumulative decay per channel, gated factors.
    for (int c = tid; c < DK; c += kSimtThreads) {
        float G = 1.f;
        float* gm = ws.Gm ? ws.Gm + ci * C * DK : nullptr;
        for (int r0 = 0; r0 < C; r0 += 8) {
            float kv[8], qv[8], bv[8], av[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = r0 + u, t = t0 + r;
                const bool in = r < L;
                kv[u] = in ? to_f32(k[pb.qk_row(b, t, hk) + c]) : 0.f;
                qv[u] = in ? to_f32(q[pb.qk_row(b, t, hk) + c]) : 0.f;
                av[u] = in ? to_f32(al[pb.gate_row(b, t, hv, APC ? DK : 1) + (APC ? c : 0)]) : 1.f;
                bv[u] = in ? to_f32(bg[pb.gate_row(b, t, hv, GPC ? DK : 1) + (GPC ? c : 0)]) : 0.f;
            }
            if (pb.gate_logits) {  // one branch after the eight rows' loads, not one per load
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (r0 + u < L) {
                        av[u] = pb.alpha_t<true>(hv, av[u]);
                        bv[u] = pb.sig_t<true>(bv[u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = r0 + u;
                G *= av[u];
                Eh[r * LD + c] = bv[u] * kv[u] * G;
                Qh[r * LD + c] = qv[u] * G;
                Kt[r * LD + c] = kv[u] / G;
                if (save_bwd) gm[r * DK + c] = G;
            }
        }
        ws.gam[ci * DK + c] = G;
        // a chunk product below the factors' range: the pair goes to the sequential kernels
        if (ws.flags && seq::decay_out_of_range(G)) ws.flags[(long)b * pb.Hv + hv] = 1;
        for (int r = 0; r < C; ++r) {
            ws.Eh[(ci * C + r) * DK + c] = Eh[r * LD + c];
            ws.Qh[(ci * C + r) * DK + c] = Qh[r * LD + c];
            // Kbar = k * gamma / Gamma_r = Ktil * gamma.
            ws.Kb[(ci * C + r) * DK + c] = Kt[r * LD + c] * G;
            if (save_bwd) ws.Kt[(ci * C + r) * DK + c] = Kt[r * LD + c];
        }
    }
    __syncthreads();

    // A = strict_lower(Ehat Ktil^T), P = lower(Qhat Ktil^T).
    using G64 = BlockGemm<C, C, kSimtThreads, 32, 16>;
    {
        G64 g;
        g.zero();
        g.mma(View{Eh, LD, 1}, View{Kt, 1, LD}, DK, scratch);
#pragma unroll
        for (int i = 0; i < G64::TM; ++i)
#pragma unroll
            for (int j = 0; j < G64::TN; ++j) {
                const int r = g.row(i), s = g.col(j);
                A[r * LC + s] = s < r ? g.acc[i][j] : 0.f;
            }
    }
    {
        G64 g;
        g.zero();
        g.mma(View{Qh, LD, 1}, View{Kt, 1, LD}, DK, scratch);
#pragma unroll
        for (int i = 0; i < G64::TM; ++i)
#pragma unroll
            for (int j = 0; j < G64::TN; ++j) {
                const int r = g.row(i), s = g.col(j);
                ws.P[(ci * C + r) * C + s] = s <= r ? g.acc[i][j] : 0.f;
            }
    }
    __syncthreads();

    // T = (I + A)^-1 by forward substitution, column j by a group of 4 lanes.
    {
        const int j = tid >> 2, part = tid & 3;
        for (int i = 0; i < C; ++i) {
            float acc = 0.f;
            for (int s = j + part; s < i; s += 4) acc += A[i * LC + s] * Tm[s * LC + j];
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (part == 0) Tm[i * LC + j] = i == j ? 1.f : (i < j ? 0.f : -acc);
            __syncwarp();
        }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += kSimtThreads)
        ws.T[ci * C * C + idx] = Tm[(idx / C) * LC + idx % C];
}

template <int DK>
constexpr size_t chunk_prep_smem() {
    static_assert(DK >= kChunk, "A and T reuse the space of Ehat and Qhat");
    return sizeof(float) * (3 * kChunk * (DK + 1) + BlockGemm<kChunk, kChunk, kSimtThreads, 32, 16>::kScratch);
}

// ------------------------------------------------------------------------------------------
// chunk_scan_fwd: grid (dv / 32, Hv, B).  Carries the fp32 state slice S[:, j0:j0+32].
// ------------------------------------------------------------------------------------------
template <class TIn, class TG, bool GPC, int DK, bool GATE>
__global__ void __launch_bounds__(kSimtThreads)
chunk_scan_fwd_kernel(Problem pb, ChunkIO io, ChunkWs ws, int write_out, int save_states) {
    constexpr int C = kChunk, W = kDvTileFwd;
    extern __shared__ float smem[];
    float* S = smem;            // [DK][W]
    float* Z = S + DK * W;      // [C][W]
    float* Y = Z + C * W;       // [C][W]
    float* V = Y + C * W;       // [C][W]
    float* scratch = V + C * W;

    const int tile = blockIdx.x, hv = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int j0 = tile * W;
    const int dv = pb.dv;
    const TIn* vin = static_cast<const TIn*>(io.v);
    const TG* wg = static_cast<const TG*>(GPC ? io.w : io.b);
    const long soff = pb.state_off(b, hv);

    cta_load<DK * W>(
        [&](int idx) { return io.h0 ? io.h0[soff + (long)(idx / W) * dv + j0 + idx % W] : 0.f; },
        [&](int idx, float v) { S[idx] = v; });

    using GCW = BlockGemm<C, W, kSimtThreads, 16>;   // [C x 32] outputs
    using GKW = BlockGemm<DK, W, kSimtThreads, 16>;  // [DK x 32] outputs
    for (int n = 0; n < pb.NT; ++n) {
        const int t0 = n * C, L = min(C, pb.T - t0);
        const long ci = chunk_index(pb, b, hv, n);
        const float* Eh = ws.Eh + ci * C * DK;
        const float* Qh = ws.Qh + ci * C * DK;
        const float* Kb = ws.Kb + ci * C * DK;
        const float* Tm = ws.T + ci * C * C;
        const float* Pm = ws.P + ci * C * C;
        const float* gam = ws.gam + ci * DK;
        __syncthreads();
        cta_load<C * W>(
            [&](int idx) {
                const int r = idx / W, j = idx % W, t = t0 + r;
                if (r >= L) return 0.f;
                return to_f32(vin[pb.v_row(b, t, hv) + j0 + j]) *
                       pb.sig_of(to_f32(wg[pb.gate_row(b, t, hv, GPC ? dv : 1) + (GPC ? j0 + j : 0)]));
            },
            [&](int idx, float v) { Z[idx] = v; });
        if (save_states)
            for (int idx = tid; idx < DK * W; idx += kSimtThreads) {
                const int c = idx / W, j = idx % W;
                ws.S0[ci * DK * dv + (long)c * dv + j0 + j] = S[idx];
            }
        // Y = Z - Ehat S0
        {
            GCW g;
            g.zero();
            g.mma(View{Eh, DK, 1}, View{S, W, 1}, DK, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) {
                    const int r = g.row(i), c = g.col(j);
                    Y[r * W + c] = Z[r * W + c] - g.acc[i][j];
                }
        }
        // V' = T Y
        {
            GCW g;
            g.zero();
            g.mma(View{Tm, C, 1}, View{Y, W, 1}, C, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) V[g.row(i) * W + g.col(j)] = g.acc[i][j];
        }
        // O = scale (Qhat S0 + P V')
        if (write_out) {
            GCW g;
            g.zero();
            g.mma(View{Qh, DK, 1}, View{S, W, 1}, DK, scratch);
            g.mma(View{Pm, C, 1}, View{V, W, 1}, C, scratch);
            TIn* o = static_cast<TIn*>(io.o);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) {
                    const int r = g.row(i), c = g.col(j);
                    if (r < L) {
                        const long off = pb.v_row(b, t0 + r, hv) + j0 + c;
                        float ov = pb.scale * g.acc[i][j];
                        if (GATE) {
                            const float zz = io.z_bf16 ? to_f32(static_cast<const __nv_bfloat16*>(io.z)[off])
                                                       : to_f32(static_cast<const TIn*>(io.z)[off]);
                            ov *= zz * sigmoidf_(zz);
                        }
                        if (io.o_type == 1) static_cast<float*>(io.o)[off] = ov;
                        else if (io.o_type == 2) static_cast<__nv_bfloat16*>(io.o)[off] = from_f32<__nv_bfloat16>(ov);
                        else o[off] = from_f32<TIn>(ov);
                    }
                }
        }
        // S = Diag(gamma) S0 + Kbar^T V'
        {
            GKW g;
            g.zero();
            g.mma(View{Kb, 1, DK}, View{V, W, 1}, C, scratch);
#pragma unroll
            for (int i = 0; i < GKW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GKW::TN; ++j) {
                    const int c = g.row(i), jj = g.col(j);
                    S[c * W + jj] = gam[c] * S[c * W + jj] + g.acc[i][j];
                }
        }
    }
    __syncthreads();
    if (io.ht)
        for (int idx = tid; idx < DK * W; idx += kSimtThreads) {
            const int c = idx / W, j = idx % W;
            io.ht[soff + (long)c * dv + j0 + j] = S[idx];
        }
}

template <int DK>
constexpr size_t chunk_scan_fwd_smem() {
    return sizeof(float) * (DK * kDvTileFwd + 3 * kChunk * kDvTileFwd +
                            BlockGemm<DK, kDvTileFwd, kSimtThreads, 16>::kScratch);
}

// ------------------------------------------------------------------------------------------
// chunk_scan_bwd: grid (dv / 32, Hv, B).  Reverse scan of the state gradient:
//   dV' = scale P^T dO + Kbar dS_end,  dY = T^T dV',
//   dS0 = scale Qhat^T dO + Diag(gamma) dS_end - Ehat^T dY.
// Saves dS_end, V', Y, dV', dY per chunk and writes dv, dw (dZ = dY).
// ------------------------------------------------------------------------------------------
template <class TIn, class TG, bool GPC, int DK>
__global__ void __launch_bounds__(kSimtThreads)
chunk_scan_bwd_kernel(Problem pb, ChunkIO io, ChunkWs ws) {
    constexpr int C = kChunk, W = kDvTile;
    extern __shared__ float smem[];
    float* dS = smem;            // [DK][W]
    float* S0 = dS + DK * W;     // [DK][W]
    float* Z = S0 + DK * W;      // [C][W]
    float* Y = Z + C * W;
    float* V = Y + C * W;
    float* dO = V + C * W;       // scale * dO
    float* dV = dO + C * W;
    float* dY = dV + C * W;
    float* scratch = dY + C * W;

    const int tile = blockIdx.x, hv = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int j0 = tile * W, dv = pb.dv, ntile = dv / W;
    const TIn* vin = static_cast<const TIn*>(io.v);
    const TIn* gout = static_cast<const TIn*>(io.dout);
    const TG* wg = static_cast<const TG*>(GPC ? io.w : io.b);
    const long soff = pb.state_off(b, hv);

    cta_load<DK * W>(
        [&](int idx) { return io.dht ? io.dht[soff + (long)(idx / W) * dv + j0 + idx % W] : 0.f; },
        [&](int idx, float v) { dS[idx] = v; });

    using GCW = BlockGemm<C, W, kSimtThreads, 16>;
    using GKW = BlockGemm<DK, W, kSimtThreads, 16>;
    for (int n = pb.NT - 1; n >= 0; --n) {
        const int t0 = n * C, L = min(C, pb.T - t0);
        const long ci = chunk_index(pb, b, hv, n);
        const float* Eh = ws.Eh + ci * C * DK;
        const float* Qh = ws.Qh + ci * C * DK;
        const float* Kb = ws.Kb + ci * C * DK;
        const float* Tm = ws.T + ci * C * C;
        const float* Pm = ws.P + ci * C * C;
        const float* gam = ws.gam + ci * DK;
        __syncthreads();
        cta_load<DK * W>(
            [&](int idx) {
                const long off = ci * DK * dv + (long)(idx / W) * dv + j0 + idx % W;
                ws.dSC[off] = dS[idx];
                return ws.S0[off];
            },
            [&](int idx, float v) { S0[idx] = v; });
        cta_load<C * W>(
            [&](int idx) {
                const int r = idx / W, j = idx % W, t = t0 + r;
                if (r >= L) return 0.f;
                return to_f32(vin[pb.v_row(b, t, hv) + j0 + j]) *
                       pb.sig_of(to_f32(wg[pb.gate_row(b, t, hv, GPC ? dv : 1) + (GPC ? j0 + j : 0)]));
            },
            [&](int idx, float v) { Z[idx] = v; });
        cta_load<C * W>(
            [&](int idx) {
                const int r = idx / W, j = idx % W;
                return r < L ? pb.scale * to_f32(gout[pb.v_row(b, t0 + r, hv) + j0 + j]) : 0.f;
            },
            [&](int idx, float v) { dO[idx] = v; });
        // Y = Z - Ehat S0 ; V' = T Y
        {
            GCW g;
            g.zero();
            g.mma(View{Eh, DK, 1}, View{S0, W, 1}, DK, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) {
                    const int r = g.row(i), c = g.col(j);
                    Y[r * W + c] = Z[r * W + c] - g.acc[i][j];
                }
        }
        {
            GCW g;
            g.zero();
            g.mma(View{Tm, C, 1}, View{Y, W, 1}, C, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) V[g.row(i) * W + g.col(j)] = g.acc[i][j];
        }
        // dV' = P^T (scale dO) + Kbar dS_end
        {
            GCW g;
            g.zero();
            g.mma(View{Pm, 1, C}, View{dO, W, 1}, C, scratch);
            g.mma(View{Kb, DK, 1}, View{dS, W, 1}, DK, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) dV[g.row(i) * W + g.col(j)] = g.acc[i][j];
        }
        // dY = T^T dV'  (= dZ): write dv, dw and the per-chunk intermediates.
        {
            GCW g;
            g.zero();
            g.mma(View{Tm, 1, C}, View{dV, W, 1}, C, scratch);
#pragma unroll
            for (int i = 0; i < GCW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GCW::TN; ++j) dY[g.row(i) * W + g.col(j)] = g.acc[i][j];
        }
        __syncthreads();
        for (int idx = tid; idx < C * W; idx += kSimtThreads) {
            const int r = idx / W, j = idx % W;
            const long off = (ci * C + r) * dv + j0 + j;
            ws.Y[off] = Y[idx];
            ws.V[off] = V[idx];
            ws.dV[off] = dV[idx];
            ws.dY[off] = dY[idx];
            if (r < L) {
                const int t = t0 + r;
                const long io_off = pb.v_row(b, t, hv) + j0 + j;
                const float ww = pb.sig_of(to_f32(wg[pb.gate_row(b, t, hv, GPC ? dv : 1) + (GPC ? j0 + j : 0)]));
                static_cast<float*>(io.dv)[io_off] = dY[idx] * ww;
                if (GPC) static_cast<float*>(io.dw)[io_off] = dY[idx] * to_f32(vin[io_off]);
            }
        }
        if (!GPC && tid < C) {
            // Scalar beta: this slice's share of sum_j dZ_j v_j.
            const int r = tid;
            float acc = 0.f;
            if (r < L)
                for (int j = 0; j < W; ++j)
                    acc += dY[r * W + j] * to_f32(vin[pb.v_row(b, t0 + r, hv) + j0 + j]);
            ws.dbw[(ci * ntile + tile) * C + r] = acc;
        }
        // dS0 = Qhat^T (scale dO) - Ehat^T dY + Diag(gamma) dS_end
        {
            GKW g;
            g.zero();
            g.mma(View{Qh, 1, DK}, View{dO, W, 1}, C, scratch);
            g.mma(View{Eh, 1, DK}, View{dY, W, 1}, C, scratch, -1.f);
#pragma unroll
            for (int i = 0; i < GKW::TM; ++i)
#pragma unroll
                for (int j = 0; j < GKW::TN; ++j) {
                    const int c = g.row(i), jj = g.col(j);
                    dS[c * W + jj] = gam[c] * dS[c * W + jj] + g.acc[i][j];
                }
        }
    }
    __syncthreads();
    if (io.dh0)
        for (int idx = tid; idx < DK * W; idx += kSimtThreads) {
            const int c = idx / W, j = idx % W;
            io.dh0[soff + (long)c * dv + j0 + j] = dS[idx];
        }
}

template <int DK>
constexpr size_t chunk_scan_bwd_smem() {
    return sizeof(float) * (2 * DK * kDvTile + 6 * kChunk * kDvTile +
                            BlockGemm<DK, kDvTile, kSimtThreads, 16>::kScratch);
}

// ------------------------------------------------------------------------------------------
// chunk_grad: grid (NT, Hv, B).  Per-chunk gradients of q, k, alpha, b (and beta):
//   dP = lower(scale dO V'^T),  dT = dV' Y^T,  dA = strict_lower(-T^T dT T^T)
//   dQhat = scale dO S0^T + dP Ktil,   dEhat = -dY S0^T + dA Ktil
//   dKtil = dA^T Ehat + dP^T Qhat,      dKbar = V' dS_end^T,  dgamma = rowsum(dS_end .* S0)
// then through Ehat = e Gamma, Qhat = q Gamma, Ktil = k / Gamma, Kbar = k gamma / Gamma and
// g = cumsum(log alpha) (reverse cumulative sum), e = b k.
// ------------------------------------------------------------------------------------------
template <class TIn, class TG, bool APC, bool GPC, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads)
chunk_grad_kernel(Problem pb, ChunkIO io, ChunkWs ws, int direct_qk) {
    constexpr int C = kChunk, LC = C + 1, LDV = DV + 1;
    extern __shared__ float smem[];
    float* dP = smem;             // [C][LC]
    float* dA = dP + C * LC;      // [C][LC]   (dT first, then dA)
    float* tmp = dA + C * LC;     // [C][LC]
    float* dO = tmp + C * LC;     // [C][LDV]  scale * dO
    float* dg = dO + C * LDV;     // [C][DK]
    float* colp = dg + C * DK;    // [8][DK] partial column sums
    float* rowsum = colp + 8 * DK;// [C]
    float* scratch = rowsum + C;

    const int n = blockIdx.x, hv = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int hk = pb.key_head(hv);
    const int t0 = n * C, L = min(C, pb.T - t0);
    const long ci = chunk_index(pb, b, hv, n);
    const float* Eh = ws.Eh + ci * C * DK;
    const float* Qh = ws.Qh + ci * C * DK;
    const float* Kt = ws.Kt + ci * C * DK;
    const float* Kb = ws.Kb + ci * C * DK;
    const float* Gm = ws.Gm + ci * C * DK;
    const float* gam = ws.gam + ci * DK;
    const float* Tm = ws.T + ci * C * C;
    const float* S0 = ws.S0 + ci * DK * DV;
    const float* dSC = ws.dSC + ci * DK * DV;
    const float* Vp = ws.V + ci * C * DV;
    const float* Yp = ws.Y + ci * C * DV;
    const float* dVp = ws.dV + ci * C * DV;
    const float* dYp = ws.dY + ci * C * DV;
    const TIn* kin = static_cast<const TIn*>(io.k);
    const TG* al = static_cast<const TG*>(io.alpha);
    const TG* bg = static_cast<const TG*>(io.b);

    cta_load<C * DV>(
        [&](int idx) {
            const int r = idx / DV, j = idx % DV;
            return r < L ? pb.scale * to_f32(static_cast<const TIn*>(io.dout)[pb.v_row(b, t0 + r, hv) + j]) : 0.f;
        },
        [&](int idx, float v) { dO[(idx / DV) * LDV + idx % DV] = v; });

    using GCC = BlockGemm<C, C, kSimtThreads, 32>;
    {   // dP = lower(scale dO V'^T)
        GCC g;
        g.zero();
        g.mma(View{dO, LDV, 1}, View{Vp, 1, DV}, DV, scratch);
#pragma unroll
        for (int i = 0; i < GCC::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCC::TN; ++j) {
                const int r = g.row(i), s = g.col(j);
                dP[r * LC + s] = s <= r ? g.acc[i][j] : 0.f;
            }
    }
    {   // dT = dV' Y^T
        GCC g;
        g.zero();
        g.mma(View{dVp, DV, 1}, View{Yp, 1, DV}, DV, scratch);
#pragma unroll
        for (int i = 0; i < GCC::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCC::TN; ++j) dA[g.row(i) * LC + g.col(j)] = g.acc[i][j];
    }
    {   // tmp = dT T^T
        GCC g;
        g.zero();
        g.mma(View{dA, LC, 1}, View{Tm, 1, C}, C, scratch);
#pragma unroll
        for (int i = 0; i < GCC::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCC::TN; ++j) tmp[g.row(i) * LC + g.col(j)] = g.acc[i][j];
    }
    {   // dA = strict_lower(-T^T tmp)
        GCC g;
        g.zero();
        g.mma(View{Tm, 1, C}, View{tmp, LC, 1}, C, scratch);
#pragma unroll
        for (int i = 0; i < GCC::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCC::TN; ++j) {
                const int r = g.row(i), s = g.col(j);
                dA[r * LC + s] = s < r ? -g.acc[i][j] : 0.f;
            }
    }

    // [C x DK] gradients, all with the same thread mapping: dk and dg accumulate in registers.
    using GCK = BlockGemm<C, DK, kSimtThreads, 32>;
    float dk_acc[GCK::TM][GCK::TN], dg_acc[GCK::TM][GCK::TN], rsum[GCK::TM];
#pragma unroll
    for (int i = 0; i < GCK::TM; ++i) {
        rsum[i] = 0.f;
#pragma unroll
        for (int j = 0; j < GCK::TN; ++j) dk_acc[i][j] = dg_acc[i][j] = 0.f;
    }
    float* dq_out = nullptr;
    float* dq_direct = nullptr;
    if (direct_qk) dq_direct = static_cast<float*>(io.dq);
    else dq_out = ws.dq_v;
    {   // dQhat = (scale dO) S0^T + dP Ktil
        GCK g;
        g.zero();
        g.mma(View{dO, LDV, 1}, View{S0, 1, DV}, DV, scratch);
        g.mma(View{dP, LC, 1}, View{Kt, DK, 1}, C, scratch);
#pragma unroll
        for (int i = 0; i < GCK::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCK::TN; ++j) {
                const int r = g.row(i), c = g.col(j);
                const float v = g.acc[i][j];
                dg_acc[i][j] += v * Qh[r * DK + c];
                if (r < L) {
                    const float gq = v * Gm[r * DK + c];
                    if (direct_qk) dq_direct[pb.qk_row(b, t0 + r, hk) + c] = gq;
                    else dq_out[pb.v_row(b, t0 + r, hv) / pb.dv * DK + c] = gq;
                }
            }
    }
    {   // dEhat = -dY S0^T + dA Ktil
        GCK g;
        g.zero();
        g.mma(View{dYp, DV, 1}, View{S0, 1, DV}, DV, scratch, -1.f);
        g.mma(View{dA, LC, 1}, View{Kt, DK, 1}, C, scratch);
#pragma unroll
        for (int i = 0; i < GCK::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCK::TN; ++j) {
                const int r = g.row(i), c = g.col(j);
                const float v = g.acc[i][j];
                dg_acc[i][j] += v * Eh[r * DK + c];
                if (r < L) {
                    const int t = t0 + r;
                    const float de = v * Gm[r * DK + c];
                    const float kv = to_f32(kin[pb.qk_row(b, t, hk) + c]);
                    const float bv = pb.sig_of(to_f32(bg[pb.gate_row(b, t, hv, GPC ? DK : 1) + (GPC ? c : 0)]));
                    dk_acc[i][j] += de * bv;
                    if (GPC) static_cast<float*>(io.db)[pb.gate_row(b, t, hv, DK) + c] = de * kv;
                    else rsum[i] += de * kv;
                }
            }
    }
    {   // dKtil = dA^T Ehat + dP^T Qhat
        GCK g;
        g.zero();
        g.mma(View{dA, 1, LC}, View{Eh, DK, 1}, C, scratch);
        g.mma(View{dP, 1, LC}, View{Qh, DK, 1}, C, scratch);
#pragma unroll
        for (int i = 0; i < GCK::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCK::TN; ++j) {
                const int r = g.row(i), c = g.col(j);
                const float v = g.acc[i][j];
                dk_acc[i][j] += v / Gm[r * DK + c];
                dg_acc[i][j] -= v * Kt[r * DK + c];
            }
    }
    float cpart[GCK::TN];
#pragma unroll
    for (int j = 0; j < GCK::TN; ++j) cpart[j] = 0.f;
    {   // dKbar = V' dS_end^T
        GCK g;
        g.zero();
        g.mma(View{Vp, DV, 1}, View{dSC, 1, DV}, DV, scratch);
#pragma unroll
        for (int i = 0; i < GCK::TM; ++i)
#pragma unroll
            for (int j = 0; j < GCK::TN; ++j) {
                const int r = g.row(i), c = g.col(j);
                const float v = g.acc[i][j];
                const float kb = Kb[r * DK + c];
                dk_acc[i][j] += v * gam[c] / Gm[r * DK + c];
                dg_acc[i][j] -= v * kb;
                cpart[j] += v * kb;
            }
    }
    // Write dk; stage dg; deterministic column sums of dKbar .* Kbar.
    {
        GCK g;  // mapping only
        float* dk_direct = static_cast<float*>(io.dk);
#pragma unroll
        for (int i = 0; i < GCK::TM; ++i) {
            const int r = g.row(i);
#pragma unroll
            for (int j = 0; j < GCK::TN; ++j) {
                const int c = g.col(j);
                dg[r * DK + c] = dg_acc[i][j];
                if (r < L) {
                    if (direct_qk) dk_direct[pb.qk_row(b, t0 + r, hk) + c] = dk_acc[i][j];
                    else ws.dk_v[pb.v_row(b, t0 + r, hv) / pb.dv * DK + c] = dk_acc[i][j];
                }
            }
        }
        const int tm = tid / 32;
#pragma unroll
        for (int j = 0; j < GCK::TN; ++j) colp[tm * DK + g.col(j)] = cpart[j];
        if (!GPC) {
            // row sums of de .* k over the 32 lanes of the warp (same rows in a warp)
#pragma unroll
            for (int i = 0; i < GCK::TM; ++i) {
                float v = rsum[i];
#pragma unroll
                for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if ((tid & 31) == 0) rowsum[g.row(i)] = v;
            }
        }
    }
    __syncthreads();
    // dgamma = rowsum(dS_end .* S0); add (sum_r dKbar .* Kbar + dgamma gamma) to the last row.
    for (int c = tid; c < DK; c += kSimtThreads) {
        float dgam = 0.f;
        for (int j = 0; j < DV; ++j) dgam += dSC[c * DV + j] * S0[c * DV + j];
        float cs = 0.f;
        for (int m = 0; m < kSimtThreads / 32; ++m) cs += colp[m * DK + c];
        dg[(C - 1) * DK + c] += cs + dgam * gam[c];
    }
    __syncthreads();
    // d log alpha_r = sum_{r' >= r} dg_r'  (reverse cumulative sum per channel).
    for (int c = tid; c < DK; c += kSimtThreads) {
        float run = 0.f;
        for (int r = C - 1; r >= 0; --r) {
            run += dg[r * DK + c];
            dg[r * DK + c] = run;
        }
    }
    __syncthreads();
    if (APC) {
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            if (r < L) {
                const long off = pb.gate_row(b, t0 + r, hv, DK) + c;
                static_cast<float*>(io.dalpha)[off] = dg[idx] / pb.alpha_of(hv, to_f32(al[off]));
            }
        }
    } else if (tid < C) {
        const int r = tid;
        if (r < L) {
            float s = 0.f;
            for (int c = 0; c < DK; ++c) s += dg[r * DK + c];
            const long off = pb.gate_row(b, t0 + r, hv, 1);
            static_cast<float*>(io.dalpha)[off] = s / pb.alpha_of(hv, to_f32(al[off]));
        }
    }
    if (!GPC && tid < C) {
        const int r = tid, ntile = DV / kDvTile;
        if (r < L) {
            float s = rowsum[r];
            for (int tl = 0; tl < ntile; ++tl) s += ws.dbw[(ci * ntile + tl) * C + r];
            static_cast<float*>(io.db)[pb.gate_row(b, t0 + r, hv, 1)] = s;
        }
    }
}

template <int DK, int DV>
constexpr size_t chunk_grad_smem() {
    return sizeof(float) * (3 * kChunk * (kChunk + 1) + kChunk * (DV + 1) + kChunk * DK + 8 * DK +
                            kChunk + BlockGemm<kChunk, DK, kSimtThreads, 32>::kScratch);
}

// Sum per-value-head dq/dk [B,T,Hv,dk] over the value heads of each key head, ascending hv
// (fixed order: deterministic).  The block first lists the value heads of every key head in
// shared memory (dynamic: Hv + Hk + 1 ints); then each thread sums float4 columns of one token
// row at a time.  dk is a multiple of 4 and every row starts 16-byte aligned.  The sums are written
// in OT (fp32, or bf16 for gradients returned in the inputs' dtype).
template <class OT>
static __global__ void __launch_bounds__(256) gqa_reduce_kernel(Problem pb, const float* part, OT* out) {
    extern __shared__ int heads[];  // heads[0 .. Hv): value heads grouped by key head; then Hk + 1 starts
    int* beg = heads + pb.Hv;
    if (threadIdx.x == 0) {
        int n = 0;
        for (int hk = 0; hk < pb.Hk; ++hk) {
            beg[hk] = n;
            for (int hv = 0; hv < pb.Hv; ++hv)
                if (pb.key_head(hv) == hk) heads[n++] = hv;
        }
        beg[pb.Hk] = n;
    }
    __syncthreads();
    const int q4 = pb.dk / 4, per_row = pb.Hk * q4;
    const long rows = (long)pb.B * pb.T;
    const float4* src = reinterpret_cast<const float4*>(part);
    for (long bt = blockIdx.x; bt < rows; bt += gridDim.x) {
        for (int i = threadIdx.x; i < per_row; i += blockDim.x) {
            const int hk = i / q4, c = i - hk * q4;
            float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = beg[hk]; j < beg[hk + 1]; ++j) {
                const float4 x = __ldg(src + (bt * pb.Hv + heads[j]) * q4 + c);
                s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
            }
            st4_g(out + (bt * per_row + i) * 4, s.x, s.y, s.z, s.w);
        }
    }
}

}  // namespace gdn
