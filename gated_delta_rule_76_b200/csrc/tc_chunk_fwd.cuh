// Fused chunkwise forward on the 5th-generation tensor cores (sm_100a): one CTA per
// (batch, value head), chunks of C = 64 tokens, dk = dv = 128, bf16 inputs, fp32 state.
//
// Per chunk (Gated DeltaNet-2 summary, «Entraînement Parallèle Efficace par Blocs»; the decay is
// absorbed into the erase and write factors, a lower-triangular system is solved):
//   Gamma_r = prod_{i<=r} alpha_i,  gamma = Gamma_63;  Ehat = (b.*k).*Gamma,  Qhat = q.*Gamma,
//   Ktil = k./Gamma,  Kbar = k.*gamma./Gamma;   A = strict_lower(Ehat Ktil^T),
//   P = lower(Qhat Ktil^T),  T = (I + A)^-1,   V' = T (Z - Ehat S0),  Z = w.*v,
//   O = scale (Qhat S0 + P V'),  S_end = Diag(gamma) S0 + Kbar^T V'.
// Every product is issued with M = 128 by putting dv on the M side (D[j][..] = sum A[j][k] B[..][k]):
//   X1 = [Ehat;Qhat] Ktil^T               (M = 128 rows of Ehat/Qhat, N = 64, K = 128)
//   X2 = S0^T [Ehat;Qhat]^T               (M = dv, N = 2 x 64, K = dk; A = S0^T in tensor memory)
//   X3 = Y^T T^T   with Y^T = Z^T - (Ehat S0)^T  (M = dv, N = 64, K = 64; A in tensor memory)
//   X4 = V'^T P^T  accumulated onto (Qhat S0)^T  (M = dv, N = 64, K = 64)
//   X5 = V'^T Kbar (B = Kbar^T, K-major)  (M = dv, N = dk, K = 64)
// Thread j of the two scan warpgroups owns TMEM lane j (= value column j) and keeps its column
// of the fp32 state in registers, split between the warpgroups by halves of dk.
//
// Roles (384 threads):
//   warps 0-7  (scan)     : the sequential chain X2 -> Y -> X3 -> V' -> X4, X5 -> output, state;
//                           thread 0 issues the scan's MMAs and the TMA loads.
//   warps 8-11 (prologue) : for the next chunk, the cumulative decay and in-place scaling of the
//                           TMA tiles, X1, the triangular solve T = (I + A)^-1, and Kbar^T.
// Shared memory (~226 KB): two slots of raw tiles (q, k, alpha, b) that are transformed in place
// into the MMA operands, two slots of v/w tiles, Kbar^T, a fp32 scratch for A.
// Tensor memory: 480 of 512 columns.  Every mbarrier wait is bounded: on expiry the kernel sets
// an error word, stops issuing work and frees its tensor memory.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "umma.cuh"

namespace gdn {
namespace tcfwd {

using namespace gdn::tc;

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 384;
constexpr uint64_t kWaitNs = 4000000000ull;

// tensor memory columns
constexpr uint32_t TM_X1 = 0;    // 64:  A (lanes 0-63), P (lanes 64-127), fp32
constexpr uint32_t TM_X2 = 64;   // 128: (Ehat S0)^T | (Qhat S0 + P V')^T
constexpr uint32_t TM_X3 = 192;  // 64:  V'^T fp32
constexpr uint32_t TM_X5 = 256;  // 128: (Kbar^T V')^T
constexpr uint32_t TM_S0 = 384;  // 64:  S0^T as bf16 pairs (A operand of X2)
constexpr uint32_t TM_Y = 448;   // 32:  Y^T, then V'^T, as bf16 pairs (A operand of X3, X4, X5)
constexpr uint32_t TM_COLS = 512;

// shared memory offsets from the 1024-byte-aligned base
constexpr uint32_t SLOT_BYTES = 65536;
constexpr uint32_t OFF_EQ = 0;       // [2 atoms][128 rows][128 B]: rows 0-63 b -> Ehat, 64-127 q -> Qhat
constexpr uint32_t OFF_KT = 32768;   // [2][64][128 B]: k -> Ktil
constexpr uint32_t OFF_AL = 49152;   // [2][64][128 B]: alpha; later T (first 8 KB) and P (next 8 KB)
constexpr uint32_t SM_VW = 131072;   // 2 slots x 32 KB: v [2][64][128B], w [2][64][128B]
constexpr uint32_t VW_BYTES = 32768;
constexpr uint32_t SM_KB = 196608;   // Kbar^T [1 atom][128 rows][128 B]
constexpr uint32_t SM_ASCR = 212992; // A fp32 [64][64], float4 columns XOR-swizzled by row
constexpr uint32_t SM_GAM = 229376;  // gamma, 3 slots x 128 floats (slot n % 3: the prologue runs at most
                                     // two chunks ahead of the scan's last read of gamma)
constexpr uint32_t SM_BAR = 230912;  // mbarriers, tensor memory base, abort flag
constexpr uint32_t SM_END = SM_BAR + 256;
constexpr size_t kSmemBytes = SM_END + 1024;

enum Bar {
    B_FULL = 0,     // +slot: raw q, k, alpha, b tiles landed
    B_VWFULL = 2,   // +slot: v, w tiles landed
    B_X1 = 4,
    B_READY = 5,    // +slot: Ehat, Qhat, Ktil written (operands of X2)
    B_TREADY = 7,   // +slot: T and P written
    B_KBREADY = 9,
    B_KBFREE = 10,
    B_X2A = 11,
    B_X2B = 12,
    B_X3 = 13,
    B_X45 = 14,
    B_COUNT = 15
};

struct Params {
    Problem pb;
    const void* alpha;  // scalar-gate reads
    const void* b;
    const void* z;
    const float* h0;
    void* o;
    int o_type;  // 0: bf16, 1: fp32
    float* ht;
    int* err;    // device error word (bit 0: a bounded wait expired)
};

__device__ __forceinline__ float bf(const uint8_t* tile, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}
__device__ __forceinline__ void put_bf(uint8_t* tile, uint32_t off, float v) {
    *reinterpret_cast<__nv_bfloat16*>(tile + off) = __float2bfloat16_rn(v);
}
__device__ __forceinline__ uint32_t ascr_index(int r, int c) {  // fp32 element index
    return (uint32_t)r * 64u + ((uint32_t)((c >> 2) ^ (r & 15)) << 2) + (uint32_t)(c & 3);
}

struct Ctx {
    uint8_t* sm;
    uint64_t* bars;
    volatile int* abort_flag;
    int* err;
};

// Bounded wait that also gives up as soon as another thread has aborted.
__device__ __forceinline__ bool wait_bar(const Ctx& cx, int bar, uint32_t parity) {
    uint64_t* b = cx.bars + bar;
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(b, parity)) return true;
        if (*cx.abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            *cx.abort_flag = 1;
            atomicOr(cx.err, 1);
            return false;
        }
    }
}

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                     int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

template <bool APC, bool GPC>
__device__ __forceinline__ void issue_tma(const Ctx& cx, int n, int b, int hk, int hv, const CUtensorMap* tq,
                                          const CUtensorMap* tk, const CUtensorMap* tv, const CUtensorMap* ta,
                                          const CUtensorMap* tb_, const CUtensorMap* tw) {
    const int s = n & 1, t0 = n * C;
    const uint32_t slot = smem_u32(cx.sm) + s * SLOT_BYTES;
    uint64_t* full = cx.bars + B_FULL + s;
    mbar_arrive_expect_tx(full, 32768u + (GPC ? 16384u : 0u) + (APC ? 16384u : 0u));
    tma4(slot + OFF_EQ + 8192, tq, full, 0, hk, t0, b);           // q -> rows 64-127, channels 0-63
    tma4(slot + OFF_EQ + 16384 + 8192, tq, full, 64, hk, t0, b);  // channels 64-127
    tma4(slot + OFF_KT, tk, full, 0, hk, t0, b);
    tma4(slot + OFF_KT + 8192, tk, full, 64, hk, t0, b);
    if (GPC) {
        tma4(slot + OFF_EQ, tb_, full, 0, hv, t0, b);              // b -> rows 0-63
        tma4(slot + OFF_EQ + 16384, tb_, full, 64, hv, t0, b);
    }
    if (APC) {
        tma4(slot + OFF_AL, ta, full, 0, hv, t0, b);
        tma4(slot + OFF_AL + 8192, ta, full, 64, hv, t0, b);
    }
    uint64_t* vwf = cx.bars + B_VWFULL + s;
    const uint32_t vw = smem_u32(cx.sm) + SM_VW + s * VW_BYTES;
    mbar_arrive_expect_tx(vwf, GPC ? 32768u : 16384u);
    tma4(vw, tv, vwf, 0, hv, t0, b);
    tma4(vw + 8192, tv, vwf, 64, hv, t0, b);
    if (GPC) {
        tma4(vw + 16384, tw, vwf, 0, hv, t0, b);
        tma4(vw + 16384 + 8192, tw, vwf, 64, hv, t0, b);
    }
}

template <bool APC, bool GPC, bool GATE, class TG>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w, Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctx cx;
    cx.sm = sm;
    cx.bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_BAR + 128);
    cx.abort_flag = reinterpret_cast<volatile int*>(sm + SM_BAR + 132);
    cx.err = p.err;
    float* gam = reinterpret_cast<float*>(sm + SM_GAM);

    const Problem& pb = p.pb;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int b = blockIdx.x / pb.Hv, hv = blockIdx.x % pb.Hv;
    const int hk = pb.key_head(hv);
    const int NT = pb.NT;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(cx.bars + i, 1);
        *cx.abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    int issued = 0;  // chunks whose TMA loads thread 0 has issued
    if (tid == 0) {
        for (; issued < 2 && issued < NT; ++issued)
            issue_tma<APC, GPC>(cx, issued, b, hk, hv, &tm_q, &tm_k, &tm_v, &tm_a, &tm_b, &tm_w);
    }

    if (warp < 8) {
        // =================================== state scan ===================================
        const int j = tid & 127, h = tid >> 7;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tl = tbase + lane_base;
        const long soff = pb.state_off(b, hv);
        float S[64];  // S[c'] = state[64h + c'][j]
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = p.h0 ? p.h0[soff + (long)(64 * h + c) * D + j] : 0.f;
        {
            uint32_t pk[16];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(S[32 * q2 + 2 * i], S[32 * q2 + 2 * i + 1]);
                tmem_st16(tl + TM_S0 + 32 * h + 16 * q2, pk);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        named_bar(1, 256);

        const TG* beta = static_cast<const TG*>(p.b);
        for (int n = 0; n < NT; ++n) {
            const int s = n & 1;
            const uint32_t par = (n >> 1) & 1, pn = n & 1;
            const int t0 = n * C, L = min(C, pb.T - t0);
            const uint32_t slot = smem_u32(sm) + s * SLOT_BYTES;
            // ---- X2 = S0^T [Ehat;Qhat]^T ------------------------------------------------------
            if (tid == 0) {
                tc_fence_after();
                if (wait_bar(cx, B_READY + s, par) && !*cx.abort_flag) {
                    const uint32_t id64 = idesc_bf16_f32(128, 64);
                    mma_ts_k(tbase + TM_X2, tbase + TM_S0, slot + OFF_EQ, 128, 128, id64, false);
                    mma_commit(cx.bars + B_X2A);
                    mma_ts_k(tbase + TM_X2 + 64, tbase + TM_S0, slot + OFF_EQ + 8192, 128, 128, id64, false);
                    mma_commit(cx.bars + B_X2B);
                }
            }
            // ---- Y^T = Z^T - (Ehat S0)^T  (tensor memory, bf16) -----------------------------
            wait_bar(cx, B_X2A, pn);
            wait_bar(cx, B_VWFULL + s, par);
            tc_fence_after();
            {
                uint32_t r[32];
                tmem_ld32(tl + TM_X2 + 32 * h, r);
                tmem_ld_wait();
                const uint8_t* vt = sm + SM_VW + s * VW_BYTES;
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float y2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int rr = 32 * h + 2 * i + e;
                        const uint32_t off = sw128_offset(rr, j, 64);
                        const float vv = bf(vt, off);
                        float ww;
                        if (GPC) ww = bf(vt + 16384, off);
                        else ww = rr < L ? to_f32(beta[pb.gate_row(b, t0 + rr, hv, 1)]) : 0.f;
                        y2[e] = vv * ww - __uint_as_float(r[2 * i + e]);
                    }
                    pk[i] = pack_bf16x2(y2[0], y2[1]);
                }
                tmem_st16(tl + TM_Y + 16 * h, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            named_bar(1, 256);
            // ---- X3 = Y^T T^T = V'^T -----------------------------------------------------------
            if (tid == 0) {
                tc_fence_after();
                if (wait_bar(cx, B_TREADY + s, par) && !*cx.abort_flag) {
                    mma_ts_k(tbase + TM_X3, tbase + TM_Y, slot + OFF_AL, 64, 64, idesc_bf16_f32(128, 64), false);
                    mma_commit(cx.bars + B_X3);
                }
            }
            wait_bar(cx, B_X3, pn);
            tc_fence_after();
            {
                uint32_t r[32], pk[16];
                tmem_ld32(tl + TM_X3 + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                tmem_st16(tl + TM_Y + 16 * h, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            named_bar(1, 256);
            // ---- X4 (O += V'^T P^T), X5 (dS^T = V'^T Kbar) --------------------------------------
            if (tid == 0) {
                tc_fence_after();
                if (wait_bar(cx, B_KBREADY, pn) && !*cx.abort_flag) {
                    mma_ts_k(tbase + TM_X2 + 64, tbase + TM_Y, slot + OFF_AL + 8192, 64, 64, idesc_bf16_f32(128, 64),
                             true);
                    mma_ts_k(tbase + TM_X5, tbase + TM_Y, smem_u32(sm) + SM_KB, 128, 64, idesc_bf16_f32(128, 128),
                             false);
                    mma_commit(cx.bars + B_X45);
                    mma_commit(cx.bars + B_KBFREE);
                }
            }
            const bool done45 = wait_bar(cx, B_X45, pn);
            tc_fence_after();
            if (tid == 0 && done45 && issued < NT && !*cx.abort_flag) {
                // slot s and its v/w slot are free again: prefetch chunk n + 2
                issue_tma<APC, GPC>(cx, issued, b, hk, hv, &tm_q, &tm_k, &tm_v, &tm_a, &tm_b, &tm_w);
                ++issued;
            }
            // ---- output rows 32h .. 32h+31 of column j -----------------------------------------
            {
                uint32_t r[32];
                tmem_ld32(tl + TM_X2 + 64 + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int rr = 32 * h + i;
                    if (rr < L) {
                        const long off = pb.v_row(b, t0 + rr, hv) + j;
                        float ov = pb.scale * __uint_as_float(r[i]);
                        if (GATE) {
                            const float zz = __bfloat162float(static_cast<const __nv_bfloat16*>(p.z)[off]);
                            ov *= zz * sigmoidf_(zz);
                        }
                        if (p.o_type == 1) static_cast<float*>(p.o)[off] = ov;
                        else static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(ov);
                    }
                }
            }
            // ---- state: S = Diag(gamma) S0 + Kbar^T V'; S0^T (bf16) for the next chunk --------------
            {
                const float* g = gam + (n % 3) * 128 + 64 * h;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t r[32], pk[16];
                    tmem_ld32(tl + TM_X5 + 64 * h + 32 * q2, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        S[32 * q2 + i] = fmaf(g[32 * q2 + i], S[32 * q2 + i], __uint_as_float(r[i]));
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(S[32 * q2 + 2 * i], S[32 * q2 + 2 * i + 1]);
                    tmem_st16(tl + TM_S0 + 32 * h + 16 * q2, pk);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            named_bar(1, 256);
            const int stop = *cx.abort_flag;
            named_bar(1, 256);
            if (stop) break;
        }
        if (p.ht && !*cx.abort_flag) {
#pragma unroll
            for (int c = 0; c < 64; ++c) p.ht[soff + (long)(64 * h + c) * D + j] = S[c];
        }
    } else {
        // =================================== chunk prologue ===================================
        const int c = tid - 256;              // key channel; also TMEM lane of X1
        const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        const TG* alpha_g = static_cast<const TG*>(p.alpha);
        const TG* beta_g = static_cast<const TG*>(p.b);
        float* ascr = reinterpret_cast<float*>(sm + SM_ASCR);
        float kr[64];
        for (int m = 0; m < NT; ++m) {
            const int s = m & 1;
            const uint32_t par = (m >> 1) & 1, pm = m & 1;
            const int t0 = m * C, L = min(C, pb.T - t0);
            uint8_t* slot = sm + s * SLOT_BYTES;
            uint8_t* EQ = slot + OFF_EQ;
            uint8_t* KT = slot + OFF_KT;
            uint8_t* AL = slot + OFF_AL;
            wait_bar(cx, B_FULL + s, par);
            // ---- cumulative decay, gated and decayed factors, in place ------------------------
            float G = 1.f;
#pragma unroll
            for (int r = 0; r < C; ++r) {
                float a = 1.f;
                if (r < L) {
                    if (APC) a = bf(AL, sw128_offset(r, c, 64));
                    else a = to_f32(alpha_g[pb.gate_row(b, t0 + r, hv, 1)]);
                }
                G *= a;
                const uint32_t oe = sw128_offset(r, c, 128), oq = sw128_offset(64 + r, c, 128);
                const uint32_t ok = sw128_offset(r, c, 64);
                const float kv = bf(KT, ok), qv = bf(EQ, oq);
                float bv;
                if (GPC) bv = bf(EQ, oe);
                else bv = r < L ? to_f32(beta_g[pb.gate_row(b, t0 + r, hv, 1)]) : 0.f;
                const float inv = 1.f / G;
                put_bf(EQ, oe, bv * kv * G);
                put_bf(EQ, oq, qv * G);
                kr[r] = kv * inv;
                put_bf(KT, ok, kr[r]);
            }
            gam[(m % 3) * 128 + c] = G;
            fence_async_shared();
            named_bar(2, 128);
            // ---- X1 = [Ehat;Qhat] Ktil^T --------------------------------------------------------
            if (c == 0) {
                tc_fence_after();
                if (!*cx.abort_flag) {
                    mma_ss_k(tbase + TM_X1, smem_u32(EQ), 128, smem_u32(KT), 64, 128, idesc_bf16_f32(128, 64), false);
                    mma_commit(cx.bars + B_X1);
                }
                mbar_arrive(cx.bars + B_READY + s);
            }
            wait_bar(cx, B_X1, pm);
            tc_fence_after();
            {
                uint32_t r[64];
                tmem_ld32(tl + TM_X1, *reinterpret_cast<uint32_t(*)[32]>(r));
                tmem_ld32(tl + TM_X1 + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
                tmem_ld_wait();
                if (c >= 64) {
                    // P row (c - 64), lower triangle with the diagonal, bf16, K-major
                    const int rr = c - 64;
                    uint8_t* Pt = AL + 8192;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s0 = 8 * ch + 2 * e;
                            const float x0 = s0 <= rr ? __uint_as_float(r[s0]) : 0.f;
                            const float x1 = s0 + 1 <= rr ? __uint_as_float(r[s0 + 1]) : 0.f;
                            w4[e] = pack_bf16x2(x0, x1);
                        }
                        *reinterpret_cast<uint4*>(Pt + sw128_offset(rr, 8 * ch, 64)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                } else {
                    // A row c, strictly lower, fp32 scratch
#pragma unroll
                    for (int q4 = 0; q4 < 16; ++q4) {
                        float4 v4;
                        v4.x = 4 * q4 + 0 < c ? __uint_as_float(r[4 * q4 + 0]) : 0.f;
                        v4.y = 4 * q4 + 1 < c ? __uint_as_float(r[4 * q4 + 1]) : 0.f;
                        v4.z = 4 * q4 + 2 < c ? __uint_as_float(r[4 * q4 + 2]) : 0.f;
                        v4.w = 4 * q4 + 3 < c ? __uint_as_float(r[4 * q4 + 3]) : 0.f;
                        *reinterpret_cast<float4*>(ascr + ascr_index(c, 4 * q4)) = v4;
                    }
                }
            }
            tc_fence_before();
            named_bar(2, 128);
            // ---- T = (I + A)^-1, column jj by the lane pair (jj, parity pp) ----------------------
            {
                const int jj = c >> 1, pp = c & 1;
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = 0.f;
                uint8_t* Tt = AL;
#pragma unroll
                for (int i = 0; i < C; ++i) {
                    float acc = 0.f;
#pragma unroll
                    for (int mm = 0; mm < (i + 1) / 2; ++mm) {
                        const int s0 = 2 * mm + pp;  // rows of this lane's parity below i
                        const float aval = ascr[ascr_index(i, s0 < C ? s0 : 0)];
                        acc = fmaf(s0 < i ? aval : 0.f, x[mm], acc);
                    }
                    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                    const float xi = i == jj ? 1.f : (i > jj ? -acc : 0.f);
                    if ((i & 1) == pp) {
                        x[i >> 1] = xi;
                        put_bf(Tt, sw128_offset(i, jj, 64), xi);
                    }
                }
            }
            fence_async_shared();
            named_bar(2, 128);
            if (c == 0) mbar_arrive(cx.bars + B_TREADY + s);
            // ---- Kbar^T row c: k * gamma / Gamma_r --------------------------------------------
            if (m > 0) wait_bar(cx, B_KBFREE, (m - 1) & 1);
            {
                uint8_t* KB = sm + SM_KB;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w4[e] = pack_bf16x2(kr[8 * ch + 2 * e] * G, kr[8 * ch + 2 * e + 1] * G);
                    *reinterpret_cast<uint4*>(KB + sw128_offset(c, 8 * ch, 128)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_async_shared();
            named_bar(2, 128);
            if (c == 0) mbar_arrive(cx.bars + B_KBREADY);
            const int stop = *cx.abort_flag;
            named_bar(2, 128);
            if (stop) break;
        }
    }

    // ---- teardown: loads still in flight after an abort are waited for (bounded) ----------------
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *cx.abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        for (int n = issued - 2 < 0 ? 0 : issued - 2; n < issued; ++n) {
            while (!mbar_try_wait(cx.bars + B_FULL + (n & 1), (n >> 1) & 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
            while (!mbar_try_wait(cx.bars + B_VWFULL + (n & 1), (n >> 1) & 1) && globaltimer_ns() - t0 < kWaitNs) {
            }
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcfwd
}  // namespace gdn
