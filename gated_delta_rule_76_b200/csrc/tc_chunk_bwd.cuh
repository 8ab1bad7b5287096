// Chunkwise backward on the 5th-generation tensor cores (sm_100a), dk = dv = 128, bf16 inputs.
//
// Reverse mode of the chunk form (Gated DeltaNet-2 summary, «Entraînement Parallèle Efficace par
// Blocs» for the forward it differentiates, «Passage Arrière Conscient des Portes» for the gated
// backward).  Per chunk, with the forward's factors Gamma, Ehat = (b.*k).*Gamma,
// Qhat = scale q.*Gamma (the readout scale is folded into Qhat, hence into P), Ktil = k./Gamma,
// Kbar = Ktil.*gamma, T = (I + A)^-1, P = lower(Qhat Ktil^T), W = T Ehat, and the forward's
// V' = T (Z - Ehat S0):
//   dV' = P^T dO + Kbar dS_end,   dY = T^T dV'   (dZ = dY: dv = w.*dY, dw = v.*dY)
//   dS0 = Qhat^T dO - W^T dV' + Diag(gamma) dS_end          (= Qhat^T dO - Ehat^T dY + ...)
//   dP = lower(dO V'^T),  dA = strict_lower(-dY V'^T)        (= -T^T (dV' Y^T) T^T)
//   dQhat = dO S0^T + dP Ktil,   dEhat = -dY S0^T + dA Ktil
//   dKtil = dA^T Ehat + dP^T Qhat,   dKbar = V' dS_end^T
// and through the factors to q, k, b (e = b.*k) and the cumulative log decay, whose gradient is
// a reverse cumulative sum over the chunk.  The derivative of gamma collects
// sum_r dKbar.*Kbar + gamma .* rowsum(dS_end .* S0).
//
// Kernels of one backward call:
//   1. the forward kernel (tc_chunk_fwd.cuh) in saving mode: the state entering every chunk
//      (fp32), V' of every token (bf16 hi/lo) and the bf16 T tile of every chunk;
//   2. chunk_bwd_scan_kernel (this file): one CTA per (batch, value head), chunks in reverse;
//      the state gradient dS is carried in registers (thread j: column j), its chain per chunk
//      is  XA = dO^T P + dS^T Kbar^T (= dV'^T)  ->  XC = dO^T Qhat - dV'^T W (= dS0^T without
//      the decay term)  ->  dS = Diag(gamma) dS + XC^T;  off the chain it forms -dY^T = -dV'^T T.
//      The prologue warps build the chunk's factors, X1 and P; T is the forward's own bf16 tile,
//      copied in from the cache (the forward solved for it already); the chain warps form W^T from
//      T and the split Ehat tiles and request the next chunk's raw tiles.  It saves dS_end of
//      every chunk (fp32) and -dY of every token (bf16 hi/lo), and writes dh0;
//   3. chunk_bwd_grad_kernel (this file): persistent, one CTA per SM walking the chunks; every
//      gradient of a chunk's inputs.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "tc_chunk_fwd.cuh"
#include "umma.cuh"

namespace gdn {
namespace tcbwd {

// Optional phase timestamps of CTA 0 of the gradient kernel (compiled only with -DGDN_BWD_TRACE,
// for profiling builds): g_bwd_trace[iteration][point] = %globaltimer.
#ifdef GDN_BWD_TRACE
__device__ unsigned long long g_bwd_trace[16][16];
#define GDN_BTRACE(it, point)                                                            \
    do {                                                                                 \
        if (blockIdx.x == 0 && (it) < 16) g_bwd_trace[(it)][(point)] = globaltimer_ns(); \
    } while (0)
// The reverse scan's CTA 0: g_scan_trace[iteration][point].
__device__ unsigned long long g_scan_trace[64][32];
#define GDN_STRACE(it, point)                                                              \
    do {                                                                                   \
        if (blockIdx.x == 0 && (it) < 64) g_scan_trace[(it)][(point)] = globaltimer_ns(); \
    } while (0)
#else
#define GDN_BTRACE(it, point) \
    do {                      \
    } while (0)
#define GDN_STRACE(it, point) \
    do {                      \
    } while (0)
#endif

using namespace gdn::tc;
using tcfwd::bf;
using tcfwd::Ctx;
using tcfwd::ld16;
using tcfwd::ldf4;
using tcfwd::split8;
using tcfwd::split_pack;
using tcfwd::store_state_block;
using tcfwd::st16;
using tcfwd::l2_evict_last_policy;
using tcfwd::tma3;
using tcfwd::tma4;
using tcfwd::tma4_pol;
using tcfwd::unpack8;
using tcfwd::wait1;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint64_t kWaitNs = tcfwd::kWaitNs;

// =========================================== scan ===========================================
namespace scan {

constexpr int kThreads = 384;

// tensor memory columns
constexpr uint32_t TM_X1 = 0;     // 64:  A (lanes 0-63), P (lanes 64-127) of the prologue's chunk
constexpr uint32_t TM_XA = 64;    // 64:  dV'^T, then -dY^T
constexpr uint32_t TM_XC = 128;   // 128: dO^T Qhat - dV'^T W
constexpr uint32_t TM_DSH = 256;  // 64:  dS^T hi (bf16 pairs)
constexpr uint32_t TM_DSL = 320;  // 64:  dS^T lo
constexpr uint32_t TM_DVH = 384;  // 32:  -dV'^T hi
constexpr uint32_t TM_DVL = 416;  // 32:  -dV'^T lo
constexpr uint32_t TM_WT = 448;   // 64:  W^T = Ehat^T T^T of the chain's chunk
constexpr uint32_t TM_COLS = 512;

// shared memory (1024-byte-aligned base; bf16 tiles with the 128-byte swizzle)
constexpr uint32_t SM_RQB = 0;        // 32 KB [2][128]: TMA b (rows 0-63), q (64-127) -> [Ehat;Qhat] lo
constexpr uint32_t SM_RK = 32768;     // 16 KB [2][64]: TMA k -> Ktil hi
constexpr uint32_t SM_RA = 49152;     // 16 KB [2][64]: TMA alpha -> Ktil lo
constexpr uint32_t SM_EQ = 65536;     // 32 KB [2][128]: [Ehat;Qhat] hi
constexpr uint32_t SM_KB = 98304;     // 32 KB: Kbar hi [2][64], Kbar lo [2][64] (token rows)
constexpr uint32_t SM_P = 131072;     // 16 KB: P hi [1][64], P lo [1][64] (row s, columns r)
constexpr uint32_t SM_T = 147456;     // 8 KB [1][64]: T (row r, columns s)
constexpr uint32_t SM_WT = 155648;    // 32 KB: W^T hi [1][128], W^T lo [1][128] (row c, columns r)
constexpr uint32_t SM_DO = 188416;    // 16 KB: dO, two boxes of 64 channels x 64 tokens
constexpr uint32_t SM_DOL = 204800;   // 16 KB: dO lo (when dO is a hi/lo pair), as SM_DO
                                      // [221184, 222208): unused
constexpr uint32_t SM_GAM = 222208;   // gamma, 3 slots x 128 floats
constexpr uint32_t SM_BAR = 223744;   // mbarriers, tensor memory base, flags
constexpr uint32_t SM_RS = SM_BAR + 256;  // 4 KB: row-group products
constexpr uint32_t SM_END = SM_RS + 4096;
constexpr size_t kSmemBytes = SM_END + 1024;

enum Bar {
    B_RAW = 0,   // q, k, alpha, b of the prologue's chunk landed
    B_DO,        // dO of the scan's chunk landed
    B_X1,        // X1 complete
    B_WT,        // W^T complete
    B_PREADY,    // prologue -> scan: P, Kbar, [Ehat;Qhat] written
    B_TREADY,    // T of the chain's chunk landed (bulk copy from the forward's cache)
    B_XA,        // XA complete
    B_XCPRE,     // dO^T Qhat complete: [Ehat;Qhat] and dO may be overwritten
    B_XC,        // XC complete
    B_DY,        // -dY^T complete: T and W^T may be overwritten
    B_COUNT
};

struct Params {
    Problem pb;
    const void* alpha;     // scalar-gate reads
    const void* b;
    const float* dht;      // [B,Hv,dk,dv] or NULL
    float* dh0;            // [B,Hv,dk,dv] or NULL
    float* dsc;            // [B*Hv][NT][dv/4][dk][4]: dS_end of every chunk
    __nv_bfloat16* ny_hi;  // [B,T,Hv,dv]: -dY of every token, hi / lo
    __nv_bfloat16* ny_lo;
    const uint8_t* t_in;   // [B*Hv][NT][8 KB]: the forward's bf16 T tile of every chunk (swizzled image)
    int do_lo;             // dO given as bf16 hi + lo (the lo tiles through the sixth tensor map)
    int* err;
    uint64_t wait_ns;      // limit of every bounded wait; 0 = kWaitNs
    int* flags;            // [B*Hv] or NULL: set for a pair with a chunk outside the decay range
};


// SPLIT (scalar gates only): q and k arrive as bf16 hi/lo pairs; ta maps k lo (into the alpha
// slot) and tb_ maps q lo (into the b rows), both indexed by the key head.
template <bool APC, bool GPC, bool SPLIT>
__device__ __forceinline__ void scan_load_raw(const Ctx& cx, int n, int b, int hk, int hv, const CUtensorMap* tq,
                                         const CUtensorMap* tk, const CUtensorMap* ta, const CUtensorMap* tb_) {
    const int t0 = n * C;
    const uint32_t base = smem_u32(cx.sm);
    uint64_t* bar = cx.bars + B_RAW;
    mbar_arrive_expect_tx(bar, 32768u + (GPC || SPLIT ? 16384u : 0u) + (APC || SPLIT ? 16384u : 0u));
    if (SPLIT) {
        tma4(base + SM_RQB, tb_, bar, 0, hk, t0, b);  // q lo -> rows 0-63
        tma4(base + SM_RQB + 16384, tb_, bar, 64, hk, t0, b);
        tma4(base + SM_RA, ta, bar, 0, hk, t0, b);    // k lo
        tma4(base + SM_RA + 8192, ta, bar, 64, hk, t0, b);
    }
    tma4(base + SM_RQB + 8192, tq, bar, 0, hk, t0, b);  // q -> rows 64-127
    tma4(base + SM_RQB + 16384 + 8192, tq, bar, 64, hk, t0, b);
    tma4(base + SM_RK, tk, bar, 0, hk, t0, b);
    tma4(base + SM_RK + 8192, tk, bar, 64, hk, t0, b);
    if (GPC) {
        tma4(base + SM_RQB, tb_, bar, 0, hv, t0, b);  // b -> rows 0-63
        tma4(base + SM_RQB + 16384, tb_, bar, 64, hv, t0, b);
    }
    if (APC) {
        tma4(base + SM_RA, ta, bar, 0, hv, t0, b);
        tma4(base + SM_RA + 8192, ta, bar, 64, hv, t0, b);
    }
}

__device__ __forceinline__ void scan_load_do(const Ctx& cx, int n, int b, int hv, const CUtensorMap* tdo,
                                             const CUtensorMap* tdol, bool lo) {
    const uint32_t dst = smem_u32(cx.sm) + SM_DO, dsl = smem_u32(cx.sm) + SM_DOL;
    uint64_t* bar = cx.bars + B_DO;
    mbar_arrive_expect_tx(bar, lo ? 32768u : 16384u);
    tma4(dst, tdo, bar, 0, hv, n * C, b);
    tma4(dst + 8192, tdo, bar, 64, hv, n * C, b);
    if (lo) {
        tma4(dsl, tdol, bar, 0, hv, n * C, b);
        tma4(dsl + 8192, tdol, bar, 64, hv, n * C, b);
    }
}

template <bool APC, bool GPC, class TG, bool SPLIT, bool LG>
__global__ void __launch_bounds__(kThreads, 1)
chunk_bwd_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dol,
                      Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.sm = sm;
    cx.bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_BAR + 128);
    cx.abort_flag = reinterpret_cast<volatile int*>(sm + SM_BAR + 132);
    cx.err = p.err;
    cx.wait_ns = p.wait_ns ? p.wait_ns : kWaitNs;
    float* gam = reinterpret_cast<float*>(sm + SM_GAM);
    const bool dol = p.do_lo != 0;

    const Problem& pb = p.pb;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int b = blockIdx.x / pb.Hv, hv = blockIdx.x % pb.Hv;
    const int hk = pb.key_head(hv);
    const int NT = pb.NT;
    const uint32_t sbase = smem_u32(sm);

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
    // Chunks are processed in reverse: iteration i works on chunk NT - 1 - i.
    int raw_issued = 0, do_issued = 0, t_issued = 0;  // meaningful in thread 0, which issues every load
    // T of chunk n: the forward's tile, copied in once the scan's last reader of the previous T (its
    // -dY product) has completed
    auto load_t = [&](int n) {
        mbar_arrive_expect_tx(cx.bars + B_TREADY, 8192u);
        bulk_g2s(sbase + SM_T, p.t_in + ((long)blockIdx.x * NT + n) * 8192, 8192u, cx.bars + B_TREADY);
        ++t_issued;
    };
    if (tid == 0) {
        scan_load_raw<APC, GPC, SPLIT>(cx, NT - 1, b, hk, hv, &tm_q, &tm_k, &tm_a, &tm_b);
        raw_issued = 1;
        scan_load_do(cx, NT - 1, b, hv, &tm_do, &tm_dol, dol);
        do_issued = 1;
        load_t(NT - 1);
    }

    if (warp < 8) {
        // ================================ state-gradient scan ================================
        const int j = tid & 127, h = tid >> 7;
        volatile int* stop_slot = reinterpret_cast<volatile int*>(sm + SM_BAR + 136);
        const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        const long soff = pb.state_off(b, hv);
        const uint32_t id64 = idesc_bf16_f32(128, 64), id128 = idesc_bf16_f32(128, 128);
        const uint32_t id_dop = idesc_bf16_f32_mn(128, 64, true, true);    // dO^T P
        const uint32_t id_doq = idesc_bf16_f32_mn(128, 128, true, true);   // dO^T Qhat
        const uint32_t id_dy = idesc_bf16_f32_mn(128, 64, false, true);    // (-dV'^T) T
        const uint32_t id_wt = idesc_bf16_f32_mn(128, 64, true, false);    // Ehat^T (MN-major) x T
        float S[64];  // S[c'] = dS[64h + c'][j]
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = p.dht ? p.dht[soff + (long)(64 * h + c) * D + j] : 0.f;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) split_pack(S[32 * q2 + 2 * i], S[32 * q2 + 2 * i + 1], hi[i], lo[i]);
            tmem_st16(tl + TM_DSH + 32 * h + 16 * q2, hi);
            tmem_st16(tl + TM_DSL + 32 * h + 16 * q2, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, 256);

        for (int i = 0; i < NT; ++i) {
            const int n = NT - 1 - i;
            const uint32_t pi = i & 1;
            const int t0 = n * C, L = min(C, pb.T - t0);
            // ---- XA = dS^T Kbar^T + dO^T P (= dV'^T);  XC = dO^T Qhat ----------------------------
            if (tid == 0) {
                GDN_STRACE(i, 0);
                tc_fence_after();
                if (wait1(cx, B_PREADY, pi) && wait1(cx, B_DO, pi) && !*cx.abort_flag) {
                    GDN_STRACE(i, 1);
                    mma_ts_u<128, 64>(tbase + TM_XA, tbase + TM_DSH, sbase + SM_KB, id64, false);
                    mma_ts_u<128, 64>(tbase + TM_XA, tbase + TM_DSL, sbase + SM_KB, id64, true);
                    mma_ts_u<128, 64>(tbase + TM_XA, tbase + TM_DSH, sbase + SM_KB + 16384, id64, true);
#pragma unroll
                    for (int k = 0; k < 64; k += 16) {
                        const uint64_t da = sdesc_mn_sw128(sbase + SM_DO + (uint32_t)k * 128u, 8192u);
                        mma_ss(tbase + TM_XA, da, sdesc_mn_sw128(sbase + SM_P + (uint32_t)k * 128u, 8192u), id_dop, 1u);
                        mma_ss(tbase + TM_XA, da, sdesc_mn_sw128(sbase + SM_P + 8192u + (uint32_t)k * 128u, 8192u),
                               id_dop, 1u);
                        if (dol)
                            mma_ss(tbase + TM_XA, sdesc_mn_sw128(sbase + SM_DOL + (uint32_t)k * 128u, 8192u),
                                   sdesc_mn_sw128(sbase + SM_P + (uint32_t)k * 128u, 8192u), id_dop, 1u);
                    }
                    mma_commit(cx.bars + B_XA);
#pragma unroll
                    for (int k = 0; k < 64; k += 16) {
                        const uint64_t da = sdesc_mn_sw128(sbase + SM_DO + (uint32_t)k * 128u, 8192u);
                        mma_ss(tbase + TM_XC, da, sdesc_mn_sw128(sbase + SM_EQ + 8192u + (uint32_t)k * 128u, 16384u),
                               id_doq, k > 0 ? 1u : 0u);
                        mma_ss(tbase + TM_XC, da, sdesc_mn_sw128(sbase + SM_RQB + 8192u + (uint32_t)k * 128u, 16384u),
                               id_doq, 1u);
                        if (dol)
                            mma_ss(tbase + TM_XC, sdesc_mn_sw128(sbase + SM_DOL + (uint32_t)k * 128u, 8192u),
                                   sdesc_mn_sw128(sbase + SM_EQ + 8192u + (uint32_t)k * 128u, 16384u), id_doq, 1u);
                    }
                    mma_commit(cx.bars + B_XCPRE);
                    wait1(cx, B_XA, pi);
                    GDN_STRACE(i, 2);
                }
            }
            named_bar(1, 256);
            tc_fence_after();
            // ---- -dV'^T, split, as the A operand of XC and -dY ------------------------------------
            {
                uint32_t r[32], hi[16], lo[16];
                tmem_ld32(tl + TM_XA + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int i2 = 0; i2 < 16; ++i2)
                    split_pack(-__uint_as_float(r[2 * i2]), -__uint_as_float(r[2 * i2 + 1]), hi[i2], lo[i2]);
                tmem_st16(tl + TM_DVH + 16 * h, hi);
                tmem_st16(tl + TM_DVL + 16 * h, lo);
                tmem_st_wait();
            }
            tc_fence_before();
            named_bar(1, 256);
            // ---- W^T = Ehat^T T^T once the prologue has written T; then the raw stage is free ------
            if (tid == 0) {
                tc_fence_after();
                GDN_STRACE(i, 3);
                if (wait1(cx, B_TREADY, pi) && !*cx.abort_flag) {
#pragma unroll
                    for (int k = 0; k < 64; k += 16) {
                        const uint64_t dt = sdesc_k_sw128(sbase + SM_T + (uint32_t)k * 2u);
                        mma_ss(tbase + TM_WT, sdesc_mn_sw128(sbase + SM_EQ + (uint32_t)k * 128u, 16384u), dt, id_wt,
                               k > 0 ? 1u : 0u);
                        mma_ss(tbase + TM_WT, sdesc_mn_sw128(sbase + SM_RQB + (uint32_t)k * 128u, 16384u), dt, id_wt, 1u);
                    }
                    mma_commit(cx.bars + B_WT);
                    wait1(cx, B_WT, pi);
                    // X1, XC's dO^T Qhat and W^T were the last readers of the raw stage.
                    if (raw_issued < NT && wait1(cx, B_XCPRE, pi) && !*cx.abort_flag) {
                        scan_load_raw<APC, GPC, SPLIT>(cx, NT - 1 - raw_issued, b, hk, hv, &tm_q, &tm_k, &tm_a, &tm_b);
                        ++raw_issued;
                    }
                }
                GDN_STRACE(i, 4);
            }
            named_bar(1, 256);
            tc_fence_after();
            {
                // W^T row j, columns 32 h .. 32 h + 31, split (K-major B operand of XC).
                uint8_t* WT = sm + SM_WT;
                uint32_t r[32];
                tmem_ld32(tl + TM_WT + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t wh[4], wl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 8 * ch + 2 * e;
                        split_pack(__uint_as_float(r[i0]), __uint_as_float(r[i0 + 1]), wh[e], wl[e]);
                    }
                    const uint32_t off = sw128_offset(j, 32 * h + 8 * ch, 128);
                    st16(WT + off, make_uint4(wh[0], wh[1], wh[2], wh[3]));
                    st16(WT + 16384 + off, make_uint4(wl[0], wl[1], wl[2], wl[3]));
                }
            }
            fence_async_shared();
            tc_fence_before();
            named_bar(1, 256);
            // ---- XC += (-dV'^T) W;  XA = (-dV'^T) T (= -dY^T);  next dO ----------------------------
            if (tid == 0) {
                tc_fence_after();
                if (!*cx.abort_flag) {
                    mma_ts_u<64, 128>(tbase + TM_XC, tbase + TM_DVH, sbase + SM_WT, id128, true);
                    mma_ts_u<64, 128>(tbase + TM_XC, tbase + TM_DVL, sbase + SM_WT, id128, true);
                    mma_ts_u<64, 128>(tbase + TM_XC, tbase + TM_DVH, sbase + SM_WT + 16384, id128, true);
                    mma_commit(cx.bars + B_XC);
#pragma unroll
                    for (int k = 0; k < 64; k += 16) {
                        const uint64_t dt = sdesc_mn_sw128(sbase + SM_T + (uint32_t)k * 128u, 8192u);
                        mma_ts(tbase + TM_XA, tbase + TM_DVH + (uint32_t)(k >> 1), dt, id_dy, k > 0 ? 1u : 0u);
                        mma_ts(tbase + TM_XA, tbase + TM_DVL + (uint32_t)(k >> 1), dt, id_dy, 1u);
                    }
                    mma_commit(cx.bars + B_DY);
                }
                if (do_issued < NT && wait1(cx, B_XCPRE, pi) && !*cx.abort_flag) {
                    scan_load_do(cx, NT - 1 - do_issued, b, hv, &tm_do, &tm_dol, dol);
                    ++do_issued;
                }
                wait1(cx, B_XC, pi);
                GDN_STRACE(i, 5);
            }
            if (p.dsc)  // dS_end of chunk n, in the layout of the forward's chunk states
                store_state_block(p.dsc + ((long)blockIdx.x * NT + n) * (D * D), S, j, h);
            named_bar(1, 256);
            tc_fence_after();
            // ---- dS <- Diag(gamma) dS + XC^T; split for the next chunk ----------------------------
            {
                const float4* g4 = reinterpret_cast<const float4*>(gam + (i % 3) * 128 + 64 * h);
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t r[32], hi[16], lo[16];
                    tmem_ld32(tl + TM_XC + 64 * h + 32 * q2, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 g = g4[8 * q2 + i4];
                        const int e = 32 * q2 + 4 * i4;
                        S[e + 0] = fmaf(g.x, S[e + 0], __uint_as_float(r[4 * i4 + 0]));
                        S[e + 1] = fmaf(g.y, S[e + 1], __uint_as_float(r[4 * i4 + 1]));
                        S[e + 2] = fmaf(g.z, S[e + 2], __uint_as_float(r[4 * i4 + 2]));
                        S[e + 3] = fmaf(g.w, S[e + 3], __uint_as_float(r[4 * i4 + 3]));
                    }
#pragma unroll
                    for (int i2 = 0; i2 < 16; ++i2)
                        split_pack(S[32 * q2 + 2 * i2], S[32 * q2 + 2 * i2 + 1], hi[i2], lo[i2]);
                    tmem_st16(tl + TM_DSH + 32 * h + 16 * q2, hi);
                    tmem_st16(tl + TM_DSL + 32 * h + 16 * q2, lo);
                }
                tmem_st_wait();
            }
            // ---- -dY of chunk n, token-major hi / lo ----------------------------------------------
            if (tid == 0) {
                GDN_STRACE(i, 6);
                tc_fence_after();
                if (wait1(cx, B_DY, pi) && i + 1 < NT && !*cx.abort_flag) load_t(n - 1);
                GDN_STRACE(i, 7);
            }
            tc_fence_before();
            named_bar(1, 256);
            tc_fence_after();
            {
                uint32_t r[32];
                tmem_ld32(tl + TM_XA + 32 * h, r);
                tmem_ld_wait();
                const long vrow = (long)pb.Hv * D;
                const long vb = pb.v_row(b, t0 + 32 * h, hv) + j;
                const int nrow = min(32, L - 32 * h);
#pragma unroll
                for (int ii = 0; ii < 32; ++ii) {
                    if (ii < nrow) {
                        const float x = __uint_as_float(r[ii]);
                        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                        p.ny_hi[vb + ii * vrow] = hi;
                        p.ny_lo[vb + ii * vrow] = __float2bfloat16_rn(x - __bfloat162float(hi));
                    }
                }
            }
            if (tid == 0) {
                GDN_STRACE(i, 8);
                *stop_slot = *cx.abort_flag;
            }
            tc_fence_before();
            named_bar(1, 256);
            if (*stop_slot) break;
        }
        if (p.dh0 && !*cx.abort_flag) {
#pragma unroll
            for (int c = 0; c < 64; ++c) p.dh0[soff + (long)(64 * h + c) * D + j] = S[c];
        }
    } else {
        // ====================================== prologue ======================================
        const int c = tid - 256;  // key channel; also the tensor-memory lane of X1 and W^T
        volatile int* stop_slot = reinterpret_cast<volatile int*>(sm + SM_BAR + 140);
        const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        const TG* alpha_g = static_cast<const TG*>(p.alpha);
        const TG* beta_g = static_cast<const TG*>(p.b);
        float* rs = reinterpret_cast<float*>(sm + SM_RS);
        uint8_t* RQB = sm + SM_RQB;
        uint8_t* RK = sm + SM_RK;
        uint8_t* RA = sm + SM_RA;
        uint8_t* EQ = sm + SM_EQ;
        uint8_t* KB = sm + SM_KB;
        const uint32_t id64 = idesc_bf16_f32(128, 64);
        const float scale = pb.scale;
        for (int i = 0; i < NT; ++i) {
            const int n = NT - 1 - i;
            const uint32_t pi = i & 1;
            const int t0 = n * C, L = min(C, pb.T - t0);
            if (c == 0) {
                GDN_STRACE(i, 16);
                wait1(cx, B_RAW, pi);
                GDN_STRACE(i, 17);
            }
            named_bar(2, 128);
            // ---- cumulative decay; split operands (hi -> EQ / RK, lo -> RQB / RA), split Kbar -----
            // Thread c: channels 8 cg .. 8 cg + 7 of rows 8 rg .. 8 rg + 7; Gamma over the chunk is
            // the product of the row groups' products.
            {
                const int cg = c & 15, rg = c >> 4, r0 = 8 * rg;
                const uint32_t a64 = (uint32_t)(cg >> 3) * 64u * 128u + (uint32_t)r0 * 128u;
                const uint32_t a128 = (uint32_t)(cg >> 3) * 128u * 128u + (uint32_t)r0 * 128u;
                const uint32_t ch = (uint32_t)(cg & 7);
                float* part = rs;  // [8][128]
                float Gl[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) Gl[e] = 1.f;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = r0 + u;
                    float a8[8];
                    if (APC) {
                        unpack8(ld16(RA + a64 + u * 128u + ((ch ^ u) << 4)), a8);
                        if constexpr (LG) {  // alpha from its logit
#pragma unroll
                            for (int e_ = 0; e_ < 8; ++e_) a8[e_] = pb.alpha_t<LG>(hv, a8[e_]);
                        }
                        if (r >= L) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) a8[e] = 1.f;
                        }
                    } else {
                        const float av = gate_or<1, LG>(alpha_g, pb, b, t0, r, L, hv, 1.f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) a8[e] = av;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) Gl[e] *= a8[e];
                }
                *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg) = make_float4(Gl[0], Gl[1], Gl[2], Gl[3]);
                *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg + 4) = make_float4(Gl[4], Gl[5], Gl[6], Gl[7]);
                named_bar(2, 128);
                float G[8], gm[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) G[e] = gm[e] = 1.f;
#pragma unroll
                for (int g2 = 0; g2 < 8; ++g2) {
                    const float4 p0 = ldf4(part + g2 * 128 + 8 * cg), p1 = ldf4(part + g2 * 128 + 8 * cg + 4);
                    const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (g2 < rg) G[e] *= pv[e];
                        gm[e] *= pv[e];
                    }
                }
                if (rg == 0) {
                    float* gs = gam + (i % 3) * 128 + 8 * cg;
                    *reinterpret_cast<float4*>(gs) = make_float4(gm[0], gm[1], gm[2], gm[3]);
                    *reinterpret_cast<float4*>(gs + 4) = make_float4(gm[4], gm[5], gm[6], gm[7]);
                    if (p.flags) {
                        bool out = false;
#pragma unroll
                        for (int e = 0; e < 8; ++e) out |= seq::decay_out_of_range(gm[e]);
                        if (out) p.flags[blockIdx.x] = 1;  // the pair is recomputed exactly
                    }
                }
#pragma unroll 2
                for (int u = 0; u < 8; ++u) {
                    const int r = r0 + u;
                    const uint32_t sw = (ch ^ (uint32_t)u) << 4;
                    const uint32_t o64 = a64 + u * 128u + sw, oe = a128 + u * 128u + sw, oq = oe + 64u * 128u;
                    float a8[8], k8[8], q8[8], b8[8];
                    if (APC) {
                        unpack8(ld16(RA + o64), a8);
                        if constexpr (LG) {  // alpha from its logit
#pragma unroll
                            for (int e_ = 0; e_ < 8; ++e_) a8[e_] = pb.alpha_t<LG>(hv, a8[e_]);
                        }
                        if (r >= L) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) a8[e] = 1.f;
                        }
                    } else {
                        const float av = gate_or<1, LG>(alpha_g, pb, b, t0, r, L, hv, 1.f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) a8[e] = av;
                    }
                    unpack8(ld16(RK + o64), k8);
                    unpack8(ld16(RQB + oq), q8);
                    if (SPLIT) {  // + the lo halves (read before this thread overwrites them below)
                        float kl[8], ql[8];
                        unpack8(ld16(RA + o64), kl);
                        unpack8(ld16(RQB + oe), ql);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            k8[e] += kl[e];
                            q8[e] += ql[e];
                        }
                    }
                    if (GPC) {
                        unpack8(ld16(RQB + oe), b8);
                        if constexpr (LG) {  // b from its logit
#pragma unroll
                            for (int e_ = 0; e_ < 8; ++e_) b8[e_] = pb.sig_t<LG>(b8[e_]);
                        }
                    } else {
                        const float bv = gate_or<2, LG>(beta_g, pb, b, t0, r, L, hv, 0.f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) b8[e] = bv;
                    }
                    float e8[8], qq[8], kt[8], kb[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        G[e] *= a8[e];
                        e8[e] = b8[e] * k8[e] * G[e];
                        qq[e] = scale * q8[e] * G[e];
                        kt[e] = __fdividef(k8[e], G[e]);
                        kb[e] = kt[e] * gm[e];
                    }
                    uint4 hi, lo;
                    split8(e8, hi, lo);
                    st16(EQ + oe, hi);
                    st16(RQB + oe, lo);
                    split8(qq, hi, lo);
                    st16(EQ + oq, hi);
                    st16(RQB + oq, lo);
                    split8(kt, hi, lo);
                    st16(RK + o64, hi);
                    st16(RA + o64, lo);
                    split8(kb, hi, lo);
                    st16(KB + o64, hi);
                    st16(KB + 16384 + o64, lo);
                }
            }
            fence_async_shared();
            named_bar(2, 128);
            // ---- X1 = [Ehat;Qhat] Ktil^T ----------------------------------------------------------
            if (c == 0) {
                GDN_STRACE(i, 18);
                tc_fence_after();
                if (!*cx.abort_flag) {
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_EQ, sbase + SM_RK, id64, false);
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_EQ, sbase + SM_RA, id64, true);
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_RQB, sbase + SM_RK, id64, true);
                    mma_commit(cx.bars + B_X1);
                }
                wait1(cx, B_X1, pi);
            }
            named_bar(2, 128);
            tc_fence_after();
            if (c >= 64) {
                // P row s = c - 64 (lanes 64-127), lower with the diagonal, split: row s, columns r.
                const int rr = c - 64;
                uint8_t* Ph = sm + SM_P;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tl + TM_X1 + 32 * half, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t wh[4], wl[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = 8 * ch + 2 * e, s0 = 32 * half + i0;
                            const float x0 = s0 <= rr ? __uint_as_float(r[i0]) : 0.f;
                            const float x1 = s0 + 1 <= rr ? __uint_as_float(r[i0 + 1]) : 0.f;
                            split_pack(x0, x1, wh[e], wl[e]);
                        }
                        const uint32_t off = sw128_offset(rr, 32 * half + 8 * ch, 64);
                        st16(Ph + off, make_uint4(wh[0], wh[1], wh[2], wh[3]));
                        st16(Ph + 8192 + off, make_uint4(wl[0], wl[1], wl[2], wl[3]));
                    }
                }
            }
            fence_async_shared();
            tc_fence_before();
            named_bar(2, 128);
            if (c == 0) {
                GDN_STRACE(i, 19);
                mbar_arrive(cx.bars + B_PREADY);
            }
            if (c == 0) *stop_slot = *cx.abort_flag;
            named_bar(2, 128);
            if (*stop_slot) break;
        }
    }

    // ---- teardown: TMA loads still in flight after an abort are waited for (bounded) -----------
    tc_fence_before();
    __syncthreads();
    if (*cx.abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        if (tid == 0 && do_issued > 0)
            while (!mbar_try_wait(cx.bars + B_DO, (uint32_t)((do_issued - 1) & 1)) && globaltimer_ns() - t0 < cx.wait_ns) {
            }
        if (tid == 0 && raw_issued > 0)
            while (!mbar_try_wait(cx.bars + B_RAW, (uint32_t)((raw_issued - 1) & 1)) &&
                   globaltimer_ns() - t0 < cx.wait_ns) {
            }
        if (tid == 0 && t_issued > 0)
            while (!mbar_try_wait(cx.bars + B_TREADY, (uint32_t)((t_issued - 1) & 1)) &&
                   globaltimer_ns() - t0 < cx.wait_ns) {
            }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace scan

// ======================================== gradients ========================================
// Persistent: one CTA per SM walks the chunks ci = blockIdx.x, blockIdx.x + gridDim.x, ...
// (ci = (b * Hv + hv) * NT + n), 256 threads in two groups of four warps.  Per chunk:
//   P6 = G V'^T,  G = [dO; -dY]                      -> [dP; dA] after the masks (lanes: rows)
//   P7 = S0 G^T + Ktil^T [dP; dA]^T                  -> [dQhat^T | dEhat^T]   (lanes: channels)
//   P8 = [Qhat^T | Ehat^T] [dP; dA]                  -> dKtil^T
//   P9 = dS_end V'^T                                 -> dKbar^T
// S0 and dS_end are A operands in tensor memory (lane c holds row c); every other operand is a
// bf16 hi/lo pair of 128-byte-swizzled shared-memory tiles.  Once P7-P9 of chunk i are complete,
// the epilogue group (warps 0-3, lane c = channel c) writes dq, dk, db, dalpha of chunk i, walking
// the tokens from last to first so that the reverse cumulative sum of the log-decay gradient is a
// running sum per thread (its q, k, alpha, b rows from a TMA copy into tiles the products have
// finished with), then dv, dw of chunk i, while the staging group (warps 4-7) loads chunk i + 1
// (S0 and dS_end into tensor memory, the TMA tiles, the split factors).
namespace grad {

constexpr int kThreads = 256;

constexpr uint32_t TM_S0H = 0;    // 64: S0 hi (lane c, bf16 pairs along j)
constexpr uint32_t TM_S0L = 64;   // 64: S0 lo
constexpr uint32_t TM_DSH = 128;  // 64: dS_end hi
constexpr uint32_t TM_DSL = 192;  // 64: dS_end lo
constexpr uint32_t TM_P6 = 256;   // 64: P6 (lanes = rows of G), then P8
constexpr uint32_t TM_P7 = 320;   // 128: P7
constexpr uint32_t TM_P9 = 448;   // 64: P9
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t SM_RQB = 0;        // 32 KB [2][128]: TMA b (rows 0-63), q (64-127) -> [Ehat;Qhat] lo
constexpr uint32_t SM_RK = 32768;     // 16 KB [2][64]: TMA k -> Ktil hi
constexpr uint32_t SM_RA = 49152;     // 16 KB [2][64]: TMA alpha -> Ktil lo
constexpr uint32_t SM_EQ = 65536;     // 32 KB [2][128]: [Ehat;Qhat] hi
constexpr uint32_t SM_GH = 98304;     // 32 KB [2][128]: dO (rows 0-63), -dY hi (rows 64-127)
constexpr uint32_t SM_GL = 131072;    // 32 KB [2][128]: zeros (rows 0-63), -dY lo (rows 64-127)
constexpr uint32_t SM_VP = 163840;    // 32 KB: V' hi [128 channel rows][64 tokens], V' lo (MN-major operands)
constexpr uint32_t SM_DPA = 196608;   // 32 KB: [dP;dA] hi [1][128], lo [1][128]
constexpr uint32_t SM_BAR = 229376;   // mbarriers, tensor memory base, flags
constexpr uint32_t SM_XSLOT = SM_BAR + 256;   // [128] rowsum(dS_end .* S0) of the staged chunk
constexpr uint32_t SM_GSLOT = SM_BAR + 768;   // [128] gamma (the chunk's total decay) of the staged chunk
constexpr uint32_t SM_END = SM_BAR + 1280;
constexpr size_t kSmemBytes = SM_END + 1024;
// Epilogue scratch: the zero rows 0-63 of the G lo tile (first atom column, 8 KB) are free while
// the epilogue runs; the epilogue zeroes what it used before the next chunk's P6.
constexpr uint32_t SX_DBV = 0;      // [64] sum_j dY v per token (scalar beta)
constexpr uint32_t SX_RA = 256;     // [4][64] per-warp sums over channels of d log alpha
constexpr uint32_t SX_RB = 1280;    // [4][64] per-warp sums over channels of de .* k
constexpr uint32_t SX_BYTES = 2304;

enum Bar {
    B_RAW = 0,  // q, k, alpha, b tiles of the staged chunk landed
    B_GV,       // G and V' tiles landed
    B_P6,
    B_P789,
    B_WK,       // the walk's q, k (and alpha, b, or q lo, k lo) tiles of the walked chunk landed
    B_COUNT
};
// The epilogue walk reads its q, k, alpha, b rows from a second TMA copy of the chunk's tiles, taken
// into tiles the products no longer need once P7-P9 are complete: q into the dO rows of the G hi
// tile (its two 64-channel boxes 16 KB apart), k into the second half of the [dP; dA] tile (the
// staging group's row-group products use the first), alpha and b (channel gates) or the lo halves
// of q and k (split inputs) into the V' tile.
constexpr uint32_t SW_Q = SM_GH, SW_K = SM_DPA + 16384, SW_A = SM_VP, SW_B = SM_VP + 16384;
constexpr uint32_t SW_QBOX = 16384;  // byte distance of q's second box (8 KB for the others)

struct Params {
    Problem pb;
    const void* alpha;   // global reads of the gates, q, k, v, w in the epilogue
    const void* b;
    const void* w;
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* q_lo;  // SPLIT: lo halves of q, k, v (hi in q, k, v)
    const __nv_bfloat16* k_lo;
    const __nv_bfloat16* v_lo;
    const float* s0;     // [B*Hv][NT + 1][dv/8][dk][8]: row c, columns 8q..8q+7 at float (q * dk + c) * 8
    const float* dsc;    // [B*Hv][NT][dv/4][dk][4]: row c, columns 4u..4u+3 at float4 (u * dk + c)
    void* dq;            // [B,T,Hk,dk] (direct, the gradients' type) or [B,T,Hv,dk] per value head (fp32)
    void* dk;
    void* dv;            // [B,T,Hv,dv]; this and the gate gradients in the gradients' type (fp32 or bf16)
    void* dalpha;
    void* db;
    void* dw;
    int direct;          // dq, dk written per key head (no head sharing)
    int do_lo;           // dO given as bf16 hi + lo: the lo tiles fill rows 0-63 of the G lo tile
    int* err;
    uint64_t wait_ns;    // limit of every bounded wait; 0 = kWaitNs
};

struct ChunkPos {
    long ci;
    int n, b, hv, hk, t0, L;
};

__device__ __forceinline__ ChunkPos chunk_pos(const Problem& pb, long ci) {
    ChunkPos cp;
    cp.ci = ci;
    cp.n = (int)(ci % pb.NT);
    const int bh = (int)(ci / pb.NT);
    cp.b = bh / pb.Hv;
    cp.hv = bh % pb.Hv;
    cp.hk = pb.key_head(cp.hv);
    cp.t0 = cp.n * C;
    cp.L = min(C, pb.T - cp.t0);
    return cp;
}

struct Maps {
    const CUtensorMap *q, *k, *a, *b, *dO, *yh, *yl, *vh, *vl, *dOl;
};

// SPLIT: as in the scan, m.a maps k lo and m.b maps q lo.
template <bool APC, bool GPC, bool SPLIT>
// The epilogue group reads the same q, k, alpha, b rows again with plain loads while the chunk is
// walked: the tiles are loaded with L2 evict_last priority so that those reads hit L2.
__device__ __forceinline__ void load_raw_g(const Ctx& cx, const ChunkPos& cp, const Maps& m) {
    const uint32_t base = smem_u32(cx.sm);
    uint64_t* bar = cx.bars + B_RAW;
    const uint64_t pol = l2_evict_last_policy();
    mbar_arrive_expect_tx(bar, 32768u + (GPC || SPLIT ? 16384u : 0u) + (APC || SPLIT ? 16384u : 0u));
    if (SPLIT) {
        tma4_pol(base + SM_RQB, m.b, bar, 0, cp.hk, cp.t0, cp.b, pol);  // q lo -> rows 0-63
        tma4_pol(base + SM_RQB + 16384, m.b, bar, 64, cp.hk, cp.t0, cp.b, pol);
        tma4_pol(base + SM_RA, m.a, bar, 0, cp.hk, cp.t0, cp.b, pol);    // k lo
        tma4_pol(base + SM_RA + 8192, m.a, bar, 64, cp.hk, cp.t0, cp.b, pol);
    }
    tma4_pol(base + SM_RQB + 8192, m.q, bar, 0, cp.hk, cp.t0, cp.b, pol);
    tma4_pol(base + SM_RQB + 16384 + 8192, m.q, bar, 64, cp.hk, cp.t0, cp.b, pol);
    tma4_pol(base + SM_RK, m.k, bar, 0, cp.hk, cp.t0, cp.b, pol);
    tma4_pol(base + SM_RK + 8192, m.k, bar, 64, cp.hk, cp.t0, cp.b, pol);
    if (GPC) {
        tma4_pol(base + SM_RQB, m.b, bar, 0, cp.hv, cp.t0, cp.b, pol);
        tma4_pol(base + SM_RQB + 16384, m.b, bar, 64, cp.hv, cp.t0, cp.b, pol);
    }
    if (APC) {
        tma4_pol(base + SM_RA, m.a, bar, 0, cp.hv, cp.t0, cp.b, pol);
        tma4_pol(base + SM_RA + 8192, m.a, bar, 64, cp.hv, cp.t0, cp.b, pol);
    }
}

__device__ __forceinline__ void load_gv(const Ctx& cx, const ChunkPos& cp, const Maps& m, bool dol) {
    const uint32_t base = smem_u32(cx.sm);
    uint64_t* bar = cx.bars + B_GV;
    mbar_arrive_expect_tx(bar, (dol ? 6u : 5u) * 16384u);
    if (dol) {  // rows 0-63 of the G lo tile: dO lo (else they hold zeros)
        tma4(base + SM_GL, m.dOl, bar, 0, cp.hv, cp.t0, cp.b);
        tma4(base + SM_GL + 16384, m.dOl, bar, 64, cp.hv, cp.t0, cp.b);
    }
    tma4(base + SM_GH, m.dO, bar, 0, cp.hv, cp.t0, cp.b);
    tma4(base + SM_GH + 16384, m.dO, bar, 64, cp.hv, cp.t0, cp.b);
    tma4(base + SM_GH + 8192, m.yh, bar, 0, cp.hv, cp.t0, cp.b);
    tma4(base + SM_GH + 16384 + 8192, m.yh, bar, 64, cp.hv, cp.t0, cp.b);
    tma4(base + SM_GL + 8192, m.yl, bar, 0, cp.hv, cp.t0, cp.b);
    tma4(base + SM_GL + 16384 + 8192, m.yl, bar, 64, cp.hv, cp.t0, cp.b);
    // V' hi, lo: the chunk's column-major tiles (128 channel rows of its 64 tokens)
    tma3(base + SM_VP, m.vh, bar, 0, 0, (int)cp.ci);
    tma3(base + SM_VP + 16384, m.vl, bar, 0, 0, (int)cp.ci);
}

// The walked chunk's q, k (and alpha, b with channel gates, or q lo, k lo with split inputs) tiles
// once more, into the tiles P7-P9 have finished with, for the epilogue walk.
template <bool APC, bool GPC, bool SPLIT>
__device__ __forceinline__ void load_walk(const Ctx& cx, const ChunkPos& cp, const Maps& m) {
    const uint32_t base = smem_u32(cx.sm);
    uint64_t* bar = cx.bars + B_WK;
    const bool ta = APC || SPLIT, tb = GPC || SPLIT;
    mbar_arrive_expect_tx(bar, 32768u + (ta ? 16384u : 0u) + (tb ? 16384u : 0u));
    tma4(base + SW_Q, m.q, bar, 0, cp.hk, cp.t0, cp.b);
    tma4(base + SW_Q + SW_QBOX, m.q, bar, 64, cp.hk, cp.t0, cp.b);
    tma4(base + SW_K, m.k, bar, 0, cp.hk, cp.t0, cp.b);
    tma4(base + SW_K + 8192, m.k, bar, 64, cp.hk, cp.t0, cp.b);
    if (ta) {  // alpha (value head), or q lo (key head; its map takes the b slot)
        const CUtensorMap* t = SPLIT ? m.b : m.a;
        const int h = SPLIT ? cp.hk : cp.hv;
        tma4(base + SW_A, t, bar, 0, h, cp.t0, cp.b);
        tma4(base + SW_A + 8192, t, bar, 64, h, cp.t0, cp.b);
    }
    if (tb) {  // b (value head), or k lo (key head; its map takes the alpha slot)
        const CUtensorMap* t = SPLIT ? m.a : m.b;
        const int h = SPLIT ? cp.hk : cp.hv;
        tma4(base + SW_B, t, bar, 0, h, cp.t0, cp.b);
        tma4(base + SW_B + 8192, t, bar, 64, h, cp.t0, cp.b);
    }
}

// Sum of v over the 32 lanes of a warp.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 32 bytes (8 floats) from global memory written by an earlier kernel, in one 256-bit load through
// the non-coherent path; p must be 32-byte aligned.
__device__ __forceinline__ void ldg_v8(const float* p, float4& x, float4& y) {
    asm("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w), "=f"(y.x), "=f"(y.y), "=f"(y.z), "=f"(y.w)
        : "l"(p));
}

// Staging group (128 threads, c = lane = channel): S0 and dS_end rows of the chunk into tensor
// memory as split A operands and rowsum(dS_end .* S0) into xslot[c]; then, once the raw TMA tiles
// have landed, the cumulative decay (gamma into gslot[c]) and the split [Ehat;Qhat], Ktil tiles.
template <bool APC, bool GPC, class TG, bool SPLIT, bool LG>
__device__ __forceinline__ void stage_chunk(const Params& p, const Ctx& cx, const ChunkPos& cp, uint32_t tl, int c,
                                            float* xslot, float* gslot, uint32_t raw_parity, int it = 15) {
    const Problem& pb = p.pb;
    {
        // row c: S0 columns 8v .. 8v + 7 are 32 contiguous bytes at float (v * D + c) * 8 (one
        // 256-bit load; a warp reads 1 KB contiguous), dS columns 4u .. 4u + 3 the float4 u * D + c
        const long bh = cp.ci / pb.NT;
        const float* s0r = p.s0 + (bh * (pb.NT + 1) + cp.n) * D * D + 8 * c;
        const float4* dsr = reinterpret_cast<const float4*>(p.dsc + cp.ci * D * D) + c;
        float dot = 0.f;
#pragma unroll 1
        for (int q8 = 0; q8 < 2; ++q8) {
            float4 a[16], d[16];
#pragma unroll
            for (int u = 0; u < 16; u += 2) ldg_v8(s0r + ((16 * q8 + u) >> 1) * (8 * D), a[u], a[u + 1]);
#pragma unroll
            for (int u = 0; u < 16; ++u) d[u] = __ldg(dsr + (16 * q8 + u) * D);
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
                uint32_t ah[16], al[16], dh[16], dl[16];
#pragma unroll
                for (int u8 = 0; u8 < 8; ++u8) {
                    const int u = 8 * hq + u8;
                    dot = fmaf(d[u].x, a[u].x, dot);
                    dot = fmaf(d[u].y, a[u].y, dot);
                    dot = fmaf(d[u].z, a[u].z, dot);
                    dot = fmaf(d[u].w, a[u].w, dot);
                    split_pack(a[u].x, a[u].y, ah[2 * u8], al[2 * u8]);
                    split_pack(a[u].z, a[u].w, ah[2 * u8 + 1], al[2 * u8 + 1]);
                    split_pack(d[u].x, d[u].y, dh[2 * u8], dl[2 * u8]);
                    split_pack(d[u].z, d[u].w, dh[2 * u8 + 1], dl[2 * u8 + 1]);
                }
                const int q4 = 2 * q8 + hq;
                tmem_st16(tl + TM_S0H + 16 * q4, ah);
                tmem_st16(tl + TM_S0L + 16 * q4, al);
                tmem_st16(tl + TM_DSH + 16 * q4, dh);
                tmem_st16(tl + TM_DSL + 16 * q4, dl);
            }
        }
        xslot[c] = dot;
        tmem_st_wait();
    }
    if (c == 0) GDN_BTRACE(it, 6);
    if (c == 0) wait1(cx, B_RAW, raw_parity);
    if (c == 0) GDN_BTRACE(it, 7);
    named_bar(2, 128);
    const TG* alpha_g = static_cast<const TG*>(p.alpha);
    const TG* beta_g = static_cast<const TG*>(p.b);
    uint8_t* RQB = cx.sm + SM_RQB;
    uint8_t* RK = cx.sm + SM_RK;
    uint8_t* RA = cx.sm + SM_RA;
    uint8_t* EQ = cx.sm + SM_EQ;
    float* part = reinterpret_cast<float*>(cx.sm + SM_DPA);  // [8][128]: before [dP;dA] is written, below the walk's k
    const float scale = pb.scale;
    const int b = cp.b, hv = cp.hv, t0 = cp.t0, L = cp.L;
    const int cg = c & 15, rg = c >> 4, r0 = 8 * rg;
    const uint32_t a64 = (uint32_t)(cg >> 3) * 64u * 128u + (uint32_t)r0 * 128u;
    const uint32_t a128 = (uint32_t)(cg >> 3) * 128u * 128u + (uint32_t)r0 * 128u;
    const uint32_t ch = (uint32_t)(cg & 7);
    float Gl[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) Gl[e] = 1.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int r = r0 + u;
        float a8[8];
        if (APC) {
            unpack8(ld16(RA + a64 + u * 128u + ((ch ^ u) << 4)), a8);
            if constexpr (LG) {  // alpha from its logit
#pragma unroll
                for (int e_ = 0; e_ < 8; ++e_) a8[e_] = pb.alpha_t<LG>(hv, a8[e_]);
            }
            if (r >= L) {
#pragma unroll
                for (int e = 0; e < 8; ++e) a8[e] = 1.f;
            }
        } else {
            const float av = gate_or<1, LG>(alpha_g, pb, b, t0, r, L, hv, 1.f);
#pragma unroll
            for (int e = 0; e < 8; ++e) a8[e] = av;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) Gl[e] *= a8[e];
    }
    *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg) = make_float4(Gl[0], Gl[1], Gl[2], Gl[3]);
    *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg + 4) = make_float4(Gl[4], Gl[5], Gl[6], Gl[7]);
    named_bar(2, 128);
    float G[8], gm[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) G[e] = gm[e] = 1.f;
#pragma unroll
    for (int g2 = 0; g2 < 8; ++g2) {
        const float4 p0 = ldf4(part + g2 * 128 + 8 * cg), p1 = ldf4(part + g2 * 128 + 8 * cg + 4);
        const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (g2 < rg) G[e] *= pv[e];
            gm[e] *= pv[e];
        }
    }
    if (rg == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) gslot[8 * cg + e] = gm[e];
    }

#pragma unroll 2
    for (int u = 0; u < 8; ++u) {
        const int r = r0 + u;
        const uint32_t sw = (ch ^ (uint32_t)u) << 4;
        const uint32_t o64 = a64 + u * 128u + sw, oe = a128 + u * 128u + sw, oq = oe + 64u * 128u;
        float a8[8], k8[8], q8[8], b8[8];
        if (APC) {
            unpack8(ld16(RA + o64), a8);
            if constexpr (LG) {  // alpha from its logit
#pragma unroll
                for (int e_ = 0; e_ < 8; ++e_) a8[e_] = pb.alpha_t<LG>(hv, a8[e_]);
            }
            if (r >= L) {
#pragma unroll
                for (int e = 0; e < 8; ++e) a8[e] = 1.f;
            }
        } else {
            const float av = gate_or<1, LG>(alpha_g, pb, b, t0, r, L, hv, 1.f);
#pragma unroll
            for (int e = 0; e < 8; ++e) a8[e] = av;
        }
        unpack8(ld16(RK + o64), k8);
        unpack8(ld16(RQB + oq), q8);
        if (SPLIT) {  // + the lo halves (read before this thread overwrites them below)
            float kl[8], ql[8];
            unpack8(ld16(RA + o64), kl);
            unpack8(ld16(RQB + oe), ql);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                k8[e] += kl[e];
                q8[e] += ql[e];
            }
        }
        if (GPC) {
            unpack8(ld16(RQB + oe), b8);
            if constexpr (LG) {  // b from its logit
#pragma unroll
                for (int e_ = 0; e_ < 8; ++e_) b8[e_] = pb.sig_t<LG>(b8[e_]);
            }
        } else {
            const float bv = gate_or<2, LG>(beta_g, pb, b, t0, r, L, hv, 0.f);
#pragma unroll
            for (int e = 0; e < 8; ++e) b8[e] = bv;
        }
        float e8[8], qq[8], kt[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            G[e] *= a8[e];
            e8[e] = b8[e] * k8[e] * G[e];
            qq[e] = scale * q8[e] * G[e];
            kt[e] = __fdividef(k8[e], G[e]);
        }
        uint4 hi, lo;
        split8(e8, hi, lo);
        st16(EQ + oe, hi);
        st16(RQB + oe, lo);
        split8(qq, hi, lo);
        st16(EQ + oq, hi);
        st16(RQB + oq, lo);
        split8(kt, hi, lo);
        st16(RK + o64, hi);
        st16(RA + o64, lo);
    }
    fence_async_shared();
    tc_fence_before();
}

// dv = w .* dY, dw = v .* dY (a scalar beta: sum_j v dY per token into scr[SX_DBV]); run by the
// epilogue group after its walk, warp w: tokens w, w + 4, ..., lane l: value channels 4l .. 4l + 3.

template <bool GPC, class TG, bool SPLIT, bool LG, class GT>
__device__ __forceinline__ void grad_dv_dw(const Params& p, const Ctx& cx, const ChunkPos& cp, int tt, float* scr) {
    const Problem& pb = p.pb;
    const int w = tt >> 5, l = tt & 31, j = 4 * l;
    const uint8_t* gh = cx.sm + SM_GH;
    const uint8_t* gl = cx.sm + SM_GL;
    // loads are unconditional (a row past the sequence reads its last token); stores are guarded
    uint2 vr[16], wr[16], vl[16];
    float bs[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = w + 4 * i;
        const long row = pb.v_row(cp.b, cp.t0 + min(r, cp.L - 1), cp.hv);
        vr[i] = __ldg(reinterpret_cast<const uint2*>(p.v + row + j));
        if (SPLIT) vl[i] = __ldg(reinterpret_cast<const uint2*>(p.v_lo + row + j));
        if (GPC) wr[i] = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.w) + row + j));
        else bs[i] = gate_or<2, LG>(static_cast<const TG*>(p.b), pb, cp.b, cp.t0, r, cp.L, cp.hv, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = w + 4 * i;
        const uint32_t off = sw128_offset(64 + r, j, 128);
        const uint2 yh = *reinterpret_cast<const uint2*>(gh + off), yl = *reinterpret_cast<const uint2*>(gl + off);
        float dy[4], v4[4], w4[4];
        dy[0] = -(__uint_as_float(yh.x << 16) + __uint_as_float(yl.x << 16));
        dy[1] = -(__uint_as_float(yh.x & 0xFFFF0000u) + __uint_as_float(yl.x & 0xFFFF0000u));
        dy[2] = -(__uint_as_float(yh.y << 16) + __uint_as_float(yl.y << 16));
        dy[3] = -(__uint_as_float(yh.y & 0xFFFF0000u) + __uint_as_float(yl.y & 0xFFFF0000u));
        v4[0] = __uint_as_float(vr[i].x << 16); v4[1] = __uint_as_float(vr[i].x & 0xFFFF0000u);
        v4[2] = __uint_as_float(vr[i].y << 16); v4[3] = __uint_as_float(vr[i].y & 0xFFFF0000u);
        if (SPLIT) {
            v4[0] += __uint_as_float(vl[i].x << 16); v4[1] += __uint_as_float(vl[i].x & 0xFFFF0000u);
            v4[2] += __uint_as_float(vl[i].y << 16); v4[3] += __uint_as_float(vl[i].y & 0xFFFF0000u);
        }
        if (GPC) {
            w4[0] = __uint_as_float(wr[i].x << 16); w4[1] = __uint_as_float(wr[i].x & 0xFFFF0000u);
            w4[2] = __uint_as_float(wr[i].y << 16); w4[3] = __uint_as_float(wr[i].y & 0xFFFF0000u);
            if constexpr (LG) {
#pragma unroll
                for (int e_ = 0; e_ < 4; ++e_) w4[e_] = pb.sig_t<LG>(w4[e_]);
            }
        } else {
            w4[0] = w4[1] = w4[2] = w4[3] = bs[i];
        }
        const long row = pb.v_row(cp.b, cp.t0 + min(r, cp.L - 1), cp.hv);
        if (r < cp.L) {
            st4_g(static_cast<GT*>(p.dv) + row + j, w4[0] * dy[0], w4[1] * dy[1], w4[2] * dy[2], w4[3] * dy[3]);
            if (GPC)
                st4_g(static_cast<GT*>(p.dw) + row + j, v4[0] * dy[0], v4[1] * dy[1], v4[2] * dy[2],
                      v4[3] * dy[3]);
        }
        if (!GPC) {
            const float sum = warp_sum(fmaf(v4[0], dy[0], fmaf(v4[1], dy[1], fmaf(v4[2], dy[2], v4[3] * dy[3]))));
            if (l == 0) scr[SX_DBV / 4 + r] = sum;
        }
    }
}

// Epilogue of one chunk once P7-P9 are complete (epilogue group, lane c = channel c).  Per token r
// (Gamma_r the cumulative decay, gamma = Gamma_63):
//   dq = scale Gamma dQhat,  de = Gamma dEhat,  db = de k,  dk = de b + (dKtil + gamma dKbar) / Gamma,
//   dg_r = dQhat Qhat + dEhat Ehat - (dKtil + gamma dKbar) Ktil   (derivative w.r.t. log Gamma_r),
//   d log alpha_r = sum_{r' >= r} dg_r' + X,   X = gamma (sum_r dKbar_r Ktil_r + rowsum(dS .* S0))
// (X: the chunk's total decay gamma enters S_end = Diag(gamma) S0 + Kbar^T V' and Kbar).  The tokens
// are walked from last to first (Gamma_{r-1} = Gamma_r / alpha_r) with the running sum.
constexpr int RB = 8;  // tokens per block

struct RowIn {
    float q[RB], k[RB], b[RB], a[RB];
};

// sum_r dKbar[r][c] Ktil[r][c], from P9 and the Ktil hi/lo tiles still in shared memory (before the
// next chunk's raw tiles are loaded over them).
__device__ __forceinline__ float grad_xs(const Ctx& cx, uint32_t tl, int c) {
    const uint8_t* RK = cx.sm + SM_RK;
    const uint8_t* RA = cx.sm + SM_RA;
    float xs = 0.f;
    // column c of a 64-row K-major tile: row r at cbase + 128 r + xo[r & 7]
    const uint32_t cbase = (uint32_t)(c >> 6) * 64u * 128u;
    uint32_t xo[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) xo[u] = ((uint32_t)(c & 63) * 2u) ^ ((uint32_t)u << 4);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        uint32_t rb[32];
        tmem_ld32(tl + TM_P9 + 32 * hf, rb);
        float kt[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t off = cbase + (uint32_t)(32 * hf + i) * 128u + xo[i & 7];
            kt[i] = bf(RK, off) + bf(RA, off);
        }
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) xs = fmaf(__uint_as_float(rb[i]), kt[i], xs);
    }
    return xs;
}

// Row addressing of one chunk for lane c: element offsets of token t0 + r are base + r * stride.
struct RowPtrs {
    long qk, qk_s;   // q, k (and dq, dk when direct) rows: [B,T,Hk,dk]
    long g, g_s;     // per-channel gate rows and per-value-head rows: [B,T,Hv,dk]
    long s1, s1_s;   // scalar gate rows: [B,T,Hv]
    long o, o_s;     // dq, dk rows (direct: the q/k rows; else per value head)
};

__device__ __forceinline__ RowPtrs row_ptrs(const Params& p, const ChunkPos& cp, int c) {
    const Problem& pb = p.pb;
    RowPtrs rp;
    rp.qk = pb.qk_row(cp.b, cp.t0, cp.hk) + c;
    rp.qk_s = (long)pb.Hk * D;
    rp.g = pb.gate_row(cp.b, cp.t0, cp.hv, D) + c;
    rp.g_s = (long)pb.Hv * D;
    rp.s1 = pb.gate_row(cp.b, cp.t0, cp.hv, 1);
    rp.s1_s = pb.Hv;
    rp.o = p.direct ? rp.qk : rp.g;
    rp.o_s = p.direct ? rp.qk_s : rp.g_s;
    return rp;
}

// Inputs of tokens r0 .. r0 + RB - 1.  FULL: every row of the chunk is inside the sequence; else rows
// past the sequence read its last token and are then replaced (a load under a branch would be waited
// for where the branch ends).
// The walk tiles hold channel c of token r at box (c >> 6), row r, 16-byte chunk ((c & 63) >> 3) ^ (r & 7)
// (128-byte swizzle), byte 2 (c & 7); boxes are 8 KB apart, q's SW_QBOX.
template <bool APC, bool GPC, bool FULL, class TG, bool SPLIT, bool LG>
__device__ __forceinline__ void load_rows(const Params& p, const Ctx& cx, const ChunkPos& cp, const RowPtrs& rp,
                                          int c, int r0, RowIn& x) {
    const TG* ag = static_cast<const TG*>(p.alpha);
    const TG* bg = static_cast<const TG*>(p.b);
    const uint32_t cb = (uint32_t)(c >> 6) * 8192u + (uint32_t)(c & 7) * 2u, cc = (uint32_t)((c & 63) >> 3);
    const uint8_t* wq = cx.sm + SW_Q + (uint32_t)(c >> 6) * (SW_QBOX - 8192u);
#pragma unroll
    for (int i = 0; i < RB; ++i) {
        const int r = r0 + i, rr = FULL ? r : min(r, cp.L - 1);
        const uint32_t off = cb + (uint32_t)r * 128u + ((cc ^ (uint32_t)(r & 7)) << 4);
        float q0 = bf(wq, off);
        float k0 = bf(cx.sm + SW_K, off);
        if (SPLIT) {
            q0 += bf(cx.sm + SW_A, off);
            k0 += bf(cx.sm + SW_B, off);
        }
        const float b0 = p.pb.sig_t<LG>(GPC ? bf(cx.sm + SW_B, off) : to_f32(__ldg(bg + rp.s1 + rr * rp.s1_s)));
        const float a0 = p.pb.alpha_t<LG>(cp.hv, APC ? bf(cx.sm + SW_A, off) : to_f32(__ldg(ag + rp.s1 + rr * rp.s1_s)));
        const bool in = FULL || r < cp.L;
        x.q[i] = in ? q0 : 0.f;
        x.k[i] = in ? k0 : 0.f;
        x.b[i] = in ? b0 : 0.f;
        x.a[i] = in ? a0 : 1.f;
    }
}

template <bool APC, bool GPC, bool FULL, class TG, bool SPLIT, bool LG, class GT, class QT>
__device__ __forceinline__ void grad_epilogue_t(const Params& p, const Ctx& cx, const ChunkPos& cp, uint32_t tl, int c,
                                                int warp, float gam, float xtot, float* scr, int it) {
    const float scale = p.pb.scale;
    const RowPtrs rp = row_ptrs(p, cp, c);
    float G = gam, rg = __fdividef(1.f, gam), run = 0.f;
    auto do_block = [&](int blk, const RowIn& x) {
        uint32_t rq[RB], re[RB], rk[RB], rb[RB];
        tmem_ld8(tl + TM_P7 + RB * blk, rq);
        tmem_ld8(tl + TM_P7 + 64 + RB * blk, re);
        tmem_ld8(tl + TM_P6 + RB * blk, rk);
        tmem_ld8(tl + TM_P9 + RB * blk, rb);
        tmem_ld_wait();
#pragma unroll
        for (int i = RB - 1; i >= 0; --i) {
            const int r = RB * blk + i;
            const float qv = x.q[i], kv = x.k[i], bv = x.b[i];
            const float ra = __fdividef(1.f, x.a[i]);
            const float dQh = __uint_as_float(rq[i]), dEh = __uint_as_float(re[i]);
            const float dkc = fmaf(gam, __uint_as_float(rb[i]), __uint_as_float(rk[i]));
            const float de = G * dEh;
            run += fmaf(dQh, scale * qv * G, fmaf(dEh, bv * kv * G, -dkc * kv * rg));
            const float dla = run + xtot;
            if (FULL || r < cp.L) {
                st_g(static_cast<QT*>(p.dq) + rp.o + r * rp.o_s, scale * G * dQh);
                st_g(static_cast<QT*>(p.dk) + rp.o + r * rp.o_s, fmaf(de, bv, dkc * rg));
                if (GPC) st_g(static_cast<GT*>(p.db) + rp.g + r * rp.g_s, de * kv);
                if (APC) st_g(static_cast<GT*>(p.dalpha) + rp.g + r * rp.g_s, dla * ra);
            }
            if (!GPC) {
                const float sum = warp_sum(de * kv);
                if ((c & 31) == 0) scr[SX_RB / 4 + warp * 64 + r] = sum;
            }
            if (!APC) {
                const float sum = warp_sum(dla);
                if ((c & 31) == 0) scr[SX_RA / 4 + warp * 64 + r] = sum;
            }
            G *= ra;       // Gamma_{r-1} = Gamma_r / alpha_r
            rg *= x.a[i];  // 1 / Gamma_{r-1}
        }
    };
    // two input buffers: a block's loads are in flight while the previous block is formed
    RowIn x0, x1;
    load_rows<APC, GPC, FULL, TG, SPLIT, LG>(p, cx, cp, rp, c, 7 * RB, x0);
#pragma unroll 1
    for (int blk = C / RB - 1; blk > 0; blk -= 2) {
        load_rows<APC, GPC, FULL, TG, SPLIT, LG>(p, cx, cp, rp, c, (blk - 1) * RB, x1);
        do_block(blk, x0);
        if (blk > 1) load_rows<APC, GPC, FULL, TG, SPLIT, LG>(p, cx, cp, rp, c, (blk - 2) * RB, x0);
        do_block(blk - 1, x1);
        if (c == 0) GDN_BTRACE(it, 10 + (C / RB - 1 - blk) / 2);
    }
}

// Full chunks (every chunk but a ragged last one) take the variant without per-token guards.
template <bool APC, bool GPC, class TG, bool SPLIT, bool LG, class GT, class QT>
__device__ __forceinline__ void grad_epilogue(const Params& p, const Ctx& cx, const ChunkPos& cp, uint32_t tl, int c,
                                              int warp, float gam, float xtot, float* scr, int it = 15) {
    if (cp.L == C) grad_epilogue_t<APC, GPC, true, TG, SPLIT, LG, GT, QT>(p, cx, cp, tl, c, warp, gam, xtot, scr, it);
    else grad_epilogue_t<APC, GPC, false, TG, SPLIT, LG, GT, QT>(p, cx, cp, tl, c, warp, gam, xtot, scr, it);
}

// Scalar gates: per-token sums over the channels (the epilogue group's per-warp partials, the
// dv/dw pass's sum_j v dY), then rows 0-63 of the G lo tile are zeroed again for the next P6.
template <bool APC, bool GPC, class TG, bool LG, class GT>
__device__ __forceinline__ void scalar_gate_finish(const Params& p, const ChunkPos& cp, int c, float* scr) {
    const Problem& pb = p.pb;
    // gradients in the inputs' dtypes: the scalar gates' in the gates' own type
    using SG = typename std::conditional<std::is_same<GT, float>::value, float, TG>::type;
    if (c < cp.L) {
        const long g1 = pb.gate_row(cp.b, cp.t0 + c, cp.hv, 1);
        if (!APC) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) sum += scr[SX_RA / 4 + w * 64 + c];
            st_g(static_cast<SG*>(p.dalpha) + g1,
                 sum / pb.alpha_t<LG>(cp.hv, to_f32(__ldg(static_cast<const TG*>(p.alpha) + g1))));
        }
        if (!GPC) {
            float sum = scr[SX_DBV / 4 + c];
#pragma unroll
            for (int w = 0; w < 4; ++w) sum += scr[SX_RB / 4 + w * 64 + c];
            st_g(static_cast<SG*>(p.db) + g1, sum);
        }
    }
    named_bar(2, 128);
    if (!p.do_lo) {  // with dO lo the next chunk's tiles overwrite the scratch instead
        uint4* z = reinterpret_cast<uint4*>(scr);
        for (int i = c; i < (int)(SX_BYTES / 16); i += 128) z[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_shared();
}

// Barrier 3 of all 256 threads: the epilogue group arrives (does not wait), the staging group waits.
__device__ __forceinline__ void bar_arrive_all(uint32_t id) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(kThreads) : "memory");
}
__device__ __forceinline__ void bar_sync_all(uint32_t id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kThreads) : "memory");
}

template <bool APC, bool GPC, class TG, bool SPLIT, bool LG, class GT, class QT>
__global__ void __launch_bounds__(kThreads, 1)
chunk_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_yh,
                      const __grid_constant__ CUtensorMap tm_yl, const __grid_constant__ CUtensorMap tm_vh,
                      const __grid_constant__ CUtensorMap tm_vl, const __grid_constant__ CUtensorMap tm_dol,
                      Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.sm = sm;
    cx.bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_BAR + 128);
    cx.abort_flag = reinterpret_cast<volatile int*>(sm + SM_BAR + 132);
    volatile int* stop_slot = reinterpret_cast<volatile int*>(sm + SM_BAR + 136);
    cx.err = p.err;
    cx.wait_ns = p.wait_ns ? p.wait_ns : kWaitNs;
    float* xslot = reinterpret_cast<float*>(sm + SM_XSLOT);
    float* gslot = reinterpret_cast<float*>(sm + SM_GSLOT);
    float* scr = reinterpret_cast<float*>(sm + SM_GL);

    const Problem& pb = p.pb;
    const int tid = threadIdx.x, warp = tid >> 5;
    const long nch = (long)pb.B * pb.Hv * pb.NT;
    const uint32_t sbase = smem_u32(sm);
    const Maps m{&tm_q, &tm_k, &tm_a, &tm_b, &tm_do, &tm_yh, &tm_yl, &tm_vh, &tm_vl, &tm_dol};
    const bool dol = p.do_lo != 0;

    if (tid == 0) {
        for (int i = 0; i < B_COUNT; ++i) mbar_init(cx.bars + i, 1);
        *cx.abort_flag = 0;
        *stop_slot = 0;
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
    const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    // raw and walk tiles: thread 0;  G and V' tiles: thread 128
    int raw_issued = 0, gv_issued = 0, wk_issued = 0;
    long ci = blockIdx.x;
    if (ci < nch) {
        const ChunkPos c0 = chunk_pos(pb, ci);
        if (tid == 0) {
            load_raw_g<APC, GPC, SPLIT>(cx, c0, m);
            raw_issued = 1;
        }
        if (tid == 128) {
            load_gv(cx, c0, m, dol);
            gv_issued = 1;
        }
        if (warp < 4) {
            uint8_t* gl = sm + SM_GL;  // rows 0-63 of the G lo tile: zeros when dO is exact in bf16
#pragma unroll
            for (int u = 0; u < 8 && !dol; ++u) {
                const int idx = tid + 128 * u;
                st16(gl + (uint32_t)(idx >> 9) * 16384u + (uint32_t)(idx & 511) * 16u, make_uint4(0u, 0u, 0u, 0u));
            }
        } else {
            stage_chunk<APC, GPC, TG, SPLIT, LG>(p, cx, c0, tl, tid - 128, xslot, gslot, 0u);
        }
    }
    for (int it = 0; ci < nch; ++it, ci += gridDim.x) {
        const ChunkPos cp = chunk_pos(pb, ci);
        const uint32_t par = (uint32_t)it & 1u;
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) GDN_BTRACE(it, 0);
        const long nx = ci + gridDim.x;
        // rowsum(dS_end .* S0) and gamma of this chunk (the staging group overwrites the slots with
        // the next chunk's after the next barrier)
        const float dot_c = xslot[tid & 127], gam_c = gslot[tid & 127];
        // ---- P6 = G V'^T --------------------------------------------------------------------------
        if (tid == 0) {
            if (wait1(cx, B_GV, par) && !*cx.abort_flag) {
                // G K-major (two 64-channel atoms of 128 rows); V' MN-major (its tile holds a
                // channel per 128-byte row of 64 tokens, so K = channels steps 16 rows)
                const uint32_t id_v = idesc_bf16_f32_mn(128, 64, false, true);
                const uint64_t gh = sdesc_k_sw128(sbase + SM_GH), gl = sdesc_k_sw128(sbase + SM_GL);
#pragma unroll
                for (int k = 0; k < 128; k += 16) {
                    const uint32_t ao = ((uint32_t)(k >> 6) * 128u * 128u + (uint32_t)(k & 63) * 2u) >> 4;
                    const uint64_t vh = sdesc_mn_sw128(sbase + SM_VP + (uint32_t)k * 128u, 8192u);
                    const uint64_t vl = sdesc_mn_sw128(sbase + SM_VP + 16384u + (uint32_t)k * 128u, 8192u);
                    mma_ss(tbase + TM_P6, gh + ao, vh, id_v, k > 0 ? 1u : 0u);
                    mma_ss(tbase + TM_P6, gl + ao, vh, id_v, 1u);
                    mma_ss(tbase + TM_P6, gh + ao, vl, id_v, 1u);
                }
                mma_commit(cx.bars + B_P6);
                wait1(cx, B_P6, par);
            }
            GDN_BTRACE(it, 1);
        }
        __syncthreads();
        tc_fence_after();
        // ---- [dP; dA]: row r' of P6, masked (dP: s <= r', dA: s < r' - 64), split ------------------
        if (!*cx.abort_flag) {
            const int rp = tid & 127, hc = tid >> 7;
            const int lim = rp < 64 ? rp : rp - 65;  // keep s <= lim
            uint8_t* dpa = sm + SM_DPA;
            uint32_t r[32];
            tmem_ld32(tl + TM_P6 + 32 * hc, r);
            tmem_ld_wait();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t wh[4], wl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i0 = 8 * ch + 2 * e, s0 = 32 * hc + i0;
                    const float x0 = s0 <= lim ? __uint_as_float(r[i0]) : 0.f;
                    const float x1 = s0 + 1 <= lim ? __uint_as_float(r[i0 + 1]) : 0.f;
                    split_pack(x0, x1, wh[e], wl[e]);
                }
                const uint32_t off = sw128_offset(rp, 32 * hc + 8 * ch, 128);
                st16(dpa + off, make_uint4(wh[0], wh[1], wh[2], wh[3]));
                st16(dpa + 16384 + off, make_uint4(wl[0], wl[1], wl[2], wl[3]));
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- P7 = S0 G^T + Ktil^T [dP;dA]^T,  P8 = [Qhat^T|Ehat^T] [dP;dA],  P9 = dS V'^T ----------
        if (tid == 0) GDN_BTRACE(it, 2);
        if (tid == 0 && !*cx.abort_flag) {
            const uint32_t id128 = idesc_bf16_f32(128, 128);
            mma_ts_u<128, 128>(tbase + TM_P7, tbase + TM_S0H, sbase + SM_GH, id128, false);
            mma_ts_u<128, 128>(tbase + TM_P7, tbase + TM_S0L, sbase + SM_GH, id128, true);
            mma_ts_u<128, 128>(tbase + TM_P7, tbase + TM_S0H, sbase + SM_GL, id128, true);
            const uint32_t id_kt = idesc_bf16_f32_mn(128, 128, true, false);
#pragma unroll
            for (int k = 0; k < 64; k += 16) {
                const uint64_t akh = sdesc_mn_sw128(sbase + SM_RK + (uint32_t)k * 128u, 8192u);
                const uint64_t akl = sdesc_mn_sw128(sbase + SM_RA + (uint32_t)k * 128u, 8192u);
                const uint64_t bdh = sdesc_k_sw128(sbase + SM_DPA + (uint32_t)k * 2u);
                const uint64_t bdl = sdesc_k_sw128(sbase + SM_DPA + 16384u + (uint32_t)k * 2u);
                mma_ss(tbase + TM_P7, akh, bdh, id_kt, 1u);
                mma_ss(tbase + TM_P7, akl, bdh, id_kt, 1u);
                mma_ss(tbase + TM_P7, akh, bdl, id_kt, 1u);
            }
            const uint32_t id_k8 = idesc_bf16_f32_mn(128, 64, true, true);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t s0 = 16u * (uint32_t)kk;
                const uint32_t arow = s0 < 64u ? 64u + s0 : s0 - 64u;  // Qhat rows, then Ehat rows
                const uint64_t ah = sdesc_mn_sw128(sbase + SM_EQ + arow * 128u, 16384u);
                const uint64_t al = sdesc_mn_sw128(sbase + SM_RQB + arow * 128u, 16384u);
                const uint64_t bh_ = sdesc_mn_sw128(sbase + SM_DPA + s0 * 128u, 8192u);
                const uint64_t bl_ = sdesc_mn_sw128(sbase + SM_DPA + 16384u + s0 * 128u, 8192u);
                mma_ss(tbase + TM_P6, ah, bh_, id_k8, kk > 0 ? 1u : 0u);
                mma_ss(tbase + TM_P6, al, bh_, id_k8, 1u);
                mma_ss(tbase + TM_P6, ah, bl_, id_k8, 1u);
            }
            {
                const uint32_t id_v = idesc_bf16_f32_mn(128, 64, false, true);
#pragma unroll
                for (int k = 0; k < 128; k += 16) {
                    const uint64_t vh = sdesc_mn_sw128(sbase + SM_VP + (uint32_t)k * 128u, 8192u);
                    const uint64_t vl = sdesc_mn_sw128(sbase + SM_VP + 16384u + (uint32_t)k * 128u, 8192u);
                    mma_ts(tbase + TM_P9, tbase + TM_DSH + (uint32_t)(k >> 1), vh, id_v, k > 0 ? 1u : 0u);
                    mma_ts(tbase + TM_P9, tbase + TM_DSL + (uint32_t)(k >> 1), vh, id_v, 1u);
                    mma_ts(tbase + TM_P9, tbase + TM_DSH + (uint32_t)(k >> 1), vl, id_v, 1u);
                }
            }
            mma_commit(cx.bars + B_P789);
            if (wait1(cx, B_P789, par) && !*cx.abort_flag) {
                // the [dP; dA] and V' tiles are free: the walk's rows of this chunk
                load_walk<APC, GPC, SPLIT>(cx, cp, m);
                ++wk_issued;
            }
            GDN_BTRACE(it, 3);
        }
        __syncthreads();
        tc_fence_after();
        // ---- chunk ci: dv, dw, then the epilogue;  chunk ci + gridDim.x: staging -------------------
        if (warp < 4) {
            const float xs = grad_xs(cx, tl, tid);
            named_bar(1, 128);  // Ktil read: the next chunk's raw tiles may land
            if (tid == 0 && nx < nch && !*cx.abort_flag) {
                load_raw_g<APC, GPC, SPLIT>(cx, chunk_pos(pb, nx), m);
                ++raw_issued;
            }
            if (tid == 0) {
                GDN_BTRACE(it, 9);
                wait1(cx, B_WK, par);
            }
            named_bar(1, 128);
            if (!*cx.abort_flag)
                grad_epilogue<APC, GPC, TG, SPLIT, LG, GT, QT>(p, cx, cp, tl, tid, warp, gam_c, gam_c * (xs + dot_c), scr,
                                                               it);
            if (tid == 0) GDN_BTRACE(it, 5);
            // dv, dw of this chunk (the staging group's loads of the next chunk's states are the longer
            // part of its work, so this group takes them after its walk)
            grad_dv_dw<GPC, TG, SPLIT, LG, GT>(p, cx, cp, tid, scr);
            if (tid == 0) GDN_BTRACE(it, 4);
            // the walk and dv/dw have read their tiles; the scalar gates' partials are written
            bar_arrive_all(3);
        } else {
            if (nx < nch)
                stage_chunk<APC, GPC, TG, SPLIT, LG>(p, cx, chunk_pos(pb, nx), tl, tid - 128, xslot, gslot, par ^ 1u, it);
            if (tid == 128) GDN_BTRACE(it, 8);
            // The next chunk's G and V' tiles may land once dv/dw (the G tiles' last reader) and the
            // walk (its alpha, b or lo rows are in the V' tile) are done, and with scalar gates once
            // their scratch (in rows of the G lo tile that dO lo overwrites) has been read.
            bar_sync_all(3);
            if ((!APC || !GPC) && !*cx.abort_flag) scalar_gate_finish<APC, GPC, TG, LG, GT>(p, cp, tid - 128, scr);
            if (tid == 128 && nx < nch && !*cx.abort_flag) {
                load_gv(cx, chunk_pos(pb, nx), m, dol);
                ++gv_issued;
            }
        }
        if (tid == 0) *stop_slot = *cx.abort_flag;
        __syncthreads();
        if (*stop_slot) break;
    }
    // ---- teardown: TMA loads still in flight after an abort are waited for (bounded) -----------
    tc_fence_before();
    __syncthreads();
    if (*cx.abort_flag && (tid == 0 || tid == 128)) {
        const uint64_t tw = globaltimer_ns();
        if (raw_issued > 0)
            while (!mbar_try_wait(cx.bars + B_RAW, (uint32_t)((raw_issued - 1) & 1)) && globaltimer_ns() - tw < cx.wait_ns) {
            }
        if (gv_issued > 0)
            while (!mbar_try_wait(cx.bars + B_GV, (uint32_t)((gv_issued - 1) & 1)) && globaltimer_ns() - tw < cx.wait_ns) {
            }
        if (wk_issued > 0)
            while (!mbar_try_wait(cx.bars + B_WK, (uint32_t)((wk_issued - 1) & 1)) && globaltimer_ns() - tw < cx.wait_ns) {
            }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}
}  // namespace grad
}  // namespace tcbwd
}  // namespace gdn
