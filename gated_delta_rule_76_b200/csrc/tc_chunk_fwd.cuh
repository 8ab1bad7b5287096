// Fused chunkwise forward on the 5th-generation tensor cores (sm_100a): one CTA per
// (batch, value head), chunks of C = 64 tokens, dk = dv = 128, bf16 inputs, fp32 state.
//
// Per chunk (Gated DeltaNet-2 summary, «Entraînement Parallèle Efficace par Blocs»; the decay is
// absorbed into the erase and write factors, a lower-triangular system is solved):
//   Gamma_r = prod_{i<=r} alpha_i,  gamma = Gamma_63;  Ehat = (b.*k).*Gamma,  Qhat = q.*Gamma,
//   Ktil = k./Gamma,  Kbar = k.*gamma./Gamma;   A = strict_lower(Ehat Ktil^T),
//   P = lower(Qhat Ktil^T),  T = (I + A)^-1,   V' = T (Z - Ehat S0),  Z = w.*v,
//   O = scale (Qhat S0 + P V'),  S_end = Diag(gamma) S0 + Kbar^T V' = Diag(gamma) (S0 + Ktil^T V').
// Every product is issued with M = 128 by putting dv on the M side (D[j][..] = sum A[j][k] B[..][k]):
//   X1 = [Ehat;Qhat] Ktil^T               (M = 128 rows of Ehat/Qhat, N = 64, K = 128)
//   X2 = S0^T [Ehat;Qhat]^T               (M = dv, N = 2 x 64, K = dk; A = S0^T in tensor memory)
//   X3 = Y^T T^T   with Y^T = Z^T - (Ehat S0)^T  (M = dv, N = 64, K = 64; A in tensor memory)
//   X4 = V'^T P^T  accumulated onto (Qhat S0)^T  (M = dv, N = 64, K = 64)
//   X5 = V'^T Ktil (B = Ktil MN-major, the tile X1 read)  (M = dv, N = dk, K = 64); gamma is
//        applied in the state update
//
// Precision.  A bf16 operand carries a relative rounding of up to 2^-9, and with seven rounded
// operand families the output error reaches ~4% of its RMS at the largest entry.  Every derived
// operand x is therefore carried as a pair hi = bf16(x), lo = bf16(x - hi) and the products take
// the cross terms that matter (hi*hi + lo*hi + hi*lo), each in fp32 in tensor memory:
//   X1: Ehat, Qhat and Ktil split (3 MMAs);  X2: S0 split, and Qhat split in Qhat S0 (2 + 3 MMAs);
//   X3: Y and T split (3);  X4: V' and P split (3);  X5: V' and Ktil split (3).
// T lo shares the fp32 scratch of the solve: the next chunk's A is written there only after X3 of
// this chunk has completed.
//
// Thread j of the two scan warpgroups owns TMEM lane j (= value column j) and keeps its column of
// the fp32 state in registers, split between the warpgroups by halves of dk.
// Roles (384 threads):
//   warps 0-7  (scan)     : the sequential chain X2 -> Y -> X3 -> V' -> X4, X5 -> output, state;
//                           while the prologue solves for T they build P (from X1).  Thread 0
//                           issues the scan's MMAs and all TMA loads (the z tile of a gated output
//                           at the top of each chunk).
//   warps 8-11 (prologue) : for the next chunk, the cumulative decay and the split operands, X1,
//                           and the triangular solve T = (I + A)^-1; thread 256 issues X1.
// The Ktil tiles (where the raw k and alpha tiles land) are double-buffered by chunk parity, so X5
// of a chunk can read them while the next chunk's are formed; the other operand tiles are single-
// buffered.  [Ehat;Qhat] and T each have a "ready" barrier (prologue -> scan) and a "free" barrier
// (the scan's MMA that read it has completed -> prologue); the raw TMA stage is reloaded as soon as
// X1 and X2 (the last readers of [Ehat;Qhat] lo) are done.  Saving mode
// (the backward cache) stores the entering state and V' while the MMAs run.  Split inputs (fp32
// q, k, v as bf16 hi/lo pairs, scalar gates only) take the lo tiles in the gate slots.  Every
// mbarrier wait is bounded: on expiry the kernel sets an error word, stops issuing work and frees
// its tensor memory.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "seq.cuh"
#include "umma.cuh"

namespace gdn {
namespace tcfwd {

using namespace gdn::tc;

// Optional phase timestamps of CTA 0 (compiled only with -DGDN_FWD_TRACE, for profiling builds):
// g_fwd_trace[chunk][point] = %globaltimer.
#ifdef GDN_FWD_TRACE
__device__ unsigned long long g_fwd_trace[64][32];
#define GDN_TRACE(chunk, point)                                                   \
    do {                                                                          \
        if (blockIdx.x == 0 && (chunk) < 64) g_fwd_trace[(chunk)][(point)] = globaltimer_ns(); \
    } while (0)
#else
#define GDN_TRACE(chunk, point) \
    do {                        \
    } while (0)
#endif

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 384;
constexpr uint64_t kWaitNs = 4000000000ull;

// tensor memory columns
constexpr uint32_t TM_X1 = 0;     // 64:  A (lanes 0-63), P (lanes 64-127), fp32
constexpr uint32_t TM_X2 = 64;    // 128: (Ehat S0)^T | (Qhat S0 + P V')^T
constexpr uint32_t TM_X5 = 192;   // 128: first V'^T = (Y^T T^T) in cols 0-63, then V'^T Ktil
constexpr uint32_t TM_S0H = 320;  // 64:  S0^T hi, bf16 pairs
constexpr uint32_t TM_S0L = 384;  // 64:  S0^T lo
constexpr uint32_t TM_YH = 448;   // 32:  Y^T (then V'^T) hi
constexpr uint32_t TM_YL = 480;   // 32:  Y^T (then V'^T) lo
constexpr uint32_t TM_COLS = 512;

// shared memory offsets from the 1024-byte-aligned base (K-major 128-byte-swizzled bf16 tiles)
constexpr uint32_t SM_RQB = 0;        // 32 KB [2 atoms][128 rows]: TMA b (rows 0-63), q (64-127) -> [Ehat;Qhat] lo
constexpr uint32_t SM_RK = 32768;     // 16 KB [2][64]: TMA k -> Ktil hi (even chunks)
constexpr uint32_t SM_RA = 49152;     // 16 KB [2][64]: TMA alpha -> Ktil lo (even chunks)
constexpr uint32_t SM_EQ = 65536;     // 32 KB [2][128]: [Ehat;Qhat] hi
constexpr uint32_t SM_Z = 98304;      // 16 KB [2][64]: TMA z tile of the scan's chunk (gated output)
constexpr uint32_t SM_T = 114688;     // 8 KB [1][64]: T
constexpr uint32_t SM_P = 122880;     // 16 KB: P hi [1][64], P lo [1][64]
constexpr uint32_t SM_KB = 139264;    // 32 KB: TMA k -> Ktil hi [2][64], TMA alpha -> Ktil lo [2][64]
                                      // (odd chunks: the Ktil tiles are double-buffered, X5 of one
                                      // chunk reads them while the next chunk's are formed)
constexpr uint32_t SM_VW = 172032;    // 32 KB: v [2][64], w [2][64]
constexpr uint32_t SM_ASCR = 204800;  // 17 KB: A, then T, fp32 [64][LDA] row-major; then T lo
constexpr uint32_t SM_TLO = SM_ASCR;   // 8 KB [1][64]: T lo (bf16), from the solve until X3 has read it
constexpr uint32_t SM_GAM = 222208;   // gamma, 3 slots x 128 floats (chunk n uses slot n % 3)
constexpr uint32_t SM_BAR = 223744;   // mbarriers, tensor memory base, abort flag
constexpr uint32_t SM_RS = SM_BAR + 256;  // 4 KB: alpha products per row group [8][128], then the
                                          // solve's products: [2][16][16], then [32][32]
constexpr uint32_t SM_SG = SM_RS + 4096;  // scalar gates of a chunk: [2 slots][alpha, beta][64] fp32
constexpr uint32_t SM_NRM = SM_SG + 1024;  // output norm: [2 halves][4 warps][32 tokens] partial sums
constexpr uint32_t SM_END = SM_NRM + 1024;
constexpr int LDA = 68;  // fp32 row stride of the A/T scratch: float4 rows, rows 16 B apart in bank
constexpr size_t kSmemBytes = SM_END + 1024;
// Ktil hi / lo tiles of chunk n
__device__ __forceinline__ uint32_t kt_hi(int n) { return (n & 1) ? SM_KB : SM_RK; }
__device__ __forceinline__ uint32_t kt_lo(int n) { return (n & 1) ? SM_KB + 16384u : SM_RA; }

enum Bar {
    B_RAW = 0,      // q, k, alpha, b tiles of the prologue's chunk landed
    B_VW,           // v, w tiles of the scan's chunk landed
    B_X1,           // X1 complete
    B_EQ_READY,     // [Ehat;Qhat] hi and Qhat lo written
    B_EQ_FREE,      // X2 complete
    B_T_READY,
    B_T_FREE,       // X3 complete
    B_X2A,
    B_X3,
    B_X45,
    B_Z,            // z tile of the scan's chunk landed (gated output)
    B_COUNT
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
    uint64_t wait_ns;  // limit of every bounded wait; 0 = kWaitNs
    // Backward support (all NULL in a plain forward).  o may be NULL then: no output is formed.
    float* s0_out;               // [B*Hv][NT + 1][dv/8][dk][8] fp32: the state entering every chunk, then
                                 //   the final state
    __nv_bfloat16* vp_hi;        // [B*Hv][NT][dv][64]: V' = T (Z - Ehat S0) of every chunk, column-major
    __nv_bfloat16* vp_lo;        //   (a column's 64 tokens contiguous), as hi = bf16(V'), lo = bf16(V' - hi)
    float* o_raw;                // GATE only, may be NULL: the output before the gate, fp32 [B,T,Hv,dv]
    uint8_t* t_out;              // [B*Hv][NT][8 KB] or NULL: the image of every chunk's bf16 T hi tile
                                 //   (64 rows of 128 swizzled bytes), read back by the reverse scan
    int* flags;                  // [B*Hv] or NULL: set for a pair with a chunk outside the decay range
    // GATE only, may be NULL: the output norm before the gate (every (token, head) row of dv values
    // divided by its root mean square, times norm_w[dv]); norm_w is bf16 unless norm_w_f32
    const void* norm_w;
    int norm_w_f32;
    float norm_eps;
};

// Reduce-scatter of 32 values over the lanes of a warp: afterwards lane l holds the sum over the
// warp of entry l.
__device__ __forceinline__ float warp_reduce_scatter32(float (&x)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i < n / 2) {
                const float send = upper ? x[i] : x[i + n / 2];
                const float keep = upper ? x[i + n / 2] : x[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
    }
    return x[0];
}

__device__ __forceinline__ float bf(const uint8_t* tile, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi), for two values at once (bf16x2 pairs).
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16x2(x0, x1);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16x2(x0 - h0, x1 - h1);
}
// 8 bf16 (one 16-byte chunk of a swizzled row) <-> 8 floats.
__device__ __forceinline__ void unpack8(const uint4 v, float (&x)[8]) {
    x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    x[4] = __uint_as_float(v.z << 16); x[5] = __uint_as_float(v.z & 0xFFFF0000u);
    x[6] = __uint_as_float(v.w << 16); x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
    split_pack(x[0], x[1], hi.x, lo.x);
    split_pack(x[2], x[3], hi.y, lo.y);
    split_pack(x[4], x[5], hi.z, lo.z);
    split_pack(x[6], x[7], hi.w, lo.w);
}
__device__ __forceinline__ uint4 ld16(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st16(uint8_t* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }
__device__ __forceinline__ float4 ldf4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void fma4(float (&acc)[4], float a, const float4 t) {
    acc[0] = fmaf(a, t.x, acc[0]);
    acc[1] = fmaf(a, t.y, acc[1]);
    acc[2] = fmaf(a, t.z, acc[2]);
    acc[3] = fmaf(a, t.w, acc[3]);
}

struct Ctx {
    uint8_t* sm;
    uint64_t* bars;
    volatile int* abort_flag;
    int* err;
    uint64_t wait_ns;  // limit of one bounded wait (kWaitNs unless a caller asks for another)
};

// Bounded wait by a single thread (the others sleep in a named barrier meanwhile).  Polls sleep in
// hardware between attempts; gives up when another thread has aborted or after cx.wait_ns.
__device__ __forceinline__ bool wait1(const Ctx& cx, int bar, uint32_t parity) {
    uint64_t* b = cx.bars + bar;
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(b, parity, 1000u)) {
        if (*cx.abort_flag) return false;
        if (globaltimer_ns() - t0 > cx.wait_ns) {
            *cx.abort_flag = 1;
            atomicOr(cx.err, 1);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                     int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Rows 64h .. 64h + 63 of state column j (thread j holds them in S) into one dk x dv block in the
// layout [j / 4][row][j % 4] (float4 (j / 4) * D + row holds columns 4 (j / 4) .. + 3 of a row, so
// a reader holding one row per thread loads it as float4s).  The four lanes of a column quad
// transpose each 4 x 4 block in two butterfly steps, so that every lane stores whole float4s (16
// 16-byte stores instead of 64 4-byte ones).  All 32 lanes of the warp take part.
__device__ __forceinline__ void store_state_block(float* blk, const float (&S)[64], int j, int h) {
    const int e = j & 3;
    const bool b0 = (e & 1) != 0, b1 = (e & 2) != 0;
    float4* dst = reinterpret_cast<float4*>(blk) + (j >> 2) * D + 64 * h + e;
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 4) {
        float v0 = S[c0], v1 = S[c0 + 1], v2 = S[c0 + 2], v3 = S[c0 + 3];
        float s0 = b0 ? v0 : v1, s1 = b0 ? v2 : v3;
        float r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
        if (b0) { v0 = r0; v2 = r1; } else { v1 = r0; v3 = r1; }
        s0 = b1 ? v0 : v2;
        s1 = b1 ? v1 : v3;
        r0 = __shfl_xor_sync(0xffffffffu, s0, 2);
        r1 = __shfl_xor_sync(0xffffffffu, s1, 2);
        if (b1) { v0 = r0; v1 = r1; } else { v2 = r0; v3 = r1; }
        dst[c0] = make_float4(v0, v1, v2, v3);  // row 64h + c0 + e, columns 4 (j / 4) .. + 3
    }
}

// A 3-D tile (the backward cache's chunk-major tiles).
__device__ __forceinline__ void tma3(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// tma4 with an L2 cache policy (from createpolicy): tiles that plain loads read again soon stay
// in L2 with evict_last priority.
__device__ __forceinline__ void tma4_pol(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                         int c3, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(pol)
        : "memory");
}
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Raw tiles of chunk n.  With SPLIT (scalar gates only) q, k, v arrive as bf16 hi + lo pairs of
// fp32 values; the lo halves take the tiles that scalar gates leave free: q lo the b rows of RQB,
// k lo the alpha tile, v lo the w tile (the maps in the tb_, ta and tw slots point at them).
template <bool APC, bool GPC, bool SPLIT>
__device__ __forceinline__ void load_raw(const Ctx& cx, int n, int b, int hk, int hv, const CUtensorMap* tq,
                                         const CUtensorMap* tk, const CUtensorMap* ta, const CUtensorMap* tb_) {
    static_assert(!SPLIT || (!APC && !GPC), "split inputs use the gate tiles");
    const int t0 = n * C;
    const uint32_t base = smem_u32(cx.sm);
    uint64_t* bar = cx.bars + B_RAW;
    mbar_arrive_expect_tx(bar, 32768u + (GPC || SPLIT ? 16384u : 0u) + (APC || SPLIT ? 16384u : 0u));
    tma4(base + SM_RQB + 8192, tq, bar, 0, hk, t0, b);           // q -> rows 64-127, channels 0-63
    tma4(base + SM_RQB + 16384 + 8192, tq, bar, 64, hk, t0, b);  // channels 64-127
    tma4(base + kt_hi(n), tk, bar, 0, hk, t0, b);
    tma4(base + kt_hi(n) + 8192, tk, bar, 64, hk, t0, b);
    if (GPC || SPLIT) {
        const int hb = SPLIT ? hk : hv;
        tma4(base + SM_RQB, tb_, bar, 0, hb, t0, b);              // b (or q lo) -> rows 0-63
        tma4(base + SM_RQB + 16384, tb_, bar, 64, hb, t0, b);
    }
    if (APC || SPLIT) {
        const int ha = SPLIT ? hk : hv;
        tma4(base + kt_lo(n), ta, bar, 0, ha, t0, b);             // alpha (or k lo)
        tma4(base + kt_lo(n) + 8192, ta, bar, 64, ha, t0, b);
    }
}

// L2 prefetch of the tiles load_raw reads for chunk n (no shared memory, no barrier), issued one
// chunk ahead so that the load, which waits for the previous chunk's readers, finds them in L2.
__device__ __forceinline__ void tma_prefetch4(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
template <bool APC, bool GPC, bool SPLIT>
__device__ __forceinline__ void prefetch_raw(int n, int b, int hk, int hv, const CUtensorMap* tq,
                                             const CUtensorMap* tk, const CUtensorMap* ta, const CUtensorMap* tb_) {
    const int t0 = n * C;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 64) {
        tma_prefetch4(tq, c0, hk, t0, b);
        tma_prefetch4(tk, c0, hk, t0, b);
        if (GPC || SPLIT) tma_prefetch4(tb_, c0, SPLIT ? hk : hv, t0, b);
        if (APC || SPLIT) tma_prefetch4(ta, c0, SPLIT ? hk : hv, t0, b);
    }
}

template <bool GPC, bool SPLIT>
__device__ __forceinline__ void load_vw(const Ctx& cx, int n, int b, int hv, const CUtensorMap* tv,
                                        const CUtensorMap* tw) {
    const int t0 = n * C;
    const uint32_t vw = smem_u32(cx.sm) + SM_VW;
    uint64_t* bar = cx.bars + B_VW;
    mbar_arrive_expect_tx(bar, GPC || SPLIT ? 32768u : 16384u);
    tma4(vw, tv, bar, 0, hv, t0, b);
    tma4(vw + 8192, tv, bar, 64, hv, t0, b);
    if (GPC || SPLIT) {
        tma4(vw + 16384, tw, bar, 0, hv, t0, b);                  // w (or v lo)
        tma4(vw + 16384 + 8192, tw, bar, 64, hv, t0, b);
    }
}

template <bool APC, bool GPC, bool GATE, class TG, bool SPLIT, bool LG>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                 const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_z, Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // Offset arithmetic on the shared array keeps the pointer in the shared state space, so the
    // compiler emits shared loads/stores and knows they cannot alias global memory.
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Ctx cx;
    cx.sm = sm;
    cx.bars = reinterpret_cast<uint64_t*>(sm + SM_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SM_BAR + 128);
    cx.abort_flag = reinterpret_cast<volatile int*>(sm + SM_BAR + 132);
    cx.err = p.err;
    cx.wait_ns = p.wait_ns ? p.wait_ns : kWaitNs;
    float* gam = reinterpret_cast<float*>(sm + SM_GAM);

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
    if (tid == 0) {
        load_raw<APC, GPC, SPLIT>(cx, 0, b, hk, hv, &tm_q, &tm_k, &tm_a, &tm_b);
        load_vw<GPC, SPLIT>(cx, 0, b, hv, &tm_v, &tm_w);
    }
    int raw_issued = 1, vw_issued = 1, z_issued = 0;  // meaningful in thread 0 only

    if (warp < 8) {
        // =================================== state scan ===================================
        const int j = tid & 127, h = tid >> 7;
        volatile int* stop_slot = reinterpret_cast<volatile int*>(sm + SM_BAR + 136);
        const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        const long soff = pb.state_off(b, hv);
        const uint32_t id64 = idesc_bf16_f32(128, 64), id128 = idesc_bf16_f32(128, 128);
        // swizzled byte offsets of column j in a 64-row tile: row r -> base + r*128 + xo[r & 7]
        const uint32_t vbase = (uint32_t)(j >> 6) * 64u * 128u;
        uint32_t xo[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) xo[u] = ((uint32_t)(j & 63) * 2u) ^ ((uint32_t)u << 4);
        const long orow = (long)pb.Hv * D;  // element stride between tokens of o / z
        float S[64];  // S[c'] = state[64h + c'][j]
#pragma unroll
        for (int c = 0; c < 64; ++c) S[c] = p.h0 ? p.h0[soff + (long)(64 * h + c) * D + j] : 0.f;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) split_pack(S[32 * q2 + 2 * i], S[32 * q2 + 2 * i + 1], hi[i], lo[i]);
            tmem_st16(tl + TM_S0H + 32 * h + 16 * q2, hi);
            tmem_st16(tl + TM_S0L + 32 * h + 16 * q2, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        named_bar(1, 256);

        for (int n = 0; n < NT; ++n) {
            const uint32_t pn = n & 1;
            const int t0 = n * C, L = min(C, pb.T - t0);
            if (GATE && tid == 0 && !*cx.abort_flag) {
                // z of this chunk for the output epilogue (the previous chunk's reads are done)
                const uint32_t zd = sbase + SM_Z;
                mbar_arrive_expect_tx(cx.bars + B_Z, 16384u);
                tma4(zd, &tm_z, cx.bars + B_Z, 0, hv, t0, b);
                tma4(zd + 8192, &tm_z, cx.bars + B_Z, 64, hv, t0, b);
                ++z_issued;
            }
            // ---- X2 = S0^T [Ehat;Qhat]^T  (S0 split; Qhat split in the Qhat half) ------------------
            if (tid == 0) {
                GDN_TRACE(n, 0);
                tc_fence_after();
                if (wait1(cx, B_EQ_READY, pn) && !*cx.abort_flag) {
                    GDN_TRACE(n, 1);
                    mma_ts_u<128, 128>(tbase + TM_X2, tbase + TM_S0H, sbase + SM_EQ, id128, false);
                    mma_ts_u<128, 128>(tbase + TM_X2, tbase + TM_S0L, sbase + SM_EQ, id128, true);
                    mma_commit(cx.bars + B_X2A);
                    // Qhat lo: rows 64-127 of the [Ehat;Qhat] lo tile
                    mma_ts_u<128, 128>(tbase + TM_X2 + 64, tbase + TM_S0H, sbase + SM_RQB + 8192, id64, true);
                    mma_commit(cx.bars + B_EQ_FREE);
                }
            }
            if (p.s0_out) {
                // state entering chunk n (saving mode): rows 64h .. 64h + 63 of column j, in the
                // layout [j / 8][row][j % 8]: each group of 8 lanes fills one 32-byte sector per
                // store (a reader holding one row per thread loads a row's 8 columns of a block as
                // one 32-byte vector).  Plain 4-byte stores: transposing the state across lanes
                // first (store_state_block, as the reverse scan does) made this chain slower.  The
                // first 32 rows are stored while X2 runs, the other 32 while X4 / X5 run (S changes
                // only in the state update): split so, the stores queue behind the chain's waits
                // instead of in one burst (all 64 in either place was slower).
                float* dst = p.s0_out + ((long)blockIdx.x * (NT + 1) + n) * (D * D) + (j >> 3) * (8 * D) + (64 * h) * 8 + (j & 7);
#pragma unroll
                for (int c = 0; c < 32; ++c) dst[8 * c] = S[c];
            }
            tc_fence_before();
            fence_async_shared();
            named_bar(1, 256);
            if (tid == 0) {
                tc_fence_after();
                // X1 and X2 of this chunk were the last readers of the [Ehat;Qhat] lo tile, and the
                // next chunk's Ktil tiles were last read by X5 of the previous chunk: the next
                // chunk's raw tiles may land.
                wait1(cx, B_X1, pn);
                wait1(cx, B_EQ_FREE, pn);
                GDN_TRACE(n, 8);
                if (raw_issued < NT && !*cx.abort_flag) {
                    load_raw<APC, GPC, SPLIT>(cx, raw_issued, b, hk, hv, &tm_q, &tm_k, &tm_a, &tm_b);
                    ++raw_issued;
                }
                wait1(cx, B_X2A, pn);
                GDN_TRACE(n, 2);
                wait1(cx, B_VW, pn);
                GDN_TRACE(n, 3);
            }
            named_bar(1, 256);
            tc_fence_after();
            // ---- Y^T = Z^T - (Ehat S0)^T  (tensor memory, split) -----------------------------------
            {
                uint32_t r[32];
                tmem_ld32(tl + TM_X2 + 32 * h, r);
                tmem_ld_wait();
                const uint8_t* vt = sm + SM_VW + vbase + 32u * h * 128u;
                const float* sgb = reinterpret_cast<const float*>(sm + SM_SG) + pn * 128 + 64;
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float y2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int ii = 2 * i + e, rr = 32 * h + ii;
                        const uint32_t off = (uint32_t)ii * 128u + xo[ii & 7];
                        const float vv = SPLIT ? bf(vt, off) + bf(vt + 16384, off) : bf(vt, off);
                        float ww;
                        if (GPC) ww = pb.sig_t<LG>(bf(vt + 16384, off));
                        else ww = sgb[rr];
                        y2[e] = vv * ww - __uint_as_float(r[ii]);
                    }
                    split_pack(y2[0], y2[1], hi[i], lo[i]);
                }
                tmem_st16(tl + TM_YH + 16 * h, hi);
                tmem_st16(tl + TM_YL + 16 * h, lo);
                tmem_st_wait();
            }
            // ---- P of this chunk (operand of X4); X1 completed before the Y step --------------------
            if (j >= 64) {
                // P row j - 64 (lanes 64-127 of X1), columns 32 h .. 32 h + 31, lower with diagonal.
                const int rr = j - 64;
                uint8_t* Ph = sm + SM_P;
                uint32_t r[32];
                tmem_ld32(tl + TM_X1 + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t wh[4], wl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i0 = 8 * ch + 2 * e, s0 = 32 * h + i0;
                        const float x0 = s0 <= rr ? __uint_as_float(r[i0]) : 0.f;
                        const float x1 = s0 + 1 <= rr ? __uint_as_float(r[i0 + 1]) : 0.f;
                        split_pack(x0, x1, wh[e], wl[e]);
                    }
                    const uint32_t off = sw128_offset(rr, 32 * h + 8 * ch, 64);
                    st16(Ph + off, make_uint4(wh[0], wh[1], wh[2], wh[3]));
                    st16(Ph + 8192 + off, make_uint4(wl[0], wl[1], wl[2], wl[3]));
                }
            }
            tc_fence_before();
            fence_async_shared();
            named_bar(1, 256);
            // ---- X3 = Y^T T^T = V'^T; v/w of the next chunk --------------------------------------
            if (tid == 0) {
                GDN_TRACE(n, 4);
                tc_fence_after();
                if (vw_issued < NT && !*cx.abort_flag) {
                    load_vw<GPC, SPLIT>(cx, vw_issued, b, hv, &tm_v, &tm_w);
                    ++vw_issued;
                }
                if (wait1(cx, B_T_READY, pn) && !*cx.abort_flag) {
                    GDN_TRACE(n, 5);
                    mma_ts_u<64, 64>(tbase + TM_X5, tbase + TM_YH, sbase + SM_T, id64, false);
                    mma_ts_u<64, 64>(tbase + TM_X5, tbase + TM_YL, sbase + SM_T, id64, true);
                    mma_ts_u<64, 64>(tbase + TM_X5, tbase + TM_YH, sbase + SM_TLO, id64, true);
                    mma_commit(cx.bars + B_X3);
                    mma_commit(cx.bars + B_T_FREE);
                    wait1(cx, B_X3, pn);
                    GDN_TRACE(n, 6);
                }
            }
            named_bar(1, 256);
            tc_fence_after();
            uint32_t vhi[16], vlo[16];  // V' of rows 32h .. 32h + 31, column j (stored after X4/X5 issue)
            {
                uint32_t r[32];
                tmem_ld32(tl + TM_X5 + 32 * h, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    split_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]), vhi[i], vlo[i]);
                tmem_st16(tl + TM_YH + 16 * h, vhi);
                tmem_st16(tl + TM_YL + 16 * h, vlo);
                tmem_st_wait();
            }
            tc_fence_before();
            named_bar(1, 256);
            // ---- X4 (O += V'^T P^T), X5 (dS^T = V'^T Kbar) ---------------------------------------
            if (tid == 0) {
                GDN_TRACE(n, 7);
                tc_fence_after();
                if (!*cx.abort_flag) {
                    const uint32_t P = sbase + SM_P, kh = sbase + kt_hi(n), kl = sbase + kt_lo(n);
                    if (p.o) {
                        mma_ts_u<64, 64>(tbase + TM_X2 + 64, tbase + TM_YH, P, id64, true);
                        mma_ts_u<64, 64>(tbase + TM_X2 + 64, tbase + TM_YL, P, id64, true);
                        mma_ts_u<64, 64>(tbase + TM_X2 + 64, tbase + TM_YH, P + 8192, id64, true);
                    }
                    // X5' = V'^T Ktil: the Ktil tiles are MN-major B operands (token rows, 64
                    // channels per 128-byte row, the two channel halves 8 KB apart); gamma is
                    // applied in the state update, S = Diag(gamma) (S0 + X5'^T)
                    const uint32_t id_x5 = idesc_bf16_f32_mn(128, 128, false, true);
#pragma unroll
                    for (int k = 0; k < C; k += 16) {
                        const uint64_t bh = sdesc_mn_sw128(kh + (uint32_t)k * 128u, 8192u);
                        const uint64_t bl = sdesc_mn_sw128(kl + (uint32_t)k * 128u, 8192u);
                        mma_ts(tbase + TM_X5, tbase + TM_YH + (uint32_t)(k >> 1), bh, id_x5, k > 0 ? 1u : 0u);
                        mma_ts(tbase + TM_X5, tbase + TM_YL + (uint32_t)(k >> 1), bh, id_x5, 1u);
                        mma_ts(tbase + TM_X5, tbase + TM_YH + (uint32_t)(k >> 1), bl, id_x5, 1u);
                    }
                    mma_commit(cx.bars + B_X45);
                }
            }
            if (p.vp_hi) {
                // V' (saving mode), stored while X4 / X5 run.  Column j's rows 32h .. 32h + 31 are 64
                // contiguous bytes of the chunk-major tile (rows past the sequence as zeros), four
                // 16-byte chunks.  A 4 x 4 transpose of those chunks within the lane quad gives lane e
                // chunk e of the quad's four columns, so that each store writes whole 64-byte column
                // pieces (8 per warp instruction instead of 32 scattered 16-byte pieces: the stores
                // of the saving mode are what throttles this chain's global-memory queue).
                uint32_t vh[16], vl[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r0 = 32 * h + 2 * i;
                    const uint32_t keep = (r0 < L ? 0x0000FFFFu : 0u) | (r0 + 1 < L ? 0xFFFF0000u : 0u);
                    vh[i] = vhi[i] & keep;
                    vl[i] = vlo[i] & keep;
                }
                const int e = j & 3;
                const bool b0 = (e & 1) != 0, b1 = (e & 2) != 0;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    // chunks (0,1) and (2,3) swap across lane pairs, then chunk pairs across lane pairs of pairs
#pragma unroll
                    for (int k = 0; k < 4; k += 2) {
                        const uint32_t sh = b0 ? vh[4 * k + w] : vh[4 * (k + 1) + w];
                        const uint32_t sl = b0 ? vl[4 * k + w] : vl[4 * (k + 1) + w];
                        const uint32_t rh = __shfl_xor_sync(0xffffffffu, sh, 1);
                        const uint32_t rl = __shfl_xor_sync(0xffffffffu, sl, 1);
                        if (b0) {
                            vh[4 * k + w] = rh;
                            vl[4 * k + w] = rl;
                        } else {
                            vh[4 * (k + 1) + w] = rh;
                            vl[4 * (k + 1) + w] = rl;
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const uint32_t sh = b1 ? vh[4 * k + w] : vh[4 * (k + 2) + w];
                        const uint32_t sl = b1 ? vl[4 * k + w] : vl[4 * (k + 2) + w];
                        const uint32_t rh = __shfl_xor_sync(0xffffffffu, sh, 2);
                        const uint32_t rl = __shfl_xor_sync(0xffffffffu, sl, 2);
                        if (b1) {
                            vh[4 * k + w] = rh;
                            vl[4 * k + w] = rl;
                        } else {
                            vh[4 * (k + 2) + w] = rh;
                            vl[4 * (k + 2) + w] = rl;
                        }
                    }
                }
                // lane e: chunk e (tokens 32h + 8e .. + 7) of columns 4 (j / 4) + i, i = 0 .. 3
                const long vo = (((long)blockIdx.x * NT + n) * D + (j & ~3)) * 64 + 32 * h + 8 * e;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    *reinterpret_cast<uint4*>(p.vp_hi + vo + 64 * i) =
                        make_uint4(vh[4 * i], vh[4 * i + 1], vh[4 * i + 2], vh[4 * i + 3]);
                    *reinterpret_cast<uint4*>(p.vp_lo + vo + 64 * i) =
                        make_uint4(vl[4 * i], vl[4 * i + 1], vl[4 * i + 2], vl[4 * i + 3]);
                }
            }
            if (p.s0_out) {
                // the other 32 rows of the state entering chunk n (see the X2 phase)
                float* dst = p.s0_out + ((long)blockIdx.x * (NT + 1) + n) * (D * D) + (j >> 3) * (8 * D) + (64 * h) * 8 + (j & 7);
#pragma unroll
                for (int c = 32; c < 64; ++c) dst[8 * c] = S[c];
            }
            if (tid == 0) {
                if (!*cx.abort_flag) {
                    wait1(cx, B_X45, pn);
                    GDN_TRACE(n, 10);
                }
                if (GATE) wait1(cx, B_Z, pn);
            }
            named_bar(1, 256);
            tc_fence_after();
            // ---- output rows 32h .. 32h+31 of column j -----------------------------------------
            if (p.o) {
                uint32_t r[32];
                tmem_ld32(tl + TM_X2 + 64 + 32 * h, r);
                tmem_ld_wait();
                const long obase = pb.v_row(b, t0 + 32 * h, hv) + j;
                const int nrow = min(32, L - 32 * h);
                float ov[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] = pb.scale * __uint_as_float(r[i]);
                if (GATE && p.o_raw) {
                    float* rp = p.o_raw + obase;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < nrow) rp[i * orow] = ov[i];
                }
                if (GATE && p.norm_w) {
                    // token row 32h + i: sum of squares over the 128 columns = the 4 warps of this
                    // half; lane l of each warp reduces token l over its 32 columns
                    float sq[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) sq[i] = ov[i] * ov[i];
                    float* nrm = reinterpret_cast<float*>(sm + SM_NRM);
                    const int lane = tid & 31, w4 = (tid >> 5) & 3;
                    nrm[(h * 4 + w4) * 32 + lane] = warp_reduce_scatter32(sq);
                    named_bar(1, 256);
                    const float tot = nrm[(h * 4) * 32 + lane] + nrm[(h * 4 + 1) * 32 + lane] +
                                      nrm[(h * 4 + 2) * 32 + lane] + nrm[(h * 4 + 3) * 32 + lane];
                    const float rs = rsqrtf(tot * (1.f / D) + p.norm_eps);
                    const float wn = p.norm_w_f32 ? static_cast<const float*>(p.norm_w)[j]
                                                  : __bfloat162float(static_cast<const __nv_bfloat16*>(p.norm_w)[j]);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] *= __shfl_sync(0xffffffffu, rs, i) * wn;
                }
                if (GATE) {
                    // z column j, rows 32h .. 32h + 31, from the TMA tile (zero past the end)
                    const uint8_t* zt = sm + SM_Z + vbase + 32u * h * 128u;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float zz = bf(zt, (uint32_t)i * 128u + xo[i & 7]);
                        ov[i] *= zz * __fdividef(1.f, 1.f + __expf(-zz));
                    }
                }
                if (p.o_type == 1) {
                    float* op = static_cast<float*>(p.o) + obase;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < nrow) op[i * orow] = ov[i];
                } else {
                    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + obase;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i < nrow) op[i * orow] = __float2bfloat16_rn(ov[i]);
                }
            }
            // ---- state: S = Diag(gamma) S0 + Kbar^T V'; split S0^T for the next chunk -------------
            if (tid == 0) GDN_TRACE(n, 13);
            {
                const float4* g4 = reinterpret_cast<const float4*>(gam + (n % 3) * 128 + 64 * h);
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t r[32], hi[16], lo[16];
                    tmem_ld32(tl + TM_X5 + 64 * h + 32 * q2, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const float4 g = g4[8 * q2 + i4];
                        const int i = 4 * i4;
                        S[32 * q2 + i + 0] = g.x * (S[32 * q2 + i + 0] + __uint_as_float(r[i + 0]));
                        S[32 * q2 + i + 1] = g.y * (S[32 * q2 + i + 1] + __uint_as_float(r[i + 1]));
                        S[32 * q2 + i + 2] = g.z * (S[32 * q2 + i + 2] + __uint_as_float(r[i + 2]));
                        S[32 * q2 + i + 3] = g.w * (S[32 * q2 + i + 3] + __uint_as_float(r[i + 3]));
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        split_pack(S[32 * q2 + 2 * i], S[32 * q2 + 2 * i + 1], hi[i], lo[i]);
                    tmem_st16(tl + TM_S0H + 32 * h + 16 * q2, hi);
                    tmem_st16(tl + TM_S0L + 32 * h + 16 * q2, lo);
                }
                tmem_st_wait();
            }
            // One thread samples the abort flag (another group may set it at any time) and the
            // group leaves the loop together.
            if (tid == 0) {
                GDN_TRACE(n, 11);
                *stop_slot = *cx.abort_flag;
            }
            tc_fence_before();
            named_bar(1, 256);
            if (*stop_slot) break;
        }
        if (p.ht && !*cx.abort_flag) {
#pragma unroll
            for (int c = 0; c < 64; ++c) p.ht[soff + (long)(64 * h + c) * D + j] = S[c];
        }
        if (p.s0_out && !*cx.abort_flag) {  // the final state follows the last chunk's entering state
            float* dst = p.s0_out + ((long)blockIdx.x * (NT + 1) + NT) * (D * D) + (j >> 3) * (8 * D) + (64 * h) * 8 + (j & 7);
#pragma unroll
            for (int c = 0; c < 64; ++c) dst[8 * c] = S[c];
        }
    } else {
        // =================================== chunk prologue ===================================
        const int c = tid - 256;  // key channel; also TMEM lane of X1
        volatile int* stop_slot = reinterpret_cast<volatile int*>(sm + SM_BAR + 140);
        const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        const TG* alpha_g = static_cast<const TG*>(p.alpha);
        const TG* beta_g = static_cast<const TG*>(p.b);
        float* ascr = reinterpret_cast<float*>(sm + SM_ASCR);
        float* rs = reinterpret_cast<float*>(sm + SM_RS);
        uint8_t* RQB = sm + SM_RQB;
        uint8_t* EQ = sm + SM_EQ;
        const uint32_t id64 = idesc_bf16_f32(128, 64);
        float ga_next = 1.f, gb_next = 0.f;  // scalar gates of the next chunk (threads c < 64)
        const float* sga = reinterpret_cast<const float*>(sm + SM_SG);
        for (int m = 0; m < NT; ++m) {
            const uint32_t pm = m & 1, pprev = (m - 1) & 1;
            const int t0 = m * C, L = min(C, pb.T - t0);
            uint8_t* RK = sm + kt_hi(m);  // raw k -> Ktil hi of this chunk
            uint8_t* RA = sm + kt_lo(m);  // raw alpha (or k lo) -> Ktil lo
            if (!APC || !GPC) {
                // Scalar gates of chunk m into slot m & 1 (the scan reads beta there); the next
                // chunk's are loaded now and held in registers, so their latency is hidden.
                float* sg = reinterpret_cast<float*>(sm + SM_SG) + pm * 128;
                if (c < 64) {
                    if (m == 0) {
                        if (!APC) ga_next = gate_or<1, LG>(alpha_g, pb, b, t0, c, L, hv, 1.f);
                        if (!GPC) gb_next = gate_or<2, LG>(beta_g, pb, b, t0, c, L, hv, 0.f);
                    }
                    sg[c] = ga_next;
                    sg[64 + c] = gb_next;
                    if (m + 1 < NT) {
                        const int t1 = t0 + C, L1 = min(C, pb.T - t1);
                        if (!APC) ga_next = gate_or<1, LG>(alpha_g, pb, b, t1, c, L1, hv, 1.f);
                        if (!GPC) gb_next = gate_or<2, LG>(beta_g, pb, b, t1, c, L1, hv, 0.f);
                    }
                }
            }
            if (c == 0) {
                GDN_TRACE(m, 16);
                wait1(cx, B_RAW, pm);
                if (m + 1 < NT) prefetch_raw<APC, GPC, SPLIT>(m + 1, b, hk, hv, &tm_q, &tm_k, &tm_a, &tm_b);
                GDN_TRACE(m, 17);
                if (m > 0) wait1(cx, B_EQ_FREE, pprev);
                GDN_TRACE(m, 18);
            }
            named_bar(2, 128);
            // ---- cumulative decay; split operands (hi -> EQ / RK, lo -> RQB / RA) -----------------
            // Thread c: channels 8 cg .. 8 cg + 7 (one 16-byte chunk of a swizzled row) of rows
            // 8 rg .. 8 rg + 7.  Gamma over the chunk is the product of the row groups' products.
            {
                const int cg = c & 15, rg = c >> 4, r0 = 8 * rg;
                const uint32_t a64 = (uint32_t)(cg >> 3) * 64u * 128u + (uint32_t)r0 * 128u;
                const uint32_t a128 = (uint32_t)(cg >> 3) * 128u * 128u + (uint32_t)r0 * 128u;
                const uint32_t ch = (uint32_t)(cg & 7);
                float* part = rs;  // [8][128]
                float Gl[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) Gl[i] = 1.f;
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
                            for (int i = 0; i < 8; ++i) a8[i] = 1.f;
                        }
                    } else {
                        const float av = sga[pm * 128 + r];
#pragma unroll
                        for (int i = 0; i < 8; ++i) a8[i] = av;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) Gl[i] *= a8[i];
                }
                *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg) = make_float4(Gl[0], Gl[1], Gl[2], Gl[3]);
                *reinterpret_cast<float4*>(part + rg * 128 + 8 * cg + 4) = make_float4(Gl[4], Gl[5], Gl[6], Gl[7]);
                named_bar(2, 128);
                float G[8], gm[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) G[i] = gm[i] = 1.f;
#pragma unroll
                for (int g2 = 0; g2 < 8; ++g2) {
                    const float4 p0 = ldf4(part + g2 * 128 + 8 * cg), p1 = ldf4(part + g2 * 128 + 8 * cg + 4);
                    const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (g2 < rg) G[i] *= pv[i];
                        gm[i] *= pv[i];
                    }
                }
                if (rg == 0) {
                    float* gs = gam + (m % 3) * 128 + 8 * cg;
                    *reinterpret_cast<float4*>(gs) = make_float4(gm[0], gm[1], gm[2], gm[3]);
                    *reinterpret_cast<float4*>(gs + 4) = make_float4(gm[4], gm[5], gm[6], gm[7]);
                    if (p.flags) {
                        bool out = false;
#pragma unroll
                        for (int i = 0; i < 8; ++i) out |= seq::decay_out_of_range(gm[i]);
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
                            for (int i = 0; i < 8; ++i) a8[i] = 1.f;
                        }
                    } else {
                        const float av = sga[pm * 128 + r];
#pragma unroll
                        for (int i = 0; i < 8; ++i) a8[i] = av;
                    }
                    unpack8(ld16(RK + o64), k8);
                    unpack8(ld16(RQB + oq), q8);
                    if (SPLIT) {
                        float kl[8], ql[8];
                        unpack8(ld16(RA + o64), kl);
                        unpack8(ld16(RQB + oe), ql);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            k8[i] += kl[i];
                            q8[i] += ql[i];
                        }
                    }
                    if (GPC) {
                        unpack8(ld16(RQB + oe), b8);
                        if constexpr (LG) {  // b from its logit
#pragma unroll
                            for (int e_ = 0; e_ < 8; ++e_) b8[e_] = pb.sig_t<LG>(b8[e_]);
                        }
                    } else {
                        const float bv = sga[pm * 128 + 64 + r];
#pragma unroll
                        for (int i = 0; i < 8; ++i) b8[i] = bv;
                    }
                    float e8[8], qq[8], kt[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        G[i] *= a8[i];
                        e8[i] = b8[i] * k8[i] * G[i];
                        qq[i] = q8[i] * G[i];
                        kt[i] = __fdividef(k8[i], G[i]);
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
            }
            if (c == 0) GDN_TRACE(m, 19);
            fence_async_shared();
            named_bar(2, 128);
            // ---- X1 = [Ehat;Qhat] Ktil^T with the split operands ----------------------------------
            if (c == 0) {
                tc_fence_after();
                if (!*cx.abort_flag) {
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_EQ, sbase + kt_hi(m), id64, false);
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_EQ, sbase + kt_lo(m), id64, true);
                    mma_ss_u<128, 128, 64>(tbase + TM_X1, sbase + SM_RQB, sbase + kt_hi(m), id64, true);
                    mma_commit(cx.bars + B_X1);
                }
                mbar_arrive(cx.bars + B_EQ_READY);
                wait1(cx, B_X1, pm);
                GDN_TRACE(m, 20);
            }
            // The fp32 scratch holds the previous chunk's T lo until X3 has read it.
            if (c == 0 && m > 0) wait1(cx, B_T_FREE, pprev);
            named_bar(2, 128);
            tc_fence_after();
            if (c < 64) {
                // A row c (lanes 0-63 of X1), strictly lower, into the fp32 scratch; warps 8-9.
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[32];
                    tmem_ld32(tl + TM_X1 + 32 * half, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const int s0 = 32 * half + 4 * q4;
                        float4 v4;
                        v4.x = s0 + 0 < c ? __uint_as_float(r[4 * q4 + 0]) : 0.f;
                        v4.y = s0 + 1 < c ? __uint_as_float(r[4 * q4 + 1]) : 0.f;
                        v4.z = s0 + 2 < c ? __uint_as_float(r[4 * q4 + 2]) : 0.f;
                        v4.w = s0 + 3 < c ? __uint_as_float(r[4 * q4 + 3]) : 0.f;
                        *reinterpret_cast<float4*>(ascr + c * LDA + s0) = v4;
                    }
                }
            }
            tc_fence_before();
            named_bar(2, 128);
            if (c == 0) GDN_TRACE(m, 31);
            // ---- T = (I + A)^-1 by 16 x 16 blocks, in place in the fp32 scratch ------------------
            // (1) diagonal blocks D_i = (I + A_ii)^-1: thread c < 64 solves column c & 15 of block
            //     c >> 4 by forward substitution.
            if (c < 64) {
                const int base = 16 * (c >> 4), jc = c & 15;
                float x[16];
#pragma unroll
                for (int s2 = 0; s2 < 16; ++s2) {
                    const float* arow = ascr + (base + s2) * LDA + base;
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int u4 = 0; u4 < (s2 + 3) / 4; ++u4) {
                        const float4 a4 = ldf4(arow + 4 * u4);
                        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int u = 4 * u4 + e;
                            if (u < s2) {
                                if (u & 1) a1 = fmaf(av[e], x[u], a1);
                                else a0 = fmaf(av[e], x[u], a0);
                            }
                        }
                    }
                    x[s2] = s2 == jc ? 1.f : (s2 > jc ? -(a0 + a1) : 0.f);
                }
                named_bar(3, 64);
#pragma unroll
                for (int s2 = 0; s2 < 16; ++s2) ascr[(base + s2) * LDA + base + jc] = x[s2];
            }
            named_bar(2, 128);
            if (c == 0) GDN_TRACE(m, 28);
            // (2) the 32 x 32 diagonal halves: T_10 = -D_1 (A_10 D_0) and T_32 = -D_3 (A_32 D_2).
            //     Thread c: block c >> 6, row i = (c >> 2) & 15 of it, columns 4 (c & 3) .. + 3.
            {
                const int bk = c >> 6, i = (c >> 2) & 15, j0 = 4 * (c & 3);
                const int r0 = 16 + 32 * bk, c0 = 32 * bk;  // the block A_{r0.., c0..}; D above it at c0
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const float* arow = ascr + (r0 + i) * LDA + c0;
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 a4 = ldf4(arow + k);
                    fma4(acc, a4.x, ldf4(ascr + (c0 + k + 0) * LDA + c0 + j0));
                    fma4(acc, a4.y, ldf4(ascr + (c0 + k + 1) * LDA + c0 + j0));
                    fma4(acc, a4.z, ldf4(ascr + (c0 + k + 2) * LDA + c0 + j0));
                    fma4(acc, a4.w, ldf4(ascr + (c0 + k + 3) * LDA + c0 + j0));
                }
                *reinterpret_cast<float4*>(rs + bk * 256 + i * 16 + j0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                named_bar(2, 128);
                float t4[4] = {0.f, 0.f, 0.f, 0.f};
                const float* drow = ascr + (r0 + i) * LDA + r0;  // D_{r0}: lower triangular, zeros above
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 d4 = ldf4(drow + k);
                    fma4(t4, d4.x, ldf4(rs + bk * 256 + (k + 0) * 16 + j0));
                    fma4(t4, d4.y, ldf4(rs + bk * 256 + (k + 1) * 16 + j0));
                    fma4(t4, d4.z, ldf4(rs + bk * 256 + (k + 2) * 16 + j0));
                    fma4(t4, d4.w, ldf4(rs + bk * 256 + (k + 3) * 16 + j0));
                }
                *reinterpret_cast<float4*>(ascr + (r0 + i) * LDA + c0 + j0) = make_float4(-t4[0], -t4[1], -t4[2], -t4[3]);
            }
            named_bar(2, 128);
            if (c == 0) GDN_TRACE(m, 29);
            // (3) the lower-left quarter: X = A_LL T_00, then T_LL = -T_11 X (T_00, T_11 the 32 x 32
            //     diagonal halves, lower triangular with zeros above, so the sums run over all 32).
            //     Thread c: rows 2 (c >> 3), + 1 of the quarter, columns 4 (c & 7) .. + 3.
            {
                const int i = 2 * (c >> 3), j0 = 4 * (c & 7);
                float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
                const float* a0p = ascr + (32 + i) * LDA;
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                    const float4 a0 = ldf4(a0p + k), a1 = ldf4(a0p + LDA + k);
                    const float4 t0 = ldf4(ascr + (k + 0) * LDA + j0), t1 = ldf4(ascr + (k + 1) * LDA + j0);
                    const float4 t2 = ldf4(ascr + (k + 2) * LDA + j0), t3 = ldf4(ascr + (k + 3) * LDA + j0);
                    fma4(x0, a0.x, t0); fma4(x1, a1.x, t0);
                    fma4(x0, a0.y, t1); fma4(x1, a1.y, t1);
                    fma4(x0, a0.z, t2); fma4(x1, a1.z, t2);
                    fma4(x0, a0.w, t3); fma4(x1, a1.w, t3);
                }
                *reinterpret_cast<float4*>(rs + i * 32 + j0) = make_float4(x0[0], x0[1], x0[2], x0[3]);
                *reinterpret_cast<float4*>(rs + (i + 1) * 32 + j0) = make_float4(x1[0], x1[1], x1[2], x1[3]);
                named_bar(2, 128);
                float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
                const float* t0p = ascr + (32 + i) * LDA + 32;
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                    const float4 d0 = ldf4(t0p + k), d1 = ldf4(t0p + LDA + k);
                    const float4 r0 = ldf4(rs + (k + 0) * 32 + j0), r1 = ldf4(rs + (k + 1) * 32 + j0);
                    const float4 r2 = ldf4(rs + (k + 2) * 32 + j0), r3 = ldf4(rs + (k + 3) * 32 + j0);
                    fma4(y0, d0.x, r0); fma4(y1, d1.x, r0);
                    fma4(y0, d0.y, r1); fma4(y1, d1.y, r1);
                    fma4(y0, d0.z, r2); fma4(y1, d1.z, r2);
                    fma4(y0, d0.w, r3); fma4(y1, d1.w, r3);
                }
                *reinterpret_cast<float4*>(ascr + (32 + i) * LDA + j0) = make_float4(-y0[0], -y0[1], -y0[2], -y0[3]);
                *reinterpret_cast<float4*>(ascr + (33 + i) * LDA + j0) = make_float4(-y1[0], -y1[1], -y1[2], -y1[3]);
            }
            named_bar(2, 128);
            if (c == 0) GDN_TRACE(m, 30);
            // (3) T (fp32) -> K-major bf16 tiles T hi (SM_T) and T lo (the first 8 KB of the scratch,
            //     once every thread holds its values): thread c converts half c >> 6 of row c & 63.
            if (c == 0) GDN_TRACE(m, 21);
            if (c == 0 && m > 0) wait1(cx, B_T_FREE, pprev);
            if (c == 0) GDN_TRACE(m, 22);
            named_bar(2, 128);
            {
                const int row = c & 63, col0 = 32 * (c >> 6);
                uint8_t* Tt = sm + SM_T;
                uint8_t* Tl = sm + SM_TLO;
                uint8_t* Tg = p.t_out ? p.t_out + ((long)blockIdx.x * NT + m) * 8192 : nullptr;
                float tv[32];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float4 f = ldf4(ascr + row * LDA + col0 + 4 * q4);
                    tv[4 * q4] = f.x; tv[4 * q4 + 1] = f.y; tv[4 * q4 + 2] = f.z; tv[4 * q4 + 3] = f.w;
                }
                named_bar(2, 128);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    uint4 hi, lo;
                    float x8[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) x8[i] = tv[8 * q8 + i];
                    split8(x8, hi, lo);
                    const uint32_t off = sw128_offset(row, col0 + 8 * q8, 64);
                    st16(Tt + off, hi);
                    st16(Tl + off, lo);
                    if (Tg) *reinterpret_cast<uint4*>(Tg + off) = hi;
                }
            }
            fence_async_shared();
            named_bar(2, 128);
            if (c == 0) {
                mbar_arrive(cx.bars + B_T_READY);
                GDN_TRACE(m, 23);
                *stop_slot = *cx.abort_flag;
            }
            named_bar(2, 128);
            if (*stop_slot) break;
        }
    }

    // ---- teardown: TMA loads still in flight after an abort are waited for (bounded) -----------
    tc_fence_before();
    __syncthreads();
    if (*cx.abort_flag && tid == 0) {
        // thread 0 issued every load; the last one of each stage completes phase (issued - 1)
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(cx.bars + B_VW, (uint32_t)((vw_issued - 1) & 1)) && globaltimer_ns() - t0 < cx.wait_ns) {
        }
        while (!mbar_try_wait(cx.bars + B_RAW, (uint32_t)((raw_issued - 1) & 1)) && globaltimer_ns() - t0 < cx.wait_ns) {
        }
        while (z_issued > 0 && !mbar_try_wait(cx.bars + B_Z, (uint32_t)((z_issued - 1) & 1)) &&
               globaltimer_ns() - t0 < cx.wait_ns) {
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcfwd
}  // namespace gdn
