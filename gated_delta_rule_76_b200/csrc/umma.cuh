// Blackwell (sm_100a) building blocks written as inline PTX: mbarriers with bounded waits,
// tensor-memory allocation, tcgen05 MMA (bf16 x bf16 -> fp32, operands in shared or tensor
// memory), tcgen05 loads/stores, TMA tiled loads, and the 128-byte-swizzled K-major shared
// memory layout that both TMA and the tensor core use.
//
// Descriptor formats (PTX ISA, tcgen05 "matrix descriptor" and "instruction descriptor" for
// .kind::f16):
//   shared-memory descriptor: start address >> 4 in bits [0,14), leading byte offset >> 4 in
//   [16,30), stride byte offset >> 4 in [32,46), version 1 in [46,48), base offset [49,52),
//   layout type in [61,64) (2 = 128-byte swizzle).
//   instruction descriptor: D format [4,6) (1 = f32), A format [7,10) and B format [10,13)
//   (1 = bf16), A major bit 15 and B major bit 16 (0 = K-major), N >> 3 in [17,23),
//   M >> 4 in [24,29).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- 128-byte swizzle, K-major tiles --------------------------------------------------------
// A tile of R rows x K bf16 columns (K a multiple of 64) is stored as K/64 "atom columns", each
// R rows x 128 bytes; inside every 1024-byte group of 8 rows the 16-byte chunk index is XORed
// with the row index mod 8.  Tile bases are 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows) {
    const uint32_t byte = (uint32_t)(col >> 6) * (uint32_t)rows * 128u + (uint32_t)row * 128u +
                          (uint32_t)(col & 63) * 2u;
    return byte ^ (((byte >> 7) & 7u) << 4);
}

// ---- mbarrier ----------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Untiled bulk copy of `bytes` from global to shared memory (both addresses 16-byte aligned, bytes
// a multiple of 16), completing on the mbarrier's transaction count (the caller has announced the
// bytes with mbar_arrive_expect_tx).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// Wait for the phase with the given parity to complete.  Gives up after `limit_ns` of wall time
// and returns false: callers record an error and leave without touching the barrier again.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// ---- fences ------------------------------------------------------------------------------------
// Generic-proxy shared-memory writes become visible to the async proxy (tensor core, TMA).
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Named barrier among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---- tensor memory -------------------------------------------------------------------------------
// Executed by one whole warp.  The allocated base address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Tensor-memory address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// 32 lanes x 32 consecutive 32-bit columns per warp: thread t gets columns [col, col+32) of
// lane (warp's lane quarter) + t.  Followed by tmem_ld_wait() before the registers are used.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// 32 lanes x 8 consecutive 32-bit columns per warp (same lane mapping as tmem_ld32).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- descriptors ---------------------------------------------------------------------------------
// K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; the leading offset is unused.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset: next 8-row group
    d |= (uint64_t)1u << 46;                 // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                 // 128-byte swizzle
    return d;
}
// bf16 x bf16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Same, with A (bit 15) and/or B (bit 16) MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_mn(int M, int N, bool a_mn, bool b_mn) {
    return idesc_bf16_f32(M, N) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16);
}
// Shared-memory descriptor of an MN-major bf16 operand with the 128-byte swizzle: one 128-byte
// row holds 64 consecutive MN elements of one k, 8 rows (k .. k + 7) form a 1024-byte swizzle
// atom; `lbo_bytes` is the distance between consecutive 64-element MN groups and the next 8
// k-rows start 1024 bytes further.  This is the layout of a token-major tile loaded by TMA in
// boxes of 64 channels (MN = channel, K = token, lbo = box size).  Advance the start address by
// 2048 bytes per K = 16 step.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t smem_addr, uint32_t lbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// D[tmem] (+)= A[smem] * B[smem]^T for one K = 16 slice.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T for one K = 16 slice.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Unrolled K-loops with the shared-memory descriptors computed once: the start-address field
// (bits [0,14), 16-byte units) advances by the K offset; tiles stay below 256 KB, so the field never
// carries into the next one.  A_ROWS / B_ROWS: rows per 128-byte-wide atom column of the tile.
template <int K, int A_ROWS, int B_ROWS>
__device__ __forceinline__ void mma_ss_u(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem, uint32_t idesc,
                                         bool accumulate) {
    const uint64_t da = sdesc_k_sw128(a_smem), db = sdesc_k_sw128(b_smem);
#pragma unroll
    for (int k = 0; k < K; k += 16) {
        const uint32_t ao = ((uint32_t)(k >> 6) * A_ROWS * 128u + (uint32_t)(k & 63) * 2u) >> 4;
        const uint32_t bo = ((uint32_t)(k >> 6) * B_ROWS * 128u + (uint32_t)(k & 63) * 2u) >> 4;
        mma_ss(d_tmem, da + ao, db + bo, idesc, (accumulate || k > 0) ? 1u : 0u);
    }
}
template <int K, int B_ROWS>
__device__ __forceinline__ void mma_ts_u(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, uint32_t idesc,
                                         bool accumulate) {
    const uint64_t db = sdesc_k_sw128(b_smem);
#pragma unroll
    for (int k = 0; k < K; k += 16) {
        const uint32_t bo = ((uint32_t)(k >> 6) * B_ROWS * 128u + (uint32_t)(k & 63) * 2u) >> 4;
        mma_ts(d_tmem, a_tmem + (uint32_t)(k >> 1), db + bo, idesc, (accumulate || k > 0) ? 1u : 0u);
    }
}

// Wait for the phase of the given parity, sleeping in hardware between polls (suspend hint in ns).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Issue a K-loop of MMAs for operands in K-major SW128 tiles.  A: M rows (a_rows rows per atom
// column), B: N rows (b_rows per atom column); K in multiples of 16.
__device__ __forceinline__ void mma_ss_k(uint32_t d_tmem, uint32_t a_smem, int a_rows, uint32_t b_smem,
                                         int b_rows, int K, uint32_t idesc, bool accumulate) {
#pragma unroll 1
    for (int k = 0; k < K; k += 16) {
        const uint32_t a = a_smem + (uint32_t)(k >> 6) * (uint32_t)a_rows * 128u + (uint32_t)(k & 63) * 2u;
        const uint32_t b = b_smem + (uint32_t)(k >> 6) * (uint32_t)b_rows * 128u + (uint32_t)(k & 63) * 2u;
        mma_ss(d_tmem, sdesc_k_sw128(a), sdesc_k_sw128(b), idesc, (accumulate || k > 0) ? 1u : 0u);
    }
}
// Same with A in tensor memory (bf16 pairs packed per 32-bit column: 8 columns per K = 16).
__device__ __forceinline__ void mma_ts_k(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem, int b_rows, int K,
                                         uint32_t idesc, bool accumulate) {
#pragma unroll 1
    for (int k = 0; k < K; k += 16) {
        const uint32_t b = b_smem + (uint32_t)(k >> 6) * (uint32_t)b_rows * 128u + (uint32_t)(k & 63) * 2u;
        mma_ts(d_tmem, a_tmem + (uint32_t)(k >> 1), sdesc_k_sw128(b), idesc, (accumulate || k > 0) ? 1u : 0u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace tc
}  // namespace gdn
