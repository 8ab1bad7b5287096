// Test-only library (libgdn_selftest.so): checks the tcgen05 / TMA building blocks of umma.cuh
// on the GPU in isolation, against plain host arithmetic in the tests.
//
//  gdn_selftest_mma: D1 = A * B1^T      (A 128x128 from shared memory, B1 64x128), then
//                    D1 += A2 * B3^T    (A2 128x64, B3 64x64; accumulate into the same TMEM),
//                    D2 = A * B2^T      (A from tensor memory, B2 128x128).
//  gdn_selftest_mma_mn: MN-major operands (a token-major tile read with M or N = channel):
//                    D1 = Ak X, D2 = X^T B2^T, D3 = Ak X with Ak in tensor memory.
//  gdn_selftest_wait_expiry: the tensor-core kernels' failure path (their bounded wait, the error
//                    word and the release of tensor memory) driven by a barrier that nothing
//                    arrives at, with a short limit.
//  gdn_selftest_tma: one 4-D TMA box (64 channels x 1 head x 64 tokens x 1 batch, 128-byte
//                    swizzle) of a [B,T,H,D] bf16 tensor copied to shared memory and read back
//                    through sw128_offset(); tokens past T must read as zero.
// Every wait is bounded; an expired wait sets *err and the kernel frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../umma.cuh"
#include "../tc_chunk_fwd.cuh"

using namespace gdn::tc;

#define SELFTEST_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

__global__ void __launch_bounds__(128) mma_selftest_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B1,
                                                           const __nv_bfloat16* A2, const __nv_bfloat16* B3,
                                                           const __nv_bfloat16* B2, float* D1, float* D2,
                                                           int* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;                  // 128 x 128  (32 KB)
    uint8_t* sB1 = sA + 32768;           // 64 x 128   (16 KB)
    uint8_t* sA2 = sB1 + 16384;          // 128 x 64   (16 KB)
    uint8_t* sB3 = sA2 + 16384;          // 64 x 64    (8 KB)
    uint8_t* sB2 = sB3 + 8192;           // 128 x 128  (32 KB)
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    const int tid = threadIdx.x, warp = tid >> 5;

    auto put = [&](uint8_t* tile, const __nv_bfloat16* src, int rows, int cols) {
        for (int i = tid; i < rows * cols; i += 128) {
            const int r = i / cols, c = i % cols;
            *reinterpret_cast<__nv_bfloat16*>(tile + sw128_offset(r, c, rows)) = src[i];
        }
    };
    put(sA, A, 128, 128);
    put(sB1, B1, 64, 128);
    put(sA2, A2, 128, 64);
    put(sB3, B3, 64, 64);
    put(sB2, B2, 128, 128);
    fence_async_shared();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tbase, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tbase;
    const uint32_t dcol1 = 0, dcol2 = 64, acol = 192;  // D1: 64 cols, D2: 128 cols, A copy: 64 cols

    // A into tensor memory as packed bf16 pairs: lane m = row m, column c holds k = 2c, 2c+1.
    {
        const int m = tid;  // lane = row
        for (int c0 = 0; c0 < 64; c0 += 16) {
            uint32_t r[16];
            for (int i = 0; i < 16; ++i) {
                const int k = 2 * (c0 + i);
                r[i] = pack_bf16x2(__bfloat162float(A[m * 128 + k]), __bfloat162float(A[m * 128 + k + 1]));
            }
            tmem_st16(tmem_addr(tb, warp * 32, acol + c0), r);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t id1 = idesc_bf16_f32(128, 64), id2 = idesc_bf16_f32(128, 128);
        mma_ss_k(tb + dcol1, smem_u32(sA), 128, smem_u32(sB1), 64, 128, id1, false);
        mma_ss_k(tb + dcol1, smem_u32(sA2), 128, smem_u32(sB3), 64, 64, id1, true);
        mma_ts_k(tb + dcol2, tb + acol, smem_u32(sB2), 128, 128, id2, false);
        mma_commit(&bar);
    }
    __syncwarp();
    const bool ok = __syncthreads_and(mbar_wait(&bar, 0, kWaitNs) ? 1 : 0) != 0;
    if (!ok && tid == 0) atomicExch(err, 1);
    tc_fence_after();
    if (ok) {
        const int m = warp * 32 + (tid & 31);
        for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tb, warp * 32, dcol1 + c0), r);
            tmem_ld_wait();
            for (int i = 0; i < 32; ++i) D1[m * 64 + c0 + i] = __uint_as_float(r[i]);
        }
        for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tb, warp * 32, dcol2 + c0), r);
            tmem_ld_wait();
            for (int i = 0; i < 32; ++i) D2[m * 128 + c0 + i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

// MN-major operands.  Ak [128 x 64] (K-major), X [64 x 128] (token-major: row k, 128 MN values),
// B2 [64 x 64] (K-major).  D1 = Ak X (B MN-major from a 64-row tile), D2 = X^T B2^T (A MN-major
// from rows 64-127 of a 128-row tile), D3 = Ak X with Ak taken from tensor memory.
__global__ void __launch_bounds__(128) mma_mn_selftest_kernel(const __nv_bfloat16* Ak, const __nv_bfloat16* X,
                                                              const __nv_bfloat16* B2, float* D1, float* D2,
                                                              float* D3, int* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sAk = smem;             // 128 x 64 K-major  (16 KB)
    uint8_t* sX64 = sAk + 16384;     // X as a 64-row tile (16 KB)
    uint8_t* sX128 = sX64 + 16384;   // X in rows 64-127 of a 128-row tile (32 KB)
    uint8_t* sB2 = sX128 + 32768;    // 64 x 64 K-major   (8 KB)
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    const int tid = threadIdx.x, warp = tid >> 5;
    for (int i = tid; i < 128 * 64; i += 128) {
        const int r = i / 64, c = i % 64;
        *reinterpret_cast<__nv_bfloat16*>(sAk + sw128_offset(r, c, 128)) = Ak[i];
    }
    for (int i = tid; i < 64 * 128; i += 128) {
        const int r = i / 128, c = i % 128;
        *reinterpret_cast<__nv_bfloat16*>(sX64 + sw128_offset(r, c, 64)) = X[i];
        *reinterpret_cast<__nv_bfloat16*>(sX128 + sw128_offset(64 + r, c, 128)) = X[i];
    }
    for (int i = tid; i < 64 * 64; i += 128) {
        const int r = i / 64, c = i % 64;
        *reinterpret_cast<__nv_bfloat16*>(sB2 + sw128_offset(r, c, 64)) = B2[i];
    }
    fence_async_shared();
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tbase;
    const uint32_t c1 = 0, c2 = 128, c3 = 192, ca = 320;  // D1 128, D2 64, D3 128, A copy 32 columns
    {
        const int m = tid;
        for (int c0 = 0; c0 < 32; c0 += 16) {
            uint32_t r[16];
            for (int i = 0; i < 16; ++i) {
                const int k = 2 * (c0 + i);
                r[i] = pack_bf16x2(__bfloat162float(Ak[m * 64 + k]), __bfloat162float(Ak[m * 64 + k + 1]));
            }
            tmem_st16(tmem_addr(tb, warp * 32, ca + c0), r);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t id1 = idesc_bf16_f32_mn(128, 128, false, true);
        const uint32_t id2 = idesc_bf16_f32_mn(128, 64, true, false);
        for (int k = 0; k < 64; k += 16) {
            const uint32_t acc = k > 0 ? 1u : 0u;
            mma_ss(tb + c1, sdesc_k_sw128(smem_u32(sAk) + (uint32_t)k * 2u),
                   sdesc_mn_sw128(smem_u32(sX64) + (uint32_t)k * 128u, 8192u), id1, acc);
            mma_ss(tb + c2, sdesc_mn_sw128(smem_u32(sX128) + 8192u + (uint32_t)k * 128u, 16384u),
                   sdesc_k_sw128(smem_u32(sB2) + (uint32_t)k * 2u), id2, acc);
            mma_ts(tb + c3, tb + ca + (uint32_t)(k >> 1), sdesc_mn_sw128(smem_u32(sX64) + (uint32_t)k * 128u, 8192u),
                   id1, acc);
        }
        mma_commit(&bar);
    }
    __syncwarp();
    const bool ok = __syncthreads_and(mbar_wait(&bar, 0, kWaitNs) ? 1 : 0) != 0;
    if (!ok && tid == 0) atomicExch(err, 1);
    tc_fence_after();
    if (ok) {
        const int m = warp * 32 + (tid & 31);
        for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tb, warp * 32, c1 + c0), r);
            tmem_ld_wait();
            for (int i = 0; i < 32; ++i) D1[m * 128 + c0 + i] = __uint_as_float(r[i]);
            tmem_ld32(tmem_addr(tb, warp * 32, c3 + c0), r);
            tmem_ld_wait();
            for (int i = 0; i < 32; ++i) D3[m * 128 + c0 + i] = __uint_as_float(r[i]);
        }
        for (int c0 = 0; c0 < 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tb, warp * 32, c2 + c0), r);
            tmem_ld_wait();
            for (int i = 0; i < 32; ++i) D2[m * 64 + c0 + i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

__global__ void __launch_bounds__(128) tma_selftest_kernel(const __grid_constant__ CUtensorMap tmap, int c0,
                                                           int hh, int t0, int bb, __nv_bfloat16* out,
                                                           int* err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar, 64 * 64 * 2);
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
            "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem)),
            "l"(reinterpret_cast<uint64_t>(&tmap)), "r"(smem_u32(&bar)), "r"(c0), "r"(hh), "r"(t0), "r"(bb)
            : "memory");
    }
    const bool ok = mbar_wait(&bar, 0, kWaitNs);
    if (!ok) {
        if (tid == 0) atomicExch(err, 2);
        return;
    }
    for (int i = tid; i < 64 * 64; i += 128) {
        const int r = i / 64, c = i % 64;
        out[i] = *reinterpret_cast<const __nv_bfloat16*>(smem + sw128_offset(r, c, 64));
    }
}

typedef CUresult (*EncodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The failure path of the tensor-core kernels on a barrier that completes only if `arrive`:
// thread 0 waits on it with the kernels' own bounded wait (gdn::tcfwd::wait1) and the given limit
// while the other threads hold tensor memory, as a kernel's roles do.  On expiry the wait sets the
// CTA's abort flag and bit 0 of *status (a workspace status word); every thread then sees the
// abort, and the CTA releases its tensor memory and returns.  out[0] = 1 if the wait succeeded,
// out[1] = number of threads that saw the abort flag.
__global__ void __launch_bounds__(128) wait_expiry_selftest_kernel(int* status, int* out, unsigned long long limit_ns,
                                                                   int arrive) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    __shared__ uint32_t tbase;
    __shared__ int seen;
    const int tid = threadIdx.x, warp = tid >> 5;
    gdn::tcfwd::Ctx cx;
    cx.sm = nullptr;
    cx.bars = &bar;
    cx.abort_flag = reinterpret_cast<volatile int*>(&abort_flag);
    cx.err = status;
    cx.wait_ns = limit_ns;
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        seen = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&tbase, 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (arrive && tid == 32) mbar_arrive(&bar);
    if (tid == 0) out[0] = gdn::tcfwd::wait1(cx, 0, 0) ? 1 : 0;
    __syncthreads();
    if (*cx.abort_flag) atomicAdd(&seen, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) out[1] = seen;
    if (warp == 0) tmem_dealloc(tbase, 32);
}

}  // namespace

SELFTEST_API int gdn_selftest_mma(const void* A, const void* B1, const void* A2, const void* B3,
                                  const void* B2, float* D1, float* D2, int* err, void* stream) {
    const size_t smem = 32768 + 16384 + 16384 + 8192 + 32768 + 1024;
    cudaError_t e = cudaFuncSetAttribute(mma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return (int)e;
    mma_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)A, (const __nv_bfloat16*)B1, (const __nv_bfloat16*)A2, (const __nv_bfloat16*)B3,
        (const __nv_bfloat16*)B2, D1, D2, err);
    return (int)cudaGetLastError();
}

SELFTEST_API int gdn_selftest_mma_mn(const void* Ak, const void* X, const void* B2, float* D1, float* D2,
                                     float* D3, int* err, void* stream) {
    const size_t smem = 16384 + 16384 + 32768 + 8192 + 1024;
    cudaError_t e = cudaFuncSetAttribute(mma_mn_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return (int)e;
    mma_mn_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)Ak, (const __nv_bfloat16*)X, (const __nv_bfloat16*)B2, D1, D2, D3, err);
    return (int)cudaGetLastError();
}

// x is [B,T,H,D] bf16 with D = 128; copies the box at (channel c0, head hh, token t0, batch bb).
SELFTEST_API int gdn_selftest_tma(const void* x, int B, int T, int H, int c0, int hh, int t0, int bb,
                                  void* out, int* err, void* stream) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || !fn) return 1000;
    CUtensorMap map;
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 128 * 2, (cuuint64_t)T * H * 128 * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = reinterpret_cast<EncodeTiled>(fn)(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x),
                                                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return 2000 + (int)r;
    const size_t smem = 8192 + 1024;
    tma_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(map, c0, hh, t0, bb, (__nv_bfloat16*)out, err);
    return (int)cudaGetLastError();
}

// status: a workspace status word (device int); out: 2 device ints.
SELFTEST_API int gdn_selftest_wait_expiry(int* status, int* out, unsigned long long limit_ns, int arrive,
                                          void* stream) {
    wait_expiry_selftest_kernel<<<1, 128, 0, (cudaStream_t)stream>>>(status, out, limit_ns, arrive);
    return (int)cudaGetLastError();
}
