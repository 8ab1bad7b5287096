/*
 * gdn_selftest.h — test-only library libgdn_selftest.so: checks of the sm_100a building blocks
 * (tcgen05 MMA with shared- and tensor-memory operands, TMA tiled loads with the 128-byte
 * swizzle) used by the tensor-core kernels of libgdn.  Not part of the recurrence's API; the
 * tests compare its results with plain host arithmetic.  All pointers are device pointers;
 * calls are asynchronous on `stream`; the return value is 0 or a CUDA error code, and *err
 * (device int, zero on entry) becomes non-zero if a bounded wait inside the kernel expired.
 */
#ifndef GDN_SELFTEST_H
#define GDN_SELFTEST_H
#ifdef __cplusplus
extern "C" {
#endif

/* A [128x128], B1 [64x128], A2 [128x64], B3 [64x64], B2 [128x128] bf16 row-major.
 * D1 [128x64] = A B1^T + A2 B3^T (shared-memory operands, second product accumulated);
 * D2 [128x128] = A B2^T (A taken from tensor memory). */
int gdn_selftest_mma(const void* A, const void* B1, const void* A2, const void* B3, const void* B2,
                     float* D1, float* D2, int* err, void* stream);

/* MN-major operands.  Ak [128x64], X [64x128], B2 [64x64] bf16 row-major.
 * D1 [128x128] = Ak X (B MN-major: X as a 64-row token-major tile), D2 [128x64] = X^T B2^T (A
 * MN-major: X in rows 64-127 of a 128-row tile), D3 [128x128] = Ak X with Ak in tensor memory. */
int gdn_selftest_mma_mn(const void* Ak, const void* X, const void* B2, float* D1, float* D2, float* D3,
                        int* err, void* stream);

/* x: [B,T,H,128] bf16.  out [64x64] bf16 receives x[bb, t0 + r, hh, c0 + c] (zero where
 * t0 + r >= T), loaded by one TMA box with the 128-byte swizzle and read back in shared memory
 * through the swizzled address map. */
int gdn_selftest_tma(const void* x, int B, int T, int H, int c0, int hh, int t0, int bb, void* out,
                     int* err, void* stream);

/* The tensor-core kernels' failure path: thread 0 of one 128-thread CTA holding tensor memory
 * waits on an mbarrier with the kernels' bounded wait and a limit of limit_ns; the barrier
 * completes only if `arrive` is non-zero.  On expiry bit 0 of *status is set (status is meant to
 * be the first word of a libgdn workspace, so that gdn_workspace_status reports it), every
 * thread sees the CTA's abort flag, and the CTA releases its tensor memory and returns.
 * out[0] = 1 if the wait succeeded, else 0; out[1] = number of threads that saw the abort. */
int gdn_selftest_wait_expiry(int* status, int* out, unsigned long long limit_ns, int arrive, void* stream);

#ifdef __cplusplus
}
#endif
#endif
