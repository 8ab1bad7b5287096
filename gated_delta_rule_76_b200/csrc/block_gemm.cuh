// CTA-wide fp32 GEMM on CUDA cores, operands staged through shared memory in K slices.
//
// acc(m, n) += alpha * sum_k A(m, k) * B(k, n), with A(m, k) = A.p[m * A.sm + k * A.sk] and
// B(k, n) = B.p[k * B.sk + n * B.sn]: any operand may be transposed or live in global or shared
// memory.  Thread t owns rows m = t / NTC + i * (NTH / NTC) and columns n = t % NTC + j * NTC.
// Used by the fp32 (FFMA) chunk kernels; the bf16 forward uses tensor cores instead.
#pragma once
#include "common.cuh"

namespace gdn {

struct View {
    const float* p;
    long sm;  // stride of the row index (m for A, k for B)
    long sk;  // stride of the column index (k for A, n for B)
};

template <int M, int N, int NTH, int NTC, int KS = 32>
struct BlockGemm {
    static constexpr int MTR = NTH / NTC;
    static constexpr int TM = M / MTR;
    static constexpr int TN = N / NTC;
    static_assert(NTH % NTC == 0 && M % MTR == 0 && N % NTC == 0, "bad GEMM tiling");
    static constexpr int LA = M + 1;  // odd leading dimensions: conflict-free strided stores
    static constexpr int LB = N + 1;
    // Shared scratch needed by mma(), in floats.
    static constexpr int kScratch = KS * (LA + LB);

    float acc[TM][TN];

    __device__ __forceinline__ int row(int i) const { return threadIdx.x / NTC + i * MTR; }
    __device__ __forceinline__ int col(int j) const { return threadIdx.x % NTC + j * NTC; }

    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
    }

    // Stage A (M x ks) and B (ks x N) slices; both loops walk the operand's contiguous axis.
    __device__ __forceinline__ void stage(const View& A, const View& B, int k0, int ks,
                                          float* As, float* Bs) {
        const int tid = threadIdx.x;
        if (A.sk == 1) {
            for (int idx = tid; idx < M * KS; idx += NTH) {
                const int m = idx / KS, kk = idx % KS;
                As[kk * LA + m] = kk < ks ? A.p[m * A.sm + (long)(k0 + kk)] : 0.f;
            }
        } else {
            for (int idx = tid; idx < M * KS; idx += NTH) {
                const int m = idx % M, kk = idx / M;
                As[kk * LA + m] = kk < ks ? A.p[m * A.sm + (long)(k0 + kk) * A.sk] : 0.f;
            }
        }
        if (B.sk == 1) {
            for (int idx = tid; idx < N * KS; idx += NTH) {
                const int n = idx % N, kk = idx / N;
                Bs[kk * LB + n] = kk < ks ? B.p[(long)(k0 + kk) * B.sm + n] : 0.f;
            }
        } else {
            for (int idx = tid; idx < N * KS; idx += NTH) {
                const int n = idx / KS, kk = idx % KS;
                Bs[kk * LB + n] = kk < ks ? B.p[(long)(k0 + kk) * B.sm + n * B.sk] : 0.f;
            }
        }
    }

    // acc += alpha * A * B over K.  Starts and ends with a CTA barrier, so operands written by
    // any thread before the call are visible and shared operands may be overwritten after it.
    // For B, View::sm is the stride of k and View::sk the stride of n.
    __device__ void mma(const View& A, const View& B, int K, float* scratch, float alpha = 1.f) {
        float* As = scratch;
        float* Bs = scratch + KS * LA;
        const int tm = threadIdx.x / NTC, tn = threadIdx.x % NTC;
        for (int k0 = 0; k0 < K; k0 += KS) {
            const int ks = K - k0 < KS ? K - k0 : KS;
            __syncthreads();
            stage(A, B, k0, ks, As, Bs);
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < ks; ++kk) {
                float a[TM], b[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i) a[i] = As[kk * LA + tm + i * MTR];
#pragma unroll
                for (int j = 0; j < TN; ++j) b[j] = Bs[kk * LB + tn + j * NTC];
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(alpha * a[i], b[j], acc[i][j]);
            }
        }
        __syncthreads();
    }
};

}  // namespace gdn
