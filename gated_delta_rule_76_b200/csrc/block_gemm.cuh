// CTA-wide fp32 GEMM on CUDA cores, operands staged through shared memory in K slices.
//
// acc(m, n) += alpha * sum_k A(m, k) * B(k, n), with A(m, k) = A.p[m * A.sm + k * A.sk] and
// B(k, n) = B.p[k * B.sk + n * B.sn]: any operand may be transposed or live in global or shared
// memory.  Thread t owns a TM x TN register tile of consecutive rows and columns.
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
    static_assert(TM % 4 == 0 && (TN == 2 || TN % 4 == 0), "register tile must be float4 / float2 loadable");
    // Leading dimensions are multiples of 4 floats so that a thread's TM rows / TN columns of one
    // k are read with 16-byte (8-byte) shared loads.
    static constexpr int LA = M + 4;
    static constexpr int LB = N + 4;
    // Shared scratch needed by mma(), in floats (its base must be 16-byte aligned).
    static constexpr int kScratch = KS * (LA + LB);

    float acc[TM][TN];

    // Thread t owns the TM consecutive rows starting at (t / NTC) * TM and the TN consecutive
    // columns starting at (t % NTC) * TN.
    __device__ __forceinline__ int row(int i) const { return (threadIdx.x / NTC) * TM + i; }
    __device__ __forceinline__ int col(int j) const { return (threadIdx.x % NTC) * TN + j; }

    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
    }

    static constexpr int NA = M * KS / NTH;  // staged A elements per thread and K slice
    static constexpr int NB = N * KS / NTH;  // staged B elements per thread and K slice
    static_assert(M * KS % NTH == 0 && N * KS % NTH == 0, "staging must divide evenly");

    // Read one K slice of A (M x KS) and B (KS x N) into registers; both walk the operand's
    // contiguous axis.  Entries past K read as 0.
    __device__ __forceinline__ void fetch(const View& A, const View& B, int k0, int K, float (&ra)[NA],
                                          float (&rb)[NB]) const {
        const int tid = threadIdx.x;
#pragma unroll
        for (int it = 0; it < NA; ++it) {
            const int idx = tid + it * NTH;
            const int m = A.sk == 1 ? idx / KS : idx % M, kk = A.sk == 1 ? idx % KS : idx / M;
            ra[it] = k0 + kk < K ? A.p[m * A.sm + (long)(k0 + kk) * A.sk] : 0.f;
        }
#pragma unroll
        for (int it = 0; it < NB; ++it) {
            const int idx = tid + it * NTH;
            const int n = B.sk == 1 ? idx % N : idx / KS, kk = B.sk == 1 ? idx / N : idx % KS;
            rb[it] = k0 + kk < K ? B.p[(long)(k0 + kk) * B.sm + n * B.sk] : 0.f;
        }
    }
    // Write the fetched slice (A scaled by alpha) to the shared staging tiles As[k][m], Bs[k][n].
    __device__ __forceinline__ void put(const View& A, const View& B, const float (&ra)[NA],
                                        const float (&rb)[NB], float alpha, float* As, float* Bs) const {
        const int tid = threadIdx.x;
#pragma unroll
        for (int it = 0; it < NA; ++it) {
            const int idx = tid + it * NTH;
            const int m = A.sk == 1 ? idx / KS : idx % M, kk = A.sk == 1 ? idx % KS : idx / M;
            As[kk * LA + m] = alpha * ra[it];
        }
#pragma unroll
        for (int it = 0; it < NB; ++it) {
            const int idx = tid + it * NTH;
            const int n = B.sk == 1 ? idx % N : idx / KS, kk = B.sk == 1 ? idx / N : idx % KS;
            Bs[kk * LB + n] = rb[it];
        }
    }

    // acc += alpha * A * B over K.  Starts and ends with a CTA barrier, so operands written by
    // any thread before the call are visible and shared operands may be overwritten after it.
    // For B, View::sm is the stride of k and View::sk the stride of n.  The next K slice is read
    // into registers while the current one is multiplied, so its load latency is hidden.
    __device__ void mma(const View& A, const View& B, int K, float* scratch, float alpha = 1.f) {
        float* As = scratch;
        float* Bs = scratch + KS * LA;
        const float* ap = As + (threadIdx.x / NTC) * TM;
        const float* bp = Bs + (threadIdx.x % NTC) * TN;
        float ra[NA], rb[NB];
        __syncthreads();  // operands written before the call are visible to fetch()
        fetch(A, B, 0, K, ra, rb);
        for (int k0 = 0; k0 < K; k0 += KS) {
            __syncthreads();
            put(A, B, ra, rb, alpha, As, Bs);
            __syncthreads();
            if (k0 + KS < K) fetch(A, B, k0 + KS, K, ra, rb);
#pragma unroll 4
            for (int kk = 0; kk < KS; ++kk) {
                float a[TM], b[TN];
#pragma unroll
                for (int i4 = 0; i4 < TM / 4; ++i4) {
                    const float4 v = *reinterpret_cast<const float4*>(ap + kk * LA + 4 * i4);
                    a[4 * i4 + 0] = v.x;
                    a[4 * i4 + 1] = v.y;
                    a[4 * i4 + 2] = v.z;
                    a[4 * i4 + 3] = v.w;
                }
                if constexpr (TN == 2) {
                    const float2 v = *reinterpret_cast<const float2*>(bp + kk * LB);
                    b[0] = v.x;
                    b[1] = v.y;
                } else {
#pragma unroll
                    for (int j4 = 0; j4 < TN / 4; ++j4) {
                        const float4 v = *reinterpret_cast<const float4*>(bp + kk * LB + 4 * j4);
                        b[4 * j4 + 0] = v.x;
                        b[4 * j4 + 1] = v.y;
                        b[4 * j4 + 2] = v.z;
                        b[4 * j4 + 3] = v.w;
                    }
                }
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
        __syncthreads();
    }
};

}  // namespace gdn
