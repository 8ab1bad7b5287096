// Pieces of the sequence-parallel forward and backward (a sequence split along time over
// several GPUs): each segment acts on the state as an affine map S -> M S + N, so the state
// entering a segment is the composition of the maps of the segments before it, and a state
// gradient is carried back across a segment by M^T.  (The state's size does not depend on the
// context length: mkdocs chapter «Gated DeltaNet», «L'état, en mémoire».)
//
//  - identity_states_kernel: S = I for every (sequence, head) (the entering state from which the
//    chunk forward computes M, with the writes zeroed);
//  - compose_kernel: S_out = M S_in + N, or M^T S_in + N, fp32 on CUDA cores, one CTA per
//    (sequence, head) and 64-column slice of S_in: M (dk x dk) and the slice of S_in are staged in
//    shared memory, each thread accumulates a 4 x 8 tile of S_out.
#include "launch.h"

namespace gdn {

namespace {

__global__ void identity_states_kernel(float* S, long pairs, int d) {
    const long n = pairs * d * d;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long e = i % ((long)d * d);
        S[i] = (e / d == e % d) ? 1.f : 0.f;
    }
}

constexpr int kComposeThreads = 256;
constexpr int kComposeCols = 64;  // columns of S_in / S_out per CTA

// grid (pairs, dv / 64), 256 threads; dynamic shared memory: M^T or M as [k][i] (dk x dk) and the
// slice of S_in [k][64].
template <int DK>
__global__ void __launch_bounds__(kComposeThreads) compose_kernel(const float* M, const float* N, const float* S_in,
                                                                  float* S_out, int dv, int transpose) {
    extern __shared__ float sm_c[];
    float* A = sm_c;               // A[k][i] = op(M)[i][k]
    float* Bs = sm_c + DK * DK;    // Bs[k][c] = S_in[k][c0 + c]
    const long pair = blockIdx.x;
    const int c0 = blockIdx.y * kComposeCols, tid = threadIdx.x;
    const float* m = M + pair * DK * DK;
    const float* s = S_in ? S_in + pair * (long)DK * dv : nullptr;
    // op(M)[i][k] = M[i][k] (plain) or M[k][i] (transposed); A is stored k-major so that a thread's
    // rows are consecutive in shared memory.
    for (int idx = tid; idx < DK * DK; idx += kComposeThreads) {
        const int r = idx / DK, c = idx % DK;  // M[r][c], coalesced read
        const float x = m[idx];
        if (transpose) A[r * DK + c] = x;      // op(M)[c][r] = M[r][c]: k = r, i = c
        else A[c * DK + r] = x;                // op(M)[r][c]: k = c, i = r
    }
    for (int idx = tid; idx < DK * kComposeCols; idx += kComposeThreads) {
        const int k = idx / kComposeCols, c = idx % kComposeCols;
        Bs[idx] = s ? s[(long)k * dv + c0 + c] : 0.f;
    }
    __syncthreads();
    // thread: rows 4 * (tid / 8) .. + 3 (DK = 128: 32 row groups; 64: 16 used twice) and
    // columns 8 * (tid % 8) .. + 7
    constexpr int RG = DK / 4;
    for (int rg = tid / 8; rg < RG; rg += kComposeThreads / 8) {
        const int i0 = 4 * rg, j0 = 8 * (tid % 8);
        float acc[4][8] = {};
        if (s) {
#pragma unroll 4
            for (int k = 0; k < DK; ++k) {
                const float4 a = *reinterpret_cast<const float4*>(A + k * DK + i0);
                const float4 b0 = *reinterpret_cast<const float4*>(Bs + k * kComposeCols + j0);
                const float4 b1 = *reinterpret_cast<const float4*>(Bs + k * kComposeCols + j0 + 4);
                const float av[4] = {a.x, a.y, a.z, a.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int ii = 0; ii < 4; ++ii)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) acc[ii][jj] = fmaf(av[ii], bv[jj], acc[ii][jj]);
            }
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
            const long row = pair * (long)DK * dv + (long)(i0 + ii) * dv + c0 + j0;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) S_out[row + jj] = acc[ii][jj] + (N ? N[row + jj] : 0.f);
        }
    }
}

}  // namespace

cudaError_t identity_states(float* S, long pairs, int d, cudaStream_t st) {
    const long n = pairs * d * d;
    const long blocks = (n + 255) / 256;
    identity_states_kernel<<<(unsigned)(blocks < 148L * 16 ? blocks : 148L * 16), 256, 0, st>>>(S, pairs, d);
    count_launch();
    return cudaGetLastError();
}

cudaError_t compose_states(const float* M, const float* N, const float* S_in, float* S_out, long pairs, int dk,
                           int dv, bool transpose, cudaStream_t st) {
    const dim3 grid((unsigned)pairs, (unsigned)(dv / kComposeCols));
    const size_t smem = (size_t)(dk * dk + dk * kComposeCols) * sizeof(float);
    cudaError_t e;
    if (dk == 128) {
        e = cudaFuncSetAttribute(compose_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        compose_kernel<128><<<grid, kComposeThreads, smem, st>>>(M, N, S_in, S_out, dv, transpose ? 1 : 0);
    } else if (dk == 64) {
        e = cudaFuncSetAttribute(compose_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        compose_kernel<64><<<grid, kComposeThreads, smem, st>>>(M, N, S_in, S_out, dv, transpose ? 1 : 0);
    } else {
        return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}

}  // namespace gdn
