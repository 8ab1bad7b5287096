// Dense copies of token-major inputs given with a token stride (gdn_strides): rows of `row_bytes`
// bytes, `stride_bytes` apart in the source, packed back to back in the destination.  The chunk
// and layer calls run this once per strided tensor before their own kernels, which all read
// dense token-major tensors.  An HBM-bound copy: each thread moves 16-, 8-, 4- or 2-byte units,
// the widest that the source address, the source stride and the row length all allow (the
// destination is a 256-byte-aligned workspace slice, and every row length is a multiple of it).
#include "launch.h"

namespace gdn {

namespace {

template <class U>
__global__ void __launch_bounds__(256) pack_rows_kernel(const char* __restrict__ src, char* __restrict__ dst,
                                                        long rows, long row_units, long stride_units) {
    const U* s = reinterpret_cast<const U*>(src);
    U* d = reinterpret_cast<U*>(dst);
    const long n = rows * row_units;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        const long r = i / row_units, c = i - r * row_units;
        d[i] = __ldg(s + r * stride_units + c);
    }
}

template <class U>
cudaError_t launch_pack(const char* src, char* dst, long rows, long row_bytes, long stride_bytes, cudaStream_t st) {
    const long units = rows * (row_bytes / (long)sizeof(U));
    const long blocks = (units + 255) / 256;
    // enough resident threads to keep HBM busy: 16 CTAs of 256 threads on each of 148 SMs at most
    const unsigned grid = (unsigned)(blocks < 148L * 16 ? (blocks > 0 ? blocks : 1) : 148L * 16);
    pack_rows_kernel<U><<<grid, 256, 0, st>>>(src, dst, rows, row_bytes / (long)sizeof(U),
                                              stride_bytes / (long)sizeof(U));
    count_launch();
    return cudaGetLastError();
}

}  // namespace

cudaError_t pack_rows(const void* src, void* dst, long rows, long row_bytes, long stride_bytes, cudaStream_t st) {
    if (rows <= 0 || row_bytes <= 0) return cudaSuccess;
    const char* s = static_cast<const char*>(src);
    char* d = static_cast<char*>(dst);
    const unsigned long a = reinterpret_cast<uintptr_t>(s) | (unsigned long)row_bytes | (unsigned long)stride_bytes;
    if ((a & 15) == 0) return launch_pack<uint4>(s, d, rows, row_bytes, stride_bytes, st);
    if ((a & 7) == 0) return launch_pack<uint2>(s, d, rows, row_bytes, stride_bytes, st);
    if ((a & 3) == 0) return launch_pack<unsigned>(s, d, rows, row_bytes, stride_bytes, st);
    if ((a & 1) == 0) return launch_pack<unsigned short>(s, d, rows, row_bytes, stride_bytes, st);
    return cudaErrorMisalignedAddress;
}

}  // namespace gdn
