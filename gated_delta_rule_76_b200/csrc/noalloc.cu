// gdn_chunk_fwd_noalloc: the chunkwise forward with its scratch memory taken from a fixed device
// array inside this library instead of a caller workspace.  Nothing here allocates memory.
#include <cstdio>

#include "gdn.h"
#include "launch.h"

namespace gdn {
// Defined with the rest of the C ABI (argument validation and the thread-local error message).
gdn_status check_fwd_args(const gdn_fwd_args* a);
gdn_status record_error(gdn_status code, const char* msg);
}  // namespace gdn

namespace {

// Scratch of the forward (status word at offset 0, then the per-chunk factors of the CUDA-core
// path; the tensor-core path uses the status word only).  Zero-initialised at module load.
constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch in the current context, looked up on every call with
// cudaGetSymbolAddress (with the device current, as that call requires).  It is not cached: after a
// cudaDeviceReset the module is loaded again and the array may sit at another address.  Once the
// module is loaded the lookup is a host-side table read.
gdn_status scratch_of_current_device(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof(msg), "gdn_chunk_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed (%s)",
                 cudaGetErrorName(e));
        return gdn::record_error(GDN_ERR_CUDA, msg);
    }
    *out = p;
    return GDN_OK;
}

}  // namespace

extern "C" GDN_API gdn_status gdn_chunk_fwd_noalloc(const gdn_fwd_args* a, gdn_stream stream) {
    gdn_status s = gdn::check_fwd_args(a);
    if (s) return s;
    const size_t need = gdn_chunk_fwd_workspace_size(a);
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "gdn_chunk_fwd_noalloc: this problem needs %zu bytes of scratch, more than the %zu built "
                 "into the library; call gdn_chunk_fwd with a workspace instead",
                 need, kScratchBytes);
        return gdn::record_error(GDN_ERR_WORKSPACE, msg);
    }
    void* ws = nullptr;
    if ((s = scratch_of_current_device(&ws))) return s;
    return gdn_chunk_fwd(a, ws, kScratchBytes, stream);
}

extern "C" GDN_API gdn_status gdn_chunk_fwd_noalloc_status(gdn_stream stream) {
    void* ws = nullptr;
    gdn_status s = scratch_of_current_device(&ws);
    if (s) return s;
    return gdn_workspace_status(ws, stream);
}
