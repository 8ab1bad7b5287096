// Kernel instantiations for __nv_bfloat16 tensors with __nv_bfloat16 gates.
#include <type_traits>
#include "launch.cuh"

namespace gdn {
GDN_DEFINE_LAUNCHERS(bf16, __nv_bfloat16, __nv_bfloat16)
}  // namespace gdn
