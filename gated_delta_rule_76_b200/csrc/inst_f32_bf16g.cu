// Kernel instantiations for float tensors with __nv_bfloat16 gates.
#include <type_traits>
#include "launch.cuh"

namespace gdn {
GDN_DEFINE_LAUNCHERS(f32_bf16g, float, __nv_bfloat16)
}  // namespace gdn
