// Kernel instantiations for __nv_bfloat16 tensors with float gates.
#include <type_traits>
#include "launch.cuh"

namespace gdn {
GDN_DEFINE_LAUNCHERS(bf16_f32g, __nv_bfloat16, float)
}  // namespace gdn
