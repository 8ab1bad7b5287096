// Kernel instantiations for float tensors with float gates.
#include <type_traits>
#include "launch.cuh"

namespace gdn {
GDN_DEFINE_LAUNCHERS(f32, float, float)
}  // namespace gdn
