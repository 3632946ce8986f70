// Launchers for the RWKV6 instantiations of the DeltaLog kernels (fp32 base,
// and the eager step).
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarRWKV6, float)
DL_DEFINE_EAGER_LAUNCHER(kVarRWKV6)
}  // namespace dl
