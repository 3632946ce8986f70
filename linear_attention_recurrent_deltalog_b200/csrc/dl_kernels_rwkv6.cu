// Launchers for the RWKV6 instantiations of the DeltaLog kernels.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_VARIANT_LAUNCHERS(kVarRWKV6)
}  // namespace dl
