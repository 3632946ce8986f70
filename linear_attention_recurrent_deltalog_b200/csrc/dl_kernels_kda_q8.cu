// Launchers for the KDA instantiations of the DeltaLog kernels with an
// int8 base.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarKDA, int8_t)
}  // namespace dl
