// Launchers for the KDA instantiations of the DeltaLog kernels.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_VARIANT_LAUNCHERS(kVarKDA)
}  // namespace dl
