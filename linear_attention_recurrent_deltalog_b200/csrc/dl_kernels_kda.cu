// Launchers for the KDA instantiations of the DeltaLog kernels (fp32 base,
// and the eager step).
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarKDA, float)
DL_DEFINE_EAGER_LAUNCHER(kVarKDA)
}  // namespace dl
