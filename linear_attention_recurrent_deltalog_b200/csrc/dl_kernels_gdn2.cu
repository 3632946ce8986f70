// Launchers for the GDN-2 instantiations of the DeltaLog kernels (fp32 base,
// and the eager step).
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarGDN2, float)
DL_DEFINE_EAGER_LAUNCHER(kVarGDN2)
}  // namespace dl
