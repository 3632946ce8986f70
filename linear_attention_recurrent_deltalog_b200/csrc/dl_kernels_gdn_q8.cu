// Launchers for the GDN instantiations of the DeltaLog kernels with an
// int8 base.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarGDN, int8_t)
}  // namespace dl
