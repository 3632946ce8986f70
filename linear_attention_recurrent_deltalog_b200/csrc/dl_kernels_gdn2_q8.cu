// Launchers for the GDN-2 instantiations of the DeltaLog kernels with an
// int8 base.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_BASE_LAUNCHERS(kVarGDN2, int8_t)
}  // namespace dl
