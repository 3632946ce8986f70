// Launchers for the GDN instantiations of the DeltaLog kernels.
#include "dl_launch.cuh"

namespace dl {
DL_DEFINE_VARIANT_LAUNCHERS(kVarGDN)
}  // namespace dl
