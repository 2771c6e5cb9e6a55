// msda_inst_bwd_e4m3_direct.cu -- explicit instantiations of the operator kernels: backward, FP8 (E4M3) value, direct reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, E4M3, false)
}  // namespace msda
