// msda_inst_fwd_e4m3.cu -- explicit instantiations of the operator kernels: forward, FP8 (E4M3) value.
#include "msda_instances.cuh"

namespace msda {
MSDA_FWD_INSTANCES(, E4M3, false)
}  // namespace msda
