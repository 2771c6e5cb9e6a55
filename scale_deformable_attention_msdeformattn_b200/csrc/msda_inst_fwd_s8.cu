// msda_inst_fwd_s8.cu -- explicit instantiations of the operator kernels: forward, INT8 value.
#include "msda_instances.cuh"

namespace msda {
MSDA_FWD_INSTANCES(, S8, false)
}  // namespace msda
