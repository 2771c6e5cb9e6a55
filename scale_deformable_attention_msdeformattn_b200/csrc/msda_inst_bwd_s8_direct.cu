// msda_inst_bwd_s8_direct.cu -- explicit instantiations of the operator kernels: backward, INT8 value, direct grad_value reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, S8, false)
}  // namespace msda
