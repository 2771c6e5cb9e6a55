// msda_inst_bwd_s8_merge.cu -- explicit instantiations of the operator kernels: backward, INT8 value, merged grad_value reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, S8, true)
}  // namespace msda
