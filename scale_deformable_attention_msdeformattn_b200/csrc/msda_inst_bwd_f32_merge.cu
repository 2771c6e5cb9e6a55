// msda_inst_bwd_f32_merge.cu -- explicit instantiations of the operator kernels: backward, float32 value, merged grad_value reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, float, true)
}  // namespace msda
