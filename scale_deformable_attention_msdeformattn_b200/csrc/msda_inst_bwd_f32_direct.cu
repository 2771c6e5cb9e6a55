// msda_inst_bwd_f32_direct.cu -- explicit instantiations of the operator kernels: backward, float32 value, direct grad_value reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, float, false)
}  // namespace msda
