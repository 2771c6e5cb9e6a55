// msda_inst_bwd_bf16_merge.cu -- explicit instantiations of the operator kernels: backward, bf16 value, merged grad_value reductions.
#include "msda_instances.cuh"

namespace msda {
MSDA_BWD_INSTANCES(, __nv_bfloat16, true)
}  // namespace msda
