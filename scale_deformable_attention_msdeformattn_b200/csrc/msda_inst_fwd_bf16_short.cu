// msda_inst_fwd_bf16_short.cu -- explicit instantiations of the operator kernels: forward, bf16 value, rows of at most 16 samples.
#include "msda_instances.cuh"

namespace msda {
MSDA_FWD_INSTANCES(, __nv_bfloat16, true)
}  // namespace msda
