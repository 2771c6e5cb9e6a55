// msda_inst_fwd_f32.cu -- explicit instantiations of the operator kernels: forward, float32 value.
#include "msda_instances.cuh"

namespace msda {
MSDA_FWD_INSTANCES(, float, false)
}  // namespace msda
