// msda_inst_fwd_split.cu -- explicit instantiations of the operator kernels: forward with rows split over lane groups (small problems).
#include "msda_instances.cuh"

namespace msda {
MSDA_FWD_SPLIT_INSTANCES()
}  // namespace msda
