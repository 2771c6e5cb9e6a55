// msda_instances.cuh -- the list of operator kernel instantiations.
//
// Each (direction, value type) is instantiated in its own translation unit
// (msda_inst_*.cu, with PFX empty) so that the library compiles in parallel;
// msda_api.cu declares the same list with PFX = extern and launches the
// kernels through their host stubs.
#pragma once

#include "msda_kernels.cuh"

// forward_kernel<T, D, FUSED, GEN, SHORT>
#define MSDA_FWD_D(PFX, T, D, SHORT)                                                         \
    PFX template __global__ void forward_kernel<T, D, false, false, SHORT>(const KernelArgs); \
    PFX template __global__ void forward_kernel<T, D, false, true, SHORT>(const KernelArgs);  \
    PFX template __global__ void forward_kernel<T, D, true, false, SHORT>(const KernelArgs);  \
    PFX template __global__ void forward_kernel<T, D, true, true, SHORT>(const KernelArgs);
#define MSDA_FWD_INSTANCES(PFX, T, SHORT)                                                  \
    MSDA_FWD_D(PFX, T, 8, SHORT) MSDA_FWD_D(PFX, T, 16, SHORT) MSDA_FWD_D(PFX, T, 32, SHORT) \
    MSDA_FWD_D(PFX, T, 64, SHORT) MSDA_FWD_D(PFX, T, 128, SHORT) MSDA_FWD_D(PFX, T, 256, SHORT)

// backward_kernel<T, D, FUSED, GEN, MERGE>
#define MSDA_BWD_D(PFX, T, D, MERGE)                                                          \
    PFX template __global__ void backward_kernel<T, D, false, false, MERGE>(const KernelArgs); \
    PFX template __global__ void backward_kernel<T, D, false, true, MERGE>(const KernelArgs);  \
    PFX template __global__ void backward_kernel<T, D, true, false, MERGE>(const KernelArgs);  \
    PFX template __global__ void backward_kernel<T, D, true, true, MERGE>(const KernelArgs);
#define MSDA_BWD_INSTANCES(PFX, T, MERGE)                                                  \
    MSDA_BWD_D(PFX, T, 8, MERGE) MSDA_BWD_D(PFX, T, 16, MERGE) MSDA_BWD_D(PFX, T, 32, MERGE) \
    MSDA_BWD_D(PFX, T, 64, MERGE) MSDA_BWD_D(PFX, T, 128, MERGE) MSDA_BWD_D(PFX, T, 256, MERGE)

#define MSDA_ALL_INSTANCES(PFX)                                                                  \
    MSDA_FWD_INSTANCES(PFX, float, false)                                                        \
    MSDA_FWD_INSTANCES(PFX, __nv_bfloat16, false) MSDA_FWD_INSTANCES(PFX, __nv_bfloat16, true)   \
    MSDA_FWD_INSTANCES(PFX, S8, false)                                                           \
    MSDA_BWD_INSTANCES(PFX, float, true) MSDA_BWD_INSTANCES(PFX, float, false)                   \
    MSDA_BWD_INSTANCES(PFX, __nv_bfloat16, true) MSDA_BWD_INSTANCES(PFX, __nv_bfloat16, false)   \
    MSDA_BWD_INSTANCES(PFX, S8, true) MSDA_BWD_INSTANCES(PFX, S8, false)
