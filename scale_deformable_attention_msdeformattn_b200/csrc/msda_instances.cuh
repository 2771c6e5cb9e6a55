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

// forward_kernel<T, D, FUSED, GEN, SHORT, SPLIT>: rows split over SPLIT
// lane groups (head dims whose rows leave room in a warp)
#define MSDA_FWD_SPLIT_D(PFX, T, D, SHORT, SPLIT)                                                   \
    PFX template __global__ void forward_kernel<T, D, false, false, SHORT, SPLIT>(const KernelArgs); \
    PFX template __global__ void forward_kernel<T, D, false, true, SHORT, SPLIT>(const KernelArgs);  \
    PFX template __global__ void forward_kernel<T, D, true, false, SHORT, SPLIT>(const KernelArgs);  \
    PFX template __global__ void forward_kernel<T, D, true, true, SHORT, SPLIT>(const KernelArgs);
#define MSDA_FWD_SPLIT_INSTANCES(PFX)                                                             \
    MSDA_FWD_SPLIT_D(PFX, float, 8, false, MSDA_FWD_SPLIT)                                         \
    MSDA_FWD_SPLIT_D(PFX, float, 16, false, MSDA_FWD_SPLIT)                                        \
    MSDA_FWD_SPLIT_D(PFX, float, 32, false, MSDA_FWD_SPLIT)                                        \
    MSDA_FWD_SPLIT_D(PFX, __nv_bfloat16, 8, true, MSDA_FWD_SPLIT)                                  \
    MSDA_FWD_SPLIT_D(PFX, __nv_bfloat16, 16, true, MSDA_FWD_SPLIT)                                 \
    MSDA_FWD_SPLIT_D(PFX, __nv_bfloat16, 32, true, MSDA_FWD_SPLIT)                                 \
    MSDA_FWD_SPLIT_D(PFX, __nv_bfloat16, 64, true, MSDA_FWD_SPLIT)

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
    MSDA_FWD_INSTANCES(PFX, S8, false) MSDA_FWD_SPLIT_INSTANCES(PFX)                             \
    MSDA_BWD_INSTANCES(PFX, float, true) MSDA_BWD_INSTANCES(PFX, float, false)                   \
    MSDA_BWD_INSTANCES(PFX, __nv_bfloat16, true) MSDA_BWD_INSTANCES(PFX, __nv_bfloat16, false)   \
    MSDA_BWD_INSTANCES(PFX, S8, true) MSDA_BWD_INSTANCES(PFX, S8, false)                         \
    MSDA_FWD_INSTANCES(PFX, E4M3, false)                                                         \
    MSDA_BWD_INSTANCES(PFX, E4M3, true) MSDA_BWD_INSTANCES(PFX, E4M3, false)
