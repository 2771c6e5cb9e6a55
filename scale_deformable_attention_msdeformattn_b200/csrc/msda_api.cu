// msda_api.cu -- the C ABI declared in include/msda.h: argument checks, kernel
// selection by (value dtype, head_dim), launch shapes, device status word.
//
// Launch shape.  Every compute kernel runs as one persistent wave: the grid is
// (SM count) x (resident CTAs per SM, from the occupancy calculator), walking
// the row tiles grid-stride (tile_walk in msda_kernels.cuh).  CTAs have up to 8 warps; fewer when
// the shared-memory records of the L*K samples of each row would exceed the
// per-CTA budget.
#include "msda.h"
#include "msda_aux.cuh"
#include "msda_gemm.cuh"
#include "msda_instances.cuh"

#include <cudaTypedefs.h>

#include <mutex>

namespace msda {
// the operator kernels are instantiated in the msda_inst_*.cu units
MSDA_ALL_INSTANCES(extern)

// Per-device status word; kernels record failures through KernelArgs::status.
__device__ int g_device_status;
}  // namespace msda

#include <nvtx3/nvToolsExt.h>

namespace {

using msda::KernelArgs;

constexpr int kMaxDevices = 64;
constexpr size_t kCtaSmemBudget = 96 * 1024;   // keeps >= 2 CTAs per SM
// shared-memory bytes per sample slot of a row: two 16-byte records, plus
// grad_A and A in the fused backward
constexpr size_t kForwardRecordBytes = 32;
constexpr size_t kBackwardRecordBytes = 32;
constexpr size_t kFusedBackwardRecordBytes = 40;

bool is_supported_head_dim(int d)
{
    return d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256;
}

bool scaled_dtype(int32_t dtype) { return dtype == MSDA_S8 || dtype == MSDA_E4M3; }

size_t elem_bytes(int32_t dtype) { return dtype == MSDA_BF16 ? 2 : (scaled_dtype(dtype) ? 1 : 4); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// A pointer may be null only when its tensor is empty.
bool ptr_ok(const void *p, int64_t numel)
{
    if (numel == 0)
        return p == nullptr || aligned16(p);
    return p != nullptr && aligned16(p);
}

// value and output are read / written with 32-byte vectors
bool vec_ptr_ok(const void *p, int64_t numel) { return ptr_ok(p, numel) && aligned32(p); }

msda_status check_problem(const msda_problem *p)
{
    if (!p)
        return MSDA_ERR_INVALID_ARG;
    if (p->batch < 0 || p->num_queries < 0 || p->num_keys < 1 || p->num_heads < 1 ||
        p->num_levels < 1 || p->num_points < 1 || p->head_dim < 1)
        return MSDA_ERR_INVALID_ARG;
    if (p->value_dtype != MSDA_F32 && p->value_dtype != MSDA_BF16 && !scaled_dtype(p->value_dtype))
        return MSDA_ERR_INVALID_ARG;
    if (scaled_dtype(p->value_dtype) &&
        (!p->value_scale || (reinterpret_cast<uintptr_t>(p->value_scale) & 3u)))
        return MSDA_ERR_INVALID_ARG;
    if (p->flags & ~(uint32_t)(MSDA_GRAD_VALUE_BF16 | MSDA_ACCUMULATE_GRADS | MSDA_STAGE_INPUTS |
                               MSDA_MERGE_REDUCTIONS | MSDA_TEST_WITHHOLD_COPY))
        return MSDA_ERR_INVALID_ARG;
    if ((p->flags & MSDA_GRAD_VALUE_BF16) && (p->flags & MSDA_ACCUMULATE_GRADS))
        return MSDA_ERR_INVALID_ARG;
    if (p->num_levels > msda::kMaxLevels || p->num_points > 32 ||
        p->num_levels * p->num_points > 128)
        return MSDA_ERR_UNSUPPORTED;
    if (!is_supported_head_dim(p->head_dim))
        return MSDA_ERR_UNSUPPORTED;
    if (p->num_keys >= (int64_t(1) << 27))
        return MSDA_ERR_UNSUPPORTED;
    if ((int64_t)p->num_heads * p->head_dim * (int64_t)elem_bytes(p->value_dtype) >= (int64_t(1) << 31))
        return MSDA_ERR_UNSUPPORTED;
    // corner offsets are int32 (key, head) row indices within one batch entry
    if (p->num_keys * (int64_t)p->num_heads >= (int64_t(1) << 31))
        return MSDA_ERR_UNSUPPORTED;
    // B * Q * M * L * K < 2^40, evaluated without overflow
    const double samples = (double)p->batch * (double)p->num_queries * p->num_heads *
                           p->num_levels * p->num_points;
    if (samples >= 1099511627776.0)
        return MSDA_ERR_UNSUPPORTED;
    const double values = (double)p->batch * (double)p->num_keys * p->num_heads * p->head_dim;
    if (values >= 9.0e18)
        return MSDA_ERR_UNSUPPORTED;
    if ((double)p->batch * (double)p->num_queries >= 2147483648.0)
        return MSDA_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(p->query_order) & 3u)
        return MSDA_ERR_INVALID_ARG;
    return MSDA_OK;
}

struct DeviceInfo {
    int sm_count = 0;
    int *status = nullptr;  // device address of msda::g_device_status
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

// SM count and status-word address of the current device, looked up once per
// device (with that device current) on its first call.
msda_status current_device(int &dev, int &sm_count, int **status = nullptr)
{
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MSDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_devices[dev].sm_count == 0) {
        int n = 0;
        void *st = nullptr;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return MSDA_ERR_CUDA;
        if (cudaGetSymbolAddress(&st, msda::g_device_status) != cudaSuccess || !st)
            return MSDA_ERR_CUDA;
        g_devices[dev].status = static_cast<int *>(st);
        g_devices[dev].sm_count = n;
    }
    sm_count = g_devices[dev].sm_count;
    if (status)
        *status = g_devices[dev].status;
    return MSDA_OK;
}

// Resident CTAs per SM of `kernel` for (threads, smem), cached per device.
// The kernel's dynamic shared-memory limit is raised once, to the device's
// opt-in maximum, so that launches of one kernel with different record sizes
// never see a limit set for a smaller one.
struct OccEntry {
    const void *kernel;
    int dev, threads;
    size_t smem;
    int blocks;
};
struct AttrEntry {
    const void *kernel;
    int dev;
};
constexpr int kOccCache = 512;
OccEntry g_occ[kOccCache];
int g_occ_n = 0;
AttrEntry g_attr[kOccCache];
int g_attr_n = 0;

msda_status raise_smem_limit(const void *kernel, int dev)
{
    for (int i = 0; i < g_attr_n; ++i)
        if (g_attr[i].kernel == kernel && g_attr[i].dev == dev)
            return MSDA_OK;
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
        return MSDA_ERR_CUDA;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes) != cudaSuccess)
        return MSDA_ERR_CUDA;
    if (g_attr_n < kOccCache)
        g_attr[g_attr_n++] = AttrEntry{kernel, dev};
    return MSDA_OK;
}

msda_status occupancy(const void *kernel, int dev, int threads, size_t smem, int &blocks)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int i = 0; i < g_occ_n; ++i) {
        const OccEntry &e = g_occ[i];
        if (e.kernel == kernel && e.dev == dev && e.threads == threads && e.smem == smem) {
            blocks = e.blocks;
            return MSDA_OK;
        }
    }
    msda_status st = raise_smem_limit(kernel, dev);
    if (st != MSDA_OK)
        return st;
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, smem) != cudaSuccess || b < 1)
        return MSDA_ERR_CUDA;
    if (g_occ_n < kOccCache)
        g_occ[g_occ_n++] = OccEntry{kernel, dev, threads, smem, b};
    blocks = b;
    return MSDA_OK;
}


// Launches one compute kernel over all rows as a persistent wave; the row
// records hold `padded_samples` slots.
msda_status launch_rows(const void *kernel, int rpw, size_t record_bytes, int padded_samples,
                        bool stages, KernelArgs &a, cudaStream_t stream)
{
    int dev = 0, sms = 0;
    msda_status st = current_device(dev, sms, &a.status);
    if (st != MSDA_OK)
        return st;
    // records of the warp's rows, then (power-of-two L*K up to 32) the warp's
    // double-buffered input stages; the kernel carves the same layout
    const size_t rec_warp = (size_t)rpw * msda::record_stride(padded_samples) * record_bytes;
    const size_t stage_warp = msda::stage_bytes_per_warp(stages, rpw, a.L * a.K);
    int warps = (int)(kCtaSmemBudget / (rec_warp + stage_warp));
    warps = warps < 1 ? 1 : (warps > msda::kMaxWarpsPerCta ? msda::kMaxWarpsPerCta : warps);
    const size_t smem = msda::align16(rec_warp * warps) + stage_warp * warps;
    const int threads = warps * 32;
    int blocks_per_sm = 0;
    st = occupancy(kernel, dev, threads, smem, blocks_per_sm);
    if (st != MSDA_OK)
        return st;
    a.rows_per_tile = (int64_t)warps * rpw;
    a.ntiles = (a.rows + a.rows_per_tile - 1) / a.rows_per_tile;
    // one resident wave, but no more CTAs than there are tiles
    int64_t ctas = (int64_t)sms * blocks_per_sm;
    if (ctas > a.ntiles)
        ctas = a.ntiles;
    void *params[] = {&a};
    if (cudaLaunchKernel(kernel, dim3((unsigned)ctas), dim3(threads), params, smem, stream) != cudaSuccess)
        return MSDA_ERR_CUDA;
    return MSDA_OK;
}

// Shared-memory budget of one CTA of the merged backward: every value type
// runs three CTAs per SM (the backward's register budget).
constexpr size_t kMergeSmemBudget = 72 * 1024;

// Launches the merged backward (tiles of one head of merge_qb consecutive
// queries of one batch; msda_kernels.cuh "merged reductions") as a
// persistent wave.  The tile takes as many warps (up to 8) as fit the budget
// with a hash table of at least one slot per contribution and 16-bit
// contribution ids; `fits` is false when not even one warp does (the caller
// then takes the direct path).
msda_status launch_merge(const void *kernel, int rpw, size_t record_bytes, int padded_samples, int D,
                         size_t budget, KernelArgs &a, const msda_problem *p, cudaStream_t stream,
                         bool &fits)
{
    fits = false;
    int dev = 0, sms = 0;
    msda_status st = current_device(dev, sms, &a.status);
    if (st != MSDA_OK)
        return st;
    const int stride = msda::record_stride(padded_samples);
    // no more warps than the queries of one batch need
    const int64_t need = (p->num_queries + rpw - 1) / rpw;
    int warps = need < msda::kMaxWarpsPerCta ? (int)need : msda::kMaxWarpsPerCta;
    int tslots = 0, tbits = 0;
    size_t smem = 0;
    for (; warps >= 1; --warps) {
        const int64_t rows = (int64_t)warps * rpw;
        const int64_t ids = rows * stride * 4;
        const int64_t items = rows * padded_samples * 4;
        tbits = 2;
        while ((int64_t(1) << tbits) < items)
            ++tbits;
        tslots = 1 << tbits;
        if (ids > 0xFFFF || tslots > 0x10000)
            continue;
        smem = msda::merge_layout((size_t)rows * stride * record_bytes, rows, stride, D, tslots).total;
        if (smem <= budget)
            break;
    }
    if (warps < 1)
        return MSDA_OK;
    fits = true;
    const int threads = warps * 32;
    int blocks_per_sm = 0;
    st = occupancy(kernel, dev, threads, smem, blocks_per_sm);
    if (st != MSDA_OK)
        return st;
    a.rows_per_tile = (int64_t)warps * rpw;
    a.merge_qb = a.rows_per_tile;
    a.merge_nqb = (p->num_queries + a.merge_qb - 1) / a.merge_qb;
    a.merge_tslots = tslots;
    a.merge_tbits = tbits;
    a.ntiles = p->batch * a.merge_nqb * p->num_heads;
    int64_t ctas = (int64_t)sms * blocks_per_sm;
    if (ctas > a.ntiles)
        ctas = a.ntiles;
    void *params[] = {&a};
    if (cudaLaunchKernel(kernel, dim3((unsigned)ctas), dim3(threads), params, smem, stream) != cudaSuccess)
        return MSDA_ERR_CUDA;
    return MSDA_OK;
}

msda_status launch_zero(float *a, int64_t na, float *b, int64_t nb, cudaStream_t stream)
{
    if (na == 0 && nb == 0)
        return MSDA_OK;
    int dev = 0, sms = 0;
    msda_status st = current_device(dev, sms);
    if (st != MSDA_OK)
        return st;
    // grid-stride over at most MSDA_ZERO_CTAS_PER_SM CTAs per SM
    int64_t work = na / 4 > nb ? na / 4 : nb;
    int64_t blocks = (work + 255) / 256;
    if (blocks > (int64_t)sms * MSDA_ZERO_CTAS_PER_SM)
        blocks = (int64_t)sms * MSDA_ZERO_CTAS_PER_SM;
    if (blocks < 1)
        blocks = 1;
    msda::zero_kernel<<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<float4 *>(a), na / 4, b, nb);
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status launch_to_bf16(const float *src, void *dst, int64_t n, cudaStream_t stream)
{
    if (n == 0)
        return MSDA_OK;
    int dev = 0, sms = 0;
    msda_status st = current_device(dev, sms);
    if (st != MSDA_OK)
        return st;
    int64_t n8 = n / 8;
    int64_t blocks = (n8 + 255) / 256;
    if (blocks > (int64_t)sms * 8)
        blocks = (int64_t)sms * 8;
    msda::f32_to_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        reinterpret_cast<const float4 *>(src), reinterpret_cast<uint4 *>(dst), n8);
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

// Kernel selection -----------------------------------------------------------

// The forward with rows split over MSDA_FWD_SPLIT lane groups
// (msda_kernels.cuh, forward_kernel SPLIT), taken for problems whose rows,
// one lane group each, would not fill one resident wave of the unsplit
// kernel.  Returns false (nothing launched) when the problem is larger.
// The general kernels split on the same rule, so that a query order never
// changes a row's summation order.
template <typename T, int DD, bool FUSED, bool SHORT>
bool try_forward_split(KernelArgs &a, bool gen, cudaStream_t s, msda_status &st)
{
    constexpr int rpw0 = msda::forward_rows_per_warp<T, DD>();
    constexpr int rpw = rpw0 / MSDA_FWD_SPLIT;
    static_assert(MSDA_FWD_SPLIT >= 1 && rpw >= 1, "split rows must fit a warp");
    if (MSDA_FWD_SPLIT == 1)
        return false;
    int dev = 0, sms = 0;
    if (current_device(dev, sms) != MSDA_OK)
        return false;
    const int64_t warps = (a.rows + rpw0 - 1) / rpw0;
    if (warps >= (int64_t)sms * msda::kMaxWarpsPerCta * msda::FwdTune<T, SHORT>::kMinCtas)
        return false;
    st = launch_rows(gen ? (const void *)msda::forward_kernel<T, DD, FUSED, true, SHORT, MSDA_FWD_SPLIT>
                         : (const void *)msda::forward_kernel<T, DD, FUSED, false, SHORT, MSDA_FWD_SPLIT>,
                     rpw, kForwardRecordBytes, a.L * a.K, false, a, s);
    return true;
}

// The general kernels (query order, DCN grid) are separate instantiations, so
// that the plain attention kernels carry none of their branches.
template <bool FUSED>
msda_status launch_forward(const msda_problem *p, KernelArgs &a, cudaStream_t s)
{
    const bool gen = a.order != nullptr || a.dcn != 0 || a.stage != 0;
    msda_status st = MSDA_OK;
    // (staged inputs, a per-call option, need whole rows per lane group)
    if (!a.stage && p->value_dtype == MSDA_F32) {
        if ((p->head_dim == 8 && try_forward_split<float, 8, FUSED, false>(a, gen, s, st)) ||
            (p->head_dim == 16 && try_forward_split<float, 16, FUSED, false>(a, gen, s, st)) ||
            (p->head_dim == 32 && try_forward_split<float, 32, FUSED, false>(a, gen, s, st)))
            return st;
    }
    if (!a.stage && p->value_dtype == MSDA_BF16 && a.L * a.K <= 16) {
        if ((p->head_dim == 8 && try_forward_split<__nv_bfloat16, 8, FUSED, true>(a, gen, s, st)) ||
            (p->head_dim == 16 && try_forward_split<__nv_bfloat16, 16, FUSED, true>(a, gen, s, st)) ||
            (p->head_dim == 32 && try_forward_split<__nv_bfloat16, 32, FUSED, true>(a, gen, s, st)) ||
            (p->head_dim == 64 && try_forward_split<__nv_bfloat16, 64, FUSED, true>(a, gen, s, st)))
            return st;
    }
#define MSDA_FWD_CASE(T, DD)                                                                      \
    case DD:                                                                                       \
        return launch_rows(gen ? (const void *)msda::forward_kernel<T, DD, FUSED, true>          \
                               : (const void *)msda::forward_kernel<T, DD, FUSED, false>,        \
                           msda::forward_rows_per_warp<T, DD>(),                                 \
                           kForwardRecordBytes, a.L * a.K,                                       \
                           msda::forward_stages<T>() || (a.stage && !a.order), a, s);
    if (p->value_dtype == MSDA_F32) {
        switch (p->head_dim) {
            MSDA_FWD_CASE(float, 8) MSDA_FWD_CASE(float, 16) MSDA_FWD_CASE(float, 32)
            MSDA_FWD_CASE(float, 64) MSDA_FWD_CASE(float, 128) MSDA_FWD_CASE(float, 256)
        }
    } else if (p->value_dtype == MSDA_BF16) {
        // bf16 rows of at most 16 samples take the SHORT tuning (msda_kernels.cuh)
        const bool short_rows = a.L * a.K <= 16;
#define MSDA_FWD_CASE_BF16(DD)                                                                     \
    case DD:                                                                                        \
        return launch_rows(                                                                         \
            short_rows ? (gen ? (const void *)msda::forward_kernel<__nv_bfloat16, DD, FUSED, true, true>    \
                              : (const void *)msda::forward_kernel<__nv_bfloat16, DD, FUSED, false, true>)  \
                       : (gen ? (const void *)msda::forward_kernel<__nv_bfloat16, DD, FUSED, true, false>   \
                              : (const void *)msda::forward_kernel<__nv_bfloat16, DD, FUSED, false, false>), \
            msda::forward_rows_per_warp<__nv_bfloat16, DD>(), kForwardRecordBytes, a.L * a.K,     \
            msda::forward_stages<__nv_bfloat16>() || (a.stage && !a.order), a, s);
        switch (p->head_dim) {
            MSDA_FWD_CASE_BF16(8) MSDA_FWD_CASE_BF16(16) MSDA_FWD_CASE_BF16(32)
            MSDA_FWD_CASE_BF16(64) MSDA_FWD_CASE_BF16(128) MSDA_FWD_CASE_BF16(256)
        }
#undef MSDA_FWD_CASE_BF16
    } else if (p->value_dtype == MSDA_S8) {
        switch (p->head_dim) {
            MSDA_FWD_CASE(msda::S8, 8) MSDA_FWD_CASE(msda::S8, 16) MSDA_FWD_CASE(msda::S8, 32)
            MSDA_FWD_CASE(msda::S8, 64) MSDA_FWD_CASE(msda::S8, 128) MSDA_FWD_CASE(msda::S8, 256)
        }
    } else {
        switch (p->head_dim) {
            MSDA_FWD_CASE(msda::E4M3, 8) MSDA_FWD_CASE(msda::E4M3, 16) MSDA_FWD_CASE(msda::E4M3, 32)
            MSDA_FWD_CASE(msda::E4M3, 64) MSDA_FWD_CASE(msda::E4M3, 128) MSDA_FWD_CASE(msda::E4M3, 256)
        }
    }
#undef MSDA_FWD_CASE
    return MSDA_ERR_UNSUPPORTED;
}

// Backward kernel for (T, D): direct grad_value reductions, or merged ones
// when the caller asks (MSDA_MERGE_REDUCTIONS), no query order is given
// (merged tiles follow the natural order) and a merged tile fits.
template <typename T, int D, bool FUSED>
msda_status launch_backward_td(const msda_problem *p, KernelArgs &a, cudaStream_t s)
{
    const bool gen = a.order != nullptr || a.dcn != 0;
    const int rpw = msda::backward_rows_per_warp<T, D>();
    const size_t rec = FUSED ? kFusedBackwardRecordBytes : kBackwardRecordBytes;
    const int pp = msda::backward_padded_samples<T, D>(a.L * a.K);
    if (!a.order && (p->flags & MSDA_MERGE_REDUCTIONS)) {
        const void *k = gen ? (const void *)msda::backward_kernel<T, D, FUSED, true, true>
                            : (const void *)msda::backward_kernel<T, D, FUSED, false, true>;
        bool fits = false;
        msda_status st = launch_merge(k, rpw, rec, pp, D, kMergeSmemBudget, a, p, s, fits);
        if (st != MSDA_OK || fits)
            return st;
    }
    const void *k = gen ? (const void *)msda::backward_kernel<T, D, FUSED, true, false>
                        : (const void *)msda::backward_kernel<T, D, FUSED, false, false>;
    return launch_rows(k, rpw, rec, pp, false, a, s);
}

template <bool FUSED>
msda_status launch_backward(const msda_problem *p, KernelArgs &a, cudaStream_t s)
{
#define MSDA_BWD_CASE(T, DD) \
    case DD:                 \
        return launch_backward_td<T, DD, FUSED>(p, a, s);
    if (p->value_dtype == MSDA_F32) {
        switch (p->head_dim) {
            MSDA_BWD_CASE(float, 8) MSDA_BWD_CASE(float, 16) MSDA_BWD_CASE(float, 32)
            MSDA_BWD_CASE(float, 64) MSDA_BWD_CASE(float, 128) MSDA_BWD_CASE(float, 256)
        }
    } else if (p->value_dtype == MSDA_BF16) {
        switch (p->head_dim) {
            MSDA_BWD_CASE(__nv_bfloat16, 8) MSDA_BWD_CASE(__nv_bfloat16, 16)
            MSDA_BWD_CASE(__nv_bfloat16, 32) MSDA_BWD_CASE(__nv_bfloat16, 64)
            MSDA_BWD_CASE(__nv_bfloat16, 128) MSDA_BWD_CASE(__nv_bfloat16, 256)
        }
    } else if (p->value_dtype == MSDA_S8) {
        switch (p->head_dim) {
            MSDA_BWD_CASE(msda::S8, 8) MSDA_BWD_CASE(msda::S8, 16) MSDA_BWD_CASE(msda::S8, 32)
            MSDA_BWD_CASE(msda::S8, 64) MSDA_BWD_CASE(msda::S8, 128) MSDA_BWD_CASE(msda::S8, 256)
        }
    } else {
        switch (p->head_dim) {
            MSDA_BWD_CASE(msda::E4M3, 8) MSDA_BWD_CASE(msda::E4M3, 16) MSDA_BWD_CASE(msda::E4M3, 32)
            MSDA_BWD_CASE(msda::E4M3, 64) MSDA_BWD_CASE(msda::E4M3, 128) MSDA_BWD_CASE(msda::E4M3, 256)
        }
    }
#undef MSDA_BWD_CASE
    return MSDA_ERR_UNSUPPORTED;
}

KernelArgs base_args(const msda_problem *p, const void *value, const int64_t *shapes,
                     const int64_t *starts)
{
    KernelArgs a = {};
    a.value = value;
    a.shapes = shapes;
    a.starts = starts;
    a.rows = p->batch * p->num_queries * p->num_heads;
    a.S = p->num_keys;
    a.Q = (int)p->num_queries;
    a.M = p->num_heads;
    a.L = p->num_levels;
    a.K = p->num_points;
    a.withhold_copy = (p->flags & MSDA_TEST_WITHHOLD_COPY) ? 1 : 0;
    a.stage = (p->flags & MSDA_STAGE_INPUTS) ? 1 : 0;
    a.order = (p->batch * p->num_queries > 0) ? p->query_order : nullptr;
    a.scale = scaled_dtype(p->value_dtype) ? p->value_scale : nullptr;
    return a;
}

struct Sizes {
    int64_t value, samples, rows_d, queries;
};

Sizes sizes_of(const msda_problem *p)
{
    Sizes z;
    z.value = p->batch * p->num_keys * p->num_heads * p->head_dim;
    z.samples = p->batch * p->num_queries * p->num_heads * p->num_levels * p->num_points;
    z.rows_d = p->batch * p->num_queries * p->num_heads * p->head_dim;
    z.queries = p->batch * p->num_queries;
    return z;
}

bool geometry_ptrs_ok(const msda_problem *p, const int64_t *shapes, const int64_t *starts)
{
    (void)p;
    return shapes != nullptr && starts != nullptr && aligned16(shapes) && aligned16(starts);
}

// Shared tail of both backward entry points: zero, run, convert.
template <bool FUSED>
msda_status run_backward(const msda_problem *p, KernelArgs &a, void *grad_value, void *workspace,
                         size_t workspace_bytes, cudaStream_t s)
{
    const Sizes z = sizes_of(p);
    const bool to_bf16 = (p->flags & MSDA_GRAD_VALUE_BF16) != 0;
    float *acc = static_cast<float *>(grad_value);
    if (to_bf16) {
        if (workspace_bytes < (size_t)z.value * sizeof(float) || !ptr_ok(workspace, z.value))
            return MSDA_ERR_INVALID_ARG;
        acc = static_cast<float *>(workspace);
    }
    a.grad_value = acc;
    msda_status st = MSDA_OK;
    if (!(p->flags & MSDA_ACCUMULATE_GRADS)) {
        st = launch_zero(acc, z.value, FUSED ? a.grad_ref : nullptr,
                         (FUSED && a.grad_ref) ? z.queries * 2 : 0, s);
        if (st != MSDA_OK)
            return st;
    }
    if (a.rows > 0) {
        st = launch_backward<FUSED>(p, a, s);
        if (st != MSDA_OK)
            return st;
    }
    if (to_bf16)
        return launch_to_bf16(acc, grad_value, z.value, s);
    return MSDA_OK;
}

// Backward without any allocation ---------------------------------------------
//
// Some callers cannot allocate device memory when they run the backward pass:
// a host framework that hands an extension only its input and output tensors
// and no workspace, or a serving process whose device memory is fixed at
// start-up and must not change while requests are in flight.  For them the
// bf16-grad_value backward can accumulate in this library-owned buffer instead
// of a caller workspace.  Every GPU that loads the library holds it until the
// process exits.
constexpr int64_t kNoAllocScratchFloats = int64_t(4) << 20;  // 16 MiB of float32
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// Device address of g_noalloc_scratch, looked up once per device (with that
// device current) on the first call there.  In host code the array's name is
// only a host-side stand-in, never a device address.
float *g_noalloc_ptr[kMaxDevices];

msda_status noalloc_scratch(int dev, float **ptr)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return MSDA_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *ptr = g_noalloc_ptr[dev];
    return MSDA_OK;
}

// DCNv3 core as the attention kernels' non-fused path: keys = the H*W input
// pixels, queries = the Ho*Wo output pixels, heads = groups, head_dim =
// group channels, levels = kernel rows, points = kernel columns.
msda_status dcn_to_problem(const msda_dcn_problem *d, msda_problem &p, int64_t &ho, int64_t &wo)
{
    if (!d)
        return MSDA_ERR_INVALID_ARG;
    if (d->batch < 0 || d->height < 1 || d->width < 1 || d->groups < 1 || d->group_channels < 1 ||
        d->kernel_h < 1 || d->kernel_w < 1 || d->stride_h < 1 || d->stride_w < 1 || d->pad_h < 0 ||
        d->pad_w < 0 || d->dilation_h < 1 || d->dilation_w < 1)
        return MSDA_ERR_INVALID_ARG;
    if (d->height > 65535 || d->width > 65535 || d->pad_h > 65535 || d->pad_w > 65535 ||
        d->stride_h > 65535 || d->stride_w > 65535 || d->dilation_h > 65535 || d->dilation_w > 65535)
        return MSDA_ERR_UNSUPPORTED;
    ho = ((int64_t)d->height + 2 * (int64_t)d->pad_h - (int64_t)d->dilation_h * (d->kernel_h - 1) - 1);
    wo = ((int64_t)d->width + 2 * (int64_t)d->pad_w - (int64_t)d->dilation_w * (d->kernel_w - 1) - 1);
    ho = ho < 0 ? 0 : ho / d->stride_h + 1;
    wo = wo < 0 ? 0 : wo / d->stride_w + 1;
    p = msda_problem{};
    p.batch = d->batch;
    p.num_keys = (int64_t)d->height * d->width;
    p.num_queries = ho * wo;
    p.num_heads = d->groups;
    p.head_dim = d->group_channels;
    p.num_levels = d->kernel_h;
    p.num_points = d->kernel_w;
    p.value_dtype = d->value_dtype;
    p.flags = d->flags;
    p.value_scale = d->value_scale;
    if (p.flags & MSDA_TEST_WITHHOLD_COPY)
        return MSDA_ERR_INVALID_ARG;
    return check_problem(&p);
}

void dcn_args(const msda_dcn_problem *d, int64_t wo, KernelArgs &a)
{
    a.dcn = 1;
    a.dcn_h = d->height;
    a.dcn_w = d->width;
    a.dcn_wo = (int)wo;
    a.stride_h = d->stride_h;
    a.stride_w = d->stride_w;
    a.pad_h = d->pad_h;
    a.pad_w = d->pad_w;
    a.dil_h = d->dilation_h;
    a.dil_w = d->dilation_w;
}

// Tensor-core dense layers (msda_gemm.cuh) ------------------------------------

// Widest output tile, in 128-column MMAs (1 or 2; a tuning knob).
#ifndef MSDA_GEMM_MAX_SUB
#define MSDA_GEMM_MAX_SUB 2
#endif
constexpr int kGemmMaxSub = MSDA_GEMM_MAX_SUB;
// Output tile of the query head, in 128-column MMAs (two measured 43.6
// against 45.0 us for one on 87040 rows of a 256 -> 384 head).
#ifndef MSDA_GEMM_HEAD_SUB
#define MSDA_GEMM_HEAD_SUB 2
#endif

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links no driver library).
PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

msda_status tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000 &fn)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_encode_tiled) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !f)
            return MSDA_ERR_CUDA;
        g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    fn = g_encode_tiled;
    return MSDA_OK;
}

// Tensor map of a row-major matrix [rows, cols] of `dtype` moved in boxes of
// box_rows x box_cols elements (box_cols * element size = 128 bytes) with the
// 128-byte swizzle the MMA descriptors and the epilogue boxes use; rows and
// columns outside the matrix read as zero and are not written.
msda_status tile_map(CUtensorMap &map, const void *ptr, CUtensorMapDataType dtype, int64_t rows, int64_t cols,
                     int box_cols, int box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    msda_status st = tensor_map_encoder(encode);
    if (st != MSDA_OK)
        return st;
    const int esize = dtype == CU_TENSOR_MAP_DATA_TYPE_FLOAT32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(&map, dtype, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MSDA_OK : MSDA_ERR_CUDA;
}

// Operand map: bf16 [rows, cols] in 128-row x 64-column boxes.
msda_status operand_map(CUtensorMap &map, const void *ptr, int64_t rows, int64_t cols)
{
    return tile_map(map, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rows, cols, msda_gemm::kBK, msda_gemm::kBM);
}

// Output map: 32-row boxes of 128 bytes (32 float32 or 64 bf16 columns).
msda_status output_map(CUtensorMap &map, void *ptr, bool bf16, int64_t rows, int64_t cols)
{
    return tile_map(map, ptr, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rows,
                    cols, bf16 ? 64 : 32, 32);
}

template <int NSUB, bool WRES>
msda_status launch_gemm_n(const CUtensorMap &mx, const CUtensorMap &mw, const CUtensorMap &mo0,
                          const CUtensorMap &mo1, msda_gemm::Params &p, int sms, int dev, cudaStream_t s)
{
    using C = msda_gemm::Cfg<NSUB, WRES>;
    const void *k = (const void *)msda_gemm::gemm_kernel<NSUB, WRES>;
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, k) != cudaSuccess)
        return MSDA_ERR_CUDA;
    msda_status st;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        st = raise_smem_limit(k, dev);
    }
    if (st != MSDA_OK)
        return st;
    // as many stages as the shared memory left after the w area holds
    const int avail = optin - (int)fa.sharedSizeBytes;
    p.stages = (avail - C::smem_bytes(p.w_bytes, 0)) / C::kStageBytes;
    if (p.stages > msda_gemm::kMaxStages)
        p.stages = msda_gemm::kMaxStages;
    if (p.stages < 2)
        return MSDA_ERR_UNSUPPORTED;
    const int smem = C::smem_bytes(p.w_bytes, p.stages);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    // one persistent CTA per SM (the shared memory admits one); with the
    // weight resident, a multiple of n_tiles CTAs, so that each CTA keeps
    // one column tile
    int64_t grid = WRES ? (int64_t)(sms / p.n_tiles) * p.n_tiles : sms;
    if (grid > tiles)
        grid = tiles;
    msda_gemm::gemm_kernel<NSUB, WRES><<<(unsigned)grid, msda_gemm::kThreads, smem, s>>>(mx, mw, mo0, mo1, p);
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

template <int NSUB>
msda_status launch_gemm_nsub(const CUtensorMap &mx, const CUtensorMap &mw, const CUtensorMap &mo0,
                             const CUtensorMap &mo1, msda_gemm::Params &p, cudaStream_t s)
{
    using C = msda_gemm::Cfg<NSUB, true>;
    int dev = 0, sms = 0;
    msda_status st = current_device(dev, sms, &p.status);
    if (st != MSDA_OK)
        return st;
    p.m_tiles = (p.rows + msda_gemm::kBM - 1) / msda_gemm::kBM;
    p.n_tiles = (p.N + C::kBN - 1) / C::kBN;
    const int nkb = (p.K + msda_gemm::kBK - 1) / msda_gemm::kBK;
    // the weight stays in shared memory when its K blocks fit the area
    if (nkb <= C::kMaxKBlocks && p.n_tiles <= sms) {
        p.w_bytes = nkb * NSUB * msda_gemm::kBSubBytes;
        return launch_gemm_n<NSUB, true>(mx, mw, mo0, mo1, p, sms, dev, s);
    }
    p.w_bytes = 0;
    return launch_gemm_n<NSUB, false>(mx, mw, mo0, mo1, p, sms, dev, s);
}

msda_status launch_gemm(int nsub, const CUtensorMap &mx, const CUtensorMap &mw, const CUtensorMap &mo0,
                        const CUtensorMap &mo1, msda_gemm::Params &p, cudaStream_t s)
{
    switch (nsub) {
    case 1: return launch_gemm_nsub<1>(mx, mw, mo0, mo1, p, s);
    case 2: return launch_gemm_nsub<2>(mx, mw, mo0, mo1, p, s);
    }
    return MSDA_ERR_UNSUPPORTED;
}

// Query-head sizes: P = M*L*K with L*K a power of two <= 32 and P a multiple
// of 32 (a 32-column chunk of the head is all offsets or whole softmax runs).
msda_status head_sizes(const msda_problem *p, int64_t &rows, int &P, int &LK)
{
    if (!p || p->batch < 0 || p->num_queries < 0 || p->num_heads < 1 || p->num_levels < 1 ||
        p->num_levels > msda::kMaxLevels || p->num_points < 1)
        return MSDA_ERR_INVALID_ARG;
    LK = p->num_levels * p->num_points;
    const int64_t P64 = (int64_t)p->num_heads * LK;
    if (LK > 32 || (LK & (LK - 1)) != 0 || P64 % 32 != 0 || 3 * P64 > (int64_t(1) << 20))
        return MSDA_ERR_UNSUPPORTED;
    rows = p->batch * p->num_queries;
    if (rows >= (int64_t(1) << 31))
        return MSDA_ERR_UNSUPPORTED;
    P = (int)P64;
    return MSDA_OK;
}

// NVTX range around each entry point that enqueues work, so that a profiler
// timeline shows the library calls (no-ops when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
#define MSDA_TRACE() NvtxRange msda_trace_range_(__func__)

}  // namespace

extern "C" {

msda_status msda_dcn_output_size(const msda_dcn_problem *problem, int64_t *out_h, int64_t *out_w)
{
    msda_problem p;
    int64_t ho = 0, wo = 0;
    msda_status st = dcn_to_problem(problem, p, ho, wo);
    if (st != MSDA_OK)
        return st;
    if (!out_h || !out_w)
        return MSDA_ERR_INVALID_ARG;
    *out_h = ho;
    *out_w = wo;
    return MSDA_OK;
}

msda_status msda_dcn_forward(const msda_dcn_problem *problem, const void *input, const float *offset,
                             const float *mask, void *output, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_problem p;
    int64_t ho = 0, wo = 0;
    msda_status st = dcn_to_problem(problem, p, ho, wo);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(&p);
    if (!vec_ptr_ok(input, z.value) || !ptr_ok(offset, z.samples * 2) || !ptr_ok(mask, z.samples) ||
        !vec_ptr_ok(output, z.rows_d))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(&p, input, nullptr, nullptr);
    if (a.rows == 0)
        return MSDA_OK;
    dcn_args(problem, wo, a);
    a.loc = offset;
    a.attn = mask;
    a.out = output;
    return launch_forward<false>(&p, a, reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_dcn_backward(const msda_dcn_problem *problem, const void *input, const float *offset,
                              const float *mask, const void *grad_output, void *grad_input,
                              float *grad_offset, float *grad_mask, void *workspace,
                              size_t workspace_bytes, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_problem p;
    int64_t ho = 0, wo = 0;
    msda_status st = dcn_to_problem(problem, p, ho, wo);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(&p);
    if (!vec_ptr_ok(input, z.value) || !ptr_ok(offset, z.samples * 2) || !ptr_ok(mask, z.samples) ||
        !ptr_ok(grad_output, z.rows_d) || !ptr_ok(grad_input, z.value) ||
        !ptr_ok(grad_offset, z.samples * 2) || !ptr_ok(grad_mask, z.samples))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(&p, input, nullptr, nullptr);
    dcn_args(problem, wo, a);
    a.loc = offset;
    a.attn = mask;
    a.grad_out = grad_output;
    a.grad_loc = grad_offset;
    a.grad_attn = grad_mask;
    return run_backward<false>(&p, a, grad_input, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_dcn_backward_workspace_size(const msda_dcn_problem *problem, size_t *bytes)
{
    msda_problem p;
    int64_t ho = 0, wo = 0;
    msda_status st = dcn_to_problem(problem, p, ho, wo);
    if (st != MSDA_OK)
        return st;
    return msda_backward_workspace_size(&p, bytes);
}

msda_status msda_forward(const msda_problem *problem, const void *value,
                         const int64_t *spatial_shapes, const int64_t *level_start_index,
                         const float *sampling_locations, const float *attention_weights,
                         void *output, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(problem);
    if (!vec_ptr_ok(value, z.value) || !geometry_ptrs_ok(problem, spatial_shapes, level_start_index) ||
        !ptr_ok(sampling_locations, z.samples * 2) || !ptr_ok(attention_weights, z.samples) ||
        !vec_ptr_ok(output, z.rows_d))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(problem, value, spatial_shapes, level_start_index);
    if (a.rows == 0)
        return MSDA_OK;
    a.loc = sampling_locations;
    a.attn = attention_weights;
    a.out = output;
    return launch_forward<false>(problem, a, reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_backward(const msda_problem *problem, const void *value,
                          const int64_t *spatial_shapes, const int64_t *level_start_index,
                          const float *sampling_locations, const float *attention_weights,
                          const void *grad_output, void *grad_value,
                          float *grad_sampling_locations, float *grad_attention_weights,
                          void *workspace, size_t workspace_bytes, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(problem);
    if (!vec_ptr_ok(value, z.value) || !geometry_ptrs_ok(problem, spatial_shapes, level_start_index) ||
        !ptr_ok(sampling_locations, z.samples * 2) || !ptr_ok(attention_weights, z.samples) ||
        !ptr_ok(grad_output, z.rows_d) || !ptr_ok(grad_value, z.value) ||
        !ptr_ok(grad_sampling_locations, z.samples * 2) || !ptr_ok(grad_attention_weights, z.samples))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(problem, value, spatial_shapes, level_start_index);
    a.loc = sampling_locations;
    a.attn = attention_weights;
    a.grad_out = grad_output;
    a.grad_loc = grad_sampling_locations;
    a.grad_attn = grad_attention_weights;
    return run_backward<false>(problem, a, grad_value, workspace, workspace_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_fused_forward(const msda_problem *problem, const void *value,
                               const int64_t *spatial_shapes, const int64_t *level_start_index,
                               const float *reference_points, const float *sampling_offsets,
                               const float *attention_logits, void *output,
                               float *attention_weights_out, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(problem);
    if (!vec_ptr_ok(value, z.value) || !geometry_ptrs_ok(problem, spatial_shapes, level_start_index) ||
        !ptr_ok(reference_points, z.queries * 2) || !ptr_ok(sampling_offsets, z.samples * 2) ||
        !ptr_ok(attention_logits, z.samples) || !vec_ptr_ok(output, z.rows_d) ||
        (attention_weights_out && !aligned16(attention_weights_out)))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(problem, value, spatial_shapes, level_start_index);
    if (a.rows == 0)
        return MSDA_OK;
    a.ref = reference_points;
    a.off = sampling_offsets;
    a.logits = attention_logits;
    a.out = output;
    a.attn_out = attention_weights_out;
    return launch_forward<true>(problem, a, reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_fused_backward(const msda_problem *problem, const void *value,
                                const int64_t *spatial_shapes, const int64_t *level_start_index,
                                const float *reference_points, const float *sampling_offsets,
                                const float *attention_logits, const void *grad_output,
                                void *grad_value, float *grad_reference_points,
                                float *grad_sampling_offsets, float *grad_attention_logits,
                                void *workspace, size_t workspace_bytes, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(problem);
    if (!vec_ptr_ok(value, z.value) || !geometry_ptrs_ok(problem, spatial_shapes, level_start_index) ||
        !ptr_ok(reference_points, z.queries * 2) || !ptr_ok(sampling_offsets, z.samples * 2) ||
        !ptr_ok(attention_logits, z.samples) || !ptr_ok(grad_output, z.rows_d) ||
        !ptr_ok(grad_value, z.value) || !ptr_ok(grad_sampling_offsets, z.samples * 2) ||
        !ptr_ok(grad_attention_logits, z.samples) ||
        (grad_reference_points && !aligned16(grad_reference_points)))
        return MSDA_ERR_INVALID_ARG;
    KernelArgs a = base_args(problem, value, spatial_shapes, level_start_index);
    a.ref = reference_points;
    a.off = sampling_offsets;
    a.logits = attention_logits;
    a.grad_out = grad_output;
    a.grad_ref = grad_reference_points;
    a.grad_off = grad_sampling_offsets;
    a.grad_logits = grad_attention_logits;
    return run_backward<true>(problem, a, grad_value, workspace, workspace_bytes,
                              reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_zero_grads(const msda_problem *problem, float *grad_value,
                            float *grad_reference_points, msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const Sizes z = sizes_of(problem);
    if (!ptr_ok(grad_value, z.value) || (grad_reference_points && !aligned16(grad_reference_points)))
        return MSDA_ERR_INVALID_ARG;
    return launch_zero(grad_value, z.value, grad_reference_points,
                       grad_reference_points ? z.queries * 2 : 0,
                       reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_backward_noalloc(const msda_problem *problem, const void *value,
                                  const int64_t *spatial_shapes, const int64_t *level_start_index,
                                  const float *sampling_locations, const float *attention_weights,
                                  const void *grad_output, void *grad_value,
                                  float *grad_sampling_locations, float *grad_attention_weights,
                                  msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    if (problem->flags & ~(uint32_t)(MSDA_GRAD_VALUE_BF16 | MSDA_MERGE_REDUCTIONS))
        return MSDA_ERR_INVALID_ARG;
    const Sizes z = sizes_of(problem);
    if (z.value > kNoAllocScratchFloats)
        return MSDA_ERR_UNSUPPORTED;
    if (!vec_ptr_ok(value, z.value) || !geometry_ptrs_ok(problem, spatial_shapes, level_start_index) ||
        !ptr_ok(sampling_locations, z.samples * 2) || !ptr_ok(attention_weights, z.samples) ||
        !ptr_ok(grad_output, z.rows_d) || !ptr_ok(grad_value, z.value) ||
        !ptr_ok(grad_sampling_locations, z.samples * 2) || !ptr_ok(grad_attention_weights, z.samples))
        return MSDA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = current_device(dev, sms);
    if (st != MSDA_OK)
        return st;
    float *acc = nullptr;
    st = noalloc_scratch(dev, &acc);
    if (st != MSDA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    KernelArgs a = base_args(problem, value, spatial_shapes, level_start_index);
    a.loc = sampling_locations;
    a.attn = attention_weights;
    a.grad_out = grad_output;
    a.grad_loc = grad_sampling_locations;
    a.grad_attn = grad_attention_weights;
    a.grad_value = acc;
    // the buffer keeps the previous call's sums: clear it first
    st = launch_zero(acc, z.value, nullptr, 0, s);
    if (st != MSDA_OK)
        return st;
    if (a.rows > 0) {
        st = launch_backward<false>(problem, a, s);
        if (st != MSDA_OK)
            return st;
    }
    return launch_to_bf16(acc, grad_value, z.value, s);
}

// Per-(b, m) absmax, scale = amax / qmax, then the codes: the INT8 and FP8
// storage entry points differ only in qmax and the quantising kernel.
static msda_status quantize_value(const msda_problem *problem, const void *value, void *codes,
                                  float *value_scale, bool e4m3, msda_stream_t stream)
{
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    if (problem->value_dtype != MSDA_F32 && problem->value_dtype != MSDA_BF16)
        return MSDA_ERR_INVALID_ARG;
    const int64_t B = problem->batch, S = problem->num_keys;
    const int M = problem->num_heads, D = problem->head_dim;
    const int64_t n = B * S * M * (int64_t)D;
    if (B == 0)
        return MSDA_OK;
    if (!ptr_ok(value, n) || !vec_ptr_ok(codes, n) || !value_scale ||
        (reinterpret_cast<uintptr_t>(value_scale) & 3u) || D % 8 != 0)
        return MSDA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = current_device(dev, sms);
    if (st != MSDA_OK)
        return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t bm = B * M;
    if (cudaMemsetAsync(value_scale, 0, (size_t)bm * sizeof(float), s) != cudaSuccess)
        return MSDA_ERR_CUDA;
    // about four CTAs per SM in the reduction, each over >= 1 key of one (b, m)
    int64_t chunks = ((int64_t)sms * 4 + bm - 1) / bm;
    if (chunks > S)
        chunks = S;
    if (chunks * bm > 0x7fffffffLL)
        chunks = 0x7fffffffLL / bm;
    if (chunks < 1)
        return MSDA_ERR_UNSUPPORTED;
    unsigned *amax = reinterpret_cast<unsigned *>(value_scale);
    int64_t qblocks = (n / 8 + 255) / 256;
    if (qblocks > (int64_t)sms * 8)
        qblocks = (int64_t)sms * 8;
    const float qmax = e4m3 ? 448.f : 127.f;
    uint2 *q = static_cast<uint2 *>(codes);
    if (problem->value_dtype == MSDA_F32) {
        const float *v = static_cast<const float *>(value);
        msda::absmax_kernel<float><<<(unsigned)(chunks * bm), 256, 0, s>>>(v, S, M, D, (int)chunks, amax);
        msda::quant_scale_kernel<<<(unsigned)((bm + 255) / 256), 256, 0, s>>>(value_scale, bm, qmax);
        if (e4m3)
            msda::quantize_e4m3_kernel<float><<<(unsigned)qblocks, 256, 0, s>>>(v, value_scale, n / 8, S, M,
                                                                              D, q);
        else
            msda::quantize_s8_kernel<float><<<(unsigned)qblocks, 256, 0, s>>>(v, value_scale, n / 8, S, M, D,
                                                                            q);
    } else {
        const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(value);
        msda::absmax_kernel<__nv_bfloat16><<<(unsigned)(chunks * bm), 256, 0, s>>>(v, S, M, D, (int)chunks,
                                                                                  amax);
        msda::quant_scale_kernel<<<(unsigned)((bm + 255) / 256), 256, 0, s>>>(value_scale, bm, qmax);
        if (e4m3)
            msda::quantize_e4m3_kernel<__nv_bfloat16><<<(unsigned)qblocks, 256, 0, s>>>(
                v, value_scale, n / 8, S, M, D, q);
        else
            msda::quantize_s8_kernel<__nv_bfloat16><<<(unsigned)qblocks, 256, 0, s>>>(
                v, value_scale, n / 8, S, M, D, q);
    }
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_quantize_value_s8(const msda_problem *problem, const void *value, void *value_s8,
                                   float *value_scale, msda_stream_t stream)
{
    MSDA_TRACE();
    return quantize_value(problem, value, value_s8, value_scale, false, stream);
}

msda_status msda_quantize_value_e4m3(const msda_problem *problem, const void *value, void *value_e4m3,
                                     float *value_scale, msda_stream_t stream)
{
    MSDA_TRACE();
    return quantize_value(problem, value, value_e4m3, value_scale, true, stream);
}

msda_status msda_sort_queries(const msda_problem *problem, const float *points, int32_t *query_order,
                              msda_stream_t stream)
{
    MSDA_TRACE();
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    const int64_t bq = problem->batch * problem->num_queries;
    if (bq == 0)
        return MSDA_OK;
    if (!ptr_ok(points, bq * 2) || !query_order || (reinterpret_cast<uintptr_t>(query_order) & 3u))
        return MSDA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    msda::sort_queries_kernel<<<(unsigned)problem->batch, msda::kSortThreads, 0, s>>>(
        reinterpret_cast<const float2 *>(points), problem->num_queries, query_order);
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_linear(int64_t rows, int32_t in_features, int32_t out_features, const void *x,
                        const void *weight, const float *bias, void *out, int32_t out_dtype,
                        msda_stream_t stream)
{
    MSDA_TRACE();
    if (rows < 0 || rows >= (int64_t(1) << 31) || in_features < 8 || in_features % 8 != 0 ||
        out_features < 8 || out_features % 8 != 0 || out_features >= (1 << 20) ||
        (out_dtype != MSDA_F32 && out_dtype != MSDA_BF16))
        return MSDA_ERR_INVALID_ARG;
    if (rows == 0)
        return MSDA_OK;
    if (!x || !weight || !out || !aligned16(x) || !aligned16(weight) || !aligned16(out) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return MSDA_ERR_INVALID_ARG;
    const bool bf16 = out_dtype == MSDA_BF16;
    CUtensorMap mx, mw, mo;
    msda_status st = operand_map(mx, x, rows, in_features);
    if (st == MSDA_OK)
        st = operand_map(mw, weight, out_features, in_features);
    if (st == MSDA_OK)
        st = output_map(mo, out, bf16, rows, out_features);
    if (st != MSDA_OK)
        return st;
    msda_gemm::Params p = {};
    p.rows = (int)rows;
    p.N = out_features;
    p.K = in_features;
    p.bias = bias;
    p.epi = msda_gemm::kEpiStore;
    p.out_bf16 = bf16;
    return launch_gemm(out_features <= 128 ? 1 : kGemmMaxSub, mx, mw, mo, mo, p,
                       reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_query_head(const msda_problem *problem, int32_t in_features, const void *query,
                            const void *weight, const float *bias, const float *reference_points,
                            const int64_t *spatial_shapes, float *sampling_locations,
                            float *attention_weights, msda_stream_t stream)
{
    MSDA_TRACE();
    int64_t rows = 0;
    int P = 0, LK = 0;
    msda_status st = head_sizes(problem, rows, P, LK);
    if (st != MSDA_OK)
        return st;
    if (in_features < 8 || in_features % 8 != 0)
        return MSDA_ERR_INVALID_ARG;
    if (rows == 0)
        return MSDA_OK;
    if (!query || !weight || !aligned16(query) || !aligned16(weight) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) || !ptr_ok(reference_points, rows * 2) ||
        !spatial_shapes || !aligned16(spatial_shapes) || !ptr_ok(sampling_locations, rows * 2 * P) ||
        !ptr_ok(attention_weights, rows * P))
        return MSDA_ERR_INVALID_ARG;
    CUtensorMap mx, mw, mloc, mattn;
    st = operand_map(mx, query, rows, in_features);
    if (st == MSDA_OK)
        st = operand_map(mw, weight, 3 * (int64_t)P, in_features);
    if (st == MSDA_OK)
        st = output_map(mloc, sampling_locations, false, rows, 2 * (int64_t)P);
    if (st == MSDA_OK)
        st = output_map(mattn, attention_weights, false, rows, P);
    if (st != MSDA_OK)
        return st;
    msda_gemm::Params p = {};
    p.rows = (int)rows;
    p.N = 3 * P;
    p.K = in_features;
    p.bias = bias;
    p.epi = msda_gemm::kEpiHead;
    p.P = P;
    p.L = problem->num_levels;
    p.LK = LK;
    p.lk_mask = LK - 1;
    int ks = 0;
    while ((1 << ks) < problem->num_points)
        ++ks;
    p.k_shift = ks;  // L*K is a power of two, so K is one too
    p.ref = reference_points;
    p.shapes = spatial_shapes;
    p.withhold = (problem->flags & MSDA_TEST_WITHHOLD_COPY) ? 1 : 0;
    return launch_gemm(3 * P <= 128 ? 1 : MSDA_GEMM_HEAD_SUB, mx, mw, mloc, mattn, p,
                       reinterpret_cast<cudaStream_t>(stream));
}

msda_status msda_query_head_backward(const msda_problem *problem, const float *attention_weights,
                                     const float *grad_sampling_locations,
                                     const float *grad_attention_weights, const int64_t *spatial_shapes,
                                     float *grad_head, float *grad_reference_points, msda_stream_t stream)
{
    MSDA_TRACE();
    int64_t rows = 0;
    int P = 0, LK = 0;
    msda_status st = head_sizes(problem, rows, P, LK);
    if (st != MSDA_OK)
        return st;
    if (rows == 0)
        return MSDA_OK;
    if (!ptr_ok(attention_weights, rows * P) || !ptr_ok(grad_sampling_locations, rows * 2 * P) ||
        !ptr_ok(grad_attention_weights, rows * P) || !spatial_shapes || !aligned16(spatial_shapes) ||
        !ptr_ok(grad_head, rows * 3 * P) || (grad_reference_points && !aligned16(grad_reference_points)))
        return MSDA_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    st = current_device(dev, sms);
    if (st != MSDA_OK)
        return st;
    int64_t blocks = (rows + 7) / 8;
    if (blocks > (int64_t)sms * 8)
        blocks = (int64_t)sms * 8;
    msda::head_backward_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        rows, P, problem->num_levels, problem->num_points, attention_weights, grad_sampling_locations,
        grad_attention_weights, spatial_shapes, grad_head, grad_reference_points);
    return cudaGetLastError() == cudaSuccess ? MSDA_OK : MSDA_ERR_CUDA;
}

msda_status msda_backward_workspace_size(const msda_problem *problem, size_t *bytes)
{
    msda_status st = check_problem(problem);
    if (st != MSDA_OK)
        return st;
    if (!bytes)
        return MSDA_ERR_INVALID_ARG;
    *bytes = (problem->flags & MSDA_GRAD_VALUE_BF16) ? (size_t)sizes_of(problem).value * sizeof(float) : 0;
    return MSDA_OK;
}

msda_status msda_get_device_status(msda_stream_t stream, int32_t *code)
{
    if (!code)
        return MSDA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MSDA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, msda::g_device_status, sizeof(int)) != cudaSuccess)
        return MSDA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(msda::g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return MSDA_ERR_CUDA;
    *code = v;
    return MSDA_OK;
}

const char *msda_status_string(msda_status status)
{
    switch (status) {
    case MSDA_OK: return "success";
    case MSDA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or bad size)";
    case MSDA_ERR_UNSUPPORTED: return "sizes outside the supported range";
    case MSDA_ERR_CUDA: return "CUDA runtime error";
    case MSDA_ERR_DEVICE_CHECK: return "kernel found inconsistent spatial_shapes / level_start_index or a query_order entry out of range";
    case MSDA_ERR_DEVICE_TIMEOUT: return "kernel gave up waiting for an input copy";
    case MSDA_ERR_DEVICE_BOUNDS: return "checked build: a kernel found a row index outside its tensor";
    }
    return "unknown status";
}

const char *msda_version(void) { return "0.1.0"; }

}  // extern "C"
