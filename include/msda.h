/*
 * msda.h -- C ABI of the B200 (sm_100a) multi-scale deformable attention core.
 *
 * The operator (Deformable DETR's MSDeformAttn without its linear
 * projections).  For every batch b, query q and head m:
 *
 *   out[b,q,m,:] = sum_{l<L} sum_{k<K} A[b,q,m,l,k] * x^l_m( loc[b,q,m,l,k] )
 *
 * where x^l_m(p) bilinearly samples head m of level l of the flattened value
 * map at the normalized point p = (x, y) in [0,1]^2.  Sources (web pages on
 * the operator, cited by page and section):
 *   - the multi-scale sum and the level map phi_l:
 *       discosf.com/news/5175395 §2.2; cf-1.com/news/4799680 §3.1
 *   - sum over levels and points of A equals 1 (softmax over L*K):
 *       cf-1.com/news/4799680 §3.1-3.2; x-humanoid.csdn.net MSDA explainer §3
 *   - the flattened value [B, sum H_l*W_l, M, D] with spatial_shapes (H, W)
 *     and level_start_index: cf-1.com/news/4799680 §3.3 and §5.3
 *   - locations = reference_points + offsets / (W_l, H_l), offsets in level
 *     pixels without a sigmoid: cf-1.com/news/4799680 §3.2
 *   - bilinear sampling, pixel coordinate x = loc_x * W - 0.5 (grid_sample
 *     with align_corners=False on grid = 2*loc - 1), out-of-range corners
 *     masked to zero: cf-1.com/news/4799680 §5.3;
 *     x-humanoid.csdn.net MSDA explainer §3 note 2;
 *     discosf.com/news/5175395 §2.1-2.2
 * Readings taken where the pages are silent: a sample is taken only when
 * -1 < x < W and -1 < y < H (else it contributes 0 and has zero gradients);
 * at an integer coordinate the derivative is the one of the cell floor(x);
 * the backward pass is the exact derivative of the sum above.
 *
 * Conventions for every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major, each 16-byte aligned; value and output 32-byte aligned (they
 *     move in 32-byte vectors).  The library keeps no pointer after the call
 *     returns and allocates no memory.
 *   - value, output and grad_output hold value_dtype elements (float32 or
 *     bfloat16; with MSDA_S8 or MSDA_E4M3 value, output and grad_output are
 *     bfloat16);
 *     every other floating-point tensor is float32.  Accumulation is float32.
 *   - Locations and offsets are (x, y) pairs; spatial_shapes rows are (H, W).
 *   - spatial_shapes [L,2] and level_start_index [L] are int64 device arrays.
 *     Their consistency (H, W >= 1, start[0] = 0, start[l+1] = start[l] +
 *     H_l*W_l, sum = S) is checked by the kernels themselves: on a mismatch the
 *     work is skipped, outputs are left unspecified, and a code is recorded in
 *     a per-device status word that msda_get_device_status() returns.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).  The
 *     host-side checks below run before anything is enqueued; a call that
 *     returns an error has enqueued nothing.
 *   - Supported sizes: D (head_dim) in {8, 16, 32, 64, 128, 256};
 *     1 <= L <= 16; 1 <= K <= 32; L*K <= 128; 1 <= M; S < 2^27; S*M < 2^31;
 *     B*Q < 2^31;
 *     B*Q*M*L*K < 2^40; B or Q may be 0 (nothing to sample).
 *   - No C++ exception crosses this boundary.
 *   - Per-device state: on its first call on a device (with that device
 *     current) the library looks up the device's SM count and the device
 *     addresses of its status word and of the msda_backward_noalloc buffer,
 *     and keeps them for the life of the process.  cudaDeviceReset() destroys
 *     the context those addresses belong to: after a reset of a device, do not
 *     call the library on that device again in the same process.
 */
#ifndef MSDA_H_
#define MSDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSDA_API __attribute__((visibility("default")))
#else
#define MSDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that callers need
 * no CUDA header. */
typedef struct CUstream_st *msda_stream_t;

typedef enum msda_status {
    MSDA_OK = 0,
    MSDA_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, bad size */
    MSDA_ERR_UNSUPPORTED = 2,   /* valid, but outside the supported sizes */
    MSDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    MSDA_ERR_DEVICE_CHECK = 4,  /* a kernel found inconsistent geometry or a bad query_order entry */
    MSDA_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up waiting for an input copy
                                   (bounded wait) and read its inputs directly
                                   instead; a copy that may still be in flight
                                   is waited for (bounded) before the kernel
                                   ends */
    MSDA_ERR_DEVICE_BOUNDS = 6  /* checked build only (MSDA_BOUNDS_CHECK): a kernel
                                   found a corner row outside its tensor and
                                   skipped the access */
} msda_status;

typedef enum msda_dtype {
    MSDA_F32 = 0,
    MSDA_BF16 = 1,
    /* INT8 value storage (the quantisation note of the x-humanoid.csdn.net
     * MSDA explainer, §4: INT8 cuts the operator's memory traffic): value is
     * int8 q with one float32 scale per (batch, head) in
     * msda_problem.value_scale, and the operator samples q * scale; output
     * and grad_output are bfloat16; grad_value is the gradient with respect
     * to the dequantized value (float32, or bf16 with MSDA_GRAD_VALUE_BF16).
     * msda_quantize_value_s8 produces q and the scales. */
    MSDA_S8 = 2,
    /* FP8 value storage (the same note's low-precision storage): value is one
     * E4M3 code per element (the OCP 8-bit floating-point E4M3 encoding:
     * sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite
     * 448, no infinity) with one float32 scale per (batch, head) in
     * msda_problem.value_scale; otherwise as MSDA_S8.
     * msda_quantize_value_e4m3 produces the codes and the scales. */
    MSDA_E4M3 = 3
} msda_dtype;

/* msda_problem.flags */
#define MSDA_GRAD_VALUE_BF16 (1u << 0) /* backward writes grad_value as bf16;
                                          needs a float32 workspace */
#define MSDA_ACCUMULATE_GRADS (1u << 1) /* backward adds into grad_value (and
                                          grad_reference_points) instead of
                                          zeroing them first; float32 only */
#define MSDA_STAGE_INPUTS (1u << 2) /* forward: each warp copies its next rows'
                                          set-up inputs into shared memory with
                                          bulk copies (completion on an
                                          mbarrier, bounded wait) while it
                                          gathers the current rows, instead of
                                          loading them directly; power-of-two
                                          L*K <= 32, natural query order.  A
                                          performance option (off by default:
                                          slower with the default lane layout) */
#define MSDA_MERGE_REDUCTIONS (1u << 3) /* backward: per tile of consecutive
                                          queries of one head, merge in shared
                                          memory the grad_value contributions
                                          that share a corner row before
                                          reducing them (one reduction per
                                          distinct row instead of one per
                                          corner).  Results agree within float32
                                          rounding.  A performance option, off
                                          by default: on B200 the merge costs
                                          more than the reductions it saves on
                                          every workload measured.  Ignored with
                                          a query_order */
#define MSDA_TEST_WITHHOLD_COPY (1u << 31) /* testing only: kernels that stage
                                          their inputs with bulk copies arm
                                          the copy but never issue it, so
                                          their bounded wait runs out and
                                          they report MSDA_ERR_DEVICE_TIMEOUT
                                          (and finish on direct loads);
                                          msda_query_head's tensor-core
                                          kernel arms each CTA's first
                                          operand stage without loading it:
                                          its waits run out (about a second
                                          each), it reports the same status,
                                          writes no output, frees its tensor
                                          memory and returns */

/* Sizes of one call.  S = sum_l H_l * W_l. */
typedef struct msda_problem {
    int64_t batch;        /* B */
    int64_t num_keys;     /* S */
    int64_t num_queries;  /* Q */
    int32_t num_heads;    /* M */
    int32_t head_dim;     /* D */
    int32_t num_levels;   /* L */
    int32_t num_points;   /* K */
    int32_t value_dtype;  /* msda_dtype of value (and of output, grad_output
                             unless MSDA_S8: then bfloat16) */
    uint32_t flags;       /* MSDA_* flags above */
    /* Optional device array [B*Q] int32, 4-byte aligned: the order in which
     * the kernels process the queries, a permutation of 0 .. B*Q-1 (query
     * index b*Q + q), e.g. from msda_sort_queries.  NULL: natural order.
     * Each query's outputs are computed as in the natural order; what can
     * change is float32 rounding where the order decides the summation
     * order (grad_value, and the fused softmax sums, whose reduction pattern
     * can differ between ordered and natural-order set-up).  An entry outside 0 .. B*Q-1 is replaced by 0 and sets the
     * device status to MSDA_ERR_DEVICE_CHECK; repeated entries are not
     * detected (the rows of queries missing from the order are not written).
     * Read by the kernels on the stream: it must stay valid until they end. */
    const int32_t *query_order;
    /* MSDA_S8 / MSDA_E4M3 value only (ignored otherwise, required then): device array
     * [B, M] float32, 4-byte aligned, the dequantization scale of each
     * (batch, head).  Read by the kernels on the stream. */
    const float *value_scale;
} msda_problem;

/*
 * Forward of the core operator (discosf.com/news/5175395 §2.2;
 * cf-1.com/news/4799680 §3.1 and the argument list of §5.3).
 *   value               [B, S, M, D]        value_dtype
 *   spatial_shapes      [L, 2] int64        (H_l, W_l)
 *   level_start_index   [L]    int64
 *   sampling_locations  [B, Q, M, L, K, 2]  float32, normalized (x, y)
 *   attention_weights   [B, Q, M, L, K]     float32 (used as given; the
 *                                            operator does not renormalize)
 *   output              [B, Q, M, D]        value_dtype, overwritten
 */
MSDA_API msda_status msda_forward(const msda_problem *problem, const void *value,
                         const int64_t *spatial_shapes, const int64_t *level_start_index,
                         const float *sampling_locations, const float *attention_weights,
                         void *output, msda_stream_t stream);

/*
 * Backward of the core operator: the exact derivative of msda_forward
 * (bilinear sampling is differentiable in the coordinates,
 * discosf.com/news/5175395 §2.1).  Inputs as msda_forward plus
 *   grad_output              [B, Q, M, D]       value_dtype
 * Outputs, all overwritten:
 *   grad_value               [B, S, M, D]       float32 (bf16 with
 *                                               MSDA_GRAD_VALUE_BF16)
 *   grad_sampling_locations  [B, Q, M, L, K, 2] float32
 *   grad_attention_weights   [B, Q, M, L, K]    float32
 * grad_value is zeroed and then accumulated with float32 atomics, so its
 * summation order (and its last bits) vary from run to run.  With
 * MSDA_ACCUMULATE_GRADS the zero-fill is skipped and the gradients are added to
 * what grad_value holds (not allowed together with MSDA_GRAD_VALUE_BF16).
 * workspace: with MSDA_GRAD_VALUE_BF16, at least msda_backward_workspace_size()
 * bytes of device memory that the call may overwrite; otherwise ignored (may
 * be NULL).
 */
MSDA_API msda_status msda_backward(const msda_problem *problem, const void *value,
                          const int64_t *spatial_shapes, const int64_t *level_start_index,
                          const float *sampling_locations, const float *attention_weights,
                          const void *grad_output, void *grad_value,
                          float *grad_sampling_locations, float *grad_attention_weights,
                          void *workspace, size_t workspace_bytes, msda_stream_t stream);

/*
 * Fused forward: computes the sampling locations and the attention softmax
 * inside the kernel (cf-1.com/news/4799680 §3.2):
 *   loc[b,q,m,l,k] = reference_points[b,q] + sampling_offsets[b,q,m,l,k] / (W_l, H_l)
 *   A[b,q,m,:]     = softmax(attention_logits[b,q,m,:])   over the L*K points
 * then the forward sum.
 *   reference_points    [B, Q, 2]          float32, normalized (x, y), shared
 *                                          by every level and head
 *   sampling_offsets    [B, Q, M, L, K, 2] float32, pixels of level l
 *   attention_logits    [B, Q, M, L*K]     float32
 *   output              [B, Q, M, D]       value_dtype, overwritten
 *   attention_weights_out [B, Q, M, L, K]  float32 or NULL: the softmax, if
 *                                          the caller wants it
 */
MSDA_API msda_status msda_fused_forward(const msda_problem *problem, const void *value,
                               const int64_t *spatial_shapes, const int64_t *level_start_index,
                               const float *reference_points, const float *sampling_offsets,
                               const float *attention_logits, void *output,
                               float *attention_weights_out, msda_stream_t stream);

/*
 * Fused backward: msda_backward followed by the chain rule through the
 * location and softmax steps of msda_fused_forward:
 *   grad_sampling_offsets = grad_loc / (W_l, H_l)
 *   grad_reference_points = sum over (m, l, k) of grad_loc   (NULL: skipped)
 *   grad_attention_logits = A * (grad_A - sum_j A_j grad_A_j)
 * Inputs as msda_fused_forward plus grad_output [B, Q, M, D] (value_dtype).
 * Outputs (overwritten): grad_value as in msda_backward, grad_reference_points
 * [B, Q, 2], grad_sampling_offsets [B, Q, M, L, K, 2], grad_attention_logits
 * [B, Q, M, L*K], all float32 except grad_value with MSDA_GRAD_VALUE_BF16.
 * grad_reference_points is accumulated with atomics over the M heads; like
 * grad_value it is zeroed first unless MSDA_ACCUMULATE_GRADS is set.
 */
MSDA_API msda_status msda_fused_backward(const msda_problem *problem, const void *value,
                                const int64_t *spatial_shapes, const int64_t *level_start_index,
                                const float *reference_points, const float *sampling_offsets,
                                const float *attention_logits, const void *grad_output,
                                void *grad_value, float *grad_reference_points,
                                float *grad_sampling_offsets, float *grad_attention_logits,
                                void *workspace, size_t workspace_bytes, msda_stream_t stream);

/*
 * Zeroes the float32 accumulators of a backward call: grad_value
 * [B, S, M, D] and, if not NULL, grad_reference_points [B, Q, 2].  Together
 * with MSDA_ACCUMULATE_GRADS this splits the zero-fill from the backward
 * kernel (e.g. to accumulate several backward calls into one buffer).
 */
MSDA_API msda_status msda_zero_grads(const msda_problem *problem, float *grad_value,
                                     float *grad_reference_points, msda_stream_t stream);

/*
 * msda_backward with grad_value written as bf16, for callers that cannot
 * allocate device memory at call time (a host framework that gives an
 * extension only its input and output tensors and no workspace, or a
 * serving process whose device memory is fixed once it has started).  The
 * pages on the operator have no counterpart of this entry point; it is an
 * interface convenience of this library.
 *   Arguments: as msda_backward, without the workspace; grad_value is
 *   [B, S, M, D] bf16 (overwritten).  problem->flags may hold
 *   MSDA_GRAD_VALUE_BF16 (the output is bf16 either way) and
 *   MSDA_MERGE_REDUCTIONS, nothing else.
 *   Scratch: the float32 sums are kept in one buffer owned by the library,
 *   4 Mi floats (16 MiB) per GPU, held until the process exits.  Problems with
 *   B*S*M*D > 4 * 2^20 are rejected with MSDA_ERR_UNSUPPORTED before anything
 *   is enqueued.  Nothing is allocated: no cudaMalloc, no cudaFree, no
 *   allocating library routine.
 *   The first call on a device looks up the buffer's device address (a CUDA
 *   runtime query, once per device, with that device current); make that
 *   first call before any stream capture.  The address is kept until the
 *   process exits: after cudaDeviceReset() of the device it is stale (see
 *   "Per-device state" above).
 *   Every call on a device shares the one buffer and clears it before use:
 *   calls that overlap on the GPU (different streams, no ordering between
 *   them) race on it and give wrong results.  Serialize them.
 */
MSDA_API msda_status msda_backward_noalloc(const msda_problem *problem, const void *value,
                                           const int64_t *spatial_shapes,
                                           const int64_t *level_start_index,
                                           const float *sampling_locations,
                                           const float *attention_weights,
                                           const void *grad_output, void *grad_value,
                                           float *grad_sampling_locations,
                                           float *grad_attention_weights, msda_stream_t stream);

/*
 * INT8 value storage for MSDA_S8 (x-humanoid.csdn.net MSDA explainer §4,
 * "quantization and low-precision inference"; the page gives no scheme, this
 * is the plain symmetric one): for each (batch b, head m)
 *   amax  = max over keys s and channels d of |value[b, s, m, d]|
 *   scale = amax / 127 (float32 division), 1 when amax = 0
 *   q     = value / scale (float32 division) rounded half to even, clipped to
 *           [-127, 127]
 *   value        [B, S, M, D]  problem->value_dtype (MSDA_F32 or MSDA_BF16),
 *                              finite, 16-byte aligned
 *   value_s8     [B, S, M, D]  int8, written, 32-byte aligned
 *   value_scale  [B, M]        float32, written (also used as scratch)
 * D must be a multiple of 8 (every supported D is).  Four operations on
 * `stream`: a fill, an absmax reduction, the scales, the quantisation.
 * Non-finite inputs give unspecified q and scales.
 */
MSDA_API msda_status msda_quantize_value_s8(const msda_problem *problem, const void *value,
                                            void *value_s8, float *value_scale,
                                            msda_stream_t stream);

/*
 * FP8 value storage for MSDA_E4M3 (the same note): for each (batch b, head m)
 *   amax  = max over keys s and channels d of |value[b, s, m, d]|
 *   scale = amax / 448 (float32 division), 1 when amax = 0
 *   code  = the E4M3 value nearest to value / scale (float32 division), ties
 *           to the even mantissa, magnitudes above 448 clipped to 448, the
 *           sign kept when the quotient rounds to zero
 *   value        [B, S, M, D]  problem->value_dtype (MSDA_F32 or MSDA_BF16),
 *                              finite, 16-byte aligned
 *   value_e4m3   [B, S, M, D]  one byte per element, written, 32-byte aligned
 *   value_scale  [B, M]        float32, written (also used as scratch)
 * D must be a multiple of 8.  Four operations on `stream`, as
 * msda_quantize_value_s8.  Non-finite inputs give unspecified codes and
 * scales.
 */
MSDA_API msda_status msda_quantize_value_e4m3(const msda_problem *problem, const void *value,
                                              void *value_e4m3, float *value_scale,
                                              msda_stream_t stream);

/*
 * Processing order that keeps spatially close queries together (the optional
 * query-sorting step of the operator's data-locality notes,
 * x-humanoid.csdn.net MSDA explainer §4 "pre-processing and reordering"):
 * writes into query_order [B*Q] (int32, 4-byte aligned) a permutation of the
 * B*Q queries sorted by batch, then by the Morton code of the 64 x 64 cell of
 * [0,1]^2 that holds the query's point (coordinates outside [0,1] are
 * clamped, NaN counts as 0; the order within a cell is unspecified).
 * points [B, Q, 2] float32 (x, y), 16-byte aligned, typically the reference
 * points.  One kernel, one CTA per batch, no workspace.  Only batch, num_queries
 * and the validity of the rest of `problem` are used.  Asynchronous on `stream`.
 */
MSDA_API msda_status msda_sort_queries(const msda_problem *problem, const float *points,
                                       int32_t *query_order, msda_stream_t stream);

/* Bytes of workspace msda_backward / msda_fused_backward need for `problem`
 * (0 unless MSDA_GRAD_VALUE_BF16 is set).  Host only; enqueues nothing. */
MSDA_API msda_status msda_backward_workspace_size(const msda_problem *problem, size_t *bytes);

/*
 * DCNv3 core (discosf.com/news/5175395 §4.2, the operator of InternImage):
 *
 *   y[n,i,j,g,:] = sum_k mask[n,i,j,g,k] * x_g( p0(i,j) + p_k + offset[n,i,j,g,k] )
 *
 * the same gather-reduce on one map, with a convolution's sampling grid.
 * Point k = r*kernel_w + c of output pixel (i, j) sits at pixel coordinate
 *   px = j*stride_w - pad_w + c*dilation_w + dx,
 *   py = i*stride_h - pad_h + r*dilation_h + dy
 * (pixel centres at integers; bilinear; corners outside the H x W map read
 * zero; a sample is taken only when -1 < px < W and -1 < py < H).  The group
 * projection w_g of the formula is a linear layer outside the core.  The page
 * gives only the formula: the grid convention, (dx, dy) order and taking the
 * mask as given (no normalisation inside the core) are this library's
 * reading.  Output size: Ho = (H + 2*pad_h - dilation_h*(kernel_h-1) - 1) /
 * stride_h + 1, likewise Wo.
 *   input        [N, H, W, G, C]          value_dtype (channels last, group-major)
 *   offset       [N, Ho, Wo, G, K, 2]     float32 (dx, dy) pixels, K = kh*kw
 *   mask         [N, Ho, Wo, G, K]        float32
 *   output       [N, Ho, Wo, G, C]        value_dtype (bf16 for MSDA_S8)
 * Supported: C (group_channels) in {8, 16, 32, 64, 128, 256}; kernel_w <= 32,
 * kernel_h <= 16, kernel_h*kernel_w <= 128; H, W <= 65535; stride and
 * dilation >= 1; pad >= 0; N*Ho*Wo < 2^31.  Flags and dtypes as for the
 * attention calls (MSDA_S8 needs value_scale [N, G]).
 */
typedef struct msda_dcn_problem {
    int64_t batch;          /* N */
    int32_t height, width;  /* H, W of the input map */
    int32_t groups;         /* G */
    int32_t group_channels; /* C */
    int32_t kernel_h, kernel_w;
    int32_t stride_h, stride_w;
    int32_t pad_h, pad_w;
    int32_t dilation_h, dilation_w;
    int32_t value_dtype;    /* msda_dtype of input (and output, grad_output) */
    uint32_t flags;         /* MSDA_GRAD_VALUE_BF16, MSDA_ACCUMULATE_GRADS */
    const float *value_scale; /* MSDA_S8 only: [N, G] float32 */
} msda_dcn_problem;

/* Ho and Wo of `problem` (host only). */
MSDA_API msda_status msda_dcn_output_size(const msda_dcn_problem *problem, int64_t *out_h,
                                          int64_t *out_w);

MSDA_API msda_status msda_dcn_forward(const msda_dcn_problem *problem, const void *input,
                                      const float *offset, const float *mask, void *output,
                                      msda_stream_t stream);

/*
 * Gradients of the DCNv3 core: grad_input (zeroed first unless
 * MSDA_ACCUMULATE_GRADS; float32, or bf16 through a float32 workspace of
 * msda_dcn_backward_workspace_size() bytes with MSDA_GRAD_VALUE_BF16),
 * grad_offset [N,Ho,Wo,G,K,2] = mask * <g, dsample/dp> (pixels) and grad_mask
 * [N,Ho,Wo,G,K] = <g, sample>, both overwritten.
 */
MSDA_API msda_status msda_dcn_backward(const msda_dcn_problem *problem, const void *input,
                                       const float *offset, const float *mask,
                                       const void *grad_output, void *grad_input,
                                       float *grad_offset, float *grad_mask, void *workspace,
                                       size_t workspace_bytes, msda_stream_t stream);

MSDA_API msda_status msda_dcn_backward_workspace_size(const msda_dcn_problem *problem,
                                                      size_t *bytes);

/* ------------------------------------------------------------------------
 * Dense layers around the operator, on the tensor cores (tcgen05, sm_100a).
 *
 * The module the pages build around the core (discosf.com/news/5175395
 * §2.2 and §3.1; cf-1.com/news/4799680 §3.1-3.2) has four linear layers: the
 * value projection W'_m (value_proj), the sampling-offset and attention-
 * weight heads that read the query, and the output projection W_m
 * (output_proj).  These entry points run them with bf16 operands and
 * float32 accumulation; the layer weights use nn.Linear's layout
 * [out_features, in_features] (row-major, in_features contiguous).
 * ------------------------------------------------------------------------ */

/*
 * out[r, n] = sum_k x[r, k] * weight[n, k] + bias[n], r < rows, n < out_features.
 *   x       [rows, in_features] bf16, device, 16-byte aligned
 *   weight  [out_features, in_features] bf16, device, 16-byte aligned
 *   bias    [out_features] float32 or NULL
 *   out     [rows, out_features] in out_dtype (MSDA_F32 or MSDA_BF16),
 *           16-byte aligned.  With MSDA_BF16 output and out_features = M*D,
 *           value_proj writes the operator's value tensor [B, S, M, D]
 *           directly (rows = B*S).
 *   in_features and out_features >= 8 and multiples of 8 (16-byte rows for
 *   the tensor-memory copies); rows < 2^31; out_features < 2^20.
 * Errors: MSDA_ERR_INVALID_ARG (null / misaligned pointer, bad size or
 * dtype), MSDA_ERR_CUDA (launch or tensor-map set-up failed).  A kernel that
 * gives up a bounded wait records MSDA_ERR_DEVICE_TIMEOUT in the status word.
 */
MSDA_API msda_status msda_linear(int64_t rows, int32_t in_features, int32_t out_features,
                                 const void *x, const void *weight, const float *bias,
                                 void *out, int32_t out_dtype, msda_stream_t stream);

/*
 * The query-side head: one linear layer from the query to the 3*M*L*K
 * outputs the module's two heads predict (cf-1.com/news/4799680 §3.2:
 * 2*M*L*K sampling offsets, M*L*K attention logits), fused with the steps
 * that turn them into the core's inputs: sampling locations
 * loc = ref + off / (W_l, H_l) and attention weights A = softmax over the
 * L*K logits of each (b, q, m).  The offsets and logits are never written.
 *   problem      sizes (B, Q, M, L, K; S, D and value_dtype unused)
 *   query        [B, Q, in_features] bf16
 *   weight       [3*M*L*K, in_features] bf16: rows 0 .. 2P-1 are the offset
 *                head in the core's [M, L, K, 2] order, rows 2P .. 3P-1 the
 *                logit head in [M, L*K] order (P = M*L*K)
 *   bias         [3*M*L*K] float32 or NULL
 *   reference_points [B, Q, 2] float32 (normalized)
 *   spatial_shapes   [L, 2] int64 (H, W), device
 *   sampling_locations [B, Q, M, L, K, 2] float32, attention_weights
 *                [B, Q, M, L, K] float32: outputs, the core's layouts
 *   Needs L*K a power of two of at most 32 and M*L*K a multiple of 32;
 *   in_features as for msda_linear.
 */
MSDA_API msda_status msda_query_head(const msda_problem *problem, int32_t in_features,
                                     const void *query, const void *weight, const float *bias,
                                     const float *reference_points, const int64_t *spatial_shapes,
                                     float *sampling_locations, float *attention_weights,
                                     msda_stream_t stream);

/*
 * Backward of msda_query_head's location and softmax step: from the core's
 * grad_sampling_locations [B, Q, M, L, K, 2] and grad_attention_weights
 * [B, Q, M, L, K] (and the attention weights the forward produced) it
 * writes grad_head [B, Q, 3*M*L*K] float32, the gradient of the head's
 * linear outputs in the weight's row order: grad_loc / (W_l, H_l) for the
 * offsets, A_j (gA_j - sum_i A_i gA_i) over each run of L*K for the logits.
 * grad_reference_points [B, Q, 2] (sum of grad_loc over the query's
 * samples) is written when not NULL.  Same size limits as msda_query_head.
 */
MSDA_API msda_status msda_query_head_backward(const msda_problem *problem,
                                              const float *attention_weights,
                                              const float *grad_sampling_locations,
                                              const float *grad_attention_weights,
                                              const int64_t *spatial_shapes, float *grad_head,
                                              float *grad_reference_points, msda_stream_t stream);

/*
 * Synchronizes `stream`, then returns in *code the status the kernels recorded
 * on the current device since the last call (MSDA_OK, MSDA_ERR_DEVICE_CHECK,
 * MSDA_ERR_DEVICE_TIMEOUT, or MSDA_ERR_DEVICE_BOUNDS in the checked build), and
 * clears it.  The word belongs to the loaded library (the checked build has its
 * own).  Returns MSDA_ERR_CUDA if the synchronization or the read fails.
 */
MSDA_API msda_status msda_get_device_status(msda_stream_t stream, int32_t *code);

/* Static English description of a status code. */
MSDA_API const char *msda_status_string(msda_status status);

/* Library version, e.g. "0.1.0". */
MSDA_API const char *msda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSDA_H_ */
