// msda_kernels.cuh -- sm_100a kernels of the multi-scale deformable attention
// core: forward, backward and their fused variants (location step + softmax
// over the L*K points inside the kernel), plus zero-fill and float32 -> bf16
// conversion helpers.
//
// Work decomposition.  A "row" is one (b, q, m) triple; rows are numbered
// r = (b * Q + q) * M + m.  A group of G lanes owns one row; each lane owns
// one vector of VB bytes (4 to 32, by value type and direction) of the
// head_dim axis, so a corner of a sample is one fully used G*VB-byte row
// segment of `value` (128 bytes for D = 32 float32).  A warp carries 32 / G
// rows, a CTA up to 8 warps (fewer when the per-row shared-memory records
// would not fit); rows too few to fill the GPU are split over several lane
// groups in the forward (SPLIT).
//
// Per tile of rows there are two phases:
//   1. set-up: the group's lanes turn the row's L*K samples into records in
//      shared memory (pixel coordinate, floor, corner in-map bits, corner
//      offsets, attention weight; in the fused kernels also the location step
//      and the softmax over the row's logits);
//   2. gather: every lane of the group reads each record (a shared-memory
//      broadcast) and issues the four corner loads for its vector; the forward
//      accumulates A * w_c * v_c in float32 registers, the backward forms the
//      four partial dot products <g, v_c>, reduces the three gradient terms over
//      the group with a reduce-scatter of shuffles (each lane ends up owning
//      one sample's results), and scatters A * w_c * g into the float32
//      grad_value with 16-byte vector reductions (red.global.add.v4.f32), laid
//      out so that a row's lanes reduce whole 128-byte lines (one L2 request
//      per line: the backward's lanes carry 4 float32 gradient channels).
//
// Floor decisions.  The pixel coordinate x = loc_x * W - 0.5 and its floor are
// taken in float64 so that the corner choice is exactly that of the defining
// formula evaluated in double precision: non-fused fma(loc, W, -0.5) rounds
// as the formula does (loc * W is exact); fused fma(ref, W, off) - 0.5
// differs from the formula's chain (loc = ref + off / W, then loc * W - 0.5)
// by far less than the distance to an integer unless x lies within 1e-9 of
// one or the magnitudes are large, and there the chain itself is evaluated.
// The fractional parts are then rounded to float32 and everything else runs
// in float32.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <type_traits>

namespace msda {

// Tuning knobs (compile-time).  The forward gathers float32 rows with 16-byte
// lane vectors, one sample in flight per lane and 4 CTAs per SM, and bf16
// rows with 16-byte vectors and four samples in flight; the backward sizes
// its lanes by value type (float32 16 B, bf16 8 B, one-byte types 4 B) so
// that a row's float32 gradient is one whole 128-byte line per reduction
// request (D = 32), with 3 CTAs per SM.
// Bulk-copy staging of the set-up inputs measured slower everywhere with
// these layouts; it stays available per call (MSDA_STAGE_INPUTS, general
// kernels) and by these switches.
#ifndef MSDA_FWD_VB_F32
#define MSDA_FWD_VB_F32 16
#endif
#ifndef MSDA_FWD_INFLIGHT_F32
#define MSDA_FWD_INFLIGHT_F32 1
#endif
#ifndef MSDA_FWD_MIN_CTAS_F32
#define MSDA_FWD_MIN_CTAS_F32 4
#endif
#ifndef MSDA_FWD_VB_BF16
#define MSDA_FWD_VB_BF16 16
#endif
#ifndef MSDA_FWD_INFLIGHT_BF16
#define MSDA_FWD_INFLIGHT_BF16 4
#endif
#ifndef MSDA_FWD_MIN_CTAS_BF16
#define MSDA_FWD_MIN_CTAS_BF16 2
#endif
#ifndef MSDA_FWD_INFLIGHT_BF16_SHORT  // bf16 rows of at most 16 samples
#define MSDA_FWD_INFLIGHT_BF16_SHORT 1
#endif
#ifndef MSDA_FWD_MIN_CTAS_BF16_SHORT
#define MSDA_FWD_MIN_CTAS_BF16_SHORT 3
#endif
#ifndef MSDA_ZERO_CTAS_PER_SM         // zero-fill grid: 256-thread CTAs per SM (2 measured
#define MSDA_ZERO_CTAS_PER_SM 8        // slower beside the decoder's forward: 57 against 48 us)
#endif
#ifndef MSDA_FWD_SPLIT               // lane groups per row of the split forward (small problems)
#define MSDA_FWD_SPLIT 4
#endif
#ifndef MSDA_FWD_STAGE_F32           // TMA-staged set-up inputs (see "input staging")
#define MSDA_FWD_STAGE_F32 0
#endif
#ifndef MSDA_FWD_STAGE_BF16
#define MSDA_FWD_STAGE_BF16 0
#endif
#ifndef MSDA_FWD_VB_S8               // one-byte (INT8, FP8) value: bytes per lane vector
#define MSDA_FWD_VB_S8 8
#endif
#ifndef MSDA_FWD_INFLIGHT_S8          // INT8: one sample in flight, 3 CTAs per SM (measured
#define MSDA_FWD_INFLIGHT_S8 1         // against 4 and 2: 1024^2 forward 377 -> 338 us, 1080p
#endif                                 // K = 8 713 -> 694 us)
#ifndef MSDA_FWD_MIN_CTAS_S8
#define MSDA_FWD_MIN_CTAS_S8 3
#endif
#ifndef MSDA_BWD_VB
#define MSDA_BWD_VB 16
#endif
#ifndef MSDA_BWD_MIN_CTAS_F32       // backward CTAs per SM (register budget) by value type
#define MSDA_BWD_MIN_CTAS_F32 3
#endif
#ifndef MSDA_BWD_MIN_CTAS_BF16
#define MSDA_BWD_MIN_CTAS_BF16 3
#endif
#ifndef MSDA_BWD_MIN_CTAS            // one-byte (INT8, FP8) value
#define MSDA_BWD_MIN_CTAS 3
#endif
#ifndef MSDA_MERGE_FLUSH_CHAINS      // merged backward: slot lists a lane group walks together
#define MSDA_MERGE_FLUSH_CHAINS 1
#endif
#ifndef MSDA_STREAM_HINTS            // 1: L2 evict-first on streaming arrays
#define MSDA_STREAM_HINTS 1
#endif

constexpr int kMaxLevels = 16;
constexpr int kMaxWarpsPerCta = 8;

#ifndef MSDA_BOUNDS_CHECK            // 1: checked build (every corner row tested)
#define MSDA_BOUNDS_CHECK 0
#endif

struct KernelArgs {
    const void *value;
    const int64_t *shapes;
    const int64_t *starts;
    const float *loc;       // non-fused inputs
    const float *attn;
    const float *ref;       // fused inputs
    const float *off;
    const float *logits;
    const void *grad_out;
    void *out;
    float *attn_out;        // fused forward, may be null
    float *grad_value;      // float32 accumulator
    float *grad_loc;        // non-fused backward
    float *grad_attn;
    float *grad_ref;        // fused backward, may be null
    float *grad_off;
    float *grad_logits;
    int64_t rows;           // B * Q * M
    int64_t rows_per_tile;  // warps per CTA * rows per warp
    int64_t ntiles;         // ceil(rows / rows_per_tile)
    int64_t S;
    int Q, M, L, K;
    int withhold_copy;      // testing: arm the input copies but never issue them
    int stage;              // forward: stage set-up inputs by bulk copies (general kernels)
    const int32_t *order;   // optional processing order of the B*Q queries
    const float *scale;     // one-byte value: dequantization scale per (batch, head)
    // DCNv3 core (non-fused kernels): levels are the kh kernel rows, points
    // the kw kernel columns, all on the one H x W map; the pixel coordinate
    // of sample (l, k) of output pixel q = (i, j) is the convolution grid
    // point plus the offset, and the offset gradient is not rescaled
    int dcn;
    int dcn_h, dcn_w, dcn_wo;
    int stride_h, stride_w, pad_h, pad_w, dil_h, dil_w;
    // backward grad_value merge (see "merged reductions"): queries per tile,
    // query blocks per batch, hash-table slots (a power of two) and log2
    int64_t merge_qb, merge_nqb;
    int merge_tslots, merge_tbits;
    int *status;            // per-device status word (device address)
};

// Records a device-side failure code in the status word (msda_status values).
__device__ __forceinline__ void report(const KernelArgs &a, int code) { atomicExch(a.status, code); }

// Checked build (MSDA_BOUNDS_CHECK): the corner row offset `off` (key * M,
// relative to the row's (batch, head) slice) that a kernel is about to read
// or reduce into must lie in [0, S*M); a violation is recorded
// (MSDA_ERR_DEVICE_BOUNDS = 6) and the access skipped.  By construction the
// set-up only produces in-range offsets, so a clean run of the checked build
// is evidence that every access stays inside value / grad_value.
__device__ __forceinline__ bool row_in_bounds(const KernelArgs &a, int off)
{
#if MSDA_BOUNDS_CHECK
    if (off < 0 || (int64_t)off >= a.S * a.M) {
        report(a, 6 /* MSDA_ERR_DEVICE_BOUNDS */);
        return false;
    }
#else
    (void)a;
    (void)off;
#endif
    return true;
}

struct Geometry {
    int H[kMaxLevels];
    int W[kMaxLevels];
    int start[kMaxLevels];
};

// Loads spatial_shapes / level_start_index into shared memory and checks
// them: H, W in [1, 65535], start[0] = 0, start[l+1] = start[l] + H_l W_l,
// sum = S.  Returns false (for the whole CTA) on a mismatch, after recording
// it in the device status word.
__device__ __forceinline__ bool load_geometry(const KernelArgs &a, Geometry &geo, int &ok)
{
    if (a.dcn) {  // every kernel row samples the one input map (host-checked sizes)
        if (threadIdx.x < a.L) {
            geo.H[threadIdx.x] = a.dcn_h;
            geo.W[threadIdx.x] = a.dcn_w;
            geo.start[threadIdx.x] = 0;
        }
        __syncthreads();
        return true;
    }
    if (threadIdx.x == 0) {
        int good = 1;
        int64_t run = 0;
        for (int l = 0; l < a.L; ++l) {
            int64_t h = a.shapes[2 * l], w = a.shapes[2 * l + 1], s = a.starts[l];
            if (h < 1 || w < 1 || h > 65535 || w > 65535 || s != run)
                good = 0;
            run += h * w;
            if (good) {
                geo.H[l] = (int)h;
                geo.W[l] = (int)w;
                geo.start[l] = (int)s;
            }
        }
        if (run != a.S)
            good = 0;
        ok = good;
        if (!good)
            report(a, 4 /* MSDA_ERR_DEVICE_CHECK */);
    }
    __syncthreads();
    return ok != 0;
}

// ---------------------------------------------------------------- vectors --

struct alignas(32) U8 {
    uint32_t w[8];
};

template <int VB> struct RawOf;
template <> struct RawOf<4> { using type = uint32_t; };
template <> struct RawOf<8> { using type = uint2; };
template <> struct RawOf<16> { using type = uint4; };
template <> struct RawOf<32> { using type = U8; };

// Read-only vector load of `value` (L1-cached).
__device__ __forceinline__ uint32_t ld_vec(const uint32_t *p) { return __ldg(p); }
__device__ __forceinline__ uint2 ld_vec(const uint2 *p) { return __ldg(p); }
__device__ __forceinline__ uint4 ld_vec(const uint4 *p) { return __ldg(p); }
__device__ __forceinline__ U8 ld_vec(const U8 *p)
{
    U8 r;
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]),
                   "=r"(r.w[6]), "=r"(r.w[7])
                 : "l"(p));
    return r;
}
__device__ __forceinline__ void st_vec(uint2 *p, const uint2 &v) { *p = v; }
__device__ __forceinline__ void st_vec(uint4 *p, const uint4 &v) { *p = v; }
__device__ __forceinline__ void st_vec(U8 *p, const U8 &v)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
                    "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
}

// Element type traits: widening of stored words to float32 and back.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kBytes = 4;
    static constexpr bool kScaled = false;  // stored codes times a (batch, head) scale
    template <int NW> __device__ __forceinline__ static void widen(const uint32_t *u, float *f)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i)
            f[i] = __uint_as_float(u[i]);
    }
    template <int NW> __device__ __forceinline__ static void narrow(const float *f, uint32_t *u)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i)
            u[i] = __float_as_uint(f[i]);
    }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr bool kScaled = false;
    // bf16 -> f32 is exact: the bf16 bits are the top half of the float.
    template <int NW> __device__ __forceinline__ static void widen(const uint32_t *u, float *f)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            f[2 * i] = __uint_as_float(u[i] << 16);
            f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
    }
    template <int NW> __device__ __forceinline__ static void narrow(const float *f, uint32_t *u)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            u[i] = *reinterpret_cast<uint32_t *>(&h);
        }
    }
};

// INT8 value storage: a signed byte per channel, dequantized by the
// (batch, head) scale of KernelArgs::scale.  Never written by the kernels.
struct S8 {
    int8_t bits;
};
template <> struct Elem<S8> {
    static constexpr int kBytes = 1;
    static constexpr bool kScaled = true;
    // Exact: byte b (offset to b + 128 by the xor) is placed in the low
    // mantissa bits of the float 2^23, which is then subtracted with the
    // offset.
    template <int NW> __device__ __forceinline__ static void widen(const uint32_t *u, float *f)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            const uint32_t x = u[i] ^ 0x80808080u;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                f[4 * i + k] = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u + k)) - 8388736.0f;
        }
    }
};

// FP8 value storage: an OCP E4M3 code per channel (sign, 4 exponent bits with
// bias 7, 3 mantissa bits), dequantized by the (batch, head) scale of
// KernelArgs::scale.  Never written by the operator kernels.
struct E4M3 {
    uint8_t bits;
};
template <> struct Elem<E4M3> {
    static constexpr int kBytes = 1;
    static constexpr bool kScaled = true;
    // Exact: every E4M3 value is a half, and every half a float.  Byte k of a
    // word is element k (the low byte of each 16-bit pair is the pair's .x).
    template <int NW> __device__ __forceinline__ static void widen(const uint32_t *u, float *f)
    {
#pragma unroll
        for (int i = 0; i < NW; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
                    (__nv_fp8x2_storage_t)((u[i] >> (16 * h)) & 0xffffu), __NV_E4M3);
                const float2 v = __half22float2(__half2(r));
                f[4 * i + 2 * h] = v.x;
                f[4 * i + 2 * h + 1] = v.y;
            }
        }
    }
};

// Element type of output and grad_output rows: the value type, except bf16
// rows for one-byte (INT8, FP8) value.
template <typename T> struct RowOf { using type = T; };
template <> struct RowOf<S8> { using type = __nv_bfloat16; };
template <> struct RowOf<E4M3> { using type = __nv_bfloat16; };

// Lane layout of one row of D channels with VB-byte lane vectors.
template <typename T, int D, int VB> struct Layout {
    static constexpr int kVB = (D * Elem<T>::kBytes < VB) ? D * Elem<T>::kBytes : VB;
    using Raw = typename RawOf<kVB>::type;
    static constexpr int kWords = kVB / 4;                   // 32-bit words per vector
    static constexpr int kEpv = kVB / Elem<T>::kBytes;       // channels per vector
    static constexpr int kNvec = D / kEpv;                   // vectors per row
    static constexpr int kG = kNvec < 32 ? kNvec : 32;       // lanes per row
    static constexpr int kCh = kNvec / kG;                   // vectors per lane
    static constexpr int kRowsPerWarp = 32 / kG;
    static constexpr int kLaneElems = kCh * kEpv;            // channels per lane
    static_assert(kVB == 4 || kVB == 8 || kVB == 16 || kVB == 32, "vector size");
    static_assert(kNvec >= 1 && kNvec % kG == 0, "unsupported head_dim");
    __device__ __forceinline__ static void widen(const Raw &r, float *f)
    {
        Elem<T>::template widen<kWords>(reinterpret_cast<const uint32_t *>(&r), f);
    }
    __device__ __forceinline__ static Raw narrow(const float *f)
    {
        Raw r;
        Elem<T>::template narrow<kWords>(f, reinterpret_cast<uint32_t *>(&r));
        return r;
    }
};

// Lane vector width and resident CTAs per SM of the backward for each value
// type.
// bf16 backward: 8-byte lanes, so that a lane's float32 gradient channels
// are one 16-byte vector and the G lanes of a row reduce whole 128-byte
// lines (16-byte lanes split each D = 32 row into two 64-byte reductions;
// measured on the fused backward alone, µs: 1024^2 1194 -> 1055, 1080p K=8
// 2048 -> 1899, decoder 70.8 -> 67.6; with 3 CTAs per SM, which the smaller
// register need then allows: 985, 1692, 59.5)
#ifndef MSDA_BWD_VB_BF16
#define MSDA_BWD_VB_BF16 8
#endif
template <typename T> struct BwdVB { static constexpr int kVB = MSDA_BWD_VB; };
template <> struct BwdVB<__nv_bfloat16> { static constexpr int kVB = MSDA_BWD_VB_BF16; };
// One-byte (INT8, FP8) value backward: 4-byte lanes for the same reason as
// bf16's 8-byte ones (whole-line reductions), at 3 CTAs per SM (fused
// backward alone, µs: 1024^2 INT8 1196 -> 996, 1080p K=8 FP8 2024 -> 1713).
#ifndef MSDA_BWD_VB_1B
#define MSDA_BWD_VB_1B 4
#endif
template <> struct BwdVB<S8> { static constexpr int kVB = MSDA_BWD_VB_1B; };
template <> struct BwdVB<E4M3> { static constexpr int kVB = MSDA_BWD_VB_1B; };
template <typename T> struct BwdMinCtas { static constexpr int kN = MSDA_BWD_MIN_CTAS; };
template <> struct BwdMinCtas<float> { static constexpr int kN = MSDA_BWD_MIN_CTAS_F32; };
template <> struct BwdMinCtas<__nv_bfloat16> { static constexpr int kN = MSDA_BWD_MIN_CTAS_BF16; };

template <int G>
__device__ __forceinline__ float group_sum(float v)
{
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int G>
__device__ __forceinline__ float group_max(float v)
{
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Packed float32 pair arithmetic (one instruction for two lanes of work).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(*reinterpret_cast<unsigned long long *>(&d))
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<unsigned long long *>(&d))
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)));
    return d;
}

// ------------------------------------------------------------ cache hints --
//
// Arrays touched once per call (locations, offsets, logits, weights,
// reference points, grad_output and the per-sample gradients) are read and
// written with an L2 evict-first policy, so that they do not push value and
// the grad_value accumulator out of L2.

__device__ __forceinline__ uint64_t stream_policy()
{
    uint64_t p = 0;
#if MSDA_STREAM_HINTS
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
#endif
    return p;
}

__device__ __forceinline__ float ld_stream(const float *ptr, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    float v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.f32 %0, [%1], %2;"
                 : "=f"(v) : "l"(ptr), "l"(pol));
    return v;
#else
    (void)pol;
    return __ldg(ptr);
#endif
}

__device__ __forceinline__ float2 ld_stream2(const float2 *ptr, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    float2 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;"
                 : "=f"(v.x), "=f"(v.y) : "l"(ptr), "l"(pol));
    return v;
#else
    (void)pol;
    return __ldg(ptr);
#endif
}

__device__ __forceinline__ uint2 ld_stream_u2(const uint2 *ptr, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
                 : "=r"(v.x), "=r"(v.y) : "l"(ptr), "l"(pol));
    return v;
#else
    (void)pol;
    return __ldg(ptr);
#endif
}

__device__ __forceinline__ uint4 ld_stream_u4(const uint4 *ptr, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(ptr), "l"(pol));
    return v;
#else
    (void)pol;
    return __ldg(ptr);
#endif
}

__device__ __forceinline__ void st_stream(float *ptr, float v, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" :: "l"(ptr), "f"(v), "l"(pol) : "memory");
#else
    (void)pol;
    *ptr = v;
#endif
}

__device__ __forceinline__ void st_stream2(float2 *ptr, float2 v, uint64_t pol)
{
#if MSDA_STREAM_HINTS
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;"
                 :: "l"(ptr), "f"(v.x), "f"(v.y), "l"(pol) : "memory");
#else
    (void)pol;
    *ptr = v;
#endif
}

// grad_value reduction of one 16-byte chunk: a vector reduction that returns
// nothing (no wait for the L2 round trip).
__device__ __forceinline__ void red_add_v4(float4 *p, float4 v)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

// 4 consecutive grad_output channels starting at element `e` of a row,
// widened to float32.
template <typename T>
__device__ __forceinline__ float4 ld_grad4(const T *row, int e, uint64_t pol);
template <>
__device__ __forceinline__ float4 ld_grad4<float>(const float *row, int e, uint64_t pol)
{
    const uint4 u = ld_stream_u4(reinterpret_cast<const uint4 *>(row + e), pol);
    return make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
}
template <>
__device__ __forceinline__ float4 ld_grad4<__nv_bfloat16>(const __nv_bfloat16 *row, int e, uint64_t pol)
{
    const uint2 u = ld_stream_u2(reinterpret_cast<const uint2 *>(row + e), pol);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

// ------------------------------------------------------------- scheduling --
//
// Persistent grid: one resident wave of CTAs walks the row tiles grid-stride
// (tile c, c + gridDim.x, ...).
//
// Processing row p maps to memory row (b * Q + q) * M + m = p in the natural
// order; with a query order the p-th query is order[p / M].

__device__ __forceinline__ int64_t memory_row(const KernelArgs &a, int64_t p)
{
    if (a.order) {
        // processing row p is head p % M of the (p / M)-th query of the order;
        // an entry outside 0 .. B*Q-1 is reported and replaced by query 0
        const int64_t qi = p / a.M;
        int64_t q = __ldg(a.order + qi);
        if (q < 0 || q * a.M >= a.rows) {
            report(a, 4 /* MSDA_ERR_DEVICE_CHECK */);
            q = 0;
        }
        return q * a.M + (p - qi * a.M);
    }
    return p;
}

// ----------------------------------------------------------------- set-up --
//
// Each sample of a row becomes a 32-byte record in shared memory, stored as
// two 16-byte arrays (structure of arrays) with an odd row stride so that the
// lane groups of a warp read distinct banks:
//   forward   wa  = {A*w00, A*w01, A*w10, A*w11}  (0 for corners outside the map)
//             off = {o00, o01, o10, o11}          corner rows (key * M) relative to
//                                                 the row's (b, m) base; o00 = -1:
//                                                 sample skipped
//   backward  fa  = {fx (-1: sample skipped), fy, A, level | in-map bits << 8}
//             off = {o00, o01, o10, o11}
// Corner c = (y0 + c/2, x0 + c%2).  A corner outside the map is redirected to
// an in-map corner of the same sample (its column / row clamped into the map),
// so every issued load is in bounds; its weight is exactly zero (forward) or
// its dot product and reduction are dropped (backward).

__host__ __device__ __forceinline__ int record_stride(int P) { return (P & 1) ? P + 2 : P + 1; }

// Non-fused: x = loc_x * W - 0.5 in float64.  The product of a float32 and
// an integer below 2^16 is exact in float64, so one fused multiply-add rounds
// exactly as the double-precision formula (product, then subtraction) does.
__device__ __forceinline__ void pixel_from_location(float lx, float ly, int H, int W,
                                                    double &x, double &y)
{
    x = __fma_rn((double)lx, (double)W, -0.5);
    y = __fma_rn((double)ly, (double)H, -0.5);
}

// Fused: the formula reads loc = ref + off / W, then x = loc * W - 0.5, each
// step rounded in float64 (the oracle's chain).  Algebraically x = ref * W +
// off - 0.5, which the kernel forms with one float64 fused multiply-add and
// one subtraction, without the division.  For |off| + |ref| * W < 2^20 the two
// values differ by less than 2^-30 (each chain rounds a few times at 2^-53
// relative to that magnitude), so they have the same floor and the same
// order against -1 and W (integers) unless the value lies within 1e-9 of an
// integer; there, and for larger magnitudes, the formula's own chain is
// evaluated, so that the corner choice is always that of the float64 formula.
__device__ __forceinline__ double fused_coord(float r, float o, int W)
{
    const double Wd = (double)W;
    const double x = __dsub_rn(__fma_rn((double)r, Wd, (double)o), 0.5);
    const double f = x - floor(x);
    if (f > 1e-9 && f < 1.0 - 1e-9 && fabsf(o) + fabsf(r) * (float)W < 1048576.f)
        return x;
    return __dsub_rn(__dmul_rn(__dadd_rn((double)r, __ddiv_rn((double)o, Wd)), Wd), 0.5);
}

__device__ __forceinline__ void pixel_from_offset(float rx, float ry, float ox, float oy,
                                                  int H, int W, double &x, double &y)
{
    x = fused_coord(rx, ox, W);
    y = fused_coord(ry, oy, H);
}

// DCNv3: sample s = r * kw + c of memory row `row` (= (b * Q + q) * G + g,
// q = i * Wo + j) sits at the convolution grid point plus its offset,
//   x = (j * stride_w - pad_w + c * dil_w) + dx,  y = (i * stride_h - pad_h + r * dil_h) + dy,
// the integer part exact and one float64 addition.
__device__ __forceinline__ void pixel_from_dcn(const KernelArgs &a, int64_t row, int s, float dx, float dy,
                                               double &x, double &y)
{
    const int64_t q = (row / a.M) % a.Q;
    const int64_t i = q / a.dcn_wo, j = q - i * a.dcn_wo;
    const int r = s / a.K, c = s - r * a.K;
    x = __dadd_rn((double)(j * a.stride_w - a.pad_w + (int64_t)c * a.dil_w), (double)dx);
    y = __dadd_rn((double)(i * a.stride_h - a.pad_h + (int64_t)r * a.dil_h), (double)dy);
}

// Corner geometry of one sample at pixel coordinate (x, y) of a level.
struct Corners {
    bool valid;          // -1 < x < W and -1 < y < H
    float fx, fy;
    int key[4];          // flattened keys, redirected into the map
    bool in[4];          // corner lies inside the map
};

__device__ __forceinline__ Corners corners_of(double x, double y, int H, int W, int start)
{
    Corners c;
    c.valid = (x > -1.0) && (x < (double)W) && (y > -1.0) && (y < (double)H);
    if (!c.valid) {
        c.fx = c.fy = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            c.key[i] = start;
            c.in[i] = false;
        }
        return c;
    }
    const double x0d = floor(x), y0d = floor(y);
    const int x0 = (int)x0d, y0 = (int)y0d;  // x0 in [-1, W-1], y0 in [-1, H-1]
    c.fx = (float)(x - x0d);
    c.fy = (float)(y - y0d);
    const bool left = x0 >= 0, right = x0 + 1 < W, top = y0 >= 0, bottom = y0 + 1 < H;
    const int xl = left ? x0 : x0 + 1, xr = right ? x0 + 1 : x0;
    const int yt = top ? y0 : y0 + 1, yb = bottom ? y0 + 1 : y0;
    c.key[0] = start + yt * W + xl;
    c.key[1] = start + yt * W + xr;
    c.key[2] = start + yb * W + xl;
    c.key[3] = start + yb * W + xr;
    c.in[0] = top && left;
    c.in[1] = top && right;
    c.in[2] = bottom && left;
    c.in[3] = bottom && right;
    return c;
}

// Row prologue of the fused kernels: softmax statistics of the row's L*K
// logits (max-subtracted, float32) and the row's reference point.  Every lane
// of the warp takes part in the shuffles; inactive groups use dummy values.
template <int G>
__device__ __forceinline__ void fused_row_stats(const KernelArgs &a, int64_t row, bool active, int gl,
                                                float &mx, float &inv_sum, float &rx, float &ry)
{
    const int P = a.L * a.K;
    const int64_t base = row * P;
    mx = -INFINITY;
    if (active)
        for (int s = gl; s < P; s += G)
            mx = fmaxf(mx, __ldg(a.logits + base + s));
    mx = group_max<G>(mx);
    float sum = 0.f;
    if (active)
        for (int s = gl; s < P; s += G)
            sum += expf(__ldg(a.logits + base + s) - mx);
    sum = group_sum<G>(sum);
    inv_sum = 1.0f / sum;
    rx = ry = 0.f;
    if (active) {
        const int64_t bq = row / a.M;
        const float2 r = __ldg(reinterpret_cast<const float2 *>(a.ref) + bq);
        rx = r.x;
        ry = r.y;
    }
}

// Pixel coordinate and attention weight of sample s of a row.
template <bool FUSED>
__device__ __forceinline__ void sample_input(const KernelArgs &a, int64_t base, int s, int H, int W,
                                             float mx, float inv_sum, float rx, float ry,
                                             uint64_t pol, double &x, double &y, float &A)
{
    if (FUSED) {
        const float2 o = ld_stream2(reinterpret_cast<const float2 *>(a.off) + base + s, pol);
        pixel_from_offset(rx, ry, o.x, o.y, H, W, x, y);
        // last read of the logits: the softmax statistics pass read them first
        A = expf(ld_stream(a.logits + base + s, pol) - mx) * inv_sum;
    } else {
        const float2 p = ld_stream2(reinterpret_cast<const float2 *>(a.loc) + base + s, pol);
        if (a.dcn)
            pixel_from_dcn(a, base / (a.L * a.K), s, p.x, p.y, x, y);
        else
            pixel_from_location(p.x, p.y, H, W, x, y);
        A = ld_stream(a.attn + base + s, pol);
    }
}

// Builds the forward records of one row; lane gl of the group does samples
// gl, gl + G, ...
// One forward record: the four corner weights A * w_c (0 outside the map)
// and the corner rows.
__device__ __forceinline__ void write_forward_record(const KernelArgs &a, const Geometry &geo, int l,
                                                     double x, double y, float A, float4 *wa, int4 *off)
{
    const Corners c = corners_of(x, y, geo.H[l], geo.W[l], geo.start[l]);
    const float ay1 = A * c.fy, ay0 = A - ay1;
    float4 w;
    w.x = c.in[0] ? ay0 * (1.f - c.fx) : 0.f;
    w.y = c.in[1] ? ay0 * c.fx : 0.f;
    w.z = c.in[2] ? ay1 * (1.f - c.fx) : 0.f;
    w.w = c.in[3] ? ay1 * c.fx : 0.f;
    *wa = w;
    *off = c.valid ? make_int4(c.key[0] * a.M, c.key[1] * a.M, c.key[2] * a.M, c.key[3] * a.M)
                   : make_int4(-1, 0, 0, 0);
}

// Samples of a row a lane of the fused forward keeps in registers between
// the softmax statistics and the records (rows of up to kFwdCache * G
// samples read each logit once and take one expf per sample).
constexpr int kFwdCache = 4;

template <int G, bool FUSED>
__device__ __forceinline__ void setup_forward_row(const KernelArgs &a, const Geometry &geo,
                                                  int64_t row, bool active, int gl, uint64_t pol,
                                                  float4 *wa, int4 *off)
{
    const int P = a.L * a.K;
    const int64_t base = row * P;
    if constexpr (FUSED) {
        if (P <= kFwdCache * G) {
            float z[kFwdCache];
            float2 o[kFwdCache];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < kFwdCache; ++i) {
                const int s = gl + i * G;
                const bool on = active && s < P;
                z[i] = on ? ld_stream(a.logits + base + s, pol) : -INFINITY;
                o[i] = on ? ld_stream2(reinterpret_cast<const float2 *>(a.off) + base + s, pol)
                          : make_float2(0.f, 0.f);
                mx = fmaxf(mx, z[i]);
            }
            mx = group_max<G>(mx);
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < kFwdCache; ++i) {
                z[i] = (active && gl + i * G < P) ? expf(z[i] - mx) : 0.f;
                sum += z[i];
            }
            sum = group_sum<G>(sum);
            if (!active)
                return;
            const float inv_sum = 1.0f / sum;
            const float2 r = __ldg(reinterpret_cast<const float2 *>(a.ref) + row / a.M);
#pragma unroll
            for (int i = 0; i < kFwdCache; ++i) {
                const int s = gl + i * G;
                if (s >= P)
                    break;
                const int l = s / a.K;
                double x, y;
                pixel_from_offset(r.x, r.y, o[i].x, o[i].y, geo.H[l], geo.W[l], x, y);
                const float A = z[i] * inv_sum;
                if (a.attn_out)
                    st_stream(a.attn_out + base + s, A, pol);
                write_forward_record(a, geo, l, x, y, A, wa + s, off + s);
            }
            return;
        }
    }
    float mx = 0.f, inv_sum = 0.f, rx = 0.f, ry = 0.f;
    if (FUSED)
        fused_row_stats<G>(a, row, active, gl, mx, inv_sum, rx, ry);
    if (!active)
        return;
    for (int s = gl; s < P; s += G) {
        const int l = s / a.K;
        const int H = geo.H[l], W = geo.W[l];
        double x, y;
        float A;
        sample_input<FUSED>(a, base, s, H, W, mx, inv_sum, rx, ry, pol, x, y, A);
        if (FUSED && a.attn_out)
            st_stream(a.attn_out + base + s, A, pol);
        write_forward_record(a, geo, l, x, y, A, wa + s, off + s);
    }
}

// Builds the backward records of one row, padded to Pp >= P samples with
// inert records (no load, no reduction); lane gl of the group does samples
// gl, gl + G, ...  For an inactive row every record is inert.  Record of
// sample s: fa = {fx, fy, A, in-map bits of the four corners | tag}, off =
// corner rows (key * M) with off.x = -1 when the sample is skipped; `tag`
// (bits 8 and up) is the row's slot in the CTA tile, which the merged
// reductions use to find the row's grad_output.
template <int G, bool FUSED>
__device__ __forceinline__ void setup_backward_row(const KernelArgs &a, const Geometry &geo,
                                                   int64_t row, bool active, int gl, uint64_t pol,
                                                   int Pp, float4 *fa, int4 *off, float *As,
                                                   unsigned tag)
{
    const int P = a.L * a.K;
    const int64_t base = row * P;
    float mx = 0.f, inv_sum = 0.f, rx = 0.f, ry = 0.f;
    if (FUSED)
        fused_row_stats<G>(a, row, active, gl, mx, inv_sum, rx, ry);
    for (int s = gl; s < Pp; s += G) {
        if (!active || s >= P) {
            fa[s] = make_float4(0.f, 0.f, 0.f, 0.f);
            off[s] = make_int4(-1, 0, 0, 0);
            continue;
        }
        const int l = s / a.K;
        const int H = geo.H[l], W = geo.W[l];
        double x, y;
        float A;
        sample_input<FUSED>(a, base, s, H, W, mx, inv_sum, rx, ry, pol, x, y, A);
        const Corners c = corners_of(x, y, H, W, geo.start[l]);
        const unsigned bits = (c.in[0] ? 1u : 0u) | (c.in[1] ? 2u : 0u) | (c.in[2] ? 4u : 0u) |
                              (c.in[3] ? 8u : 0u);
        fa[s] = make_float4(c.fx, c.fy, A, __uint_as_float(bits | tag));
        off[s] = c.valid ? make_int4(c.key[0] * a.M, c.key[1] * a.M, c.key[2] * a.M, c.key[3] * a.M)
                         : make_int4(-1, 0, 0, 0);
        if (FUSED)
            As[s] = A;
    }
}

// ----------------------------------------------------------- input staging --
//
// For L*K = P a power of two <= 32, each warp copies the set-up inputs of its
// rows for the *next* tile (locations or offsets, and weights or logits) into
// a shared-memory double buffer with the TMA bulk-copy engine
// (cp.async.bulk, completion on an mbarrier) while it gathers the current
// tile, so set-up loads leave the L1 load path and their latency is hidden.
// A copy needs 16-byte aligned source and size: a warp slice qualifies when
// (first row * P) and (rows * P) are multiples of 4; other slices (ragged
// tails) and other P read global memory directly.  Waits are bounded: after
// kStageSpinLimit polls the kernel records MSDA_ERR_DEVICE_TIMEOUT (5), stops
// staging and reads the rest of its inputs directly; before the CTA exits it
// waits (bounded again) for every copy it issued and has not seen complete,
// so that no copy is left writing the shared memory of a finished CTA.

constexpr int kStageSpinLimit = 1 << 22;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *b)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, unsigned parity)
{
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                 " selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait; false after kStageSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, unsigned parity)
{
    for (int i = 0; i < kStageSpinLimit; ++i) {
        if (mbar_test(b, parity))
            return true;
        __nanosleep(32);
    }
    return false;
}
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, unsigned bytes, uint64_t *bar,
                                              uint64_t pol)
{
#if MSDA_STREAM_HINTS
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                 " [%0], [%1], %2, [%3], %4;"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol) : "memory");
#else
    (void)pol;
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
#endif
}

// A warp's double buffer: per stage RPW * P location pairs and RPW * P
// weights; two mbarriers.
struct WarpStage {
    float2 *p;      // [2][rpw * P]
    float *z;       // [2][rpw * P]
    uint64_t *bar;  // [2]
    int cap;        // rpw * P
};

// Stage capacity (elements per stage) of a warp of rpw rows, 0 when the
// inputs are never staged; bytes of a warp's stages and barriers.
__host__ __device__ __forceinline__ int stage_cap(bool enabled, int rpw, int P)
{
    return (enabled && P <= 32 && (P & (P - 1)) == 0) ? ((rpw * P + 3) & ~3) : 0;
}
__host__ __device__ __forceinline__ size_t stage_bytes_per_warp(bool enabled, int rpw, int P)
{
    const int c = stage_cap(enabled, rpw, P);
    return c ? (size_t)c * 2 * 12 + 16 : 0;
}
__host__ __device__ __forceinline__ size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Carves a warp's stages out of the shared memory after the records.
__device__ __forceinline__ WarpStage warp_stage(unsigned char *base, int warp, int nwarps, int cap)
{
    WarpStage ws;
    ws.cap = cap;
    float2 *p_all = reinterpret_cast<float2 *>(base);
    float *z_all = reinterpret_cast<float *>(p_all + (size_t)nwarps * 2 * cap);
    uint64_t *b_all = reinterpret_cast<uint64_t *>(z_all + (size_t)nwarps * 2 * cap);
    ws.p = p_all + (size_t)warp * 2 * cap;
    ws.z = z_all + (size_t)warp * 2 * cap;
    ws.bar = b_all + warp * 2;
    return ws;
}

// Tiles of this CTA: a grid-stride walk (c, c + G, c + 2G, ...), so that the
// resident wave sweeps one narrow band of queries at a time and the corner
// rows it gathers and reduces into stay in L2.  The host launches at most
// ntiles CTAs.
struct TileWalk {
    int64_t first, end, step;
};

__device__ __forceinline__ TileWalk tile_walk(const KernelArgs &a)
{
    return TileWalk{(int64_t)blockIdx.x, a.ntiles, (int64_t)gridDim.x};
}

__device__ __forceinline__ bool stage_ok(int64_t prow0, int nv, int P)
{
    return nv > 0 && P <= 32 && (P & (P - 1)) == 0 && ((prow0 * P) & 3) == 0 && ((nv * P) & 3) == 0;
}

// Lane 0 starts the copies of the inputs of rows prow0 .. prow0 + nv - 1 into
// stage st (the caller checked stage_ok).
template <bool FUSED>
__device__ __forceinline__ void stage_issue(const KernelArgs &a, const WarpStage &ws, int st, int64_t prow0,
                                            int nv, int lane, uint64_t pol)
{
    if (lane != 0)
        return;
    const int P = a.L * a.K;
    const unsigned np = (unsigned)(nv * P);
    const float2 *src_p = reinterpret_cast<const float2 *>(FUSED ? a.off : a.loc) + prow0 * P;
    const float *src_z = (FUSED ? a.logits : a.attn) + prow0 * P;
    mbar_expect_tx(ws.bar + st, np * 12u);
    if (a.withhold_copy)
        return;  // the wait for this stage runs out (failure-path test)
    bulk_copy_g2s(ws.p + st * ws.cap, src_p, np * 8u, ws.bar + st, pol);
    bulk_copy_g2s(ws.z + st * ws.cap, src_z, np * 4u, ws.bar + st, pol);
}

// Warp-wide set-up of the backward for L*K = P a power of two <= 32: lane L
// of round t takes sample (32 t + L) % P of the warp's row (32 t + L) / P, so
// every input array is read with one contiguous load per round (the loads of
// up to kWarpSetupRounds rounds are issued together), and the softmax of a row
// is a reduction over its P lanes (one expf per sample).  (The forward keeps the
// per-group set-up: its register budget is spent on gathers in flight, and the
// warp-wide form measured slower there.)

__host__ __device__ __forceinline__ bool warp_setup_ok(int P) { return P <= 32 && (P & (P - 1)) == 0; }

template <bool FUSED>
__device__ __forceinline__ float seg_max(float v, int P)
{
    for (int o = P / 2; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float seg_sum(float v, int P)
{
    for (int o = P / 2; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Raw inputs of one sample of the warp-wide set-up, loaded ahead of the math
// so that the loads of all rounds are in flight together.
struct WarpIn {
    float2 p;    // location (non-fused) or offset (fused)
    float z;     // attention weight (non-fused) or logit (fused)
    float2 r;    // reference point (fused)
};

template <bool FUSED>
__device__ __forceinline__ WarpIn warp_load(const KernelArgs &a, int64_t row, bool active, int s,
                                            int P, uint64_t pol)
{
    WarpIn in;
    in.p = make_float2(0.f, 0.f);
    in.r = make_float2(0.f, 0.f);
    in.z = FUSED ? -INFINITY : 0.f;
    if (active) {
        const int64_t idx = row * P + s;
        if (FUSED) {
            in.p = ld_stream2(reinterpret_cast<const float2 *>(a.off) + idx, pol);
            in.z = ld_stream(a.logits + idx, pol);
            in.r = __ldg(reinterpret_cast<const float2 *>(a.ref) + row / a.M);
        } else {
            in.p = ld_stream2(reinterpret_cast<const float2 *>(a.loc) + idx, pol);
            in.z = ld_stream(a.attn + idx, pol);
        }
    }
    return in;
}

// Same inputs from a shared-memory stage (element k of the warp's slice).
template <bool FUSED>
__device__ __forceinline__ WarpIn warp_load_staged(const KernelArgs &a, const float2 *sp, const float *sz,
                                                   int k, int64_t row, bool active)
{
    WarpIn in;
    in.p = make_float2(0.f, 0.f);
    in.r = make_float2(0.f, 0.f);
    in.z = FUSED ? -INFINITY : 0.f;
    if (active) {
        in.p = sp[k];
        in.z = sz[k];
        if (FUSED)
            in.r = __ldg(reinterpret_cast<const float2 *>(a.ref) + row / a.M);
    }
    return in;
}

// Pixel coordinate and weight from the loaded inputs.  Every lane of the warp
// must call (the softmax shuffles).
template <bool FUSED>
__device__ __forceinline__ void warp_sample(const KernelArgs &a, const Geometry &geo, const WarpIn &in,
                                            bool active, int64_t row, int s, int P, int &l, double &x,
                                            double &y, float &A)
{
    l = s / a.K;
    const int H = geo.H[l], W = geo.W[l];
    if (FUSED) {
        const float mx = seg_max<true>(in.z, P);
        const float e = active ? expf(in.z - mx) : 0.f;
        const float sum = seg_sum(e, P);
        A = active ? e / sum : 0.f;
        pixel_from_offset(in.r.x, in.r.y, in.p.x, in.p.y, H, W, x, y);
    } else {
        A = in.z;
        if (a.dcn)
            pixel_from_dcn(a, row, s, in.p.x, in.p.y, x, y);
        else
            pixel_from_location(in.p.x, in.p.y, H, W, x, y);
    }
}

#ifndef MSDA_WARP_SETUP_ROUNDS
#define MSDA_WARP_SETUP_ROUNDS 8
#endif
constexpr int kWarpSetupRounds = MSDA_WARP_SETUP_ROUNDS;  // rounds whose loads are issued together

// Backward records of the warp's rows (inactive rows and pad slots inert).
// row_of(rr) is the memory row of the warp's rr-th row, or -1 when that row
// is inactive; record k = rr * stride + s; tag0 + (rr << 8) tags the records
// of row rr with the row's slot in the CTA tile (see setup_backward_row).
// ROUNDS: rounds whose loads are issued together; nrows <= ROUNDS * 32 / P
// rows fit one batch of rounds when ROUNDS >= nrows.
template <bool FUSED, int ROUNDS, typename RowFn>
__device__ __forceinline__ void setup_backward_warp(const KernelArgs &a, const Geometry &geo, RowFn row_of,
                                                    int nrows, int lane, uint64_t pol, int Pp, float4 *fa0,
                                                    int4 *off0, float *As0, int stride, unsigned tag0)
{
    const int P = a.L * a.K;
    const int per_round = 32 / P;
    for (int rb = 0; rb < nrows; rb += per_round * ROUNDS) {
        WarpIn in[ROUNDS];
#pragma unroll
        for (int t = 0; t < ROUNDS; ++t) {
            const int rr = rb + t * per_round + lane / P;
            const int64_t row = rr < nrows ? row_of(rr) : -1;
            in[t] = warp_load<FUSED>(a, row >= 0 ? row : 0, row >= 0, lane % P, P, pol);
        }
#pragma unroll
        for (int t = 0; t < ROUNDS; ++t) {
            if (rb + t * per_round >= nrows)
                break;
            const int rr = rb + t * per_round + lane / P, s = lane % P;
            const int64_t row = rr < nrows ? row_of(rr) : -1;
            const bool active = row >= 0;
            int l;
            double x, y;
            float A;
            warp_sample<FUSED>(a, geo, in[t], active, active ? row : 0, s, P, l, x, y, A);
            if (rr >= nrows)
                continue;
            const int k = rr * stride + s;
            if (!active) {
                fa0[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                off0[k] = make_int4(-1, 0, 0, 0);
                continue;
            }
            const Corners c = corners_of(x, y, geo.H[l], geo.W[l], geo.start[l]);
            const unsigned bits = (c.in[0] ? 1u : 0u) | (c.in[1] ? 2u : 0u) | (c.in[2] ? 4u : 0u) |
                                  (c.in[3] ? 8u : 0u);
            fa0[k] = make_float4(c.fx, c.fy, A, __uint_as_float(bits | (tag0 + ((unsigned)rr << 8))));
            off0[k] = c.valid ? make_int4(c.key[0] * a.M, c.key[1] * a.M, c.key[2] * a.M, c.key[3] * a.M)
                              : make_int4(-1, 0, 0, 0);
            if (FUSED)
                As0[k] = A;
        }
    }
    // pad slots P .. Pp-1 (only when P is below the reduce-scatter chunk)
    for (int k = lane; k < nrows * (Pp - P); k += 32) {
        const int rr = k / (Pp - P), s = P + k % (Pp - P);
        fa0[rr * stride + s] = make_float4(0.f, 0.f, 0.f, 0.f);
        off0[rr * stride + s] = make_int4(-1, 0, 0, 0);
    }
}

// Forward records of the warp's rows from a shared-memory stage (staged
// tiles only; the per-group set-up serves the others).
template <bool FUSED>
__device__ __forceinline__ void setup_forward_staged(const KernelArgs &a, const Geometry &geo,
                                                     int64_t prow0, int nrows, int lane, uint64_t pol,
                                                     float4 *wa0, int4 *off0, int stride,
                                                     const float2 *sp, const float *sz)
{
    const int P = a.L * a.K;
    const int per_round = 32 / P;
    for (int r0 = 0; r0 < nrows; r0 += per_round) {
        const int rr = r0 + lane / P, s = lane % P;
        const int64_t prow = prow0 + rr;
        const bool active = rr < nrows && prow < a.rows;
        const int64_t row = active ? memory_row(a, prow) : 0;
        const WarpIn in = warp_load_staged<FUSED>(a, sp, sz, rr * P + s, row, active);
        int l;
        double x, y;
        float A;
        warp_sample<FUSED>(a, geo, in, active, row, s, P, l, x, y, A);
        if (!active)
            continue;
        if (FUSED && a.attn_out)
            st_stream(a.attn_out + row * P + s, A, pol);
        const Corners c = corners_of(x, y, geo.H[l], geo.W[l], geo.start[l]);
        const float ay1 = A * c.fy, ay0 = A - ay1;
        float4 w;
        w.x = c.in[0] ? ay0 * (1.f - c.fx) : 0.f;
        w.y = c.in[1] ? ay0 * c.fx : 0.f;
        w.z = c.in[2] ? ay1 * (1.f - c.fx) : 0.f;
        w.w = c.in[3] ? ay1 * c.fx : 0.f;
        wa0[rr * stride + s] = w;
        off0[rr * stride + s] = c.valid ? make_int4(c.key[0] * a.M, c.key[1] * a.M, c.key[2] * a.M,
                                                    c.key[3] * a.M)
                                        : make_int4(-1, 0, 0, 0);
    }
}

// ---------------------------------------------------------------- forward --

// Forward tuning per value type.  SHORT: rows of at most 16 samples (L*K <=
// 16), where bf16 runs faster with one sample in flight per lane and 3 CTAs
// per SM than with four samples in flight and 2 CTAs (measured: 1024^2
// encoder forward 342 -> 281 us, decoder 31 -> 27 us; the 32-sample rows of
// the K = 8 workload prefer the deeper pipeline).
template <typename T, bool SHORT> struct FwdTune;
template <bool SHORT> struct FwdTune<float, SHORT> {
    static constexpr int kVB = MSDA_FWD_VB_F32, kInFlight = MSDA_FWD_INFLIGHT_F32,
                         kMinCtas = MSDA_FWD_MIN_CTAS_F32;
    static constexpr bool kStage = MSDA_FWD_STAGE_F32 != 0;
};
template <> struct FwdTune<__nv_bfloat16, false> {
    static constexpr int kVB = MSDA_FWD_VB_BF16, kInFlight = MSDA_FWD_INFLIGHT_BF16,
                         kMinCtas = MSDA_FWD_MIN_CTAS_BF16;
    static constexpr bool kStage = MSDA_FWD_STAGE_BF16 != 0;
};
template <> struct FwdTune<__nv_bfloat16, true> {
    static constexpr int kVB = MSDA_FWD_VB_BF16, kInFlight = MSDA_FWD_INFLIGHT_BF16_SHORT,
                         kMinCtas = MSDA_FWD_MIN_CTAS_BF16_SHORT;
    static constexpr bool kStage = MSDA_FWD_STAGE_BF16 != 0;
};
template <bool SHORT> struct FwdTune<S8, SHORT> {
    static constexpr int kVB = MSDA_FWD_VB_S8, kInFlight = MSDA_FWD_INFLIGHT_S8,
                         kMinCtas = MSDA_FWD_MIN_CTAS_S8;
    static constexpr bool kStage = false;
};
template <bool SHORT> struct FwdTune<E4M3, SHORT> : FwdTune<S8, SHORT> {};

// GEN = false: the plain attention kernel (natural query order, no DCN grid),
// with those branches removed at compile time; GEN = true honours
// KernelArgs::order and KernelArgs::dcn.
//
// SPLIT > 1: SPLIT lane groups share a row, group ph
// gathering samples ph*U .. ph*U + U-1, then (ph + SPLIT)*U ..., and the
// partial sums meet in a shuffle reduction before group 0 stores the row.
// For problems with too few rows to fill the GPU (the decoder's 300 queries
// per image), this gives each row SPLIT times the loads in flight and the
// grid SPLIT times the warps.
template <typename T, int D, bool FUSED, bool GEN, bool SHORT = false, int SPLIT = 1>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32, FwdTune<T, SHORT>::kMinCtas)
forward_kernel(const KernelArgs a_in)
{
    KernelArgs a = a_in;
    if constexpr (!GEN) {
        a.order = nullptr;
        a.dcn = 0;
        a.stage = 0;
    }
    using Tune = FwdTune<T, SHORT>;
    using Lay = Layout<T, D, Tune::kVB>;
    using Raw = typename Lay::Raw;
    constexpr int G = Lay::kG, CH = Lay::kCh, E = Lay::kLaneElems, EPV = Lay::kEpv;
    constexpr int U = Tune::kInFlight;  // samples in flight per lane (4 corners each)
    static_assert(SPLIT == 1 || SPLIT * G <= 32, "row split: G * SPLIT <= 32");
    constexpr int GS = G * SPLIT;       // lanes of one row

    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ Geometry geo;
    __shared__ int geo_ok;
    if (!load_geometry(a, geo, geo_ok))
        return;

    const int P = a.L * a.K;
    const int stride = record_stride(P);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int RPW = 32 / GS;  // rows per warp
    const int grp = lane / GS, ph = (lane / G) % SPLIT, gl = lane % G;
    const int slot = warp * RPW + grp;
    float4 *wa = reinterpret_cast<float4 *>(smem_raw) + slot * stride;
    int4 *off = reinterpret_cast<int4 *>(smem_raw) + a.rows_per_tile * stride + slot * stride;
    const uint64_t pol = stream_policy();
    // staged slices are contiguous rows: not with a query order nor a split
    const int cap = (a.order || SPLIT > 1) ? 0 : stage_cap(Tune::kStage || a.stage, RPW, P);
    const WarpStage ws = warp_stage(smem_raw + align16((size_t)a.rows_per_tile * stride * 32), warp,
                                    blockDim.x >> 5, cap);
    if (cap) {
        if (lane == 0) {
            mbar_init(ws.bar);
            mbar_init(ws.bar + 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        __syncwarp();
    }
    unsigned phase = 0;    // bit st: parity of the next completion of stage st
    unsigned pending = 0;  // bit st: a copy into stage st was issued and not yet seen complete
    bool live = cap != 0;  // staging on; off after a wait ran out
    int k = 0;
    const TileWalk tw = tile_walk(a);
    int64_t tile = tw.first;
    if (live && tile < tw.end) {
        const int64_t p0 = tile * a.rows_per_tile + warp * RPW;
        const int nv = (int)max((int64_t)0, min((int64_t)RPW, a.rows - p0));
        if (stage_ok(p0, nv, P)) {
            stage_issue<FUSED>(a, ws, 0, p0, nv, lane, pol);
            if (!a.withhold_copy)
                pending |= 1u;
        }
    }
    for (; tile < tw.end; tile += tw.step, ++k) {
        const int st = k & 1;
        const int64_t nxt = tile + tw.step;
        if (live && nxt < tw.end) {
            const int64_t p0n = nxt * a.rows_per_tile + warp * RPW;
            const int nvn = (int)max((int64_t)0, min((int64_t)RPW, a.rows - p0n));
            if (stage_ok(p0n, nvn, P)) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                stage_issue<FUSED>(a, ws, st ^ 1, p0n, nvn, lane, pol);
                if (!a.withhold_copy)
                    pending |= 1u << (st ^ 1);
            }
        }
        const int64_t prow = tile * a.rows_per_tile + slot;
        const bool active = prow < a.rows;
        const int64_t row = active ? memory_row(a, prow) : prow;
        const int64_t p0 = tile * a.rows_per_tile + warp * RPW;
        const int nv = (int)max((int64_t)0, min((int64_t)RPW, a.rows - p0));
        bool staged = false;
        if (live && stage_ok(p0, nv, P)) {
            staged = __all_sync(0xffffffffu, mbar_wait(ws.bar + st, (phase >> st) & 1u));
            if (staged) {
                pending &= ~(1u << st);
                phase ^= 1u << st;
            } else {
                // the copy did not land in time: report it, stop staging and
                // read the inputs directly from here on (the copies still in
                // flight are waited for before the CTA exits)
                if (lane == 0)
                    report(a, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                live = false;
            }
        }
        if (staged)
            setup_forward_staged<FUSED>(a, geo, p0, RPW, lane, pol, wa - grp * stride, off - grp * stride,
                                        stride, ws.p + st * cap, ws.z + st * cap);
        else
            setup_forward_row<GS, FUSED>(a, geo, row, active, lane % GS, pol, wa, off);
        __syncwarp();
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e)
            acc[e] = 0.f;
        const int64_t bq = row / a.M;
        const int m = (int)(row - bq * a.M);
        const int64_t b = bq / a.Q;
        if (active) {
            // this lane's first vector of head m of batch b, key 0; corner rows
            // are D channels apart
            const Raw *vbase = reinterpret_cast<const Raw *>(static_cast<const T *>(a.value) +
                                                             (b * a.S * a.M + m) * D) + gl;
            for (int s0 = ph * U; s0 < P; s0 += U * SPLIT) {
                Raw v[U][4][CH];
                float4 w[U];
                bool ok[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int s = s0 + u;
                    const int4 o = s < P ? off[s] : make_int4(-1, 0, 0, 0);
                    w[u] = s < P ? wa[s] : make_float4(0.f, 0.f, 0.f, 0.f);
                    ok[u] = o.x >= 0;
                    const int oc[4] = {o.x, o.y, o.z, o.w};
                    if (ok[u]) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int j = 0; j < CH; ++j)
                                v[u][c][j] = row_in_bounds(a, oc[c])
                                                 ? ld_vec(vbase + (int64_t)oc[c] * Lay::kNvec + j * G)
                                                 : Raw{};
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!ok[u])
                        continue;
                    const float wc[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int j = 0; j < CH; ++j) {
                            float f[EPV];
                            Lay::widen(v[u][c][j], f);
#pragma unroll
                            for (int e = 0; e < EPV; ++e)
                                acc[j * EPV + e] = fmaf(wc[c], f[e], acc[j * EPV + e]);
                        }
                }
            }
        }
        if constexpr (SPLIT > 1) {
            // the row's partial sums: lanes gl of its SPLIT groups are G apart
#pragma unroll
            for (int i = G; i < GS; i <<= 1)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], i);
        }
        if (active && ph == 0) {
            if constexpr (Elem<T>::kScaled) {
                // dequantize once per row, store bf16 (EPV = 8 channels, 16 bytes)
                static_assert(EPV == 8, "one-byte lanes hold 8 channels");
                const float sc = __ldg(a.scale + b * a.M + m);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    acc[e] *= sc;
                uint4 *obase = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + row * D) + gl;
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    uint4 r;
                    Elem<__nv_bfloat16>::narrow<4>(acc + j * EPV, reinterpret_cast<uint32_t *>(&r));
                    obase[j * G] = r;
                }
            } else {
                Raw *obase = reinterpret_cast<Raw *>(static_cast<T *>(a.out) + row * D) + gl;
#pragma unroll
                for (int j = 0; j < CH; ++j)
                    st_vec(obase + j * G, Lay::narrow(acc + j * EPV));
            }
        }
        __syncwarp();
    }
    // no copy may still be writing this CTA's shared memory when it exits:
    // after a time-out, wait (bounded) for the copies issued and not yet seen
    for (int st = 0; st < 2; ++st)
        if (pending & (1u << st))
            mbar_wait(ws.bar + st, (phase >> st) & 1u);
}

// --------------------------------------------------------------- backward --

// Reduce-scatter of C samples x 3 partial sums over the G lanes of a group:
// afterwards v[0][0..2] of lane gl holds the group totals of chunk sample
// gl % C (halving exchange over the sample index for C lanes, then a plain
// butterfly over the remaining G / C lanes).  Every lane of the warp must call.
template <int G, int C>
__device__ __forceinline__ void reduce_scatter3(float (&v)[C][3], int gl)
{
#pragma unroll
    for (int o = C / 2; o >= 1; o >>= 1) {
        const bool hi = (gl & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i)
#pragma unroll
            for (int t = 0; t < 3; ++t) {
                const float lo_v = v[i][t], hi_v = v[i + o][t];
                const float send = hi ? lo_v : hi_v;
                const float keep = hi ? hi_v : lo_v;
                v[i][t] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
    }
#pragma unroll
    for (int o = C; o < G; o <<= 1)
#pragma unroll
        for (int t = 0; t < 3; ++t)
            v[0][t] += __shfl_xor_sync(0xffffffffu, v[0][t], o);
}

// Samples per backward reduce-scatter chunk for G lanes per row.
template <int G> struct BwdChunk { static constexpr int kC = G < 4 ? G : 4; };

// ------------------------------------------------------ merged reductions --
//
// grad_value receives A * w_c * g for every in-map corner of every sample.
// Neighbouring queries of one head sample largely the same corner rows (on
// the encoder workloads only about a third of the contributions of 32
// consecutive queries of one head go to distinct rows), so in the MERGE
// kernels a CTA tile is one head m of Qb consecutive queries of one batch
// and the CTA merges the tile's contributions before they reach L2:
//   1. each warp keeps its rows' grad_output in shared memory and enters the
//      in-map corners of its records into a shared-memory open-addressing
//      table keyed by corner row (multiplicative hash, linear probing, slots
//      claimed with atomicCAS); each contribution is linked into its row's
//      list with atomicExch on the list head, and a newly claimed slot is
//      appended to the tile's list of occupied slots;
//   2. after a CTA barrier, groups of FG lanes take the occupied slots, walk
//      each list summing A * w_c * g (the weights are recomputed from the
//      record, the row's grad_output read from shared memory) and reduce the
//      sum into grad_value with one vector reduction per lane (a row is a whole line);
//      each walked slot is reset for the next tile;
//   3. a second barrier closes the tile.
// The table has at least as many slots as the tile has contributions, so a
// free slot always exists; the probe loop is bounded all the same, and a
// contribution that finds no slot is reduced directly.  Contribution ids
// (record * 4 + corner) and slots are 16-bit; the host sizes tiles so that
// they fit.
//
// Measured on B200, the merge costs more than the L2 reductions it saves
// (fused backward, direct / merged: encoder float32 270 / 469 us, 1080p K = 8
// bf16 2045 / 6439 us, DCNv3 7 x 7 bf16 697 / 2711 us): a shared-memory
// atomic takes about one L1 wavefront per lane, and the list walks are
// latency-bound between the CTA barriers.  It is therefore an option
// (MSDA_MERGE_REDUCTIONS); the default reduces each contribution directly.

constexpr int kMergeEmpty = -1;         // free table slot
constexpr unsigned kMergeEnd = 0xFFFFu;  // end of a contribution list

// Byte offsets of the merge arrays after the records (host and device agree).
struct MergeLayout {
    size_t gsm, tkey, thead, occ, next, total;
};

__host__ __device__ __forceinline__ MergeLayout merge_layout(size_t record_bytes, int64_t rows, int stride,
                                                            int D, int tslots)
{
    MergeLayout m;
    size_t o = align16(record_bytes);
    m.gsm = o;      // float32 grad_output rows of the tile [rows][D]
    o += (size_t)rows * D * 4;
    m.tkey = o;     // int   [tslots]: corner row (key * M) or kMergeEmpty
    o += (size_t)tslots * 4;
    m.thead = o;    // int   [tslots]: first contribution id of the slot's list
    o += (size_t)tslots * 4;
    m.occ = o;      // u16   [tslots]: occupied slots in claim order
    o += align16((size_t)tslots * 2);
    m.next = o;     // u16   [rows * stride * 4]: next contribution id
    o += align16((size_t)rows * stride * 4 * 2);
    m.total = o;
    return m;
}

// Enters contribution `id` (record id >> 2, corner id & 3) of corner row
// `key` into the table; false when no slot was found.
__device__ __forceinline__ bool merge_insert(int *tkey, int *thead, uint16_t *occ, uint16_t *next, int *nocc,
                                             int tslots, int tbits, int key, int id)
{
    unsigned h = ((unsigned)key * 2654435761u) >> (32 - tbits);
    for (int probe = 0; probe < tslots; ++probe) {
        const int prev = atomicCAS(tkey + h, kMergeEmpty, key);
        if (prev == kMergeEmpty)
            occ[atomicAdd(nocc, 1)] = (uint16_t)h;
        if (prev == kMergeEmpty || prev == key) {
            next[id] = (uint16_t)atomicExch(thead + h, id);
            return true;
        }
        h = (h + 1) & (unsigned)(tslots - 1);
    }
    return false;
}

// --------------------------------------------------------------- backward --

// GEN = false: the plain attention kernel (natural query order, no DCN grid);
// GEN = true honours KernelArgs::order (without MERGE only) and ::dcn.
// MERGE = true: a CTA tile is one head of merge_qb consecutive queries of one
// batch and grad_value contributions are merged per tile (above); MERGE =
// false: a tile is rows_per_tile consecutive processing rows and every
// contribution is reduced into grad_value directly.
template <typename T, int D, bool FUSED, bool GEN, bool MERGE>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32, BwdMinCtas<T>::kN)
backward_kernel(const KernelArgs a_in)
{
    KernelArgs a = a_in;
    if constexpr (!GEN) {
        a.order = nullptr;
        a.dcn = 0;
    }
    if constexpr (MERGE)
        a.order = nullptr;  // merged tiles follow the natural order (host-checked)
    a.stage = 0;
    using Lay = Layout<T, D, BwdVB<T>::kVB>;
    using R = typename RowOf<T>::type;  // grad_output element
    using Raw = typename Lay::Raw;
    constexpr int G = Lay::kG, CH = Lay::kCh, E = Lay::kLaneElems, EPV = Lay::kEpv;
    constexpr int C = BwdChunk<G>::kC;
    // grad_value reductions: a float32 row is D / 4 chunks of 16 bytes;
    // reduction h of lane gl covers chunk h * G + gl, so each reduction
    // instruction of a group fills whole sectors
    constexpr int NR = D / 4 / G;
    static_assert(NR >= 1 && (D / 4) % G == 0, "reduction layout");
    static_assert(EPV % 2 == 0, "pairs");
    constexpr int RPW = Lay::kRowsPerWarp;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ Geometry geo;
    __shared__ int geo_ok;
    __shared__ int nocc[2];
    if (!load_geometry(a, geo, geo_ok))
        return;

    const int P = a.L * a.K;
    const int Pp = (P + C - 1) / C * C;
    const int stride = record_stride(Pp);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int grp = lane / G, gl = lane % G;
    const int slot = warp * RPW + grp;
    const int64_t arr = a.rows_per_tile * stride;  // one record array, in 16-byte units
    float4 *fa_all = reinterpret_cast<float4 *>(smem_raw);
    int4 *off_all = reinterpret_cast<int4 *>(fa_all + arr);
    float4 *fa = fa_all + slot * stride;
    int4 *off = off_all + slot * stride;
    // fused: grad_A and A of each sample, kept for the softmax Jacobian.
    // Layout in floats: fa, off: 4 * arr each; gA, As: arr each (10 * arr
    // floats = 40 bytes per record slot, as the host sizes it).
    float *gA = reinterpret_cast<float *>(fa_all + 2 * arr) + slot * stride;
    float *As = gA + arr;
    const uint64_t pol = stream_policy();

    // merge arrays (MERGE only)
#define MSDA_MERGE_ARRAYS                                                                             \
    const MergeLayout ml = merge_layout((size_t)arr * (FUSED ? 40 : 32), a.rows_per_tile, stride, D, \
                                        a.merge_tslots);                                             \
    float4 *gsm = reinterpret_cast<float4 *>(smem_raw + ml.gsm);                                     \
    int *tkey = reinterpret_cast<int *>(smem_raw + ml.tkey);                                         \
    int *thead = reinterpret_cast<int *>(smem_raw + ml.thead);                                       \
    uint16_t *occ = reinterpret_cast<uint16_t *>(smem_raw + ml.occ);                                 \
    uint16_t *cnext = reinterpret_cast<uint16_t *>(smem_raw + ml.next);                              \
    (void)gsm, (void)tkey, (void)thead, (void)occ, (void)cnext;
    if constexpr (MERGE) {
        MSDA_MERGE_ARRAYS
        for (int i = threadIdx.x; i < a.merge_tslots; i += blockDim.x) {
            tkey[i] = kMergeEmpty;
            thead[i] = (int)kMergeEnd;
        }
        if (threadIdx.x == 0)
            nocc[0] = nocc[1] = 0;
        __syncthreads();
    }

    int k = 0;
    for (int64_t tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x, ++k) {
        // rows of this warp: row_of(rr) for rr < RPW, -1 when inactive
        int64_t tb = 0, tm = 0, mrow0 = 0, prow0 = 0;
        int nact;
        if constexpr (MERGE) {
            tm = tile % a.M;
            const int64_t rest = tile / a.M;
            const int64_t qblk = rest % a.merge_nqb;
            tb = rest / a.merge_nqb;
            const int64_t q0 = qblk * a.merge_qb + warp * RPW;
            nact = (int)max((int64_t)0, min((int64_t)RPW, (int64_t)a.Q - q0));
            mrow0 = (tb * a.Q + q0) * a.M + tm;
        } else {
            prow0 = tile * a.rows_per_tile + warp * RPW;
            nact = (int)max((int64_t)0, min((int64_t)RPW, a.rows - prow0));
        }
        auto row_of = [&](int rr) -> int64_t {
            if (rr >= nact)
                return -1;
            return MERGE ? mrow0 + (int64_t)rr * a.M : memory_row(a, prow0 + rr);
        };
        const int64_t row0 = row_of(grp);
        const bool active = row0 >= 0;
        const int64_t row = active ? row0 : 0;
        const unsigned tag0 = (unsigned)(warp * RPW) << 8;
        if (warp_setup_ok(P))
            setup_backward_warp<FUSED, (RPW < kWarpSetupRounds ? RPW : kWarpSetupRounds)>(
                a, geo, row_of, RPW, lane, pol, Pp, fa - grp * stride,
                                       off - grp * stride, As - grp * stride, stride, tag0);
        else
            setup_backward_row<G, FUSED>(a, geo, row, active, gl, pol, Pp, fa, off, As,
                                         tag0 + ((unsigned)grp << 8));
        __syncwarp();
        const int64_t bq = row / a.M;
        const int m = (int)(row - bq * a.M);
        const int64_t b = bq / a.Q;
        const int64_t rbase = b * a.S * a.M + m;  // (b, key 0, m) row
        const Raw *vbase = reinterpret_cast<const Raw *>(static_cast<const T *>(a.value) + rbase * D) + gl;
        float4 *gvbase = reinterpret_cast<float4 *>(a.grad_value + rbase * D) + gl;
        // grad_output of the row: pairs in the load layout (dot products) and
        // float4s in the reduction layout (scatter)
        float2 g2[E / 2];
        float4 gr[NR];
        if (active) {
            const R *grow = static_cast<const R *>(a.grad_out) + row * D;
#pragma unroll
            for (int j = 0; j < CH; ++j)
#pragma unroll
                for (int q4 = 0; q4 < EPV / 4; ++q4) {
                    const float4 t4 = ld_grad4<R>(grow, (j * G + gl) * EPV + 4 * q4, pol);
                    g2[(j * EPV + 4 * q4) / 2] = make_float2(t4.x, t4.y);
                    g2[(j * EPV + 4 * q4) / 2 + 1] = make_float2(t4.z, t4.w);
                }
#pragma unroll
            for (int h = 0; h < NR; ++h)
                gr[h] = ld_grad4<R>(grow, (h * G + gl) * 4, pol);
        } else {
#pragma unroll
            for (int e = 0; e < E / 2; ++e)
                g2[e] = make_float2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < NR; ++h)
                gr[h] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if constexpr (MERGE) {
            MSDA_MERGE_ARRAYS
            // the tile's grad_output rows, then this warp's contributions
            float4 *gvt = reinterpret_cast<float4 *>(a.grad_value + (tb * a.S * a.M + tm) * D);
#pragma unroll
            for (int h = 0; h < NR; ++h)
                gsm[slot * (D / 4) + h * G + gl] = gr[h];
            __syncwarp();
            for (int e = lane; e < nact * Pp; e += 32) {
                const int rr = e / Pp, s = e - rr * Pp;
                const int rec = (warp * RPW + rr) * stride + s;
                const unsigned bits = __float_as_uint(fa_all[rec].w) & 15u;
                if (!bits)
                    continue;
                const int4 o = off_all[rec];
                const int oc[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!(bits & (1u << c)))
                        continue;
                    if (!merge_insert(tkey, thead, occ, cnext, &nocc[k & 1], a.merge_tslots, a.merge_tbits,
                                      oc[c], rec * 4 + c) &&
                        row_in_bounds(a, oc[c])) {
                        // no slot (never with the host's table size): reduce directly
                        const float4 r = fa_all[rec];
                        const float wxy = ((c & 1) ? r.x : 1.f - r.x) * ((c & 2) ? r.y : 1.f - r.y);
                        const float coef = r.z * wxy;
                        const float4 *gq = gsm + (warp * RPW + rr) * (D / 4);
                        for (int f = 0; f < D / 4; ++f) {
                            const float4 g4 = gq[f];
                            red_add_v4(gvt + (int64_t)oc[c] * (D / 4) + f,
                                      make_float4(coef * g4.x, coef * g4.y, coef * g4.z, coef * g4.w));
                        }
                    }
                }
            }
        }
        const int64_t base = row * P;
        float dot = 0.f, ref_gx = 0.f, ref_gy = 0.f;  // fused: per-owner partial sums
        float vsc = 1.f;  // one-byte value: the dot products are in code units
        if constexpr (Elem<T>::kScaled)
            vsc = active ? __ldg(a.scale + b * a.M + m) : 0.f;
        for (int c0 = 0; c0 < Pp; c0 += C) {
            float part[C][3];
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const int s = c0 + i;
                const int4 o = off[s];
                float d[4] = {0.f, 0.f, 0.f, 0.f};  // partial <g, v_c>
                if (o.x >= 0) {
                    const int oc[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float2 dp = make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < CH; ++j) {
                            float f[EPV];
                            Lay::widen(row_in_bounds(a, oc[c])
                                           ? ld_vec(vbase + (int64_t)oc[c] * Lay::kNvec + j * G)
                                           : Raw{},
                                       f);
#pragma unroll
                            for (int e = 0; e < EPV; e += 2)
                                dp = fma2(g2[(j * EPV + e) / 2], make_float2(f[e], f[e + 1]), dp);
                        }
                        d[c] = dp.x + dp.y;
                    }
                }
                const float4 r = fa[s];
                const unsigned inm = __float_as_uint(r.w);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    d[c] = (inm & (1u << c)) ? (Elem<T>::kScaled ? d[c] * vsc : d[c])
                                             : 0.f;  // corners outside the map read 0
                const float fx = r.x, fy = r.y, A = r.z, ex = 1.f - fx, ey = 1.f - fy;
                const float w[4] = {ex * ey, fx * ey, ex * fy, fx * fy};
                part[i][0] = w[0] * d[0] + w[1] * d[1] + w[2] * d[2] + w[3] * d[3];
                part[i][1] = A * (ey * (d[1] - d[0]) + fy * (d[3] - d[2]));
                part[i][2] = A * (ex * (d[2] - d[0]) + fx * (d[3] - d[1]));
                if constexpr (!MERGE) {
                    // scatter A * w_c * g into grad_value (in-map corners of
                    // taken samples; skipped samples have no in-map bits)
                    const int ocs[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (!(inm & (1u << c)))
                            continue;
                        const float awc = A * w[c];
                        if (!row_in_bounds(a, ocs[c]))
                            continue;
                        float4 *q = gvbase + (int64_t)ocs[c] * (D / 4);
                        const float2 ww = make_float2(awc, awc);
#pragma unroll
                        for (int h = 0; h < NR; ++h) {
                            const float2 lo = mul2(ww, make_float2(gr[h].x, gr[h].y));
                            const float2 hi = mul2(ww, make_float2(gr[h].z, gr[h].w));
                            red_add_v4(q + h * G, make_float4(lo.x, lo.y, hi.x, hi.y));
                        }
                    }
                }
            }
            reduce_scatter3<G, C>(part, gl);
            const int s = c0 + gl;
            if (active && gl < C && s < P) {
                const int l = s / a.K;
                const float W = (float)geo.W[l], H = (float)geo.H[l];
                if (FUSED) {
                    st_stream2(reinterpret_cast<float2 *>(a.grad_off) + base + s,
                               make_float2(part[0][1], part[0][2]), pol);
                    gA[s] = part[0][0];
                    ref_gx += W * part[0][1];
                    ref_gy += H * part[0][2];
                } else {
                    // DCN offsets are in pixels: no normalized-unit factor
                    const float sx = a.dcn ? 1.f : W, sy = a.dcn ? 1.f : H;
                    st_stream2(reinterpret_cast<float2 *>(a.grad_loc) + base + s,
                               make_float2(sx * part[0][1], sy * part[0][2]), pol);
                    st_stream(a.grad_attn + base + s, part[0][0], pol);
                }
            }
        }
        if (FUSED) {
            // softmax Jacobian: grad_z_j = A_j (gA_j - sum_i A_i gA_i)
            if (active && gl < C)
                for (int s = gl; s < P; s += C)
                    dot += As[s] * gA[s];
            dot = group_sum<G>(dot);
            ref_gx = group_sum<G>(ref_gx);
            ref_gy = group_sum<G>(ref_gy);
            if (active && gl < C) {
                for (int s = gl; s < P; s += C)
                    st_stream(a.grad_logits + base + s, As[s] * (gA[s] - dot), pol);
                if (a.grad_ref && gl == 0) {
                    atomicAdd(a.grad_ref + 2 * bq, ref_gx);
                    atomicAdd(a.grad_ref + 2 * bq + 1, ref_gy);
                }
            }
        }
        if constexpr (MERGE) {
            // every warp's contributions are in the table: reduce one sum per
            // occupied slot, FG lanes per grad_value row
            MSDA_MERGE_ARRAYS
            __syncthreads();
            const int n = nocc[k & 1];
            if (threadIdx.x == 0)
                nocc[(k + 1) & 1] = 0;  // last read in the previous tile, before its second barrier
            constexpr int FG = (D / 4) < 32 ? (D / 4) : 32, NRF = D / 4 / FG, GPW = 32 / FG;
            const int fg = lane / FG, fl = lane % FG;
            float4 *gvt = reinterpret_cast<float4 *>(a.grad_value + (tb * a.S * a.M + tm) * D) + fl;
            const int limit = (int)(arr * 4);
            // NCH slots per lane group at a time, their lists walked in step so
            // that the dependent shared-memory loads of different lists overlap
            constexpr int NCH = MSDA_MERGE_FLUSH_CHAINS;
            // (warp-uniform trip count: the __syncwarp below is reached by every lane)
            for (int jw = warp * GPW * NCH; jw < n; jw += nwarps * GPW * NCH) {
                const int j0 = jw + fg * NCH;
                int hs[NCH], id[NCH];
                float4 acc[NCH][NRF];
#pragma unroll
                for (int u = 0; u < NCH; ++u) {
                    hs[u] = j0 + u < n ? occ[j0 + u] : -1;
                    id[u] = hs[u] >= 0 ? thead[hs[u]] : (int)kMergeEnd;
#pragma unroll
                    for (int f = 0; f < NRF; ++f)
                        acc[u][f] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                for (int guard = 0; guard < limit; ++guard) {
                    bool more = false;
#pragma unroll
                    for (int u = 0; u < NCH; ++u) {
                        if (id[u] == (int)kMergeEnd)
                            continue;
                        more = true;
                        const float4 r = fa_all[id[u] >> 2];
                        const int c = id[u] & 3;
                        const float wxy = ((c & 1) ? r.x : 1.f - r.x) * ((c & 2) ? r.y : 1.f - r.y);
                        const float coef = r.z * wxy;
                        const float4 *gq = gsm + (__float_as_uint(r.w) >> 8) * (D / 4) + fl;
#pragma unroll
                        for (int f = 0; f < NRF; ++f) {
                            const float4 g4 = gq[f * FG];
                            acc[u][f].x = fmaf(coef, g4.x, acc[u][f].x);
                            acc[u][f].y = fmaf(coef, g4.y, acc[u][f].y);
                            acc[u][f].z = fmaf(coef, g4.z, acc[u][f].z);
                            acc[u][f].w = fmaf(coef, g4.w, acc[u][f].w);
                        }
                        id[u] = cnext[id[u]];
                    }
                    if (!more)
                        break;
                }
#pragma unroll
                for (int u = 0; u < NCH; ++u) {
                    if (hs[u] < 0)
                        continue;
                    const int key = tkey[hs[u]];
                    if (row_in_bounds(a, key)) {
#pragma unroll
                        for (int f = 0; f < NRF; ++f)
                            red_add_v4(gvt + (int64_t)key * (D / 4) + f * FG, acc[u][f]);
                    }
                }
                __syncwarp();  // every lane of the group has read tkey before the reset
#pragma unroll
                for (int u = 0; u < NCH; ++u)
                    if (hs[u] >= 0 && fl == 0) {
                        tkey[hs[u]] = kMergeEmpty;
                        thead[hs[u]] = (int)kMergeEnd;
                    }
            }
            __syncthreads();
        } else {
            __syncwarp();
        }
    }
#undef MSDA_MERGE_ARRAYS
}

// Rows per warp of each kernel (the host sizes CTAs and shared memory by it).
template <typename T, int D> constexpr int forward_rows_per_warp() { return Layout<T, D, FwdTune<T, false>::kVB>::kRowsPerWarp; }
template <typename T> constexpr bool forward_stages() { return FwdTune<T, false>::kStage; }
template <typename T, int D> constexpr int backward_rows_per_warp() { return Layout<T, D, BwdVB<T>::kVB>::kRowsPerWarp; }
// Record slots of a backward row: L*K rounded up to the reduce-scatter chunk.
template <typename T, int D> inline int backward_padded_samples(int P)
{
    constexpr int C = BwdChunk<Layout<T, D, BwdVB<T>::kVB>::kG>::kC;
    return (P + C - 1) / C * C;
}

}  // namespace msda
