// msda_aux.cuh -- sm_100a helper kernels of the library: grad_value zero-fill,
// float32 -> bf16 conversion, INT8 value quantisation and the query sort.
// Included by msda_api.cu only (the operator kernels live in
// msda_kernels.cuh and are instantiated in their own translation units).
#pragma once

#include "msda_kernels.cuh"

namespace msda {

// ----------------------------------------------------------------- helpers --

// Zeroes n4 float4 of `a` and n floats of `b` (grid-stride).
__global__ void zero_kernel(float4 *a, int64_t n4, float *b, int64_t n)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // four independent stores per step
    for (; i + 3 * stride < n4; i += 4 * stride) {
        a[i] = z;
        a[i + stride] = z;
        a[i + 2 * stride] = z;
        a[i + 3 * stride] = z;
    }
    for (; i < n4; i += stride)
        a[i] = z;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        b[i] = 0.f;
}

// float32 -> bf16 (round to nearest even), 8 elements per thread step.
__global__ void f32_to_bf16_kernel(const float4 *src, uint4 *dst, int64_t n8)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const float4 x = src[2 * i], y = src[2 * i + 1];
        const float f[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
        uint4 r;
        Elem<__nv_bfloat16>::narrow<4>(f, reinterpret_cast<uint32_t *>(&r));
        dst[i] = r;
    }
}

// ------------------------------------------------------ INT8 quantisation --
//
// value [B, S, M, D] (float32 or bf16) -> int8 with one symmetric scale per
// (batch, head): amax = max |value[b, :, m, :]|, scale = amax / 127 (1 when
// amax = 0), q = value / scale rounded half to even, clipped to +-127.  Three
// kernels: per-(b, m) absmax (into the scale array as float bits, zeroed by
// the host), scale = amax / 127 in place, quantise.

// Eight consecutive channels starting at p, widened to float32.
__device__ __forceinline__ void load8(const float *p, float (&f)[8])
{
    const float4 x = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 y = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&f)[8])
{
    const uint4 r = __ldg(reinterpret_cast<const uint4 *>(p));
    Elem<__nv_bfloat16>::widen<4>(reinterpret_cast<const uint32_t *>(&r), f);
}

// CTA blockIdx.x covers (b, m) = blockIdx.x / chunks and the chunk
// blockIdx.x % chunks of the S keys; one atomicMax per CTA.  |x| >= 0, so the
// float bit patterns order like the values.
template <typename T>
__global__ void __launch_bounds__(256) absmax_kernel(const T *v, int64_t S, int M, int D, int chunks,
                                                     unsigned *amax)
{
    __shared__ float part[8];
    const int64_t bm = blockIdx.x / chunks;
    const int64_t chunk = blockIdx.x % chunks;
    const int64_t b = bm / M, m = bm % M;
    const int nv = D / 8;
    const int64_t s0 = S * chunk / chunks, s1 = S * (chunk + 1) / chunks;
    float mx = 0.f;
    for (int64_t i = threadIdx.x; i < (s1 - s0) * nv; i += blockDim.x) {
        const int64_t s = s0 + i / nv;
        const int j = (int)(i % nv);
        float f[8];
        load8(v + ((b * S + s) * M + m) * D + j * 8, f);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            mx = fmaxf(mx, fabsf(f[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0)
        part[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            mx = fmaxf(mx, part[w]);
        atomicMax(amax + bm, __float_as_uint(mx));
    }
}

// scale = amax / qmax in place (1 when amax = 0): qmax 127 for INT8, 448 for
// FP8 E4M3.
__global__ void quant_scale_kernel(float *scale, int64_t n, float qmax)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const float amax = scale[i];
        scale[i] = amax > 0.f ? __fdiv_rn(amax, qmax) : 1.f;
    }
}

// Eight channels per thread step (D is a multiple of 8).
template <typename T>
__global__ void quantize_s8_kernel(const T *v, const float *scale, int64_t n8, int64_t S, int M, int D,
                                   uint2 *q)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const int64_t row = i * 8 / D;  // (b * S + s) * M + m
        const int64_t m = row % M, b = row / ((int64_t)S * M);
        const float sc = __ldg(scale + b * M + m);
        float f[8];
        load8(v + i * 8, f);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int r = __float2int_rn(__fdiv_rn(f[e], sc));  // half to even
            r = r > 127 ? 127 : (r < -127 ? -127 : r);
            w[e >> 2] |= ((uint32_t)r & 0xffu) << (8 * (e & 3));
        }
        q[i] = make_uint2(w[0], w[1]);
    }
}

// FP8 storage: the E4M3 code nearest to value / scale (the division in
// float32, round to nearest even, magnitudes above 448 clipped to 448, the
// sign kept on zero), eight channels per thread step.
template <typename T>
__global__ void quantize_e4m3_kernel(const T *v, const float *scale, int64_t n8, int64_t S, int M, int D,
                                     uint2 *q)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const int64_t row = i * 8 / D;  // (b * S + s) * M + m
        const int64_t m = row % M, b = row / ((int64_t)S * M);
        const float sc = __ldg(scale + b * M + m);
        float f[8];
        load8(v + i * 8, f);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
                make_float2(__fdiv_rn(f[e], sc), __fdiv_rn(f[e + 1], sc)), __NV_SATFINITE, __NV_E4M3);
            w[e >> 2] |= (uint32_t)c << (8 * (e & 3));
        }
        q[i] = make_uint2(w[0], w[1]);
    }
}

// ------------------------------------------------------------ query order --
//
// Counting sort of each batch's queries by the Morton code of the 64 x 64 cell
// of [0,1]^2 holding their point, in one kernel: one CTA of 1024 threads per
// batch counts the queries per cell in shared memory, scans the counts, then
// hands each query the next slot of its cell.  Each pass reads the batch's
// points with kSortInFlight loads in flight per thread.

constexpr int kSortCells = 64;  // cells per axis of [0,1]^2
constexpr int kSortThreads = 1024, kSortInFlight = 8;

__device__ __forceinline__ uint32_t spread_bits6(uint32_t v)  // 6 bits -> even bit positions
{
    v &= 63u;
    v = (v | (v << 4)) & 0x0f0fu;
    v = (v | (v << 2)) & 0x3333u;
    v = (v | (v << 1)) & 0x5555u;
    return v;
}

__device__ __forceinline__ uint32_t cell_code(float2 p)
{
    // fminf / fmaxf map NaN to the other operand, so every point gets a cell
    const float fx = fminf(fmaxf(p.x * kSortCells, 0.f), kSortCells - 1.f);
    const float fy = fminf(fmaxf(p.y * kSortCells, 0.f), kSortCells - 1.f);
    return spread_bits6((uint32_t)fx) | (spread_bits6((uint32_t)fy) << 1);
}

// Cell codes of the points i0 + j * kSortThreads + t (j < kSortInFlight);
// ~0u past the end.
__device__ __forceinline__ void cell_codes(const float2 *p, int64_t Q, int64_t i0, int t,
                                           uint32_t (&code)[kSortInFlight])
{
    float2 v[kSortInFlight];
#pragma unroll
    for (int j = 0; j < kSortInFlight; ++j) {
        const int64_t i = i0 + (int64_t)j * kSortThreads + t;
        v[j] = i < Q ? __ldg(p + i) : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kSortInFlight; ++j)
        code[j] = i0 + (int64_t)j * kSortThreads + t < Q ? cell_code(v[j]) : ~0u;
}

__global__ void __launch_bounds__(kSortThreads) sort_queries_kernel(const float2 *pts, int64_t Q,
                                                                    int32_t *order)
{
    constexpr int kCells = kSortCells * kSortCells;
    static_assert(kCells == 4 * kSortThreads, "the scan takes 4 counters per thread");
    __shared__ __align__(16) int cnt[kCells];
    __shared__ int warp_base[kSortThreads / 32];
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    const int64_t base = (int64_t)blockIdx.x * Q;  // first query of this batch
    const float2 *p = pts + base;
    reinterpret_cast<int4 *>(cnt)[t] = make_int4(0, 0, 0, 0);
    __syncthreads();
    for (int64_t i0 = 0; i0 < Q; i0 += (int64_t)kSortThreads * kSortInFlight) {
        uint32_t code[kSortInFlight];
        cell_codes(p, Q, i0, t, code);
#pragma unroll
        for (int j = 0; j < kSortInFlight; ++j)
            if (code[j] != ~0u)
                atomicAdd(cnt + code[j], 1);
    }
    __syncthreads();
    // exclusive scan of the counters: 4 per thread, warp shuffles, warp totals
    const int4 c = reinterpret_cast<const int4 *>(cnt)[t];
    const int own = c.x + c.y + c.z + c.w;
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        warp_base[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        const int tot = warp_base[lane];
        int x = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o)
                x += y;
        }
        warp_base[lane] = x - tot;
    }
    __syncthreads();
    int4 r;
    r.x = warp_base[wid] + incl - own;
    r.y = r.x + c.x;
    r.z = r.y + c.y;
    r.w = r.z + c.z;
    reinterpret_cast<int4 *>(cnt)[t] = r;
    __syncthreads();
    for (int64_t i0 = 0; i0 < Q; i0 += (int64_t)kSortThreads * kSortInFlight) {
        uint32_t code[kSortInFlight];
        cell_codes(p, Q, i0, t, code);
#pragma unroll
        for (int j = 0; j < kSortInFlight; ++j)
            if (code[j] != ~0u) {
                const int slot = atomicAdd(cnt + code[j], 1);
                order[base + slot] = (int32_t)(base + i0 + (int64_t)j * kSortThreads + t);
            }
    }
}

// ------------------------------------------------ query head: chain rule --
//
// Backward of the query head's location / softmax step (cf-1.com/news/4799680
// §3.2): with loc = ref + off / (W_l, H_l) and A = softmax over each run of
// L*K logits, the gradient of the head's pre-activations is
//   grad_off_x = grad_loc_x / W_l,  grad_off_y = grad_loc_y / H_l,
//   grad_logit_j = A_j * (grad_A_j - sum_{i in run} A_i grad_A_i),
// and grad_ref = sum over the query's samples of grad_loc.  One warp per
// query row; L*K a power of two of at most 32 (a run is LK consecutive lanes).
__global__ void __launch_bounds__(256) head_backward_kernel(int64_t rows, int P, int L, int K,
                                                            const float *attn, const float *gloc,
                                                            const float *gattn, const int64_t *shapes,
                                                            float *ghead, float *gref)
{
    __shared__ float Hs[kMaxLevels], Ws[kMaxLevels];
    if (threadIdx.x < L) {
        Hs[threadIdx.x] = (float)shapes[2 * threadIdx.x];
        Ws[threadIdx.x] = (float)shapes[2 * threadIdx.x + 1];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int LK = L * K;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const float *gl = gloc + r * 2 * P;
        float *gh = ghead + r * 3 * P;
        float sx = 0.f, sy = 0.f;
        for (int h = lane; h < 2 * P; h += 32) {
            const int l = (h >> 1) / K % L;
            const float g = __ldg(gl + h);
            gh[h] = g / ((h & 1) ? Hs[l] : Ws[l]);
            if (h & 1)
                sy += g;
            else
                sx += g;
        }
        for (int j0 = 0; j0 < P; j0 += 32) {
            const int j = j0 + lane;
            const float a = j < P ? __ldg(attn + r * P + j) : 0.f;
            const float g = j < P ? __ldg(gattn + r * P + j) : 0.f;
            float dot = a * g;
            for (int o = 1; o < LK; o <<= 1)
                dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (j < P)
                gh[2 * P + j] = a * (g - dot);
        }
        if (gref) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sx += __shfl_xor_sync(0xffffffffu, sx, o);
                sy += __shfl_xor_sync(0xffffffffu, sy, o);
            }
            if (lane == 0) {
                gref[2 * r] = sx;
                gref[2 * r + 1] = sy;
            }
        }
    }
}

}  // namespace msda
