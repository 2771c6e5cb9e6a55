// msda_kernels.cuh -- sm_100a kernels of the multi-scale deformable attention
// core: forward, backward and their fused variants (location + softmax in the
// kernel), plus the zero-fill and float32 -> bf16 conversion helpers.
//
// Work decomposition.  A "row" is one (b, q, m) triple, rows are numbered
// r = (b * Q + q) * M + m, so consecutive rows are the heads of one query and
// consecutive queries follow.  A group of G lanes owns one row; each lane owns
// one 16-byte vector (4 float32 or 8 bf16 channels) of the head_dim axis, so a
// corner of a sample is one fully used 16*G-byte row segment of `value`
// (128 bytes for D = 32 float32).  A warp carries 32 / G rows, a CTA up to 8
// warps (fewer when the per-row shared-memory records would not fit).
// Each CTA walks a contiguous range of row tiles (persistent grid, one wave),
// so neighbouring queries -- which sample neighbouring pixels -- stay on one SM
// and share its L1.
//
// Per tile there are two phases:
//   1. set-up: the group's lanes turn the row's L*K samples into 16-byte
//      records {fx, fy, A, key|mask} in shared memory (pixel coordinate, floor,
//      the four corner in-map bits, the attention weight -- in the fused
//      kernels also the location step and the softmax over the L*K logits);
//   2. gather: every lane of the group reads each record (a shared-memory
//      broadcast) and issues the four corner loads for its vector; the forward
//      accumulates A * w_c * v_c in float32 registers, the backward forms the
//      four partial dot products <g, v_c>, reduces the three gradient terms over
//      the group with butterfly shuffles and scatters A * w_c * g into
//      grad_value with 16-byte vector float32 reductions (red.global.add.v4.f32).
//
// Floor decisions.  The pixel coordinate x = loc_x * W - 0.5 and its floor are
// taken in float64 with the same operations, in the same order, as the
// defining formula (fused: loc = ref + off / W first, then loc * W - 0.5), so
// the corner choice is exactly that of the formula evaluated in double
// precision; the fractional parts are then rounded to float32 and everything
// else runs in float32.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace msda {

constexpr int kMaxLevels = 16;
constexpr int kMaxWarpsPerCta = 8;
constexpr int kKeyBias = 1 << 27;  // keys are stored biased into 28 bits

// Per-device status word; kernels record inconsistent geometry here.
__device__ int g_device_status;

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
    int64_t tiles_per_cta;
    int64_t S;
    int Q, M, L, K;
};

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
            atomicExch(&g_device_status, 4 /* MSDA_ERR_DEVICE_CHECK */);
    }
    __syncthreads();
    return ok != 0;
}

// ---------------------------------------------------------------- vectors --

template <typename T> struct Vec;

template <> struct Vec<float> {
    static constexpr int kElems = 4;
    using Raw = float4;
    __device__ __forceinline__ static void widen(const Raw &r, float *f)
    {
        f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
    }
    __device__ __forceinline__ static Raw narrow(const float *f)
    {
        return make_float4(f[0], f[1], f[2], f[3]);
    }
};

template <> struct Vec<__nv_bfloat16> {
    static constexpr int kElems = 8;
    using Raw = uint4;
    // bf16 -> f32 is exact: the bf16 bits are the top half of the float.
    __device__ __forceinline__ static void widen(const Raw &r, float *f)
    {
        const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(u[i] << 16);
            f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static Raw narrow(const float *f)
    {
        uint32_t u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            u[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        return make_uint4(u[0], u[1], u[2], u[3]);
    }
};

template <typename T, int D> struct Layout {
    static constexpr int kEpv = Vec<T>::kElems;              // channels per vector
    static constexpr int kNvec = D / kEpv;                   // vectors per row
    static constexpr int kG = kNvec < 32 ? kNvec : 32;       // lanes per row
    static constexpr int kCh = kNvec / kG;                   // vectors per lane
    static constexpr int kRowsPerWarp = 32 / kG;
    static constexpr int kLaneElems = kCh * kEpv;            // channels per lane
    static_assert(kNvec >= 1 && kNvec % kG == 0, "unsupported head_dim");
};

template <typename T>
__device__ __forceinline__ typename Vec<T>::Raw load_value(const typename Vec<T>::Raw *p)
{
    return __ldg(p);
}

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

// ----------------------------------------------------------------- set-up --

// One sample's record: fractional parts, attention weight, and the biased key
// of its top-left corner (start_l + y0 * W + x0) with the four corner in-map
// bits in the top nibble (bit c: corner c = (y0 + c/2, x0 + c%2) is inside).
struct Record {
    float fx, fy, A;
    uint32_t packed;
};

__device__ __forceinline__ Record make_record(double x, double y, int H, int W, int start, float A)
{
    Record r;
    r.A = A;
    bool valid = (x > -1.0) && (x < (double)W) && (y > -1.0) && (y < (double)H);
    if (!valid) {
        r.fx = 0.f;
        r.fy = 0.f;
        r.packed = (uint32_t)kKeyBias;  // mask 0: nothing is read
        return r;
    }
    double x0d = floor(x), y0d = floor(y);
    int x0 = (int)x0d, y0 = (int)y0d;  // x0 in [-1, W-1], y0 in [-1, H-1]
    r.fx = (float)(x - x0d);
    r.fy = (float)(y - y0d);
    uint32_t mask = 0;
    bool left = x0 >= 0, right = x0 + 1 < W, top = y0 >= 0, bottom = y0 + 1 < H;
    mask |= (top && left) ? 1u : 0u;
    mask |= (top && right) ? 2u : 0u;
    mask |= (bottom && left) ? 4u : 0u;
    mask |= (bottom && right) ? 8u : 0u;
    int key = start + y0 * W + x0;
    r.packed = (uint32_t)(key + kKeyBias) | (mask << 28);
    return r;
}

__device__ __forceinline__ int record_key(uint32_t packed)
{
    return (int)(packed & 0x0fffffffu) - kKeyBias;
}

// Non-fused: x = loc_x * W - 0.5 in float64 (the product of a float32 and an
// integer below 2^16 is exact, so this equals the double-precision formula).
__device__ __forceinline__ void pixel_from_location(float lx, float ly, int H, int W,
                                                    double &x, double &y)
{
    x = __dsub_rn(__dmul_rn((double)lx, (double)W), 0.5);
    y = __dsub_rn(__dmul_rn((double)ly, (double)H), 0.5);
}

// Fused: loc = ref + off / (W, H) then x = loc * W - 0.5, each operation
// rounded in float64 exactly as the formula reads.
__device__ __forceinline__ void pixel_from_offset(float rx, float ry, float ox, float oy,
                                                  int H, int W, double &x, double &y)
{
    double lx = __dadd_rn((double)rx, __ddiv_rn((double)ox, (double)W));
    double ly = __dadd_rn((double)ry, __ddiv_rn((double)oy, (double)H));
    x = __dsub_rn(__dmul_rn(lx, (double)W), 0.5);
    y = __dsub_rn(__dmul_rn(ly, (double)H), 0.5);
}

// Level of flattened sample s = l * K + k.
__device__ __forceinline__ int level_of(int s, int K) { return s / K; }

// Builds the records of one row into rec[0 .. P-1]; lane `gl` of the group
// does samples gl, gl + G, ...  For the fused kernels the softmax over the
// row's logits is taken here as well (max-subtracted, float32).
template <int G, bool FUSED>
__device__ __forceinline__ void setup_row(const KernelArgs &a, const Geometry &geo, int64_t row,
                                          bool active, int gl, Record *rec, float *attn_out)
{
    const int P = a.L * a.K;
    const int64_t base = row * P;
    float mx = -INFINITY, inv_sum = 0.f;
    float rx = 0.f, ry = 0.f;
    if (FUSED) {
        // softmax statistics of the row (every lane of the warp takes part in
        // the shuffles, inactive groups on dummy values)
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
        if (active) {
            int64_t bq = row / a.M;
            rx = __ldg(a.ref + 2 * bq);
            ry = __ldg(a.ref + 2 * bq + 1);
        }
    }
    if (!active)
        return;
    for (int s = gl; s < P; s += G) {
        const int l = level_of(s, a.K);
        const int H = geo.H[l], W = geo.W[l];
        double x, y;
        float A;
        if (FUSED) {
            const float2 o = __ldg(reinterpret_cast<const float2 *>(a.off) + base + s);
            pixel_from_offset(rx, ry, o.x, o.y, H, W, x, y);
            A = expf(__ldg(a.logits + base + s) - mx) * inv_sum;
            if (attn_out)
                attn_out[base + s] = A;
        } else {
            const float2 p = __ldg(reinterpret_cast<const float2 *>(a.loc) + base + s);
            pixel_from_location(p.x, p.y, H, W, x, y);
            A = __ldg(a.attn + base + s);
        }
        rec[s] = make_record(x, y, H, W, geo.start[l], A);
    }
}

// ---------------------------------------------------------------- forward --

template <typename T, int D, bool FUSED>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32)
forward_kernel(const KernelArgs a)
{
    using Lay = Layout<T, D>;
    using Raw = typename Vec<T>::Raw;
    constexpr int G = Lay::kG, CH = Lay::kCh, E = Lay::kLaneElems;
    constexpr int UNROLL = 4;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ Geometry geo;
    __shared__ int geo_ok;
    if (!load_geometry(a, geo, geo_ok))
        return;

    const int P = a.L * a.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / G, gl = lane % G;
    Record *rec = reinterpret_cast<Record *>(smem_raw) + (warp * Lay::kRowsPerWarp + grp) * P;
    const int64_t rows_per_tile = a.rows_per_tile;
    const int64_t MD = (int64_t)a.M * D;

    const int64_t t0 = (int64_t)blockIdx.x * a.tiles_per_cta;
    const int64_t t1 = min(t0 + a.tiles_per_cta, a.ntiles);
    for (int64_t tile = t0; tile < t1; ++tile) {
        const int64_t row = tile * rows_per_tile + warp * Lay::kRowsPerWarp + grp;
        const bool active = row < a.rows;
        setup_row<G, FUSED>(a, geo, row, active, gl, rec, a.attn_out);
        __syncwarp();
        if (active) {
            const int64_t bq = row / a.M;
            const int m = (int)(row - bq * a.M);
            const int64_t b = bq / a.Q;
            // this lane's first vector of head m of batch b, key 0
            const Raw *vbase = reinterpret_cast<const Raw *>(static_cast<const T *>(a.value) +
                                                             (b * a.S * a.M + m) * D) + gl;
            float acc[E];
#pragma unroll
            for (int e = 0; e < E; ++e)
                acc[e] = 0.f;
            for (int l = 0; l < a.L; ++l) {
                const int64_t row_step = (int64_t)geo.W[l] * MD / Vec<T>::kElems;  // vectors
                const int64_t col_step = MD / Vec<T>::kElems;
                for (int k0 = 0; k0 < a.K; k0 += UNROLL) {
                    Raw v[UNROLL][4][CH];
                    float w[UNROLL][4];
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u) {
                        const bool in = k0 + u < a.K;
                        const Record r = in ? rec[l * a.K + k0 + u] : Record{0.f, 0.f, 0.f, (uint32_t)kKeyBias};
                        const uint32_t mask = r.packed >> 28;
                        const float ay1 = r.A * r.fy, ay0 = r.A - ay1;
                        w[u][0] = ay0 - ay0 * r.fx;
                        w[u][1] = ay0 * r.fx;
                        w[u][2] = ay1 - ay1 * r.fx;
                        w[u][3] = ay1 * r.fx;
                        const Raw *p0 = vbase + (int64_t)record_key(r.packed) * col_step;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const Raw *pc = p0 + ((c >> 1) ? row_step : 0) + ((c & 1) ? col_step : 0);
#pragma unroll
                            for (int j = 0; j < CH; ++j) {
                                if (mask & (1u << c))
                                    v[u][c][j] = load_value<T>(pc + j * G);
                                else
                                    v[u][c][j] = Raw{};
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < UNROLL; ++u)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int j = 0; j < CH; ++j) {
                                float f[Vec<T>::kElems];
                                Vec<T>::widen(v[u][c][j], f);
#pragma unroll
                                for (int e = 0; e < Vec<T>::kElems; ++e)
                                    acc[j * Vec<T>::kElems + e] = fmaf(w[u][c], f[e], acc[j * Vec<T>::kElems + e]);
                            }
                }
            }
            Raw *obase = reinterpret_cast<Raw *>(static_cast<T *>(a.out) + row * D) + gl;
#pragma unroll
            for (int j = 0; j < CH; ++j)
                obase[j * G] = Vec<T>::narrow(acc + j * Vec<T>::kElems);
        }
        __syncwarp();
    }
}

// --------------------------------------------------------------- backward --

template <typename T, int D, bool FUSED>
__global__ void __launch_bounds__(kMaxWarpsPerCta * 32)
backward_kernel(const KernelArgs a)
{
    using Lay = Layout<T, D>;
    using Raw = typename Vec<T>::Raw;
    constexpr int G = Lay::kG, CH = Lay::kCh, E = Lay::kLaneElems, EPV = Vec<T>::kElems;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ Geometry geo;
    __shared__ int geo_ok;
    if (!load_geometry(a, geo, geo_ok))
        return;

    const int P = a.L * a.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / G, gl = lane % G;
    const int row_slot = warp * Lay::kRowsPerWarp + grp;
    const int rows_per_cta = (int)a.rows_per_tile;
    Record *rec = reinterpret_cast<Record *>(smem_raw) + row_slot * P;
    // per-sample results of the row: (grad_x, grad_y, grad_A)
    float *res = reinterpret_cast<float *>(reinterpret_cast<Record *>(smem_raw) + rows_per_cta * P)
                 + row_slot * P * 3;
    const int64_t MD = (int64_t)a.M * D;

    const int64_t t0 = (int64_t)blockIdx.x * a.tiles_per_cta;
    const int64_t t1 = min(t0 + a.tiles_per_cta, a.ntiles);
    for (int64_t tile = t0; tile < t1; ++tile) {
        const int64_t row = tile * rows_per_cta + row_slot;
        const bool active = row < a.rows;
        setup_row<G, FUSED>(a, geo, row, active, gl, rec, nullptr);
        __syncwarp();
        const int64_t bq = active ? row / a.M : 0;
        const int m = active ? (int)(row - bq * a.M) : 0;
        const int64_t b = bq / a.Q;
        const Raw *vbase = reinterpret_cast<const Raw *>(static_cast<const T *>(a.value) +
                                                         (b * a.S * a.M + m) * D) + gl;
        float4 *gvbase = reinterpret_cast<float4 *>(a.grad_value + (b * a.S * a.M + m) * D) + gl * (EPV / 4);
        // grad_output chunk of this lane, widened
        float g[E];
        if (active) {
            const Raw *gp = reinterpret_cast<const Raw *>(static_cast<const T *>(a.grad_out) + row * D) + gl;
#pragma unroll
            for (int j = 0; j < CH; ++j)
                Vec<T>::widen(__ldg(gp + j * G), g + j * EPV);
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e)
                g[e] = 0.f;
        }
        float ref_gx = 0.f, ref_gy = 0.f;  // fused: sum over the row of grad_loc
        for (int l = 0; l < a.L; ++l) {
            const int W = geo.W[l], H = geo.H[l];
            const int64_t row_step = (int64_t)W * MD / EPV;
            const int64_t col_step = MD / EPV;
            for (int k = 0; k < a.K; ++k) {
                const int s = l * a.K + k;
                const Record r = active ? rec[s] : Record{0.f, 0.f, 0.f, (uint32_t)kKeyBias};
                const uint32_t mask = r.packed >> 28;
                const Raw *p0 = vbase + (int64_t)record_key(r.packed) * col_step;
                float d[4] = {0.f, 0.f, 0.f, 0.f};  // partial <g, v_c>
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int64_t coff = ((c >> 1) ? row_step : 0) + ((c & 1) ? col_step : 0);
#pragma unroll
                    for (int j = 0; j < CH; ++j) {
                        if (mask & (1u << c)) {
                            float f[EPV];
                            Vec<T>::widen(load_value<T>(p0 + coff + j * G), f);
#pragma unroll
                            for (int e = 0; e < EPV; ++e)
                                d[c] = fmaf(g[j * EPV + e], f[e], d[c]);
                        }
                    }
                }
                const float fx = r.fx, fy = r.fy;
                const float w00 = (1.f - fx) * (1.f - fy), w01 = fx * (1.f - fy);
                const float w10 = (1.f - fx) * fy, w11 = fx * fy;
                float ga = w00 * d[0] + w01 * d[1] + w10 * d[2] + w11 * d[3];
                float gx = (1.f - fy) * (d[1] - d[0]) + fy * (d[3] - d[2]);
                float gy = (1.f - fx) * (d[2] - d[0]) + fx * (d[3] - d[1]);
                ga = group_sum<G>(ga);
                gx = group_sum<G>(gx);
                gy = group_sum<G>(gy);
                if (active && mask) {
                    // scatter A * w_c * g into grad_value
                    const float wc[4] = {r.A * w00, r.A * w01, r.A * w10, r.A * w11};
                    float4 *q0 = gvbase + (int64_t)record_key(r.packed) * (MD / 4);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (!(mask & (1u << c)))
                            continue;
                        float4 *qc = q0 + ((c >> 1) ? (int64_t)W * MD / 4 : 0) + ((c & 1) ? MD / 4 : 0);
#pragma unroll
                        for (int j = 0; j < CH; ++j)
#pragma unroll
                            for (int h = 0; h < EPV / 4; ++h) {
                                const float *gg = g + j * EPV + 4 * h;
                                atomicAdd(qc + j * G * (EPV / 4) + h,
                                          make_float4(wc[c] * gg[0], wc[c] * gg[1], wc[c] * gg[2], wc[c] * gg[3]));
                            }
                    }
                }
                // gradients w.r.t. the pixel coordinate, scaled to the caller's units
                const float gxA = r.A * gx, gyA = r.A * gy;
                if (active && gl == (s % G)) {
                    if (FUSED) {
                        res[3 * s] = gxA;         // grad offset (level pixels)
                        res[3 * s + 1] = gyA;
                    } else {
                        res[3 * s] = (float)W * gxA;   // grad location (normalized)
                        res[3 * s + 1] = (float)H * gyA;
                    }
                    res[3 * s + 2] = ga;
                }
                if (FUSED) {
                    ref_gx += (float)W * gxA;
                    ref_gy += (float)H * gyA;
                }
            }
        }
        __syncwarp();
        // softmax Jacobian: grad_z_j = A_j (gA_j - sum_i A_i gA_i); every lane
        // of the warp takes part in the shuffles
        float dot = 0.f;
        if (FUSED) {
            if (active)
                for (int s = gl; s < P; s += G)
                    dot += rec[s].A * res[3 * s + 2];
            dot = group_sum<G>(dot);
        }
        if (active) {
            const int64_t base = row * P;
            if (FUSED) {
                for (int s = gl; s < P; s += G) {
                    a.grad_logits[base + s] = rec[s].A * (res[3 * s + 2] - dot);
                    reinterpret_cast<float2 *>(a.grad_off)[base + s] = make_float2(res[3 * s], res[3 * s + 1]);
                }
                if (a.grad_ref && gl == 0) {
                    atomicAdd(a.grad_ref + 2 * bq, ref_gx);
                    atomicAdd(a.grad_ref + 2 * bq + 1, ref_gy);
                }
            } else {
                for (int s = gl; s < P; s += G) {
                    reinterpret_cast<float2 *>(a.grad_loc)[base + s] = make_float2(res[3 * s], res[3 * s + 1]);
                    a.grad_attn[base + s] = res[3 * s + 2];
                }
            }
        }
        __syncwarp();
    }
}

// ----------------------------------------------------------------- helpers --

// Zeroes n4 float4 of `a` and n floats of `b` (grid-stride).
__global__ void zero_kernel(float4 *a, int64_t n4, float *b, int64_t n)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride)
        a[i] = make_float4(0.f, 0.f, 0.f, 0.f);
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
        dst[i] = Vec<__nv_bfloat16>::narrow(f);
    }
}

}  // namespace msda
