// msda_gemm.cuh -- dense layers around the operator on the 5th-generation
// tensor cores (tcgen05, sm_100a): the value / output projections W'_m, W_m
// and the query-side head that predicts the sampling offsets and attention
// logits (discosf.com/news/5175395 §2.2 and §3.1; cf-1.com/news/4799680
// §3.1-3.2).
//
//   out[r, n] = sum_k x[r, k] * w[n, k] + bias[n]
//
// x [rows, K] and w [N, K] are bf16, row-major (K contiguous: nn.Linear's
// weight layout); the products accumulate in float32 in tensor memory (TMEM).
//
// Persistent kernel, one CTA per SM walking 128-row x BN-column output tiles
// (BN = 128 * NSUB; the column tiles of one row block are consecutive, so the
// CTAs working on them share the x tile through L2), 10 warps with fixed
// roles:
//   warp 0, one lane   TMA producer: per 64-wide K block, a 128 x 64 tile of
//                      x and NSUB 128 x 64 tiles of w (128-byte swizzle) into
//                      a STAGES-deep shared-memory ring; completion on a
//                      "full" mbarrier per stage (transaction bytes);
//   warp 1             allocates the TMEM columns; one lane issues the MMAs
//                      (M = 128, N = BN, K = 16 per instruction,
//                      cta_group::1, kind::f16 with bf16 operands, float32
//                      accumulation), frees each stage with tcgen05.commit on
//                      its "empty" barrier and, after a tile's last K block,
//                      commits the tile's accumulator buffer to the epilogue;
//   warps 2..9         epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31
//                      (its 32 output rows; kEpiWarps / 4 warps per lane
//                      quarter, two by default, each taking every
//                      kEpiParts-th column chunk) 32 columns at a
//                      time, applies the epilogue, writes 32-row x 128-byte
//                      boxes into shared memory (128-byte swizzle, one box
//                      per warp by default) and stores them with TMA; then it
//                      hands the accumulator buffer back to the MMA lane.
// Measured on 87040 x 256 -> 256 (bf16 out, B200): the K-block cadence is set
// by the stage ring (a 16 KB TMA load takes about 1.1 us to land under load,
// so the ring's depth bounds the MMA rate); one epilogue box per warp instead
// of two frees 32 KB for two more stages (21.8 -> 19.2 us), the bias from
// shared memory instead of 32 shuffles per 32 columns takes a third off each
// box (-> 19.0 us), and one N = 256 MMA instead of two of N = 128 per K step
// 23.1 -> 21.8 us.  Twelve epilogue warps instead of eight: no change
// (19.3 us; query head 42.7 against 43.5 us).
// With NSUB <= 2 there are two accumulator buffers (2 x BN <= 512 columns),
// so a tile's epilogue overlaps the next tile's loads and MMAs.
// No TMA multicast and no clusters: the tensor maps cover this GPU's memory
// and every CTA loads its own tiles.
//
// Every wait is bounded (kGemmSpinLimit suspending tries of an mbarrier,
// about a second in all); a wait that runs out records
// MSDA_ERR_DEVICE_TIMEOUT (5) in the status word, every role stops issuing
// work, the CTA waits (bounded) for what it issued, frees its TMEM and
// returns.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace msda_gemm {

constexpr int kBM = 128;           // rows per tile (TMEM lanes)
constexpr int kBK = 64;            // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kSubN = 128;         // columns per MMA (and per TMA box of w)
#ifndef MSDA_GEMM_EPI_WARPS
#define MSDA_GEMM_EPI_WARPS 8                       // epilogue warps (a multiple of 4)
#endif
constexpr int kEpiWarps = MSDA_GEMM_EPI_WARPS;
constexpr int kEpiParts = kEpiWarps / 4;          // epilogue warps per TMEM lane quarter
static_assert(kEpiWarps % 4 == 0, "epilogue warps come in lane quarters");
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kATileBytes = kBM * kBK * 2;      // 16 KB
constexpr int kBSubBytes = kSubN * kBK * 2;     // 16 KB
constexpr int kBoxBytes = 32 * 128;             // one epilogue box: 32 rows x 128 bytes
#ifndef MSDA_GEMM_EPI_BOXES
#define MSDA_GEMM_EPI_BOXES 1                       // epilogue boxes per warp (1 or 2)
#endif
constexpr int kEpiBoxes = MSDA_GEMM_EPI_BOXES;
constexpr int kGemmSpinLimit = 1 << 20;
constexpr int kMaxLevels = 16;

// Epilogue kinds.
enum : int {
    kEpiStore = 0,   // out[r, n] (+ bias), float32 or bf16
    kEpiHead = 1,    // query head: head columns [0, 2P) -> sampling locations,
                     // [2P, 3P) -> softmax over runs of L*K -> attention weights
};

struct Params {
    int rows, N, K;           // out is rows x N
    int m_tiles, n_tiles;
    const float *bias;        // [N] or null
    int epi;
    int out_bf16;             // kEpiStore: bf16 output (else float32)
    // kEpiHead: tile column c is head column c of a head whose first 2P
    // columns are the (x, y) offsets in level pixels of the samples
    // s = (m * L + l) * K + k and whose last P columns are their logits,
    // P = M*L*K; the level of sample s is (s & lk_mask) >> k_shift (L*K and
    // K are powers of two)
    int P, L, LK, lk_mask, k_shift;
    const float *ref;         // [rows, 2] normalized reference points
    const int64_t *shapes;    // [L, 2] (H, W), device
    int stages;               // stage ring depth (<= kMaxStages)
    int w_bytes;              // weight-resident: bytes of the w area
    int withhold;             // testing: arm the CTA's first stage without loading it
    int *status;
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_addr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_addr(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(b)) : "memory");
}
// One potentially blocking test: the thread is suspended until the phase
// completes or about kTryWaitNs nanoseconds pass, and woken as soon as it
// completes (no sleep quantum added to the hand-off latency).
#ifndef MSDA_GEMM_TRY_WAIT_NS
#define MSDA_GEMM_TRY_WAIT_NS 1000
#endif
constexpr unsigned kTryWaitNs = MSDA_GEMM_TRY_WAIT_NS;
__device__ __forceinline__ bool mbar_try(uint64_t *b, unsigned parity)
{
    uint32_t ok;
    if constexpr (kTryWaitNs > 0)
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
                     " selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(ok) : "r"(smem_addr(b)), "r"(parity), "n"(kTryWaitNs) : "memory");
    else
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                     " selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(ok) : "r"(smem_addr(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait for the completion of the phase with the given parity: at
// most kGemmSpinLimit tries of about a microsecond each.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, unsigned parity)
{
    for (int i = 0; i < kGemmSpinLimit; ++i)
        if (mbar_try(b, parity))
            return true;
    return false;
}

// 2-D TMA load of box (x = column coordinate, y = row coordinate).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
                    "r"(smem_addr(bar))
                 : "memory");
}
// 2-D TMA store of a shared-memory box; rows and columns outside the tensor
// are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, const void *src)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(src)) : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most N committed stores are still reading shared memory.
template <int N> __device__ __forceinline__ void tma_store_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory");
}
__device__ __forceinline__ void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major bf16 tile with 128-byte rows
// in the 128-byte swizzle TMA writes: start address (16-byte units), leading
// offset 1 (unused for swizzled K-major), stride between 8-row groups 1024
// bytes, descriptor version 1, swizzle mode 2 (128 B).  The tile base must be
// 1024-byte aligned; a K step of 16 elements adds 32 bytes to the start.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: kind::f16 with bf16 A and B, float32 D, both
// K-major, M = 128, N columns (a multiple of 16, at most 256).
template <int N>
constexpr uint32_t idesc_bf16()
{
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

// D[128 x N] (+)= A[128 x 16] * B[N x 16]^T; B's N rows are consecutive
// 128-byte rows (8-row groups 1024 bytes apart), as NSUB 128-row boxes of w
// stored back to back are.
template <int N>
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t acc)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc_bf16<N>()), "r"(acc)
                 : "memory");
}
// Arrives on `bar` when every MMA this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_addr(bar)) : "memory");
}

// 32 consecutive float32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32"
                 " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
                 " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
                 " [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
                   "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
                   "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
                   "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared memory (dynamic, 1024-byte aligned): the stage ring, the epilogue
// boxes (kEpiBoxes per epilogue warp), then the barriers.  Host and device
// agree.
// WRES (weight-resident): the CTA's BN x K block of w (p.w_bytes, at most
// kWMaxBytes) is loaded once and only x streams through the ring; every tile
// of the CTA then has the same column tile.  The ring has p.stages stages
// (at most kMaxStages), as many as the shared memory left over holds.
constexpr int kWMaxBytes = 128 * 1024;
constexpr int kMaxStages = 12;

template <int NSUB, bool WRES> struct Cfg {
    static constexpr int kBN = kSubN * NSUB;
    static constexpr int kStageBytes = WRES ? kATileBytes : kATileBytes + NSUB * kBSubBytes;
    static constexpr int kAcc = 2;                                 // TMEM accumulator buffers
    static constexpr int kTmemCols = 2 * kBN;
    static constexpr int kMaxKBlocks = kWMaxBytes / (NSUB * kBSubBytes);  // WRES: K blocks w may have
    static constexpr int kEpiBytes = kEpiWarps * kEpiBoxes * kBoxBytes;
    // full, empty per stage; accumulator full / empty; drain; w full
    static constexpr int kBarBytes = 8 * (2 * kMaxStages + 2 * kAcc + 2) + 16;
    // dynamic shared memory for a w area of w_bytes and `stages` stages
    static constexpr int smem_bytes(int w_bytes, int stages)
    {
        return 1024 + w_bytes + stages * kStageBytes + kEpiBytes + kBarBytes;
    }
};

// Writes this lane's row of a 32 x 128-byte box in the 128-byte swizzle
// (16-byte chunk j of row i at chunk j ^ (i % 8)).
__device__ __forceinline__ void box_put_row(uint8_t *box, int i, const uint4 (&chunks)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4 *>(box + i * 128 + ((j ^ (i & 7)) << 4)) = chunks[j];
}

__device__ __forceinline__ void pack_f32(const float (&v)[32], uint4 (&c)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        c[j] = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]), __float_as_uint(v[4 * j + 2]),
                          __float_as_uint(v[4 * j + 3]));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// bias[col + lane] (0 past N or without a bias): one coalesced load for a
// warp's 32 columns.
__device__ __forceinline__ float bias_lane(const float *bias, int col, int N, int lane)
{
    return (bias && col + lane < N) ? __ldg(bias + col + lane) : 0.f;
}

// Adds the 32 columns' bias to v: lane i holds element i (bias_lane), the
// values reach every lane by shuffles.
__device__ __forceinline__ void add_bias32(float mine, float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] += __shfl_sync(0xffffffffu, mine, i);
}

// Adds b[0 .. 31] (shared memory, 16-byte aligned; every lane reads the
// same words, a broadcast) to v.
__device__ __forceinline__ void add_bias32_smem(const float *b, float (&v)[32])
{
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(b + i);
        v[i] += t.x;
        v[i + 1] += t.y;
        v[i + 2] += t.z;
        v[i + 3] += t.w;
    }
}

template <int LK>
__device__ __forceinline__ void softmax_runs(float (&v)[32])
{
    constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
    for (int j = 0; j < 32; j += LK) {
        float mx = v[j];
#pragma unroll
        for (int t = 1; t < LK; ++t)
            mx = fmaxf(mx, v[j + t]);
        const float mxl = mx * kLog2e;
        float sum = 0.f;
#pragma unroll
        for (int t = 0; t < LK; ++t) {
            v[j + t] = exp2f(fmaf(v[j + t], kLog2e, -mxl));  // exp(z - max)
            sum += v[j + t];
        }
        const float inv = 1.0f / sum;
#pragma unroll
        for (int t = 0; t < LK; ++t)
            v[j + t] *= inv;
    }
}

// ------------------------------------------------------------------ kernel --

template <int NSUB, bool WRES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
            const __grid_constant__ CUtensorMap map_o0, const __grid_constant__ CUtensorMap map_o1, Params p)
{
    using C = Cfg<NSUB, WRES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int S = p.stages;
    uint8_t *w_area = base;                       // WRES only
    uint8_t *smem = base + (WRES ? p.w_bytes : 0);  // stage ring
    uint8_t *epi_smem = smem + S * C::kStageBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(epi_smem + C::kEpiBytes);
    uint64_t *empty = full + kMaxStages;
    uint64_t *acc_full = empty + kMaxStages;
    uint64_t *acc_empty = acc_full + C::kAcc;
    uint64_t *drain = acc_empty + C::kAcc;
    uint64_t *wfull = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(wfull + 1);
    // query head: 1 / W_l or 1 / H_l of head column h, at h % (2 L K)
    __shared__ float colscale[2 * 32];
    // weight-resident: the bias of the CTA's column tile (0 past N), added
    // from shared memory (a shuffle per column costs the epilogue more than
    // its whole tensor-memory read)
    __shared__ __align__(16) float sbias[WRES ? C::kBN : 4];
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = (p.K + kBK - 1) / kBK;
    const int ntiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < C::kAcc; ++b) {
            mbar_init(acc_full + b, 1);
            mbar_init(acc_empty + b, kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(wfull, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    if (WRES) {
        const int nb0 = (blockIdx.x % p.n_tiles) * C::kBN;
        for (int i = threadIdx.x; i < C::kBN; i += blockDim.x)
            sbias[i] = (p.bias && nb0 + i < p.N) ? p.bias[nb0 + i] : 0.f;
    }
    if (p.epi == kEpiHead && threadIdx.x < 2 * p.LK) {
        const int j = threadIdx.x, l = ((j >> 1) & p.lk_mask) >> p.k_shift;
        colscale[j] = 1.0f / (float)p.shapes[2 * l + ((j & 1) ? 0 : 1)];
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(tmem_slot)), "r"(C::kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int g = 0;  // k blocks issued so far (all tiles)
            if (WRES && blockIdx.x < ntiles) {
                // the CTA's column tile (the grid is a multiple of n_tiles):
                // all K blocks of w, once
                const int n0 = (blockIdx.x % p.n_tiles) * C::kBN;
                mbar_expect_tx(wfull, (unsigned)(nkb * NSUB * kBSubBytes));
                for (int kb = 0; kb < nkb; ++kb)
#pragma unroll
                    for (int j = 0; j < NSUB; ++j)
                        tma_load_2d(w_area + (kb * NSUB + j) * kBSubBytes, &map_w, kb * kBK, n0 + j * kSubN,
                                    wfull);
            }
            for (int t = blockIdx.x; t < ntiles && !*(volatile int *)&abort_flag; t += gridDim.x) {
                const int m0 = (t / p.n_tiles) * kBM, n0 = (t % p.n_tiles) * C::kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(empty + s, ((g / S) - 1) & 1)) {
                        atomicExch(p.status, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                        abort_flag = 1;
                        break;
                    }
                    uint8_t *a_tile = smem + s * C::kStageBytes;
                    mbar_expect_tx(full + s, (unsigned)C::kStageBytes);
                    if (p.withhold && g == 0)
                        continue;  // the stage never fills: the MMA lane's wait runs out
                    tma_load_2d(a_tile, &map_x, kb * kBK, m0, full + s);
                    if (!WRES) {
#pragma unroll
                        for (int j = 0; j < NSUB; ++j)
                            tma_load_2d(a_tile + kATileBytes + j * kBSubBytes, &map_w, kb * kBK,
                                        n0 + j * kSubN, full + s);
                    }
                }
            }
            // everything issued has landed before the CTA may exit
            for (int h = g - S < 0 ? 0 : g - S; h < g; ++h)
                mbar_wait(full + h % S, (h / S) & 1);
            if (WRES && blockIdx.x < ntiles)
                mbar_wait(wfull, 0);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int g = 0, local = 0;
            if (WRES && blockIdx.x < ntiles && !mbar_wait(wfull, 0)) {
                atomicExch(p.status, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                abort_flag = 1;
            }
            for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
                const int buf = local % C::kAcc, use = local / C::kAcc;
                bool ok = !*(volatile int *)&abort_flag;
                if (ok && use > 0)
                    ok = mbar_wait(acc_empty + buf, (use - 1) & 1);
                if (!ok) {
                    atomicExch(p.status, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                    abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + buf * C::kBN;
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!mbar_wait(full + s, (g / S) & 1) || *(volatile int *)&abort_flag) {
                        atomicExch(p.status, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                        abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_addr(smem + s * C::kStageBytes);
                    const uint32_t b_base = WRES ? smem_addr(w_area + kb * NSUB * kBSubBytes)
                                                 : a_base + kATileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // one MMA over all BN columns (the w sub-tiles are
                        // consecutive rows of one operand)
                        mma_bf16<C::kBN>(d, smem_desc(a_base + kk * 32), smem_desc(b_base + kk * 32),
                                         (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(empty + s);  // frees the stage once these MMAs have read it
                }
                mma_commit(acc_full + buf);  // the tile's accumulator is complete
                if (!ok)
                    break;
            }
            // no MMA may be in flight when the TMEM is freed
            mma_commit(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;                     // TMEM lane quarter
        const int e = warp - 2;                     // epilogue warp index
        const int part = e >> 2;                    // which column chunks of the quarter
        uint8_t *boxes = epi_smem + e * kEpiBoxes * kBoxBytes;
        int nbox = 0, local = 0;
        const int step = (p.epi == kEpiStore && p.out_bf16) ? 64 : 32;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++local) {
            const int buf = local % C::kAcc, use = local / C::kAcc;
            const int m0 = (t / p.n_tiles) * kBM, n0 = (t % p.n_tiles) * C::kBN;
            // this warp's bias values of the tile (chunks c0 = part*step +
            // kEpiParts*step*k, 32 columns each), loaded before the
            // accumulator wait
            constexpr int kNb = WRES ? 1 : (C::kBN / 32 + kEpiParts - 1) / kEpiParts;
            float bl[kNb];
#pragma unroll
            for (int k = 0; k < kNb; ++k) {
                const int c = part * step + (k / (step / 32)) * kEpiParts * step + (k % (step / 32)) * 32;
                bl[k] = (!WRES && c < C::kBN) ? bias_lane(p.bias, n0 + c, p.N, lane) : 0.f;
            }
            const bool ready = __all_sync(0xffffffffu, mbar_wait(acc_full + buf, use & 1) &&
                                                           !*(volatile int *)&abort_flag);
            if (!ready) {
                if (lane == 0) {
                    atomicExch(p.status, 5 /* MSDA_ERR_DEVICE_TIMEOUT */);
                    abort_flag = 1;
                }
                break;
            }
            tc_fence_after();
            const int row0 = m0 + 32 * q;           // first row of this warp
            const int r = row0 + lane;
            const uint32_t tbase = tmem + buf * C::kBN + ((uint32_t)(32 * q) << 16);
            float rx = 0.f, ry = 0.f;
            if (p.epi == kEpiHead && r < p.rows) {
                rx = __ldg(p.ref + 2 * (int64_t)r);
                ry = __ldg(p.ref + 2 * (int64_t)r + 1);
            }
#pragma unroll 1
            for (int c0 = part * step, kc = 0; c0 < C::kBN && n0 + c0 < p.N; c0 += kEpiParts * step, ++kc) {
                float v[32], v2[32];
                tmem_ld32(tbase + c0, v);
                if (step == 64)
                    tmem_ld32(tbase + c0 + 32, v2);
                const int col = n0 + c0;
                uint4 chunks[8];
                const CUtensorMap *map = &map_o0;
                int x = col;
                // this chunk's bias values (kc < kNb: registers, no dynamic index)
                float b0 = 0.f, b1 = 0.f;
#pragma unroll
                for (int k = 0; k < kNb; ++k) {
                    if (k == kc * (step / 32))
                        b0 = bl[k];
                    if (step == 64 && k == kc * 2 + 1)
                        b1 = bl[k];
                }
                if (p.epi == kEpiStore) {
                    if (WRES) {
                        if (p.bias) {
                            add_bias32_smem(sbias + c0, v);
                            if (step == 64)
                                add_bias32_smem(sbias + c0 + 32, v2);
                        }
                    } else if (p.bias) {
                        add_bias32(b0, v);
                        if (step == 64)
                            add_bias32(b1, v2);
                    }
                    if (step == 64) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            chunks[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                                                   pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                                                   pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                                                   pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            chunks[4 + j] = make_uint4(pack_bf16x2(v2[8 * j], v2[8 * j + 1]),
                                                       pack_bf16x2(v2[8 * j + 2], v2[8 * j + 3]),
                                                       pack_bf16x2(v2[8 * j + 4], v2[8 * j + 5]),
                                                       pack_bf16x2(v2[8 * j + 6], v2[8 * j + 7]));
                    } else {
                        pack_f32(v, chunks);
                    }
                } else {
                    // query head: a 32-column chunk is all offsets or whole runs of logits
                    if (WRES)
                        add_bias32_smem(sbias + c0, v);
                    else if (p.bias)
                        add_bias32(b0, v);
                    if (col < 2 * p.P) {
                        const int cmask = 2 * p.LK - 1;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            v[i] = fmaf(v[i], colscale[(col + i) & cmask], (i & 1) ? ry : rx);
                    } else {
                        switch (p.LK) {
                        case 1: softmax_runs<1>(v); break;
                        case 2: softmax_runs<2>(v); break;
                        case 4: softmax_runs<4>(v); break;
                        case 8: softmax_runs<8>(v); break;
                        case 16: softmax_runs<16>(v); break;
                        default: softmax_runs<32>(v); break;
                        }
                        map = &map_o1;
                        x = col - 2 * p.P;
                    }
                    pack_f32(v, chunks);
                }
                // stage the box (kEpiBoxes buffers: the store issued kEpiBoxes
                // boxes ago must have finished reading it) and store it with TMA
                uint8_t *box = boxes + (nbox % kEpiBoxes) * kBoxBytes;
                if (lane == 0)
                    tma_store_wait_read<kEpiBoxes - 1>();
                __syncwarp();
                box_put_row(box, lane, chunks);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0)
                    tma_store_2d(map, x, row0, box);
                ++nbox;
            }
            // the accumulator buffer may be refilled once every lane has read it
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acc_empty + buf);
        }
        if (lane == 0)
            tma_store_wait_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(C::kTmemCols)
                     : "memory");
}

}  // namespace msda_gemm
