// gemm_kernel.cuh -- persistent, warp-specialized NVFP4 x NVFP4 GEMM for
// sm_100a on the 5th-generation tensor cores, with the per-module
// global-scale epilogue of a fused-module linear layer.
//
//   out[m, n] = round( acc[m, n] * fl32(g_a * g_w[seg(n)]) )
//   acc[m, n] = sum_k qa[m,k] sa[m,k/16] qw[n,k] sw[n,k/16]   (fp32, TMEM)
//
// The block-scaled product runs on the tensor cores without emulation ("Why
// Gated DeltaNet Survives 4-Bit Quantization", kipquest.com, "The deep
// dive"); applying each module's own FP32 global scale to its columns is the
// repair of the global-scale mismatch: modules calibrated one by one, then
// run as a single fused GEMM under one scale, give wrong outputs
// (same page, "The abstract" and "The deep dive").
//
// Tile 128 x 256 (x 256 of K per pipeline stage), one CTA per SM, 12 warps:
//   warps 0, 3  TMA producers (4-stage ring): warp 0 the activation codes
//               (2-D tiled TMA, 128-byte swizzle) and their scale tiles (1-D
//               bulk copies), warp 3 the weight codes and scale tiles.  One
//               issuing thread cannot stream a stage's 54 KB as fast as the
//               MMAs consume it; two independent issuers can.
//   warp 1      allocates 512 TMEM columns; one lane issues the MMAs.  The
//               256-column tile is two 128-column accumulators and the
//               128x128x64 kind::mxf4nvf4 MMAs alternate between them:
//               back-to-back MMAs into one accumulator wait on each other,
//               two independent chains keep the tensor pipe full.
//   warp 2      one lane copies each stage's scale factors shared -> TMEM
//               (tcgen05.cp) into that stage's own TMEM buffer; copies issued
//               from a warp other than the MMA warp overlap the MMAs.
//   warps 4..11 epilogue: two warps per TMEM lane quarter, each drains 128
//               accumulator columns into registers, releases TMEM (so the next
//               tile's MMAs start), then applies alpha[n] and stores.
// No load uses cluster multicast.  Every mbarrier wait is bounded in time;
// when a wait runs out the kernel latches kStatusTimeout and unwinds.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "quantize_kernels.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;             // rows of A per tile (TMEM lanes)
constexpr int BN = 256;             // rows of W per tile (accumulator columns)
constexpr int HALF_N = 128;         // N of one MMA / one accumulator
constexpr int BK_BYTES = 128;       // 256 fp4 values of K per stage = one swizzle row
constexpr int KB_PER_STAGE = 4;     // MMA K-steps (64 values) per stage
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK_BYTES;                 // 16 KB
constexpr uint32_t B_BYTES = BN * BK_BYTES;                 // 32 KB
constexpr uint32_t SF_TILE = 512;                           // one 128-row x 4-block scale tile
constexpr uint32_t SFA_BYTES = KB_PER_STAGE * SF_TILE;      // 2 KB
constexpr uint32_t SFB_BYTES = 2 * KB_PER_STAGE * SF_TILE;  // 4 KB (two 128-row tiles)
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 54 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = BN;                            // scale buffers after the accumulator
constexpr uint32_t SF_BUF_COLS = 4 * KB_PER_STAGE + 8 * KB_PER_STAGE;  // 16 (A) + 32 (B) per stage
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int EPI_THREADS = 256;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 5120 /*barriers, alpha*/;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;           // default bound of every wait: 2 s

static_assert(SF_COL0 + STAGES * SF_BUF_COLS <= TMEM_COLS, "TMEM budget");
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");

// Instruction descriptor: dense, A/B = E2M1 (kind::mxf4nvf4 format 1),
// K-major A and B, scale format UE4M3, N = 128 (>>3), M = 128 (>>4).
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(HALF_N >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct Params {
    int32_t M, N, K;
    int32_t num_m, num_n, num_tiles;
    int32_t pair_m, pair_n, pair_tiles;  // 256 x 256 tiles of the CTA-pair kernel
    // Bytes of the activation box the single-CTA kernel loads per stage: all
    // 128 rows, or only round_up(M, 8) of them when M < 128 (decode).  The
    // stage's other rows keep stale codes; they meet only the zero or stale
    // scales of rows >= M and feed accumulator rows that are never stored.
    uint32_t a_box_bytes;
    // Split-K (single-CTA kernel, small M): work item t covers tile
    // t % num_tiles over the K steps of split t / num_tiles; with splits > 1
    // the epilogue writes alpha * acc as fp32 to partial[split][M][N] and a
    // finalize kernel adds the splits in order.
    int32_t splits;
    int32_t kt_per_split;
    float *partial;
    // the partials of a CTA's last work item go out through shared memory,
    // a row per store instruction (store_partial_staged); set for M >= 64
    int32_t staged_partials;
    // the weight producer may load before the previous kernel on the stream
    // has finished (that kernel does not write W)
    int32_t w_early;
    int32_t kb_total;    // K / 64
    int32_t kt_total;    // ceil(kb_total / 4)
    int32_t n_row_tiles; // ceil(N / 128): scale tiles of W per K-step
    uint32_t sf_box_bytes;  // bytes of one scale row-tile per stage (2 KB unless K < 256)
    uint32_t sfb_box_rows;  // scale row-tiles of W per stage load (2, or 1 when N <= 128)
    const uint8_t *sfa;
    const uint8_t *sfb;
    const float *g_a;
    const float *g_w;
    int32_t nseg;
    int32_t seg_end[kMaxSeg];
    void *out;
    int32_t out_fp32;
    int32_t vec_ok;      // rows of `out` are 16-byte aligned
    int32_t tma_out;     // bf16 output stored by TMA from swizzled staging boxes (pair kernel)
    uint32_t *status;
    // gated MLP epilogue (template flag GATED): the weight is [gate F | up F]
    // interleaved in 128-row blocks; out is h [M, F] bf16 and the largest
    // |h| (bf16 magnitude bits) is folded into *h_amax.
    int32_t F;
    uint32_t *h_amax;
    // Tile order: consecutive tiles (run at the same time by neighbouring
    // CTAs) share their A block when n_fastest, else their W block, so the
    // operand re-read for every tile column / row is the smaller one and stays
    // in L2.
    int32_t n_fastest;
    // Failure-path check: the producer issues nothing, so every consumer's
    // bounded wait runs out after wait_limit_ns and the kernel unwinds.
    int32_t inject_stall;
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ void tile_coords(const Params &p, int tile, int &m_blk, int &n_blk)
{
    if (p.n_fastest) {
        n_blk = tile % p.num_n;
        m_blk = tile / p.num_n;
    } else {
        m_blk = tile % p.num_m;
        n_blk = tile / p.num_m;
    }
}

__device__ __forceinline__ void work_item(const Params &p, int item, int &tile, int &split, int &kt0, int &kt1)
{
    split = item / p.num_tiles;
    tile = item - split * p.num_tiles;
    kt0 = split * p.kt_per_split;
    kt1 = min(kt0 + p.kt_per_split, p.kt_total);
}

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t sf_ready[STAGES];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    volatile int32_t abort_flag;
    alignas(16) float alpha[EPI_THREADS / 32][HALF_N];  // per epilogue warp, read as float4
};

static_assert(offsetof(Smem, alpha) % 16 == 0, "alpha is read as float4");

__device__ __forceinline__ void raise_timeout(Smem *sm, uint32_t *status)
{
    sm->abort_flag = 1;
    atomicOr(status, kStatusTimeout);
}

// Module segment of output column n (n < N).
__device__ __forceinline__ int column_segment(const Params &p, int32_t n)
{
    int s = 0;
#pragma unroll 1
    while (s + 1 < p.nseg && n >= p.seg_end[s])
        ++s;
    return s;
}

__device__ __forceinline__ float column_alpha(const Params &p, float ga, int32_t n)
{
    if (n >= p.N)
        return 0.0f;
    int s = 0;
#pragma unroll 1
    while (s + 1 < p.nseg && n >= p.seg_end[s])
        ++s;
    return __fmul_rn(ga, __ldg(p.g_w + s));
}

// Scale 64 accumulator columns by alpha and store them for one row.
__device__ __forceinline__ void store_64(const Params &p, const float *alpha, int32_t row, int32_t col0,
                                         const uint32_t (&v)[64])
{
    if (row >= p.M || col0 >= p.N)
        return;
    const int64_t off = static_cast<int64_t>(row) * p.N + col0;
    const bool full = p.vec_ok && (col0 + 64 <= p.N);
    if (p.out_fp32) {
        float *o = static_cast<float *>(p.out) + off;
        if (full) {
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 a = *reinterpret_cast<const float4 *>(&alpha[j]);
                *reinterpret_cast<float4 *>(o + j) =
                    make_float4(__fmul_rn(__uint_as_float(v[j]), a.x), __fmul_rn(__uint_as_float(v[j + 1]), a.y),
                                __fmul_rn(__uint_as_float(v[j + 2]), a.z), __fmul_rn(__uint_as_float(v[j + 3]), a.w));
            }
        } else {
            for (int j = 0; j < 64 && col0 + j < p.N; ++j)
                o[j] = __fmul_rn(__uint_as_float(v[j]), alpha[j]);
        }
    } else {
        __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + off;
        if (full) {
#pragma unroll
            for (int j = 0; j < 64; j += 8) {
                const float4 a0 = *reinterpret_cast<const float4 *>(&alpha[j]);
                const float4 a1 = *reinterpret_cast<const float4 *>(&alpha[j + 4]);
                __nv_bfloat162 b0 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j]), a0.x),
                                                          __fmul_rn(__uint_as_float(v[j + 1]), a0.y));
                __nv_bfloat162 b1 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j + 2]), a0.z),
                                                          __fmul_rn(__uint_as_float(v[j + 3]), a0.w));
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j + 4]), a1.x),
                                                          __fmul_rn(__uint_as_float(v[j + 5]), a1.y));
                __nv_bfloat162 b3 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j + 6]), a1.z),
                                                          __fmul_rn(__uint_as_float(v[j + 7]), a1.w));
                uint4 w;
                w.x = *reinterpret_cast<uint32_t *>(&b0);
                w.y = *reinterpret_cast<uint32_t *>(&b1);
                w.z = *reinterpret_cast<uint32_t *>(&b2);
                w.w = *reinterpret_cast<uint32_t *>(&b3);
                *reinterpret_cast<uint4 *>(o + j) = w;
            }
        } else {
            for (int j = 0; j < 64 && col0 + j < p.N; ++j)
                o[j] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(v[j]), alpha[j]));
        }
    }
}

// Split-K partial: alpha * acc for 64 columns of one row, fp32, into the
// split's [M, N] slice of p.partial.
__device__ __forceinline__ void store_partial_64(const Params &p, int split, const float *alpha, int32_t row,
                                                 int32_t col0, const uint32_t (&v)[64])
{
    if (row >= p.M || col0 >= p.N)
        return;
    float *o = p.partial + (static_cast<int64_t>(split) * p.M + row) * p.N + col0;
    if ((p.N & 3) == 0 && col0 + 64 <= p.N) {
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(&alpha[j]);
            *reinterpret_cast<float4 *>(o + j) =
                make_float4(__fmul_rn(__uint_as_float(v[j]), a.x), __fmul_rn(__uint_as_float(v[j + 1]), a.y),
                            __fmul_rn(__uint_as_float(v[j + 2]), a.z), __fmul_rn(__uint_as_float(v[j + 3]), a.w));
        }
    } else {
        for (int j = 0; j < 64 && col0 + j < p.N; ++j)
            o[j] = __fmul_rn(__uint_as_float(v[j]), alpha[j]);
    }
}

// Staging rows of store_partial_staged: 64 values + 4 of padding, so that
// the 16-byte writes of a warp spread over the shared-memory banks.
constexpr int STG_LD = 68;
constexpr uint32_t STG_WARP_BYTES = 32 * STG_LD * 4;
static_assert((EPI_THREADS / 32) * STG_WARP_BYTES <= STAGES * STAGE_BYTES, "staging rows fit in the pipeline ring");

// Split-K partial of the warp's 32 x 64 block (lane = row, v = 64
// accumulator columns), alpha * acc as fp32, through shared memory: every
// lane writes its row's values, then the warp stores the block one row at a
// time, two columns per lane, so one store instruction covers 256 contiguous
// bytes of one row instead of 16 bytes of each of 32 rows (store_partial_64).
// stg: this warp's STG_WARP_BYTES of idle shared memory; rows: valid rows
// from row0 (1..32).
__device__ __forceinline__ void store_partial_staged(const Params &p, int split, float *stg, const float *alpha,
                                                     int lane, int32_t rows, int32_t row0, int32_t col0,
                                                     const uint32_t (&v)[64])
{
    float *my = stg + lane * STG_LD;
#pragma unroll
    for (int j = 0; j < 64; j += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(&alpha[j]);
        *reinterpret_cast<float4 *>(my + j) =
            make_float4(__fmul_rn(__uint_as_float(v[j]), a.x), __fmul_rn(__uint_as_float(v[j + 1]), a.y),
                        __fmul_rn(__uint_as_float(v[j + 2]), a.z), __fmul_rn(__uint_as_float(v[j + 3]), a.w));
    }
    __syncwarp();
    const int32_t c = col0 + 2 * lane;
    const bool pairs = (p.N & 1) == 0;
    float *base = p.partial + static_cast<int64_t>(split) * p.M * p.N;
    for (int r = 0; r < rows; ++r) {
        const float2 x = *reinterpret_cast<const float2 *>(stg + r * STG_LD + 2 * lane);
        float *o = base + static_cast<int64_t>(row0 + r) * p.N + c;
        if (pairs && c + 1 < p.N) {
            *reinterpret_cast<float2 *>(o) = x;
        } else {
            if (c < p.N)
                o[0] = x.x;
            if (c + 1 < p.N)
                o[1] = x.y;
        }
    }
    __syncwarp();  // the block is read before the next one overwrites it
}

// out[m, n] = round( sum over splits s = 0, 1, ... of partial[s][m][n] ), the
// splits added in order (deterministic), bf16 round-to-nearest-even or fp32.
__global__ void __launch_bounds__(256) splitk_finalize_kernel(const float *__restrict__ partial, int32_t splits,
                                                              int64_t M, int64_t N, void *out, int32_t out_fp32)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    const int64_t total = M * N;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        float acc = partial[i];
        for (int s = 1; s < splits; ++s)
            acc = __fadd_rn(acc, partial[static_cast<int64_t>(s) * total + i]);
        if (out_fp32)
            static_cast<float *>(out)[i] = acc;
        else
            static_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(acc);
    }
}

// Store 128 bf16 values of one row (as 64 packed pairs) at [row, col0).
__device__ __forceinline__ void store_bf16_packed_128(const Params &p, int32_t row, int32_t col0,
                                                      const uint32_t (&pk)[64])
{
    if (row >= p.M || col0 >= p.N)
        return;
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + static_cast<int64_t>(row) * p.N + col0;
    if (p.vec_ok && col0 + 128 <= p.N) {
#pragma unroll
        for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<uint4 *>(o + 2 * j) = make_uint4(pk[j], pk[j + 1], pk[j + 2], pk[j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 128; ++j)
            if (col0 + j < p.N)
                o[j] = __ushort_as_bfloat16(static_cast<unsigned short>((j & 1) ? (pk[j >> 1] >> 16) : (pk[j >> 1] & 0xFFFFu)));
    }
}

// 1 / d for 1 <= d < 2^126 on the FMA pipe: a seed from the exponent and
// significand bits (within 12.5% of 1/d), then three Newton steps
// r <- r + r (1 - d r), each squaring the relative error (2e-2, 2e-4,
// 4e-8), the last one rounded: within about 1 ulp.  The SwiGLU epilogue
// evaluates one of these per h value, and the special-function unit's
// reciprocal was a tenth of the gated GEMM's time.
__device__ __forceinline__ float rcp_newton(float d)
{
    float r = __int_as_float(0x7EF311C3 - __float_as_int(d));
#pragma unroll
    for (int i = 0; i < 3; ++i)
        r = __fmaf_rn(r, __fmaf_rn(-d, r, 1.0f), r);
    return r;
}

// h = silu(g) * u, silu(g) = g / (1 + exp(-g)), in fp32.  The quotient is g
// times rcp_newton(1 + exp(-g)); g is clamped at -87 so that the divisor
// stays finite (e^87 < 2^126): below that silu(g) is under 1e-35 anyway.  The
// result is checked against the fp64 oracle with a 1e-6 relative allowance
// for fp32 evaluation before bf16 rounding.
__device__ __forceinline__ float silu_mul(float g, float u)
{
    const float gc = fmaxf(g, -87.0f);
    return __fmul_rn(__fmul_rn(gc, rcp_newton(__fadd_rn(1.0f, expf(-gc)))), u);
}

template <bool GATED>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                     const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *sm = reinterpret_cast<Smem *>(smem + STAGES * STAGE_BYTES);
    const uint32_t smem_base = smem_u32(smem);
    auto a_smem = [&](int s) { return smem_base + s * STAGE_BYTES; };
    auto b_smem = [&](int s) { return smem_base + s * STAGE_BYTES + A_BYTES; };
    auto sfa_smem = [&](int s) { return smem_base + s * STAGE_BYTES + A_BYTES + B_BYTES; };
    auto sfb_smem = [&](int s) { return smem_base + s * STAGE_BYTES + A_BYTES + B_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm->full[s]), 2);  // one arrival per producer warp
            mbar_init(smem_u32(&sm->empty[s]), 1);
            mbar_init(smem_u32(&sm->sf_ready[s]), 1);
        }
        mbar_init(smem_u32(&sm->acc_full), 1);
        mbar_init(smem_u32(&sm->acc_empty), EPI_THREADS / 32);
        mbar_init(smem_u32(&sm->drain), 1);
        sm->abort_flag = 0;
        fence_mbarrier_init();
    }
    if ((warp == 0 || warp == 3) && lane == 0) {
        prefetch_tensormap(warp == 0 ? &tmA : &tmB);
        prefetch_tensormap(warp == 0 ? &tmSFA : &tmSFB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    // set-up above touches no global memory; from here on the previous
    // kernel's outputs (the quantized activation) are read.  With w_early the
    // weight producer skips the wait: the kernel before this one does not
    // write W, and everything before that kernel had completed when it
    // allowed this launch, so the weights stream in while it finishes.
    if (!(p.w_early && warp == 3)) {
        grid_dep_wait();
        grid_dep_launch_dependents();
    }

    if (warp == 0 || warp == 3) {
        // ----------------------------------------------------- producers
        // Two warps share the loads of a stage: warp 0 the activation tile and
        // its scales, warp 3 the weight tile and its scales.  One thread's
        // stream of TMA instructions is slower than the stage's bytes need;
        // two independent issuers double it.  Each arrives once on the
        // stage's full barrier with its own byte count.
        const bool w_side = (warp == 3);
        if (lane == 0 && !p.inject_stall) {
            int stage = 0;
            uint32_t phase = 0;
            for (int item = blockIdx.x; item < p.num_tiles * p.splits && !sm->abort_flag; item += gridDim.x) {
                int tile, split, kt0, kt1, m_blk, n_blk;
                work_item(p, item, tile, split, kt0, kt1);
                tile_coords(p, tile, m_blk, n_blk);
                const int m0 = m_blk * BM, n0 = n_blk * BN;
                const int rb0 = n0 >> 7;  // first 128-row scale tile of W
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->empty[stage]), phase ^ 1u, p.wait_limit_ns)) {
                        raise_timeout(sm, p.status);
                        break;
                    }
                    // Scale tiles come as 2-D boxes of 8-byte elements over the
                    // [row tile][K/64 x 512 B] scale array: one instruction for
                    // the stage's 4 K-steps (both W row tiles at once).  A box
                    // reaching past the last K-step or row tile is zero-filled and
                    // still counts its full size.
                    const uint32_t bar = smem_u32(&sm->full[stage]);
                    const int32_t sf_x = kt * KB_PER_STAGE * (SF_TILE / 8);
                    if (!w_side) {
                        mbar_arrive_expect_tx(bar, p.a_box_bytes + p.sf_box_bytes);
                        tma_load_2d(a_smem(stage), &tmA, kt * BK_BYTES, m0, bar);
                        tma_load_2d(sfa_smem(stage), &tmSFA, sf_x, m_blk, bar);
                    } else {
                        mbar_arrive_expect_tx(bar, B_BYTES + p.sf_box_bytes * p.sfb_box_rows);
                        tma_load_2d(b_smem(stage), &tmB, kt * BK_BYTES, n0, bar);
                        tma_load_2d(sfb_smem(stage), &tmSFB, sf_x, rb0, bar);
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            // Operand descriptors of stage 0; a stage adds STAGE_BYTES and a
            // K-step 32 bytes to the 14-bit start-address field (shared
            // addresses stay below 2^18, so it never carries).  Computing them
            // once keeps the gap between two stages' MMAs short.
            const uint64_t adesc0 = smem_desc(a_smem(0), 16, 1024, 2);
            const uint64_t bdesc0 = smem_desc(b_smem(0), 16, 1024, 2);
            constexpr uint32_t HALF_B = (HALF_N * BK_BYTES) >> 4;  // second 128 rows of W
            for (int item = blockIdx.x; item < p.num_tiles * p.splits && !sm->abort_flag;
                 item += gridDim.x, ++local) {
                int tile, split, kt0, kt1;
                work_item(p, item, tile, split, kt0, kt1);
                if (!mbar_wait_bounded(smem_u32(&sm->acc_empty), (local & 1) ^ 1u, p.wait_limit_ns)) {
                    raise_timeout(sm, p.status);
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->full[stage]), phase, p.wait_limit_ns) ||
                        !mbar_wait_bounded(smem_u32(&sm->sf_ready[stage]), phase, p.wait_limit_ns)) {
                        raise_timeout(sm, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(KB_PER_STAGE, p.kb_total - kt * KB_PER_STAGE);
                    const uint32_t sfa_t = tmem + SF_COL0 + stage * SF_BUF_COLS;
                    const uint32_t sfb_t = sfa_t + 4 * KB_PER_STAGE;
                    const uint32_t soff = (static_cast<uint32_t>(stage) * STAGE_BYTES) >> 4;
                    const uint64_t ad = adesc0 + soff, bd = bdesc0 + soff;
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint32_t acc_flag = (kt > kt0 || kb > 0) ? 1u : 0u;
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_mma_nvf4(tmem + h * HALF_N, ad + 2 * kb, bd + h * HALF_B + 2 * kb, IDESC,
                                        sfa_t + kb * 4, sfb_t + kb * 8 + h * 4, acc_flag);
                    }
                    tc_commit(smem_u32(&sm->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(smem_u32(&sm->acc_full));
            }
            // let every tcgen05 operation this thread issued finish before TMEM is freed
            tc_commit(smem_u32(&sm->drain));
            if (!mbar_wait_bounded(smem_u32(&sm->drain), 0, p.wait_limit_ns))
                raise_timeout(sm, p.status);
        }
    } else if (warp == 2) {
        // ------------------------------------- scale factors -> TMEM
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int item = blockIdx.x; item < p.num_tiles * p.splits && !sm->abort_flag; item += gridDim.x) {
                int tile, split, kt0, kt1;
                work_item(p, item, tile, split, kt0, kt1);
                bool ok = true;
                for (int kt = kt0; kt < kt1; ++kt) {
                    // The stage's TMEM scale buffer is free: the producer only refilled this
                    // stage after the MMAs that read the buffer last time had completed.
                    if (!mbar_wait_bounded(smem_u32(&sm->full[stage]), phase, p.wait_limit_ns)) {
                        raise_timeout(sm, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(KB_PER_STAGE, p.kb_total - kt * KB_PER_STAGE);
                    const uint32_t sfa_t = tmem + SF_COL0 + stage * SF_BUF_COLS;
                    const uint32_t sfb_t = sfa_t + 4 * KB_PER_STAGE;
                    for (int kb = 0; kb < nkb; ++kb) {
                        tc_cp_32x128b_x4(sfa_t + kb * 4, smem_desc(sfa_smem(stage) + kb * SF_TILE, 0, 128, 0));
                        tc_cp_32x128b_x4(sfb_t + kb * 8, smem_desc(sfb_smem(stage) + kb * SF_TILE, 0, 128, 0));
                        tc_cp_32x128b_x4(sfb_t + kb * 8 + 4,
                                         smem_desc(sfb_smem(stage) + p.sf_box_bytes + kb * SF_TILE, 0, 128, 0));
                    }
                    tc_commit(smem_u32(&sm->sf_ready[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
            }
        }
    } else if (warp >= EPI_WARP0 && GATED) {
        // ------------------------------------------- gated MLP epilogue
        // Tile columns [0, 128) are gate rows and [128, 256) the matching up
        // rows; each warp takes 64 of the tile's 128 h columns for its lane quarter.
        const int q = warp & 3;
        const int hc = (warp - EPI_WARP0) >> 2;
        const float ga = __ldg(p.g_a);
        const float a_gate = __fmul_rn(ga, __ldg(p.g_w));
        const float a_up = __fmul_rn(ga, __ldg(p.g_w + 1));
        uint32_t hmax = 0;
        int local = 0;
        for (int item = blockIdx.x; item < p.num_tiles * p.splits && !sm->abort_flag; item += gridDim.x, ++local) {
            int tile, split, kt0, kt1, m_blk, n_blk;
            work_item(p, item, tile, split, kt0, kt1);  // the gated path never splits K
            tile_coords(p, tile, m_blk, n_blk);
            const int m0 = m_blk * BM, n0 = n_blk * BN;
            const bool ok = mbar_wait_bounded(smem_u32(&sm->acc_full), local & 1, p.wait_limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                if (lane == 0)
                    raise_timeout(sm, p.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + hc * 64;
            uint32_t vg[64], vu[64];
            tc_ld_32x32b_x64(taddr, vg);
            tc_ld_32x32b_x64(taddr + HALF_N, vu);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm->acc_empty));
            const int row = m0 + q * 32 + lane;
            const int col0 = (n0 >> 1) + hc * 64;  // h column
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float h0 = silu_mul(__fmul_rn(__uint_as_float(vg[2 * j]), a_gate),
                                          __fmul_rn(__uint_as_float(vu[2 * j]), a_up));
                const float h1 = silu_mul(__fmul_rn(__uint_as_float(vg[2 * j + 1]), a_gate),
                                          __fmul_rn(__uint_as_float(vu[2 * j + 1]), a_up));
                __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
                pk[j] = *reinterpret_cast<uint32_t *>(&b);
            }
            if (row < p.M && col0 < p.F) {
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + static_cast<int64_t>(row) * p.F + col0;
                const int nval = min(64, p.F - col0);
                if (p.vec_ok && nval == 64) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<uint4 *>(o + 2 * j) = make_uint4(pk[j], pk[j + 1], pk[j + 2], pk[j + 3]);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        hmax = vmax_mag(hmax, pk[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        if (j < nval) {
                            const uint32_t hb = (j & 1) ? (pk[j >> 1] >> 16) : (pk[j >> 1] & 0xFFFFu);
                            o[j] = __ushort_as_bfloat16(static_cast<unsigned short>(hb));
                            hmax = vmax_mag(hmax, hb);
                        }
                    }
                }
            }
        }
        uint32_t v = hmax16(hmax);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0 && v != 0)
            atomicMax(p.h_amax, v);
    } else if (warp >= EPI_WARP0) {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter this warp may access
        const int hc = (warp - EPI_WARP0) >> 2;    // which 128-column half of the tile
        float *alpha = sm->alpha[warp - EPI_WARP0];
        const float ga = __ldg(p.g_a);
        int local = 0;
        for (int item = blockIdx.x; item < p.num_tiles * p.splits && !sm->abort_flag; item += gridDim.x, ++local) {
            int tile, split, kt0, kt1, m_blk, n_blk;
            work_item(p, item, tile, split, kt0, kt1);
            tile_coords(p, tile, m_blk, n_blk);
            const int m0 = m_blk * BM, n0 = n_blk * BN;
            __syncwarp();  // this warp's reads of the previous tile's alpha are done
#pragma unroll
            for (int j = 0; j < HALF_N / 32; ++j)
                alpha[lane + 32 * j] = column_alpha(p, ga, n0 + hc * HALF_N + lane + 32 * j);
            __syncwarp();
            // every lane waits (bounded); the vote keeps the warp's decision uniform
            const bool ok = mbar_wait_bounded(smem_u32(&sm->acc_full), local & 1, p.wait_limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                if (lane == 0)
                    raise_timeout(sm, p.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + hc * HALF_N;
            uint32_t v0[64], v1[64];
            tc_ld_32x32b_x64(taddr, v0);
            tc_ld_32x32b_x64(taddr + 64, v1);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&sm->acc_empty));
            const int row = m0 + q * 32 + lane;
            const int col0 = n0 + hc * HALF_N;
            const int rows = min(32, p.M - (m0 + q * 32));
            if (p.splits > 1 && p.staged_partials && item + static_cast<int>(gridDim.x) >= p.num_tiles * p.splits) {
                // This CTA's last work item: its MMAs are complete (acc_full) and the
                // producers have nothing left to load, so the pipeline ring is idle
                // and holds each warp's staging rows.
                float *stg = reinterpret_cast<float *>(smem + (warp - EPI_WARP0) * STG_WARP_BYTES);
                if (rows > 0 && col0 < p.N) {
                    store_partial_staged(p, split, stg, alpha, lane, rows, m0 + q * 32, col0, v0);
                    store_partial_staged(p, split, stg, alpha + 64, lane, rows, m0 + q * 32, col0 + 64, v1);
                }
            } else if (p.splits > 1) {
                store_partial_64(p, split, alpha, row, col0, v0);
                store_partial_64(p, split, alpha + 64, row, col0 + 64, v1);
            } else {
                store_64(p, alpha, row, n0 + hc * HALF_N, v0);
                store_64(p, alpha + 64, row, n0 + hc * HALF_N + 64, v1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace nvfp4
