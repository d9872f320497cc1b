// gemm_kernel.cuh -- persistent, warp-specialized NVFP4 x NVFP4 GEMM for
// sm_100a on the 5th-generation tensor cores, with the per-module
// global-scale epilogue of a fused-module linear layer.
//
//   out[m, n] = round( acc[m, n] * fl32(g_a * g_w[seg(n)]) )
//   acc[m, n] = sum_k qa[m,k] sa[m,k/16] qw[n,k] sw[n,k/16]   (fp32, TMEM)
//
// The block-scaled product runs "natively on current tensor cores" ("Why
// Gated DeltaNet Survives 4-Bit Quantization", kipquest.com, "The deep
// dive"); applying each module's own FP32 global scale to its columns is the
// repair of the global-scale mismatch that appears when per-module-calibrated
// checkpoints are served by a kernel that fuses those modules into one GEMM
// (same page, "The abstract" and "The deep dive").
//
// Structure (one CTA per SM, 6 warps):
//   warp 0      TMA producer: codes tiles by 2-D tiled TMA (128-byte swizzle),
//               scale-factor tiles by 1-D bulk copies, into a 4-stage ring.
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.cp for the
//               scale factors and tcgen05.mma (kind::mxf4nvf4, 128x192x64 per
//               instruction) and commits stage / accumulator barriers.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, x alpha[n],
//               bf16 (or fp32) stores.  Two accumulator buffers in TMEM let the
//               epilogue of tile i overlap the main loop of tile i+1.
// No load uses cluster multicast.  Every mbarrier wait is bounded in time;
// when a wait runs out the kernel latches kStatusTimeout and unwinds.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "quantize_kernels.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;            // rows of A per tile (TMEM lanes)
constexpr int BN = 192;            // rows of W per tile (accumulator columns)
constexpr int BK_BYTES = 128;      // 256 fp4 values of K per stage = one swizzle row
constexpr int KB_PER_STAGE = 4;    // MMA K-steps (64 values) per stage
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK_BYTES;                 // 16 KB
constexpr uint32_t B_BYTES = BN * BK_BYTES;                 // 24 KB
constexpr uint32_t SFA_BYTES = KB_PER_STAGE * 512;          // one 128-row scale tile per K-step
constexpr uint32_t SFB_BYTES = 2 * KB_PER_STAGE * 512;      // two 128-row scale tiles per K-step
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 46 KB, 1024-aligned
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = 2 * BN;                        // scale factors after both accumulators
constexpr uint32_t SF_BUF_COLS = 4 * KB_PER_STAGE + 8 * KB_PER_STAGE;  // 16 (A) + 32 (B)
constexpr int NUM_THREADS = 192;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;           // 2 s per wait

static_assert(SF_COL0 + 2 * SF_BUF_COLS <= TMEM_COLS, "TMEM budget");
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");

// Instruction descriptor: dense, A/B = E2M1 (kind::mxf4nvf4 format 1),
// K-major A and B, scale format UE4M3, N = 192 (>>3), M = 128 (>>4).
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct Params {
    int32_t M, N, K;
    int32_t num_m, num_n, num_tiles;
    int32_t kb_total;    // K / 64
    int32_t kt_total;    // ceil(kb_total / 4)
    int32_t n_row_tiles; // ceil(N / 128): scale tiles of W per K-step
    const uint8_t *sfa;
    const uint8_t *sfb;
    const float *g_a;
    const float *g_w;
    int32_t nseg;
    int32_t seg_end[kMaxSeg];
    void *out;
    int32_t out_fp32;
    int32_t vec_ok;      // rows of `out` are 16-byte aligned
    uint32_t *status;
};

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int32_t abort_flag;
};

__device__ __forceinline__ void raise_timeout(Smem *sm, uint32_t *status)
{
    sm->abort_flag = 1;
    atomicOr(status, kStatusTimeout);
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

__device__ __forceinline__ void store_chunk(const Params &p, int32_t row, int32_t col0, const float (&f)[32])
{
    if (row >= p.M)
        return;
    const int64_t off = static_cast<int64_t>(row) * p.N + col0;
    const bool full = p.vec_ok && (col0 + 32 <= p.N);
    if (p.out_fp32) {
        float *o = static_cast<float *>(p.out) + off;
        if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4 *>(o + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
        } else {
            for (int j = 0; j < 32 && col0 + j < p.N; ++j)
                o[j] = f[j];
        }
    } else {
        __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + off;
        if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
                uint4 v;
                __nv_bfloat162 b0 = __floats2bfloat162_rn(f[j], f[j + 1]);
                __nv_bfloat162 b1 = __floats2bfloat162_rn(f[j + 2], f[j + 3]);
                __nv_bfloat162 b2 = __floats2bfloat162_rn(f[j + 4], f[j + 5]);
                __nv_bfloat162 b3 = __floats2bfloat162_rn(f[j + 6], f[j + 7]);
                v.x = *reinterpret_cast<uint32_t *>(&b0);
                v.y = *reinterpret_cast<uint32_t *>(&b1);
                v.z = *reinterpret_cast<uint32_t *>(&b2);
                v.w = *reinterpret_cast<uint32_t *>(&b3);
                *reinterpret_cast<uint4 *>(o + j) = v;
            }
        } else {
            for (int j = 0; j < 32 && col0 + j < p.N; ++j)
                o[j] = __float2bfloat16_rn(f[j]);
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
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
            mbar_init(smem_u32(&sm->full[s]), 1);
            mbar_init(smem_u32(&sm->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sm->acc_full[b]), 1);
            mbar_init(smem_u32(&sm->acc_empty[b]), 4);
        }
        mbar_init(smem_u32(&sm->drain), 1);
        sm->abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && !sm->abort_flag; tile += gridDim.x) {
                const int m_blk = tile % p.num_m, n_blk = tile / p.num_m;
                const int m0 = m_blk * BM, n0 = n_blk * BN;
                const int rb0 = n0 >> 7;
                const int nb_tiles = (rb0 + 1 < p.n_row_tiles) ? 2 : 1;
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->empty[stage]), phase ^ 1u, WAIT_LIMIT_NS)) {
                        raise_timeout(sm, p.status);
                        break;
                    }
                    const int nkb = min(KB_PER_STAGE, p.kb_total - kt * KB_PER_STAGE);
                    const uint32_t sf_bytes = nkb * 512u;
                    const uint32_t bar = smem_u32(&sm->full[stage]);
                    mbar_arrive_expect_tx(bar, A_BYTES + B_BYTES + sf_bytes * (1 + nb_tiles));
                    tma_load_2d(a_smem(stage), &tmA, kt * BK_BYTES, m0, bar);
                    tma_load_2d(b_smem(stage), &tmB, kt * BK_BYTES, n0, bar);
                    bulk_load(sfa_smem(stage),
                              p.sfa + (static_cast<int64_t>(m_blk) * p.kb_total + kt * KB_PER_STAGE) * 512,
                              sf_bytes, bar);
                    for (int j = 0; j < nb_tiles; ++j)
                        bulk_load(sfb_smem(stage) + j * (KB_PER_STAGE * 512),
                                  p.sfb + (static_cast<int64_t>(rb0 + j) * p.kb_total + kt * KB_PER_STAGE) * 512,
                                  sf_bytes, bar);
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
            uint32_t sf_buf = 0;
            int local = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && !sm->abort_flag; tile += gridDim.x, ++local) {
                const int n0 = (tile / p.num_m) * BN;
                const uint32_t sfb_shift = (n0 & 127) >> 5;  // 0 or 2 columns: first W row of the tile
                const int acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait_bounded(smem_u32(&sm->acc_empty[acc]), acc_phase ^ 1u, WAIT_LIMIT_NS)) {
                    raise_timeout(sm, p.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * BN;
                bool ok = true;
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->full[stage]), phase, WAIT_LIMIT_NS)) {
                        raise_timeout(sm, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(KB_PER_STAGE, p.kb_total - kt * KB_PER_STAGE);
                    const uint32_t sfa_t = tmem + SF_COL0 + sf_buf * SF_BUF_COLS;
                    const uint32_t sfb_t = sfa_t + 4 * KB_PER_STAGE;
                    sf_buf ^= 1u;
                    for (int kb = 0; kb < nkb; ++kb) {
                        tc_cp_32x128b_x4(sfa_t + kb * 4, smem_desc(sfa_smem(stage) + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_x4(sfb_t + kb * 8, smem_desc(sfb_smem(stage) + kb * 512, 0, 128, 0));
                        tc_cp_32x128b_x4(sfb_t + kb * 8 + 4,
                                         smem_desc(sfb_smem(stage) + KB_PER_STAGE * 512 + kb * 512, 0, 128, 0));
                    }
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t adesc = smem_desc(a_smem(stage) + kb * 32, 16, 1024, 2);
                        const uint64_t bdesc = smem_desc(b_smem(stage) + kb * 32, 16, 1024, 2);
                        tc_mma_nvf4(d_tmem, adesc, bdesc, IDESC, sfa_t + kb * 4, sfb_t + kb * 8 + sfb_shift,
                                    (kt > 0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&sm->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(smem_u32(&sm->acc_full[acc]));
            }
            // let every tcgen05 operation this thread issued finish before TMEM is freed
            tc_commit(smem_u32(&sm->drain));
            if (!mbar_wait_bounded(smem_u32(&sm->drain), 0, WAIT_LIMIT_NS))
                raise_timeout(sm, p.status);
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const float ga = __ldg(p.g_a);
        int local = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles && !sm->abort_flag; tile += gridDim.x, ++local) {
            const int m0 = (tile % p.num_m) * BM, n0 = (tile / p.num_m) * BN;
            const int acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            if (!mbar_wait_bounded(smem_u32(&sm->acc_full[acc]), acc_phase, WAIT_LIMIT_NS)) {
                raise_timeout(sm, p.status);
                break;
            }
            tc_fence_after();
            const int row = m0 + q * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tc_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c * 32, v);
                tc_wait_ld();
                if (c == BN / 32 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(smem_u32(&sm->acc_empty[acc]));
                }
                const int col0 = n0 + c * 32;
                const float al = column_alpha(p, ga, col0 + lane);
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    f[j] = __fmul_rn(__uint_as_float(v[j]), __shfl_sync(0xFFFFFFFFu, al, j));
                store_chunk(p, row, col0, f);
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
