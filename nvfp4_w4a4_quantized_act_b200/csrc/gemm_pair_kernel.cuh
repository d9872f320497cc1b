// gemm_pair_kernel.cuh -- the NVFP4 x NVFP4 GEMM of gemm_kernel.cuh on CTA
// pairs: a cluster of two CTAs on neighbouring SMs computes a 256 x 256 tile
// with tcgen05.mma.cta_group::2 (M = 256: 128 rows of A from each CTA; the
// tile's 256 rows of W split 128/128 between the two CTAs' shared memory).
// Each SM therefore stages only half of the W tile, and one MMA instruction
// covers the work of two 128 x 128 single-CTA MMAs.
//
//   out[m, n] = round( acc[m, n] * fl32(g_a * g_w[seg(n)]) )     (same math,
//   same epilogue and same gated-MLP variant as the single-CTA kernel)
//
// Per CTA, 16 warps:
//   warp 0      A producer: this CTA's 128 x 256-value A box per stage
//   warp 3      W producer: this CTA's 128 x 256-value half of the W box
//               Both are pair-form TMA loads completing on the LEADER's full
//               barrier, which therefore counts the bytes of both CTAs.
//   warp 2      scale producer: the stage's A scale tile (this CTA's rows)
//               and both W scale tiles (all 256 columns: every CTA's MMA
//               half reads the scales of the whole N range), pair-form loads
//               completing on the leader's sf_full barrier, into a scale ring
//               twice as deep as the code ring: a scale slot is free again
//               once its scales are in TMEM, so scales arrive stages ahead of
//               the codes.
//   warp 1      TMEM allocation (both CTAs, cta_group::2); in the leader one
//               lane issues the pair MMAs (4 per stage, 256 x 256 x 64) and
//               releases each stage in both CTAs with one commit fan-out.
//   warps 4..7  scale copiers (leader only): warp 4 + kb copies K-step kb's A
//               tile and both W tiles into both CTAs' TMEM (pair-mode
//               tcgen05.cp reads each CTA's own shared memory) and commits to
//               the stage's full barrier.  While MMAs occupy the tensor pipe a copy takes its
//               issuing thread about 70 cycles; twelve per stage from one
//               thread (or from the MMA thread itself) would outlast the
//               stage's MMAs, four threads overlap them.
//   warps 8..15 epilogue: this CTA's 128 rows x 256 columns, two warps per
//               lane quarter; each converts its 128 columns to bf16 as it
//               loads them (one scalar scale when the slice lies in one
//               module segment), releases TMEM, then writes 32 x 64 boxes
//               into a 128-byte-swizzled staging buffer that one TMA store
//               per box copies out.  (A thread per output row storing its own
//               16-byte pieces took longer than the next tile's mainloop.)
// No load uses cluster multicast.  Every mbarrier wait is bounded; a wait
// that runs out latches kStatusTimeout and the kernel unwinds (the other CTA
// of the pair runs out of its own bounded waits).
#pragma once

#include "gemm_kernel.cuh"

namespace nvfp4 {
namespace gemm {
namespace pair {

constexpr int PAIR_M = 256;                               // rows of A per pair tile
constexpr int PAIR_N = 256;                               // rows of W per pair tile
constexpr int STAGES = 5;
constexpr uint32_t A_BYTES = 128 * BK_BYTES;              // 16 KB: this CTA's rows
constexpr uint32_t B_BYTES = 128 * BK_BYTES;              // 16 KB: this CTA's half of W
constexpr uint32_t SFA_BYTES = KB_PER_STAGE * SF_TILE;    // 2 KB
constexpr uint32_t SFB_BYTES = 2 * KB_PER_STAGE * SF_TILE;// 4 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;      // 32 KB of codes per stage
// Scale tiles have their own ring: a slot is free again as soon as its
// copies into TMEM are done, long before the MMAs free the codes' stage, so
// the scale loads run ahead of the codes.
constexpr int SF_SLOTS = STAGES;
constexpr uint32_t SF_SLOT_BYTES = SFA_BYTES + SFB_BYTES; // 6 KB
constexpr uint32_t STAGING_BYTES = 32 * 128;             // per epilogue warp: 32 rows x 128 B (64 bf16)
constexpr uint32_t SF_COL0 = PAIR_N;                      // scale buffers after the accumulator
constexpr uint32_t SF_BUF_COLS = 16 + 32;                 // per stage: A 4 x 4, W 4 x 8 columns
constexpr int NUM_THREADS = 512;
constexpr int WRITER_WARP0 = 4;
constexpr int EPI_WARP0 = 8;
constexpr int EPI_WARPS = 8;
constexpr uint32_t SF_READY_COUNT = KB_PER_STAGE;         // one commit per copier warp
// full[stage]: the leader's A and W producers (arrive with the stage's byte
// count) and the four copier warps (commit once their copies are done).  One
// barrier per stage: a satisfied mbarrier wait still costs the MMA thread
// ~70 cycles, and the pipe holds only about one MMA of queued work.
constexpr uint32_t FULL_COUNT = 2 + SF_READY_COUNT;
constexpr uint32_t ACC_EMPTY_COUNT = 2 * EPI_WARPS;       // epilogue warps of both CTAs

static_assert(SF_COL0 + STAGES * SF_BUF_COLS <= TMEM_COLS, "TMEM budget");
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment for the 128-byte swizzle");

// Instruction descriptor: kind::mxf4nvf4, E2M1 A/B, UE4M3 scales, K-major,
// N = 256 (>>3), M = 256 (>>4, the pair's rows).
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (uint32_t(PAIR_N >> 3) << 17) | (uint32_t(PAIR_M >> 4) << 24);

struct Smem {
    uint64_t full[STAGES];      // leader: A and W boxes of both CTAs and the stage's scales in TMEM
    uint64_t empty[STAGES];     // each CTA: stage consumed (MMA commit fan-out)
    uint64_t sf_full[SF_SLOTS]; // leader: both CTAs' scale boxes landed
    uint64_t sf_empty[SF_SLOTS];// each CTA: scale slot copied (copier commit fan-out)
    uint64_t acc_full;          // each CTA: accumulator complete (commit fan-out)
    uint64_t acc_empty;         // leader: both CTAs' epilogues drained TMEM
    uint64_t drain;             // leader: every MMA finished before teardown
    uint32_t tmem_base;
    volatile int32_t abort_flag;
    alignas(16) float alpha[EPI_WARPS][64];  // read as float4
};

constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + EPI_WARPS * STAGING_BYTES +
                                1024 /*align*/ + ((sizeof(Smem) + 1023) / 1024) * 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
static_assert(offsetof(Smem, alpha) % 16 == 0, "alpha is read as float4");
static_assert((STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES) % 1024 == 0, "staging boxes need 1024-byte alignment");

// Write 32 packed bf16 pairs (64 values of row `lane`) into a 32 x 128 B
// staging box in the 128-byte-swizzled layout the output tensor map uses:
// 16-byte chunk k of row r lives at r * 128 + ((k ^ (r % 8)) * 16).
__device__ __forceinline__ void stage_row_swizzled(uint32_t box, int lane, const uint32_t *pk)
{
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t a = box + lane * 128 + (((k ^ (lane & 7)) & 7) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * k]), "r"(pk[4 * k + 1]),
                     "r"(pk[4 * k + 2]), "r"(pk[4 * k + 3])
                     : "memory");
    }
}

__device__ __forceinline__ void pair_tile_coords(const Params &p, int tile, int &mp, int &np)
{
    if (p.n_fastest) {
        np = tile % p.pair_n;
        mp = tile / p.pair_n;
    } else {
        mp = tile % p.pair_m;
        np = tile / p.pair_m;
    }
}

__device__ __forceinline__ void raise_timeout_pair(Smem *sm, uint32_t *status)
{
    sm->abort_flag = 1;
    atomicOr(status, kStatusTimeout);
}

template <bool GATED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                          const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *sm = reinterpret_cast<Smem *>(smem + STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES +
                                        EPI_WARPS * STAGING_BYTES);
    const uint32_t smem_base = smem_u32(smem);
    const uint32_t sf_base = smem_base + STAGES * STAGE_BYTES;
    // epilogue staging for TMA stores: one 1024-aligned 4 KB box per warp
    const uint32_t stage_out_base = sf_base + SF_SLOTS * SF_SLOT_BYTES;
    auto a_smem = [&](int s) { return smem_base + s * STAGE_BYTES; };
    auto b_smem = [&](int s) { return smem_base + s * STAGE_BYTES + A_BYTES; };
    auto sfa_smem = [&](int j) { return sf_base + j * SF_SLOT_BYTES; };
    auto sfb_smem = [&](int j) { return sf_base + j * SF_SLOT_BYTES + SFA_BYTES; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(cluster_count_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm->full[s]), FULL_COUNT);
            mbar_init(smem_u32(&sm->empty[s]), 1);
        }
        for (int j = 0; j < SF_SLOTS; ++j) {
            mbar_init(smem_u32(&sm->sf_full[j]), 1);
            mbar_init(smem_u32(&sm->sf_empty[j]), SF_READY_COUNT);  // one commit per copier warp
        }
        mbar_init(smem_u32(&sm->acc_full), 1);
        mbar_init(smem_u32(&sm->acc_empty), ACC_EMPTY_COUNT);
        mbar_init(smem_u32(&sm->drain), 1);
        sm->abort_flag = 0;
        fence_mbarrier_init();
    }
    if (lane == 0) {
        if (warp == 0)
            prefetch_tensormap(&tmA);
        else if (warp == 3)
            prefetch_tensormap(&tmB);
        else if (warp == 2) {
            prefetch_tensormap(&tmSFA);
            prefetch_tensormap(&tmSFB);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&sm->tmem_base), TMEM_COLS);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised and both TMEM bases known before any
    // cross-CTA arrival or load
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    // set-up above touches no global memory
    grid_dep_wait();
    grid_dep_launch_dependents();
    const uint32_t tmem = sm->tmem_base;
    auto leader_bar = [&](uint64_t *b) { return mapa_shared(smem_u32(b), 0); };

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------ code producers
        const bool w_side = (warp == 3);
        if (lane == 0 && !p.inject_stall) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl) {
                int mp, np;
                pair_tile_coords(p, tile, mp, np);
                const int y = (w_side ? np * PAIR_N : mp * PAIR_M) + static_cast<int>(rank) * 128;
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->empty[stage]), phase ^ 1u, p.wait_limit_ns)) {
                        raise_timeout_pair(sm, p.status);
                        break;
                    }
                    if (leader)
                        mbar_arrive_expect_tx(smem_u32(&sm->full[stage]), 2 * (w_side ? B_BYTES : A_BYTES));
                    tma_load_2d_pair(w_side ? b_smem(stage) : a_smem(stage), w_side ? &tmB : &tmA, kt * BK_BYTES, y,
                                     leader_bar(&sm->full[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 2) {
        // ----------------------------------------------- scale producer
        if (lane == 0 && !p.inject_stall) {
            int slot = 0;
            uint32_t sphase = 0;
            const uint32_t sf_bytes = p.sf_box_bytes * (1u + p.sfb_box_rows);
            for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl) {
                int mp, np;
                pair_tile_coords(p, tile, mp, np);
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    if (!mbar_wait_bounded(smem_u32(&sm->sf_empty[slot]), sphase ^ 1u, p.wait_limit_ns)) {
                        raise_timeout_pair(sm, p.status);
                        break;
                    }
                    const int32_t sf_x = kt * KB_PER_STAGE * (SF_TILE / 8);
                    const uint32_t bar = leader_bar(&sm->sf_full[slot]);
                    if (leader)
                        mbar_arrive_expect_tx(smem_u32(&sm->sf_full[slot]), 2 * sf_bytes);
                    tma_load_2d_pair(sfa_smem(slot), &tmSFA, sf_x, mp * 2 + static_cast<int>(rank), bar);
                    tma_load_2d_pair(sfb_smem(slot), &tmSFB, sf_x, np * 2, bar);
                    if (++slot == SF_SLOTS) {
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------- MMA issuer (leader only)
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            // Operand descriptors of stage 0; a stage adds STAGE_BYTES and a
            // K-step 32 bytes to the 14-bit start-address field (shared
            // addresses stay below 2^18, so the field never carries).  Kept
            // out of the gap between one stage's last MMA and the next
            // stage's first, where the tensor pipe has at most one MMA queued.
            const uint64_t adesc0 = smem_desc(a_smem(0), 16, 1024, 2);
            const uint64_t bdesc0 = smem_desc(b_smem(0), 16, 1024, 2);
            const uint32_t full0 = smem_u32(&sm->full[0]), empty0 = smem_u32(&sm->empty[0]);
            const int kt_whole = p.kb_total / KB_PER_STAGE;  // stages with all four K-steps
            for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl, ++local) {
                if (!mbar_wait_bounded_cluster(smem_u32(&sm->acc_empty), (local & 1) ^ 1u, p.wait_limit_ns)) {
                    raise_timeout_pair(sm, p.status);
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    const uint32_t soff = (static_cast<uint32_t>(stage) * STAGE_BYTES) >> 4;
                    const uint64_t ad = adesc0 + soff, bd = bdesc0 + soff;
                    const uint32_t sf_t = tmem + SF_COL0 + stage * SF_BUF_COLS;
                    const uint32_t acc0 = kt > 0 ? 1u : 0u;
                    // codes of both CTAs landed and the stage's scales are in TMEM
                    if (!mbar_wait_bounded(full0 + 8u * stage, phase, p.wait_limit_ns)) {
                        raise_timeout_pair(sm, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (kt < kt_whole) {
#pragma unroll
                        for (int kb = 0; kb < KB_PER_STAGE; ++kb)
                            tc_mma_pair_nvf4(tmem, ad + 2 * kb, bd + 2 * kb, IDESC, sf_t + kb * 4, sf_t + 16 + kb * 8,
                                             kb > 0 ? 1u : acc0);
                    } else {
                        const int nkb = p.kb_total - kt * KB_PER_STAGE;
                        for (int kb = 0; kb < nkb; ++kb)
                            tc_mma_pair_nvf4(tmem, ad + 2 * kb, bd + 2 * kb, IDESC, sf_t + kb * 4, sf_t + 16 + kb * 8,
                                             kb > 0 ? 1u : acc0);
                    }
                    tc_commit_pair_both(empty0 + 8u * stage, 3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit_pair_both(smem_u32(&sm->acc_full), 3);
            }
            // every MMA this thread issued has finished before TMEM is freed
            tc_commit_pair(smem_u32(&sm->drain));
            if (!mbar_wait_bounded(smem_u32(&sm->drain), 0, p.wait_limit_ns))
                raise_timeout_pair(sm, p.status);
        }
    } else if (warp < EPI_WARP0) {
        // ------------------------------------- scale copiers (leader only)
        // TMEM scale buffer of a stage (48 columns): A tile of K-step kb at
        // columns 4*kb (lane m reads column 4*kb + m/32), W tiles at 16 + 8*kb
        // (columns 16 + 8*kb + n/32 in every lane quarter).
        const int kb = warp - WRITER_WARP0;
        if (leader && lane == 0 && !p.inject_stall) {
            int stage = 0, slot = 0;
            uint32_t phase = 0, sphase = 0;
            for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl) {
                bool ok = true;
                for (int kt = 0; kt < p.kt_total; ++kt) {
                    // scales landed, and the stage's TMEM scale buffer is free: the
                    // MMAs of the stage that used it last (STAGES back) are done
                    if (!mbar_wait_bounded(smem_u32(&sm->sf_full[slot]), sphase, p.wait_limit_ns) ||
                        !mbar_wait_bounded(smem_u32(&sm->empty[stage]), phase ^ 1u, p.wait_limit_ns)) {
                        raise_timeout_pair(sm, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_t = tmem + SF_COL0 + stage * SF_BUF_COLS;
                    tc_cp_pair_32x128b_x4(sf_t + kb * 4, smem_desc(sfa_smem(slot) + kb * SF_TILE, 0, 128, 0));
                    tc_cp_pair_32x128b_x4(sf_t + 16 + kb * 8, smem_desc(sfb_smem(slot) + kb * SF_TILE, 0, 128, 0));
                    tc_cp_pair_32x128b_x4(sf_t + 16 + kb * 8 + 4,
                                          smem_desc(sfb_smem(slot) + p.sf_box_bytes + kb * SF_TILE, 0, 128, 0));
                    tc_commit_pair(smem_u32(&sm->full[stage]));
                    tc_commit_pair_both(smem_u32(&sm->sf_empty[slot]), 3);  // scale slot free in both CTAs
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++slot == SF_SLOTS) {
                        slot = 0;
                        sphase ^= 1u;
                    }
                }
                if (!ok)
                    break;
            }
        }
    } else if (GATED) {
        // ------------------------------------------- gated MLP epilogue
        // Tile columns [0, 128) are gate rows and [128, 256) the matching up
        // rows; each warp takes 64 of the tile's 128 h columns for its lane
        // quarter, 32 at a time.
        const int q = warp & 3;
        const int hc = (warp - EPI_WARP0) >> 2;
        const uint32_t box = stage_out_base + (warp - EPI_WARP0) * STAGING_BYTES;
        const float ga = __ldg(p.g_a);
        const float a_gate = __fmul_rn(ga, __ldg(p.g_w));
        const float a_up = __fmul_rn(ga, __ldg(p.g_w + 1));
        uint32_t hmax = 0;
        int local = 0;
        for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl, ++local) {
            int mp, np;
            pair_tile_coords(p, tile, mp, np);
            const int m0 = mp * PAIR_M + static_cast<int>(rank) * 128, n0 = np * PAIR_N;
            const bool ok = mbar_wait_bounded(smem_u32(&sm->acc_full), local & 1, p.wait_limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                if (lane == 0)
                    raise_timeout_pair(sm, p.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + hc * 64;
            const int row = m0 + q * 32 + lane;
            const int col0 = (n0 >> 1) + hc * 64;  // h column
            const bool row_ok = row < p.M;
            uint32_t pk[32];  // 64 h values as bf16 pairs
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t vg[32], vu[32];
                tc_ld_32x32b_x32(taddr + c * 32, vg);
                tc_ld_32x32b_x32(taddr + 128 + c * 32, vu);
                tc_wait_ld();
                if (c == 1) {
                    // the whole accumulator slice of this warp is in registers
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_remote(leader_bar(&sm->acc_empty));
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float h0 = silu_mul(__fmul_rn(__uint_as_float(vg[2 * j]), a_gate),
                                              __fmul_rn(__uint_as_float(vu[2 * j]), a_up));
                    const float h1 = silu_mul(__fmul_rn(__uint_as_float(vg[2 * j + 1]), a_gate),
                                              __fmul_rn(__uint_as_float(vu[2 * j + 1]), a_up));
                    __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
                    pk[16 * c + j] = *reinterpret_cast<uint32_t *>(&b);
                }
            }
            if (p.tma_out) {
                // stage the 32 x 64 h box and store it with one TMA copy
                if (lane == 0)
                    bulk_wait_group_read<0>();  // the previous store has read the box
                __syncwarp();
                stage_row_swizzled(box, lane, pk);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && m0 + q * 32 < p.M && col0 < p.F) {
                    tma_store_2d(&tmOut, col0, m0 + q * 32, box);
                    bulk_commit_group();
                }
            }
            if (row_ok && col0 < p.F) {
                __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + static_cast<int64_t>(row) * p.F + col0;
                const int nval = min(64, p.F - col0);
                if (p.tma_out) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (2 * j < nval)
                            hmax = vmax_mag(hmax, (2 * j + 1 < nval) ? pk[j] : (pk[j] & 0xFFFFu));
                    }
                } else if (p.vec_ok && nval == 64) {
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
        if (lane == 0)
            bulk_wait_group_all();  // every store of this warp has landed
        uint32_t v = hmax16(hmax);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0 && v != 0)
            atomicMax(p.h_amax, v);
    } else {
        // ------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int hc = (warp - EPI_WARP0) >> 2;  // which 128-column half of the tile
        float *alpha = sm->alpha[warp - EPI_WARP0];
        const uint32_t box = stage_out_base + (warp - EPI_WARP0) * STAGING_BYTES;
        const float ga = __ldg(p.g_a);
        int local = 0;
        for (int tile = cid; tile < p.pair_tiles && !sm->abort_flag; tile += ncl, ++local) {
            int mp, np;
            pair_tile_coords(p, tile, mp, np);
            const int m0 = mp * PAIR_M + static_cast<int>(rank) * 128, n0 = np * PAIR_N;
            const int row = m0 + q * 32 + lane;
            const int col0 = n0 + hc * 128;
            // Column scales first: they do not depend on the accumulator.  A
            // slice inside one module segment (the usual case) needs one scalar.
            const bool uniform = col0 >= p.N || column_segment(p, col0) == column_segment(p, min(col0 + 127, p.N - 1));
            const float a_u = column_alpha(p, ga, min(col0, p.N - 1));
            __syncwarp();  // this warp's reads of the previous alpha are done
            if (!uniform || p.out_fp32) {
                alpha[lane] = column_alpha(p, ga, col0 + lane);
                alpha[lane + 32] = column_alpha(p, ga, col0 + lane + 32);
            }
            __syncwarp();
            const bool ok = mbar_wait_bounded(smem_u32(&sm->acc_full), local & 1, p.wait_limit_ns);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                if (lane == 0)
                    raise_timeout_pair(sm, p.status);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + hc * 128;
            if (!p.out_fp32) {
                // 128 columns as bf16 pairs: scaled and rounded as they arrive
                uint32_t pk[64];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t v[64];
                    tc_ld_32x32b_x64(taddr + c * 64, v);
                    tc_wait_ld();
                    if (c == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive_remote(leader_bar(&sm->acc_empty));
                        if (!uniform) {
                            // second chunk's column scales (the rare mixed-segment slice)
                            __syncwarp();
                            alpha[lane] = column_alpha(p, ga, col0 + 64 + lane);
                            alpha[lane + 32] = column_alpha(p, ga, col0 + 96 + lane);
                            __syncwarp();
                        }
                    }
                    if (uniform) {
#pragma unroll
                        for (int j = 0; j < 64; j += 2) {
                            __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j]), a_u),
                                                                     __fmul_rn(__uint_as_float(v[j + 1]), a_u));
                            pk[32 * c + j / 2] = *reinterpret_cast<uint32_t *>(&b);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; j += 2) {
                            __nv_bfloat162 b =
                                __floats2bfloat162_rn(__fmul_rn(__uint_as_float(v[j]), alpha[j]),
                                                      __fmul_rn(__uint_as_float(v[j + 1]), alpha[j + 1]));
                            pk[32 * c + j / 2] = *reinterpret_cast<uint32_t *>(&b);
                        }
                    }
                }
                if (p.tma_out) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        if (lane == 0)
                            bulk_wait_group_read<0>();  // the previous store has read the box
                        __syncwarp();
                        stage_row_swizzled(box, lane, pk + 32 * c);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && m0 + q * 32 < p.M && col0 + 64 * c < p.N) {
                            tma_store_2d(&tmOut, col0 + 64 * c, m0 + q * 32, box);
                            bulk_commit_group();
                        }
                    }
                } else {
                    store_bf16_packed_128(p, row, col0, pk);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t v[64];
                    tc_ld_32x32b_x64(taddr + c * 64, v);
                    tc_wait_ld();
                    if (c == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            mbar_arrive_remote(leader_bar(&sm->acc_empty));
                        __syncwarp();
                        alpha[lane] = column_alpha(p, ga, col0 + 64 + lane);
                        alpha[lane + 32] = column_alpha(p, ga, col0 + 96 + lane);
                        __syncwarp();
                    }
                    store_64(p, alpha, row, col0 + 64 * c, v);
                }
            }
        }
        if (lane == 0)
            bulk_wait_group_all();  // every store of this warp has landed
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace pair
}  // namespace gemm
}  // namespace nvfp4
