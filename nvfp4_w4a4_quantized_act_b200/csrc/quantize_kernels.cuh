// quantize_kernels.cuh -- HBM-bound NVFP4 codec kernels for sm_100a.
//
//  amax_kernel      max|x| per module segment (per tensor for activations):
//                   one warp per row, 16-byte loads, packed 16-bit integer
//                   max of bf16 magnitudes (non-negative floats order like
//                   their bit patterns), one shared then one global atomic
//                   per CTA and segment.
//  quantize_kernel  per 16-element block: E4M3 scale and E2M1 codes, two
//                   codes per byte, scales written straight into the 128x4
//                   tile layout the block-scaled MMA reads (four neighbouring
//                   blocks of a row form one 32-bit word, gathered by warp
//                   shuffles).
//  swiglu_kernel    h = bf16(silu(gate) * up) for a fused gate/up output, plus
//                   max|h| for its dynamic global scale.
//
// Format and scale conventions: NVFP4 = E2M1 codes, each group of 16
// consecutive codes sharing one E4M3 scale ("NVFP4 W4A4 quantization compresses 27B hybrid models",
// thevalue.engineering, "Challenging the Recurrence Fragility Assumption"),
// one FP32 global scale per calibrated module ("Why Gated DeltaNet Survives
// 4-Bit Quantization", kipquest.com, "The abstract").
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "fp_div.cuh"
#include "ptx_sm100.cuh"

namespace nvfp4 {

constexpr int kMaxSeg = 16;
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusNonFinite = 2u;

// Rows [0, end[0]) belong to segment 0, [end[i-1], end[i]) to segment i.
struct SegRows {
    int32_t nseg;
    int64_t end[kMaxSeg];
};

__device__ __forceinline__ int seg_of(const SegRows &s, int64_t r)
{
    int k = 0;
#pragma unroll 1
    while (k + 1 < s.nseg && r >= s.end[k])
        ++k;
    return k;
}

// Packed max of the magnitudes of the two bf16 in `w`, each kept as
// (magnitude << 1) in its 16-bit half: w + w pushes the upper sign bit out
// and the lower sign bit into the upper half's lowest bit, which hmax16()
// shifts away again.
__device__ __forceinline__ uint32_t vmax_mag(uint32_t acc, uint32_t w)
{
    return __vmaxu2(acc, w + w);
}

__device__ __forceinline__ uint32_t vmax_mag(uint32_t acc, const uint4 &v)
{
    acc = vmax_mag(acc, v.x);
    acc = vmax_mag(acc, v.y);
    acc = vmax_mag(acc, v.z);
    acc = vmax_mag(acc, v.w);
    return acc;
}

// Largest bf16 magnitude (bits, sign cleared) of a vmax_mag() accumulator.
__device__ __forceinline__ uint32_t hmax16(uint32_t packed) { return max(packed & 0xFFFFu, packed >> 16) >> 1; }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ amax

// words[0, n) = 0: clears amax accumulators in stream order as a kernel (so
// the launches around it keep their programmatic dependencies).
__global__ void zero_words_kernel(uint32_t *__restrict__ words, int32_t n)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        words[i] = 0;
}

// amax_bits[seg] = max over the segment's rows of the bf16 magnitude bits
// (the float max|x| is amax_bits << 16).  amax_bits must be zero on entry,
// except with `direct` (a launch of one CTA), where the CTA stores its maxima.
// Each row is cut into `slices` contiguous ranges of 16-byte chunks, one warp
// per (row, range): one range per row when there are rows enough to fill the
// GPU, several when there are few (decode-sized inputs), so that a short
// input is read by many warps at once instead of a few long loops.
__global__ void __launch_bounds__(1024) amax_kernel(const uint16_t *__restrict__ X, int64_t rows, int64_t K,
                                                    int64_t ld, int64_t slices, SegRows seg,
                                                    uint32_t *__restrict__ amax_bits, uint32_t *__restrict__ status,
                                                    int32_t direct)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    __shared__ uint32_t s_max[kMaxSeg];
    if (threadIdx.x < kMaxSeg)
        s_max[threadIdx.x] = 0;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t chunks = K >> 3;  // 16-byte chunks per row
    const int64_t per_slice = (chunks + slices - 1) / slices;

    int slot = 0;
    uint32_t m = 0;
    for (int64_t item = warp; item < rows * slices; item += nwarps) {
        const int64_t r = item / slices;
        const int64_t c0 = (item - r * slices) * per_slice;
        const int64_t c1 = min(c0 + per_slice, chunks);
        const int s = seg_of(seg, r);
        if (s != slot) {  // warp-uniform: every lane works on row r
            atomicMax(&s_max[slot], hmax16(m));
            m = 0;
            slot = s;
        }
        const uint4 *p = reinterpret_cast<const uint4 *>(X + r * ld);
        int64_t j = c0 + lane;
        for (; j + 96 < c1; j += 128) {
            const uint4 a = __ldg(p + j), b = __ldg(p + j + 32), c = __ldg(p + j + 64), d = __ldg(p + j + 96);
            m = vmax_mag(m, a);
            m = vmax_mag(m, b);
            m = vmax_mag(m, c);
            m = vmax_mag(m, d);
        }
        for (; j < c1; j += 32)
            m = vmax_mag(m, __ldg(p + j));
    }
    atomicMax(&s_max[slot], hmax16(m));
    __syncthreads();
    if (threadIdx.x < seg.nseg) {
        const uint32_t v = s_max[threadIdx.x];
        if (direct)
            amax_bits[threadIdx.x] = v;
        else if (v != 0)
            atomicMax(&amax_bits[threadIdx.x], v);
        if (v >= 0x7F80u)  // Inf or NaN magnitude
            atomicOr(status, kStatusNonFinite);
    }
}

// ------------------------------------------------------------- quantize

struct QuantParams {
    const uint16_t *X;       // bf16 [rows, K], leading dimension ld
    int64_t ld;
    int32_t rows;
    int32_t K;
    int32_t rows_pad;        // rows rounded up to 128
    int32_t groups;          // ceil(K / 64): 32-bit scale words per row
    SegRows seg;
    const uint32_t *amax_bits;  // mode 0: per-segment amax bits
    const float *g_in;          // mode 1: per-segment global scale
    float *g_out;               // modes 0, 2: per-segment global scale written here (may be null)
    int32_t mode;               // 0: g from amax_bits, 1: g given, 2: g from max|x| taken by every CTA
    uint32_t *status = nullptr; // mode 2: latched error bits (non-finite input)
    uint8_t *codes;          // [rows, K/2]
    uint8_t *sf;             // swizzled scale tiles
    int32_t gate_up_F;       // > 0: rows are [gate F | up F]; stored interleaved in 128-row blocks
    uint32_t *zero = nullptr;  // one word block 0 clears (the next GEMM's max|h|), or null
};

// Stored row of input row r.  With a gate/up pair of F rows each, block b of
// gate rows goes to stored rows [256 b, 256 b + 128) and block b of up rows to
// [256 b + 128, 256 b + 256), so one 256-row GEMM tile holds matching gate
// and up columns.
__device__ __forceinline__ uint32_t stored_row(const QuantParams &p, uint32_t r)
{
    if (p.gate_up_F <= 0)
        return r;
    const uint32_t F = static_cast<uint32_t>(p.gate_up_F);
    const uint32_t m = r >= F ? 1u : 0u;
    const uint32_t i = r - m * F;
    return (((i >> 7) << 1) + m) * 128u + (i & 127u);
}

__device__ __forceinline__ float global_scale_from_amax(uint32_t bits)
{
    const float a = __uint_as_float(bits << 16);
    return a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// E4M3 scale byte of a block whose largest magnitude is bamax:
// s32 = fl32(fl32(bamax / 6) / g), by the shared-divisor division where it is
// exact, then E4M3 round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t block_scale_byte(float bamax, float g, float rg, bool g_ok)
{
    float s32;
    const float t_fast = div_shared(bamax, 6.0f, 0x1.555556p-3f /* RN(1/6) */);
    if (g_ok && bamax >= 0x1p-17f && bamax <= 0x1p100f && div_shared_ok(g, t_fast))
        s32 = div_shared(t_fast, g, rg);
    else
        s32 = __fdiv_rn(__fdiv_rn(bamax, 6.0f), g);
    return f32_to_e4m3_satfinite(s32);
}

// Codes of a block outside the shared-divisor range: a zero decode scale
// gives +-0 with the sign of each input, anything else the IEEE quotients.
__device__ __forceinline__ void block_codes_slow(const uint32_t (&w)[8], float d, uint32_t (&packed)[2])
{
    packed[0] = packed[1] = 0u;
    if (d == 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t lo = (w[i] >> 15) & 1u, hi = (w[i] >> 31) & 1u;
            packed[i >> 2] |= ((lo << 3) | (hi << 7)) << ((i & 3) * 8);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float y0 = __fdiv_rn(bf16_lo(w[i]), d);
            const float y1 = __fdiv_rn(bf16_hi(w[i]), d);
            packed[i >> 2] |= f32x2_to_e2m1x2(y0, y1) << ((i & 3) * 8);
        }
    }
}

// Block scale and codes of one 16-element block held as two 16-byte words.
// Returns the E4M3 scale byte and writes the 8 code bytes to packed[0..1].
__device__ __forceinline__ uint32_t quantize_block(const uint4 &v0, const uint4 &v1, float g, float rg, bool g_ok,
                                                   uint32_t (&packed)[2])
{
    const uint32_t bmax = hmax16(vmax_mag(vmax_mag(0u, v0), v1));
    const float bamax = __uint_as_float(bmax << 16);
    const uint32_t sbyte = block_scale_byte(bamax, g, rg, g_ok);
    const float d = __fmul_rn(e4m3_to_f32(sbyte), g);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    if (d != 0.0f && div_shared_ok(d, bamax)) {
        const float nr = -__frcp_rn(d);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                div_shared_x2(w[4 * h + i], d, nr, y[2 * i], y[2 * i + 1]);
            packed[h] = e2m1x8(y);
        }
    } else {
        block_codes_slow(w, d, packed);
    }
    return sbyte;
}

// Eight E2M1 codes of the quotients x / d of the eight bf16 values in v (low
// half of each word first), for a divisor in the shared-divisor range and
// nr = -RN(1/d): the negated quotients are encoded and every code's sign bit
// flipped back (div_shared_neg_x2).
__device__ __forceinline__ uint32_t codes8_shared(const uint4 &v, float d, float nr)
{
    float y[8];
    div_shared_neg_x2(v.x, d, nr, y[0], y[1]);
    div_shared_neg_x2(v.y, d, nr, y[2], y[3]);
    div_shared_neg_x2(v.z, d, nr, y[4], y[5]);
    div_shared_neg_x2(v.w, d, nr, y[6], y[7]);
    return e2m1x8(y) ^ 0x88888888u;
}

// Work item = one 512-element chunk of one row (32 blocks = 8 scale words),
// one lane per 16-element block.  Warps stride over the rows_pad x chunks
// items; the next item's input is loaded before the current one is
// quantized.  Rows past `rows` (up to the 128-row padding) and blocks past K
// only write zero scale bytes.
__global__ void __launch_bounds__(256) quantize_kernel(const QuantParams p)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (p.zero != nullptr && blockIdx.x == 0 && threadIdx.x == 0)
        *p.zero = 0;
    __shared__ float s_g[kMaxSeg], s_rg[kMaxSeg];
    __shared__ int s_gok[kMaxSeg];
    if (threadIdx.x < p.seg.nseg) {
        const float g = (p.mode == 0) ? global_scale_from_amax(p.amax_bits[threadIdx.x]) : p.g_in[threadIdx.x];
        s_g[threadIdx.x] = g;
        s_rg[threadIdx.x] = __frcp_rn(g);
        s_gok[threadIdx.x] = (g >= 0x1p-80f && g <= 0x1p100f) ? 1 : 0;
        if (p.mode == 0 && p.g_out != nullptr && blockIdx.x == 0)
            p.g_out[threadIdx.x] = g;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const uint32_t cpr = (static_cast<uint32_t>(p.groups) + 7u) >> 3;  // chunks per row
    const uint32_t items = static_cast<uint32_t>(p.rows_pad) * cpr;
    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t drow = nwarps / cpr, dchunk = nwarps - drow * cpr;
    const int nblk = p.K >> 4;
    const bool one_seg = p.seg.nseg == 1;

    uint32_t row = warp0 / cpr, chunk = warp0 - row * cpr;
    auto load = [&](uint32_t r, uint32_t c, uint4 &a, uint4 &b) {
        const int blk = static_cast<int>(c * 32u) + lane;
        if (r < static_cast<uint32_t>(p.rows) && blk < nblk) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.X + static_cast<int64_t>(r) * p.ld + blk * 16);
            a = __ldg(src);
            b = __ldg(src + 1);
        }
    };
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (warp0 < items)
        load(row, chunk, v0, v1);
    for (uint32_t item = warp0; item < items; item += nwarps) {
        // advance to the next item and start its loads
        uint32_t nrow = row + drow, nchunk = chunk + dchunk;
        if (nchunk >= cpr) {
            nchunk -= cpr;
            ++nrow;
        }
        uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
        if (item + nwarps < items)
            load(nrow, nchunk, n0, n1);

        const int blk = static_cast<int>(chunk * 32u) + lane;
        uint32_t sbyte = 0;
        if (row < static_cast<uint32_t>(p.rows) && blk < nblk) {
            const int sg = one_seg ? 0 : seg_of(p.seg, row);
            uint32_t packed[2];
            sbyte = quantize_block(v0, v1, s_g[sg], s_rg[sg], s_gok[sg] != 0, packed);
            *reinterpret_cast<uint2 *>(p.codes + static_cast<int64_t>(stored_row(p, row)) * (p.K >> 1) + blk * 8) =
                make_uint2(packed[0], packed[1]);
        }
        // four neighbouring blocks -> one 32-bit scale word, in lanes 0, 4, 8, ...
        const uint32_t pair = sbyte | (__shfl_down_sync(0xFFFFFFFFu, sbyte, 1) << 8);
        const uint32_t word = pair | (__shfl_down_sync(0xFFFFFFFFu, pair, 2) << 16);
        const uint32_t cg = chunk * 8u + (lane >> 2);
        if ((lane & 3) == 0 && cg < static_cast<uint32_t>(p.groups)) {
            const uint32_t srow = stored_row(p, row);
            const uint64_t tile = static_cast<uint64_t>(srow >> 7) * p.groups + cg;
            const uint32_t rr = srow & 127u;
            *reinterpret_cast<uint32_t *>(p.sf + tile * 512 + (rr & 31u) * 16 + (rr >> 5) * 4) = word;
        }
        row = nrow;
        chunk = nchunk;
        v0 = n0;
        v1 = n1;
    }
}

// quantize_kernel for one module segment with rows stored in order (every
// activation): the same work items and the same results.  The decode scale
// d = fl32(s g), nr = -RN(1/d) and the largest block amax for which the
// shared-divisor quotients are exact (d 2^100) depend only on the block's
// scale byte s, so each CTA tabulates them once for the 127 finite bytes and
// a block looks its entry up instead of decoding s and taking a correctly
// rounded reciprocal; the quotients are taken on the unnegated inputs
// (codes8_shared).
template <bool CTA_AMAX = false>
__global__ void __launch_bounds__(256) quantize_act_kernel(const QuantParams p)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    __shared__ float4 s_tab[128];  // {d, nr, d 2^100 or -1 outside the shared-divisor range, 0}
    __shared__ uint32_t s_amax;
    float g;
    if (CTA_AMAX) {
        // mode 2, a decode-sized input: every CTA reads all of it (from L2) for max|x|,
        // so the global scale needs neither an amax launch nor a grid barrier
        if (threadIdx.x == 0)
            s_amax = 0;
        __syncthreads();
        const int64_t cpr16 = p.K >> 3;  // 16-byte chunks per row
        uint32_t m = 0;
        for (int64_t i = threadIdx.x; i < static_cast<int64_t>(p.rows) * cpr16; i += blockDim.x) {
            const int64_t r = i / cpr16, c = i - r * cpr16;
            m = vmax_mag(m, __ldg(reinterpret_cast<const uint4 *>(p.X + r * p.ld) + c));
        }
        uint32_t v = hmax16(m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if ((threadIdx.x & 31) == 0 && v != 0)
            atomicMax(&s_amax, v);
        __syncthreads();
        if (blockIdx.x == 0 && threadIdx.x == 0 && s_amax >= 0x7F80u)  // Inf or NaN magnitude
            atomicOr(p.status, kStatusNonFinite);
        g = global_scale_from_amax(s_amax);
    } else {
        g = (p.mode == 0) ? global_scale_from_amax(p.amax_bits[0]) : p.g_in[0];
    }
    if (threadIdx.x < 128) {
        // byte 0x7F is E4M3's NaN; the saturating conversion never produces it
        const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), g);
        const bool fast = threadIdx.x < 127 && d >= 0x1p-80f && d <= 0x1p100f;
        s_tab[threadIdx.x] =
            make_float4(d, fast ? -__frcp_rn(d) : 0.0f, fast ? __fmul_rn(d, 0x1p100f) : -1.0f, 0.0f);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (p.zero != nullptr)
            *p.zero = 0;
        if (p.mode != 1 && p.g_out != nullptr)
            p.g_out[0] = g;
    }
    const float rg = __frcp_rn(g);
    const bool g_ok = g >= 0x1p-80f && g <= 0x1p100f;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const uint32_t cpr = (static_cast<uint32_t>(p.groups) + 7u) >> 3;  // chunks per row
    const uint32_t items = static_cast<uint32_t>(p.rows_pad) * cpr;
    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    const uint32_t drow = nwarps / cpr, dchunk = nwarps - drow * cpr;
    const int nblk = p.K >> 4;
    const uint32_t rows = static_cast<uint32_t>(p.rows);

    uint32_t row = warp0 / cpr, chunk = warp0 - row * cpr;
    auto load = [&](uint32_t r, uint32_t c, uint4 &a, uint4 &b) {
        const int blk = static_cast<int>(c * 32u) + lane;
        if (r < rows && blk < nblk) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.X + static_cast<int64_t>(r) * p.ld + blk * 16);
            a = __ldg(src);
            b = __ldg(src + 1);
        }
    };
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
    if (warp0 < items)
        load(row, chunk, v0, v1);
    for (uint32_t item = warp0; item < items; item += nwarps) {
        uint32_t nrow = row + drow, nchunk = chunk + dchunk;
        if (nchunk >= cpr) {
            nchunk -= cpr;
            ++nrow;
        }
        uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
        if (item + nwarps < items)
            load(nrow, nchunk, n0, n1);

        const int blk = static_cast<int>(chunk * 32u) + lane;
        uint32_t sbyte = 0;
        if (row < rows && blk < nblk) {
            const float bamax = __uint_as_float(hmax16(vmax_mag(vmax_mag(0u, v0), v1)) << 16);
            sbyte = block_scale_byte(bamax, g, rg, g_ok);
            const float4 e = s_tab[sbyte];
            uint32_t packed[2];
            if (bamax <= e.z) {
                packed[0] = codes8_shared(v0, e.x, e.y);
                packed[1] = codes8_shared(v1, e.x, e.y);
            } else {
                const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                block_codes_slow(w, e.x, packed);
            }
            *reinterpret_cast<uint2 *>(p.codes + static_cast<int64_t>(row) * (p.K >> 1) + blk * 8) =
                make_uint2(packed[0], packed[1]);
        }
        // four neighbouring blocks -> one 32-bit scale word, in lanes 0, 4, 8, ...
        const uint32_t pair = sbyte | (__shfl_down_sync(0xFFFFFFFFu, sbyte, 1) << 8);
        const uint32_t word = pair | (__shfl_down_sync(0xFFFFFFFFu, pair, 2) << 16);
        const uint32_t cg = chunk * 8u + (lane >> 2);
        if ((lane & 3) == 0 && cg < static_cast<uint32_t>(p.groups)) {
            const uint64_t tile = static_cast<uint64_t>(row >> 7) * p.groups + cg;
            const uint32_t rr = row & 127u;
            *reinterpret_cast<uint32_t *>(p.sf + tile * 512 + (rr & 31u) * 16 + (rr >> 5) * 4) = word;
        }
        row = nrow;
        chunk = nchunk;
        v0 = n0;
        v1 = n1;
    }
}

// --------------------------------------------------------------- SwiGLU

// h[r, j] = bf16( silu(gate[r, j]) * up[r, j] ), silu(v) = v / (1 + exp(-v))
// in fp32; gate_up is [rows, 2F] with leading dimension ld.  Also folds
// max|h| into *amax_bits (zero on entry).
__global__ void __launch_bounds__(256) swiglu_kernel(const uint16_t *__restrict__ GU, int64_t ld, int32_t rows,
                                                     int32_t F, uint16_t *__restrict__ H,
                                                     uint32_t *__restrict__ amax_bits)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    const uint32_t cpr = static_cast<uint32_t>(F) >> 3;
    const uint32_t total = static_cast<uint32_t>(rows) * cpr;
    uint32_t m = 0;
    for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
        const uint32_t r = t / cpr, j = t - r * cpr;
        const uint16_t *rowp = GU + static_cast<int64_t>(r) * ld;
        const uint4 gv = __ldg(reinterpret_cast<const uint4 *>(rowp) + j);
        const uint4 uv = __ldg(reinterpret_cast<const uint4 *>(rowp + F) + j);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
        uint32_t hw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float h2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float g = k ? bf16_hi(gw[i]) : bf16_lo(gw[i]);
                const float u = k ? bf16_hi(uw[i]) : bf16_lo(uw[i]);
                const float sg = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
                h2[k] = __fmul_rn(sg, u);
            }
            const __nv_bfloat162 b = __floats2bfloat162_rn(h2[0], h2[1]);
            hw[i] = *reinterpret_cast<const uint32_t *>(&b);
            m = vmax_mag(m, hw[i]);
        }
        reinterpret_cast<uint4 *>(H + static_cast<int64_t>(r) * F)[j] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    uint32_t v = hmax16(m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    __shared__ uint32_t s_max;
    if (threadIdx.x == 0)
        s_max = 0;
    __syncthreads();
    if ((threadIdx.x & 31) == 0)
        atomicMax(&s_max, v);
    __syncthreads();
    if (threadIdx.x == 0 && s_max != 0)
        atomicMax(amax_bits, s_max);
}

}  // namespace nvfp4
