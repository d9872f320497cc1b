// kv_cache_kernels.cuh -- FP8 (E4M3) KV-cache quantization with a calibrated
// per-tensor scale: the recipe ships calibrated KV-cache scales, which the
// pages report as costing nothing (freegardner.com, "Quantizing All Layers
// Reveals Recurrent Memory Is Robust", section "The Calibrated Cache That
// Ships for Free"; thevalue.engineering, "NVFP4 W4A4 quantization compresses
// 27B hybrid models", section "Efficiency Gains and Serving Optimization").
//
//   s    = fl32(amax / 448), 1 when amax == 0       (calibration, one pass)
//   code = E4M3_RNE_satfinite( fl32(x / s) )         (sign kept)
//
// s is a decode multiplier (x ~= e4m3(code) * s) held on the device.  The
// division by the shared s uses one reciprocal and a Markstein correction
// per element (fp_div.cuh), with the IEEE division where that is not exact.
#pragma once

#include <cstdint>

#include "fp_div.cuh"
#include "ptx_sm100.cuh"
#include "quantize_kernels.cuh"

namespace nvfp4 {
namespace kv {

// s = fl32(amax / 448) (1 when amax == 0) from the amax pass's bf16 bits.
__global__ void kv_scale_kernel(const uint32_t *__restrict__ amax_bits, float *__restrict__ scale)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const float a = __uint_as_float(amax_bits[0] << 16);
        scale[0] = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 448.0f);
    }
}

// Two E4M3 bytes (round to nearest even, saturating at +-448): lo in the
// low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(hi), "f"(lo));
    return pair;
}

struct KvParams {
    const uint16_t *X;  // bf16 [rows, cols], leading dimension ld (elements)
    int64_t ld;
    int64_t rows;
    int64_t cols;       // multiple of 8
    const float *scale; // device, one fp32
    uint8_t *out;       // [rows, cols] bytes, leading dimension ldo
    int64_t ldo;
    uint32_t *status;
};

// Grid-stride over 8-element groups: one 16-byte load, eight quotients, four
// conversions, one 8-byte store.
__global__ void __launch_bounds__(256) kv_quantize_kernel(const KvParams p)
{
    grid_dep_wait();
    grid_dep_launch_dependents();
    const float s = __ldg(p.scale);
    if (!(s > 0.0f) || !(s <= 3.40282347e38f)) {
        // a scale that is not a positive finite number: nothing is written
        if (blockIdx.x == 0 && threadIdx.x == 0)
            atomicOr(p.status, kStatusNonFinite);
        return;
    }
    const float r = __frcp_rn(s);
    const int64_t gpr = p.cols >> 3;
    const int64_t total = p.rows * gpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t row = i / gpr;
        const int64_t g = i - row * gpr;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.X + row * p.ld + g * 8));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        // the shared-divisor quotient is exact while every |x| / s stays below 2^100
        const float gmax = __uint_as_float(hmax16(vmax_mag(0u, v)) << 16);
        const bool fast = div_shared_ok(s, gmax);
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float x0 = bf16_lo(w[k]), x1 = bf16_hi(w[k]);
            const float y0 = fast ? div_shared(x0, s, r) : __fdiv_rn(x0, s);
            const float y1 = fast ? div_shared(x1, s, r) : __fdiv_rn(x1, s);
            b[k] = e4m3x2(y0, y1);
        }
        *reinterpret_cast<uint2 *>(p.out + row * p.ldo + g * 8) = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
    }
}

}  // namespace kv
}  // namespace nvfp4
