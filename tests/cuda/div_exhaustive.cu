// Compares the quantizer's shared-divisor division (div_shared, its packed
// two-lane form div_shared_x2 and the negated form div_shared_neg_x2, from
// fp_div.cuh) with CUDA's IEEE division __fdiv_rn, bit for bit (the packed
// forms on the pair (x, -x); div_shared_neg_x2 against -__fdiv_rn):
//  (1) every bf16 significand x (128) against every fp32 significand d (2^23),
//      with exponents chosen so x/d spans [2^-5, 2^5), both signs;
//  (2) every finite bf16 value against pseudo-random divisors over the whole
//      range div_shared_ok() accepts: quotients >= 2^-20 bit for bit, smaller
//      ones below 0.25 with the sign of x (they all encode to +-0).
// Prints "checked=<n> mismatches=<m> accepted=<a>" and exits 0.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "fp_div.cuh"

using nvfp4::div_shared;
using nvfp4::div_shared_ok;
using nvfp4::div_shared_x2;
using nvfp4::div_shared_neg_x2;

// bf16 bits of x (x is a bf16 value) in the low half, of -x in the high half
__device__ uint32_t pair_of(float x)
{
    const uint32_t b = __float_as_uint(x) >> 16;
    return b | ((b ^ 0x8000u) << 16);
}

__device__ unsigned int g_nrec;
__device__ float g_rec[64][4];

__device__ void record(float x, float d, float y, float ref)
{
    const unsigned i = atomicAdd(&g_nrec, 1u);
    if (i < 64) {
        g_rec[i][0] = x;
        g_rec[i][1] = d;
        g_rec[i][2] = y;
        g_rec[i][3] = ref;
    }
}

__global__ void sweep_significands(unsigned long long *checked, unsigned long long *bad)
{
    const uint32_t n_d = 1u << 23;
    unsigned long long c = 0, b = 0;
    for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < n_d; t += gridDim.x * blockDim.x) {
        const float d0 = __uint_as_float(0x3F800000u | t);  // [1, 2)
#pragma unroll 1
        for (int ed = -1; ed <= 0; ++ed) {
            const float d = ldexpf(d0, ed);
            const float r = __frcp_rn(d);
#pragma unroll 1
            for (uint32_t m = 0; m < 128; ++m) {
#pragma unroll 1
                for (int ex = -4; ex <= 4; ++ex) {
                    const float x = ldexpf(__uint_as_float(0x3F800000u | (m << 16)), ex);
#pragma unroll
                    for (int sgn = 0; sgn < 2; ++sgn) {
                        const float xs = sgn ? -x : x;
                        const float y = div_shared(xs, d, r);
                        const float ref = __fdiv_rn(xs, d);
                        if (__float_as_uint(y) != __float_as_uint(ref)) {
                            ++b;
                            record(xs, d, y, ref);
                        }
                        ++c;
                        float y2lo, y2hi;
                        div_shared_x2(pair_of(xs), d, -r, y2lo, y2hi);
                        const float ref_neg = __fdiv_rn(-xs, d);
                        if (__float_as_uint(y2lo) != __float_as_uint(ref) ||
                            __float_as_uint(y2hi) != __float_as_uint(ref_neg)) {
                            ++b;
                            record(xs, d, y2lo, ref);
                        }
                        c += 2;
                        float n2lo, n2hi;
                        div_shared_neg_x2(pair_of(xs), d, -r, n2lo, n2hi);
                        if (__float_as_uint(n2lo) != (__float_as_uint(ref) ^ 0x80000000u) ||
                            __float_as_uint(n2hi) != (__float_as_uint(ref_neg) ^ 0x80000000u)) {
                            ++b;
                            record(xs, d, -n2lo, ref);
                        }
                        c += 2;
                    }
                }
            }
        }
    }
    atomicAdd(checked, c);
    atomicAdd(bad, b);
}

__device__ uint32_t hash32(uint32_t x)
{
    x ^= x >> 16; x *= 0x7feb352dU; x ^= x >> 15; x *= 0x846ca68bU; x ^= x >> 16;
    return x;
}

__global__ void sweep_range(unsigned long long *checked, unsigned long long *bad, unsigned long long *accepted)
{
    unsigned long long c = 0, b = 0, a = 0;
    for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < (1u << 16) * 256u; t += gridDim.x * blockDim.x) {
        const uint32_t xb = t & 0xFFFFu;
        const float x = __uint_as_float(xb << 16);
        if (!isfinite(x))
            continue;
        // divisor: random significand, exponent uniform over [2^-110, 2^110]
        const uint32_t h = hash32(t * 2654435761u + 12345u);
        const int e = static_cast<int>(hash32(h) % 201u) - 90;
        const float d = ldexpf(__uint_as_float(0x3F800000u | (h & 0x7FFFFFu)), e);
        if (!div_shared_ok(d, fabsf(x)))
            continue;
        ++a;
        const float r = __frcp_rn(d);
        float y2[2], n2[2];
        div_shared_x2(pair_of(x), d, -r, y2[0], y2[1]);
        div_shared_neg_x2(pair_of(x), d, -r, n2[0], n2[1]);
        const float ys[5] = {div_shared(x, d, r), y2[0], y2[1], -n2[0], -n2[1]};
        const float refs[5] = {__fdiv_rn(x, d), __fdiv_rn(x, d), __fdiv_rn(-x, d), __fdiv_rn(x, d), __fdiv_rn(-x, d)};
        // quotients >= 2^-20 must be the IEEE ones; smaller ones must stay below
        // 0.25 (all encode to +-0) with the sign of x
        for (int k = 0; k < 5; ++k) {
            const float y = ys[k], ref = refs[k];
            if (fabsf(ref) >= 0x1p-20f || fabsf(y) >= 0x1p-20f) {
                if (__float_as_uint(y) != __float_as_uint(ref)) {
                    ++b;
                    record(x, d, y, ref);
                }
            } else {
                b += (signbit(y) != signbit(ref)) || !(fabsf(y) < 0.25f);
            }
            ++c;
        }
    }
    atomicAdd(checked, c);
    atomicAdd(bad, b);
    atomicAdd(accepted, a);
}

int main()
{
    unsigned long long *d_c, *d_b, *d_a;
    cudaMalloc(&d_c, 8);
    cudaMalloc(&d_b, 8);
    cudaMalloc(&d_a, 8);
    cudaMemset(d_c, 0, 8);
    cudaMemset(d_b, 0, 8);
    cudaMemset(d_a, 0, 8);
    sweep_significands<<<148 * 8, 256>>>(d_c, d_b);
    sweep_range<<<148 * 8, 256>>>(d_c, d_b, d_a);
    cudaError_t e = cudaDeviceSynchronize();
    unsigned long long c = 0, b = 0, a = 0;
    cudaMemcpy(&c, d_c, 8, cudaMemcpyDeviceToHost);
    cudaMemcpy(&b, d_b, 8, cudaMemcpyDeviceToHost);
    cudaMemcpy(&a, d_a, 8, cudaMemcpyDeviceToHost);
    printf("checked=%llu mismatches=%llu accepted=%llu err=%s\n", c, b, a, cudaGetErrorString(e));
    unsigned nrec = 0;
    float rec[64][4];
    cudaMemcpyFromSymbol(&nrec, g_nrec, sizeof(nrec));
    cudaMemcpyFromSymbol(rec, g_rec, sizeof(rec));
    for (unsigned i = 0; i < nrec && i < 16; ++i)
        printf("mismatch x=%a d=%a div_shared=%a ieee=%a\n", rec[i][0], rec[i][1], rec[i][2], rec[i][3]);
    return e == cudaSuccess ? 0 : 1;
}
