// e4m3.cuh -- per-row e4m3 quantization helpers shared by the kernels that
// quantize expert activations (the one-launch permutation's row copies, the
// gather of the permuted rows, the rows of h between the expert GEMMs).
//
// "PCoMoE" summary, "Improvements", 3 (Mixed Precision Execution): a row is
// divided by the smallest power of two s with 448 s >= max|row| and rounded
// to the nearest e4m3 value (ties to even, saturating); s is kept beside the
// row for the GEMM's epilogue.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// The smallest power of two s with 448 s >= amax (1 for amax == 0).  448 * 2^e
// is exact in fp32, so the comparisons decide exactly.
__device__ __forceinline__ float pow2_scale(float amax)
{
    if (!(amax > 0.f)) return 1.f;
    int ex;
    frexpf(amax, &ex);                  // amax in [2^(ex-1), 2^ex)
    int e = max(ex - 9, -126);
    while (448.f * ldexpf(1.f, e) < amax) ++e;
    while (e > -126 && 448.f * ldexpf(1.f, e - 1) >= amax) --e;
    return ldexpf(1.f, e);
}

// Eight values -> eight e4m3 codes (nearest, ties to even, saturating).
__device__ __forceinline__ uint2 to_e4m3x8(const float (&v)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = __nv_cvt_float2_to_fp8x2(make_float2(v[2 * i], v[2 * i + 1]), __NV_SATFINITE, __NV_E4M3);
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Eight bf16 values (one 16-byte vector) -> fp32.
__device__ __forceinline__ void bf16x8(const uint4 u, float (&v)[8])
{
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

}  // namespace moe
