// quant.cu -- e4m3 quantization of the expert activations.
//
// "PCoMoE" summary, "Improvements", 3 (Mixed Precision Execution): the expert
// computation in FP8, the gating in BF16.  Each activation row (a token's x
// on its way into the gate/up GEMM, a row of the hidden activation h on its
// way into the down GEMM) is divided by the smallest power of two s with
// 448 s >= max|row| and rounded to the nearest e4m3 value (ties to even,
// saturating).  Dividing by a power of two is exact, so the rounding is the
// only approximation, and s is kept beside the row for the GEMM's epilogue.
//   gather_quant_kernel: x_sorted codes[r] = e4m3(x[token_of[r]] / s_r), one
//     warp per row (the permutation's gather and the quantization in one pass;
//     layers with four or more destination rows per token quantize each
//     token's row once inside the one-launch permutation instead);
//   quant_rows_kernel: h8[r] = e4m3(h[r] / s_r), one block per row.
// The row scale and the code conversion are in e4m3.cuh.

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "e4m3.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr unsigned FULL = 0xffffffffu;

// Rows r < offsets[n_last] (capped at rows_cap): codes[r] = e4m3(x[t] / s),
// scale[r] = s, t = token_of[r].  d a multiple of 256 (32 lanes x 8).
__global__ void __launch_bounds__(256) gather_quant_kernel(const int32_t* __restrict__ token_of,
                                                           const int32_t* __restrict__ offsets, int n_last,
                                                           const __nv_bfloat16* __restrict__ x, int d, int T,
                                                           uint8_t* __restrict__ codes, float* __restrict__ scale,
                                                           long long rows_cap)
{
    const int lane = threadIdx.x & 31;
    const long long total = min((long long)offsets[n_last], rows_cap);
    const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
    const int nv = d / 256;                                 // 8-element vectors per lane
    for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < total; r += nw) {
        const int t = token_of[r];
        if (t < 0 || t >= T) { if (lane == 0) set_status(MOE_ERR_DEVICE_BOUNDS); continue; }
        const uint4* src = reinterpret_cast<const uint4*>(x + (long long)t * d);
        float amax = 0.f;
        for (int i = 0; i < nv; ++i) {
            float v[8];
            bf16x8(__ldg(src + i * 32 + lane), v);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        const float s = pow2_scale(amax), inv = 1.f / s;   // inverse of a power of two: exact
        uint2* dst = reinterpret_cast<uint2*>(codes + r * d);
        for (int i = 0; i < nv; ++i) {
            float v[8];
            bf16x8(__ldg(src + i * 32 + lane), v);          // second read: from L1 / L2
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] *= inv;
            dst[i * 32 + lane] = to_e4m3x8(v);
        }
        if (lane == 0) scale[r] = s;
    }
}

// Rows r < offsets[n_last] of h [rows, H] bf16: h8[r] = e4m3(h[r] / s), s_h[r] = s.
// One block of 256 threads per row; H a multiple of 8.
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ h,
                                                         const int32_t* __restrict__ offsets, int n_last, int H,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scale,
                                                         long long rows_cap)
{
    __shared__ float red[8];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const long long total = min((long long)offsets[n_last], rows_cap);
    const int nv = H / 8;
    for (long long r = blockIdx.x; r < total; r += gridDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(h + r * H);
        float amax = 0.f;
        for (int i = threadIdx.x; i < nv; i += 256) {
            float v[8];
            bf16x8(src[i], v);
#pragma unroll
            for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
        if (lane == 0) red[wib] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
        const float s = pow2_scale(amax), inv = 1.f / s;
        uint2* dst = reinterpret_cast<uint2*>(codes + r * H);
        for (int i = threadIdx.x; i < nv; i += 256) {
            float v[8];
            bf16x8(src[i], v);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] *= inv;
            dst[i] = to_e4m3x8(v);
        }
        if (threadIdx.x == 0) scale[r] = s;
        __syncthreads();                                  // red[] is rewritten for the next row
    }
}

}  // namespace

moe_status launch_gather_quant(const int32_t* token_of, const int32_t* offsets, int n_last, const void* x, int d,
                               int T, void* codes, float* scale, long long rows_cap, cudaStream_t st)
{
    if (d % 256 != 0) return MOE_ERR_UNSUPPORTED;
    const int grid = (int)std::max<long long>(1, std::min<long long>((rows_cap + 7) / 8, num_sms() * 16));
    gather_quant_kernel<<<grid, 256, 0, st>>>(token_of, offsets, n_last, static_cast<const __nv_bfloat16*>(x), d, T,
                                              static_cast<uint8_t*>(codes), scale, rows_cap);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_quant_rows(const void* h, const int32_t* offsets, int n_last, int H, void* codes, float* scale,
                             long long rows_cap, cudaStream_t st)
{
    if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
    const int grid = (int)std::max<long long>(1, std::min<long long>(rows_cap, num_sms() * 8));
    quant_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h), offsets, n_last, H,
                                            static_cast<uint8_t*>(codes), scale, rows_cap);
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
