// ffn_simt.cu -- grouped SwiGLU experts in fp32 on the CUDA cores.
//
// The fp32 layer keeps fp32 end to end (a 1e-4 relative bar that TF32 or
// bf16 tensor-core inputs cannot meet), so its grouped GEMMs run on the FMA
// pipes: 32-row x 64-column tiles per expert group, K staged through shared
// memory in chunks of 32, each thread 2 rows x 4 columns (x2 for gate/up).
//   phase 1: h[r, :] = silu(x_s[r] . W_gate[e]^T) * (x_s[r] . W_up[e]^T)
//   phase 2: y_s[r, :] = h[r] . W_down[e]^T
// Tiles are enumerated on the device from the group offsets, as in the
// tensor-core path.

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int FM = 32, FN = 64, FK = 32;

template <bool SWIGLU>
__global__ void __launch_bounds__(256) ffn_f32_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                                                      int n_groups, int n_first,
                                                      const float* __restrict__ B0, const float* __restrict__ B1,
                                                      const float* __restrict__ B2, const float* __restrict__ B3,
                                                      int N, int K, float* __restrict__ out, long long rows_cap)
{
    __shared__ float As[FM][FK + 1];
    __shared__ float Bs[FN][FK + 1];
    __shared__ float Cs[SWIGLU ? FN : 1][FK + 1];
    __shared__ int s_tile[2];
    const int ntn = cdiv(N, FN);
    if (threadIdx.x == 0) {
        // this block's tile: walk the groups (few groups on this path)
        int tile = blockIdx.x, g = -1, local = 0;
        for (int gg = 0; gg < n_groups; ++gg) {
            const int cnt = max(offsets[gg + 1] - offsets[gg], 0);
            const int nt = cdiv(cnt, FM) * ntn;
            if (tile < nt) { g = gg; local = tile; break; }
            tile -= nt;
        }
        s_tile[0] = g;
        s_tile[1] = local;
    }
    __syncthreads();
    const int g = s_tile[0];
    if (g < 0) return;
    const int cnt = offsets[g + 1] - offsets[g];
    const int mt = cdiv(cnt, FM);
    const int m = s_tile[1] % mt, n = s_tile[1] / mt;
    const int row0 = offsets[g] + m * FM, rows = min(FM, cnt - m * FM);
    const int col0 = n * FN;
    const bool first = g < n_first;
    const long long gb = first ? g : g - n_first;
    const float* Wa = (first ? B0 : B2) + gb * (long long)N * K;
    const float* Wb = SWIGLU ? (first ? B1 : B3) + gb * (long long)N * K : nullptr;

    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16
    float acc[2][4], acc2[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { acc[i][j] = 0.f; acc2[i][j] = 0.f; }

    for (int k0 = 0; k0 < K; k0 += FK) {
        for (int i = threadIdx.x; i < FM * FK; i += 256) {
            const int r = i / FK, k = i % FK;
            As[r][k] = (r < rows && k0 + k < K) ? A[(long long)(row0 + r) * K + k0 + k] : 0.f;
        }
        for (int i = threadIdx.x; i < FN * FK; i += 256) {
            const int c = i / FK, k = i % FK;
            const bool ok = col0 + c < N && k0 + k < K;
            Bs[c][k] = ok ? Wa[(long long)(col0 + c) * K + k0 + k] : 0.f;
            if (SWIGLU) Cs[c][k] = ok ? Wb[(long long)(col0 + c) * K + k0 + k] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < FK; ++k) {
            const float a0 = As[ty][k], a1 = As[ty + 16][k];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float b = Bs[tx + 16 * j][k];
                acc[0][j] = fmaf(a0, b, acc[0][j]);
                acc[1][j] = fmaf(a1, b, acc[1][j]);
                if (SWIGLU) {
                    const float c = Cs[tx + 16 * j][k];
                    acc2[0][j] = fmaf(a0, c, acc2[0][j]);
                    acc2[1][j] = fmaf(a1, c, acc2[1][j]);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = ty + 16 * i;
        const long long grow = (long long)row0 + r;
        if (r >= rows || grow >= rows_cap) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = col0 + tx + 16 * j;
            if (c >= N) continue;
            float v = acc[i][j];
            if (SWIGLU) v = v / (1.0f + expf(-v)) * acc2[i][j];
            out[grow * N + c] = v;
        }
    }
}

}  // namespace

moe_status launch_ffn_f32(const FfnF32Args& a, int phase, cudaStream_t st)
{
    const long long row_tiles = (a.rows_cap + FM - 1) / FM + a.n_groups;
    if (phase == 1) {
        const long long grid = row_tiles * cdiv(a.H, FN);
        ffn_f32_kernel<true><<<(unsigned)grid, 256, 0, st>>>(a.xs, a.offsets, a.n_groups, a.n_first, a.wg, a.wu,
                                                            a.sg, a.su, a.H, a.d, a.h, a.rows_cap);
    } else {
        const long long grid = row_tiles * cdiv(a.d, FN);
        ffn_f32_kernel<false><<<(unsigned)grid, 256, 0, st>>>(a.h, a.offsets, a.n_groups, a.n_first, a.wd, nullptr,
                                                             a.sd, nullptr, a.d, a.H, a.ys, a.rows_cap);
    }
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
