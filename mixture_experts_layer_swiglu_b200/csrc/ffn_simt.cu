// ffn_simt.cu -- grouped SwiGLU experts in fp32 on the CUDA cores.
//
// The fp32 layer keeps fp32 end to end (a 1e-4 relative bar that TF32 or
// bf16 tensor-core inputs cannot meet), so its grouped GEMMs run on the FMA
// pipes: 16-row x 32-column tiles per expert group, each thread 1 row x 2
// columns (x2 for gate/up).
//   phase 1: h[r, :] = silu(x_s[r] . W_gate[e]^T) * (x_s[r] . W_up[e]^T)
//   phase 2: y_s[r, :] = h[r] . W_down[e]^T
// The layers on this path are small (a few MB of weights, a few rows per
// expert), so a tile's time is load latency and the length of each thread's
// FMA chain, not the FMA rate: each block copies its rows of A and of the
// weights for up to 256 elements of K at once (16-byte cp.async, all in
// flight together) and waits once, and tiles are small so that the work
// spreads over many SMs.  Tiles are enumerated on the device from the group offsets, as in
// the tensor-core path.

#include <algorithm>

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int FM = 16, FN = 32;
constexpr int FKMAX = 256;              // K elements staged per step
constexpr int fpitch(int kc) { return kc + 4; }   // floats per staged row (16-byte aligned rows)

template <bool SWIGLU>
constexpr int ffn_f32_smem(int kc) { return (FM + FN * (SWIGLU ? 2 : 1)) * fpitch(kc) * 4; }

// K % 4 == 0 and 16-byte aligned bases (checked by the caller), so every row
// starts on a 16-byte boundary.
template <bool SWIGLU>
__global__ void __launch_bounds__(256) ffn_f32_kernel(const float* __restrict__ A, const int32_t* __restrict__ offsets,
                                                      int n_groups, int n_first,
                                                      const float* __restrict__ B0, const float* __restrict__ B1,
                                                      const float* __restrict__ B2, const float* __restrict__ B3,
                                                      int N, int K, int KC, float* __restrict__ out, long long rows_cap)
{
    extern __shared__ __align__(16) float fsm[];
    const int pitch = fpitch(KC);
    float* As = fsm;                         // [FM][pitch]
    float* Bs = As + FM * pitch;             // [FN][pitch]
    float* Cs = Bs + FN * pitch;             // [FN][pitch] (SwiGLU: the up rows)
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

    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 columns (x2) x 16 rows
    float acc[2], acc2[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) { acc[j] = 0.f; acc2[j] = 0.f; }

    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += KC) {
        const int kc = min(KC, K - k0);       // a multiple of 4
        const int nv = kc >> 2;               // 16-byte vectors per row
        // every copy of this step in flight at once; rows past the tile and
        // columns past N are zero-filled
        for (int i = threadIdx.x; i < FM * nv; i += 256) {
            const int r = i / nv, v = i - r * nv;
            float* dst = As + r * pitch + 4 * v;
            if (r < rows) cp_async16(dst, A + (long long)(row0 + r) * K + k0 + 4 * v);
            else *reinterpret_cast<float4*>(dst) = zero4;
        }
        for (int i = threadIdx.x; i < FN * nv; i += 256) {
            const int c = i / nv, v = i - c * nv;
            const bool ok = col0 + c < N;
            const long long src = (long long)(col0 + c) * K + k0 + 4 * v;
            float* db = Bs + c * pitch + 4 * v;
            if (ok) cp_async16(db, Wa + src); else *reinterpret_cast<float4*>(db) = zero4;
            if (SWIGLU) {
                float* dc = Cs + c * pitch + 4 * v;
                if (ok) cp_async16(dc, Wb + src); else *reinterpret_cast<float4*>(dc) = zero4;
            }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < kc; k += 4) {
            const float4 a0 = *reinterpret_cast<const float4*>(As + ty * pitch + k);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float4 b = *reinterpret_cast<const float4*>(Bs + (tx + 16 * j) * pitch + k);
                acc[j] = fmaf(a0.x, b.x, acc[j]); acc[j] = fmaf(a0.y, b.y, acc[j]);
                acc[j] = fmaf(a0.z, b.z, acc[j]); acc[j] = fmaf(a0.w, b.w, acc[j]);
                if (SWIGLU) {
                    const float4 c = *reinterpret_cast<const float4*>(Cs + (tx + 16 * j) * pitch + k);
                    acc2[j] = fmaf(a0.x, c.x, acc2[j]); acc2[j] = fmaf(a0.y, c.y, acc2[j]);
                    acc2[j] = fmaf(a0.z, c.z, acc2[j]); acc2[j] = fmaf(a0.w, c.w, acc2[j]);
                }
            }
        }
        __syncthreads();
    }
    const int r = ty;
    const long long grow = (long long)row0 + r;
    if (r < rows && grow < rows_cap) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int c = col0 + tx + 16 * j;
            if (c >= N) continue;
            float v = acc[j];
            if (SWIGLU) v = v / (1.0f + expf(-v)) * acc2[j];
            out[grow * N + c] = v;
        }
    }
}

}  // namespace

moe_status launch_ffn_f32(const FfnF32Args& a, int phase, cudaStream_t st)
{
    const long long row_tiles = (a.rows_cap + FM - 1) / FM + a.n_groups;
    const int K = phase == 1 ? a.d : a.H;
    const int kc = std::min(K, FKMAX);
    if (phase == 1) {
        const long long grid = row_tiles * cdiv(a.H, FN);
        const int smem = ffn_f32_smem<true>(kc);
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(ffn_f32_kernel<true>), smem);
        if (e != cudaSuccess) return cuda_status(e);
        ffn_f32_kernel<true><<<(unsigned)grid, 256, smem, st>>>(a.xs, a.offsets, a.n_groups, a.n_first, a.wg, a.wu,
                                                               a.sg, a.su, a.H, a.d, kc, a.h, a.rows_cap);
    } else {
        const long long grid = row_tiles * cdiv(a.d, FN);
        const int smem = ffn_f32_smem<false>(kc);
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(ffn_f32_kernel<false>), smem);
        if (e != cudaSuccess) return cuda_status(e);
        ffn_f32_kernel<false><<<(unsigned)grid, 256, smem, st>>>(a.h, a.offsets, a.n_groups, a.n_first, a.wd, nullptr,
                                                                a.sd, nullptr, a.d, a.H, kc, a.ys, a.rows_cap);
    }
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
