// combine.cu -- gate-weighted combine back to token order, MoE++
// zero-computation experts, and the two passes of the atomic-expert layer.
//
// Combine ("OmniMoE" technical summary, 2.1: the routed outputs are
// assembled per token, the shared dense branch is always added; "MoE++"
// summary, "Approach": zero expert = discard, copy expert = identity,
// constant expert = trainable vector mixed with the input):
//   y_t = sum_s y_sorted[shared row of t] + sum_j g_tj O_tj
// accumulated in fp32 in slot order and rounded once.  Four warps per token,
// each a quarter of the row, 16- and 32-byte vector loads (HBM-bound: reads
// the k expert rows and, for copy/constant experts, x; writes y).
//
// Atomic experts ("OmniMoE" 2.1 Atomic Experts E_i(x) = sigma(x . u_i) v_i,
// Dynamic Expert Assembly; 2.2 Expert-Centric Scheduling):
//   phase A, over the expert-sorted tasks: the dot products u_e . x_t of 16
//     consecutive tasks are one m16n8k16 tile sequence (x stays in L2, each
//     touched u_e is read once): c[s] = g[s] * GELU(u_e . x_t);
//   phase B, token by token: y_t = sum_j c[t, j] v_{e_tj}, fp32 in slot order.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr unsigned FULL = 0xffffffffu;

template <typename T> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const void* p, long long i, float (&v)[8])
    {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
        v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
        v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
    }
    __device__ static void store(void* p, long long i, const float (&v)[8])
    {
        reinterpret_cast<uint4*>(p)[i] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                    pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
    }
};
template <> struct Chunk<float> {
    static constexpr int N = 4;
    __device__ static void load(const void* p, long long i, float (&v)[4])
    {
        const float4 f = __ldg(reinterpret_cast<const float4*>(p) + i);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
    __device__ static void store(void* p, long long i, const float (&v)[4])
    {
        reinterpret_cast<float4*>(p)[i] = make_float4(v[0], v[1], v[2], v[3]);
    }
};

constexpr int CMB_MAXK = 32;

// y_sorted rows are fp32 (expert outputs are not rounded before the combine);
// x, the constant vectors and y are T.  Chunks of 8 elements for both types.
template <typename T>
__device__ __forceinline__ void load8(const void* p, long long i8, float (&v)[8])
{
    if constexpr (sizeof(T) == 2) {
        Chunk<__nv_bfloat16>::load(p, i8, v);
    } else {
        float a[4], b[4];
        Chunk<float>::load(p, 2 * i8, a);
        Chunk<float>::load(p, 2 * i8 + 1, b);
#pragma unroll
        for (int i = 0; i < 4; ++i) { v[i] = a[i]; v[4 + i] = b[i]; }
    }
}

template <typename T>
__device__ __forceinline__ void store8(void* p, long long i8, const float (&v)[8])
{
    if constexpr (sizeof(T) == 2) {
        Chunk<__nv_bfloat16>::store(p, i8, v);
    } else {
        const float a[4] = {v[0], v[1], v[2], v[3]}, b[4] = {v[4], v[5], v[6], v[7]};
        Chunk<float>::store(p, 2 * i8, a);
        Chunk<float>::store(p, 2 * i8 + 1, b);
    }
}

// One token per group of CMB_SPLIT warps, each warp a contiguous quarter of
// the row (more rows in flight per SM than one warp per token).
constexpr int CMB_SPLIT = 4;

template <typename T, typename TO>
__global__ void __launch_bounds__(256, 3) combine_kernel(const CombineArgs a)
{
    constexpr int V = 8;
    constexpr int WPB = 256 / 32;                    // warps per block
    constexpr int TPB = WPB / CMB_SPLIT;             // tokens per block
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int tib = wib / CMB_SPLIT, part = wib % CMB_SPLIT;
    const int vecs = a.d / V;
    const int per = cdiv(vecs, CMB_SPLIT);
    const int i0 = part * per, i1 = min(vecs, i0 + per);
    const int zero0 = a.n_ffn, copy0 = zero0 + a.n_zero, const0 = copy0 + a.n_copy;
    const int n_ids = const0 + a.n_const;
    __shared__ int s_e[TPB][CMB_MAXK], s_r[TPB][CMB_MAXK];
    __shared__ float s_g[TPB][CMB_MAXK], s_a1[TPB][CMB_MAXK], s_a2[TPB][CMB_MAXK];
    for (long long base = (long long)blockIdx.x * TPB; base < a.T; base += (long long)gridDim.x * TPB) {
        const long long t = base + tib;
        const bool live = t < a.T;
        // slot j's id, gate, row and constant mix, staged by lane j of part 0
        if (live && part == 0 && lane < a.k) {
            int e = a.idx[t * a.k + lane];
            const int r = a.row_of[t * a.k + lane];
            bool bad = e < 0 || e >= n_ids;
            if (!bad && e < zero0 && (r < 0 || r >= a.rows_cap)) bad = true;
            if (bad) { set_status(MOE_ERR_DEVICE_BOUNDS); e = -1; }
            float a1 = 0.f, a2 = 0.f;
            if (e >= const0) {
                const int c = e - const0;
                a1 = a.const_mix[(t * a.n_const + c) * 2 + 0];
                a2 = a.const_mix[(t * a.n_const + c) * 2 + 1];
            }
            s_e[tib][lane] = e;
            s_r[tib][lane] = r;
            s_g[tib][lane] = a.gate[t * a.k + lane];
            s_a1[tib][lane] = a1;
            s_a2[tib][lane] = a2;
        }
        __syncthreads();
        if (live) {
            // two chunks per lane and step: their row loads are independent
            for (int i = i0 + lane; i < i1; i += 64) {
                const bool two = i + 32 < i1;
                float acc[2][V];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[u][v] = 0.f;
                for (int s = 0; s < a.n_shared; ++s) {
                    const long long r = (long long)a.offsets[a.n_ffn + s] + t;
                    if (r < a.rows_cap) {
                        float w[2][V];
                        load8<float>(a.ys, r * vecs + i, w[0]);
                        if (two) load8<float>(a.ys, r * vecs + i + 32, w[1]);
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[u][v] += w[u][v];
                    }
                }
                bool have_x = false;
                float xv[2][V];
                for (int j = 0; j < a.k; ++j) {
                    const int e = s_e[tib][j];
                    const float g = s_g[tib][j];
                    if (e < 0) continue;
                    if (e < zero0) {
                        const long long rb = (long long)s_r[tib][j] * vecs;
                        float w[2][V];
                        load8<float>(a.ys, rb + i, w[0]);
                        if (two) load8<float>(a.ys, rb + i + 32, w[1]);
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[u][v] = fmaf(g, w[u][v], acc[u][v]);
                    } else if (e < copy0) {
                        // zero expert: contributes nothing
                    } else {
                        if (!have_x) {
                            load8<T>(a.x, t * vecs + i, xv[0]);
                            if (two) load8<T>(a.x, t * vecs + i + 32, xv[1]);
                            have_x = true;
                        }
                        if (e < const0) {
#pragma unroll
                            for (int u = 0; u < 2; ++u)
#pragma unroll
                                for (int v = 0; v < V; ++v) acc[u][v] = fmaf(g, xv[u][v], acc[u][v]);
                        } else {
                            const float a1 = s_a1[tib][j], a2 = s_a2[tib][j];
                            const long long cb = (long long)(e - const0) * vecs;
                            float cv[2][V];
                            load8<T>(a.const_vec, cb + i, cv[0]);
                            if (two) load8<T>(a.const_vec, cb + i + 32, cv[1]);
#pragma unroll
                            for (int u = 0; u < 2; ++u)
#pragma unroll
                                for (int v = 0; v < V; ++v) acc[u][v] = fmaf(g, a1 * xv[u][v] + a2 * cv[u][v], acc[u][v]);
                        }
                    }
                }
                store8<TO>(a.y, t * vecs + i, acc[0]);
                if (two) store8<TO>(a.y, t * vecs + i + 32, acc[1]);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- atomic

// Expert of every task: task_expert[p] = e for p in [offsets[e], offsets[e+1]).
__global__ void atomic_task_expert_kernel(const int32_t* offsets, int N, long long cap, int32_t* te)
{
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < N;
         e += (long long)gridDim.x * blockDim.x) {
        const int lo = offsets[e], hi = offsets[e + 1];
        if (lo < 0 || hi > cap || lo > hi) {
            set_status(MOE_ERR_DEVICE_BOUNDS);
            continue;
        }
        for (int p = lo; p < hi; ++p) te[p] = (int)e;
    }
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

constexpr int AT_M = 16;       // tasks per warp unit
constexpr int AT_UNROLL = 4;   // 32-element chunks of d whose loads are issued together

// D[i][j] += x_{t_i} . u_{e_j} over d for the 16 task rows i and NT*8 expert
// columns j.  Chunk c covers elements [32c, 32c + 32); lane (g, q) loads the
// 16 bytes at 32c + 8q of its A rows (tasks g, g + 8) and B rows (columns g,
// g + 8) and feeds them to two k16 steps, so A and B agree on the k order.
template <int NT>
__device__ __forceinline__ void atomic_dot_tiles(const uint4* xr0, const uint4* xr1, const uint4* ur0,
                                                 const uint4* ur1, int chunks, int q, float (&d0)[4],
                                                 float (&d1)[4])
{
    for (int c0 = 0; c0 < chunks; c0 += AT_UNROLL) {
        uint4 xa[AT_UNROLL], xb[AT_UNROLL], ua[AT_UNROLL], ub[AT_UNROLL];
#pragma unroll
        for (int c = 0; c < AT_UNROLL; ++c) {
            const int o = (c0 + c) * 4 + q;
            xa[c] = __ldg(xr0 + o);
            xb[c] = __ldg(xr1 + o);
            ua[c] = __ldg(ur0 + o);
            if (NT == 2) ub[c] = __ldg(ur1 + o);
        }
#pragma unroll
        for (int c = 0; c < AT_UNROLL; ++c) {
            mma_16816(d0, xa[c].x, xb[c].x, xa[c].y, xb[c].y, ua[c].x, ua[c].y);
            mma_16816(d0, xa[c].z, xb[c].z, xa[c].w, xb[c].w, ua[c].z, ua[c].w);
            if (NT == 2) {
                mma_16816(d1, xa[c].x, xb[c].x, xa[c].y, xb[c].y, ub[c].x, ub[c].y);
                mma_16816(d1, xa[c].z, xb[c].z, xa[c].w, xb[c].w, ub[c].z, ub[c].w);
            }
        }
    }
}

// phase A: c[s] = g[s] * GELU(u_e . x_t) for every task (s = slot t*K + j,
// e its expert).  A warp takes 16 consecutive tasks of the expert-sorted
// order; their distinct experts (at most 16, about 7 at 2.4 tasks per
// expert) are the columns of one or two m16n8 tiles, and task i keeps
// D[i][column of its expert].  Each touched u_e is read once per unit it
// appears in (x stays in L2); the tensor cores do the dot products.
__global__ void __launch_bounds__(256, 2) atomic_phase_a_kernel(const AtomicArgs a)
{
    __shared__ int col_expert[8][AT_M];
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int wib = threadIdx.x >> 5;
    const long long cap = (long long)a.T * a.K;
    const int R = (int)min((long long)a.offsets[a.N], cap);
    const int units = (R + AT_M - 1) / AT_M;
    const int vecs = a.d >> 3;
    const int chunks = a.d >> 5;
    const uint4* x = reinterpret_cast<const uint4*>(a.x);
    const uint4* u = reinterpret_cast<const uint4*>(a.u);
    const int nw = gridDim.x * (blockDim.x >> 5);
    for (int un = blockIdx.x * (blockDim.x >> 5) + wib; un < units; un += nw) {
        const int p = un * AT_M + (lane & (AT_M - 1));
        int s = -1, e = -1;
        float gt = 0.f;
        if (lane < AT_M && p < R) {
            s = a.token_of[p];
            e = a.task_expert[p];
            if (s < 0 || s >= cap || e < 0 || e >= a.N) {
                set_status(MOE_ERR_DEVICE_BOUNDS);
                s = -1;
                e = -1;
            } else {
                gt = a.gate[s];
            }
        }
        const int eprev = __shfl_up_sync(FULL, e, 1);
        const bool fresh = lane < AT_M && e >= 0 && (lane == 0 || e != eprev);
        const unsigned nm = __ballot_sync(FULL, fresh);
        const int ndist = __popc(nm);
        if (ndist == 0) continue;
        const int col = __popc(nm & ((2u << (lane & (AT_M - 1))) - 1u)) - 1;   // tasks: own column
        if (fresh) col_expert[wib][col] = e;
        __syncwarp();
        const int s0 = __shfl_sync(FULL, s, g), s1 = __shfl_sync(FULL, s, g + 8);
        const int k0 = __shfl_sync(FULL, col, g), k1 = __shfl_sync(FULL, col, g + 8);
        const float g0 = __shfl_sync(FULL, gt, g), g1 = __shfl_sync(FULL, gt, g + 8);
        const uint4* xr0 = x + (long long)(s0 >= 0 ? s0 / a.K : 0) * vecs;
        const uint4* xr1 = x + (long long)(s1 >= 0 ? s1 / a.K : 0) * vecs;
        const uint4* ur0 = u + (long long)col_expert[wib][min(g, ndist - 1)] * vecs;
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
        if (ndist <= 8) {
            atomic_dot_tiles<1>(xr0, xr1, ur0, ur0, chunks, q, d0, d1);
        } else {
            const uint4* ur1 = u + (long long)col_expert[wib][min(g + 8, ndist - 1)] * vecs;
            atomic_dot_tiles<2>(xr0, xr1, ur0, ur1, chunks, q, d0, d1);
        }
        __syncwarp();
        // D fragment: d[0], d[1] = row g, columns 2q, 2q+1; d[2], d[3] = row g+8.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int sr = h ? s1 : s0, kr = h ? k1 : k0;
            if (sr < 0) continue;
            const int tile = kr >> 3, cc = kr & 7;
            if ((cc >> 1) != q) continue;
            const float lo = tile ? d1[2 * h] : d0[2 * h];
            const float hi = tile ? d1[2 * h + 1] : d0[2 * h + 1];
            const float dot = (cc & 1) ? hi : lo;
            const float gel = 0.5f * dot * (1.0f + erff(dot * 0.70710678118654752f));
            a.c[sr] = (h ? g1 : g0) * gel;
        }
    }
}

// phase B: one warp per token; 4 v rows in flight per lane.
template <int NV>
__global__ void __launch_bounds__(256) atomic_phase_b_kernel(const AtomicArgs a)
{
    const int lane = threadIdx.x & 31;
    const uint4* v = reinterpret_cast<const uint4*>(a.v);
    const int vecs = a.d / 8;
    const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); t < a.T; t += nw) {
        float acc[NV][8];
#pragma unroll
        for (int q = 0; q < NV; ++q)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[q][i] = 0.f;
        for (int j0 = 0; j0 < a.K; j0 += 32) {
            const int my_e = (j0 + lane < a.K) ? a.idx[t * a.K + j0 + lane] : -1;
            const float my_c = (j0 + lane < a.K) ? a.c[t * a.K + j0 + lane] : 0.f;
            const int jn = min(32, a.K - j0);
            for (int jj = 0; jj < jn; ++jj) {
                const int e = __shfl_sync(FULL, my_e, jj);
                const float c = __shfl_sync(FULL, my_c, jj);
                if (e < 0 || e >= a.N) { if (lane == 0) set_status(MOE_ERR_DEVICE_BOUNDS); continue; }
                uint4 w[NV];
#pragma unroll
                for (int q = 0; q < NV; ++q) w[q] = __ldg(v + (long long)e * vecs + q * 32 + lane);
#pragma unroll
                for (int q = 0; q < NV; ++q) {
                    acc[q][0] = fmaf(c, bf16_lo(w[q].x), acc[q][0]); acc[q][1] = fmaf(c, bf16_hi(w[q].x), acc[q][1]);
                    acc[q][2] = fmaf(c, bf16_lo(w[q].y), acc[q][2]); acc[q][3] = fmaf(c, bf16_hi(w[q].y), acc[q][3]);
                    acc[q][4] = fmaf(c, bf16_lo(w[q].z), acc[q][4]); acc[q][5] = fmaf(c, bf16_hi(w[q].z), acc[q][5]);
                    acc[q][6] = fmaf(c, bf16_lo(w[q].w), acc[q][6]); acc[q][7] = fmaf(c, bf16_hi(w[q].w), acc[q][7]);
                }
            }
        }
        if (a.out_f32) {
            float4* y = reinterpret_cast<float4*>(a.y);
#pragma unroll
            for (int q = 0; q < NV; ++q) {
                const long long o = (t * vecs + q * 32 + lane) * 2;
                y[o] = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
                y[o + 1] = make_float4(acc[q][4], acc[q][5], acc[q][6], acc[q][7]);
            }
        } else {
            uint4* y = reinterpret_cast<uint4*>(a.y);
#pragma unroll
            for (int q = 0; q < NV; ++q)
                y[t * vecs + q * 32 + lane] = make_uint4(pack_bf16(acc[q][0], acc[q][1]), pack_bf16(acc[q][2], acc[q][3]),
                                                         pack_bf16(acc[q][4], acc[q][5]), pack_bf16(acc[q][6], acc[q][7]));
        }
    }
}

template <template <int> class K, typename... Args>
moe_status launch_nv(int nv, int grid, cudaStream_t st, const AtomicArgs& a)
{
    switch (nv) {
        case 1: K<1>::launch(grid, st, a); break;
        case 2: K<2>::launch(grid, st, a); break;
        case 4: K<4>::launch(grid, st, a); break;
        case 8: K<8>::launch(grid, st, a); break;
        default: return MOE_ERR_UNSUPPORTED;
    }
    count_launch();
    return cuda_status(cudaGetLastError());
}

template <int NV> struct PhaseB {
    static void launch(int grid, cudaStream_t st, const AtomicArgs& a)
    {
        atomic_phase_b_kernel<NV><<<grid, 256, 0, st>>>(a);
    }
};

}  // namespace

moe_status launch_combine(int dtype, const CombineArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    if (a.k > CMB_MAXK) return MOE_ERR_UNSUPPORTED;
    const int grid = std::max(1, std::min(cdiv(a.T, 256 / 32 / CMB_SPLIT), num_sms() * 16));
    if (dtype == MOE_BF16 && !a.out_f32) combine_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, st>>>(a);
    else if (dtype == MOE_BF16) combine_kernel<__nv_bfloat16, float><<<grid, 256, 0, st>>>(a);
    else combine_kernel<float, float><<<grid, 256, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_atomic_phase_a(const AtomicArgs& a, cudaStream_t st)
{
    const long long cap = (long long)a.T * a.K;
    if (cap == 0) return MOE_OK;
    if (a.d % 256 != 0) return MOE_ERR_UNSUPPORTED;
    const int g0 = (int)std::min<long long>((a.N + 255) / 256, num_sms() * 8);
    atomic_task_expert_kernel<<<std::max(1, g0), 256, 0, st>>>(a.offsets, a.N, cap, a.task_expert);
    count_launch();
    const long long units = (cap + AT_M - 1) / AT_M;
    const int grid = (int)std::max(1LL, std::min<long long>((units + 7) / 8, num_sms() * 2));
    atomic_phase_a_kernel<<<grid, 256, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_atomic_phase_b(const AtomicArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    const int grid = std::max(1, std::min(cdiv(a.T, 8), num_sms() * 16));
    return launch_nv<PhaseB>(a.d / 256, grid, st, a);
}

}  // namespace moe
