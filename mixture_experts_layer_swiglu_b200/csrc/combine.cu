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
// Phase A loads its operands straight into registers with 32-byte loads;
// phase B streams whole v rows through a warp-private ring of shared-memory
// stages filled by bulk copies.

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

// C: 8-element chunks per lane and step; BYP: the layer has zero-computation
// experts (without them the x and constant-vector paths are compiled out and
// the registers go to more loads in flight).
template <typename T, typename TO, int C, int MINB, bool BYP>
__global__ void __launch_bounds__(256, MINB) combine_kernel(const CombineArgs a)
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
    __shared__ int s_ffn[TPB];                       // the token has an FFN slot (accumulator row written)
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
        if (live && part == 0) {
            const bool f = lane < a.k && a.idx[t * a.k + lane] >= 0 && a.idx[t * a.k + lane] < zero0;
            const unsigned m = __ballot_sync(FULL, f);
            if (lane == 0) s_ffn[tib] = m != 0u;
        }
        __syncthreads();
        if (live) {
            // C chunks of 8 elements per lane and step; the slots are
            // taken in pairs, the rows of both (expert output, or constant
            // vector) loaded before either is added, so 2 C independent
            // 32-byte row loads per lane are in flight; the sum runs in slot order
            for (int i = i0 + lane; i < i1; i += 32 * C) {
                float acc[C][V];
#pragma unroll
                for (int u = 0; u < C; ++u)
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[u][v] = 0.f;
                if (a.acc_rows && s_ffn[tib]) {      // the FFN slots' sum, formed by the down GEMM
                    for (int u = 0; u < C; ++u)
                        if (i + 32 * u < i1) load8<float>(a.ys, t * vecs + i + 32 * u, acc[u]);
                }
                for (int s = 0; s < a.n_shared; ++s) {
                    const long long r = (long long)a.offsets[a.n_ffn + s] + t;
                    if (r < a.rows_cap) {
                        float w[C][V];
                        for (int u = 0; u < C; ++u)
                            if (i + 32 * u < i1) load8<float>(a.ys, r * vecs + i + 32 * u, w[u]);
#pragma unroll
                        for (int u = 0; u < C; ++u)
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[u][v] += w[u][v];
                    }
                }
                bool have_x = false;
                float xv[C][V];
                for (int j0 = 0; j0 < a.k; j0 += 2) {
                    float pw[2][C][V];                       // slot j0 + p: its row (FFN output or constant vector)
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int j = j0 + p;
                        const int e = j < a.k ? s_e[tib][j] : -1;
                        if (e < 0) continue;
                        if (e < zero0) {
                            if (!a.acc_rows) {
                                const long long rb = (long long)s_r[tib][j] * vecs;
                                for (int u = 0; u < C; ++u)
                                    if (i + 32 * u < i1) load8<float>(a.ys, rb + i + 32 * u, pw[p][u]);
                            }
                        } else if (BYP && e >= copy0) {      // copy and constant experts read x
                            if (!have_x) {
                                for (int u = 0; u < C; ++u)
                                    if (i + 32 * u < i1) load8<T>(a.x, t * vecs + i + 32 * u, xv[u]);
                                have_x = true;
                            }
                            if (e >= const0) {
                                const long long cb = (long long)(e - const0) * vecs;
                                for (int u = 0; u < C; ++u)
                                    if (i + 32 * u < i1) load8<T>(a.const_vec, cb + i + 32 * u, pw[p][u]);
                            }
                        }
                    }
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int j = j0 + p;
                        const int e = j < a.k ? s_e[tib][j] : -1;
                        if (e < 0) continue;
                        const float g = s_g[tib][j];
                        if (e < zero0) {
                            if (a.acc_rows) continue;            // already in the accumulator row
#pragma unroll
                            for (int u = 0; u < C; ++u)
#pragma unroll
                                for (int v = 0; v < V; ++v) acc[u][v] = fmaf(g, pw[p][u][v], acc[u][v]);
                        } else if (!BYP || e < copy0) {
                            // zero expert: contributes nothing
                        } else if (e < const0) {
#pragma unroll
                            for (int u = 0; u < C; ++u)
#pragma unroll
                                for (int v = 0; v < V; ++v) acc[u][v] = fmaf(g, xv[u][v], acc[u][v]);
                        } else {
                            const float a1 = s_a1[tib][j], a2 = s_a2[tib][j];
#pragma unroll
                            for (int u = 0; u < C; ++u)
#pragma unroll
                                for (int v = 0; v < V; ++v)
                                    acc[u][v] = fmaf(g, a1 * xv[u][v] + a2 * pw[p][u][v], acc[u][v]);
                        }
                    }
                }
                for (int u = 0; u < C; ++u)
                    if (i + 32 * u < i1) store8<TO>(a.y, t * vecs + i + 32 * u, acc[u]);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- atomic

// Per task p of the expert-sorted order: its expert (task_expert[p] = e for
// p in [offsets[e], offsets[e+1])) and its gate (task_gate[p] = gate[slot]).
__global__ void atomic_task_meta_kernel(const AtomicArgs a)
{
    const long long cap = (long long)a.T * a.K;
    const int R = (int)min((long long)a.offsets[a.N], cap);
    const long long n = max((long long)a.N, (long long)R);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        if (i < a.N) {
            const int lo = a.offsets[i], hi = a.offsets[i + 1];
            if (lo < 0 || hi > cap || lo > hi) set_status(MOE_ERR_DEVICE_BOUNDS);
            else
                for (int p = lo; p < hi; ++p) a.task_expert[p] = (int)i;
        }
        if (i < R) {
            const int s = a.token_of[i];
            a.task_gate[i] = (s >= 0 && s < cap) ? a.gate[s] : 0.f;
        }
    }
}


// ---- phase A: c[s] = g[s] * GELU(u_e . x_t) for every task.
//
// A warp takes units of 16 consecutive tasks of the expert-sorted order.
// The unit's distinct experts (at most 16, about 7 at 2.4 tasks per expert)
// are the columns of one or two m16n8 tiles; D[i][j] = x_{t_i} . u_{e_j}
// accumulates over d on the tensor cores and task i keeps D[i][its column].
// Operands come straight from global memory into registers with 32-byte
// loads: for each 64-element slice of d, lane (g, q) loads bytes
// [32q, 32q + 32) of its A rows (tasks g, g+8) and B rows (columns g, g+8),
// so one warp instruction reads 8 whole 128-byte lines, and those 16
// elements feed four k16 steps.  The k order this implies (step s takes
// elements 16q + 4s + {0,1} as k = 2q, 2q+1 and 16q + 4s + {2,3} as k = 2q+8,
// 2q+9) is the same for A and B, so the sums are the dot products.  x rows
// come from L2, each touched u row from HBM once per unit it appears in;
// occupancy (16 warps per SM, each with up to 12 KiB of loads in flight)
// hides the latency.
constexpr int AT_M = 16;
constexpr int PA_WARPS = 4;
#ifndef MOE_PA_U1
#define MOE_PA_U1 4      // 64-element slices loaded together, one-tile units
#endif
#ifndef MOE_PA_U2
#define MOE_PA_U2 2      // the same, two-tile units
#endif
#ifndef MOE_PA_MINB
#define MOE_PA_MINB 4    // resident blocks per SM
#endif
static_assert(4 % MOE_PA_U1 == 0 && 4 % MOE_PA_U2 == 0, "slice groups must divide d / 64 for d = 256");

struct PaRaw {       // lane i < 16: task i of a unit
    int s, e;
    float g;
};

__device__ __forceinline__ PaRaw pa_load(const AtomicArgs& a, int un, int units, int R, long long cap, int lane)
{
    PaRaw r{-1, -1, 0.f};
    const int p = un * AT_M + lane;
    if (un < units && lane < AT_M && p < R) {
        const int s = a.token_of[p], e = a.task_expert[p];
        if (s < 0 || s >= cap || e < 0 || e >= a.N) {
            set_status(MOE_ERR_DEVICE_BOUNDS);
        } else {
            r.s = s;
            r.e = e;
            r.g = a.task_gate[p];
        }
    }
    return r;
}


// D += the products of the 64-element slices of d, in groups of U slices
// whose loads are issued together (one tile: U * 3 KiB per warp in flight,
// two tiles: U * 4 KiB).  Measured on B200 for d = 1024, groups of 4 / 2
// slices at 16 warps per SM beat both smaller groups at higher occupancy and
// double-buffered groups.  U divides the slice count for every supported d.
template <int NT>
__device__ __forceinline__ void pa_dot(const unsigned char* xr0, const unsigned char* xr1, const unsigned char* ur0,
                                       const unsigned char* ur1, int nsc, int q, float (&d0)[4], float (&d1)[4])
{
    constexpr int U = NT == 1 ? MOE_PA_U1 : MOE_PA_U2;
#pragma unroll 1
    for (int sc = 0; sc < nsc; sc += U) {
        uint32_t xa[U][8], xb[U][8], ua[U][8], ub[NT == 2 ? U : 1][8];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int off = (sc + u) * 128 + q * 32;
            ld256(xr0 + off, xa[u]);
            ld256(xr1 + off, xb[u]);
            ld256(ur0 + off, ua[u]);
            if constexpr (NT == 2) ld256(ur1 + off, ub[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                mma_16816(d0, xa[u][2 * st], xb[u][2 * st], xa[u][2 * st + 1], xb[u][2 * st + 1], ua[u][2 * st],
                          ua[u][2 * st + 1]);
                if constexpr (NT == 2)
                    mma_16816(d1, xa[u][2 * st], xb[u][2 * st], xa[u][2 * st + 1], xb[u][2 * st + 1], ub[u][2 * st],
                              ub[u][2 * st + 1]);
            }
    }
}

__global__ void __launch_bounds__(PA_WARPS * 32, MOE_PA_MINB) atomic_phase_a_kernel(const AtomicArgs a)
{
    __shared__ int col_expert[PA_WARPS][AT_M];
    __shared__ int task_slot[PA_WARPS][AT_M], task_col[PA_WARPS][AT_M];
    __shared__ float task_g[PA_WARPS][AT_M];
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, wib = threadIdx.x >> 5;
    const long long cap = (long long)a.T * a.K;
    const int R = (int)min((long long)a.offsets[a.N], cap);
    const int units = (R + AT_M - 1) / AT_M;
    const int nsc = a.d / 64;
    const size_t rowb = (size_t)a.d * 2;
    const unsigned char* xb = static_cast<const unsigned char*>(a.x);
    const unsigned char* ub = static_cast<const unsigned char*>(a.u);
    const int nw = gridDim.x * PA_WARPS;
    int un = blockIdx.x * PA_WARPS + wib;
    PaRaw r = pa_load(a, un, units, R, cap, lane);
    for (; un < units; un += nw) {
        const int eprev = __shfl_up_sync(FULL, r.e, 1);
        const bool fresh = r.e >= 0 && (lane == 0 || r.e != eprev);
        const unsigned nm = __ballot_sync(FULL, fresh);
        const int ndist = __popc(nm);
        const int col = __popc(nm & ((2u << (lane & (AT_M - 1))) - 1u)) - 1;
        if (fresh) col_expert[wib][col] = r.e;
        if (lane < AT_M) {
            task_slot[wib][lane] = r.s;
            task_col[wib][lane] = col;
            task_g[wib][lane] = r.g;
        }
        __syncwarp();
        const int s0 = task_slot[wib][g], s1 = task_slot[wib][g + 8];
        const int last = max(ndist - 1, 0);
        const unsigned char* xr0 = xb + (size_t)(s0 >= 0 ? s0 / a.K : 0) * rowb;
        const unsigned char* xr1 = xb + (size_t)(s1 >= 0 ? s1 / a.K : 0) * rowb;
        const unsigned char* ur0 = ub + (size_t)(ndist ? col_expert[wib][min(g, last)] : 0) * rowb;
        const unsigned char* ur1 = ub + (size_t)(ndist ? col_expert[wib][min(g + 8, last)] : 0) * rowb;
        r = pa_load(a, un + nw, units, R, cap, lane);   // next unit, in flight meanwhile
        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
        if (ndist > 8) pa_dot<2>(xr0, xr1, ur0, ur1, nsc, q, d0, d1);
        else pa_dot<1>(xr0, xr1, ur0, ur1, nsc, q, d0, d1);
        // D fragment: d[0], d[1] = row g, columns 2q, 2q+1; d[2], d[3] = row g+8.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int sr = task_slot[wib][g + 8 * h], kr = task_col[wib][g + 8 * h];
            if (sr < 0) continue;
            const int tile = kr >> 3, cc = kr & 7;
            if ((cc >> 1) != q) continue;
            const float lo = tile ? d1[2 * h] : d0[2 * h];
            const float hi = tile ? d1[2 * h + 1] : d0[2 * h + 1];
            const float dot = (cc & 1) ? hi : lo;
            const float gel = 0.5f * dot * (1.0f + erff(dot * 0.70710678118654752f));
            a.c[sr] = task_g[wib][g + 8 * h] * gel;
        }
    }
}

// Waits (bounded) for every stage still being filled; used on the way out
// after a failed wait, so that no copy into this block's shared memory is
// in flight when it exits.
template <int NST>
__device__ __forceinline__ void drain_stages(uint64_t* full, uint32_t pend, uint32_t ph)
{
    for (int st = 0; st < NST; ++st)
        if ((pend >> st) & 1u) mbar_wait(&full[st], (ph >> st) & 1u);
}

// ---- phase B: y_t = sum_j c[t, j] v_{e_tj}, one warp per token, fp32 in slot order.
//
// The token's v rows stream through a warp-private ring of 4 KiB stages
// (8/NV rows each, one bulk copy per row), three stages ahead and across
// tokens; lane l accumulates the 16-byte vectors l + 32 i of the row with
// packed fp32x2 FMAs.
constexpr int PB_WARPS = 12;
constexpr int PB_STAGES = 4;
constexpr int PB_STAGE = 4096;

template <int NV>
__global__ void __launch_bounds__(PB_WARPS * 32, 1) atomic_phase_b_kernel(const AtomicArgs a)
{
    extern __shared__ __align__(16) unsigned char pb_smem[];
    constexpr int RPS = 8 / NV;          // rows per stage
    constexpr int ROWB = NV * 512;       // bytes per row
    const int wib = threadIdx.x >> 5;
    unsigned char* ring = pb_smem + wib * (PB_STAGES * PB_STAGE);
    uint64_t* full = reinterpret_cast<uint64_t*>(pb_smem + PB_WARPS * PB_STAGES * PB_STAGE) + wib * PB_STAGES;
    const int lane = threadIdx.x & 31;
    const int ns = (a.K + RPS - 1) / RPS;
    const int nw = gridDim.x * PB_WARPS;
    const int t0 = blockIdx.x * PB_WARPS + wib;
    if (t0 >= a.T) return;
    if (lane == 0) {
        for (int st = 0; st < PB_STAGES; ++st) mbar_init(&full[st], 1);
        fence_barrier_init();
    }
    __syncwarp();
    const unsigned char* vb = static_cast<const unsigned char*>(a.v);

    auto pick = [](const int (&r)[4], int j) { return j < 32 ? r[0] : j < 64 ? r[1] : j < 96 ? r[2] : r[3]; };
    auto pickf = [](const float (&r)[4], int j) { return j < 32 ? r[0] : j < 64 ? r[1] : j < 96 ? r[2] : r[3]; };
    // expert ids of token t (lane + 32 i); an invalid id reads row 0 with weight 0
    auto load_e = [&](int t, int (&E)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = lane + 32 * i;
            int e = 0;
            if (t < a.T && j < a.K) {
                e = a.idx[(long long)t * a.K + j];
                if (e < 0 || e >= a.N) e = 0;
            }
            E[i] = e;
        }
    };
    auto load_c = [&](int t, float (&C)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = lane + 32 * i;
            float c = 0.f;
            if (t < a.T && j < a.K) {
                const int e = a.idx[(long long)t * a.K + j];
                if (e < 0 || e >= a.N) set_status(MOE_ERR_DEVICE_BOUNDS);
                else c = a.c[(long long)t * a.K + j];
            }
            C[i] = c;
        }
    };

    uint32_t ph = 0, pend = 0;
    int ti = t0, ki = 0;
    int Ei[4], Ep[4];
    load_e(ti, Ei);
    load_e(ti + nw, Ep);
    auto issue = [&](int st) {
        if (ti >= a.T) return;
        const int j0 = ki * RPS;
        const int rows = min(RPS, a.K - j0);
        if (lane == 0) mbar_arrive_expect_tx(&full[st], rows * ROWB);
        __syncwarp();
        // lane rr < rows copies row rr of the stage
        int e = 0;
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr) {
            const int j = min(j0 + rr, a.K - 1);
            const int er = __shfl_sync(FULL, pick(Ei, j), j & 31);
            if (lane == rr) e = er;
        }
        if (lane < rows) bulk_g2s(ring + st * PB_STAGE + lane * ROWB, vb + (size_t)e * ROWB, ROWB, &full[st]);
        pend |= 1u << st;
        if (++ki == ns) {
            ki = 0;
            ti += nw;
#pragma unroll
            for (int i = 0; i < 4; ++i) Ei[i] = Ep[i];
            load_e(ti + nw, Ep);
        }
    };

    int tc = t0, kc = 0;
    float Cc[4], Cp[4];
    load_c(tc, Cc);
    load_c(tc + nw, Cp);
    float acc[NV][8];
#pragma unroll
    for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[v][i] = 0.f;
    for (int s = 0; s < PB_STAGES - 1; ++s) issue(s);
    int cons = 0;
    while (tc < a.T) {
        const int cst = cons % PB_STAGES;
        if (!__all_sync(FULL, mbar_wait(&full[cst], (ph >> cst) & 1u))) {
            drain_stages<PB_STAGES>(full, pend & ~(1u << cst), ph);
            return;
        }
        ph ^= 1u << cst;
        pend &= ~(1u << cst);
        const unsigned char* st = ring + cst * PB_STAGE;
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr) {
            const int j = kc * RPS + rr;
            if (j < a.K) {
                const float c = __shfl_sync(FULL, pickf(Cc, j), j & 31);
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    const uint4 w = *reinterpret_cast<const uint4*>(st + rr * ROWB + (lane + 32 * v) * 16);
                    fma2(acc[v][0], acc[v][1], c, bf16_lo(w.x), bf16_hi(w.x));
                    fma2(acc[v][2], acc[v][3], c, bf16_lo(w.y), bf16_hi(w.y));
                    fma2(acc[v][4], acc[v][5], c, bf16_lo(w.z), bf16_hi(w.z));
                    fma2(acc[v][6], acc[v][7], c, bf16_lo(w.w), bf16_hi(w.w));
                }
            }
        }
        __syncwarp();
        issue((cons + PB_STAGES - 1) % PB_STAGES);
        ++cons;
        if (++kc == ns) {
            const int vecs = a.d / 8;
            if (a.shared_out) {   // the shared dense branch, added before the one rounding
                const float4* sp = reinterpret_cast<const float4*>(a.shared_out);
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    const long long o = ((long long)tc * vecs + v * 32 + lane) * 2;
                    const float4 s0 = sp[o], s1 = sp[o + 1];
                    acc[v][0] += s0.x; acc[v][1] += s0.y; acc[v][2] += s0.z; acc[v][3] += s0.w;
                    acc[v][4] += s1.x; acc[v][5] += s1.y; acc[v][6] += s1.z; acc[v][7] += s1.w;
                }
            }
            if (a.out_f32) {
                float4* y = reinterpret_cast<float4*>(a.y);
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    const long long o = ((long long)tc * vecs + v * 32 + lane) * 2;
                    y[o] = make_float4(acc[v][0], acc[v][1], acc[v][2], acc[v][3]);
                    y[o + 1] = make_float4(acc[v][4], acc[v][5], acc[v][6], acc[v][7]);
                }
            } else {
                uint4* y = reinterpret_cast<uint4*>(a.y);
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    y[(long long)tc * vecs + v * 32 + lane] =
                        make_uint4(pack_bf16(acc[v][0], acc[v][1]), pack_bf16(acc[v][2], acc[v][3]),
                                   pack_bf16(acc[v][4], acc[v][5]), pack_bf16(acc[v][6], acc[v][7]));
            }
#pragma unroll
            for (int v = 0; v < NV; ++v)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[v][i] = 0.f;
            kc = 0;
            tc += nw;
#pragma unroll
            for (int i = 0; i < 4; ++i) Cc[i] = Cp[i];
            load_c(tc + nw, Cp);
        }
    }
}

template <template <int> class K, typename... Args>
moe_status launch_nv(int nv, int grid, cudaStream_t st, const AtomicArgs& a)
{
    cudaError_t e;
    switch (nv) {
        case 1: e = K<1>::launch(grid, st, a); break;
        case 2: e = K<2>::launch(grid, st, a); break;
        case 4: e = K<4>::launch(grid, st, a); break;
        case 8: e = K<8>::launch(grid, st, a); break;
        default: return MOE_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return cuda_status(e);
    count_launch();
    return cuda_status(cudaGetLastError());
}

constexpr int kPbSmem = PB_WARPS * PB_STAGES * (PB_STAGE + 8);

template <int NV> struct PhaseB {
    static cudaError_t launch(int grid, cudaStream_t st, const AtomicArgs& a)
    {
        const cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(atomic_phase_b_kernel<NV>), kPbSmem);
        if (e != cudaSuccess) return e;
        atomic_phase_b_kernel<NV><<<grid, PB_WARPS * 32, kPbSmem, st>>>(a);
        return cudaSuccess;
    }
};

}  // namespace

moe_status launch_combine(int dtype, const CombineArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    if (a.k > CMB_MAXK) return MOE_ERR_UNSUPPORTED;
    const int grid = std::max(1, std::min(cdiv(a.T, 256 / 32 / CMB_SPLIT), num_sms() * 16));
    // FFN slots only (no zero-computation experts, no shared rows): two chunks per lane
    // (measured on the Mixtral-shaped layer: 38.4 -> 37.0 us; with shared rows it did not gain)
    const bool ffn_only = a.n_zero + a.n_copy + a.n_const == 0 && a.n_shared == 0;
    if (dtype == MOE_BF16 && !a.out_f32 && ffn_only) combine_kernel<__nv_bfloat16, __nv_bfloat16, 2, 3, false><<<grid, 256, 0, st>>>(a);
    else if (dtype == MOE_BF16 && !a.out_f32) combine_kernel<__nv_bfloat16, __nv_bfloat16, 1, 4, true><<<grid, 256, 0, st>>>(a);
    else if (dtype == MOE_BF16) combine_kernel<__nv_bfloat16, float, 1, 4, true><<<grid, 256, 0, st>>>(a);
    else combine_kernel<float, float, 1, 4, true><<<grid, 256, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_atomic_phase_a(const AtomicArgs& a, cudaStream_t st)
{
    const long long cap = (long long)a.T * a.K;
    if (cap == 0) return MOE_OK;
    if (a.d % 256 != 0) return MOE_ERR_UNSUPPORTED;
    const long long n = std::max((long long)a.N, cap);
    const int g0 = (int)std::max(1LL, std::min<long long>((n + 255) / 256, num_sms() * 8));
    atomic_task_meta_kernel<<<g0, 256, 0, st>>>(a);
    count_launch();
    const long long units = (cap + AT_M - 1) / AT_M;
    const int grid = (int)std::max(1LL, std::min<long long>((units + PA_WARPS - 1) / PA_WARPS, num_sms() * MOE_PA_MINB));
    atomic_phase_a_kernel<<<grid, PA_WARPS * 32, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_atomic_phase_b(const AtomicArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    if (a.K > 128) return MOE_ERR_UNSUPPORTED;
    const int grid = std::max(1, std::min(cdiv(a.T, PB_WARPS), num_sms()));
    return launch_nv<PhaseB>(a.d / 256, grid, st, a);
}

}  // namespace moe
