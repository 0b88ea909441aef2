// permute.cu -- expert-centric grouping of the routing decisions.
//
// "OmniMoE" technical summary, 2.2 Expert-Centric Scheduling: all routing
// decisions of the batch form one task list, grouped by expert id and, inside
// a group, sorted by token id.  For a given routing this order is unique, and
// it is produced deterministically (no atomics decide any position):
//
// SwiGLU kind (few experts, <= 1024):
//   1. count:   each block takes 256 tokens; a bitmask per expert marks the
//               block's tokens that chose it; popcounts give the counts;
//   2. scan:    one block turns the [blocks x experts] counts into exclusive
//               bases in (expert, block) order and writes the offsets;
//   3. scatter: a task's row = base(block, expert) + number of earlier
//               tokens of the block in the expert's mask;
//   4. gather:  x_sorted[r] = x[token_of[r]] with 16-byte vector copies,
//               one warp per row.
// Shared experts get groups n_ffn.. holding every token in order.
//
// Atomic kind (N up to millions of experts, ~2 tasks each):
//   histogram with integer atomics, a three-kernel exclusive scan (no
//   cross-block waits), placement through per-expert cursors, then each
//   expert's short segment is sorted by slot id (= token order), which fixes
//   the order whatever order the atomics took.

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int P_TOK = 256;        // tokens per count / scatter block
constexpr int P_MAXE = 1024;      // max FFN experts of the mask kernels
constexpr int SCAN_ELEMS = 4096;  // elements per block of the atomic-kind scan

__device__ __forceinline__ bool build_masks(const PermuteArgs& a, uint32_t (*mask)[8], int b)
{
    for (int i = threadIdx.x; i < a.n_ffn * 8; i += blockDim.x) mask[i >> 3][i & 7] = 0u;
    __syncthreads();
    const int t = b * P_TOK + threadIdx.x;
    bool ok = true;
    if (t < a.T) {
        for (int j = 0; j < a.k; ++j) {
            const int e = a.idx[(long long)t * a.k + j];
            if (e < 0 || e >= a.n_ids) { ok = false; continue; }
            if (e < a.n_ffn) {
                const uint32_t bit = 1u << (threadIdx.x & 31);
                const uint32_t old = atomicOr(&mask[e][threadIdx.x >> 5], bit);
                if (old & bit) ok = false;      // same expert twice in one token
            }
        }
    }
    __syncthreads();
    return ok;
}

__global__ void __launch_bounds__(P_TOK) perm_count_kernel(const PermuteArgs a)
{
    __shared__ uint32_t mask[P_MAXE][8];
    const int b = blockIdx.x;
    if (!build_masks(a, mask, b)) set_status(MOE_ERR_DEVICE_BOUNDS);
    for (int e = threadIdx.x; e < a.n_ffn; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) c += __popc(mask[e][w]);
        a.ws_counts[(long long)b * a.n_ffn + e] = c;
    }
}

// Exclusive scan of counts in (expert, block) order; in place.
__global__ void __launch_bounds__(1024) perm_scan_kernel(const PermuteArgs a, int nb)
{
    __shared__ int warp_tot[32];
    __shared__ int s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long L = (long long)a.n_ffn * nb;
    const long long per = (L + 1023) / 1024;
    const long long lo = std::min<long long>(L, tid * per), hi = std::min<long long>(L, lo + per);
    int s = 0;
    for (long long l = lo; l < hi; ++l) {
        const long long e = l / nb, b = l % nb;
        s += a.ws_counts[b * a.n_ffn + e];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        warp_tot[lane] = wi - w;
        if (lane == 31) s_total = wi;
    }
    __syncthreads();
    int base = warp_tot[warp] + incl - s;
    for (long long l = lo; l < hi; ++l) {
        const long long e = l / nb, b = l % nb;
        const long long ix = b * a.n_ffn + e;
        const int c = a.ws_counts[ix];
        a.ws_counts[ix] = base;
        if (b == 0) a.offsets[e] = base;
        base += c;
    }
    if (nb == 0)
        for (int e = tid; e < a.n_ffn; e += blockDim.x) a.offsets[e] = 0;
    if (tid == 0) {
        const int R = nb == 0 ? 0 : s_total;
        a.offsets[a.n_ffn] = R;
        for (int sh = 0; sh < a.n_shared; ++sh) a.offsets[a.n_ffn + sh + 1] = R + (sh + 1) * a.T;
    }
}

__global__ void __launch_bounds__(P_TOK) perm_scatter_kernel(const PermuteArgs a)
{
    __shared__ uint32_t mask[P_MAXE][8];
    const int b = blockIdx.x;
    build_masks(a, mask, b);
    const int t = b * P_TOK + threadIdx.x;
    if (t >= a.T) return;
    const int w = threadIdx.x >> 5;
    const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
    for (int j = 0; j < a.k; ++j) {
        const int e = a.idx[(long long)t * a.k + j];
        int r = -1;
        if (e >= 0 && e < a.n_ffn) {
            r = a.ws_counts[(long long)b * a.n_ffn + e];
            for (int ww = 0; ww < w; ++ww) r += __popc(mask[e][ww]);
            r += __popc(mask[e][w] & below);
            a.token_of[r] = t;
        }
        a.row_of[(long long)t * a.k + j] = r;
    }
    const int R = a.offsets[a.n_ffn];
    for (int sh = 0; sh < a.n_shared; ++sh) a.token_of[(long long)R + (long long)sh * a.T + t] = t;
}

// x_sorted[r] = x[token_of[r]] for r < offsets[n_last]; row of `vecs` 16-byte vectors.
__global__ void __launch_bounds__(256) gather_rows_kernel(const int32_t* __restrict__ token_of,
                                                          const int32_t* __restrict__ offsets,
                                                          int n_last, const uint4* __restrict__ x,
                                                          uint4* __restrict__ xs, int vecs,
                                                          long long rows_cap, int T)
{
    const int lane = threadIdx.x & 31;
    const long long total = std::min<long long>(offsets[n_last], rows_cap);
    const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long r = blockIdx.x * (long long)(blockDim.x >> 5) + (threadIdx.x >> 5); r < total; r += nw) {
        const int t = token_of[r];
        if (t < 0 || t >= T) { if (lane == 0) set_status(MOE_ERR_DEVICE_BOUNDS); continue; }
        const uint4* src = x + (long long)t * vecs;
        uint4* dst = xs + r * vecs;
        int i = lane;
        for (; i + 96 < vecs; i += 128) {
            const uint4 v0 = __ldg(src + i), v1 = __ldg(src + i + 32);
            const uint4 v2 = __ldg(src + i + 64), v3 = __ldg(src + i + 96);
            dst[i] = v0; dst[i + 32] = v1; dst[i + 64] = v2; dst[i + 96] = v3;
        }
        for (; i < vecs; i += 32) dst[i] = __ldg(src + i);
    }
}

// ------------------------------------------------------------- atomic kind

__global__ void zero_i32_kernel(int32_t* p, long long n)
{
    const long long n4 = n / 4;   // p is 16-byte aligned
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x)
        reinterpret_cast<int4*>(p)[i] = make_int4(0, 0, 0, 0);
    for (long long i = n4 * 4 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        p[i] = 0;
}

__global__ void atomic_count_kernel(const PermuteArgs a)
{
    const long long n = (long long)a.T * a.k;
    for (long long s = blockIdx.x * (long long)blockDim.x + threadIdx.x; s < n;
         s += (long long)gridDim.x * blockDim.x) {
        const int e = a.idx[s];
        if (e < 0 || e >= a.n_ids) { set_status(MOE_ERR_DEVICE_BOUNDS); continue; }
        atomicAdd(&a.ws_counts[e], 1);
    }
}

__device__ __forceinline__ int block_excl_scan_1024(int v, int* warp_tot, int* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_tot[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        warp_tot[lane] = wi - w;
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    const int r = warp_tot[warp] + incl - v;
    __syncthreads();
    return r;
}

// pass 1: per-block totals of SCAN_ELEMS counts
__global__ void __launch_bounds__(1024) atomic_scan1_kernel(const int32_t* counts, int N, int32_t* blocksum)
{
    __shared__ int wt[32];
    __shared__ int tot;
    const long long base = (long long)blockIdx.x * SCAN_ELEMS + threadIdx.x * 4;
    int s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) if (base + i < N) s += counts[base + i];
    block_excl_scan_1024(s, wt, &tot);
    if (threadIdx.x == 0) blocksum[blockIdx.x] = tot;
}

// pass 2: offsets[e] = (sum of the totals of the blocks before this one) +
// exclusive scan inside the block; each block sums the preceding totals
// itself (nb <= 4096), so no third pass is needed.
__global__ void __launch_bounds__(1024) atomic_scan2_kernel(const int32_t* counts, int N,
                                                            const int32_t* blocksum, int32_t* offsets)
{
    __shared__ int wt[32];
    __shared__ int tot;
    int pre = 0;
    for (int i = threadIdx.x; i < (int)blockIdx.x; i += blockDim.x) pre += blocksum[i];
    block_excl_scan_1024(pre, wt, &tot);
    const int base_sum = tot;                  // sum of all preceding block totals
    const long long base = (long long)blockIdx.x * SCAN_ELEMS + threadIdx.x * 4;
    int v[4], s = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[i] = (base + i < N) ? counts[base + i] : 0; s += v[i]; }
    int run = base_sum + block_excl_scan_1024(s, wt, &tot);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (base + i < N) offsets[base + i] = run;
        run += v[i];
        if (base + i == N - 1) offsets[N] = run;
    }
}

__global__ void atomic_place_kernel(const PermuteArgs a)
{
    const long long n = (long long)a.T * a.k;
    for (long long s = blockIdx.x * (long long)blockDim.x + threadIdx.x; s < n;
         s += (long long)gridDim.x * blockDim.x) {
        const int e = a.idx[s];
        if (e < 0 || e >= a.n_ids) { a.row_of[s] = -1; continue; }
        const int pos = a.offsets[e] + atomicSub(&a.ws_counts[e], 1) - 1;   // any order; sorted next
        a.token_of[pos] = (int)s;
    }
}

// Sort each expert's segment by slot id and record row_of.
__global__ void atomic_sort_kernel(const PermuteArgs a)
{
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < a.n_ids;
         e += (long long)gridDim.x * blockDim.x) {
        const int lo = a.offsets[e], hi = a.offsets[e + 1];
        for (int i = lo + 1; i < hi; ++i) {
            const int v = a.token_of[i];
            int j = i - 1;
            while (j >= lo && a.token_of[j] > v) { a.token_of[j + 1] = a.token_of[j]; --j; }
            a.token_of[j + 1] = v;
        }
        for (int i = lo; i < hi; ++i) a.row_of[a.token_of[i]] = i;
    }
}

}  // namespace

int permute_blocks(int T) { return std::max(1, cdiv(T, P_TOK)); }
int atomic_scan_blocks(int N) { return std::max(1, cdiv(N, SCAN_ELEMS)); }

moe_status launch_permute_swiglu(const PermuteArgs& a, cudaStream_t st)
{
    if (a.n_ffn > P_MAXE) return MOE_ERR_UNSUPPORTED;
    const int nb = permute_blocks(a.T);
    if (a.T > 0 && a.n_ffn > 0) {
        perm_count_kernel<<<nb, P_TOK, 0, st>>>(a);
        count_launch();
    }
    perm_scan_kernel<<<1, 1024, 0, st>>>(a, a.T > 0 ? nb : 0);
    count_launch();
    if (a.T > 0) {
        perm_scatter_kernel<<<nb, P_TOK, 0, st>>>(a);
        count_launch();
        if (a.x_sorted && a.xs_scale) {   // e4m3 codes of the rows and their scales
            const long long rows_cap = (long long)a.T * a.k + (long long)a.n_shared * a.T;
            moe_status s = launch_gather_quant(a.token_of, a.offsets, a.n_ffn + a.n_shared, a.x, a.d, a.T, a.x_sorted,
                                               a.xs_scale, rows_cap, st);
            if (s != MOE_OK) return s;
        } else if (a.x_sorted) {
            const int vecs = a.d * a.elt_bytes / 16;
            const long long rows_cap = (long long)a.T * a.k + (long long)a.n_shared * a.T;
            const int grid = (int)std::max<long long>(1, std::min<long long>((rows_cap + 7) / 8, num_sms() * 16));
            gather_rows_kernel<<<grid, 256, 0, st>>>(a.token_of, a.offsets, a.n_ffn + a.n_shared,
                                                     reinterpret_cast<const uint4*>(a.x),
                                                     reinterpret_cast<uint4*>(a.x_sorted), vecs, rows_cap, a.T);
            count_launch();
        }
    }
    return cuda_status(cudaGetLastError());
}

moe_status launch_permute_atomic(const PermuteArgs& a, cudaStream_t st)
{
    const int N = a.n_ids;
    const int grid_n = std::max(1, std::min(cdiv(N, 256), num_sms() * 8));
    zero_i32_kernel<<<std::max(1, std::min(cdiv(N, 1024), num_sms() * 4)), 256, 0, st>>>(a.ws_counts, N);
    const long long n = (long long)a.T * a.k;
    const int grid_t = (int)std::max<long long>(1, std::min<long long>((n + 255) / 256, num_sms() * 8));
    atomic_count_kernel<<<grid_t, 256, 0, st>>>(a);
    const int nb = atomic_scan_blocks(N);
    if (nb > 4096) return MOE_ERR_UNSUPPORTED;
    atomic_scan1_kernel<<<nb, 1024, 0, st>>>(a.ws_counts, N, a.ws_blocksum);
    atomic_scan2_kernel<<<nb, 1024, 0, st>>>(a.ws_counts, N, a.ws_blocksum, a.offsets);
    atomic_place_kernel<<<grid_t, 256, 0, st>>>(a);
    atomic_sort_kernel<<<grid_n, 256, 0, st>>>(a);
    count_launch(6);
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
