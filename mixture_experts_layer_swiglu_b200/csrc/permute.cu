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
// Atomic kind (N up to millions of experts, ~2 tasks each), two launches:
//   a kernel zeroes the counts and a barrier counter; one cooperative kernel
//   (every block resident) then runs histogram (integer atomics, each slot
//   keeping the count its atomic returned as its rank) -> per-block totals ->
//   exclusive scan -> placement at the expert's offset plus the rank ->
//   per-expert sort of each short segment by slot id (= token order), which
//   fixes the order whatever order the atomics took; the phases are separated
//   by a grid barrier whose waits are bounded (2 s, then MOE_ERR_TIMEOUT).

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <climits>

#include "common.cuh"
#include "e4m3.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int P_TOK = 256;        // tokens per count / scatter block
constexpr int P_MAXE = 1024;      // max FFN experts of the mask kernels

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

// ---- the atomic-kind permutation in one cooperative kernel

constexpr int AP_THREADS = 1024;       // one block per SM: few spinners at each grid barrier
constexpr int AP_MAX_BLOCKS = 4096;    // blocksum entries in the workspace

// Grid barrier number `phase` (1, 2, ...) on a counter zeroed before the
// launch: every block adds one and waits for phase * gridDim.x arrivals.
// The cooperative launch makes every block resident, so the wait ends; it is
// still bounded.  Returns false (MOE_ERR_TIMEOUT recorded) if it gave up.
__device__ __forceinline__ bool ap_grid_sync(unsigned* bar, unsigned phase, int* s_ok)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();                                    // this block's writes before its arrival
        atomicAdd(bar, 1u);
        const unsigned target = phase * gridDim.x;
        bool ok = true;
        const uint64_t t0 = globaltimer();
        unsigned v;
        for (uint32_t i = 0;; ++i) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
            if (v >= target) break;
            if (i >= 32) __nanosleep(64);                   // then back off: every block polls one line
            if ((i & 63u) == 63u && globaltimer() - t0 > kWaitLimitNs) { ok = false; break; }
        }
        if (!ok) set_status(MOE_ERR_TIMEOUT);
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Sum of v over the block (all threads get it).
__device__ __forceinline__ int ap_block_sum(int v, int* red)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int i = 0; i < AP_THREADS / 32; ++i) t += red[i];
    return t;
}

// ---- the SwiGLU-kind permutation in one cooperative kernel
//
// The same count / scan / scatter steps as the kernels above, in one launch
// (every block resident, one grid barrier after the counts), with the scan
// done by every block for itself (it reads all [chunks x experts] counts and
// keeps the bases of the chunks it places: no second barrier) and the gather
// turned around: each block takes an equal range of tokens, rebuilds the
// expert masks of the 256-token chunks its range touches, places its tokens'
// tasks, and copies each of its tokens' x row once from HBM into all its
// destination rows (the token's FFN slots and the shared experts' rows),
// 16-byte vectors, eight in flight per lane.  The small steps then cost no
// launch of their own and the row copies start right after the barrier.
constexpr int PF_THREADS = 512;
constexpr int PF_MAXDST = 8;        // destination rows per token held in shared memory (k + n_shared)
constexpr int PF_MAXCOUNTS = 16384; // [chunks x experts] counts that every block reads
static_assert(P_TOK * PF_MAXDST >= 2 * P_MAXE, "per-expert sums share s_dst's storage");

// Expert masks of chunk c (threads < P_TOK each take one token); false on a bad id.
__device__ __forceinline__ bool pf_masks(const PermuteArgs& a, uint32_t (*mask)[8], int c)
{
    for (int i = threadIdx.x; i < a.n_ffn * 8; i += blockDim.x) mask[i >> 3][i & 7] = 0u;
    __syncthreads();
    bool ok = true;
    const int t = c * P_TOK + threadIdx.x;
    if (threadIdx.x < P_TOK && t < a.T) {
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

// Exclusive prefix of v over the block's threads in thread order, and the
// block total in *total (all threads).
__device__ __forceinline__ int pf_block_scan(int v, int* warp_tot, int* total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    __syncthreads();                        // warp_tot of an earlier call read by everyone
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < PF_THREADS / 32; ++w) {
        const int x = warp_tot[w];
        before += w < warp ? x : 0;
        all += x;
    }
    *total = all;
    return before + incl - v;
}

// QUANT: the destination rows get the e4m3 codes of the token's row (and its
// scale); a separate instance, so the bf16 copy keeps its registers.
template <bool QUANT>
__global__ void __launch_bounds__(PF_THREADS, 2) perm_fused_kernel(const PermuteArgs a, unsigned* bar, int nb)
{
    __shared__ uint32_t mask[P_MAXE][8];
    __shared__ int s_dst[P_TOK][PF_MAXDST];        // destination rows of the chunk-range's tokens
    __shared__ int sbase[P_MAXE];                  // next row of each expert's tasks
    __shared__ int warp_tot[32];
    __shared__ int s_ok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = PF_THREADS / 32;

    // 1. counts of chunk c in [blocks x experts]
    for (int c = blockIdx.x; c < nb; c += gridDim.x) {
        if (!pf_masks(a, mask, c)) set_status(MOE_ERR_DEVICE_BOUNDS);
        for (int e = tid; e < a.n_ffn; e += PF_THREADS) {
            int n = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) n += __popc(mask[e][w]);
            a.ws_counts[(long long)c * a.n_ffn + e] = n;
        }
        __syncthreads();   // the masks are rebuilt for the next chunk
    }
    if (!ap_grid_sync(bar, 1, &s_ok)) return;

    // 2. every block: from all the counts, the row at which each expert's
    //    tasks of the first chunk it places begin (the exclusive sum in
    //    (expert, chunk) order); block 0 also writes the offsets
    const int tpb = cdiv(a.T, gridDim.x);
    const int lo = min(a.T, (int)blockIdx.x * tpb), hi = min(a.T, lo + tpb);
    const int cfirst = lo / P_TOK;
    // per expert, its total and its count before chunk cfirst: every thread
    // adds a strided share of the counts with shared-memory integer atomics
    // (into s_dst's storage, free until the placement)
    int* tot_s = &s_dst[0][0];
    int* cum_s = tot_s + P_MAXE;
    for (int e = tid; e < a.n_ffn; e += PF_THREADS) { tot_s[e] = 0; cum_s[e] = 0; }
    __syncthreads();
    {
        const int L = nb * a.n_ffn;
        const int lim = cfirst * a.n_ffn;          // entries of the chunks before cfirst
#pragma unroll 4
        for (int l = tid; l < L; l += PF_THREADS) {
            const int v = a.ws_counts[l];
            const int e = l % a.n_ffn;
            if (v) {
                atomicAdd(&tot_s[e], v);
                if (l < lim) atomicAdd(&cum_s[e], v);
            }
        }
    }
    __syncthreads();
    int tot[2] = {0, 0}, cum[2] = {0, 0};       // experts tid and tid + PF_THREADS
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int e = tid + u * PF_THREADS;
        if (e < a.n_ffn) { tot[u] = tot_s[e]; cum[u] = cum_s[e]; }
    }
    int tot0, tot1;
    const int ex0 = pf_block_scan(tot[0], warp_tot, &tot0);
    const int ex1 = pf_block_scan(tot[1], warp_tot, &tot1) + tot0;
    const int R = tot0 + tot1;                  // rows of the FFN experts
    if (tid < a.n_ffn) sbase[tid] = ex0 + cum[0];
    if (tid + PF_THREADS < a.n_ffn) sbase[tid + PF_THREADS] = ex1 + cum[1];
    if (blockIdx.x == 0) {
        if (tid < a.n_ffn) a.offsets[tid] = ex0;
        if (tid + PF_THREADS < a.n_ffn) a.offsets[tid + PF_THREADS] = ex1;
        if (tid == 0) {
            a.offsets[a.n_ffn] = R;
            for (int sh = 0; sh < a.n_shared; ++sh) a.offsets[a.n_ffn + sh + 1] = R + (sh + 1) * a.T;
        }
    }
    __syncthreads();

    // 3. this block's tokens: their rows, then the row copies
    const int ndst = a.k + a.n_shared;
    const long long rows_cap = (long long)a.T * a.k + (long long)a.n_shared * a.T;
    const int vecs = a.d * a.elt_bytes / 16;
    const uint4* x = reinterpret_cast<const uint4*>(a.x);
    uint4* xs = reinterpret_cast<uint4*>(a.x_sorted);
    for (int c = lo / P_TOK; c * P_TOK < hi; ++c) {
        pf_masks(a, mask, c);
        const int t0 = max(lo, c * P_TOK), t1 = min(hi, c * P_TOK + P_TOK);
        const int t = c * P_TOK + tid;
        if (tid < P_TOK && t >= t0 && t < t1) {
            const int w = tid >> 5;
            const uint32_t below = (1u << (tid & 31)) - 1u;
            for (int j = 0; j < a.k; ++j) {
                const int e = a.idx[(long long)t * a.k + j];
                int r = -1;
                if (e >= 0 && e < a.n_ffn) {
                    r = sbase[e];
                    for (int ww = 0; ww < w; ++ww) r += __popc(mask[e][ww]);
                    r += __popc(mask[e][w] & below);
                    a.token_of[r] = t;
                }
                a.row_of[(long long)t * a.k + j] = r;
                if (j < PF_MAXDST) s_dst[tid][j] = r;
            }
            for (int sh = 0; sh < a.n_shared; ++sh) {
                const long long r = (long long)R + (long long)sh * a.T + t;
                a.token_of[r] = t;
                if (a.k + sh < PF_MAXDST) s_dst[tid][a.k + sh] = (int)r;
            }
        }
        __syncthreads();
        // the next chunk's tasks of expert e begin after this chunk's
        for (int e = tid; e < a.n_ffn; e += PF_THREADS) {
            int n = 0;
#pragma unroll
            for (int w = 0; w < 8; ++w) n += __popc(mask[e][w]);
            sbase[e] += n;
        }
        if (QUANT && xs) {
            // e4m3 rows (d a multiple of 256): one warp per token reads x[t]
            // for its max, then again (from L1 / L2) to write the same codes
            // into every destination row, and the row scale beside each
            uint8_t* xq = static_cast<uint8_t*>(a.x_sorted);
            const int nv = a.d / 256;                      // 8-element vectors per lane
            for (int tt = t0 + warp; tt < t1; tt += NW) {
                const int ti = tt - c * P_TOK;
                const uint4* src = x + (long long)tt * vecs;
                float amax = 0.f;
                for (int i = 0; i < nv; ++i) {
                    float v[8];
                    bf16x8(__ldg(src + i * 32 + lane), v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const float sc = pow2_scale(amax), inv = 1.f / sc;   // inverse of a power of two: exact
                for (int i = 0; i < nv; ++i) {
                    float v[8];
                    bf16x8(__ldg(src + i * 32 + lane), v);
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[j] *= inv;
                    const uint2 q = to_e4m3x8(v);
                    for (int j = 0; j < ndst && j < PF_MAXDST; ++j) {
                        const int r = s_dst[ti][j];
                        if (r < 0 || r >= rows_cap) continue;
                        reinterpret_cast<uint2*>(xq + (long long)r * a.d)[i * 32 + lane] = q;
                    }
                }
                if (lane < ndst && lane < PF_MAXDST) {
                    const int r = s_dst[ti][lane];
                    if (r >= rows_cap) set_status(MOE_ERR_DEVICE_BOUNDS);
                    else if (r >= 0) a.xs_scale[r] = sc;
                }
            }
        } else if (!QUANT && xs) {
            // one warp per token: each 16-byte vector of x[t] is read once and
            // stored to every destination row
            for (int tt = t0 + warp; tt < t1; tt += NW) {
                const int ti = tt - c * P_TOK;
                const uint4* src = x + (long long)tt * vecs;
                for (int i0 = 0; i0 < vecs; i0 += 32 * 8) {
                    uint4 v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (i0 + u * 32 + lane < vecs) v[u] = __ldg(src + i0 + u * 32 + lane);
                    for (int j = 0; j < ndst && j < PF_MAXDST; ++j) {
                        const int r = s_dst[ti][j];
                        if (r < 0) continue;
                        if (r >= rows_cap) { if (lane == 0) set_status(MOE_ERR_DEVICE_BOUNDS); continue; }
                        uint4* dst = xs + (long long)r * vecs;
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            if (i0 + u * 32 + lane < vecs) dst[i0 + u * 32 + lane] = v[u];
                    }
                }
            }
        }
        __syncthreads();   // s_dst and the masks are rebuilt for the next chunk
    }
}

constexpr int AP_SORT = 16;            // segment length sorted in registers

// Ascending bitonic sort of N (a power of two) values held in registers.
template <int N>
__device__ __forceinline__ void sort_net_asc(int (&v)[N])
{
#pragma unroll
    for (int k = 2; k <= N; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool up = (i & k) == 0;
                    const int lo = min(v[i], v[l]), hi = max(v[i], v[l]);
                    v[i] = up ? lo : hi;
                    v[l] = up ? hi : lo;
                }
            }
}

__global__ void __launch_bounds__(AP_THREADS) atomic_permute_kernel(const PermuteArgs a, unsigned* bar)
{
    __shared__ int red[AP_THREADS / 32];
    __shared__ int s_ok;
    const long long n = (long long)a.T * a.k;
    const int N = a.n_ids;
    const long long gstride = (long long)gridDim.x * blockDim.x;
    const long long gtid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    // 1. histogram; each slot keeps the count its atomic returned (its rank
    //    among its expert's tasks, in whatever order the atomics took) in
    //    row_of until the placement, four slots per thread and step
    for (long long s0 = gtid; s0 < n; s0 += 4 * gstride) {
        int e[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long sl = s0 + u * gstride;
            e[u] = sl < n ? a.idx[sl] : -1;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long sl = s0 + u * gstride;
            if (sl >= n) continue;
            if (e[u] < 0 || e[u] >= N) {
                set_status(MOE_ERR_DEVICE_BOUNDS);
                a.row_of[sl] = -1;
            } else {
                a.row_of[sl] = atomicAdd(&a.ws_counts[e[u]], 1);
            }
        }
    }
    if (!ap_grid_sync(bar, 1, &s_ok)) return;
    // 2. this block's chunk of experts and its total
    const int chunk = cdiv(N, gridDim.x);
    const int lo = min(N, (int)blockIdx.x * chunk), hi = min(N, lo + chunk);
    int part = 0;
    for (int e = lo + threadIdx.x; e < hi; e += AP_THREADS) part += a.ws_counts[e];
    const int total = ap_block_sum(part, red);
    if (threadIdx.x == 0) a.ws_blocksum[blockIdx.x] = total;
    if (!ap_grid_sync(bar, 2, &s_ok)) return;
    // 3. exclusive scan: the totals of the blocks before this one, then the chunk
    int pre = 0;
    for (int b = threadIdx.x; b < (int)blockIdx.x; b += AP_THREADS) pre += a.ws_blocksum[b];
    int run = ap_block_sum(pre, red);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int base = lo; base < hi; base += AP_THREADS) {
        const int e = base + threadIdx.x;
        const int c = e < hi ? a.ws_counts[e] : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        __syncthreads();
        if (lane == 31) red[w] = incl;
        __syncthreads();
        int wpre = 0;
        for (int i = 0; i < w; ++i) wpre += red[i];
        int step = 0;
#pragma unroll
        for (int i = 0; i < AP_THREADS / 32; ++i) step += red[i];
        if (e < hi) a.offsets[e] = run + wpre + incl - c;
        run += step;
    }
    if (hi == N && lo < hi && threadIdx.x == 0) a.offsets[N] = run;
    if (!ap_grid_sync(bar, 3, &s_ok)) return;
    // 4. placement at the expert's offset plus the slot's rank from the
    //    histogram (any order inside a segment; sorted next): no atomics
    for (long long s0 = gtid; s0 < n; s0 += 4 * gstride) {
        int e[4], r[4], o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const long long sl = s0 + u * gstride;
            e[u] = sl < n ? a.idx[sl] : -1;
            r[u] = sl < n ? a.row_of[sl] : -1;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) o[u] = (e[u] >= 0 && e[u] < N && r[u] >= 0) ? a.offsets[e[u]] : -1;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (o[u] >= 0) a.token_of[o[u] + r[u]] = (int)(s0 + u * gstride);
    }
    if (!ap_grid_sync(bar, 4, &s_ok)) return;
    // 5. each expert's segment sorted by slot id, and row_of.  A segment of
    // up to AP_SORT tasks (product-key routing gives 2.4 per touched expert,
    // 14 at most on the 8192-token workload) is loaded into registers with
    // independent loads, sorted by a fixed compare-exchange network and
    // written back: one memory round trip instead of the dependent global
    // reads and writes of an in-place insertion sort, whose longest segments
    // bounded the whole phase.  Longer segments are sorted in place.
    // (the next expert's offsets are loaded while this one is sorted)
    int nx0 = gtid < N ? a.offsets[gtid] : 0, nx1 = gtid < N ? a.offsets[gtid + 1] : 0;
    for (long long e = gtid; e < N; e += gstride) {
        const int s0 = nx0, s1 = nx1;
        if (e + gstride < N) { nx0 = a.offsets[e + gstride]; nx1 = a.offsets[e + gstride + 1]; }
        if (s1 - s0 <= AP_SORT) {
            int v[AP_SORT];
#pragma unroll
            for (int i = 0; i < AP_SORT; ++i) v[i] = s0 + i < s1 ? a.token_of[s0 + i] : INT_MAX;
            sort_net_asc(v);
#pragma unroll
            for (int i = 0; i < AP_SORT; ++i)
                if (s0 + i < s1) {
                    a.token_of[s0 + i] = v[i];
                    a.row_of[v[i]] = s0 + i;
                }
            continue;
        }
        for (int i = s0 + 1; i < s1; ++i) {
            const int v = a.token_of[i];
            int j = i - 1;
            while (j >= s0 && a.token_of[j] > v) { a.token_of[j + 1] = a.token_of[j]; --j; }
            a.token_of[j + 1] = v;
        }
        for (int i = s0; i < s1; ++i) a.row_of[a.token_of[i]] = i;
    }
}

int ap_grid(int N)
{
    static std::atomic<int> per_sm[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    int b = per_sm[dev].load(std::memory_order_relaxed);
    if (b == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, atomic_permute_kernel, AP_THREADS, 0) != cudaSuccess ||
            b <= 0)
            b = 1;
        per_sm[dev].store(b, std::memory_order_relaxed);
    }
    (void)N;
    return std::max(1, std::min(std::min(b, 1) * num_sms(), AP_MAX_BLOCKS));
}

}  // namespace

int permute_blocks(int T) { return std::max(1, cdiv(T, P_TOK)); }
// ints after the counts in the atomic kind's workspace: the block totals, then the barrier counter
int atomic_scan_blocks(int N) { (void)N; return AP_MAX_BLOCKS + 64; }

// Blocks of the fused kernel that are resident together (0 if none fit).
static int pf_grid()
{
    static int per_sm[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (per_sm[dev] == 0) {
        int n = 0, m = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, perm_fused_kernel<false>, PF_THREADS, 0) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, perm_fused_kernel<true>, PF_THREADS, 0) != cudaSuccess)
            n = 0;
        n = std::min(n, m);
        per_sm[dev] = n > 0 ? n : -1;
    }
    return per_sm[dev] > 0 ? std::min(per_sm[dev], 2) * num_sms() : 0;
}

moe_status launch_permute_swiglu(const PermuteArgs& a, cudaStream_t st)
{
    if (a.n_ffn > P_MAXE) return MOE_ERR_UNSUPPORTED;
    const int nb = permute_blocks(a.T);
    // (every block reads all the counts: the one-launch form is for up to PF_MAXCOUNTS of them;
    // small batches take one block per 8 tokens, so the grid barrier waits on few blocks)
    const int grid = a.bar && a.T > 0 && a.k + a.n_shared <= PF_MAXDST && (long long)nb * a.n_ffn <= PF_MAXCOUNTS
                         ? std::min(pf_grid(), std::max(1, cdiv(a.T, 8))) : 0;
    if (grid > 0) {   // one cooperative launch (its barrier counter cleared first)
        cudaError_t e = cudaMemsetAsync(a.bar, 0, sizeof(unsigned), st);
        if (e != cudaSuccess) return cuda_status(e);
        PermuteArgs args = a;
        // e4m3 rows: with four or more destination rows per token (shared
        // experts, large k) this kernel quantizes each token's row once and
        // writes its codes to all of them; with fewer, the quantizing gather
        // below (one warp per permuted row) measured faster
        const bool quant_here = a.xs_scale && a.d % 256 == 0 && a.k + a.n_shared >= 4;
        if (a.xs_scale && !quant_here) args.x_sorted = nullptr;
        unsigned* bar = a.bar;
        int nbv = nb;
        void* params[3] = {&args, &bar, &nbv};
        e = cudaLaunchCooperativeKernel(quant_here ? reinterpret_cast<const void*>(perm_fused_kernel<true>)
                                                   : reinterpret_cast<const void*>(perm_fused_kernel<false>),
                                        dim3(grid), dim3(PF_THREADS), params, 0, st);
        if (e != cudaSuccess) return cuda_status(e);
        count_launch();
        if (a.x_sorted && a.xs_scale && !quant_here) {
            const long long rows_cap = (long long)a.T * a.k + (long long)a.n_shared * a.T;
            moe_status s = launch_gather_quant(a.token_of, a.offsets, a.n_ffn + a.n_shared, a.x, a.d, a.T, a.x_sorted,
                                               a.xs_scale, rows_cap, st);
            if (s != MOE_OK) return s;
        }
        return cuda_status(cudaGetLastError());
    }
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
    unsigned* bar = reinterpret_cast<unsigned*>(a.ws_blocksum + AP_MAX_BLOCKS);
    // counts, block totals and the barrier counter are one contiguous zeroed
    // range (the counts' 256-byte padding included)
    int32_t* zero_end = a.ws_blocksum + AP_MAX_BLOCKS + 64;
    const long long nz = zero_end - a.ws_counts;
    zero_i32_kernel<<<std::max(1, (int)std::min<long long>((nz + 1023) / 1024, num_sms() * 4)), 256, 0, st>>>(a.ws_counts, nz);
    count_launch();
    PermuteArgs args = a;
    void* params[2] = {&args, &bar};
    cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(atomic_permute_kernel), dim3(ap_grid(N)),
                                                dim3(AP_THREADS), params, 0, st);
    if (e != cudaSuccess) return cuda_status(e);
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
