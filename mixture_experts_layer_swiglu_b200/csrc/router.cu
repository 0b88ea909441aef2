// router.cu -- router logits with warp-level top-k / softmax, and the
// Cartesian-product (product-key) selection of atomic experts.
//
// Router ("PCoMoE" summary, "The Limitation of Monolithic Expert
// Selection": a fixed set of k experts per token; "MoE++" summary,
// "Approach": gating residuals add the previous layer's router scores):
//   z = W_r x + bias + prev;  top-k by descending z, ties to the lower id;
//   gates = softmax over the selected logits.  Constant experts' mixing
//   logits W_c x are computed in the same pass over x.
// The pass over x is the cost (x is read once from HBM): each warp takes
// 4 tokens, lanes split d into 16-byte vectors, 8 router rows at a time are
// accumulated in fp32 and reduced across the warp with a transposing
// butterfly (31 shuffles for 32 sums).
//
// Product-key selection ("OmniMoE" technical summary, 2.2 Cartesian Product
// Router): from the row and column sub-key scores of each token, keep the
// best kh of each half, then merge the kh x kh candidate sums (each row's
// candidates are already sorted) into the best K.  Candidate sums of two
// fp32 scores are formed in fp64, which is exact, so the order is the exact
// order of the sums.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int R_TPW = 4;         // tokens per warp
constexpr int R_WARPS = 4;       // warps per block
constexpr int R_MAXROWS = 256;   // router rows + constant-mix rows

template <typename Tin> struct VecOf;
template <> struct VecOf<__nv_bfloat16> { static constexpr int N = 8; };
template <> struct VecOf<float> { static constexpr int N = 4; };

__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&v)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

__device__ __forceinline__ void load_vec(const float* p, float (&v)[4])
{
    const float4 f = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

// 32 values per lane -> lane l holds the warp-wide sum of value l.
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(FULL, send, off);
        }
    }
    return v[0];
}

// (value desc, id asc) order; NaN values never win.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

template <typename Tin>
__global__ void __launch_bounds__(R_WARPS * 32) router_kernel(const RouterArgs a)
{
    constexpr int V = VecOf<Tin>::N;
    __shared__ float s_logit[R_WARPS][R_TPW][R_MAXROWS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = a.E_r + 2 * a.n_const;
    const int n_tgroups = cdiv(a.T, R_TPW);
    const Tin* x = reinterpret_cast<const Tin*>(a.x);
    const Tin* wr = reinterpret_cast<const Tin*>(a.w_router);
    const Tin* wc = reinterpret_cast<const Tin*>(a.w_const_mix);
    float (*zs)[R_MAXROWS] = s_logit[warp];

    for (int grp = blockIdx.x * R_WARPS + warp; grp < n_tgroups; grp += gridDim.x * R_WARPS) {
        const int t0 = grp * R_TPW;
        for (int rc = 0; rc < R; rc += 8) {
            float acc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = 0.f;
            for (int i = lane * V; i < a.d; i += 32 * V) {
                float xv[R_TPW][V];
#pragma unroll
                for (int tt = 0; tt < R_TPW; ++tt) {
                    if (t0 + tt < a.T) load_vec(x + (long long)(t0 + tt) * a.d + i, xv[tt]);
                    else {
#pragma unroll
                        for (int v = 0; v < V; ++v) xv[tt][v] = 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int r = rc + q;
                    if (r < R) {
                        const Tin* wrow = r < a.E_r ? wr + (long long)r * a.d
                                                    : wc + (long long)(r - a.E_r) * a.d;
                        float wv[V];
                        load_vec(wrow + i, wv);
#pragma unroll
                        for (int tt = 0; tt < R_TPW; ++tt)
#pragma unroll
                            for (int v = 0; v < V; ++v)
                                acc[tt * 8 + q] = fmaf(xv[tt][v], wv[v], acc[tt * 8 + q]);
                    }
                }
            }
            const float s = transpose_reduce32(acc, lane);
            const int r = rc + (lane & 7);
            if (r < R) zs[lane >> 3][r] = s;
        }
        __syncwarp();

        for (int tt = 0; tt < R_TPW; ++tt) {
            const int t = t0 + tt;
            if (t >= a.T) break;
            float* z = zs[tt];
            for (int e = lane; e < a.E_r; e += 32) {
                float v = z[e];
                if (a.bias) v += a.bias[e];
                if (a.prev) v += a.prev[(long long)t * a.E_r + e];
                z[e] = v;
                if (a.logits_out) a.logits_out[(long long)t * a.E_r + e] = v;
            }
            __syncwarp();
            uint32_t taken = 0;   // bit i: expert lane + 32 i already selected
            float zsel = 0.f, z0 = 0.f;
            int isel = -1;
            for (int j = 0; j < a.k; ++j) {
                float bv = -INFINITY;
                int bi = INT_MAX;
                for (int i = 0; lane + 32 * i < a.E_r; ++i) {
                    if ((taken >> i) & 1u) continue;
                    const int e = lane + 32 * i;
                    const float v = z[e];
                    if (better(v, e, bv, bi)) { bv = v; bi = e; }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const float ov = __shfl_xor_sync(FULL, bv, o);
                    const int oi = __shfl_xor_sync(FULL, bi, o);
                    if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
                }
                if (bi != INT_MAX && (bi & 31) == lane) taken |= 1u << (bi >> 5);
                if (lane == j) { zsel = bv; isel = (bi == INT_MAX) ? -1 : bi; }
                if (j == 0) z0 = bv;
            }
            const float ex = (lane < a.k) ? expf(zsel - z0) : 0.f;
            float sum = ex;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
            if (lane < a.k) {
                a.idx[(long long)t * a.k + lane] = isel;
                a.gate[(long long)t * a.k + lane] = ex / sum;
            }
            for (int c = lane; c < a.n_const; c += 32) {
                const float l0 = z[a.E_r + 2 * c], l1 = z[a.E_r + 2 * c + 1];
                const float m = fmaxf(l0, l1);
                const float e0 = expf(l0 - m), e1 = expf(l1 - m);
                a.const_mix[((long long)t * a.n_const + c) * 2 + 0] = e0 / (e0 + e1);
                a.const_mix[((long long)t * a.n_const + c) * 2 + 1] = e1 / (e0 + e1);
            }
            __syncwarp();
        }
        __syncwarp();
    }
}

// ------------------------------------------------------- product-key selection

// Best kh of n scores (per lane: elements lane + 32 i, i < MAXV); lane j < kh
// receives the j-th best value and its index.
template <int MAXV>
__device__ __forceinline__ void top_half(const float* s, int n, int kh, int lane, float& out_v,
                                         int& out_i)
{
    float vals[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        vals[i] = e < n ? s[e] : -INFINITY;
    }
    uint32_t taken = 0;
    out_v = -INFINITY;
    out_i = -1;
    for (int j = 0; j < kh; ++j) {
        float bv = -INFINITY;
        int bi = INT_MAX;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) {
            const int e = lane + 32 * i;
            if (e < n && !((taken >> i) & 1u) && better(vals[i], e, bv, bi)) { bv = vals[i]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(FULL, bv, o);
            const int oi = __shfl_xor_sync(FULL, bi, o);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if (bi != INT_MAX && (bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == j) { out_v = bv; out_i = (bi == INT_MAX) ? -1 : bi; }
    }
}

template <int MAXV>
__global__ void __launch_bounds__(256) pk_select_kernel(const PkSelectArgs a)
{
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < a.T; t += warps) {
        const float* sr = a.s_row + (long long)t * a.rows;
        const float* sc = a.s_col + (long long)t * a.cols;
        if (a.logits_out) {
            float* lo = a.logits_out + (long long)t * (a.rows + a.cols);
            for (int e = lane; e < a.rows; e += 32) lo[e] = sr[e];
            for (int e = lane; e < a.cols; e += 32) lo[a.rows + e] = sc[e];
        }
        float rv, cv;
        int ri, ci;
        top_half<MAXV>(sr, a.rows, a.kh, lane, rv, ri);
        top_half<MAXV>(sc, a.cols, a.kh, lane, cv, ci);

        // merge: lane i < kh walks row candidate i along its sorted columns
        int p = 0;
        double v0 = 0.0;
        double selv[4];
        int selid[4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            selv[blk] = -INFINITY;
            selid[blk] = -1;
            for (int jj = 0; jj < 32; ++jj) {
                const int j = blk * 32 + jj;
                if (j >= a.K) break;
                const float cvp = __shfl_sync(FULL, cv, p & 31);
                const int cip = __shfl_sync(FULL, ci, p & 31);
                double hv = -INFINITY;
                int hid = INT_MAX, wl = lane;
                if (lane < a.kh && p < a.kh && ri >= 0 && cip >= 0) {
                    hv = (double)rv + (double)cvp;
                    hid = ri * a.cols + cip;
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const double ov = __shfl_xor_sync(FULL, hv, o);
                    const int oi = __shfl_xor_sync(FULL, hid, o);
                    const int ol = __shfl_xor_sync(FULL, wl, o);
                    if (ov > hv || (ov == hv && oi < hid)) { hv = ov; hid = oi; wl = ol; }
                }
                if (lane == wl) ++p;
                if (j == 0) v0 = hv;
                if (jj == lane) { selv[blk] = hv; selid[blk] = (hid == INT_MAX) ? -1 : hid; }
            }
        }
        float ex[4];
        float sum = 0.f;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int j = blk * 32 + lane;
            ex[blk] = (j < a.K) ? expf((float)(selv[blk] - v0)) : 0.f;
            sum += ex[blk];
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int j = blk * 32 + lane;
            if (j < a.K) {
                a.idx[(long long)t * a.K + j] = selid[blk];
                a.gate[(long long)t * a.K + j] = ex[blk] / sum;
            }
        }
    }
}

// W3[g][n][p * half + i] = K_g[n][i]  for g in {row, col}, p in {0, 1, 2}.
__global__ void pk_prep_keys_kernel(const __nv_bfloat16* kr, const __nv_bfloat16* kc,
                                    __nv_bfloat16* w3, int rows, int cols, int half)
{
    const long long total = (long long)(rows + cols) * 3 * half;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long n = i / (3 * half);
        const int c = (int)(i % (3 * half)) % half;
        w3[i] = n < rows ? kr[n * half + c] : kc[(n - rows) * half + c];
    }
}

}  // namespace

moe_status launch_router(int dtype, const RouterArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    const int tgroups = cdiv(a.T, R_TPW);
    const int grid = std::max(1, std::min(cdiv(tgroups, R_WARPS), num_sms() * 8));
    if (dtype == MOE_BF16) router_kernel<__nv_bfloat16><<<grid, R_WARPS * 32, 0, st>>>(a);
    else router_kernel<float><<<grid, R_WARPS * 32, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_pk_select(const PkSelectArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    const int grid = std::max(1, std::min(cdiv(a.T, 8), num_sms() * 8));
    const int n = std::max(a.rows, a.cols);
    if (n <= 512) pk_select_kernel<16><<<grid, 256, 0, st>>>(a);
    else pk_select_kernel<32><<<grid, 256, 0, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_pk_prep_keys(const void* k_row, const void* k_col, void* w3, int rows, int cols,
                               int half, cudaStream_t st)
{
    const long long total = (long long)(rows + cols) * 3 * half;
    const int grid = (int)std::min<long long>((total + 255) / 256, num_sms() * 4);
    pk_prep_keys_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k_row),
                                              reinterpret_cast<const __nv_bfloat16*>(k_col),
                                              reinterpret_cast<__nv_bfloat16*>(w3), rows, cols, half);
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace moe
