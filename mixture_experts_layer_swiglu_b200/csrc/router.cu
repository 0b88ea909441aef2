// router.cu -- router logits with warp-level top-k / softmax, and the
// Cartesian-product (product-key) selection of atomic experts.
//
// Router ("PCoMoE" summary, "The Limitation of Monolithic Expert
// Selection": a fixed set of k experts per token; "MoE++" summary,
// "Approach": gating residuals add the previous layer's router scores):
//   z = W_r x + bias + prev;  top-k by descending z, ties to the lower id;
//   gates = softmax over the selected logits.  Constant experts' mixing
//   logits W_c x are computed in the same pass over x.
// The pass over x is the cost (x is read once from HBM): tiles of 32 tokens
// are staged in shared memory with asynchronous copies, each warp takes 4
// tokens, lanes split d into 16-byte vectors, 8 router rows at a time are
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

// Block: 8 warps x 4 tokens = a tile of 32 tokens.  The tile's x rows are
// staged in shared memory in chunks of 1 KiB per row with cp.async (a ring of
// 3 chunks, ~96 KiB in flight per SM), each warp computes its 4 tokens from
// shared memory; router rows are read through L1.  If the whole tile fits
// in the staging buffer (d <= 2048 for bf16) it is loaded once and every
// group of 8 router rows reuses it.
constexpr int R_WARPS = 8;
constexpr int R_TILE = R_WARPS * R_TPW;      // 32 tokens
constexpr int R_CHUNK_BYTES = 1024;          // per row per chunk
constexpr int R_STAGES = 4;
constexpr int R_W_BYTES = 8 * 4096;          // 8 router rows of <= 4 KiB (resident tiles)
constexpr int R_SMEM = R_STAGES * R_TILE * R_CHUNK_BYTES + 2 * R_W_BYTES + R_WARPS * R_TPW * R_MAXROWS * 4;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename Tin>
__global__ void __launch_bounds__(R_WARPS * 32) router_kernel(const RouterArgs a)
{
    constexpr int V = VecOf<Tin>::N;
    constexpr int CE = R_CHUNK_BYTES / sizeof(Tin);          // elements per row per chunk
    extern __shared__ __align__(16) uint8_t r_smem[];
    uint8_t* xs = r_smem;                                     // [stage][32 rows][CE]
    uint8_t* wbuf = r_smem + R_STAGES * R_TILE * R_CHUNK_BYTES;   // [2][8 rows][d] (resident tiles)
    float (*s_logit)[R_TPW][R_MAXROWS] =
        reinterpret_cast<float (*)[R_TPW][R_MAXROWS]>(wbuf + 2 * R_W_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = a.E_r + 2 * a.n_const;
    const int n_tiles = cdiv(a.T, R_TILE);
    const int n_chunks = cdiv(a.d, CE);
    // whole tile fits (and 8 router rows fit a W buffer): load once
    const bool resident = n_chunks <= R_STAGES && a.d * (int)sizeof(Tin) <= R_W_BYTES / 8;
    const Tin* x = reinterpret_cast<const Tin*>(a.x);
    const Tin* wr = reinterpret_cast<const Tin*>(a.w_router);
    const Tin* wc = reinterpret_cast<const Tin*>(a.w_const_mix);
    float (*zs)[R_MAXROWS] = s_logit[warp];

    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int t_tile = tile * R_TILE;
        // copy chunk c of the tile's 32 rows into stage st (rows past T repeat row T-1)
        auto issue = [&](int c, int st) {
            const int e0 = c * CE;
            const int vec_per_row = min(CE, a.d - e0) / V;
            for (int q = threadIdx.x; q < R_TILE * vec_per_row; q += blockDim.x) {
                const int row = q / vec_per_row, vi = q % vec_per_row;
                const long long t = min(t_tile + row, a.T - 1);
                cp_async16(xs + ((size_t)st * R_TILE + row) * R_CHUNK_BYTES + vi * 16,
                           x + t * a.d + e0 + (long long)vi * V);
            }
        };
        // 8 router rows (rows past R repeat row R-1) into W buffer wb
        const int row_bytes = a.d * (int)sizeof(Tin);
        auto issue_w = [&](int rc, int wb) {
            const int vec_per_row = a.d / V;
            for (int q = threadIdx.x; q < 8 * vec_per_row; q += blockDim.x) {
                const int qr = q / vec_per_row, vi = q % vec_per_row;
                const int r = min(rc + qr, R - 1);
                const Tin* wrow = r < a.E_r ? wr + (long long)r * a.d : wc + (long long)(r - a.E_r) * a.d;
                cp_async16(wbuf + (size_t)wb * R_W_BYTES + (size_t)qr * row_bytes + vi * 16, wrow + (long long)vi * V);
            }
        };
        const int passes = resident ? 1 : cdiv(R, 8);
        for (int pass = 0; pass < passes; ++pass) {
            __syncthreads();                                  // stage buffers free
            const int npro = min(R_STAGES - 1, n_chunks);
            for (int c = 0; c < (resident ? n_chunks : npro); ++c) { issue(c, c); cp_async_commit(); }
            if (resident) { issue_w(0, 0); cp_async_commit(); }
            const int rc_lo = resident ? 0 : pass * 8, rc_hi = resident ? R : min(R, pass * 8 + 8);
            for (int rc = rc_lo; rc < rc_hi; rc += 8) {
                float acc[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) acc[i] = 0.f;
                const int wb = (rc / 8) & 1;
                if (resident) {
                    // next 8 rows in flight while these compute; x tile and
                    // this W buffer complete
                    if (rc + 8 < rc_hi) { issue_w(rc + 8, wb ^ 1); cp_async_commit(); cp_async_wait<1>(); }
                    else cp_async_wait<0>();
                    __syncthreads();
                }
                for (int c = 0; c < n_chunks; ++c) {
                    const int st = resident ? c : c % R_STAGES;
                    if (!resident) {
                        if (c + R_STAGES - 1 < n_chunks) cp_async_wait<R_STAGES - 2>();
                        else cp_async_wait<0>();
                        __syncthreads();
                    }
                    const int e0 = c * CE;
                    const int ce = min(CE, a.d - e0);
                    for (int vi = lane; vi < ce / V; vi += 32) {
                        float xv[R_TPW][V];
#pragma unroll
                        for (int tt = 0; tt < R_TPW; ++tt) {
                            const Tin* src = reinterpret_cast<const Tin*>(
                                xs + ((size_t)st * R_TILE + warp * R_TPW + tt) * R_CHUNK_BYTES) + vi * V;
                            if constexpr (V == 8) {
                                const uint4 u = *reinterpret_cast<const uint4*>(src);
                                xv[tt][0] = bf16_lo(u.x); xv[tt][1] = bf16_hi(u.x); xv[tt][2] = bf16_lo(u.y); xv[tt][3] = bf16_hi(u.y);
                                xv[tt][4] = bf16_lo(u.z); xv[tt][5] = bf16_hi(u.z); xv[tt][6] = bf16_lo(u.w); xv[tt][7] = bf16_hi(u.w);
                            } else {
                                const float4 f = *reinterpret_cast<const float4*>(src);
                                xv[tt][0] = f.x; xv[tt][1] = f.y; xv[tt][2] = f.z; xv[tt][3] = f.w;
                            }
                        }
                        // all 8 router-row loads issued together: rows past R
                        // repeat row R-1 and land in accumulators never read
                        float wv[8][V];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (resident) {
                                const Tin* src = reinterpret_cast<const Tin*>(
                                    wbuf + (size_t)wb * R_W_BYTES + (size_t)q * row_bytes) + e0 + vi * V;
                                if constexpr (V == 8) {
                                    const uint4 u = *reinterpret_cast<const uint4*>(src);
                                    wv[q][0] = bf16_lo(u.x); wv[q][1] = bf16_hi(u.x); wv[q][2] = bf16_lo(u.y); wv[q][3] = bf16_hi(u.y);
                                    wv[q][4] = bf16_lo(u.z); wv[q][5] = bf16_hi(u.z); wv[q][6] = bf16_lo(u.w); wv[q][7] = bf16_hi(u.w);
                                } else {
                                    const float4 f = *reinterpret_cast<const float4*>(src);
                                    wv[q][0] = f.x; wv[q][1] = f.y; wv[q][2] = f.z; wv[q][3] = f.w;
                                }
                            } else {
                                const int r = min(rc + q, R - 1);
                                const Tin* wrow = r < a.E_r ? wr + (long long)r * a.d : wc + (long long)(r - a.E_r) * a.d;
                                load_vec(wrow + e0 + vi * V, wv[q]);
                            }
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q)
#pragma unroll
                            for (int tt = 0; tt < R_TPW; ++tt)
#pragma unroll
                                for (int v = 0; v < V; ++v)
                                    acc[tt * 8 + q] = fmaf(xv[tt][v], wv[q][v], acc[tt * 8 + q]);
                    }
                    if (!resident) {
                        __syncthreads();                      // everyone done with stage st
                        if (c + R_STAGES - 1 < n_chunks) { issue(c + R_STAGES - 1, (c + R_STAGES - 1) % R_STAGES); }
                        cp_async_commit();
                    }
                }
                if (resident) __syncthreads();                // W buffer wb free for rc + 16
                const float sres = transpose_reduce32(acc, lane);
                const int r = rc + (lane & 7);
                if (r < R) zs[lane >> 3][r] = sres;
            }
        }
        __syncwarp();

        for (int tt = 0; tt < R_TPW; ++tt) {
            const int t = t_tile + warp * R_TPW + tt;
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
    const int grid = std::max(1, std::min(cdiv(a.T, R_TILE), num_sms()));
    static bool attr_done = false;
    if (!attr_done) {
        cudaFuncSetAttribute(router_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, R_SMEM);
        cudaFuncSetAttribute(router_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, R_SMEM);
        attr_done = true;
    }
    if (dtype == MOE_BF16) router_kernel<__nv_bfloat16><<<grid, R_WARPS * 32, R_SMEM, st>>>(a);
    else router_kernel<float><<<grid, R_WARPS * 32, R_SMEM, st>>>(a);
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
