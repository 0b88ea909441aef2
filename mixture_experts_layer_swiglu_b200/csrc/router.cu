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

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr unsigned FULL = 0xffffffffu;

#ifndef MOE_ROUTER_STREAM
#define MOE_ROUTER_STREAM 1       // bf16: the streaming tensor-core router (else router_mma_kernel)
#endif
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
// An unsigned key with the order of the float comparison: a > b exactly when
// key(a) > key(b), -0 and +0 equal, -inf the smallest (key > 0); NaN key 0.
__device__ __forceinline__ uint32_t logit_key(float v)
{
    if (v != v) return 0u;
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
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


// One token's routing from its raw router logits z[0, E_r) (and the constant
// experts' mixing logits z[E_r, E_r + 2 n_const)), in shared memory: adds the
// bias and the previous layer's logits, writes logits_out, selects the k
// largest (value desc, ties to the lower id) with a warp argmax, softmax gates
// over the selected, and the constant experts' (a1, a2).
// (E_r <= 64 and `pre` given: the bias and previous-layer logits of experts
// lane and lane + 32, loaded ahead by the caller; the sum order is the same.)
__device__ __forceinline__ void route_token(const RouterArgs& a, int t, float* z, int lane,
                                            const float (*pre)[2] = nullptr)
{
    if (pre) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            if (e < a.E_r) {
                float v = z[e];
                if (a.bias) v += pre[i][0];
                if (a.prev) v += pre[i][1];
                z[e] = v;
                if (a.logits_out) a.logits_out[(long long)t * a.E_r + e] = v;
            }
        }
    } else {
        for (int e = lane; e < a.E_r; e += 32) {
            float v = z[e];
            if (a.bias) v += a.bias[e];
            if (a.prev) v += a.prev[(long long)t * a.E_r + e];
            z[e] = v;
            if (a.logits_out) a.logits_out[(long long)t * a.E_r + e] = v;
        }
    }
    __syncwarp();
    float zsel = 0.f, z0 = 0.f;
    int isel = -1;
    if (a.E_r <= 32 && a.k <= 2) {
        // one logit per lane: the best two of the warp in one butterfly that
        // carries each lane's best pair of keys (order-preserving value, then
        // the complemented id, so equal values go to the lower id; a NaN has
        // key 0 and is never chosen) -- the same choice as the loop below
        unsigned long long k1 = 0ull, k2 = 0ull;
        if (lane < a.E_r) {
            const uint32_t kv = logit_key(z[lane]);
            if (kv) k1 = ((unsigned long long)kv << 32) | (uint32_t)~(uint32_t)lane;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const unsigned long long b1 = __shfl_xor_sync(FULL, k1, o), b2 = __shfl_xor_sync(FULL, k2, o);
            const unsigned long long lo = k1 > b1 ? b1 : k1, m2 = k2 > b2 ? k2 : b2;
            k1 = k1 > b1 ? k1 : b1;
            k2 = lo > m2 ? lo : m2;
        }
        const unsigned long long mine = lane == 0 ? k1 : k2;
        if (lane < a.k) {
            isel = mine != 0ull ? (int)~(uint32_t)mine : -1;
            zsel = isel >= 0 ? z[isel] : -INFINITY;
        }
        z0 = k1 != 0ull ? z[(int)~(uint32_t)k1] : -INFINITY;
    } else {
        uint32_t taken = 0;   // bit i: expert lane + 32 i already selected
        for (int j = 0; j < a.k; ++j) {
            // the best untaken logit (value desc, ties to the lower id): each lane
            // its own best as an order-preserving key (NaN never selected, as
            // with the float comparison), then the largest key of the warp and the
            // lowest id holding it, two warp reductions instead of a shuffle tree
            uint32_t bk = 0;
            int bi = INT_MAX;
            for (int i = 0; lane + 32 * i < a.E_r; ++i) {
                if ((taken >> i) & 1u) continue;
                const int e = lane + 32 * i;
                const uint32_t kk = logit_key(z[e]);
                if (kk > bk) { bk = kk; bi = e; }
            }
            const uint32_t mk = __reduce_max_sync(FULL, bk);
            bi = __reduce_min_sync(FULL, (mk != 0u && bk == mk) ? bi : INT_MAX);
            const float bv = bi != INT_MAX ? z[bi] : -INFINITY;
            if (bi != INT_MAX && (bi & 31) == lane) taken |= 1u << (bi >> 5);
            if (lane == j) { zsel = bv; isel = (bi == INT_MAX) ? -1 : bi; }
            if (j == 0) z0 = bv;
        }
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
            route_token(a, t, zs[tt], lane);
        }
    }
}

// Router logits on the tensor cores (bf16 inputs).  A block takes 16 tokens;
// its 4 warps split d into quarters (split-K) and each computes the partial
// logits of all router rows (and the constant experts' mixing rows) as the N
// side of m16n8k16 tiles, in groups of 64 rows.  For each 64-element slice of
// d, lane (g, q) loads 32 contiguous bytes of its A rows (tokens g, g+8) and
// B rows (router row g of each n8 tile), which feed four k16 steps in the
// same k order for A and B.  bf16 x bf16 products are exact in fp32 and
// accumulate in fp32, as in the FMA kernel (only the order of the sums
// differs); the four partials are added in warp order.  Each warp then
// routes 4 of the 16 tokens with route_token.
constexpr int RM_WARPS = 4;
constexpr int RM_NG = 8;                     // n8 tiles per group: 64 router rows

__global__ void __launch_bounds__(RM_WARPS * 32) router_mma_kernel(const RouterArgs a)
{
    extern __shared__ __align__(16) float rm_z[];   // [RM_WARPS][16][zpitch] partial logits
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3, wib = threadIdx.x >> 5;
    const int R = a.E_r + 2 * a.n_const;
    const int zpitch = (R + 7) & ~7;
    float* zw = rm_z + (size_t)wib * 16 * zpitch;
    const size_t rowb = (size_t)a.d * 2;
    const unsigned char* xb = static_cast<const unsigned char*>(a.x);
    const unsigned char* wr = static_cast<const unsigned char*>(a.w_router);
    const unsigned char* wc = static_cast<const unsigned char*>(a.w_const_mix);
    const int nsc = a.d / 64;
    const int sc0 = wib * nsc / RM_WARPS, sc1 = (wib + 1) * nsc / RM_WARPS;   // this warp's slices
    const int tiles = (a.T + 15) / 16;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int t0 = tile * 16;
        const unsigned char* xr0 = xb + (size_t)min(t0 + g, a.T - 1) * rowb;
        const unsigned char* xr1 = xb + (size_t)min(t0 + g + 8, a.T - 1) * rowb;
        for (int n0 = 0; n0 < R; n0 += 8 * RM_NG) {
            const unsigned char* wrow[RM_NG];
#pragma unroll
            for (int nt = 0; nt < RM_NG; ++nt) {
                const int j = min(n0 + nt * 8 + g, R - 1);   // rows past R repeat the last; never read
                wrow[nt] = j < a.E_r ? wr + (size_t)j * rowb : wc + (size_t)(j - a.E_r) * rowb;
            }
            const int ntiles = min(RM_NG, (R - n0 + 7) / 8);
            float acc[RM_NG][4];
#pragma unroll
            for (int nt = 0; nt < RM_NG; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 1
            for (int sc = sc0; sc < sc1; ++sc) {
                const int off = sc * 128 + q * 32;
                uint32_t xa[8], xb2[8];
                ld256(xr0 + off, xa);
                ld256(xr1 + off, xb2);
#pragma unroll
                for (int nt = 0; nt < RM_NG; ++nt) {
                    if (nt < ntiles) {
                        uint32_t w[8];
                        ld256(wrow[nt] + off, w);
#pragma unroll
                        for (int st = 0; st < 4; ++st)
                            mma_16816(acc[nt], xa[2 * st], xb2[2 * st], xa[2 * st + 1], xb2[2 * st + 1], w[2 * st],
                                      w[2 * st + 1]);
                    }
                }
            }
            // D fragment: acc[0], acc[1] = token g, rows 2q, 2q+1; acc[2], acc[3] = token g+8
#pragma unroll
            for (int nt = 0; nt < RM_NG; ++nt) {
                const int col = n0 + nt * 8 + 2 * q;
                if (nt < ntiles && col < zpitch) {
                    zw[g * zpitch + col] = acc[nt][0];
                    zw[g * zpitch + col + 1] = acc[nt][1];
                    zw[(g + 8) * zpitch + col] = acc[nt][2];
                    zw[(g + 8) * zpitch + col + 1] = acc[nt][3];
                }
            }
        }
        __syncthreads();
        // sum the partials in warp order into warp 0's buffer
        for (int i = threadIdx.x; i < 16 * zpitch; i += RM_WARPS * 32) {
            float v = rm_z[i];
#pragma unroll
            for (int w2 = 1; w2 < RM_WARPS; ++w2) v += rm_z[(size_t)w2 * 16 * zpitch + i];
            rm_z[i] = v;
        }
        __syncthreads();
        for (int tt = wib; tt < 16; tt += RM_WARPS) {
            const int t = t0 + tt;
            if (t < a.T) route_token(a, t, rm_z + tt * zpitch, lane);
        }
        __syncthreads();   // buffers free for the next tile
    }
}

// Streaming form of the tensor-core router (bf16 x, d a multiple of 64, at
// most 64 router + mixing rows): x is read once from HBM, so the kernel is
// built to keep HBM busy.  One persistent block per SM; a producer warp
// copies each 16-token tile's rows into shared memory with bulk copies
// (cp.async.bulk, no multicast), chunk by chunk (16 rows x 1024 elements of d
// per chunk, one copy per row), into a ring of stages with mbarrier
// completion, running ahead across tiles (100-130 KiB in flight per SM).
// The router rows are copied into shared memory once per block when they fit
// (else read through L1).  The 16 consumer warps split each chunk's d: warp w
// takes the 64-wide slice w of the chunk and accumulates, in
// registers across the tile's chunks, the m16n8k16 tiles of those slices as
// router_mma_kernel does (lane (g, q) uses 32 contiguous bytes of token rows g
// and g + 8 and of router row g of each n8 tile, in the same k order for A and
// B); rows are padded by 16 bytes in shared memory so the fragment reads are
// conflict-free.  At the tile's end the 16 partial logits are summed in warp
// order (fixed, so the logits do not depend on timing) and each warp routes
// one token with route_token (its bias and previous-layer logits loaded
// before the MMAs), while the producer already streams the next tile.
constexpr int RS_WARPS = 16;                   // consumer warps
constexpr int RS_THREADS = (RS_WARPS + 1) * 32;
constexpr int RS_KC = 64 * RS_WARPS;           // d elements per chunk: one 64-wide slice per consumer warp
constexpr int RS_PITCH = RS_KC * 2 + 16;       // bytes per staged row
constexpr int RS_STAGE = 16 * RS_PITCH;        // 16 token rows
constexpr int RS_MAXSTAGES = 4;
constexpr int RS_MAXROWS = 8 * RM_NG;          // router + mixing rows (one group of n8 tiles)
constexpr int RS_SMEM_LIMIT = 227 * 1024;

__host__ __device__ constexpr int rs_zpitch(int R) { return (R + 7) & ~7; }
__host__ __device__ constexpr int rs_partial_bytes(int R) { return (RS_WARPS + 1) * 16 * rs_zpitch(R) * 4; }
__host__ __device__ constexpr int rs_wpitch(int d) { return d * 2 + 16; }

// Consumer-warp barrier (the producer warp never takes part).
__device__ __forceinline__ void rs_consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(RS_WARPS * 32) : "memory"); }

// Consumer-warp barrier that also returns whether `v` holds in every consumer thread.
__device__ __forceinline__ bool rs_consumer_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "n"(RS_WARPS * 32) : "memory");
    return r != 0;
}

__device__ __forceinline__ void lds256(uint32_t saddr, uint32_t (&r)[8])
{
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%8];\n\t"
                 "ld.shared.v4.u32 {%4,%5,%6,%7}, [%8+16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(saddr));
}

// 32-byte read-only global load that may allocate in L1 (router rows: every
// tile of the block reads them again).
__device__ __forceinline__ void ld256_l1(const unsigned char* p, uint32_t (&r)[8])
{
    asm("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "l"(p));
}

struct RsLayout {
    int stages;
    bool w_smem;      // router rows staged in shared memory
    int w_off, z_off, bar_off, bytes;
};

__host__ __device__ inline RsLayout rs_layout(int R, int d)
{
    RsLayout L;
    const int part = rs_partial_bytes(R);
    const int wbytes = ((R * rs_wpitch(d)) + 127) & ~127;
    const int fixed = part + (2 * RS_MAXSTAGES + 1) * 8 + 16;
    L.w_smem = RS_SMEM_LIMIT - fixed - wbytes >= 3 * RS_STAGE;
    const int avail = RS_SMEM_LIMIT - fixed - (L.w_smem ? wbytes : 0);
    L.stages = avail / RS_STAGE < RS_MAXSTAGES ? avail / RS_STAGE : RS_MAXSTAGES;
    L.w_off = L.stages * RS_STAGE;
    L.z_off = L.w_off + (L.w_smem ? wbytes : 0);
    L.bar_off = L.z_off + part;
    L.bytes = L.bar_off + (2 * RS_MAXSTAGES + 1) * 8 + 16;
    return L;
}

// NT: n8 tiles of router + mixing rows (R <= 8 NT); the accumulators of
// exactly those tiles live in registers.
template <int NT>
__global__ void __launch_bounds__(RS_THREADS, 1) router_stream_kernel(const RouterArgs a)
{
    extern __shared__ __align__(128) unsigned char rs_smem[];
    const int R = a.E_r + 2 * a.n_const;
    const int zpitch = rs_zpitch(R);
    const RsLayout L = rs_layout(R, a.d);
    const int stages = L.stages;
    unsigned char* ring = rs_smem;                                          // [stages][16 rows][RS_PITCH]
    unsigned char* wsm = rs_smem + L.w_off;                                 // [R][wpitch] (if w_smem)
    float* zpart = reinterpret_cast<float*>(rs_smem + L.z_off);             // [RS_WARPS][16][zpitch]
    float* zsum = zpart + (size_t)RS_WARPS * 16 * zpitch;                   // [16][zpitch]
    uint64_t* full = reinterpret_cast<uint64_t*>(rs_smem + L.bar_off);
    uint64_t* empty = full + RS_MAXSTAGES;
    uint64_t* wbar = empty + RS_MAXSTAGES;                                  // router rows landed
    volatile int* abort_flag = reinterpret_cast<volatile int*>(wbar + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t rowb = (size_t)a.d * 2;
    const int wpitch = rs_wpitch(a.d);
    const int nchunk = cdiv(a.d, RS_KC);
    const int tiles = cdiv(a.T, 16);
    const unsigned char* wr = static_cast<const unsigned char*>(a.w_router);
    const unsigned char* wc = static_cast<const unsigned char*>(a.w_const_mix);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], RS_WARPS); }
        mbar_init(wbar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == RS_WARPS) {
        // ---------------------------------------------------- producer warp
        // first the router rows (then the mixing rows) into shared memory, one
        // bulk copy per row, landing while the first x chunks are in flight
        if (L.w_smem) {
            if (lane == 0) mbar_arrive_expect_tx(wbar, (uint32_t)(R * a.d * 2));
            __syncwarp();
            for (int j = lane; j < R; j += 32) {
                const unsigned char* src = j < a.E_r ? wr + (size_t)j * rowb : wc + (size_t)(j - a.E_r) * rowb;
                bulk_g2s(wsm + (size_t)j * wpitch, src, (uint32_t)(a.d * 2), wbar);
            }
        }
        // lanes 0..15 each copy one token row of a chunk; lane 0 arms the stage
        const unsigned char* xb = static_cast<const unsigned char*>(a.x);
        int s = 0;
        uint32_t ph = 0, pend = 0, pend_ph = 0;
        bool bad = false;
        for (int tile = blockIdx.x; tile < tiles && !bad; tile += gridDim.x) {
            const int t0 = tile * 16;
            const int rows = min(16, a.T - t0);
            for (int c = 0; c < nchunk; ++c) {
                const bool ok = *abort_flag == 0 && mbar_wait(&empty[s], ph ^ 1);
                if (!__all_sync(FULL, ok)) { *abort_flag = 1; bad = true; break; }
                const int e0 = c * RS_KC;
                const int bytes = min(RS_KC, a.d - e0) * 2;
                if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(rows * bytes));
                __syncwarp();
                if (lane < rows)
                    bulk_g2s(ring + (size_t)s * RS_STAGE + (size_t)lane * RS_PITCH,
                             xb + (size_t)(t0 + lane) * rowb + (size_t)e0 * 2, (uint32_t)bytes, &full[s]);
                pend |= 1u << s;
                pend_ph = (pend_ph & ~(1u << s)) | (ph << s);
                if (++s == stages) { s = 0; ph ^= 1; }
            }
        }
        // copies still in flight land before the block may exit
        if (lane == 0) {
            for (int i = 0; i < stages; ++i)
                if ((pend >> i) & 1u) mbar_wait(&full[i], (pend_ph >> i) & 1u);
            if (L.w_smem) mbar_wait(wbar, 0);
        }
        return;
    }

    // -------------------------------------------------------- consumer warps
    bool ok = !L.w_smem || __all_sync(FULL, mbar_wait(wbar, 0));   // the router rows are in shared memory
    const int g = lane >> 2, q = lane & 3;
    float* zw = zpart + (size_t)warp * 16 * zpitch;
    const uint32_t ring_s = smem_u32(ring), wsm_s = smem_u32(wsm);
    int s = 0;
    uint32_t ph = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int t0 = tile * 16;
        // the bias and previous-layer logits of this warp's token, loaded now so
        // that routing it after the MMAs does not wait on them
        float pre[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        if (t0 + warp < a.T) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int e = lane + 32 * i;
                if (e < a.E_r) {
                    if (a.bias) pre[i][0] = a.bias[e];
                    if (a.prev) pre[i][1] = a.prev[(long long)(t0 + warp) * a.E_r + e];
                }
            }
        }
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        for (int c = 0; c < nchunk; ++c) {
            if (ok) ok = __all_sync(FULL, mbar_wait(&full[s], ph));   // warp-uniform: the MMAs need every lane
            const int e0 = c * RS_KC;
            const int nsl = min(RS_KC, a.d - e0) / 64;           // 64-wide slices in this chunk
            const uint32_t st = ring_s + (uint32_t)(s * RS_STAGE);
#pragma unroll 1
            for (int sl = warp; sl < nsl && ok; sl += RS_WARPS) {
                uint32_t xa[8], xb2[8];
                lds256(st + (uint32_t)(g * RS_PITCH + sl * 128 + q * 32), xa);
                lds256(st + (uint32_t)((g + 8) * RS_PITCH + sl * 128 + q * 32), xb2);
                const int off = (e0 + sl * 64) * 2 + q * 32;      // byte offset in a router row
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int j = min(nt * 8 + g, R - 1);          // rows past R repeat the last; never read
                    uint32_t w[8];
                    if (L.w_smem) {
                        lds256(wsm_s + (uint32_t)(j * wpitch + off), w);
                    } else {
                        const unsigned char* wrow = j < a.E_r ? wr + (size_t)j * rowb : wc + (size_t)(j - a.E_r) * rowb;
                        ld256_l1(wrow + off, w);
                    }
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        mma_16816(acc[nt], xa[2 * k4], xb2[2 * k4], xa[2 * k4 + 1], xb2[2 * k4 + 1], w[2 * k4],
                                  w[2 * k4 + 1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);      // this warp is done with the stage
            if (++s == stages) { s = 0; ph ^= 1; }
        }
        // D fragment: acc[0], acc[1] = token g, rows 2q, 2q+1; acc[2], acc[3] = token g+8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int col = nt * 8 + 2 * q;
            if (col < zpitch) {
                zw[g * zpitch + col] = acc[nt][0];
                zw[g * zpitch + col + 1] = acc[nt][1];
                zw[(g + 8) * zpitch + col] = acc[nt][2];
                zw[(g + 8) * zpitch + col + 1] = acc[nt][3];
            }
        }
        // all consumer warps agree to go on (a timed-out wait stops them together)
        if (!rs_consumer_all(ok)) { *abort_flag = 1; break; }
        // sum the partials in warp order, then route one token per warp
        for (int i = threadIdx.x; i < 16 * zpitch; i += RS_WARPS * 32) {
            float v = zpart[i];
#pragma unroll
            for (int w2 = 1; w2 < RS_WARPS; ++w2) v += zpart[(size_t)w2 * 16 * zpitch + i];
            zsum[i] = v;
        }
        rs_consumer_sync();
        if (t0 + warp < a.T) route_token(a, t0 + warp, zsum + warp * zpitch, lane, pre);
        rs_consumer_sync();   // zsum and the partials are free for the next tile
    }
}

// Shared-memory bytes of router_stream_kernel, or 0 if the layer does not
// fit its limits (more than 64 rows, or fewer than 2 stages).
int router_stream_smem(int R, int d)
{
    if (R > RS_MAXROWS) return 0;
    const RsLayout L = rs_layout(R, d);
    return L.stages >= 2 ? L.bytes : 0;
}

// ------------------------------------------------------- product-key selection
//
// Every candidate gets one unsigned 64-bit key whose order is the selection
// order (descending score, ties to the lower index): the high word maps the
// score to an unsigned integer with the same order, the low word is the
// complement of the index.  The best of 32 lane keys is then two (three for
// the merge, whose scores are fp64) __reduce_max_sync steps, with no
// shuffles.

__device__ __forceinline__ uint32_t order_key32(float v)
{
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;                    // -0 orders as +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key32_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ unsigned long long order_key64(double v)
{
    unsigned long long b = (unsigned long long)__double_as_longlong(v);
    if (b == 0x8000000000000000ull) b = 0ull;
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Bitonic sort of a lane's keys, descending.
template <int MAXV>
__device__ __forceinline__ void sort_desc(unsigned long long (&c)[MAXV])
{
#pragma unroll
    for (int k = 2; k <= MAXV; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < MAXV; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const unsigned long long a = c[i], b = c[l];
                    const bool sw = ((i & k) == 0) ? (a < b) : (a > b);
                    c[i] = sw ? b : a;
                    c[l] = sw ? a : b;
                }
            }
}

// Walk of the candidates list[0..C): lane l sorts candidates l + 32 j
// (j < SZ) in registers; each step the warp takes the best lane head (two
// __reduce_max_sync on the 64-bit key) and the winning lane shifts its list
// by one (compile-time register indices, no shared-memory round trip).
template <int SZ>
__device__ __forceinline__ void walk_half(const unsigned long long* list, int C, int kh, int lane, float* out_v,
                                          int* out_i)
{
    unsigned long long c[SZ];
#pragma unroll
    for (int j = 0; j < SZ; ++j) c[j] = (j * 32 + lane < C) ? list[j * 32 + lane] : 0ull;
    sort_desc<SZ>(c);
    for (int j = 0; j < kh; ++j) {
        const uint32_t hi = (uint32_t)(c[0] >> 32), lo = (uint32_t)c[0];
        const uint32_t m1 = __reduce_max_sync(FULL, hi);
        const uint32_t m2 = __reduce_max_sync(FULL, hi == m1 ? lo : 0u);
        if (hi == m1 && lo == m2) {
            out_v[j] = key32_value(hi);
            out_i[j] = (int)~lo;
#pragma unroll
            for (int q = 0; q + 1 < SZ; ++q) c[q] = c[q + 1];
            c[SZ - 1] = 0ull;
        }
    }
    __syncwarp();
}

// Best kh of the n scores s[0..n) (32 <= n, kh <= 32), best first, into
// out_v / out_i.  Prefilter: each lane's maximum is one score, so at least
// 32 scores are >= tau = the smallest lane maximum, and the kh-th best score
// is >= tau; only scores >= tau (about 110 of 512 for random scores) are
// sorted and walked.
template <int MAXV>
__device__ __forceinline__ void select_half(const float* s, int n, int kh, int lane,
                                            unsigned long long* list, float* out_v, int* out_i)
{
    uint32_t k[MAXV];
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const int e = lane + 32 * i;
        k[i] = e < n ? order_key32(__ldg(s + e)) : 0u;   // valid keys are > 0
        mx = max(mx, k[i]);
    }
    const uint32_t tau = __reduce_min_sync(FULL, mx);
    const unsigned lt = (1u << lane) - 1u;
    int C = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
        const bool take = k[i] >= tau;
        const unsigned b = __ballot_sync(FULL, take);
        if (take) list[C + __popc(b & lt)] = ((unsigned long long)k[i] << 32) | (uint32_t)~(lane + 32 * i);
        C += __popc(b);
    }
    __syncwarp();
    if (C <= 128) walk_half<4>(list, C, kh, lane, out_v, out_i);
    else if (C <= 256) walk_half<8>(list, C, kh, lane, out_v, out_i);
    else if (C <= 512) walk_half<16>(list, C, kh, lane, out_v, out_i);
    else walk_half<32>(list, C, kh, lane, out_v, out_i);
}

__device__ __forceinline__ double key64_value(unsigned long long k)
{
    return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

template <int MAXV> struct PkWarpSmem {
    unsigned long long list[MAXV * 32];   // half candidates; then each row's merge candidates
    unsigned long long sel_k[128];
    int sel_i[128];
    float rv[32], cv[32];
    int ri[32], ci[32];
};

// One warp per token.  The merge relies on both halves being sorted: lane
// i < kh walks row candidate i along the sorted columns, so its next
// candidate is always its best remaining one, and the best of the lanes'
// heads is the best remaining pair.  A pair (i, j) (ranks in the sorted
// halves) is dominated by the (i+1)(j+1) pairs (i' <= i, j' <= j), none of
// which ranks after it (sums of the sorted scores are monotone and the ids
// order ties the same way), so only pairs with (i+1)(j+1) <= K can be
// selected: lane i precomputes the keys of its first min(kh, K/(i+1)) pairs.
#ifndef MOE_PK_MINB
#define MOE_PK_MINB 3     // resident blocks of 8 warps per SM
#endif

template <int MAXV>
__global__ void __launch_bounds__(256, MOE_PK_MINB) pk_select_kernel(const PkSelectArgs a)
{
    extern __shared__ __align__(16) unsigned char pk_smem[];
    const int lane = threadIdx.x & 31;
    PkWarpSmem<MAXV>& w = reinterpret_cast<PkWarpSmem<MAXV>*>(pk_smem)[threadIdx.x >> 5];
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < a.T; t += warps) {
        const float* sr = a.s_row + (long long)t * a.rows;
        const float* sc = a.s_col + (long long)t * a.cols;
        if (a.logits_out) {
            float* lo = a.logits_out + (long long)t * (a.rows + a.cols);
            for (int e = lane; e < a.rows; e += 32) lo[e] = sr[e];
            for (int e = lane; e < a.cols; e += 32) lo[a.rows + e] = sc[e];
        }
        select_half<MAXV>(sr, a.rows, a.kh, lane, w.list, w.rv, w.ri);
        select_half<MAXV>(sc, a.cols, a.kh, lane, w.list, w.cv, w.ci);

        // merge candidates: lane i < kh owns list[off, off + np)
        const bool rowl = lane < a.kh;
        const int np = rowl ? min(a.kh, a.K / (lane + 1)) : 0;
        int off = np;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(FULL, off, o);
            if (lane >= o) off += u;
        }
        off -= np;
        const double my_r = rowl ? (double)w.rv[lane] : 0.0;
        const int my_base = rowl ? w.ri[lane] * a.cols : 0;
        for (int pp = 0; pp < np; ++pp) w.list[off + pp] = order_key64(my_r + (double)w.cv[pp]);
        __syncwarp();
        int p = 0;
        unsigned long long key = np > 0 ? w.list[off] : 0ull;
        for (int j = 0; j < a.K; ++j) {
            const uint32_t hi = (uint32_t)(key >> 32), lo = (uint32_t)key;
            const uint32_t m1 = __reduce_max_sync(FULL, hi);
            bool win = hi == m1;
            const uint32_t id = (uint32_t)(my_base + w.ci[p < a.kh ? p : 0]);
            if (__popc(__ballot_sync(FULL, win)) > 1) {        // equal high words: rare
                const uint32_t m2 = __reduce_max_sync(FULL, win ? lo : 0u);
                win = win && lo == m2;
                const uint32_t m3 = __reduce_max_sync(FULL, win ? ~id : 0u);
                win = win && ~id == m3;
            }
            if (win) {
                w.sel_k[j] = key;
                w.sel_i[j] = (int)id;
                ++p;
                key = p < np ? w.list[off + p] : 0ull;
            }
        }
        __syncwarp();
        const double v0 = key64_value(w.sel_k[0]);
        float ex[4];
        float tot = 0.f;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int j = blk * 32 + lane;
            ex[blk] = (j < a.K) ? expf((float)(key64_value(w.sel_k[j]) - v0)) : 0.f;
            tot += ex[blk];
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) tot += __shfl_xor_sync(FULL, tot, o);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int j = blk * 32 + lane;
            if (j < a.K) {
                a.idx[(long long)t * a.K + j] = w.sel_i[j];
                a.gate[(long long)t * a.K + j] = ex[blk] / tot;
            }
        }
        __syncwarp();
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
    if (dtype == MOE_BF16 && a.d % 64 == 0 && MOE_ROUTER_STREAM) {
        const int R = a.E_r + 2 * a.n_const;
        const int smem = router_stream_smem(R, a.d);
        if (smem > 0) {
            const int grid = std::max(1, std::min(cdiv(a.T, 16), num_sms()));
            auto go = [&](auto kernel) {
                cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kernel), smem);
                if (e != cudaSuccess) return cuda_status(e);
                kernel<<<grid, RS_THREADS, smem, st>>>(a);
                count_launch();
                return cuda_status(cudaGetLastError());
            };
            const int nt = (R + 7) / 8;
            if (nt <= 1) return go(router_stream_kernel<1>);
            if (nt <= 2) return go(router_stream_kernel<2>);
            if (nt <= 3) return go(router_stream_kernel<3>);
            if (nt <= 4) return go(router_stream_kernel<4>);
            return go(router_stream_kernel<8>);
        }
    }
    if (dtype == MOE_BF16 && a.d % 64 == 0) {
        const int R = a.E_r + 2 * a.n_const;
        const int smem = RM_WARPS * 16 * ((R + 7) & ~7) * 4;
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(router_mma_kernel), smem);
        if (e != cudaSuccess) return cuda_status(e);
        const int tiles = cdiv(a.T, 16);
        const int grid = std::max(1, std::min(tiles, num_sms() * 8));
        router_mma_kernel<<<grid, RM_WARPS * 32, smem, st>>>(a);
        count_launch();
        return cuda_status(cudaGetLastError());
    }
    const int grid = std::max(1, std::min(cdiv(a.T, R_TILE), num_sms()));
    cudaError_t e = dtype == MOE_BF16
                        ? ensure_smem_attr(reinterpret_cast<const void*>(router_kernel<__nv_bfloat16>), R_SMEM)
                        : ensure_smem_attr(reinterpret_cast<const void*>(router_kernel<float>), R_SMEM);
    if (e != cudaSuccess) return cuda_status(e);
    if (dtype == MOE_BF16) router_kernel<__nv_bfloat16><<<grid, R_WARPS * 32, R_SMEM, st>>>(a);
    else router_kernel<float><<<grid, R_WARPS * 32, R_SMEM, st>>>(a);
    count_launch();
    return cuda_status(cudaGetLastError());
}

moe_status launch_pk_select(const PkSelectArgs& a, cudaStream_t st)
{
    if (a.T == 0) return MOE_OK;
    constexpr int warps = 8;
    const int n_max = std::max(a.rows, a.cols);
    cudaError_t e = n_max <= 512 ? ensure_smem_attr(reinterpret_cast<const void*>(pk_select_kernel<16>),
                                                    warps * (int)sizeof(PkWarpSmem<16>))
                                 : ensure_smem_attr(reinterpret_cast<const void*>(pk_select_kernel<32>),
                                                    warps * (int)sizeof(PkWarpSmem<32>));
    if (e != cudaSuccess) return cuda_status(e);
    const int grid = std::max(1, std::min(cdiv(a.T, warps), num_sms() * MOE_PK_MINB));
    const int n = std::max(a.rows, a.cols);
    if (n <= 512) pk_select_kernel<16><<<grid, warps * 32, warps * sizeof(PkWarpSmem<16>), st>>>(a);
    else pk_select_kernel<32><<<grid, warps * 32, warps * sizeof(PkWarpSmem<32>), st>>>(a);
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
