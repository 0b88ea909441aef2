// gemm_tc.cu -- persistent grouped GEMM on 5th-generation tensor cores.
//
// The expert-centric step of the layer ("OmniMoE" technical summary, 2.2
// Expert-Centric Scheduling, Grouped GEMM): rows that chose the same expert
// are contiguous, so one block of that expert's weights, once in shared
// memory, serves up to 128 rows.  Groups have data-dependent sizes; the
// tile schedule is built on the device from the group offsets, so nothing
// is copied back to the host.
//
// Structure (one CTA per SM, 6 warps):
//   warp 0   TMA producer: A tile [128 x 64] + B tile [256 x 64] per stage,
//            128-byte swizzle, 4-stage mbarrier ring (no multicast); the
//            CTA-pair forms below use 3 stages of 128-wide K instead.
//   warp 1   TMEM allocator and MMA issuer: tcgen05.mma kind::f16,
//            M=128 N=256 K=16, fp32 accumulators in TMEM, two accumulator
//            buffers (512 columns) so the epilogue of one tile overlaps the
//            MMAs of the next.
//   warps 2-5 epilogue: tcgen05.ld of their 32-lane quarter, fused
//            activation (SwiGLU: silu(gate) * up), bf16/fp32 store.
// Two more forms run on clusters of two CTAs (tcgen05.mma.cta_group::2,
// M = 256): 256-row tiles of a group's rows, and the token-column form
// (weight rows as M, a group's rows as N in steps of 16), which the pair form
// uses for the fp32 down projection and for SwiGLU from K = 2048; its SwiGLU
// instance runs eight epilogue warps (10 in all).
// Every mbarrier wait is bounded (2 s); a timeout sets MOE_ERR_TIMEOUT, all
// roles leave their loops, in-flight TMA copies are drained and TMEM freed.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

#ifndef MOE_KB_FENCE
#define MOE_KB_FENCE 0            // tcgen05 fence after every stage wait (TMA -> MMA needs none)
#endif

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_MMA = 256;
constexpr int STAGES = 4;
constexpr int TILE_A = BM * BK * 2;        // 16 KB
constexpr int TILE_B = BN_MMA * BK * 2;    // 32 KB
constexpr int STAGE_BYTES = TILE_A + TILE_B;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int NTHREADS = 192;
constexpr int SMEM_TABLE_INTS = 4 * kMaxGemmGroups + 2;   // + the token-column tile widths and schedule flag
constexpr int EPI_STAGE_BYTES = 32 * 128;      // one 32-row x 128-byte output box per epilogue warp
constexpr int EPI_WARPS = 4;
__host__ __device__ constexpr int epi_stage_offset(int stage_bytes)
{
    return ((stage_bytes + 256 + SMEM_TABLE_INTS * 4) + 1023) / 1024 * 1024;
}
constexpr int SMEM_BYTES = 1024 + epi_stage_offset(STAGES * STAGE_BYTES) + EPI_WARPS * EPI_STAGE_BYTES;

struct DevArgs {
    const int32_t* offsets;
    int n_groups, n_first, group_rows, N, K;
    int b_kmod;                 // > 0: B's k coordinate is k mod b_kmod
    void* out;
    long long ldo;
    long long rows_cap;
    int pk_T, pk_dq;
    // fused permutation / combine (token-column form only)
    const int32_t* rows;        // row r of the grouped operand is token rows[r] (token_of)
    int rows_T;                 // tokens (bound of rows[r])
    float* acc;                 // [rows_T, acc_d] fp32 combine accumulator
    int acc_d;
    const int32_t* idx;         // [rows_T, k] routing (gate lookup of the scatter-add epilogue)
    const float* gate;          // [rows_T, k]
    int k;
    // e4m3 operands (token-column form): out = acc * sa[weight row] * sb[token row]
    const float* sa0;           // row scales of B0 (gate / down), B1 (up), B2, B3 (shared experts)
    const float* sa1;
    const float* sa2;
    const float* sa3;
    const float* sb;            // [rows] row scales of the token-row operand
};

struct TileInfo {
    int g;        // group
    int row0;     // first A row of the tile
    int rows;     // valid rows in the tile (<= BM)
    int n;        // n-tile index inside the group
};

template <int TBM = BM>
__device__ __forceinline__ TileInfo decode_tile(int tile, const int* tile_start, const int* g_lo,
                                                const int* g_cnt, int n_groups)
{
    int lo = 0, hi = n_groups - 1;   // last g with tile_start[g] <= tile
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    TileInfo ti;
    ti.g = lo;
    const int cnt = g_cnt[lo];
    const int mt = cdiv(cnt, TBM);
    const int local = tile - tile_start[lo];
    const int m = local % mt;       // m-tiles of a group are adjacent: they share B
    ti.n = local / mt;
    ti.row0 = g_lo[lo] + m * TBM;
    ti.rows = min(TBM, cnt - m * TBM);
    return ti;
}

// silu(g) * u uses the fast divide: the IEEE division was the cost of the
// SwiGLU epilogue, which short-K GEMMs (K = 1024-2048) cannot hide behind
// their mainloop (measured: shared-branch gate/up 114.6 -> 69.8 us).  The
// result is within 2 ulp of g / (1 + e^-g) for 1 + e^-g < 2^126 and 0 below
// g = -87 (where silu(g) < 1e-36).
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const DevArgs& a, uint32_t tacc, const TileInfo& ti,
                                              int r)
{
    const long long grow = (long long)ti.row0 + r;
    const bool valid = (r < ti.rows) && (grow < a.rows_cap);
    if constexpr (EPI == EPI_SWIGLU) {
        // accumulator columns [0,128) = gate, [128,256) = up for h columns n*128 ...
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
        const int col0 = ti.n * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t g[32], u[32];
            tmem_ld32(tacc + c * 32, g);
            tmem_ld32(tacc + 128 + c * 32, u);
            tc_wait_ld();
            if (valid) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                    float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                    float h0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
                    float h1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
                    pk[i] = pack_bf16(h0, h1);
                }
                uint4* dst = reinterpret_cast<uint4*>(out + grow * a.ldo + col0 + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    } else if constexpr (EPI == EPI_BF16) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
        const int col0 = ti.n * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld32(tacc + c * 32, v);
            tc_wait_ld();
            if (valid && col0 + c * 32 < a.N) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                uint4* dst = reinterpret_cast<uint4*>(out + grow * a.ldo + col0 + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        }
    } else if constexpr (EPI == EPI_F32) {
        float* out = reinterpret_cast<float*>(a.out);
        const int col0 = ti.n * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld32(tacc + c * 32, v);
            tc_wait_ld();
            if (valid && col0 + c * 32 < a.N) {
                uint4* dst = reinterpret_cast<uint4*>(out + grow * a.ldo + col0 + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    } else {   // EPI_PK_SPLIT: q = x W_q^T split into three bf16 parts per half
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
        const int col0 = ti.n * 256;
        const int half = a.pk_dq / 2;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld32(tacc + c * 32, v);
            tc_wait_ld();
            const int col = col0 + c * 32;
            if (valid && col < a.N) {
                const int hf = col / half, cc = col % half;
                __nv_bfloat16* dst = out + ((long long)hf * a.pk_T + grow) * a.ldo + cc;
                uint32_t p0[16], p1[16], p2[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float q0 = __uint_as_float(v[2 * i]), q1 = __uint_as_float(v[2 * i + 1]);
                    __nv_bfloat16 a0 = __float2bfloat16_rn(q0), a1 = __float2bfloat16_rn(q1);
                    float r0 = q0 - __bfloat162float(a0), r1 = q1 - __bfloat162float(a1);
                    __nv_bfloat16 b0 = __float2bfloat16_rn(r0), b1 = __float2bfloat16_rn(r1);
                    float s0 = r0 - __bfloat162float(b0), s1 = r1 - __bfloat162float(b1);
                    p0[i] = pack_bf16(__bfloat162float(a0), __bfloat162float(a1));
                    p1[i] = pack_bf16(__bfloat162float(b0), __bfloat162float(b1));
                    p2[i] = pack_bf16(s0, s1);
                }
                uint4* d0 = reinterpret_cast<uint4*>(dst);
                uint4* d1 = reinterpret_cast<uint4*>(dst + half);
                uint4* d2 = reinterpret_cast<uint4*>(dst + 2 * half);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    d0[i] = make_uint4(p0[4 * i], p0[4 * i + 1], p0[4 * i + 2], p0[4 * i + 3]);
                    d1[i] = make_uint4(p1[4 * i], p1[4 * i + 1], p1[4 * i + 2], p1[4 * i + 3]);
                    d2[i] = make_uint4(p2[4 * i], p2[4 * i + 1], p2[4 * i + 2], p2[4 * i + 3]);
                }
            }
        }
    }
}

// The epilogue of one warp's 32 rows when all of them are valid: each
// 128-byte column chunk of the 32 rows (32 fp32 or 64 bf16 values per row)
// is written into the warp's 4 KiB staging box in the 128-byte swizzled
// layout (16-byte unit j of row r at unit j ^ (r & 7): conflict-free) and
// stored with one TMA store, so global memory sees whole lines instead of
// one 16-byte piece per row per instruction.  The next chunk's TMEM load
// overlaps the wait for the previous store to finish reading the box.
// Blocks with invalid rows (the end of a group) take epilogue_tile.
template <int EPI>
__device__ __forceinline__ void epilogue_block_tma(const DevArgs& a, const CUtensorMap* tm_out, uint32_t tacc,
                                                   const TileInfo& ti, int q, int lane, uint8_t* box)
{
    if (ti.rows < q * 32 + 32) {
        epilogue_tile<EPI>(a, tacc, ti, q * 32 + lane);
        return;
    }
    const int row = ti.row0 + q * 32;
    uint4* mine = reinterpret_cast<uint4*>(box + lane * 128);
    auto put = [&](const uint32_t (&w)[32], int col) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j) mine[j ^ (lane & 7)] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tm_out, box, col, row);
            bulk_commit();
        }
    };
    if constexpr (EPI == EPI_SWIGLU) {
        const int col0 = ti.n * 128;
#pragma unroll 1
        for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t w[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c = 2 * c2 + hh;
                uint32_t g[32], u[32];
                tmem_ld32(tacc + c * 32, g);
                tmem_ld32(tacc + 128 + c * 32, u);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                    const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                    w[16 * hh + i] = pack_bf16(__fdividef(g0, 1.0f + __expf(-g0)) * u0, __fdividef(g1, 1.0f + __expf(-g1)) * u1);
                }
            }
            put(w, col0 + c2 * 64);
        }
    } else if constexpr (EPI == EPI_BF16) {
        const int col0 = ti.n * 256;
#pragma unroll 1
        for (int c2 = 0; c2 < 4; ++c2) {
            if (col0 + c2 * 64 >= a.N) break;
            uint32_t w[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t v[32];
                tmem_ld32(tacc + (2 * c2 + hh) * 32, v);
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[16 * hh + i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            }
            put(w, col0 + c2 * 64);
        }
    } else {   // EPI_F32
        const int col0 = ti.n * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            if (col0 + c * 32 >= a.N) break;
            uint32_t v[32];
            tmem_ld32(tacc + c * 32, v);
            tc_wait_ld();
            put(v, col0 + c * 32);
        }
    }
}

template <int EPI>
__device__ __forceinline__ void epilogue_any(const DevArgs& a, const CUtensorMap* tm_out, uint32_t tacc,
                                             const TileInfo& ti, int q, int lane, uint8_t* box)
{
    // the split query keeps direct stores: its three parts per chunk would
    // serialise on the one staging box (measured slower)
    if constexpr (EPI == EPI_PK_SPLIT) epilogue_tile<EPI>(a, tacc, ti, q * 32 + lane);
    else epilogue_block_tma<EPI>(a, tm_out, tacc, ti, q, lane, box);
}

// Warp 0 builds, for every group, its first row, its row count and the index
// of its first output tile (tiles of TBM rows x one n-tile).
template <int TBM>
__device__ __forceinline__ void build_group_table(const DevArgs& a, int ntn, int lane, int* tile_start,
                                                  int* g_lo, int* g_cnt)
{
    const int n = a.n_groups;
    const int chunk = cdiv(n, 32);
    const int g0 = min(n, lane * chunk), g1 = min(n, g0 + chunk);
    int local = 0;
    for (int g = g0; g < g1; ++g) {
        int lo, hi;
        if (a.offsets) { lo = a.offsets[g]; hi = a.offsets[g + 1]; }
        else { lo = g * a.group_rows; hi = lo + a.group_rows; }
        int cnt = hi - lo;
        if (cnt < 0 || lo < 0) { set_status(MOE_ERR_DEVICE_BOUNDS); cnt = 0; lo = 0; }
        g_lo[g] = lo;
        g_cnt[g] = cnt;
        local += cdiv(cnt, TBM) * ntn;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
        tile_start[g] = run;
        run += cdiv(g_cnt[g], TBM) * ntn;
    }
    if (lane == 31) tile_start[n] = incl;
}

template <int EPI>
__global__ void __launch_bounds__(NTHREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmOut,
                    const DevArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * TILE_A;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * TILE_B);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* tile_start = reinterpret_cast<int*>(smem + STAGES * STAGE_BYTES + 256);
    int* g_lo = tile_start + (kMaxGemmGroups + 1);
    int* g_cnt = g_lo + kMaxGemmGroups;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntn = (EPI == EPI_SWIGLU) ? cdiv(a.N, 128) : cdiv(a.N, 256);

    if (warp == 0) build_group_table<BM>(a, ntn, lane, tile_start, g_lo, g_cnt);
    if (threadIdx.x == 32) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 128); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB0); tma_prefetch_desc(&tmB1);
        tma_prefetch_desc(&tmB2); tma_prefetch_desc(&tmB3);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[a.n_groups];
    const int nk = cdiv(a.K, BK);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, arm_par = 0;   // per stage: copies in flight, their parity
            bool bad = false;
            for (int tile = blockIdx.x; tile < total && !bad; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, tile_start, g_lo, g_cnt, a.n_groups);
                const bool first = ti.g < a.n_first;
                const int gb = first ? ti.g : ti.g - a.n_first;
                const CUtensorMap* mlo = first ? &tmB0 : &tmB2;
                const CUtensorMap* mhi;
                int brow_lo, brow_hi;
                if (EPI == EPI_SWIGLU) {
                    mhi = first ? &tmB1 : &tmB3;
                    brow_lo = gb * a.N + ti.n * 128;
                    brow_hi = brow_lo;
                } else {
                    mhi = mlo;
                    brow_lo = gb * a.N + ti.n * 256;
                    brow_hi = brow_lo + 128;
                }
                for (int kb = 0; kb < nk; ++kb) {
                    if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1)) { *abort_flag = 1; bad = true; break; }
                    armed &= ~(1u << s);
                    mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                    tma_load_2d(sA + s * TILE_A, &tmA, &full[s], kb * BK, ti.row0);
                    const int kbb = a.b_kmod ? (kb * BK) % a.b_kmod : kb * BK;
                    tma_load_2d(sB + s * TILE_B, mlo, &full[s], kbb, brow_lo);
                    tma_load_2d(sB + s * TILE_B + TILE_B / 2, mhi, &full[s], kbb, brow_hi);
                    armed |= 1u << s;
                    arm_par = (arm_par & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (bad) {   // let copies already in flight land before the CTA exits
                for (int i = 0; i < STAGES; ++i)
                    if (armed & (1u << i)) mbar_wait(&full[i], (arm_par >> i) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idesc = idesc_bf16_f32(BM, BN_MMA);
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool bad = false;
            for (int tile = blockIdx.x; tile < total && !bad; tile += gridDim.x) {
                if (*abort_flag || !mbar_wait(&acc_empty[acc], aph ^ 1)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < nk; ++kb) {
                    if (*abort_flag || !mbar_wait(&full[s], ph)) { *abort_flag = 1; bad = true; break; }
#if MOE_KB_FENCE
                    tc_fence_after();
#endif
                    const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * TILE_A));
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * TILE_B));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                    tc_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (bad) break;
                tc_commit(&acc_full[acc]);
                if (++acc == 2) { acc = 0; aph ^= 1; }
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        uint8_t* epi_box = smem + epi_stage_offset(STAGES * STAGE_BYTES) + (warp - 2) * EPI_STAGE_BYTES;
        int acc = 0;
        uint32_t aph = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileInfo ti = decode_tile(tile, tile_start, g_lo, g_cnt, a.n_groups);
            if (*abort_flag || !mbar_wait(&acc_full[acc], aph)) { *abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
            epilogue_any<EPI>(a, &tmOut, tacc, ti, q, lane, epi_box);
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
            if (++acc == 2) { acc = 0; aph ^= 1; }
        }
        if (lane == 0) bulk_wait<0>();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------ CTA-pair kernel
//
// Same schedule and epilogues, but each output tile is 256 rows x 256 columns
// computed by a cluster of two CTAs on two SMs with tcgen05.mma.cta_group::2:
// CTA r stages A rows [128 r, 128 r + 128) of the tile and half of B (SwiGLU:
// CTA 0 the gate rows, CTA 1 the up rows; otherwise output columns
// [128 r, 128 r + 128)), and holds accumulator rows [128 r, 128 r + 128) in
// its own TMEM.  B is read from L2 once per pair instead of once per SM.
// The leader CTA (rank 0) issues the MMAs; both CTAs' TMA copies complete on
// the leader's stage barrier; the leader's commits arrive on both CTAs'
// barriers; the peer's epilogue warps release the accumulator remotely.
// No multicast loads.

constexpr int P_BM = 256;
// K per stage = 64 * MOE_P_KH: one issuing thread drives the tensor cores of
// both SMs and pays a wait / commit / loop per stage, so wider stages (more
// MMAs each) keep it ahead of the tensor pipe.
#ifndef MOE_P_KH
#define MOE_P_KH 2
#endif
#ifndef MOE_P_STAGES
#define MOE_P_STAGES (6 / MOE_P_KH)
#endif
constexpr int P_KH = MOE_P_KH;

constexpr int P_STAGES = MOE_P_STAGES;
constexpr int P_HALF = 128 * BK * 2;         // one 128-row x 64-K box: 16 KB
constexpr int P_TILE_A = P_KH * P_HALF;      // A: 128 rows x 64*KH of K
constexpr int P_TILE_B = P_KH * P_HALF;
constexpr int P_STAGE_BYTES = P_TILE_A + P_TILE_B;
constexpr int P_SMEM_BYTES = 1024 + epi_stage_offset(P_STAGES * P_STAGE_BYTES) + EPI_WARPS * EPI_STAGE_BYTES;
static_assert(SMEM_BYTES <= 232448 && P_SMEM_BYTES <= 232448, "shared memory per block");

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                         const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                         const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmOut,
                         const DevArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + P_STAGES * P_TILE_A;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + P_STAGES * P_TILE_B);
    uint64_t* empty = full + P_STAGES;
    uint64_t* acc_full = empty + P_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* tile_start = reinterpret_cast<int*>(smem + P_STAGES * P_STAGE_BYTES + 256);
    int* g_lo = tile_start + (kMaxGemmGroups + 1);
    int* g_cnt = g_lo + kMaxGemmGroups;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int ntn = (EPI == EPI_SWIGLU) ? cdiv(a.N, 128) : cdiv(a.N, 256);

    if (warp == 0) build_group_table<P_BM>(a, ntn, lane, tile_start, g_lo, g_cnt);
    if (threadIdx.x == 32) {
        for (int s = 0; s < P_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 8); }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc_pair(tmem_slot, TMEM_COLS); tmem_relinquish_pair(); }
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB0); tma_prefetch_desc(&tmB1);
        tma_prefetch_desc(&tmB2); tma_prefetch_desc(&tmB3);
    }
    tc_fence_before();
    cluster_sync_all();          // both CTAs: barriers initialised, TMEM allocated
    tc_fence_after();

    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[a.n_groups];
    const int pnk = cdiv(a.K, BK * P_KH);          // stages of K per tile
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const uint32_t full_leader = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(&acc_empty[0]), 0);

    if (warp == 0) {
        if (lane == 0) {
            // -------------------------------------------- TMA producer (both CTAs)
            int s = 0;
            uint32_t ph = 0;
            bool bad = false;
            for (int tile = cluster; tile < total && !bad; tile += n_clusters) {
                const TileInfo ti = decode_tile<P_BM>(tile, tile_start, g_lo, g_cnt, a.n_groups);
                const bool first = ti.g < a.n_first;
                const int gb = first ? ti.g : ti.g - a.n_first;
                const CUtensorMap* mb;
                int brow;
                if (EPI == EPI_SWIGLU) {
                    mb = rank == 0 ? (first ? &tmB0 : &tmB2) : (first ? &tmB1 : &tmB3);
                    brow = gb * a.N + ti.n * 128;
                } else {
                    mb = first ? &tmB0 : &tmB2;
                    brow = gb * a.N + ti.n * 256 + (int)rank * 128;
                }
                const int arow = ti.row0 + (int)rank * 128;
                if (*abort_flag) { bad = true; break; }
                for (int kb = 0; kb < pnk; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1)) { *abort_flag = 1; bad = true; break; }
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * P_STAGE_BYTES);
#pragma unroll
                    for (int h = 0; h < P_KH; ++h) {
                        const int k0 = (kb * P_KH + h) * BK;      // past K: zero fill
                        tma_load_2d_pair(sA + s * P_TILE_A + h * P_HALF, &tmA, full_leader + 8 * s, k0, arow);
                        tma_load_2d_pair(sB + s * P_TILE_B + h * P_HALF, mb, full_leader + 8 * s,
                                         a.b_kmod ? k0 % a.b_kmod : k0, brow);
                    }
                    if (++s == P_STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (bad) {   // copies already issued land within microseconds; let them
                const uint64_t t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) { }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------- MMA issuer (leader only)
            const uint32_t idesc = idesc_bf16_f32(P_BM, BN_MMA);
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool bad = false;
            const uint64_t ad0 = sw128_kmajor_desc(smem_u32(sA));
            const uint64_t bd0 = sw128_kmajor_desc(smem_u32(sB));
            for (int tile = cluster; tile < total && !bad; tile += n_clusters) {
                if (*abort_flag || !mbar_wait(&acc_empty[acc], aph ^ 1)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < pnk; ++kb) {
                    if (!mbar_wait(&full[s], ph)) { *abort_flag = 1; bad = true; break; }
#if MOE_KB_FENCE
                    tc_fence_after();
#endif
                    // descriptor start addresses advance in 16-byte units
                    const uint64_t ad = ad0 + (uint64_t)((s * P_TILE_A) >> 4);
                    const uint64_t bd = bd0 + (uint64_t)((s * P_TILE_B) >> 4);
#pragma unroll
                    for (int h = 0; h < P_KH; ++h)
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc_mma_bf16_pair(d_tmem, ad + (h * P_HALF >> 4) + 2 * kk, bd + (h * P_HALF >> 4) + 2 * kk,
                                             idesc, (kb | h | kk) != 0);
                    tc_commit_pair(&empty[s], 0x3);
                    if (++s == P_STAGES) { s = 0; ph ^= 1; }
                }
                if (bad) break;
                tc_commit_pair(&acc_full[acc], 0x3);
                if (++acc == 2) { acc = 0; aph ^= 1; }
            }
            // every MMA issued has completed before the CTAs may leave
            tc_commit_pair(mma_done, 0x1);
            mbar_wait(mma_done, 0);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        uint8_t* epi_box = smem + epi_stage_offset(P_STAGES * P_STAGE_BYTES) + (warp - 2) * EPI_STAGE_BYTES;
        int acc = 0;
        uint32_t aph = 0;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            TileInfo ti = decode_tile<P_BM>(tile, tile_start, g_lo, g_cnt, a.n_groups);
            ti.row0 += (int)rank * 128;
            ti.rows = max(0, min(128, ti.rows - (int)rank * 128));
            if (*abort_flag || !mbar_wait(&acc_full[acc], aph)) { *abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
            epilogue_any<EPI>(a, &tmOut, tacc, ti, q, lane, epi_box);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader + 8 * acc);
            if (++acc == 2) { acc = 0; aph ^= 1; }
        }
        if (lane == 0) bulk_wait<0>();
    }

    tc_fence_before();
    cluster_sync_all();          // all MMAs done and all TMEM reads issued in both CTAs
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------ token-column pair kernel
//
// The pair kernel above makes a group's rows the MMA's M side, so a group
// whose row count is not a multiple of 256 pays for a whole 256-row tile at
// its end: Mixtral-shaped groups of about 1024 +- 30 rows cost 36 tiles of
// MMA work for 32 tiles of rows, and the last wave of the static schedule
// decides the time.  This form swaps the operands: the expert's weight rows
// are M (256 per pair, always full) and the group's rows are N, which the
// tensor cores take in steps of 16.  A group of c rows is cut into
// ceil(c / 256) token tiles of one width w = ceil16(c / that count), so the
// tiles of a group cost the same, the round-robin schedule stays balanced and
// the padding is under 16 rows per tile.  Tile order: group, weight block,
// token tile (the token tiles sharing a weight block run side by side).
//   fp32 epilogue (down projection): TMEM lane = output feature, column =
//     token; each warp stores one token's 32 features (128 B) per instruction.
//   SwiGLU epilogue: each CTA stages 64 gate rows and the 64 up rows of the
//     same hidden units as its 128 A rows, so TMEM lanes 0-63 hold gate and
//     lanes 64-127 up of the same units; epilogue warps q and q + 2 swap
//     half of each 32-column chunk through shared memory and each applies
//     silu(gate) * up to its half.
// Used for the pair form's SwiGLU (N % 128 == 0) and fp32 (N % 256 == 0)
// epilogues; the other forms keep the row-tiled kernels.

#ifndef MOE_GEMM_TN
#define MOE_GEMM_TN 1
#endif
#ifndef MOE_TN_SWIGLU_MIN_K
#define MOE_TN_SWIGLU_MIN_K 2048
#endif
#ifndef MOE_TN_INTERLEAVE
#define MOE_TN_INTERLEAVE 1
#endif
#ifndef MOE_TN_FILL
#define MOE_TN_FILL 1
#endif

// Token-column kernel layout.  Its tile table holds at most TN_MAX_GROUPS
// groups.  SwiGLU runs eight epilogue warps (two per TMEM lane quarter, each
// taking every other 32-column chunk of a tile): with short K (e4m3 MoE++,
// K = 2048: a ~7 us mainloop per tile) four warps did not finish a tile's
// SwiGLU before the next accumulator was ready.  Each SwiGLU epilogue warp
// has a 3.5 KiB box: the exchange with its partner warp (2 KiB), the bf16
// output rows (1 KiB), and the e4m3 token-row scales of its chunks (512 B);
// an fp32 epilogue warp a 4 KiB box (one 32 x 32 fp32 chunk).
constexpr int TN_MAX_GROUPS = 256;
constexpr int TN_TABLE_INTS = 4 * TN_MAX_GROUPS + 2;
template <int EPI> constexpr int tn_epi_warps() { return EPI == EPI_SWIGLU ? 8 : 4; }
template <int EPI> constexpr int tn_threads() { return 64 + 32 * tn_epi_warps<EPI>(); }
template <int EPI> constexpr int tn_box_bytes() { return EPI == EPI_SWIGLU ? 3584 : 4096; }
constexpr int tn_epi_offset() { return ((P_STAGES * P_STAGE_BYTES + 256 + TN_TABLE_INTS * 4) + 1023) / 1024 * 1024; }
template <int EPI> constexpr int tn_smem_bytes() { return 1024 + tn_epi_offset() + tn_epi_warps<EPI>() * tn_box_bytes<EPI>(); }
static_assert(tn_smem_bytes<EPI_SWIGLU>() <= 232448 && tn_smem_bytes<EPI_F32>() <= 232448, "shared memory per block");

struct TnTile {
    int g;        // group
    int m;        // weight block (256 output features, or 128 hidden units for SwiGLU)
    int tok0;     // first row of the token tile
    int valid;    // rows of the tile (1..256)
    int nt;       // MMA N: valid rounded up to 16
};

__device__ __forceinline__ int tn_width(int cnt)
{
    const int t = cdiv(cnt, 256);
    return (cdiv(cnt, t) + 15) & ~15;
}

// Token-tile width of a group of cnt rows cut into t tiles (t >= ceil(cnt / 256)).
__device__ __forceinline__ int tn_width_t(int cnt, int t)
{
    return (cdiv(cnt, t) + 15) & ~15;
}

__device__ __forceinline__ TnTile decode_tn(int tile, const int* tile_start, const int* g_lo, const int* g_cnt,
                                            const int* g_w, int n_groups, int ntm)
{
    int lo = 0, hi = n_groups - 1;   // last g with tile_start[g] <= tile
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    TnTile ti;
    ti.g = lo;
    const int cnt = g_cnt[lo];
    const int w = g_w[lo];
    const int nj = cdiv(cnt, w);
    const int local = tile - tile_start[lo];
    ti.m = local / nj;
    const int j = local - ti.m * nj;
    ti.tok0 = g_lo[lo] + j * w;
    ti.valid = min(w, cnt - j * w);
    ti.nt = (ti.valid + 15) & ~15;
    return ti;
}

// Schedule position s (tile s of the round-robin over n_clusters pairs) ->
// tile id.  Plain: the identity (group, weight block, token tile order).
// Mixed: the positions of each wave are dealt alternately from the front and
// from the back of the tile list, and a pair alternates between the two from
// one wave to the next.  With long-tail groups the front holds the head
// experts' wide tiles (MMA-bound: N = 256 with the weight block shared by
// several token tiles in L2) and the back the tail experts' narrow ones
// (bound by streaming a weight block for N = 16..64 columns), so every wave
// keeps both the tensor pipes and the DRAM busy instead of running the MMA
// phase and then the streaming phase.  The token tiles of a weight block stay
// next to one another in each half.  A bijection of [0, total): the front
// takes tiles [0, F) in order and the back tiles [F, total) from the end,
// where F is the number of front positions.
__device__ __forceinline__ int tn_order(int s, int total, int n_clusters, bool mixed)
{
    if (!mixed) return s;
    if (n_clusters & 1)   // odd: the position's parity alternates per pair and wave by itself
        return (s & 1) ? total - 1 - (s >> 1) : (s >> 1);
    const int half = n_clusters >> 1;
    const int w = s / n_clusters, p = s - w * n_clusters;
    const int f = (w & 1) ? (p >> 1) : ((p + 1) >> 1);   // front positions before p in wave w
    return ((p + w) & 1) == 0 ? w * half + f : total - 1 - (w * half + (p - f));
}

// Warp 0 builds the token-column tile table: each group's first row, row
// count and token-tile width, the first tile of each group, and the schedule
// flag.  A group of c rows starts with ceil(c / 256) token tiles of one width
// (tn_width).  When the groups are alike (not mixed), the round-robin's last
// wave is then often a fraction of the pairs (Mixtral-shaped down GEMM: 608
// tiles of 208-256 columns on 74 pairs, 8.2 waves), so token tiles are added
// one at a time to the group whose tiles are widest for as long as the tile
// count stays within the same number of waves: the waves fill up with tiles
// of nearly equal width (656 tiles of 176-256 columns) and the pairs finish
// together.  The MMA columns stay those of the rows, rounded to 16 per tile.
__device__ __forceinline__ void build_group_table_tn(const DevArgs& a, int ntm, int n_clusters, int lane,
                                                     int* tile_start, int* g_lo, int* g_cnt, int* g_w, int* mixed)
{
    const int n = a.n_groups;
    const int chunk = cdiv(n, 32);
    const int g0 = min(n, lane * chunk), g1 = min(n, g0 + chunk);
    int local = 0, wmin = 1 << 30, wmax = 0;
    for (int g = g0; g < g1; ++g) {
        int lo, hi;
        if (a.offsets) { lo = a.offsets[g]; hi = a.offsets[g + 1]; }
        else { lo = g * a.group_rows; hi = lo + a.group_rows; }
        int cnt = hi - lo;
        if (cnt < 0 || lo < 0) { set_status(MOE_ERR_DEVICE_BOUNDS); cnt = 0; lo = 0; }
        g_lo[g] = lo;
        g_cnt[g] = cnt;
        if (cnt > 0) { wmin = min(wmin, tn_width(cnt)); wmax = max(wmax, tn_width(cnt)); }
    }
    // groups whose tiles differ in width by 2x or more: the interleaved schedule
    wmin = __reduce_min_sync(0xffffffffu, wmin);
    wmax = __reduce_max_sync(0xffffffffu, wmax);
    const bool mix = MOE_TN_INTERLEAVE && wmax >= 2 * wmin;
    if (lane == 0) *mixed = mix;
    // token tiles per group (kept in g_w until the widths are set)
    int tsum = 0;
    for (int g = g0; g < g1; ++g) {
        const int t = g_cnt[g] > 0 ? cdiv(g_cnt[g], 256) : 0;
        g_w[g] = t;
        tsum += t;
    }
    tsum = __reduce_add_sync(0xffffffffu, tsum);
    if (MOE_TN_FILL && !mix && tsum > 0) {
        const long long cap = (long long)cdiv(ntm * tsum, n_clusters) * n_clusters;   // whole waves
        int budget = min((int)(cap / ntm) - tsum, 256);
        __syncwarp();
        for (; budget > 0; --budget) {
            // the group with the widest token tiles (ties: the lower id) that can still narrow
            int bw = 0, bg = -1;
            for (int g = g0; g < g1; ++g) {
                const int c = g_cnt[g];
                if (c <= 0) continue;
                const int w = tn_width_t(c, g_w[g]);
                if (w > 16 && w > bw) { bw = w; bg = g; }
            }
            const int best = __reduce_max_sync(0xffffffffu, bw);
            if (best == 0) break;
            const unsigned cand = __ballot_sync(0xffffffffu, bw == best);
            if (lane == __ffs(cand) - 1) g_w[bg] += 1;   // lower lanes own lower ids
            __syncwarp();
        }
    }
    local = 0;
    for (int g = g0; g < g1; ++g) {
        const int c = g_cnt[g];
        const int w = c > 0 ? tn_width_t(c, g_w[g]) : 16;
        g_w[g] = w;
        local += c > 0 ? cdiv(c, w) * ntm : 0;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int g = g0; g < g1; ++g) {
        tile_start[g] = run;
        run += g_cnt[g] > 0 ? cdiv(g_cnt[g], g_w[g]) * ntm : 0;
    }
    if (lane == 31) tile_start[n] = incl;
}

// Named barrier of the two warps (64 threads) of one SwiGLU epilogue team.
__device__ __forceinline__ void team_sync(int id)
{
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// Team barrier that also returns whether `v` holds in every thread of both warps.
__device__ __forceinline__ bool team_all(bool v, int id)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, 64, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(id) : "memory");
    return r != 0;
}

// Runs body(v, ch) over the 32-column chunks ch0, ch0 + step, ... < nch of an
// accumulator, loading the next of them from TMEM while one is processed.
template <typename F>
__device__ __forceinline__ void tmem_chunks(uint32_t tacc, int nch, F&& body, int ch0 = 0, int step = 1)
{
    if (ch0 >= nch) return;
    uint32_t va[32], vb[32];
    tmem_ld32(tacc + ch0 * 32, va);
    tc_wait_ld_regs(va);
#pragma unroll 1
    for (int ch = ch0; ch < nch; ch += 2 * step) {
        const int c1 = ch + step, c2 = ch + 2 * step;
        const bool more = c1 < nch;
        if (more) tmem_ld32(tacc + c1 * 32, vb);
        body(va, ch);
        if (more) {
            tc_wait_ld_regs(vb);
            if (c2 < nch) tmem_ld32(tacc + c2 * 32, va);
            body(vb, c1);
            if (c2 < nch) tc_wait_ld_regs(va);
        }
    }
}

// MODE flags: TN_GATHER (SwiGLU: the token rows of the B operand are gathered
// from x by `rows` with tile::gather4 loads instead of read from x_sorted),
// TN_ZERO_ACC (SwiGLU: each tile zeroes its share of its tokens' fp32 combine
// accumulator rows), TN_SCATTER_ADD (fp32: each output row is scaled by its
// token's gate for this group's expert and added into the accumulator row of
// its token with vector atomics).
enum TnMode { TN_PLAIN = 0, TN_GATHER = 1, TN_SCATTER_ADD = 2, TN_ZERO_ACC = 4 };

// FP8: both operands e4m3 (kind::f8f6f4); a 128-byte box row holds 128
// elements of K instead of 64, and the epilogue applies the row scales.
template <int EPI, int MODE, bool FP8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(tn_threads<EPI>(), 1)
grouped_gemm_tn_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW0,
                       const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                       const __grid_constant__ CUtensorMap tmW3, const DevArgs a)
{
    static_assert(EPI == EPI_SWIGLU || EPI == EPI_F32, "token-column form: SwiGLU or fp32 epilogue");
    static_assert(MODE == TN_PLAIN || (EPI == EPI_SWIGLU && (MODE == TN_ZERO_ACC || MODE == (TN_GATHER | TN_ZERO_ACC))) ||
                  (EPI == EPI_F32 && MODE == TN_SCATTER_ADD), "fused modes: gather / zeroing with SwiGLU, scatter-add with fp32");
    static_assert(!FP8 || MODE == TN_PLAIN, "e4m3 operands: the plain form");
    constexpr bool GATHER = (MODE & TN_GATHER) != 0;
    constexpr bool ZERO_ACC = (MODE & TN_ZERO_ACC) != 0;
    constexpr int BKE = FP8 ? 2 * BK : BK;        // K elements per 128-byte box row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + P_STAGES * P_TILE_A;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + P_STAGES * P_TILE_B);
    uint64_t* empty = full + P_STAGES;
    uint64_t* acc_full = empty + P_STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* mma_done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* tile_start = reinterpret_cast<int*>(smem + P_STAGES * P_STAGE_BYTES + 256);
    int* g_lo = tile_start + (TN_MAX_GROUPS + 1);
    int* g_cnt = g_lo + TN_MAX_GROUPS;
    int* g_w = g_cnt + TN_MAX_GROUPS;
    int* sched_mixed = g_w + TN_MAX_GROUPS;
    constexpr int EW = tn_epi_warps<EPI>();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int ntm = (EPI == EPI_SWIGLU) ? a.N / 128 : a.N / 256;   // weight blocks per expert

    if (warp == 0) build_group_table_tn(a, ntm, (int)gridDim.x >> 1, lane, tile_start, g_lo, g_cnt, g_w, sched_mixed);
    if (threadIdx.x == 32) {
        for (int s = 0; s < P_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        // every epilogue warp of both CTAs releases an accumulator
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 2 * EW); }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) { tmem_alloc_pair(tmem_slot, TMEM_COLS); tmem_relinquish_pair(); }
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tmX); tma_prefetch_desc(&tmW0); tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmW2); tma_prefetch_desc(&tmW3);
    }
    tc_fence_before();
    cluster_sync_all();          // both CTAs: barriers initialised, TMEM allocated
    tc_fence_after();

    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[a.n_groups];
    const int pnk = cdiv(a.K, BKE * P_KH);
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const bool mixed = *sched_mixed != 0;
    const uint32_t full_leader = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(&acc_empty[0]), 0);

    if (warp == 0) {
        if (GATHER || lane == 0) {
            // -------------------------------------------- TMA producer (both CTAs)
            // (gather: all 32 lanes; lane L loads rows 4L .. 4L + 3 of the CTA's
            // half of the token tile, lane 0 also the weights and the barriers)
            int s = 0;
            uint32_t ph = 0;
            bool bad = false;
            for (int tile = cluster; tile < total && !bad; tile += n_clusters) {
                const TnTile ti = decode_tn(tn_order(tile, total, n_clusters, mixed), tile_start, g_lo, g_cnt, g_w,
                                            a.n_groups, ntm);
                const bool first = ti.g < a.n_first;
                const int gb = first ? ti.g : ti.g - a.n_first;
                // A: weight rows of this CTA's half of M; B: this CTA's half of the tokens
                const int wrow = (EPI == EPI_SWIGLU) ? gb * a.N + ti.m * 128 + (int)rank * 64
                                                     : gb * a.N + ti.m * 256 + (int)rank * 128;
                const CUtensorMap* mw = first ? &tmW0 : &tmW2;
                const CUtensorMap* mu = first ? &tmW1 : &tmW3;
                const int half_n = ti.nt >> 1;
                const int xrow = ti.tok0 + (int)rank * half_n;
                int xr[4] = {0, 0, 0, 0};
                if constexpr (GATHER) {
                    // token of each of this lane's rows; columns past the tile's
                    // valid rows repeat its last row (their results are dropped)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int lrow = min((int)rank * half_n + 4 * lane + j, ti.valid - 1);
                        int t = a.rows[ti.tok0 + lrow];
                        if (t < 0 || t >= a.rows_T) { set_status(MOE_ERR_DEVICE_BOUNDS); t = 0; }
                        xr[j] = t;
                    }
                }
                const bool stop = GATHER ? __shfl_sync(0xffffffffu, *abort_flag, 0) != 0 : *abort_flag != 0;
                if (stop) { bad = true; break; }
                for (int kb = 0; kb < pnk; ++kb) {
                    bool ok = lane != 0 || mbar_wait(&empty[s], ph ^ 1);
                    if constexpr (GATHER) ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) { *abort_flag = 1; bad = true; break; }
                    // both CTAs' bytes of this stage: A, then B (gathered: half_n rows of 128 B per box)
                    if (lane == 0 && leader)
                        mbar_arrive_expect_tx(&full[s], GATHER ? 2 * P_KH * (P_HALF + half_n * 128) : 2 * P_STAGE_BYTES);
#pragma unroll
                    for (int h = 0; h < P_KH; ++h) {
                        const int k0 = (kb * P_KH + h) * BKE;     // past K: zero fill
                        uint8_t* da = sA + s * P_TILE_A + h * P_HALF;
                        uint8_t* db = sB + s * P_TILE_B + h * P_HALF;
                        if (lane == 0) {
                            if (EPI == EPI_SWIGLU) {   // 64 gate rows, then the 64 up rows of the same units
                                tma_load_2d_pair(da, mw, full_leader + 8 * s, k0, wrow);
                                tma_load_2d_pair(da + P_HALF / 2, mu, full_leader + 8 * s, k0, wrow);
                            } else {
                                tma_load_2d_pair(da, mw, full_leader + 8 * s, k0, wrow);
                            }
                            if (!GATHER) tma_load_2d_pair(db, &tmX, full_leader + 8 * s, k0, xrow);
                        }
                        if constexpr (GATHER) {
                            if (4 * lane < half_n)
                                tma_gather4_pair(db + 4 * lane * 128, &tmX, full_leader + 8 * s, k0, xr[0], xr[1], xr[2],
                                                 xr[3]);
                        }
                    }
                    if (++s == P_STAGES) { s = 0; ph ^= 1; }
                }
            }
            if (bad) {   // copies already issued land within microseconds; let them
                const uint64_t t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) { }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------- MMA issuer (leader only)
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool bad = false;
            const uint64_t ad0 = sw128_kmajor_desc(smem_u32(sA));
            const uint64_t bd0 = sw128_kmajor_desc(smem_u32(sB));
            for (int tile = cluster; tile < total && !bad; tile += n_clusters) {
                const TnTile ti = decode_tn(tn_order(tile, total, n_clusters, mixed), tile_start, g_lo, g_cnt, g_w,
                                            a.n_groups, ntm);
                const uint32_t idesc = FP8 ? idesc_e4m3_f32(P_BM, ti.nt) : idesc_bf16_f32(P_BM, ti.nt);
                if (*abort_flag || !mbar_wait(&acc_empty[acc], aph ^ 1)) { *abort_flag = 1; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < pnk; ++kb) {
                    if (!mbar_wait(&full[s], ph)) { *abort_flag = 1; bad = true; break; }
                    const uint64_t ad = ad0 + (uint64_t)((s * P_TILE_A) >> 4);
                    const uint64_t bd = bd0 + (uint64_t)((s * P_TILE_B) >> 4);
                    // four 32-byte K steps per 128-byte row (16 bf16 or 32 e4m3 elements each)
#pragma unroll
                    for (int h = 0; h < P_KH; ++h)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            if constexpr (FP8)
                                tc_mma_e4m3_pair(d_tmem, ad + (h * P_HALF >> 4) + 2 * kk,
                                                 bd + (h * P_HALF >> 4) + 2 * kk, idesc, (kb | h | kk) != 0);
                            else
                                tc_mma_bf16_pair(d_tmem, ad + (h * P_HALF >> 4) + 2 * kk,
                                                 bd + (h * P_HALF >> 4) + 2 * kk, idesc, (kb | h | kk) != 0);
                        }
                    tc_commit_pair(&empty[s], 0x3);
                    if (++s == P_STAGES) { s = 0; ph ^= 1; }
                }
                if (bad) break;
                tc_commit_pair(&acc_full[acc], 0x3);
                if (++acc == 2) { acc = 0; aph ^= 1; }
            }
            tc_commit_pair(mma_done, 0x1);
            mbar_wait(mma_done, 0);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;                   // TMEM lanes 32q .. 32q + 31
        const int ew = warp - 2;                  // epilogue warp 0 .. EW - 1
        const int half = ew >> 2;                 // SwiGLU: this warp's chunks are half, half + 2, ...
        constexpr int CSTEP = EW / 4;             // chunk step (1 with four epilogue warps)
        uint8_t* epi0 = smem + tn_epi_offset();
        float* mine = reinterpret_cast<float*>(epi0 + ew * tn_box_bytes<EPI>());
        const float* theirs = reinterpret_cast<const float*>(epi0 + (ew ^ 2) * tn_box_bytes<EPI>());
        const bool gate_warp = q < 2;
        const int team = 1 + (q & 1) + 2 * half;  // named barrier id of warps q and q ^ 2 of this half
        int acc = 0;
        uint32_t aph = 0;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            const TnTile ti = decode_tn(tn_order(tile, total, n_clusters, mixed), tile_start, g_lo, g_cnt, g_w,
                                            a.n_groups, ntm);
            // e4m3: the scales this tile's epilogue applies, loaded before the wait for
            // the accumulator so their latency hides behind it (loaded per chunk, the
            // scale of the token rows stalled every chunk: the short-K e4m3 SwiGLU GEMMs
            // were bound by their epilogue)
            float slp[8];                             // token-row scale of column (half + CSTEP c) * 32 + lane
            float s_lane = 1.f;                       // this lane's weight-row scale
            if constexpr (FP8) {
#pragma unroll
                for (int c = 0; c < 8 / CSTEP; ++c) {
                    const int cl = (half + CSTEP * c) * 32 + lane;
                    slp[c] = cl < ti.valid ? a.sb[ti.tok0 + cl] : 0.f;
                }
                const bool first = ti.g < a.n_first;
                const int gb = first ? ti.g : ti.g - a.n_first;
                if constexpr (EPI == EPI_F32) {
                    s_lane = (first ? a.sa0 : a.sa2)[(long long)gb * a.N + ti.m * 256 + (int)rank * 128 + q * 32 + lane];
                } else {
                    const float* sa = gate_warp ? (first ? a.sa0 : a.sa2) : (first ? a.sa1 : a.sa3);
                    s_lane = sa[(long long)gb * a.N + ti.m * 128 + (int)rank * 64 + (q & 1) * 32 + lane];
                }
            }
            bool ok = !*abort_flag && mbar_wait(&acc_full[acc], aph);
            if (EPI == EPI_SWIGLU) ok = team_all(ok, team);   // both warps of a team leave together
            if (!ok) { *abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + acc * ACC_COLS;
            const int nch = cdiv(ti.valid, 32);
            // Each chunk is turned in shared memory from (lane = feature, column =
            // token) into token rows, which the warp writes as 16-byte pieces.
            if constexpr (EPI == EPI_F32) {
                float* out = reinterpret_cast<float*>(a.out);
                float* stg = mine;                        // [32 tokens][32 features]
                const int f0 = ti.m * 256 + (int)rank * 128 + q * 32;
                tmem_chunks(tacc, nch, [&](const uint32_t (&v)[32], int ch) {
                    __syncwarp();                         // the previous chunk has been read
                    if constexpr (FP8) {                  // out = acc * s_weight_row * s_token_row
                        const float sl = slp[ch];
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            stg[i * 32 + lane] = __uint_as_float(v[i]) * s_lane * __shfl_sync(0xffffffffu, sl, i);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) stg[i * 32 + lane] = __uint_as_float(v[i]);
                    }
                    __syncwarp();
                    if constexpr (MODE == TN_SCATTER_ADD) {
                        // lane l: the token of row ch * 32 + l and its gate for this group's expert
                        int tl = -1;
                        float gl = 0.f;
                        const int cl = ch * 32 + lane;
                        if (cl < ti.valid) {
                            const int t = a.rows[ti.tok0 + cl];
                            if (t < 0 || t >= a.rows_T) {
                                set_status(MOE_ERR_DEVICE_BOUNDS);
                            } else {
                                for (int j = 0; j < a.k; ++j)
                                    if (a.idx[(long long)t * a.k + j] == ti.g) { tl = t; gl = a.gate[(long long)t * a.k + j]; }
                                if (tl < 0) set_status(MOE_ERR_DEVICE_BOUNDS);
                            }
                        }
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            const int idx = r * 32 + lane, row = idx >> 3, piece = idx & 7;
                            const int t = __shfl_sync(0xffffffffu, tl, row);
                            const float gg = __shfl_sync(0xffffffffu, gl, row);
                            if (t >= 0) {
                                const float4 w = *reinterpret_cast<const float4*>(stg + row * 32 + piece * 4);
                                red_add_v4(a.acc + (long long)t * a.acc_d + f0 + piece * 4, gg * w.x, gg * w.y,
                                           gg * w.z, gg * w.w);
                            }
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < 8; ++r) {
                            const int idx = r * 32 + lane, row = idx >> 3, piece = idx & 7;
                            const int c = ch * 32 + row;
                            const long long grow = (long long)ti.tok0 + c;
                            if (c < ti.valid && grow < a.rows_cap)
                                *reinterpret_cast<float4*>(out + grow * a.ldo + f0 + piece * 4) =
                                    *reinterpret_cast<const float4*>(stg + row * 32 + piece * 4);
                        }
                    }
                });
            } else {
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
                __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(mine) + 2048);
                const int unit0 = ti.m * 128 + (int)rank * 64 + (q & 1) * 32;
                // the gate warp finishes columns 0-15 of each chunk, the up warp 16-31
                auto finish = [&](const float (&g)[16], const float (&u)[16], int c0) {
                    __syncwarp();                         // the previous chunk has been read
#pragma unroll
                    for (int i = 0; i < 16; ++i)          // [16 tokens][32 units]
                        stg[i * 32 + lane] = __float2bfloat16_rn(__fdividef(g[i], 1.0f + __expf(-g[i])) * u[i]);
                    __syncwarp();
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int idx = r * 32 + lane, row = idx >> 2, piece = idx & 3;
                        const int c = c0 + row;
                        const long long grow = (long long)ti.tok0 + c;
                        if (c < ti.valid && grow < a.rows_cap)
                            *reinterpret_cast<uint4*>(out + grow * a.ldo + unit0 + piece * 8) =
                                *reinterpret_cast<const uint4*>(stg + row * 32 + piece * 8);
                    }
                };
                // e4m3: the tile's token-row scales in this warp's staging box (bytes
                // 3072-4095, untouched by the exchange and the bf16 rows), read back
                // as broadcast vectors instead of one shuffle per column
                float* scs = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(mine) + 3072);
                if constexpr (FP8) {
#pragma unroll
                    for (int c = 0; c < 8 / CSTEP; ++c) scs[c * 32 + lane] = slp[c];
                    __syncwarp();
                }
                tmem_chunks(tacc, nch, [&](const uint32_t (&v)[32], int ch) {
                    team_sync(team);                      // the partner has read the previous chunk
                    float vv[32];                         // (e4m3: acc * s_weight_row * s_token_row)
                    if constexpr (FP8) {
                        const float4* sc4 = reinterpret_cast<const float4*>(scs + (ch - half) / CSTEP * 32);
#pragma unroll
                        for (int i4 = 0; i4 < 8; ++i4) {
                            const float4 sc = sc4[i4];
                            vv[4 * i4 + 0] = __uint_as_float(v[4 * i4 + 0]) * s_lane * sc.x;
                            vv[4 * i4 + 1] = __uint_as_float(v[4 * i4 + 1]) * s_lane * sc.y;
                            vv[4 * i4 + 2] = __uint_as_float(v[4 * i4 + 2]) * s_lane * sc.z;
                            vv[4 * i4 + 3] = __uint_as_float(v[4 * i4 + 3]) * s_lane * sc.w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) vv[i] = __uint_as_float(v[i]);
                    }
                    float g[16], u[16];
                    if (gate_warp) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) mine[i * 32 + lane] = vv[16 + i];
                        team_sync(team);
#pragma unroll
                        for (int i = 0; i < 16; ++i) { g[i] = vv[i]; u[i] = theirs[i * 32 + lane]; }
                        finish(g, u, ch * 32);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) mine[i * 32 + lane] = vv[i];
                        team_sync(team);
#pragma unroll
                        for (int i = 0; i < 16; ++i) { g[i] = theirs[i * 32 + lane]; u[i] = vv[16 + i]; }
                        finish(g, u, ch * 32 + 16);
                    }
                }, half, CSTEP);
                if constexpr (ZERO_ACC) {
                    // this tile's share of zeroing its tokens' combine accumulator rows:
                    // 16-byte units [m U / ntm, (m + 1) U / ntm) of each row, so the
                    // ntm weight blocks of a token tile clear its rows between them
                    const int U = a.acc_d / 4;
                    const int v0 = (int)((long long)ti.m * U / ntm), v1 = (int)((long long)(ti.m + 1) * U / ntm);
                    // (with eight warps, each half of them clears half of the units)
                    const int u0 = v0 + (v1 - v0) * half / CSTEP, u1 = v0 + (v1 - v0) * (half + 1) / CSTEP;
                    const int c = (int)rank * 128 + (ew & 3) * 32 + lane;
                    if (c < ti.valid) {
                        const int t = a.rows[ti.tok0 + c];
                        if (t >= 0 && t < a.rows_T) {
                            float4* row = reinterpret_cast<float4*>(a.acc + (long long)t * a.acc_d);
                            for (int u = u0; u < u1; ++u) row[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader + 8 * acc);
            if (++acc == 2) { acc = 0; aph ^= 1; }
        }
    }

    tc_fence_before();
    cluster_sync_all();          // all MMAs done and all TMEM reads issued in both CTAs
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 [rows, K] row-major, box {64 (K), box_rows}, 128-byte swizzle; or
// (e4m3) bytes [rows, K], box {128 (K), box_rows}: 128-byte box rows either way.
bool make_map(CUtensorMap* m, const void* base, long long rows, int K, int box_rows = 128, bool e4m3 = false)
{
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    if (rows <= 0 || base == nullptr) {   // unused operand: point at something valid
        rows = 128;
    }
    const int esz = e4m3 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * esz};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output [rows, N] (row stride ldo elements) as boxes of 32 rows x 128 bytes,
// 128-byte swizzle, for the TMA-store epilogues.
bool make_out_map(CUtensorMap* m, void* base, long long rows, int N, long long ldo, bool f32)
{
    EncodeTiledFn enc = get_encode();
    if (!enc || !base || rows <= 0) return false;
    const int elt = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ldo * elt};
    cuuint32_t box[2] = {(cuuint32_t)(128 / elt), 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int EPI>
moe_status launch_epi(const GemmProblem& p, cudaStream_t st)
{
    CUtensorMap mA, m0, m1, m2, m3, mo;
    const void* b1 = p.B1 ? p.B1 : p.B0;
    const void* b2 = p.B2 ? p.B2 : p.B0;
    const void* b3 = p.B3 ? p.B3 : (p.B2 ? p.B2 : b1);
    const long long r23 = p.B2 ? p.b23_rows : p.b01_rows;
    const int kb = p.b_kmod > 0 ? p.b_kmod : p.K;   // B's own K extent
    // token-column form: weight rows are the MMA's M side (SwiGLU stages 64
    // gate + 64 up rows per CTA, so its weight boxes are 64 rows high)
    // (SwiGLU from K = MOE_TN_SWIGLU_MIN_K: its epilogue swaps halves between
    // warps, which a short mainloop does not hide; measured on B200, K = 1024
    // shared-branch gate/up 72 us row-tiled vs 84 us in this form)
    // (its epilogue writes 16-byte pieces of output rows: row stride and base aligned)
    // (the fused and e4m3 forms exist only in the token-column form, for any K)
    const bool tn = MOE_GEMM_TN && (p.pair || p.tn_any || p.fuse) && p.b_kmod == 0 && p.ldo % 8 == 0 &&
                    p.n_groups <= TN_MAX_GROUPS &&
                    reinterpret_cast<uintptr_t>(p.out) % 16 == 0 &&
                    ((EPI == EPI_SWIGLU && p.N % 128 == 0 && (p.K >= MOE_TN_SWIGLU_MIN_K || p.fuse || p.fp8)) ||
                     (EPI == EPI_F32 && p.N % 256 == 0));
    // fuse: 1 = gathered B rows + zeroing, 3 = zeroing (B from x_sorted) -- SwiGLU; 2 = scatter-add -- fp32
    const bool swiglu_fuse = p.fuse == 1 || p.fuse == 3;
    if (p.fp8 && (!tn || p.fuse || p.K % 128 != 0 || !p.sb || !p.sa0 || (EPI == EPI_SWIGLU && !p.sa1) ||
                  (p.n_first < p.n_groups && (!p.sa2 || (EPI == EPI_SWIGLU && !p.sa3)))))
        return MOE_ERR_UNSUPPORTED;
    if (p.fuse && (!tn || swiglu_fuse != (EPI == EPI_SWIGLU) || (p.fuse == 2) != (EPI == EPI_F32) ||
                   !p.rows || !p.acc || p.acc_d % 256 != 0 || p.rows_T <= 0 ||
                   (p.fuse == 1 && p.K % (BK * P_KH) != 0) || (p.fuse == 2 && (!p.idx || !p.gate || p.k <= 0)) ||
                   reinterpret_cast<uintptr_t>(p.acc) % 16 != 0))
        return MOE_ERR_UNSUPPORTED;
    const int wbox = (tn && EPI == EPI_SWIGLU) ? 64 : 128;
    // gathered rows: x itself, one-row boxes (tile::gather4 loads)
    const bool f8 = p.fp8 != 0;
    const bool mapA_ok = p.fuse == 1 ? make_map(&mA, p.A, p.rows_T, p.K, 1)
                                     : make_map(&mA, p.A, p.a_rows, p.K, 128, f8);
    if (!mapA_ok || !make_map(&m0, p.B0, p.b01_rows, kb, wbox, f8) ||
        !make_map(&m1, b1, p.b01_rows, kb, wbox, f8) || !make_map(&m2, b2, r23, kb, wbox, f8) ||
        !make_map(&m3, b3, r23, kb, wbox, f8))
        return MOE_ERR_CUDA;
    if (EPI == EPI_PK_SPLIT) mo = mA;   // direct stores; the map is unused
    else if (!make_out_map(&mo, p.out, std::min<long long>(p.rows_cap, 1ll << 31), p.N, p.ldo, EPI == EPI_F32))
        return MOE_ERR_CUDA;
    DevArgs a;
    a.offsets = p.offsets;
    a.n_groups = p.n_groups;
    a.n_first = p.n_first;
    a.group_rows = p.group_rows;
    a.N = p.N;
    a.K = p.K;
    a.b_kmod = p.b_kmod;
    a.out = p.out;
    a.ldo = p.ldo;
    a.rows_cap = p.rows_cap;
    a.pk_T = p.pk_T;
    a.pk_dq = p.pk_dq;
    a.rows = p.rows;
    a.rows_T = p.rows_T;
    a.acc = p.acc;
    a.acc_d = p.acc_d;
    a.idx = p.idx;
    a.gate = p.gate;
    a.k = p.k;
    a.sa0 = p.sa0;
    a.sa1 = p.sa1;
    a.sa2 = p.sa2;
    a.sa3 = p.sa3;
    a.sb = p.sb;
    const int ntn = (EPI == EPI_SWIGLU) ? cdiv(p.N, 128) : cdiv(p.N, 256);
    const long long rows = std::min<long long>(p.rows_cap, 1ll << 30);
    if constexpr (EPI == EPI_SWIGLU || EPI == EPI_F32) {
        if (tn) {
            // a group of c rows has at most ceil(c / 256) token tiles
            const long long tiles_ub = (long long)(cdiv((int)rows, P_BM) + p.n_groups) * ntn;
            const int clusters = (int)std::max<long long>(1, std::min<long long>(tiles_ub, num_sms() / 2));
            auto go = [&](auto kernel) {
                cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kernel), tn_smem_bytes<EPI>());
                if (e != cudaSuccess) return cuda_status(e);
                kernel<<<2 * clusters, tn_threads<EPI>(), tn_smem_bytes<EPI>(), st>>>(mA, m0, m1, m2, m3, a);
                count_launch();
                return cuda_status(cudaGetLastError());
            };
            if (p.fp8) return go(grouped_gemm_tn_kernel<EPI, TN_PLAIN, true>);
            if constexpr (EPI == EPI_SWIGLU) {
                if (p.fuse == 1) return go(grouped_gemm_tn_kernel<EPI, TN_GATHER | TN_ZERO_ACC>);
                if (p.fuse == 3) return go(grouped_gemm_tn_kernel<EPI, TN_ZERO_ACC>);
            } else {
                if (p.fuse == 2) return go(grouped_gemm_tn_kernel<EPI, TN_SCATTER_ADD>);
            }
            return go(grouped_gemm_tn_kernel<EPI, TN_PLAIN>);
        }
    } else if (p.fuse || p.fp8) {
        return MOE_ERR_UNSUPPORTED;
    }
    if (p.pair) {
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(grouped_gemm_pair_kernel<EPI>), P_SMEM_BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        const long long tiles_ub = (long long)(cdiv((int)rows, P_BM) + p.n_groups) * ntn;
        const int clusters = (int)std::max<long long>(1, std::min<long long>(tiles_ub, num_sms() / 2));
        grouped_gemm_pair_kernel<EPI><<<2 * clusters, NTHREADS, P_SMEM_BYTES, st>>>(mA, m0, m1, m2, m3, mo, a);
    } else {
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(grouped_gemm_kernel<EPI>), SMEM_BYTES);
        if (e != cudaSuccess) return cuda_status(e);
        const long long tiles_ub = (long long)(cdiv((int)rows, BM) + p.n_groups) * ntn;
        const int grid = (int)std::max<long long>(1, std::min<long long>(tiles_ub, num_sms()));
        grouped_gemm_kernel<EPI><<<grid, NTHREADS, SMEM_BYTES, st>>>(mA, m0, m1, m2, m3, mo, a);
    }
    count_launch();
    return cuda_status(cudaGetLastError());
}

}  // namespace

moe_status launch_grouped_gemm(const GemmProblem& p, cudaStream_t st)
{
    if (p.n_groups <= 0 || p.n_groups > kMaxGemmGroups || p.K <= 0 || p.K % 8 != 0 || p.N <= 0 ||
        p.N % 32 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (p.epi == EPI_SWIGLU && p.N % 128 != 0) return MOE_ERR_UNSUPPORTED;
    switch (p.epi) {
        case EPI_SWIGLU: return launch_epi<EPI_SWIGLU>(p, st);
        case EPI_BF16: return launch_epi<EPI_BF16>(p, st);
        case EPI_F32: return launch_epi<EPI_F32>(p, st);
        case EPI_PK_SPLIT: return launch_epi<EPI_PK_SPLIT>(p, st);
        default: return MOE_ERR_INVALID_ARG;
    }
}

}  // namespace moe
