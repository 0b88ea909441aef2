// moe_api.cu -- the C ABI: argument checks, workspace layout, and the order
// of kernel launches for each entry point.  Everything here runs on the
// host; every step of the layer runs in the kernels of the other files.

#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {

__device__ int g_status = 0;
thread_local int t_launches = 0;

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

cudaError_t ensure_smem_attr(const void* func, int bytes)
{
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, int> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    int& have = done[{func, dev}];
    if (have >= bytes) return cudaSuccess;
    if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) == cudaSuccess)
        have = bytes;
    return e;
}

int num_sms()
{
    static std::atomic<int> cache[64];         // per device; 0 = not looked up yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) dev = 0;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {

inline size_t al(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int elt(const moe_layer_desc* d) { return d->dtype == MOE_F32 ? 4 : 2; }
inline int n_router_rows(const moe_layer_desc* d) { return d->n_ffn + d->n_zero + d->n_copy + d->n_const; }

moe_status check_desc(const moe_layer_desc* d)
{
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->d_model <= 0 || d->top_k <= 0) return MOE_ERR_INVALID_ARG;
    if (d->dtype != MOE_F32 && d->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (d->out_f32 != 0 && d->out_f32 != 1) return MOE_ERR_INVALID_ARG;
    if (d->expert_fp8 != 0 && d->expert_fp8 != 1) return MOE_ERR_INVALID_ARG;
    if (d->expert_fp8 && (d->kind != MOE_EXPERT_SWIGLU || d->dtype != MOE_BF16 || d->d_model % 256 != 0 ||
                          (d->n_ffn + d->n_shared > 0 && d->hidden % 128 != 0)))
        return MOE_ERR_UNSUPPORTED;
    if (d->kind == MOE_EXPERT_SWIGLU) {
        if (d->n_ffn < 0 || d->n_shared < 0 || d->n_zero < 0 || d->n_copy < 0 || d->n_const < 0)
            return MOE_ERR_INVALID_ARG;
        const int E = n_router_rows(d);
        if (E <= 0 || d->top_k > E) return MOE_ERR_INVALID_ARG;
        if (d->n_ffn > 0 && d->hidden <= 0) return MOE_ERR_INVALID_ARG;
        if (d->n_shared > 0 && d->hidden_shared != d->hidden) return MOE_ERR_UNSUPPORTED;
        if (d->top_k > 32 || E + 2 * d->n_const > 256 || d->n_ffn > 1024) return MOE_ERR_UNSUPPORTED;
        if (d->n_ffn + d->n_shared > kMaxGemmGroups) return MOE_ERR_UNSUPPORTED;
        if (d->pk_rows || d->pk_cols || d->pk_topk_half || d->d_query) return MOE_ERR_INVALID_ARG;
        if (d->dtype == MOE_BF16) {
            if (d->d_model % 64 != 0 || (d->n_ffn + d->n_shared > 0 && d->hidden % 128 != 0))
                return MOE_ERR_UNSUPPORTED;
        } else {
            if (d->d_model % 8 != 0 || (d->hidden > 0 && d->hidden % 4 != 0)) return MOE_ERR_UNSUPPORTED;
        }
        const long long cap = (long long)d->T * d->top_k + (long long)d->n_shared * d->T;
        if (cap >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
        return MOE_OK;
    }
    if (d->kind == MOE_EXPERT_ATOMIC_GELU) {
        if (d->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
        if (d->n_ffn || d->n_zero || d->n_copy || d->n_const || d->hidden) return MOE_ERR_INVALID_ARG;
        // one shared dense SwiGLU branch beside the atomic experts (the full OmniMoE layer)
        if (d->n_shared < 0 || d->n_shared > 1 || (d->n_shared == 0 && d->hidden_shared != 0))
            return MOE_ERR_INVALID_ARG;
        if (d->n_shared == 1 && (d->hidden_shared <= 0 || d->hidden_shared % 128 != 0)) return MOE_ERR_UNSUPPORTED;
        if (d->pk_rows <= 0 || d->pk_cols <= 0 || d->pk_topk_half <= 0 || d->d_query <= 0)
            return MOE_ERR_INVALID_ARG;
        if (d->pk_topk_half > d->pk_rows || d->pk_topk_half > d->pk_cols) return MOE_ERR_INVALID_ARG;
        if (d->top_k > d->pk_topk_half * d->pk_topk_half) return MOE_ERR_INVALID_ARG;
        if (d->pk_rows != d->pk_cols || d->pk_rows % 32 != 0 || d->pk_rows > 1024) return MOE_ERR_UNSUPPORTED;
        if (d->pk_topk_half > 32 || d->top_k > 128) return MOE_ERR_UNSUPPORTED;
        if (d->d_query % 64 != 0) return MOE_ERR_UNSUPPORTED;
        const int nv = d->d_model / 256;
        if (d->d_model % 256 != 0 || !(nv == 1 || nv == 2 || nv == 4 || nv == 8)) return MOE_ERR_UNSUPPORTED;
        if ((long long)d->pk_rows * d->pk_cols >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
        if ((long long)d->T * d->top_k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
        return MOE_OK;
    }
    return MOE_ERR_INVALID_ARG;
}

// -------------------------------------------------------------- workspace

struct Scratch {   // byte sizes of each call's scratch
    size_t route, permute, ffn;
};

Scratch scratch_sizes(const moe_layer_desc* d)
{
    Scratch s{0, 0, 0};
    const long long cap = moe_row_capacity(d);
    if (d->kind == MOE_EXPERT_SWIGLU) {
        // the counts of every 256-token chunk and expert, then the grid-barrier counter
        s.permute = al((size_t)permute_blocks(d->T) * std::max(d->n_ffn, 1) * 4) + 256;
        s.ffn = (d->n_ffn + d->n_shared > 0) ? al((size_t)cap * d->hidden * elt(d)) : 0;
        if (d->expert_fp8 && s.ffn)   // h (bf16), then its e4m3 codes and row scales
            s.ffn += al((size_t)cap * d->hidden) + al((size_t)cap * 4);
    } else {
        const size_t half = d->d_query / 2;
        s.route = al((size_t)2 * d->T * 3 * half * 2) + al((size_t)(d->pk_rows + d->pk_cols) * 3 * half * 2) +
                  al((size_t)2 * d->T * d->pk_rows * 4);
        const size_t N = (size_t)d->pk_rows * d->pk_cols;
        s.permute = al(N * 4) + al((size_t)atomic_scan_blocks((int)N) * 4);
        s.ffn = 2 * al((size_t)d->T * d->top_k * 4) + (d->n_shared ? al((size_t)d->T * d->hidden_shared * 2) : 0);
    }
    return s;
}

size_t scratch_max(const moe_layer_desc* d)
{
    const Scratch s = scratch_sizes(d);
    return std::max(std::max(s.route, s.permute), std::max(s.ffn, (size_t)256));
}

// moe_layer_forward's expert step: the two-pass one (gather copy, GEMMs, combine
// kernel).  The fused step was measured on B200 alongside it, interleaved, and
// is slower on the Mixtral-shaped and MoE++ layers (2.203 vs 2.158 ms and 1.398
// vs 1.377 ms): zeroing the accumulator in the gate/up epilogue costs ~40 us
// and the atomic epilogue ~15 us more than plain stores, against the ~15-20 us
// the finish kernel saves over the combine.  1 makes the layer take it.
#ifndef MOE_FUSED_LAYER
#define MOE_FUSED_LAYER 0
#endif

// The fused expert step (gather in the gate/up GEMM's loads, combine in the
// down GEMM's epilogue): token-column GEMM forms, and at most two FFN
// contributions per token so that their fp32 sum does not depend on the
// order the atomics land in.
bool fused_eligible(const moe_layer_desc* d)
{
    return d->kind == MOE_EXPERT_SWIGLU && d->dtype == MOE_BF16 && !d->expert_fp8 && d->n_ffn > 0 && d->n_shared == 0 &&
           d->top_k <= 2 && d->d_model % 256 == 0 && d->hidden % 128 == 0;
}

struct FusedScratch {
    size_t h, acc, total;     // hidden activation [cap, H] bf16, accumulator [T, d] fp32
};

FusedScratch fused_scratch(const moe_layer_desc* d)
{
    FusedScratch f;
    f.h = al((size_t)moe_row_capacity(d) * d->hidden * 2);
    f.acc = al((size_t)d->T * d->d_model * 4);
    f.total = std::max(f.h + f.acc, (size_t)256);
    return f;
}

struct LayerBufs {
    int32_t* idx;
    float* gate;
    float* cmix;
    int32_t* offsets;
    int32_t* row_of;
    int32_t* token_of;
    void* xs;
    void* ys;
    void* scratch;
    size_t scratch_bytes;
    size_t total;
};

LayerBufs layer_layout(const moe_layer_desc* d, void* base)
{
    LayerBufs b;
    char* p = static_cast<char*>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) { char* r = p ? p + o : nullptr; o += al(bytes); return r; };
    const long long Tk = (long long)d->T * d->top_k;
    const long long cap = moe_row_capacity(d);
    b.idx = reinterpret_cast<int32_t*>(take(Tk * 4));
    b.gate = reinterpret_cast<float*>(take(Tk * 4));
    b.cmix = reinterpret_cast<float*>(take((size_t)d->T * std::max(d->n_const, 0) * 2 * 4));
    b.offsets = reinterpret_cast<int32_t*>(take((moe_num_groups(d) + 1) * 4));
    b.row_of = reinterpret_cast<int32_t*>(take(Tk * 4));
    b.token_of = reinterpret_cast<int32_t*>(take(cap * 4));
    if (d->kind == MOE_EXPERT_SWIGLU && MOE_FUSED_LAYER && fused_eligible(d)) {
        b.xs = take((size_t)cap * d->d_model * elt(d));
        b.ys = nullptr;   // the fused step combines into its own accumulator
    } else if (d->kind == MOE_EXPERT_SWIGLU) {
        // (FP8 experts: the rows' e4m3 codes, then their fp32 scales)
        b.xs = take(d->expert_fp8 ? al((size_t)cap * d->d_model) + (size_t)cap * 4 : (size_t)cap * d->d_model * elt(d));
        b.ys = take((size_t)cap * d->d_model * 4);
    } else {
        b.xs = nullptr;
        b.ys = take(al((size_t)Tk * 4) + (size_t)d->n_shared * d->T * d->d_model * 4);   // c, then the shared rows
    }
    b.scratch_bytes = scratch_max(d);
    if (d->kind == MOE_EXPERT_SWIGLU && MOE_FUSED_LAYER && fused_eligible(d))
        b.scratch_bytes = std::max(b.scratch_bytes, fused_scratch(d).total);
    b.scratch = take(b.scratch_bytes);
    b.total = o;
    return b;
}

// --------------------------------------------------------- implementations

moe_status route_impl(const moe_layer_desc* d, const moe_layer_weights* w, const void* x,
                      const float* prev, float* logits_out, int32_t* idx, float* gate, float* cmix,
                      void* ws, size_t ws_bytes, cudaStream_t st)
{
    if (d->T == 0) return MOE_OK;
    if (d->kind == MOE_EXPERT_SWIGLU) {
        if (!w->w_router || !aligned16(w->w_router) || !aligned16(x)) return MOE_ERR_INVALID_ARG;
        if (d->n_const > 0 && (!cmix || !w->w_const_mix || !aligned16(w->w_const_mix)))
            return MOE_ERR_INVALID_ARG;
        RouterArgs a;
        a.x = x;
        a.w_router = w->w_router;
        a.w_const_mix = w->w_const_mix;
        a.bias = w->router_bias;
        a.prev = prev;
        a.logits_out = logits_out;
        a.idx = idx;
        a.gate = gate;
        a.const_mix = cmix;
        a.T = d->T;
        a.d = d->d_model;
        a.E_r = n_router_rows(d);
        a.n_const = d->n_const;
        a.k = d->top_k;
        return launch_router(d->dtype, a, st);
    }
    // atomic: q = W_q x split into bf16 parts -> sub-key scores -> selection
    if (!w->w_query || !w->subkeys_row || !w->subkeys_col) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->w_query) || !aligned16(w->subkeys_row) || !aligned16(w->subkeys_col) || !aligned16(x))
        return MOE_ERR_INVALID_ARG;
    const Scratch sc = scratch_sizes(d);
    if (!ws || ws_bytes < sc.route || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    const int half = d->d_query / 2;
    char* p = static_cast<char*>(ws);
    void* a3 = p;
    p += al((size_t)2 * d->T * 3 * half * 2);
    void* w3 = p;
    p += al((size_t)(d->pk_rows + d->pk_cols) * 3 * half * 2);
    float* scores = reinterpret_cast<float*>(p);
    // The score GEMM's B operand is [K|K|K] along k (one copy per bf16 part
    // of q).  When a copy spans whole 64-wide k blocks the GEMM reads the
    // sub-keys directly with k taken mod half; otherwise it reads a tripled
    // copy built here.
    const bool kmod = half % 64 == 0;
    moe_status s = MOE_OK;
    if (!kmod && (s = launch_pk_prep_keys(w->subkeys_row, w->subkeys_col, w3, d->pk_rows, d->pk_cols, half, st)) !=
                     MOE_OK)
        return s;
    GemmProblem q{};
    q.epi = EPI_PK_SPLIT;
    q.A = x;
    q.a_rows = d->T;
    q.K = d->d_model;
    q.B0 = w->w_query;
    q.b01_rows = d->d_query;
    q.offsets = nullptr;
    q.n_groups = 1;
    q.n_first = 1;
    q.group_rows = d->T;
    q.N = d->d_query;
    q.out = a3;
    q.ldo = 3 * half;
    q.rows_cap = d->T;
    q.pk_T = d->T;
    q.pk_dq = d->d_query;
    q.pair = d->T >= 512 ? 1 : 0;
    if ((s = launch_grouped_gemm(q, st)) != MOE_OK) return s;
    GemmProblem g{};
    g.epi = EPI_F32;
    g.A = a3;
    g.a_rows = 2ll * d->T;
    g.K = 3 * half;
    if (kmod) {                 // group 0: row sub-keys, group 1: column sub-keys
        g.B0 = w->subkeys_row;
        g.b01_rows = d->pk_rows;
        g.B2 = w->subkeys_col;
        g.b23_rows = d->pk_cols;
        g.n_first = 1;
        g.b_kmod = half;
    } else {
        g.B0 = w3;
        g.b01_rows = d->pk_rows + d->pk_cols;
        g.n_first = 2;
    }
    g.offsets = nullptr;
    g.n_groups = 2;
    g.group_rows = d->T;
    g.N = d->pk_rows;
    g.out = scores;
    g.ldo = d->pk_rows;
    g.rows_cap = 2ll * d->T;
    g.pair = d->T >= 512 ? 1 : 0;
    if ((s = launch_grouped_gemm(g, st)) != MOE_OK) return s;
    PkSelectArgs ps;
    ps.s_row = scores;
    ps.s_col = scores + (size_t)d->T * d->pk_rows;
    ps.logits_out = logits_out;
    ps.idx = idx;
    ps.gate = gate;
    ps.T = d->T;
    ps.rows = d->pk_rows;
    ps.cols = d->pk_cols;
    ps.kh = d->pk_topk_half;
    ps.K = d->top_k;
    return launch_pk_select(ps, st);
}

moe_status permute_impl(const moe_layer_desc* d, const int32_t* idx, const void* x, int32_t* offsets,
                        int32_t* row_of, int32_t* token_of, void* xs, void* ws, size_t ws_bytes,
                        cudaStream_t st)
{
    const Scratch sc = scratch_sizes(d);
    if (!ws || ws_bytes < sc.permute || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    PermuteArgs a{};
    a.idx = idx;
    a.x = x;
    a.offsets = offsets;
    a.row_of = row_of;
    a.token_of = token_of;
    a.x_sorted = xs;
    a.T = d->T;
    a.k = d->top_k;
    a.d = d->d_model;
    a.elt_bytes = elt(d);
    if (d->kind == MOE_EXPERT_SWIGLU) {
        if (xs && (!x || !aligned16(x) || !aligned16(xs))) return MOE_ERR_INVALID_ARG;
        if (xs && d->expert_fp8)   // e4m3 codes of the rows, then their scales
            a.xs_scale = reinterpret_cast<float*>(static_cast<char*>(xs) + al((size_t)moe_row_capacity(d) * d->d_model));
        a.ws_counts = static_cast<int32_t*>(ws);
        a.bar = reinterpret_cast<unsigned*>(static_cast<char*>(ws) +
                                            al((size_t)permute_blocks(d->T) * std::max(d->n_ffn, 1) * 4));
        a.n_ffn = d->n_ffn;
        a.n_shared = d->n_shared;
        a.n_ids = n_router_rows(d);
        return launch_permute_swiglu(a, st);
    }
    const size_t N = (size_t)d->pk_rows * d->pk_cols;
    char* p = static_cast<char*>(ws);
    a.ws_counts = reinterpret_cast<int32_t*>(p);
    a.ws_blocksum = reinterpret_cast<int32_t*>(p + al(N * 4));
    a.n_ffn = 0;
    a.n_shared = 0;
    a.n_ids = (int)N;
    a.x_sorted = nullptr;
    return launch_permute_atomic(a, st);
}

// The shared dense SwiGLU branch of the atomic kind: phase 1 h = silu(x Ws_gate^T) * (x Ws_up^T)
// (bf16, after the task metadata in the workspace), phase 2 ys_shared = h Ws_down^T (fp32, after c
// in y_sorted).  One group of all T tokens on the grouped tcgen05 GEMM, A read straight from x.
moe_status atomic_shared_phase(const moe_layer_desc* d, const moe_layer_weights* w, int phase, const void* x,
                               void* ys, void* ws, size_t ws_bytes, cudaStream_t st)
{
    if (d->n_shared == 0 || d->T == 0) return MOE_OK;
    const Scratch sc = scratch_sizes(d);
    if (!ws || ws_bytes < sc.ffn || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (!w->ws_gate || !w->ws_up || !w->ws_down || !ys || !aligned16(ys)) return MOE_ERR_INVALID_ARG;
    const void* ptrs[4] = {w->ws_gate, w->ws_up, w->ws_down, x};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    const size_t Tk4 = al((size_t)d->T * d->top_k * 4);
    void* h = static_cast<char*>(ws) + 2 * Tk4;
    GemmProblem g{};
    g.offsets = nullptr;
    g.n_groups = 1;
    g.n_first = 1;
    g.group_rows = d->T;
    g.rows_cap = d->T;
    g.pair = d->T >= 512 ? 1 : 0;
    if (phase == 1) {
        if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
        g.epi = EPI_SWIGLU;
        g.A = x;
        g.a_rows = d->T;
        g.K = d->d_model;
        g.B0 = w->ws_gate;
        g.B1 = w->ws_up;
        g.b01_rows = d->hidden_shared;
        g.N = d->hidden_shared;
        g.out = h;
        g.ldo = d->hidden_shared;
    } else {
        g.epi = EPI_F32;
        g.A = h;
        g.a_rows = d->T;
        g.K = d->hidden_shared;
        g.B0 = w->ws_down;
        g.b01_rows = d->d_model;
        g.N = d->d_model;
        g.out = static_cast<char*>(ys) + Tk4;
        g.ldo = d->d_model;
    }
    return launch_grouped_gemm(g, st);
}

// The SwiGLU step with FP8 experts.  Phase 1: h = SwiGLU on the e4m3 rows of
// x_sorted (epilogue: acc * weight-row scale * row scale), h rounded to bf16,
// then each h row quantized to e4m3 with its power-of-two scale.  Phase 2:
// y_sorted = (h8 W_down8^T) * weight-row scale * row scale.  Workspace: h
// [cap, H] bf16, h8 [cap, H], s_h [cap].
moe_status ffn_phase_fp8(const moe_layer_desc* d, const moe_layer_weights* w, int phase, const void* xs,
                         const int32_t* offsets, void* ys, void* ws, long long cap, cudaStream_t st)
{
    if ((d->n_ffn && (!w->s_gate || !w->s_up || !w->s_down)) ||
        (d->n_shared && (!w->ss_gate || !w->ss_up || !w->ss_down)))
        return MOE_ERR_INVALID_ARG;
    char* h = static_cast<char*>(ws);
    char* h8 = h + al((size_t)cap * d->hidden * 2);
    float* s_h = reinterpret_cast<float*>(h8 + al((size_t)cap * d->hidden));
    const float* s_x = reinterpret_cast<const float*>(static_cast<const char*>(xs) + al((size_t)cap * d->d_model));
    GemmProblem g{};
    g.offsets = offsets;
    g.n_groups = d->n_ffn + d->n_shared;
    g.n_first = d->n_ffn;
    g.rows_cap = cap;
    g.pair = 1;
    g.tn_any = 1;
    g.fp8 = 1;
    g.a_rows = cap;
    if (phase == 1) {
        g.epi = EPI_SWIGLU;
        g.A = xs;
        g.K = d->d_model;
        g.B0 = d->n_ffn ? w->w_gate : w->ws_gate;
        g.B1 = d->n_ffn ? w->w_up : w->ws_up;
        g.sa0 = d->n_ffn ? w->s_gate : w->ss_gate;
        g.sa1 = d->n_ffn ? w->s_up : w->ss_up;
        g.b01_rows = (long long)std::max(d->n_ffn, 1) * d->hidden;
        g.B2 = w->ws_gate;
        g.B3 = w->ws_up;
        g.sa2 = w->ss_gate;
        g.sa3 = w->ss_up;
        g.b23_rows = (long long)d->n_shared * d->hidden;
        g.N = d->hidden;
        g.sb = s_x;
        g.out = h;
        g.ldo = d->hidden;
        moe_status s = launch_grouped_gemm(g, st);
        if (s != MOE_OK) return s;
        return launch_quant_rows(h, offsets, d->n_ffn + d->n_shared, d->hidden, h8, s_h, cap, st);
    }
    g.epi = EPI_F32;
    g.A = h8;
    g.K = d->hidden;
    g.B0 = d->n_ffn ? w->w_down : w->ws_down;
    g.sa0 = d->n_ffn ? w->s_down : w->ss_down;
    g.b01_rows = (long long)std::max(d->n_ffn, 1) * d->d_model;
    g.B2 = w->ws_down;
    g.sa2 = w->ss_down;
    g.b23_rows = (long long)d->n_shared * d->d_model;
    g.N = d->d_model;
    g.sb = s_h;
    g.out = ys;
    g.ldo = d->d_model;
    return launch_grouped_gemm(g, st);
}

moe_status ffn_phase_impl(const moe_layer_desc* d, const moe_layer_weights* w, int phase, const void* xs,
                          const int32_t* offsets, void* ys, void* ws, size_t ws_bytes, cudaStream_t st)
{
    if (d->n_ffn + d->n_shared == 0) return MOE_OK;
    const Scratch sc = scratch_sizes(d);
    if (!ws || ws_bytes < sc.ffn || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (d->n_ffn > 0 && (!w->w_gate || !w->w_up || !w->w_down)) return MOE_ERR_INVALID_ARG;
    if (d->n_shared > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down)) return MOE_ERR_INVALID_ARG;
    const long long cap = moe_row_capacity(d);
    if (d->dtype == MOE_F32) {
        FfnF32Args a;
        a.xs = static_cast<const float*>(xs);
        a.offsets = offsets;
        a.wg = static_cast<const float*>(w->w_gate);
        a.wu = static_cast<const float*>(w->w_up);
        a.wd = static_cast<const float*>(w->w_down);
        a.sg = static_cast<const float*>(w->ws_gate);
        a.su = static_cast<const float*>(w->ws_up);
        a.sd = static_cast<const float*>(w->ws_down);
        a.h = static_cast<float*>(ws);
        a.ys = static_cast<float*>(ys);
        a.n_groups = d->n_ffn + d->n_shared;
        a.n_first = d->n_ffn;
        a.d = d->d_model;
        a.H = d->hidden;
        a.rows_cap = cap;
        return launch_ffn_f32(a, phase, st);
    }
    const void* ptrs[8] = {xs, ys, w->w_gate, w->w_up, w->w_down, w->ws_gate, w->ws_up, w->ws_down};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (d->expert_fp8) return ffn_phase_fp8(d, w, phase, xs, offsets, ys, ws, cap, st);
    GemmProblem g{};
    g.offsets = offsets;
    g.n_groups = d->n_ffn + d->n_shared;
    g.n_first = d->n_ffn;
    g.rows_cap = cap;
    // 256-row tiles on CTA pairs halve the B traffic per SM; with small groups
    // their padding costs more than that saves, so they need >= 512 rows per
    // group on average (the group sizes are only known on the device).  The
    // token-column pair form pads a group only to a multiple of 16 rows and
    // reads each weight block once per 256 rows of a group (a 128-row tile
    // reads it once per 128), so it runs whatever the group sizes.
    g.pair = (long long)d->T * d->top_k >= 512ll * std::max(d->n_ffn, 1) ? 1 : 0;
    g.tn_any = 1;
    if (phase == 1) {
        g.epi = EPI_SWIGLU;
        g.A = xs;
        g.a_rows = cap;
        g.K = d->d_model;
        g.B0 = d->n_ffn ? w->w_gate : w->ws_gate;
        g.B1 = d->n_ffn ? w->w_up : w->ws_up;
        g.b01_rows = (long long)std::max(d->n_ffn, 1) * d->hidden;
        g.B2 = w->ws_gate;
        g.B3 = w->ws_up;
        g.b23_rows = (long long)d->n_shared * d->hidden;
        g.N = d->hidden;
        g.out = ws;
        g.ldo = d->hidden;
    } else {
        g.epi = EPI_F32;
        g.A = ws;
        g.a_rows = cap;
        g.K = d->hidden;
        g.B0 = d->n_ffn ? w->w_down : w->ws_down;
        g.b01_rows = (long long)std::max(d->n_ffn, 1) * d->d_model;
        g.B2 = w->ws_down;
        g.b23_rows = (long long)d->n_shared * d->d_model;
        g.N = d->d_model;
        g.out = ys;
        g.ldo = d->d_model;
    }
    return launch_grouped_gemm(g, st);
}

moe_status ffn_impl(const moe_layer_desc* d, const moe_layer_weights* w, const void* xs,
                    const int32_t* offsets, const int32_t* token_of, const void* x, const float* gate,
                    void* ys, void* ws, size_t ws_bytes, cudaStream_t st)
{
    if (d->kind == MOE_EXPERT_SWIGLU) {
        moe_status s = ffn_phase_impl(d, w, 1, xs, offsets, ys, ws, ws_bytes, st);
        if (s != MOE_OK) return s;
        return ffn_phase_impl(d, w, 2, xs, offsets, ys, ws, ws_bytes, st);
    }
    if (!w->u || !aligned16(w->u) || !x || !aligned16(x) || !gate || !token_of) return MOE_ERR_INVALID_ARG;
    const Scratch sc = scratch_sizes(d);
    if (!ws || ws_bytes < sc.ffn || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    AtomicArgs a{};
    a.x = x;
    a.task_expert = static_cast<int32_t*>(ws);
    a.task_gate = reinterpret_cast<float*>(static_cast<char*>(ws) + al((size_t)d->T * d->top_k * 4));
    a.u = w->u;
    a.v = w->v;
    a.offsets = offsets;
    a.token_of = token_of;
    a.gate = gate;
    a.c = static_cast<float*>(ys);
    a.T = d->T;
    a.d = d->d_model;
    a.K = d->top_k;
    a.N = d->pk_rows * d->pk_cols;
    moe_status s = launch_atomic_phase_a(a, st);
    if (s != MOE_OK || d->n_shared == 0) return s;
    if ((s = atomic_shared_phase(d, w, 1, x, ys, ws, ws_bytes, st)) != MOE_OK) return s;
    return atomic_shared_phase(d, w, 2, x, ys, ws, ws_bytes, st);
}

moe_status combine_impl(const moe_layer_desc* d, const moe_layer_weights* w, const void* ys,
                        const int32_t* offsets, const int32_t* row_of, const int32_t* idx,
                        const float* gate, const float* cmix, const void* x, void* y, cudaStream_t st)
{
    if (d->T == 0) return MOE_OK;
    if (!y || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    if (d->kind == MOE_EXPERT_ATOMIC_GELU) {
        if (!w->v || !aligned16(w->v)) return MOE_ERR_INVALID_ARG;
        AtomicArgs a{};
        a.v = w->v;
        a.idx = idx;
        a.c = const_cast<float*>(static_cast<const float*>(ys));
        a.shared_out = d->n_shared ? reinterpret_cast<const float*>(static_cast<const char*>(ys) +
                                                                     al((size_t)d->T * d->top_k * 4))
                                   : nullptr;
        a.y = y;
        a.T = d->T;
        a.d = d->d_model;
        a.K = d->top_k;
        a.N = d->pk_rows * d->pk_cols;
        a.out_f32 = d->out_f32;
        return launch_atomic_phase_b(a, st);
    }
    if ((d->n_copy + d->n_const > 0) && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    if (d->n_const > 0 && (!cmix || !w->const_vec || !aligned16(w->const_vec))) return MOE_ERR_INVALID_ARG;
    if ((d->n_ffn + d->n_shared > 0) && (!ys || !aligned16(ys))) return MOE_ERR_INVALID_ARG;
    CombineArgs a{};
    a.ys = ys;
    a.offsets = offsets;
    a.row_of = row_of;
    a.idx = idx;
    a.gate = gate;
    a.const_mix = cmix;
    a.const_vec = w->const_vec;
    a.x = x;
    a.y = y;
    a.T = d->T;
    a.d = d->d_model;
    a.k = d->top_k;
    a.n_ffn = d->n_ffn;
    a.n_shared = d->n_shared;
    a.n_zero = d->n_zero;
    a.n_copy = d->n_copy;
    a.n_const = d->n_const;
    a.rows_cap = moe_row_capacity(d);
    a.out_f32 = d->out_f32;
    return launch_combine(d->dtype, a, st);
}

// One phase of the fused expert step (0: all three).
moe_status fused_impl(const moe_layer_desc* d, const moe_layer_weights* w, int phase, const void* x,
                      const void* xs, const int32_t* idx, const float* gate, const float* cmix, const int32_t* offsets,
                      const int32_t* row_of, const int32_t* token_of, void* y, void* ws, size_t ws_bytes,
                      cudaStream_t st)
{
    if (!fused_eligible(d)) return MOE_ERR_UNSUPPORTED;
    if (d->T == 0) return MOE_OK;
    const FusedScratch fs = fused_scratch(d);
    if (!ws || ws_bytes < fs.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    if (!w->w_gate || !w->w_up || !w->w_down || !x || !offsets || !token_of) return MOE_ERR_INVALID_ARG;
    const void* ptrs[4] = {w->w_gate, w->w_up, w->w_down, x};
    for (const void* q : ptrs)
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    void* h = ws;
    float* acc = reinterpret_cast<float*>(static_cast<char*>(ws) + fs.h);
    const long long cap = moe_row_capacity(d);
    moe_status s = MOE_OK;
    if (phase == 0 || phase == 1) {
        // B rows from x_sorted, or (x_sorted NULL) gathered from x by the GEMM's own loads
        if (xs && !aligned16(xs)) return MOE_ERR_INVALID_ARG;
        GemmProblem g{};
        g.epi = EPI_SWIGLU;
        g.A = xs ? xs : x;
        g.a_rows = xs ? cap : d->T;
        g.K = d->d_model;
        g.B0 = w->w_gate;
        g.B1 = w->w_up;
        g.b01_rows = (long long)d->n_ffn * d->hidden;
        g.offsets = offsets;
        g.n_groups = d->n_ffn;
        g.n_first = d->n_ffn;
        g.N = d->hidden;
        g.out = h;
        g.ldo = d->hidden;
        g.rows_cap = cap;
        g.pair = 1;
        g.fuse = xs ? 3 : 1;
        g.rows = token_of;
        g.rows_T = d->T;
        g.acc = acc;
        g.acc_d = d->d_model;
        if ((s = launch_grouped_gemm(g, st)) != MOE_OK) return s;
    }
    if (phase == 0 || phase == 2) {
        if (!idx || !gate) return MOE_ERR_INVALID_ARG;
        GemmProblem g{};
        g.epi = EPI_F32;
        g.A = h;
        g.a_rows = cap;
        g.K = d->hidden;
        g.B0 = w->w_down;
        g.b01_rows = (long long)d->n_ffn * d->d_model;
        g.offsets = offsets;
        g.n_groups = d->n_ffn;
        g.n_first = d->n_ffn;
        g.N = d->d_model;
        g.out = acc;
        g.ldo = d->d_model;
        g.rows_cap = d->T;
        g.pair = 1;
        g.fuse = 2;
        g.rows = token_of;
        g.rows_T = d->T;
        g.acc = acc;
        g.acc_d = d->d_model;
        g.idx = idx;
        g.gate = gate;
        g.k = d->top_k;
        if ((s = launch_grouped_gemm(g, st)) != MOE_OK) return s;
    }
    if (phase == 0 || phase == 3) {
        if (!y || !aligned16(y) || !idx || !gate || !row_of) return MOE_ERR_INVALID_ARG;
        if (d->n_const > 0 && (!cmix || !w->const_vec || !aligned16(w->const_vec))) return MOE_ERR_INVALID_ARG;
        CombineArgs a{};
        a.ys = acc;
        a.offsets = offsets;
        a.row_of = row_of;
        a.idx = idx;
        a.gate = gate;
        a.const_mix = cmix;
        a.const_vec = w->const_vec;
        a.x = x;
        a.y = y;
        a.T = d->T;
        a.d = d->d_model;
        a.k = d->top_k;
        a.n_ffn = d->n_ffn;
        a.n_shared = 0;
        a.n_zero = d->n_zero;
        a.n_copy = d->n_copy;
        a.n_const = d->n_const;
        a.rows_cap = cap;
        a.out_f32 = d->out_f32;
        a.acc_rows = 1;
        if ((s = launch_combine(d->dtype, a, st)) != MOE_OK) return s;
    }
    return MOE_OK;
}

}  // namespace

moe_status validate_desc(const moe_layer_desc* d) { return check_desc(d); }

}  // namespace moe

using namespace moe;

// ----------------------------------------------------- host-to-host layer

namespace {

constexpr int kMaxHostChunks = 8;

struct HostPipe {                       // per device: two copy streams and their events
    // Held while one call enqueues its copies, records and waits: the events
    // are shared, and a wait binds to an event's latest record, so another
    // call's records in between would make this call wait on the wrong work.
    std::mutex call_mu;
    bool ok = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t fork = nullptr;
    cudaEvent_t join_in = nullptr, join_out = nullptr;   // error exits: the copy streams' last work
    cudaEvent_t in_done[kMaxHostChunks], comp_done[kMaxHostChunks], out_done[kMaxHostChunks];
};

HostPipe* host_pipe()
{
    static std::mutex mu;
    static HostPipe pipes[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    HostPipe& p = pipes[dev];
    if (!p.ok) {
        bool good = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&p.fork, cudaEventDisableTiming) == cudaSuccess &&
                    cudaEventCreateWithFlags(&p.join_in, cudaEventDisableTiming) == cudaSuccess &&
                    cudaEventCreateWithFlags(&p.join_out, cudaEventDisableTiming) == cudaSuccess;
        for (int c = 0; good && c < kMaxHostChunks; ++c)
            good = cudaEventCreateWithFlags(&p.in_done[c], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&p.comp_done[c], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&p.out_done[c], cudaEventDisableTiming) == cudaSuccess;
        if (!good) return nullptr;
        p.ok = true;
    }
    return &p;
}

int host_chunks(const moe_layer_desc* d, int chunks)
{
    // About 3.5k tokens a range (host_range_start gives the lengths).  Measured
    // on B200, end-to-end ms by range count: Mixtral-shaped (T 4096) 1 / 2 / 3
    // / 4: 3.29 / 2.97 / 3.05 / 3.28; MoE++ (T 16384) 3 / 4 / 5 / 6: 2.68 /
    // 2.40 / 2.33 / 2.51, with FP8 experts 2.43 / 2.20 / 2.06 / 2.04; atomic
    // (T 8192) 1 / 2 / 3: 1.14 / 0.95-1.11 / 0.95-1.10; long-tail (T 2048) 1 /
    // 2: 0.78 / 0.86.  A range hides the copies of the next, but re-reads the
    // expert weights and pays the fixed routing costs.
    if (chunks <= 0) chunks = d->T >= 4096 ? std::max(2, (d->T + 2048) / 3584) : 1;
    return std::max(1, std::min(std::min(chunks, kMaxHostChunks), std::max(d->T, 1)));
}

struct HostLayout {
    moe_layer_desc dc;                  // one token range (the largest)
    size_t layer_bytes, x_bytes, y_bytes, z_bytes, total;
};

// First token of range c of nch (c = nch: T).  With three or more ranges the
// first and the last are half as long as the others: only the first range's
// host->device copy and the last range's device->host copy are not hidden
// behind computation.
int host_range_start(int T, int nch, int c)
{
    if (nch < 3 || T < 2 * (nch - 1)) return (int)((long long)T * c / nch);   // (every range non-empty)
    const long long W = 2ll * (nch - 1);                  // weights 1, 2, ..., 2, 1
    const long long before = c == 0 ? 0 : (c >= nch ? W : 2ll * c - 1);
    return (int)((long long)T * before / W);
}

HostLayout host_layout(const moe_layer_desc* d, int nch)
{
    HostLayout h;
    h.dc = *d;
    int longest = 1;
    for (int c = 0; c < nch; ++c)
        longest = std::max(longest, host_range_start(d->T, nch, c + 1) - host_range_start(d->T, nch, c));
    h.dc.T = longest;
    h.layer_bytes = al((size_t)moe_layer_workspace_size(&h.dc));
    h.x_bytes = al((size_t)h.dc.T * d->d_model * elt(d));
    h.y_bytes = al((size_t)h.dc.T * d->d_model * (d->out_f32 ? 4 : elt(d)));
    h.z_bytes = d->kind == MOE_EXPERT_SWIGLU ? al((size_t)h.dc.T * n_router_rows(d) * 4) : 0;
    h.total = h.layer_bytes + 2 * (h.x_bytes + h.y_bytes + h.z_bytes);
    return h;
}

}  // namespace

extern "C" {

int64_t moe_num_groups(const moe_layer_desc* d)
{
    if (check_desc(d) != MOE_OK) return -1;
    if (d->kind == MOE_EXPERT_SWIGLU) return d->n_ffn + d->n_shared;
    return (int64_t)d->pk_rows * d->pk_cols;
}

int64_t moe_row_capacity(const moe_layer_desc* d)
{
    if (check_desc(d) != MOE_OK) return -1;
    const int64_t Tk = (int64_t)d->T * d->top_k;
    if (d->kind == MOE_EXPERT_SWIGLU) return Tk + (int64_t)d->n_shared * d->T;
    return Tk;
}

int64_t moe_workspace_size(const moe_layer_desc* d)
{
    if (check_desc(d) != MOE_OK) return -1;
    return (int64_t)scratch_max(d);
}

int64_t moe_layer_workspace_size(const moe_layer_desc* d)
{
    if (check_desc(d) != MOE_OK) return -1;
    return (int64_t)layer_layout(d, nullptr).total;
}

int64_t moe_fused_workspace_size(const moe_layer_desc* d)
{
    if (check_desc(d) != MOE_OK || !fused_eligible(d)) return -1;
    return (int64_t)fused_scratch(d).total;
}

moe_status moe_fused_ffn_combine(const moe_layer_desc* d, const moe_layer_weights* w, int phase, const void* x,
                                 const void* x_sorted, const int32_t* topk_idx, const float* topk_gate,
                                 const float* const_mix, const int32_t* expert_offsets, const int32_t* row_of,
                                 const int32_t* token_of, void* y, void* workspace, size_t ws_bytes,
                                 moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || phase < 0 || phase > 3) return MOE_ERR_INVALID_ARG;
    return fused_impl(d, w, phase, x, x_sorted, topk_idx, topk_gate, const_mix, expert_offsets, row_of, token_of, y,
                      workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

moe_status moe_route(const moe_layer_desc* d, const moe_layer_weights* w, const void* x,
                     const float* prev_logits, float* logits_out, int32_t* topk_idx, float* topk_gate,
                     float* const_mix, void* workspace, size_t ws_bytes, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || (d->T > 0 && (!x || !topk_idx || !topk_gate))) return MOE_ERR_INVALID_ARG;
    return route_impl(d, w, x, prev_logits, logits_out, topk_idx, topk_gate, const_mix, workspace, ws_bytes,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_permute(const moe_layer_desc* d, const int32_t* topk_idx, const void* x,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* token_of, void* x_sorted,
                       void* workspace, size_t ws_bytes, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!expert_offsets || (d->T > 0 && (!topk_idx || !row_of || !token_of))) return MOE_ERR_INVALID_ARG;
    return permute_impl(d, topk_idx, x, expert_offsets, row_of, token_of, x_sorted, workspace, ws_bytes,
                        static_cast<cudaStream_t>(stream));
}

moe_status moe_grouped_ffn(const moe_layer_desc* d, const moe_layer_weights* w, const void* x_sorted,
                           const int32_t* expert_offsets, const int32_t* token_of, const void* x,
                           const float* topk_gate, void* y_sorted, void* workspace, size_t ws_bytes,
                           moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || !expert_offsets || (d->T > 0 && !y_sorted)) return MOE_ERR_INVALID_ARG;
    if (d->kind == MOE_EXPERT_SWIGLU && d->T > 0 && !x_sorted) return MOE_ERR_INVALID_ARG;
    return ffn_impl(d, w, x_sorted, expert_offsets, token_of, x, topk_gate, y_sorted, workspace, ws_bytes,
                    static_cast<cudaStream_t>(stream));
}

moe_status moe_grouped_ffn_phase(const moe_layer_desc* d, const moe_layer_weights* w, int phase,
                                 const void* x_sorted, const int32_t* expert_offsets, void* y_sorted,
                                 void* workspace, size_t ws_bytes, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (phase != 1 && phase != 2) return MOE_ERR_INVALID_ARG;
    if (d->kind == MOE_EXPERT_ATOMIC_GELU) {   // the shared dense branch; x_sorted is x itself
        if (!w || d->n_shared == 0 || (d->T > 0 && (!x_sorted || !y_sorted))) return MOE_ERR_INVALID_ARG;
        return atomic_shared_phase(d, w, phase, x_sorted, y_sorted, workspace, ws_bytes,
                                   static_cast<cudaStream_t>(stream));
    }
    if (!w || !expert_offsets || (d->T > 0 && (!x_sorted || !y_sorted))) return MOE_ERR_INVALID_ARG;
    return ffn_phase_impl(d, w, phase, x_sorted, expert_offsets, y_sorted, workspace, ws_bytes,
                          static_cast<cudaStream_t>(stream));
}

moe_status moe_combine(const moe_layer_desc* d, const moe_layer_weights* w, const void* y_sorted,
                       const int32_t* expert_offsets, const int32_t* row_of, const int32_t* topk_idx,
                       const float* topk_gate, const float* const_mix, const void* x, void* y,
                       moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || (d->T > 0 && (!topk_idx || !topk_gate || !y))) return MOE_ERR_INVALID_ARG;
    if (d->kind == MOE_EXPERT_SWIGLU && d->T > 0 && (!row_of || !expert_offsets)) return MOE_ERR_INVALID_ARG;
    if (d->kind == MOE_EXPERT_ATOMIC_GELU && d->T > 0 && !y_sorted) return MOE_ERR_INVALID_ARG;
    return combine_impl(d, w, y_sorted, expert_offsets, row_of, topk_idx, topk_gate, const_mix, x, y,
                        static_cast<cudaStream_t>(stream));
}

moe_status moe_layer_forward(const moe_layer_desc* d, const moe_layer_weights* w, const void* x,
                             const float* prev_logits, void* y, float* logits_out, void* workspace,
                             size_t ws_bytes, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || (d->T > 0 && (!x || !y))) return MOE_ERR_INVALID_ARG;
    const LayerBufs need = layer_layout(d, nullptr);
    if (!workspace || ws_bytes < need.total || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
    const LayerBufs b = layer_layout(d, workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d->T == 0) return MOE_OK;
    if ((s = route_impl(d, w, x, prev_logits, logits_out, b.idx, b.gate, b.cmix, b.scratch, b.scratch_bytes, st)) != MOE_OK)
        return s;
    if ((s = permute_impl(d, b.idx, x, b.offsets, b.row_of, b.token_of, b.xs, b.scratch, b.scratch_bytes, st)) != MOE_OK)
        return s;
    if (d->kind == MOE_EXPERT_SWIGLU && MOE_FUSED_LAYER && fused_eligible(d))
        return fused_impl(d, w, 0, x, b.xs, b.idx, b.gate, b.cmix, b.offsets, b.row_of, b.token_of, y, b.scratch,
                          b.scratch_bytes, st);
    if ((s = ffn_impl(d, w, b.xs, b.offsets, b.token_of, x, b.gate, b.ys, b.scratch, b.scratch_bytes, st)) != MOE_OK)
        return s;
    return combine_impl(d, w, b.ys, b.offsets, b.row_of, b.idx, b.gate, b.cmix, x, y, st);
}

int64_t moe_layer_host_workspace_size(const moe_layer_desc* d, int chunks)
{
    if (check_desc(d) != MOE_OK) return -1;
    return (int64_t)host_layout(d, host_chunks(d, chunks)).total;
}

moe_status moe_layer_forward_host(const moe_layer_desc* d, const moe_layer_weights* w, const void* x_host,
                                  const float* prev_logits_host, void* y_host, int chunks, void* workspace,
                                  size_t ws_bytes, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = check_desc(d);
    if (s != MOE_OK) return s;
    if (!w || (d->T > 0 && (!x_host || !y_host))) return MOE_ERR_INVALID_ARG;
    if (prev_logits_host && d->kind != MOE_EXPERT_SWIGLU) return MOE_ERR_INVALID_ARG;
    const int nch = host_chunks(d, chunks);
    const HostLayout h = host_layout(d, nch);
    if (!workspace || ws_bytes < h.total || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
    if (d->T == 0) return MOE_OK;
    HostPipe* pp = host_pipe();
    if (!pp) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> call_lock(pp->call_mu);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(workspace);
    void* layer_ws = base;
    char* xb[2] = {base + h.layer_bytes, base + h.layer_bytes + h.x_bytes};
    char* yb[2] = {xb[1] + h.x_bytes, xb[1] + h.x_bytes + h.y_bytes};
    char* zb[2] = {yb[1] + h.y_bytes, yb[1] + h.y_bytes + h.z_bytes};
    const size_t xrow = (size_t)d->d_model * elt(d);
    const size_t yrow = (size_t)d->d_model * (d->out_f32 ? 4 : elt(d));
    const size_t zrow = (size_t)n_router_rows(d) * 4;
    // Everything after the fork runs in `run`; whatever it returns, the copy
    // streams are joined back into `stream` first, so a caller that
    // synchronises `stream` after an error has no copy still in flight into
    // the workspace or the host buffers.
    int launches = 0;
    auto run = [&]() -> moe_status {
#define MOE_CU(call)                                              \
    do {                                                          \
        if ((call) != cudaSuccess) return MOE_ERR_CUDA;           \
    } while (0)
        for (int c = 0; c < nch; ++c) {
            const int t0 = host_range_start(d->T, nch, c);
            const int tc = host_range_start(d->T, nch, c + 1) - t0;
            if (tc <= 0) break;
            const int b = c & 1;
            if (c >= 2) MOE_CU(cudaStreamWaitEvent(pp->in, pp->comp_done[c - 2], 0));   // staging b read
            MOE_CU(cudaMemcpyAsync(xb[b], static_cast<const char*>(x_host) + (size_t)t0 * xrow, (size_t)tc * xrow,
                                   cudaMemcpyHostToDevice, pp->in));
            if (prev_logits_host)
                MOE_CU(cudaMemcpyAsync(zb[b], reinterpret_cast<const char*>(prev_logits_host) + (size_t)t0 * zrow,
                                       (size_t)tc * zrow, cudaMemcpyHostToDevice, pp->in));
            MOE_CU(cudaEventRecord(pp->in_done[c], pp->in));
            MOE_CU(cudaStreamWaitEvent(st, pp->in_done[c], 0));
            if (c >= 2) MOE_CU(cudaStreamWaitEvent(st, pp->out_done[c - 2], 0));     // output b copied out
            moe_layer_desc dcc = h.dc;
            dcc.T = tc;
            const moe_status sl = moe_layer_forward(&dcc, w, xb[b],
                                                    prev_logits_host ? reinterpret_cast<const float*>(zb[b]) : nullptr,
                                                    yb[b], nullptr, layer_ws, h.layer_bytes, stream);
            launches += t_launches;
            if (sl != MOE_OK) return sl;
            MOE_CU(cudaEventRecord(pp->comp_done[c], st));
            MOE_CU(cudaStreamWaitEvent(pp->out, pp->comp_done[c], 0));
            MOE_CU(cudaMemcpyAsync(static_cast<char*>(y_host) + (size_t)t0 * yrow, yb[b], (size_t)tc * yrow,
                                   cudaMemcpyDeviceToHost, pp->out));
            MOE_CU(cudaEventRecord(pp->out_done[c], pp->out));
        }
        return MOE_OK;
#undef MOE_CU
    };
    if (cudaEventRecord(pp->fork, st) != cudaSuccess) return MOE_ERR_CUDA;   // the copy streams join `stream`'s work
    if (cudaStreamWaitEvent(pp->in, pp->fork, 0) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(pp->out, pp->fork, 0) != cudaSuccess) {
        // `in` already waits on the fork: join it back before leaving
        if (cudaEventRecord(pp->join_in, pp->in) == cudaSuccess) cudaStreamWaitEvent(st, pp->join_in, 0);
        return MOE_ERR_CUDA;
    }
    s = run();
    // join both copy streams back into `stream` (on success as on error)
    const bool joined = cudaEventRecord(pp->join_in, pp->in) == cudaSuccess &&
                        cudaStreamWaitEvent(st, pp->join_in, 0) == cudaSuccess &&
                        cudaEventRecord(pp->join_out, pp->out) == cudaSuccess &&
                        cudaStreamWaitEvent(st, pp->join_out, 0) == cudaSuccess;
    if (s != MOE_OK) return s;
    if (!joined) return MOE_ERR_CUDA;
    t_launches = launches;
    return MOE_OK;
}

moe_status moe_get_device_status(moe_status* out, int reset, moe_stream_t stream)
{
    if (!out) return MOE_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int))) != cudaSuccess) return MOE_ERR_CUDA;
    if (reset) {
        const int zero = 0;
        if ((e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int))) != cudaSuccess) return MOE_ERR_CUDA;
    }
    *out = static_cast<moe_status>(v);
    return MOE_OK;
}

const char* moe_status_string(moe_status s)
{
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or option";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE_BOUNDS: return "kernel saw an invalid index";
        case MOE_ERR_TIMEOUT: return "kernel wait timed out";
    }
    return "unknown status";
}

int32_t moe_last_launch_count(void) { return t_launches; }

}  // extern "C"
