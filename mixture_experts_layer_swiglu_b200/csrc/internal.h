// internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Kernel launches enqueued by the current C-ABI call (per host thread).
extern thread_local int t_launches;
inline void count_launch(int n = 1) { t_launches += n; }

moe_status cuda_status(cudaError_t e);
int num_sms();
// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device (the attribute belongs to each device's context), once per device.
cudaError_t ensure_smem_attr(const void* func, int bytes);
moe_status validate_desc(const moe_layer_desc* d);   // the descriptor checks of every entry point

// ------------------------------------------------------------ grouped GEMM
enum EpiKind { EPI_SWIGLU = 0, EPI_BF16 = 1, EPI_F32 = 2, EPI_PK_SPLIT = 3 };

constexpr int kMaxGemmGroups = 1024;

// One grouped GEMM  out[r, :] = epi(A[r, :] . B_g^T)  for rows r of group g.
// A [a_rows, K] bf16 row-major.  B for groups g < n_first: rows
// [g*N, (g+1)*N) of B0 (and of B1 for SwiGLU); for g >= n_first the same rows
// (g - n_first) of B2 (/B3).  SwiGLU: B0/B2 are W_gate, B1/B3 W_up and the
// output h has N columns.  Groups: offsets [n_groups+1] on the device, or
// uniform groups of group_rows rows when offsets == nullptr.
struct GemmProblem {
    int epi;
    const void* A;
    long long a_rows;
    int K;
    const void* B0;
    const void* B1;
    long long b01_rows;
    const void* B2;
    const void* B3;
    long long b23_rows;
    const int32_t* offsets;
    int n_groups;
    int n_first;
    int group_rows;
    int N;
    void* out;
    long long ldo;
    long long rows_cap;   // rows of `out` (stores beyond are dropped)
    int pk_T;             // EPI_PK_SPLIT: tokens
    int pk_dq;            // EPI_PK_SPLIT: query width
    int pair;             // 1: 256-row tiles on CTA pairs (cta_group::2); 0: 128-row tiles per CTA
    int tn_any;           // 1: the token-column pair form may run whatever `pair` says (groups of any size)
    int b_kmod;           // > 0: B has b_kmod columns and is repeated along K (B k = k mod b_kmod)
    // fused permutation / combine (token-column pair form only; else MOE_ERR_UNSUPPORTED):
    //   fuse == 1 (SwiGLU): row r of the grouped operand is row rows[r] of A (A = x [rows_T, K]),
    //             and the tiles zero the rows rows[r] of acc [rows_T, acc_d];
    //   fuse == 3 (SwiGLU): A is x_sorted as usual; the tiles zero the rows rows[r] of acc;
    //   fuse == 2 (fp32):   out row r is added, scaled by the gate of (token rows[r], the
    //             group's expert) from idx / gate [rows_T, k], into acc row rows[r].
    int fuse;
    const int32_t* rows;
    int rows_T;
    float* acc;
    int acc_d;
    const int32_t* idx;
    const float* gate;
    int k;
    // e4m3 operands (token-column pair form only; else MOE_ERR_UNSUPPORTED): A and B hold
    // e4m3 codes, K a multiple of 128; out = acc * sa[weight row] * sb[token row], with
    // sa0 / sa1 the row scales of B0 / B1 and sa2 / sa3 those of B2 / B3.
    int fp8;
    const float* sa0;
    const float* sa1;
    const float* sa2;
    const float* sa3;
    const float* sb;
};

moe_status launch_grouped_gemm(const GemmProblem& p, cudaStream_t st);

// ------------------------------------------------------------ router
struct RouterArgs {
    const void* x;
    const void* w_router;
    const void* w_const_mix;
    const float* bias;
    const float* prev;
    float* logits_out;
    int32_t* idx;
    float* gate;
    float* const_mix;
    int T, d, E_r, n_const, k;
};
moe_status launch_router(int dtype, const RouterArgs& a, cudaStream_t st);

struct PkSelectArgs {
    const float* s_row;   // [T, rows]
    const float* s_col;   // [T, cols]
    float* logits_out;    // [T, rows + cols] nullable
    int32_t* idx;         // [T, K]
    float* gate;          // [T, K]
    int T, rows, cols, kh, K;
};
moe_status launch_pk_select(const PkSelectArgs& a, cudaStream_t st);
moe_status launch_pk_prep_keys(const void* k_row, const void* k_col, void* w3, int rows,
                               int cols, int half, cudaStream_t st);

// ------------------------------------------------------------ permute
struct PermuteArgs {
    const int32_t* idx;
    const void* x;
    int32_t* offsets;
    int32_t* row_of;
    int32_t* token_of;
    void* x_sorted;
    int32_t* ws_counts;   // [n_blocks, n_ffn] (SwiGLU) or [N] (atomic)
    int32_t* ws_blocksum; // atomic scan: [scan blocks]
    int T, k, d, n_ffn, n_shared, n_ids, elt_bytes;
    float* xs_scale;      // non-null: x_sorted gets e4m3 codes of the rows and these their scales
    unsigned* bar;        // SwiGLU: grid-barrier counter of the one-launch form (null: the four kernels)
};
moe_status launch_permute_swiglu(const PermuteArgs& a, cudaStream_t st);
moe_status launch_permute_atomic(const PermuteArgs& a, cudaStream_t st);
int permute_blocks(int T);
int atomic_scan_blocks(int N);

// ------------------------------------------------------------ e4m3 activations
// codes[r] = e4m3(x[token_of[r]] / scale[r]) for r < offsets[n_last] (x bf16 [T, d], d % 256 == 0)
moe_status launch_gather_quant(const int32_t* token_of, const int32_t* offsets, int n_last, const void* x, int d,
                               int T, void* codes, float* scale, long long rows_cap, cudaStream_t st);
// codes[r] = e4m3(h[r] / scale[r]) for r < offsets[n_last] (h bf16 [rows, H])
moe_status launch_quant_rows(const void* h, const int32_t* offsets, int n_last, int H, void* codes, float* scale,
                             long long rows_cap, cudaStream_t st);

// ------------------------------------------------------------ experts
struct FfnF32Args {
    const float* xs;
    const int32_t* offsets;
    const float* wg; const float* wu; const float* wd;      // routed
    const float* sg; const float* su; const float* sd;      // shared
    float* h;
    float* ys;
    int n_groups, n_first, d, H;
    long long rows_cap;
};
moe_status launch_ffn_f32(const FfnF32Args& a, int phase, cudaStream_t st);

struct AtomicArgs {
    const void* x;        // [T, d] bf16
    const void* u;        // [N, d]
    const void* v;        // [N, d]
    const int32_t* offsets;
    const int32_t* token_of;   // task -> slot id
    int32_t* task_expert;      // task -> expert (scratch, written by phase A's first kernel)
    float* task_gate;          // task -> gate of its slot (scratch, same kernel)
    const int32_t* idx;        // [T, K]
    const float* gate;         // [T, K]
    float* c;                  // [T*K]
    const float* shared_out;   // [T, d] fp32 output of the shared dense branch, nullable
    void* y;                   // [T, d] bf16, or fp32 if out_f32
    int T, d, K, N;
    int out_f32;
};
moe_status launch_atomic_phase_a(const AtomicArgs& a, cudaStream_t st);
moe_status launch_atomic_phase_b(const AtomicArgs& a, cudaStream_t st);

// ------------------------------------------------------------ combine
struct CombineArgs {
    const void* ys;
    const int32_t* offsets;
    const int32_t* row_of;
    const int32_t* idx;
    const float* gate;
    const float* const_mix;
    const void* const_vec;
    const void* x;
    void* y;
    int T, d, k, n_ffn, n_shared, n_zero, n_copy, n_const;
    long long rows_cap;
    int out_f32;               // y fp32 whatever the input dtype
    int acc_rows;              // 1: ys is [T, d] fp32 per-token sums of the FFN slots' gated outputs
                               //    (the fused combine); only the zero-computation slots are added here
};
moe_status launch_combine(int dtype, const CombineArgs& a, cudaStream_t st);

}  // namespace moe
