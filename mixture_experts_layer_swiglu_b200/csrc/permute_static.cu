// permute_static.cu -- moe_permute for callers that cannot allocate device
// memory.
//
// moe_permute needs a small scratch buffer (the per-block expert counts of
// the histogram / scan / scatter kernels) that the caller normally passes as
// `workspace`.  Some callers have no way to provide it: a plugin running
// inside a host framework that owns all device memory and gives the plugin
// no allocator, or a service whose device memory budget is fixed and fully
// committed when it starts.  moe_permute_static runs the same kernels with
// that scratch in a fixed-size array in this library's own device memory
// instead, so the call needs no allocation by anyone.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (kStaticPermuteInts * 4 bytes = 256 KiB) until the process
// exits.  In host code its name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress, with the device current, on
// the first call made in each CUDA context (a device's primary context, and
// again after cudaDeviceReset replaces it), and passed to the kernels.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kStaticPermuteInts = 65536;   // 256 KiB of per-block counts
constexpr int kMaxDevices = 64;

static __device__ __align__(256) int32_t g_permute_scratch[kStaticPermuteInts];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

struct ScratchAddr {
    CUcontext ctx;     // the context the address belongs to
    int32_t* ptr;
};

std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices] = {};

// Device address of g_permute_scratch in the current device's current context.
// A cached address is reused only while that context is still the current
// one: after a device reset the array lives at a new address in a new context.
moe_status static_scratch(int32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    CtxGetCurrentFn get_ctx = ctx_get_current();
    if (!get_ctx) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    ScratchAddr& c = g_scratch[dev];
    if (!c.ptr || !ctx || ctx != c.ctx) {
        void* p = nullptr;    // also makes the device's primary context current if none was
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return MOE_ERR_CUDA;
        c.ctx = ctx;
        c.ptr = static_cast<int32_t*>(p);
    }
    *out = c.ptr;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status moe_permute_static(const moe_layer_desc* desc, const int32_t* topk_idx,
                                                 const void* x, int32_t* expert_offsets, int32_t* row_of,
                                                 int32_t* token_of, void* x_sorted, moe_stream_t stream)
{
    t_launches = 0;
    moe_status s = validate_desc(desc);
    if (s != MOE_OK) return s;
    if (desc->kind != MOE_EXPERT_SWIGLU) return MOE_ERR_UNSUPPORTED;
    if (!expert_offsets || (desc->T > 0 && (!topk_idx || !row_of || !token_of))) return MOE_ERR_INVALID_ARG;
    if (desc->T > 0 && desc->n_ffn + desc->n_shared > 0 && !x_sorted) return MOE_ERR_INVALID_ARG;
    if (x_sorted && (!x || (reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_sorted) & 15u)))
        return MOE_ERR_INVALID_ARG;
    // the counts of every 256-token block for every FFN expert must fit the array
    const long long need = (long long)permute_blocks(desc->T) * (desc->n_ffn > 0 ? desc->n_ffn : 1);
    if (need > kStaticPermuteInts) return MOE_ERR_UNSUPPORTED;
    int32_t* scratch = nullptr;
    if ((s = static_scratch(&scratch)) != MOE_OK) return s;
    // The count kernel writes every entry the scan and scatter kernels read,
    // so nothing left in the array by an earlier call is used.
    PermuteArgs a{};
    a.idx = topk_idx;
    a.x = x;
    a.offsets = expert_offsets;
    a.row_of = row_of;
    a.token_of = token_of;
    a.x_sorted = x_sorted;
    a.ws_counts = scratch;
    a.T = desc->T;
    a.k = desc->top_k;
    a.d = desc->d_model;
    a.elt_bytes = desc->dtype == MOE_F32 ? 4 : 2;
    a.n_ffn = desc->n_ffn;
    a.n_shared = desc->n_shared;
    a.n_ids = desc->n_ffn + desc->n_zero + desc->n_copy + desc->n_const;
    return launch_permute_swiglu(a, static_cast<cudaStream_t>(stream));
}
