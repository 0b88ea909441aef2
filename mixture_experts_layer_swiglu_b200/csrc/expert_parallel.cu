// expert_parallel.cu -- the exchange plan of an expert-parallel layer (host
// code only).
//
// With experts split over G ranks, a rank keeps routing, permuting and
// combining its own tokens, but its expert rows are computed by the ranks
// that own those experts.  Ownership follows the grouping of tasks by
// contiguous ranges of expert ids ("OmniMoE" technical summary, 2.2
// Expert-Centric Scheduling): rank r owns experts [r E / G, (r + 1) E / G).
// Each rank's rows for expert e are already contiguous in its x_sorted
// (expert-major, token order inside), so a rank sends, per expert, one block
// of rows to the expert's owner, and the owner lays the received blocks out
// expert-major (source rank inside), which makes the owned experts ordinary
// groups of the grouped GEMM.  The results travel back the same blocks to the
// positions they came from, so the combine is the single-rank one.  This
// file computes where every block lands from the matrix of per-rank expert
// counts; the exchange itself is done by the caller (NCCL send/recv).

#include <stdint.h>

#include "moe.h"

namespace {

inline int32_t owner_lo(int G, int E, int r) { return (int32_t)(((int64_t)r * E) / G); }

}  // namespace

extern "C" {

MOE_API moe_status moe_ep_expert_range(int G, int E, int rank, int32_t* lo, int32_t* hi)
{
    if (G <= 0 || E <= 0 || rank < 0 || rank >= G || !lo || !hi) return MOE_ERR_INVALID_ARG;
    *lo = owner_lo(G, E, rank);
    *hi = owner_lo(G, E, rank + 1);
    return MOE_OK;
}

MOE_API int32_t moe_ep_owner(int G, int E, int expert)
{
    if (G <= 0 || E <= 0 || expert < 0 || expert >= E) return -1;
    // the r with lo(r) <= expert < lo(r + 1)
    int32_t r = (int32_t)((((int64_t)expert + 1) * G - 1) / E);
    while (r > 0 && owner_lo(G, E, r) > expert) --r;
    while (r + 1 < G && owner_lo(G, E, r + 1) <= expert) ++r;
    return r;
}

MOE_API int64_t moe_ep_plan(const int32_t* counts, int G, int E, int rank, int32_t* recv_offsets,
                            int32_t* recv_counts, int32_t* local_offsets)
{
    if (!counts || G <= 0 || E <= 0 || rank < 0 || rank >= G || !recv_offsets || !recv_counts || !local_offsets)
        return -1;
    const int32_t lo = owner_lo(G, E, rank), hi = owner_lo(G, E, rank + 1);
    int64_t run = 0;
    for (int32_t e = lo; e < hi; ++e) {
        const int i = e - lo;
        local_offsets[i] = (int32_t)run;
        for (int q = 0; q < G; ++q) {
            const int32_t c = counts[(int64_t)q * E + e];
            if (c < 0) return -1;
            recv_offsets[(int64_t)i * G + q] = (int32_t)run;
            recv_counts[(int64_t)i * G + q] = c;
            run += c;
            if (run >= (1ll << 31)) return -1;
        }
    }
    local_offsets[hi - lo] = (int32_t)run;
    return run;
}

}  // extern "C"
