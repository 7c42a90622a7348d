// ep.cuh -- bookkeeping of the expert-parallel layer: where the token rows a
// rank receives go in its experts' grouped GEMMs, and back.
//
// "K2 inference engineer's answer", 2.1: the deployment spreads the routed
// experts over many GPUs (EP = 128: two or three experts per rank for
// DeepSeek-V3) with data parallelism over tokens.  Each rank routes and permutes
// its own tokens; its permuted rows are expert-contiguous, so the rows bound
// for the rank owning experts [q E_l, (q + 1) E_l) are one contiguous block.
// After the all-to-all, the receiving rank holds, source by source, each
// source's rows grouped by local expert (source-major).  Its grouped GEMMs want
// them expert-major: expert e's rows from source 0, then source 1, ...  (the
// order within a (source, expert) segment is the source's, ascending tokens).
//
// ep_plan_kernel turns the received counts [R][E_l] into
//   exp_offsets [E_l + 1]  expert-major segment starts (exclusive scan);
//   src_of_exp [rows]      expert-major row -> received (source-major) row;
//   exp_of_src [rows]      received row -> expert-major row.
// One block of 1024 threads; R * E_l <= 1024 (= E).  A count total other than
// `rows` records kStatusInvalidArg, leaves every expert empty and sets every
// map entry to -1.
#pragma once

#include "common.cuh"
#include "permute.cuh"

namespace moe {

__global__ void __launch_bounds__(1024) ep_plan_kernel(const int* __restrict__ recv_counts, int R,
                                                       int El, int rows,
                                                       int* __restrict__ exp_offsets,
                                                       int* __restrict__ src_of_exp,
                                                       int* __restrict__ exp_of_src) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ int scratch[32];
    __shared__ int s_seg[1024];    // source-major start of segment (s, e), index s * El + e
    __shared__ int s_exp[1024];    // expert-major start of segment (s, e), index s * El + e
    __shared__ int s_total;
    const int n = R * El;
    const int i = threadIdx.x;
    int c = 0;
    if (i < n) {
        c = recv_counts[i];
        if (c < 0) c = 0;
    }
    int total;
    // source-major: segments in (s, e) order, i = s * El + e
    s_seg[i] = block_exclusive_scan(c, &total, scratch);
    // expert-major: segments in (e, s) order; thread j = e * R + s takes segment (s, e)
    int ce = 0;
    int se = 0, ee = 0;
    if (i < n) {
        ee = i / R;
        se = i - ee * R;
        ce = recv_counts[se * El + ee];
        if (ce < 0) ce = 0;
    }
    int total2;
    const int base_e = block_exclusive_scan(ce, &total2, scratch);
    if (i < n) s_exp[se * El + ee] = base_e;
    if (i == 0) s_total = total;
    __syncthreads();
    const bool ok = (s_total == rows);
    if (i == 0 && !ok) record_status(kStatusInvalidArg);
    // expert offsets: the expert-major start of (0, e); the end is the total
    for (int e = i; e <= El; e += blockDim.x) exp_offsets[e] = (ok && e < El) ? s_exp[e] : (ok ? rows : 0);
    if (!ok) {
        // no expert gets rows; the row maps point nowhere (the gathers that
        // read them write zero rows)
        for (int r = i; r < rows; r += blockDim.x) src_of_exp[r] = exp_of_src[r] = -1;
        return;
    }
    // maps, one warp per segment
    const int lane = i & 31;
    for (int seg = i >> 5; seg < n; seg += blockDim.x >> 5) {
        const int cnt = recv_counts[seg];
        const int a = s_seg[seg], b = s_exp[seg];
        for (int r = lane; r < cnt; r += 32) {
            src_of_exp[b + r] = a + r;
            exp_of_src[a + r] = b + r;
        }
    }
}

}  // namespace moe
