// route.cuh -- sigmoid scoring, selection-only bias, top-k and weights.
//
// Steps 1-4 of the MoE dataflow ("Kimi K2.5 deep dive", CH4.2 and CH10.2;
// "Kimi K2.5 Q&A", Q8.3): s = sigmoid(logits), b = s + bias, top-k of b over
// all experts (n_group = 1, "K2 inference" answer, 2.4), w = scale * s / sum(s)
// over the selected experts, with s the UNBIASED score.
//
// One warp per token.  The router GEMM (gemm.cuh, fp32 partial sums over K
// splits) leaves logits in `partials[split][t][e]`; this kernel adds the
// splits in a fixed order, so the result is deterministic.
#pragma once

#include "common.cuh"

namespace moe {

// NPL = experts held per lane (E <= 32 * NPL); expert of slot i on lane l is i*32+l.
template <int NPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ partials, int splits,
                                                   long long split_stride, int T, int E, int k,
                                                   const float* __restrict__ bias, float scale,
                                                   int* __restrict__ topk_idx,
                                                   float* __restrict__ topk_w) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float s[NPL], b[NPL];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
            const float* p = partials + (long long)t * E + e;
            float acc = p[0];
            for (int sp = 1; sp < splits; ++sp) acc += p[sp * split_stride];
            s[i] = sigmoid_f32(acc);
            b[i] = s[i] + bias[e];
        } else {
            s[i] = 0.0f;
            b[i] = -INFINITY;
            taken |= 1u << i;      // padding never wins
        }
    }
    float my_s = 0.0f;             // lane j keeps the score of slot j
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        // lane-local best: largest b, then lowest expert index (slots visited in e order)
        float bv = -INFINITY;
        int be = 0x7FFFFFFF;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            if (!(taken & (1u << i)) && (bi < 0 || b[i] > bv)) {
                bv = b[i];
                be = i * 32 + lane;
                bi = i;
            }
        }
        // warp argmax, ties to the lower expert index
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        // owner marks it taken and publishes the unbiased score
        float sv = 0.0f;
        if ((be & 31) == lane) {
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i == (be >> 5)) {
                    taken |= 1u << i;
                    sv = s[i];
                }
        }
        sv = __shfl_sync(0xffffffffu, sv, be & 31);
        if (lane == j) {
            my_s = sv;
            my_e = be;
        }
    }
    // sum of the selected unbiased scores with a fixed reduction shape over
    // expert positions, so it depends on the selected set only
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        const bool sel = e < E && (taken & (1u << i));
        float v = sel ? s[i] : 0.0f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        part += v;
    }
    if (lane < k) {
        topk_idx[(long long)t * k + lane] = my_e;
        topk_w[(long long)t * k + lane] = scale * (my_s / part);
    }
}

}  // namespace moe
