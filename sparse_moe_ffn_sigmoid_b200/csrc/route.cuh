// route.cuh -- sigmoid scoring, selection-only bias, top-k and weights.
//
// Steps 1-4 of the MoE dataflow ("Kimi K2.5 deep dive", CH4.2 and CH10.2;
// "Kimi K2.5 Q&A", Q8.3): s = sigmoid(logits), b = s + bias, top-k of b over
// all experts (n_group = 1, "K2 inference" answer, 2.4), w = scale * s / sum(s)
// over the selected experts, with s the UNBIASED score.
//
// The router GEMM (gemm.cuh, fp32 partial sums over K splits) leaves logits
// in `partials[split][t][e]`; each expert's splits are added in split order,
// so the result is deterministic.  Two launch shapes share the selection: a
// warp per token for large batches, a block per token (one thread per
// expert) for small batches with many splits.
#pragma once

#include "common.cuh"

namespace moe {

// Sum of expert e's K-split logit partials in split order (deterministic),
// loads issued kBatch at a time so the sum waits on memory once per batch.
template <int kBatch>
__device__ __forceinline__ float split_sum(const float* __restrict__ p, int splits,
                                           long long split_stride) {
    float acc = 0.0f;
    int sp = 0;
    for (; sp + kBatch <= splits; sp += kBatch) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) v[u] = p[(sp + u) * split_stride];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) acc += v[u];
    }
    for (; sp < splits; ++sp) acc += p[sp * split_stride];
    return acc;
}

// Top-k selection of one token by one warp.  Lane l holds slot i = expert
// i*32+l: unbiased score s[i] and biased score b[i]; `taken` marks padding
// slots (E <= e).  Writes topk_idx/topk_w of token t.
template <int NPL>
__device__ __forceinline__ void select_topk(const float (&s)[NPL], const float (&b)[NPL],
                                            uint32_t taken, int E, int k, float scale, int lane,
                                            int* __restrict__ idx_out, float* __restrict__ w_out) {
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
        idx_out[lane] = my_e;
        w_out[lane] = scale * (my_s / part);
    }
}

// Large batches: one warp per token (8 tokens per 256-thread block); lane l
// scores experts i*32+l itself.  NPL = experts per lane (E <= 32 * NPL).
template <int NPL>
__global__ void __launch_bounds__(256) topk_warp_kernel(const float* __restrict__ partials,
                                                        int splits, long long split_stride, int T,
                                                        int E, int k,
                                                        const float* __restrict__ bias,
                                                        float scale, int* __restrict__ topk_idx,
                                                        float* __restrict__ topk_w) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
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
    select_topk<NPL>(s, b, taken, E, k, scale, lane, topk_idx + (long long)t * k,
                     topk_w + (long long)t * k);
}

// Small batches (many K splits, few tokens): one block of 32 * NPL threads per
// token, thread e scoring expert e, so every partial of the token is in
// flight at once; warp 0 then selects from shared memory.
template <int NPL>
__global__ void __launch_bounds__(32 * NPL) topk_block_kernel(const float* __restrict__ partials,
                                                              int splits, long long split_stride,
                                                              int T, int E, int k,
                                                              const float* __restrict__ bias,
                                                              float scale,
                                                              int* __restrict__ topk_idx,
                                                              float* __restrict__ topk_w) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ float sh_s[32 * NPL], sh_b[32 * NPL];
    const int t = blockIdx.x;
    if (t >= T) return;
    {
        const int e = threadIdx.x;
        float sv = 0.0f, bv = -INFINITY;      // padding never wins
        if (e < E) {
            sv = sigmoid_f32(split_sum<8>(partials + (long long)t * E + e, splits, split_stride));
            bv = sv + bias[e];
        }
        sh_s[e] = sv;
        sh_b[e] = bv;
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float s[NPL], b[NPL];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        s[i] = sh_s[i * 32 + lane];
        b[i] = sh_b[i * 32 + lane];
        if (i * 32 + lane >= E) taken |= 1u << i;
    }
    select_topk<NPL>(s, b, taken, E, k, scale, lane, topk_idx + (long long)t * k,
                     topk_w + (long long)t * k);
}

}  // namespace moe
