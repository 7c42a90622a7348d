// balance.cuh -- expert load balancing: the loss-free bias update and the
// sequence-level auxiliary balance loss ("Kimi K2.5 Q&A", Q7.2; "Kimi K2.5
// deep dive", CH10.2 step 2).
//
// The selection bias is a buffer outside the gradient: after a step, experts
// that took more than their share T*k/E of the step's routed rows have it
// lowered by gamma, experts that took less have it raised (an expert exactly at
// the mean keeps it).  The load is compared with the mean exactly, in integers,
// and the update is made in the buffer's fp32.  The sequence-level loss (the
// pages give alpha = 0.001 but no formula) is the sequence-wise balance loss
// of the DeepSeek-V3 line:
//   f_i = E / (k S) #{t in seq : i in topk(t)},   P_i = mean_t s_ti / sum_j s_tj,
//   L   = alpha sum_i f_i P_i.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kBalanceThreads = 256;

__global__ void __launch_bounds__(kBalanceThreads) bias_update_kernel(
    const int* __restrict__ counts, long long total, int E, float gamma, float* __restrict__ bias) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const long long scaled = static_cast<long long>(counts[e]) * E;
    float b = bias[e];
    if (scaled > total)
        b = __fsub_rn(b, gamma);
    else if (scaled < total)
        b = __fadd_rn(b, gamma);
    bias[e] = b;
}

// scores[t, e] = sigmoid(sum of the K-split logit partials in split order):
// the same fp32 values the top-k kernel selects from.
__global__ void __launch_bounds__(kBalanceThreads) router_scores_kernel(
    const float* __restrict__ partials, int splits, long long split_stride, long long n,
    float* __restrict__ scores) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float acc = partials[i];
    for (int sp = 1; sp < splits; ++sp) acc += partials[i + sp * split_stride];
    scores[i] = sigmoid_f32(acc);
}

// Fixed-shape block sum (deterministic): warp shuffles, then warp 0 over the
// per-warp sums in warp order.
__device__ __forceinline__ float block_sum(float v, float* scratch /*[32]*/) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    __syncthreads();
    if (lane == 0) scratch[w] = v;
    __syncthreads();
    float r = 0.0f;
    if (w == 0) {
        r = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : 0.0f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
        if (lane == 0) scratch[0] = r;
    }
    __syncthreads();
    return scratch[0];
}

// One block per sequence b of S tokens.  Dynamic shared memory: E ints (the
// selection counts) + S floats (each token's 1 / sum_j s_tj).
__global__ void __launch_bounds__(kBalanceThreads) seq_aux_loss_kernel(
    const float* __restrict__ scores, const int* __restrict__ topk_idx, int S, int E, int k,
    float alpha, float* __restrict__ loss, float* __restrict__ f_out, float* __restrict__ p_out) {
    extern __shared__ int bal_smem[];
    int* cnt = bal_smem;
    float* inv_tot = reinterpret_cast<float*>(bal_smem + E);
    __shared__ float scratch[32];
    const long long t0 = static_cast<long long>(blockIdx.x) * S;
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    // selection counts (integer atomics: order-free) and per-token totals
    for (long long j = threadIdx.x; j < static_cast<long long>(S) * k; j += blockDim.x) {
        const int e = topk_idx[t0 * k + j];
        if (e >= 0 && e < E)
            atomicAdd(&cnt[e], 1);
        else
            record_status(kStatusInvalidArg);
    }
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int t = w; t < S; t += nw) {
        const float* row = scores + (t0 + t) * E;
        float v = 0.0f;
        for (int i = lane; i < E; i += 32) v += row[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) inv_tot[t] = 1.0f / v;
    }
    __syncthreads();
    // thread i: f_i and P_i (tokens in order), then the block sum of f_i P_i
    float part = 0.0f;
    const float fscale = static_cast<float>(E) / (static_cast<float>(k) * S);
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        float p = 0.0f;
        for (int t = 0; t < S; ++t) p = fmaf(scores[(t0 + t) * E + i], inv_tot[t], p);
        p /= static_cast<float>(S);
        const float f = cnt[i] * fscale;
        if (f_out) f_out[static_cast<long long>(blockIdx.x) * E + i] = f;
        if (p_out) p_out[static_cast<long long>(blockIdx.x) * E + i] = p;
        part = fmaf(f, p, part);
    }
    const float total = block_sum(part, scratch);
    if (threadIdx.x == 0) loss[blockIdx.x] = alpha * total;
}

}  // namespace moe
