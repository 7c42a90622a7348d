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
// All reductions run in fixed orders, so every run gives the same bits.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kBalanceThreads = 256;

__global__ void __launch_bounds__(kBalanceThreads) bias_update_kernel(
    const int* __restrict__ counts, long long total, int E, float gamma, float* __restrict__ bias) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
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
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float acc = partials[i];
    for (int sp = 1; sp < splits; ++sp) acc += partials[i + sp * split_stride];
    scores[i] = sigmoid_f32(acc);
}

constexpr int kAuxExperts = 32;            // experts per block of the loss kernel
constexpr int kAuxWarps = 8;

// inv_tot[t] = 1 / sum_j scores[t, j]: one warp per token, lanes over experts,
// a fixed-shape shuffle sum.
__global__ void __launch_bounds__(kBalanceThreads) token_totals_kernel(
    const float* __restrict__ scores, long long T, int E, float* __restrict__ inv_tot) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const long long t = static_cast<long long>(blockIdx.x) * (kBalanceThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const float* row = scores + t * E;
    float v = 0.0f;
    for (int i = lane; i < E; i += 32) v += row[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) inv_tot[t] = 1.0f / v;
}

constexpr int kAuxTokens = 256;            // tokens per block of the loss kernel

// Block (b, c, s): experts i = 32 c + lane of sequence b over its tokens
// [256 s, 256 s + 256).  Warp w sums 32 consecutive tokens (coalesced 128-byte
// rows of scores), the warps' sums are added in warp order into
// part[(b * nsplit + s) * E + i] = sum_t scores[t, i] / sum_j scores[t, j].
__global__ void __launch_bounds__(32 * kAuxWarps) seq_aux_partial_kernel(
    const float* __restrict__ scores, const float* __restrict__ inv_tot, int S, int E,
    float* __restrict__ part) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ float sp[kAuxWarps][kAuxExperts];
    const int b = blockIdx.x, c = blockIdx.y, sblk = blockIdx.z;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int i = c * kAuxExperts + lane;
    const long long t0 = static_cast<long long>(b) * S;
    const int tb = sblk * kAuxTokens + w * (kAuxTokens / kAuxWarps);
    const int te = min(S, tb + kAuxTokens / kAuxWarps);
    float acc = 0.0f;
    if (i < E)
        for (int t = tb; t < te; ++t) acc = fmaf(scores[(t0 + t) * E + i], inv_tot[t0 + t], acc);
    sp[w][lane] = acc;
    __syncthreads();
    if (w == 0 && i < E) {
        float v = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kAuxWarps; ++ww) v += sp[ww][lane];
        part[(static_cast<long long>(b) * gridDim.z + sblk) * E + i] = v;
    }
}

// cnt[b * E + e] += 1 for every selection of sequence b (integer atomics).
__global__ void __launch_bounds__(kBalanceThreads) seq_aux_count_kernel(
    const int* __restrict__ topk_idx, long long n, int Sk, int E, int* __restrict__ cnt) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const long long j = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= n) return;
    const int e = topk_idx[j];
    if (e < 0 || e >= E) {
        record_status(kStatusInvalidArg);
        return;
    }
    atomicAdd(&cnt[(j / Sk) * E + e], 1);
}

// One block per sequence: P_i = (sum over token blocks, in order) / S,
// f_i = cnt * E / (k S), loss[b] = alpha * (fixed-shape block sum of f_i P_i).
__global__ void __launch_bounds__(kBalanceThreads) seq_aux_finish_kernel(
    const float* __restrict__ part, const int* __restrict__ cnt, int nsplit, int S, int E, int k,
    float alpha, float* __restrict__ loss, float* __restrict__ f_out, float* __restrict__ p_out) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ float scratch[32];
    const int b = blockIdx.x;
    const float fscale = static_cast<float>(E) / (static_cast<float>(k) * S);
    float acc = 0.0f;
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        float p = 0.0f;
        for (int s = 0; s < nsplit; ++s) p += part[(static_cast<long long>(b) * nsplit + s) * E + i];
        p /= static_cast<float>(S);
        const float f = cnt[static_cast<long long>(b) * E + i] * fscale;
        if (f_out) f_out[static_cast<long long>(b) * E + i] = f;
        if (p_out) p_out[static_cast<long long>(b) * E + i] = p;
        acc = fmaf(f, p, acc);
    }
    // fixed-shape block sum
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) scratch[w] = acc;
    __syncthreads();
    if (w == 0) {
        float r = lane < static_cast<int>(blockDim.x >> 5) ? scratch[lane] : 0.0f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
        if (lane == 0) loss[b] = alpha * r;
    }
}

}  // namespace moe
