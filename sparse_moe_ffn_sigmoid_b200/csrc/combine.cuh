// combine.cuh -- deterministic weighted gather-reduce of the expert outputs.
//
// Step 7 of the MoE dataflow ("Kimi K2.5 deep dive", CH10.2): the routed
// outputs, weighted by the scaled routing weights, are added to the shared
// expert's output.  The pages accumulate with index_add_ (whose order on a GPU
// is not fixed); here each token gathers its own k rows:
//   out[t] = bf16( y_shared[t] + sum_{j=0..k-1} w[t,j] * y[slot_row[t*k+j]] )
// in fp32, slot order j = 0..k-1, so every run gives the same bits.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = 128;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(p[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 f32_to_bf16x8(const float (&f)[8]) {
    uint4 v;
    __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
}

// Block (t, c) combines the 8-element vectors v = c * blockDim.x + threadIdx.x
// (+ gridDim.y * blockDim.x ...) of token t's row.  Each thread issues the
// loads of up to 8 routed rows before it accumulates them (in slot order), so
// it waits on memory once per 8 rows; at small T the row is split over
// several blocks (gridDim.y > 1) to keep enough loads in flight.
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const bf16* __restrict__ y, const bf16* __restrict__ y_shared, const float* __restrict__ topk_w,
    const int* __restrict__ slot_row, int T, int d, int k, long long y_rows,
    bf16* __restrict__ out) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ int s_row[32];
    __shared__ float s_w[32];
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        int r = slot_row[(long long)t * k + threadIdx.x];
        if (r < 0 || r >= y_rows) {
            if (blockIdx.y == 0) record_status(kStatusInvalidArg);
            r = -1;
        }
        s_row[threadIdx.x] = r;
        s_w[threadIdx.x] = topk_w[(long long)t * k + threadIdx.x];
    }
    __syncthreads();
    const int nv = d / 8;
    for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nv; v += gridDim.y * blockDim.x) {
        float acc[8];
        if (y_shared != nullptr) {
            const uint4* ys = reinterpret_cast<const uint4*>(y_shared + (long long)t * d);
            bf16x8_to_f32(__ldg(ys + v), acc);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        }
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 raw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = (j0 + u < k) ? s_row[j0 + u] : -1;
                raw[u] = r >= 0 ? __ldg(reinterpret_cast<const uint4*>(y + (long long)r * d) + v)
                                : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int j = j0 + u;
                if (j >= k || s_row[j] < 0) continue;
                float f[8];
                bf16x8_to_f32(raw[u], f);
                const float wj = s_w[j];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
            }
        }
        reinterpret_cast<uint4*>(out + (long long)t * d)[v] = f32_to_bf16x8(acc);
    }
}

}  // namespace moe
