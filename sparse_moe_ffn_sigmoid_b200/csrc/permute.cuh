// permute.cuh -- deterministic token dispatch: per-expert histogram, exclusive
// scan, stable scatter into expert-contiguous rows, and the row gather.
//
// The pages dispatch with one boolean mask per expert ("Kimi K2.5 deep dive",
// CH10.2 step 6: token_mask = topk_indices == expert_i), which visits the
// tokens of an expert in ascending order.  This file builds the same grouping
// in three passes, bit-exact and independent of scheduling:
//   1. permute_hist:    per 128-token block, a bitmask per (warp, expert) of
//                       the lanes that chose the expert (atomicOr: order-free),
//                       popcounts -> block counts [nblk][E]
//   2. scan_plan:       block counts -> per-(block, expert) bases, counts,
//                       offsets (exclusive scan), optional GEMM tile lists
//   3. permute_scatter: rank inside the block = warp prefix + popc(mask & lanes
//                       below) -> row_token[row] = t, slot_row[t*k+j] = row
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int kPermTokens = 128;   // tokens per block (4 warps)

__global__ void __launch_bounds__(kPermTokens) permute_hist_kernel(
    const int* __restrict__ topk_idx, int T, int E, int k, int* __restrict__ blk_counts) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    extern __shared__ uint32_t mask[];   // [4][E]
    for (int i = threadIdx.x; i < 4 * E; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kPermTokens + threadIdx.x;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(long long)t * k + j];
            if (e >= 0 && e < E)
                atomicOr(&mask[w * E + e], 1u << lane);
            else
                record_status(kStatusInvalidArg);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int ww = 0; ww < 4; ++ww) c += __popc(mask[ww * E + e]);
        blk_counts[(long long)blockIdx.x * E + e] = c;
    }
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* scratch /*[32]*/) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = scratch[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        scratch[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int warp_base = w > 0 ? scratch[w - 1] : 0;
    const int tot = scratch[31];
    __syncthreads();
    *total = tot;
    return warp_base + x - v;
}

// Tile plan of the grouped SwiGLU FFN.  Expert g (0..G-1) owns rows
// [row0_g, row0_g + c_g); the shared expert (if present) is g = G-1 and reads
// its tokens from the unpermuted map.  Each expert's rows are cut into
// ceil(c/tile_n) token tiles of equal 16-multiple size; tiles are listed expert
// by expert, feature tile by feature tile, token tile fastest, so that tiles
// sharing a weight slab or a token tile run side by side.
struct PlanArgs {
    int E;                 // routed experts
    int has_shared;        // 1: append the shared expert over T tokens
    int T, d, inter;
    int rows_routed;       // T*k
    int4* tiles1;          // gate|up tiles
    int4* tiles2;          // down tiles
    int* ntiles;           // [0] = gate|up count, [1] = down count, [2], [3]: routed ones
    int kstep = kBK;       // K elements per GEMM step (FP8 compute: 2 * kBK)
    int tile_n = kTileN;   // largest token tile (a multiple of 16, <= kTileN)
};

constexpr int kPlanMaxG = 1025;   // up to 1024 routed experts and the shared one

// Writes tile `local` of expert g (c rows from row0, cut into nt token tiles
// of `chunk` rows): gate|up tiles (down = false) or down tiles, at list
// position pos.  Within an expert the tiles run feature tile by feature tile,
// token tile fastest: local = f * nt + tt.
__device__ __forceinline__ void plan_tile(const PlanArgs& p, int g, int c, int row0, int nt,
                                          int chunk, int local, bool down, int pos) {
    const bool shared = (g == p.E);
    const int f = nt == 1 ? local : local / nt;
    const int tt = local - f * nt;
    const int n = min(chunk, c - tt * chunk);
    const int map = shared ? 1 : 0;
    const int e = shared ? 0 : g;
    const int out_row = (shared ? p.rows_routed : row0) + tt * chunk;
    const int b_row = (shared ? 0 : row0) + tt * chunk;
    if (!down) {
        const int a0 = e * 2 * p.inter + f * kSlabRows;
        p.tiles1[2 * pos] = make_int4(a0, a0 + p.inter, b_row, n | (map << 16));
        p.tiles1[2 * pos + 1] = make_int4(out_row, f * kSlabRows, 0, p.d / p.kstep);
    } else {
        const int a0 = e * p.d + f * 2 * kSlabRows;
        // down reads h rows where gate|up wrote them; both B map slots of the
        // down launch point at h, the slot only picks routed / shared weights
        p.tiles2[2 * pos] = make_int4(a0, a0 + kSlabRows, out_row, n | (map << 16));
        p.tiles2[2 * pos + 1] = make_int4(out_row, f * 2 * kSlabRows, 0, p.inter / p.kstep);
    }
}

__device__ __forceinline__ void plan_counts(const PlanArgs& p, int c, int* n1, int* n2) {
    if (c <= 0) {
        *n1 = *n2 = 0;
        return;
    }
    const int nt = (c + p.tile_n - 1) / p.tile_n;
    *n1 = nt * ((p.inter + kSlabRows - 1) / kSlabRows);
    *n2 = nt * ((p.d + 2 * kSlabRows - 1) / (2 * kSlabRows));
}

// Plan over experts g = tid and g = tid + 1024 (G <= kPlanMaxG).  offsets: [E+1].
// Tile counts per expert are scanned into first positions; then each warp
// writes whole experts' tiles, its lanes taking consecutive list positions.
__device__ void plan_tiles(const PlanArgs& p, const int* offsets, int* scratch) {
    __shared__ int s_c[kPlanMaxG], s_row0[kPlanMaxG], s_first1[kPlanMaxG], s_first2[kPlanMaxG];
    const int G = p.E + p.has_shared;
    int c[2], r0[2], n1[2], n2[2];
    for (int h = 0; h < 2; ++h) {
        const int g = threadIdx.x + h * 1024;
        c[h] = 0;
        r0[h] = 0;
        if (g < p.E) {
            r0[h] = offsets[g];
            c[h] = offsets[g + 1] - offsets[g];
            // caller-supplied offsets must describe rows inside [0, T*k): a
            // malformed range gets no tiles (nothing is read or written for it)
            if (r0[h] < 0 || c[h] < 0 || offsets[g + 1] > p.rows_routed) {
                record_status(kStatusInvalidArg);
                c[h] = 0;
            }
        } else if (g < G) {
            c[h] = p.T;
        }
        plan_counts(p, c[h], &n1[h], &n2[h]);
    }
    int tot1a, tot2a, tot1b, tot2b;
    const int s1a = block_exclusive_scan(n1[0], &tot1a, scratch);
    const int s2a = block_exclusive_scan(n2[0], &tot2a, scratch);
    const int s1b = block_exclusive_scan(n1[1], &tot1b, scratch);
    const int s2b = block_exclusive_scan(n2[1], &tot2b, scratch);
    const int first1[2] = {s1a, tot1a + s1b};
    const int first2[2] = {s2a, tot2a + s2b};
    for (int h = 0; h < 2; ++h) {
        const int g = threadIdx.x + h * 1024;
        if (g < G) {
            s_c[g] = c[h];
            s_row0[g] = r0[h];
            s_first1[g] = first1[h];
            s_first2[g] = first2[h];
        }
    }
    // [0], [1]: tiles of the gate|up and down lists; [2], [3]: how many of them
    // are routed experts' (the shared expert's tiles come last)
    if (threadIdx.x == 0) {
        p.ntiles[0] = tot1a + tot1b;
        p.ntiles[1] = tot2a + tot2b;
        if (!p.has_shared) {
            p.ntiles[2] = tot1a + tot1b;
            p.ntiles[3] = tot2a + tot2b;
        }
    }
    for (int h = 0; h < 2; ++h)
        if (p.has_shared && threadIdx.x + h * 1024 == p.E) {
            p.ntiles[2] = first1[h];
            p.ntiles[3] = first2[h];
        }
    __syncthreads();
    const int ft1 = (p.inter + kSlabRows - 1) / kSlabRows;
    const int ft2 = (p.d + 2 * kSlabRows - 1) / (2 * kSlabRows);
    const int lane = threadIdx.x & 31;
    for (int g = threadIdx.x >> 5; g < G; g += blockDim.x >> 5) {
        const int cg = s_c[g];
        if (cg <= 0) continue;
        const int nt = (cg + p.tile_n - 1) / p.tile_n;
        const int chunk = pad16((cg + nt - 1) / nt);
        const int row0 = s_row0[g];
        for (int l = lane; l < nt * ft1; l += 32)
            plan_tile(p, g, cg, row0, nt, chunk, l, false, s_first1[g] + l);
        for (int l = lane; l < nt * ft2; l += 32)
            plan_tile(p, g, cg, row0, nt, chunk, l, true, s_first2[g] + l);
    }
}

// One block of 1024 threads.  blk_counts [nblk][E] is turned into per-block
// bases in place.  If plan.tiles1 is set, the GEMM tile lists are built too.
// When nblk * E counts fit the dynamic shared memory the launch provides
// (smem_counts), the per-expert scans over blocks run out of shared memory.
__global__ void __launch_bounds__(1024) scan_plan_kernel(int* __restrict__ blk_counts, int nblk,
                                                         int E, int* __restrict__ counts,
                                                         int* __restrict__ offsets, PlanArgs plan,
                                                         int smem_counts) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    extern __shared__ int sc[];
    __shared__ int scratch[32];
    __shared__ int s_total[2];
    const long long n = static_cast<long long>(nblk) * E;
    const bool staged = n <= smem_counts;
    int* cnt = staged ? sc : blk_counts;
    if (staged) {
        for (long long i = threadIdx.x; i < n; i += blockDim.x) sc[i] = blk_counts[i];
        __syncthreads();
    }
    int tot[2];
    for (int h = 0; h < 2; ++h) {
        const int e = threadIdx.x + h * 1024;
        int run = 0;
        if (e < E) {
            for (int b = 0; b < nblk; ++b) {
                const int v = cnt[(long long)b * E + e];
                cnt[(long long)b * E + e] = run;
                run += v;
            }
        }
        tot[h] = run;
    }
    int sum0, sum1;
    const int base0 = block_exclusive_scan(tot[0], &sum0, scratch);
    const int base1 = block_exclusive_scan(tot[1], &sum1, scratch) + sum0;
    if (threadIdx.x == 0) {
        s_total[0] = sum0 + sum1;
    }
    for (int h = 0; h < 2; ++h) {
        const int e = threadIdx.x + h * 1024;
        const int base = h == 0 ? base0 : base1;
        if (e < E) {
            counts[e] = tot[h];
            offsets[e] = base;
            for (int b = 0; b < nblk; ++b) cnt[(long long)b * E + e] += base;
        }
    }
    __syncthreads();
    if (staged)
        for (long long i = threadIdx.x; i < n; i += blockDim.x) blk_counts[i] = sc[i];
    if (threadIdx.x == 0) offsets[E] = s_total[0];
    if (plan.tiles1 != nullptr) {
        __syncthreads();
        plan_tiles(plan, offsets, scratch);
    }
}

// Tile plan alone, from offsets already in memory (staged expert FFN).
__global__ void __launch_bounds__(1024) plan_kernel(const int* __restrict__ offsets, PlanArgs plan) {
    __shared__ int scratch[32];
    plan_tiles(plan, offsets, scratch);
}

__global__ void __launch_bounds__(kPermTokens) permute_scatter_kernel(
    const int* __restrict__ topk_idx, int T, int E, int k, const int* __restrict__ blk_base,
    int* __restrict__ row_token, int* __restrict__ slot_row) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    extern __shared__ uint32_t sm[];
    uint32_t* mask = sm;                                  // [4][E]
    int* wbase = reinterpret_cast<int*>(sm + 4 * E);      // [4][E]
    for (int i = threadIdx.x; i < 4 * E; i += blockDim.x) mask[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kPermTokens + threadIdx.x;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(long long)t * k + j];
            if (e >= 0 && e < E) atomicOr(&mask[w * E + e], 1u << lane);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = blk_base[(long long)blockIdx.x * E + e];
        for (int ww = 0; ww < 4; ++ww) {
            wbase[ww * E + e] = run;
            run += __popc(mask[ww * E + e]);
        }
    }
    __syncthreads();
    if (t < T) {
        const uint32_t below = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(long long)t * k + j];
            if (e < 0 || e >= E) continue;
            const int row = wbase[w * E + e] + __popc(mask[w * E + e] & below);
            row_token[row] = t;
            slot_row[(long long)t * k + j] = row;
        }
    }
}

// xperm[r, :] = x[row_token[r], :]   (one warp per row, 16-byte vectors)
__global__ void __launch_bounds__(256) gather_rows_kernel(const bf16* __restrict__ x,
                                                          const int* __restrict__ row_token,
                                                          int T, int rows, int d,
                                                          bf16* __restrict__ xperm) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int t = row_token[r];
    uint4* dst = reinterpret_cast<uint4*>(xperm + (long long)r * d);
    const int nv = d / 8;
    if (t < 0 || t >= T) {
        if (lane == 0) record_status(kStatusInvalidArg);
        for (int v = lane; v < nv; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        return;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (long long)t * d);
    int v = lane;
    for (; v + 96 < nv; v += 128) {
        const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64),
                    e = __ldg(src + v + 96);
        dst[v] = a;
        dst[v + 32] = b;
        dst[v + 64] = c;
        dst[v + 96] = e;
    }
    for (; v < nv; v += 32) dst[v] = __ldg(src + v);
}

// The same permuted rows built token by token: x[t] is read once and written to
// its k rows slot_row[t*k + j] (one warp per token, 16-byte vectors, lane j
// holding the j-th destination).  At prefill this reads x once instead of k
// times (the row-by-row gather's re-reads miss L2 behind its write stream).
// A destination outside [0, rows) records kStatusInvalidArg and is skipped.
__global__ void __launch_bounds__(256) scatter_rows_kernel(const bf16* __restrict__ x,
                                                           const int* __restrict__ slot_row,
                                                           int T, int k, int rows, int d,
                                                           bf16* __restrict__ xperm) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    int dst = lane < k ? slot_row[static_cast<long long>(t) * k + lane] : 0;
    if (lane < k && (dst < 0 || dst >= rows)) {
        record_status(kStatusInvalidArg);
        dst = -1;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(t) * d);
    const int nv = d / 8;
    // every lane runs every round (the shuffles need the whole warp); only the
    // lanes with a vector in the row load and store
    for (int base = 0; base < nv; base += 32) {
        const int v = base + lane;
        const bool has = v < nv;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (has) val = __ldg(src + v);
        for (int j = 0; j < k; ++j) {
            const int r = __shfl_sync(0xffffffffu, dst, j);
            if (has && r >= 0)
                reinterpret_cast<uint4*>(xperm + static_cast<long long>(r) * d)[v] = val;
        }
    }
}

// Token rows of the FP8-compute layer, token by token: x[t] (bf16, d columns)
// is quantized once (rule above) and its codes and exponent written to the k
// permuted rows slot_row[t*k + j] and to row rows_routed + t (token order).
// One warp per token; the second pass re-reads the row from L1/L2.  A
// destination outside [0, rows_routed) records kStatusInvalidArg and is skipped.
__global__ void __launch_bounds__(32 * kRowQuantWarps) fp8_quantize_tokens_kernel(
    const bf16* __restrict__ x, const int* __restrict__ slot_row, int T, int k,
    long long rows_routed, int d, uint8_t* __restrict__ q, int8_t* __restrict__ sexp) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int t = blockIdx.x * kRowQuantWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const long long tok_row = rows_routed + t;
    long long dst = lane < k ? static_cast<long long>(slot_row[static_cast<long long>(t) * k + lane])
                             : -1;
    if (lane < k && (dst < 0 || dst >= rows_routed)) {
        record_status(kStatusInvalidArg);
        dst = -1;
    }
    const uint4* s = reinterpret_cast<const uint4*>(x + static_cast<long long>(t) * d);
    const int nv = d / 8;
    float amax = 0.0f;
#pragma unroll 4
    for (int v = lane; v < nv; v += 32) {
        const uint4 u = __ldg(s + v);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const int e = fp8_block_exponent(amax);
    if (dst >= 0) sexp[dst] = static_cast<int8_t>(e);
    if (lane == 0) sexp[tok_row] = static_cast<int8_t>(e);
    const float m1 = pow2f(-(e / 2));
    const float m2 = pow2f(-(e - e / 2));
    // every lane runs every round (the shuffles need the whole warp); only the
    // lanes with a vector in the row load, convert and store
    for (int base = 0; base < nv; base += 32) {
        const int v = base + lane;
        const bool has = v < nv;
        uint2 out = make_uint2(0u, 0u);
        if (has) {
            const uint4 u = __ldg(s + v);
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
            uint8_t* o = reinterpret_cast<uint8_t*>(&out);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(p[j]);
                o[2 * j] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.x, m1), m2), __NV_SATFINITE,
                                                 __NV_E4M3);
                o[2 * j + 1] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.y, m1), m2),
                                                     __NV_SATFINITE, __NV_E4M3);
            }
        }
        for (int j = 0; j < k; ++j) {
            const long long r = __shfl_sync(0xffffffffu, dst, j);
            if (has && r >= 0) reinterpret_cast<uint2*>(q + r * d)[v] = out;
        }
        if (has) reinterpret_cast<uint2*>(q + tok_row * d)[v] = out;
    }
}

}  // namespace moe
