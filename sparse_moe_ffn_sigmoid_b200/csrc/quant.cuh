// quant.cuh -- FP8 (E4M3) storage of the routed experts' weights.
//
// "Kimi K2.5 Q&A", Q7.1: the deployment quantizes the routed experts' weight
// storage while compute stays in BF16, and the shared experts stay BF16.  The
// pages give no FP8 format; the one used here is OCP E4M3 elements with one
// power-of-two scale 2^s per block of 128 rows x 128 columns (K), s an int8:
//   s = the smallest integer with amax <= 448 * 2^s, clamped to [-124, 127]
//       (s = 0 for an all-zero block), amax = the block's largest |w|;
//   q = E4M3 nearest to w * 2^-s (ties to even; the scaling is exact).
// Dequantization q * 2^s is then exact in bf16, so the expert GEMMs compute
// with exactly the weights the codes stand for.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

constexpr int kQuantBlock = 128;          // rows and columns per scale block
constexpr int kQuantThreads = 256;

// 2^e as a float, e in [-126, 127] (a normal number, built from its bits).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// Block exponent from the block's largest magnitude (rule above), from the
// bits of amax: amax = 1.f * 2^E lies within 448 * 2^(E-8) = 1.75 * 2^E exactly
// when 1.f <= 1.75.
__device__ __forceinline__ int fp8_block_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    const uint32_t bits = __float_as_uint(amax);
    const int ef = static_cast<int>(bits >> 23) & 0xFF;
    if (ef == 0) return -124;                               // below 2^-126: clamped
    int s = ef - 127 - 8 + ((bits & 0x7FFFFF) > 0x600000 ? 1 : 0);
    return max(-124, min(127, s));
}

// One block of kQuantThreads threads per 128 x 128 block (blockIdx.x = row
// block, blockIdx.y = column block) of w [rows, cols] bf16 row-major.
__global__ void __launch_bounds__(kQuantThreads) fp8_quantize_kernel(const bf16* __restrict__ w,
                                                                     long long cols,
                                                                     uint8_t* __restrict__ q,
                                                                     int8_t* __restrict__ sexp) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    __shared__ float s_max[kQuantThreads / 32];
    const long long r0 = static_cast<long long>(blockIdx.x) * kQuantBlock;
    const long long c0 = static_cast<long long>(blockIdx.y) * kQuantBlock;
    // thread -> 8 consecutive columns of rows r = tid / 16 + 16 i
    const int cc = (threadIdx.x & 15) * 8;
    const int rr = threadIdx.x >> 4;
    float amax = 0.0f;
    for (int i = 0; i < kQuantBlock / 16; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(w + (r0 + rr + 16 * i) * cols + c0 + cc);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = s_max[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) amax = fmaxf(amax, s_max[i]);
    const int s = fp8_block_exponent(amax);
    if (threadIdx.x == 0)
        sexp[static_cast<long long>(blockIdx.x) * gridDim.y + blockIdx.y] = static_cast<int8_t>(s);
    // w * 2^-s in two exact steps (2^-s alone may be below the normal range)
    const float m1 = pow2f(-(s / 2));
    const float m2 = pow2f(-(s - s / 2));
    for (int i = 0; i < kQuantBlock / 16; ++i) {
        const long long off = (r0 + rr + 16 * i) * cols + c0 + cc;
        const uint4 v = *reinterpret_cast<const uint4*>(w + off);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
        uint2 out;
        uint8_t* o = reinterpret_cast<uint8_t*>(&out);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            o[2 * j] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.x, m1), m2), __NV_SATFINITE,
                                             __NV_E4M3);
            o[2 * j + 1] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.y, m1), m2),
                                                 __NV_SATFINITE, __NV_E4M3);
        }
        *reinterpret_cast<uint2*>(q + off) = out;
    }
}

// A pair of bf16x2 multipliers m1, m2 (both lanes alike) that turn a scaled
// E4M3 value into code * 2^s in two exact power-of-two multiplies.
struct Fp8Scale {
    __nv_bfloat162 m1, m2;
};

__device__ __forceinline__ __nv_bfloat162 bf16x2_pow2(int e) {
    // 2^e, -126 <= e <= 127: exponent field e + 127, zero mantissa, both lanes
    const uint32_t b = static_cast<uint32_t>(e + 127) << 7;
    const uint32_t w = b | (b << 16);
    return *reinterpret_cast<const __nv_bfloat162*>(&w);
}

// Two E4M3 codes (the bytes of v16, the low byte first) -> one bf16x2 word whose
// values are code * 2^-112, bit for bit.  The hardware conversion to f16x2 is
// exact (every E4M3 value, subnormals included, is a normal f16 number or zero);
// an f16 number with exponent field E and mantissa m, moved three bits down
// under its sign, is the bf16 number with exponent field E and mantissa m >> 3,
// i.e. its value times 2^(15 - 127); E4M3 values leave the low seven mantissa
// bits of the f16 number zero, so nothing is lost and nothing crosses into the
// other lane.
__device__ __forceinline__ uint32_t fp8x2_to_bf16x2_pow2m112(uint16_t v16) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v16));
    return ((h & 0x7FFF7FFFu) >> 3) | (h & 0x80008000u);
}

// Multipliers for a block exponent s with the 2^-112 form above: m1 =
// 2^(112 + min(s, 15)), m2 = 2^(s - min(s, 15)), both normal bf16 numbers for
// s in [-238, 142]; each product is exact.
__device__ __forceinline__ Fp8Scale fp8_scale_m112(int s) {
    const int a = min(s, 15);
    return Fp8Scale{bf16x2_pow2(112 + a), bf16x2_pow2(s - a)};
}

// Eight E4M3 codes (little-endian in `v`) -> eight bf16 values code * 2^s, exact
// (sc from fp8_scale_m112).
__device__ __forceinline__ uint4 fp8x8_to_bf16x8_cvt(uint2 v, const Fp8Scale& sc) {
    const uint32_t w[4] = {fp8x2_to_bf16x2_pow2m112(static_cast<uint16_t>(v.x)),
                           fp8x2_to_bf16x2_pow2m112(static_cast<uint16_t>(v.x >> 16)),
                           fp8x2_to_bf16x2_pow2m112(static_cast<uint16_t>(v.y)),
                           fp8x2_to_bf16x2_pow2m112(static_cast<uint16_t>(v.y >> 16))};
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        const __nv_bfloat162 y = __hmul2(__hmul2(x, sc.m1), sc.m2);
        o[i] = *reinterpret_cast<const uint32_t*>(&y);
    }
    return out;
}

// ------------------------------------------------------------ INT4 storage
// "Kimi K2.5 deep dive", CH7.2: the K2.5 routed experts' weights are 4-bit
// integers, symmetric, one scale per group of 32 K elements of a row ("Kimi
// K2.5 Q&A", Q7.1: storage quantized, compute BF16).  Rule (the config gives
// none): s = bf16(amax / 7), q = clamp(nearest integer to w / s, ties to even,
// -8, 7) (0 when s = 0); the weight computed with is bf16(q * s).
// Device layout (this library's packing):
//   codes  [rows, cols / 2] bytes: 32-bit word j of a row (little-endian) holds
//          elements 8j .. 8j+7, element 8j + 2i in bits 4i .. 4i+3 and element
//          8j + 2i + 1 in bits 16 + 4i .. 16 + 4i + 3, each as q + 8 (0 .. 15);
//   scales [cols / 32, rows] bf16, group-major, so one TMA box brings a K step's
//          scales of 128 rows.
constexpr int kInt4Group = 32;
constexpr int kInt4Warps = 8;             // groups per block of the quantizer

// One warp per (row, group); lane = element of the group.  amax / 7 and w / s
// are taken in fp32: amax / 7 never lies on a bf16 rounding midpoint and w / s
// (two bf16 values) is either exactly on a half-integer or at least 2^-9 of
// its size away from one, so both decisions equal the exact ones.
__global__ void __launch_bounds__(32 * kInt4Warps) int4_quantize_kernel(
    const bf16* __restrict__ w, long long rows, int cols, uint32_t* __restrict__ codes,
    bf16* __restrict__ scale) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int gpr = cols / kInt4Group;
    const long long gid = static_cast<long long>(blockIdx.x) * kInt4Warps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gid >= rows * gpr) return;
    const long long r = gid / gpr;
    const int g = static_cast<int>(gid - r * gpr);
    const float v = __bfloat162float(w[r * cols + static_cast<long long>(g) * kInt4Group + lane]);
    float amax = fabsf(v);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const bf16 sb = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
    const float sv = __bfloat162float(sb);
    int n = 0;
    if (sv != 0.0f) n = max(-8, min(7, __float2int_rn(__fdiv_rn(v, sv))));
    const int e = lane & 7;                              // element within the word
    const int nib = (e & 1) ? (e >> 1) + 4 : (e >> 1);
    uint32_t bits = static_cast<uint32_t>(n + 8) << (4 * nib);
    bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
    bits |= __shfl_xor_sync(0xffffffffu, bits, 2);
    bits |= __shfl_xor_sync(0xffffffffu, bits, 4);
    if (e == 0) codes[(r * cols + static_cast<long long>(g) * kInt4Group) / 8 + (lane >> 3)] = bits;
    if (lane == 0) scale[static_cast<long long>(g) * rows + r] = sb;
}

// Eight packed codes (one word, layout above) -> eight bf16 weights bf16(q * s):
// 0x4300 | n is the bf16 value 128 + n, so (128 + n) - 136 = q exactly, and one
// bf16 multiply rounds q * s to nearest-even.
// Pair i (elements 2i and 2i + 1 of the word's eight) of int4x8_to_bf16x8.
__device__ __forceinline__ uint32_t int4_pair_to_bf16x2(uint32_t wd, int i, __nv_bfloat162 s2) {
    const uint32_t v = ((wd >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
    const uint32_t off_bits = 0x43084308u;               // 136.0 in both halves
    const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v),
                                     *reinterpret_cast<const __nv_bfloat162*>(&off_bits));
    const __nv_bfloat162 y = __hmul2(q, s2);
    return *reinterpret_cast<const uint32_t*>(&y);
}

__device__ __forceinline__ uint4 int4x8_to_bf16x8(uint32_t wd, __nv_bfloat162 s2) {
    const uint32_t magic = 0x43004300u;
    uint32_t v[4];
    v[0] = (wd & 0x000F000Fu) | magic;
    v[1] = ((wd >> 4) & 0x000F000Fu) | magic;
    v[2] = ((wd >> 8) & 0x000F000Fu) | magic;
    v[3] = ((wd >> 12) & 0x000F000Fu) | magic;
    const uint32_t off_bits = 0x43084308u;               // 136.0 in both halves
    const __nv_bfloat162 off = *reinterpret_cast<const __nv_bfloat162*>(&off_bits);
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 q = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v[i]), off);
        const __nv_bfloat162 y = __hmul2(q, s2);
        o[i] = *reinterpret_cast<const uint32_t*>(&y);
    }
    return out;
}

// ------------------------------------------------------------- FP8 compute
// Operands of the FP8-compute GEMMs ("Kimi K2.5 Q&A", Q7.1: V3 computes in
// FP8): E4M3 codes with one power-of-two exponent per ROW (a weight row is an
// output channel, an activation row a token), by the same smallest-exponent
// rule as the blocks above.  The exponents factor out of every K sum, so the
// tensor cores multiply codes and the epilogue applies 2^(s_w + s_x) exactly.

constexpr int kRowQuantWarps = 8;         // rows per block (one warp each)

// Row r of q [rows, cols] / sexp [rows] is the quantization of source row
// row_map[r] (r < n_map: a gather) or r - n_map (after it) of src (bf16,
// leading dimension ld, src_rows rows).  A source index out of range zeroes
// the row and records kStatusInvalidArg.  cols: a multiple of 8.
__global__ void __launch_bounds__(32 * kRowQuantWarps) fp8_quantize_rows_kernel(
    const bf16* __restrict__ src, long long ld, const int* __restrict__ row_map, long long n_map,
    long long src_rows, long long rows, int cols, uint8_t* __restrict__ q,
    int8_t* __restrict__ sexp) {
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const long long r = static_cast<long long>(blockIdx.x) * kRowQuantWarps + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const long long sr = r < n_map ? static_cast<long long>(row_map[r]) : r - n_map;
    uint2* qr = reinterpret_cast<uint2*>(q + r * cols);
    const int nv = cols / 8;
    if (sr < 0 || sr >= src_rows) {
        if (lane == 0) {
            record_status(kStatusInvalidArg);
            sexp[r] = 0;
        }
        for (int v = lane; v < nv; v += 32) qr[v] = make_uint2(0u, 0u);
        return;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src + sr * ld);
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
    if (lane == 0) sexp[r] = static_cast<int8_t>(e);
    // w * 2^-e in two exact steps (2^-e alone may be below the normal range)
    const float m1 = pow2f(-(e / 2));
    const float m2 = pow2f(-(e - e / 2));
#pragma unroll 4
    for (int v = lane; v < nv; v += 32) {
        const uint4 u = __ldg(s + v);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint2 out;
        uint8_t* o = reinterpret_cast<uint8_t*>(&out);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            o[2 * j] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.x, m1), m2), __NV_SATFINITE,
                                             __NV_E4M3);
            o[2 * j + 1] = __nv_cvt_float_to_fp8(__fmul_rn(__fmul_rn(f.y, m1), m2),
                                                 __NV_SATFINITE, __NV_E4M3);
        }
        qr[v] = out;
    }
}

// v * 2^e for the sum of two row exponents (e in [-248, 254] for exponents the
// quantizers produce), in two power-of-two factors that are normal floats.
__device__ __forceinline__ float mul_pow2(float v, int e) {
    const int e1 = max(-126, min(127, e >> 1));
    const int e2 = max(-126, min(127, e - e1));
    return __fmul_rn(__fmul_rn(v, pow2f(e1)), pow2f(e2));
}

}  // namespace moe
