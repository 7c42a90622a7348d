// gemv.cuh -- decode-sized grouped expert GEMMs for routed weights stored as
// INT4 or E4M3 codes: the codes stream from HBM into shared memory by TMA, are
// dequantized in registers and multiplied on the warp-level tensor-core MMA,
// whose A operand comes from registers.
//
// At decode an expert sees one or two tokens on average ("Kimi K2.5 Q&A",
// Q8.3: the per-expert work is a small matrix times a few rows), so the layer
// streams the touched experts' weights once and does 2 FLOPs per weight and
// token.  The tcgen05 GEMM takes its A operand from shared memory only: INT4
// codes would have to be converted into a bf16 copy there first, which costs
// more SM time per byte than the HBM stream.  Here each code is read once from
// shared memory into registers, converted there to the exact bf16 weight it
// stands for (INT4: bf16(q * s); E4M3: q * 2^s; the same weights as the
// converting tcgen05 modes) and enters mma.sync.m16n8k16 as the A fragment; the
// expert's tokens (<= 16 per tile, two MMA n-tiles of 8) are the B fragment.
//
// Work: the plan's tile list with token tiles of at most 16 rows.  A tile is
// (expert, 256 weight rows, <= 16 tokens): gate|up tiles hold 128 gate rows and
// the matching 128 up rows, down tiles two 128-row blocks.  The 8 warps of a CTA
// take the 8 units of one tile (two sets of 16 weight rows each: 16 gate + the
// matching 16 up rows, or 32 consecutive down rows), so the tile's token rows
// are read from L1 by all of them; CTAs walk the tile list round-robin.  The
// shared expert's bf16 tiles are a launch of their own (the plan lists them
// after the routed ones), which the host runs on a second stream beside the
// routed launch.
//
// Pipeline.  Every warp streams its own units with its own ring of
// gemv_depth() stages in shared memory: lane 0 issues a step's TMA loads (one
// box of both row sets, 32 rows x 128 bytes, 128-byte swizzle; INT4 also one
// box of the sets' group scales) on the stage's mbarrier, gemv_depth() - 1
// steps ahead of the step the warp computes; the walk over (unit, step) is
// flat, so the loads of the next unit start while the current one finishes.
// Every wait is bounded.
//
// K order.  A step is 128 bytes of a weight row: 256 K for INT4 (8 groups), 128
// for E4M3 (one scale block), 64 for bf16 (the shared expert).  Lane (g, c) =
// (lane / 4, lane % 4) owns bytes [32c, 32c + 32) of its rows' step, i.e. the K
// slice [step base + 8Pc, + 8P) (P = 8, 4, 2 MMA pairs per step).  MMA pair m
// takes the 8 elements [8m, 8m + 8) of every lane's slice: the first MMA of the
// pair its elements 0..3 as logical k {2c, 2c+1, 2c+8, 2c+9}, the second its
// elements 4..7.  The B fragment (token g) is loaded with the same slice, so A
// and B agree on every k; the sum over k is the same, only its order differs
// from a row-major walk.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "quant.cuh"

namespace moe {

constexpr int kGemvWarps = 8;                  // one warp per unit of a tile
constexpr int kGemvTileN = 16;                 // token rows per tile: two MMA n-tiles
constexpr int kGemvRowBytes = 128;             // bytes of a weight row per step
constexpr int kGemvSetBytes = 16 * kGemvRowBytes;      // one 16-row set per step
constexpr int kGemvStageBytes = 2 * kGemvSetBytes;     // both sets (1024-byte aligned)
constexpr int kGemvScaleBytes = 2 * 8 * 16 * 2;        // INT4: 2 sets x 8 groups x 16 rows bf16

enum GemvWeights : int {
    kGemvInt4 = 0,   // INT4 codes, a bf16 scale per group of 32 (routed experts)
    kGemvBF16 = 1,   // bf16 weights (the shared expert)
    kGemvFp8 = 2,    // E4M3 codes, a power-of-two scale per 128 x 128 block (routed experts)
};

// Stages per warp ring; 2 CTAs per SM.  The routed formats run 3 stages (the
// shared memory of an SM holds no more).  The shared expert's launch has few
// tiles (its token tiles x 256-row blocks), so its warps are few and each
// streams a long K walk: 6 stages keep 5 steps in flight per warp instead of 2.
__host__ __device__ constexpr int gemv_depth(int wf) { return wf == kGemvBF16 ? 6 : 3; }
// CTAs per tile: the shared expert's launch splits each tile's 8 units over 2
// CTAs of 4 warps, so that its few tiles reach more SMs.
__host__ __device__ constexpr int gemv_split(int wf) { return wf == kGemvBF16 ? 2 : 1; }
__host__ __device__ constexpr int gemv_warps(int wf) { return kGemvWarps / gemv_split(wf); }
__host__ __device__ constexpr int gemv_threads(int wf) { return 32 * gemv_warps(wf); }
__host__ __device__ constexpr int gemv_ctas_per_sm(int) { return 2; }

// K elements per step (one 128-byte row chunk) of a weight format.
__host__ __device__ constexpr int gemv_step_k(int wf) {
    return wf == kGemvInt4 ? 256 : wf == kGemvFp8 ? 128 : 64;
}

// Dynamic shared memory of one CTA: 1024 bytes of alignment slack, the warps'
// code rings, their scale rings (INT4), their stage barriers and abort flags.
__host__ __device__ constexpr int gemv_smem_bytes(int wf) {
    return 1024 +
           gemv_warps(wf) * gemv_depth(wf) * (kGemvStageBytes + (wf == kGemvInt4 ? kGemvScaleBytes : 0)) +
           gemv_warps(wf) * gemv_depth(wf) * 8 + gemv_warps(wf) * 4;
}

struct __align__(64) GemvArgs {
    // weights: routed INT4 codes [code_rows, K / 2] or E4M3 codes [code_rows, K]
    // (uint8), or the shared expert's bf16 weights [rows, K], as a 4-D view
    // (x, row in half, half, expert) with 128-byte swizzle; one box is a unit's
    // 128-byte step of 16 gate rows and the matching 16 up rows (gate|up) or of
    // 32 consecutive rows (down)
    CUtensorMap a_map;
    // INT4 group scales [K / 32, code_rows] bf16 as (row in half, half, expert,
    // group): one box is the same rows' 8 groups of a step
    CUtensorMap s_map;
    const int4* tiles;          // the plan's tile list (token tiles of <= kGemvTileN rows)
    const int* first;           // tiles [*first, *last) of the list (device; null first = 0)
    const int* last;
    const int8_t* exps;         // E4M3 block exponents [code_rows / 128, K / 128]
    const bf16* b[2];           // token rows [.., K] bf16: [0] routed tiles, [1] shared tiles
    bf16* out;                  // h (SwiGLU epilogue) or Y, row-major, leading dim out_ld
    long long out_ld;
    int K;                      // contraction length, a multiple of the format's step
    int col_limit;              // output features >= col_limit are not stored
    int expert_rows;            // rows of one expert's stack: 2 * inter (gate|up) or d (down)
    unsigned long long timeout_ns;
};

// The unit of warp u in a tile: its two 16-row sets (lane row g reads rows
// set + g and set + g + 8 of each) and its first output feature.
struct GemvRows {
    int set0, set1;
    int f0;
    int te, tr;     // the weight box's expert and row-in-half coordinates
    bool ok;
};

template <int EPI>
__device__ __forceinline__ GemvRows gemv_rows(const Tile& t, int u, int col_limit,
                                              int expert_rows) {
    GemvRows R;
    if constexpr (EPI == kEpiSwiGLU) {
        R.set0 = t.a_row0 + 16 * u;        // gate rows
        R.set1 = t.a_row1 + 16 * u;        // the matching up rows
        R.f0 = t.out_col0 + 16 * u;
    } else {
        const int slab = u >> 2;
        R.set0 = (slab ? t.a_row1 : t.a_row0) + (u & 3) * 32;
        R.set1 = R.set0 + 16;
        R.f0 = t.out_col0 + slab * 128 + (u & 3) * 32;
    }
    R.te = R.set0 / expert_rows;
    R.tr = R.set0 - R.te * expert_rows;
    // col_limit is a multiple of 64 and f0 of 16 (32 for down units), so a unit's
    // features are all inside or all outside
    R.ok = R.f0 < col_limit;
    return R;
}

// A warp's position in its flat walk over (unit, step).
struct GemvCursor {
    int i;          // tile index (>= last: done)
    int st;         // step within the unit
    Tile t;
    GemvRows R;
};

// Moves `cu` to the first unit `unit` at tile index >= cu.i (this CTA's
// stride through the list) that has work; false when there is none.  A tile
// that does not belong to this kernel's plan is recorded and skipped (nothing
// is read).
template <int EPI, int WF>
__device__ __forceinline__ bool gemv_seek(const GemvArgs& a, GemvCursor& cu, int last, int warp) {
    for (; cu.i < last; cu.i += gridDim.x / gemv_split(WF)) {
        cu.t = tile_at(a.tiles, cu.i);
        if (cu.t.n <= 0) continue;
        if (cu.t.n > kGemvTileN || cu.t.map != (WF == kGemvBF16 ? 1 : 0)) {
            if ((threadIdx.x & 31) == 0) record_status(kStatusInvalidArg);
            continue;
        }
        cu.R = gemv_rows<EPI>(cu.t, warp, a.col_limit, a.expert_rows);
        if (cu.R.ok) {
            cu.st = 0;
            return true;
        }
    }
    return false;
}

template <int EPI, int WF>
__device__ __forceinline__ bool gemv_advance(const GemvArgs& a, GemvCursor& cu, int nsteps,
                                             int last, int warp) {
    if (++cu.st < nsteps) return true;
    cu.i += gridDim.x / gemv_split(WF);
    return gemv_seek<EPI, WF>(a, cu, last, warp);
}

// Waits for a stage: all lanes test its barrier at once (every lane that
// sees the phase complete has acquired the stage's bytes), and only a stage
// that has not landed yet takes the bounded lane-0 wait.
__device__ __forceinline__ bool gemv_wait_stage(uint64_t* bar, uint32_t parity,
                                                volatile int* abort_flag, uint64_t tmo, int lane) {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    return wait_lane0(bar, parity, abort_flag, tmo, lane);
}

// Lane 0: the TMA loads of one step into a stage, completing on `bar`: one
// box of both row sets' codes and, for INT4, one box of their group scales.
template <int WF>
__device__ __forceinline__ void gemv_issue(const GemvArgs& a, const GemvCursor& cu, uint8_t* codes,
                                           uint8_t* scales, uint64_t* bar, uint64_t pol) {
    constexpr uint32_t bytes = kGemvStageBytes + (WF == kGemvInt4 ? kGemvScaleBytes : 0);
    // x in the map's elements: 128 bytes per step (uint8 codes) or 64 bf16
    const int x = cu.st * (WF == kGemvBF16 ? kGemvRowBytes / 2 : kGemvRowBytes);
    ptx::mbar_arrive_expect_tx(bar, bytes);
    ptx::tma_load_4d_hint(codes, &a.a_map, bar, x, cu.R.tr, 0, cu.R.te, pol);
    if constexpr (WF == kGemvInt4)
        ptx::tma_load_4d_hint(scales, &a.s_map, bar, cu.R.tr, 0, cu.R.te, 8 * cu.st, pol);
}

__device__ __forceinline__ uint32_t u4_word(const uint4& v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 16-byte chunk q (0..7) of row rr (0..15) of a set in a 128-byte-swizzled stage
__device__ __forceinline__ uint4 gemv_chunk(const uint8_t* set, int rr, int q) {
    return *reinterpret_cast<const uint4*>(set + rr * kGemvRowBytes + ((q ^ (rr & 7)) << 4));
}

template <int EPI>
__device__ __forceinline__ void gemv_epilogue(const GemvArgs& a, const GemvCursor& cu,
                                              float (&acc)[2][2][4], int lane) {
    const int g = lane >> 2, c = lane & 3;
    const Tile& t = cu.t;
    const GemvRows& R = cu.R;
    const int NT = t.n > 8 ? 2 : 1;
    // acc[so][nt] = {D[g][2c], D[g][2c+1], D[g+8][2c], D[g+8][2c+1]} of row set so
    // (rows = features, columns = tokens nt * 8 + ...).  Lanes g and g ^ 1 swap
    // halves so each stores two adjacent features of one token as one 4-byte
    // word: even g the features (g, g + 1), odd g (g + 7, g + 8).
    bf16* out = a.out;
    const bool odd = g & 1;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        if (nt >= NT) break;
        float v[2][4];     // per output block (SwiGLU: one; down: set 0 and set 1)
        if constexpr (EPI == kEpiSwiGLU) {
#pragma unroll
            for (int i = 0; i < 4; ++i) v[0][i] = silu_fast(acc[0][nt][i]) * acc[1][nt][i];
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[0][i] = acc[0][nt][i];
                v[1][i] = acc[1][nt][i];
            }
        }
        constexpr int nblk = (EPI == kEpiSwiGLU) ? 1 : 2;
#pragma unroll
        for (int b = 0; b < nblk; ++b) {
            const float s0 = odd ? v[b][0] : v[b][2];
            const float s1 = odd ? v[b][1] : v[b][3];
            const float r0 = __shfl_xor_sync(0xffffffffu, s0, 4);
            const float r1 = __shfl_xor_sync(0xffffffffu, s1, 4);
            // token 2c: (lo, hi) features; token 2c + 1 likewise
            const float lo0 = odd ? r0 : v[b][0], hi0 = odd ? v[b][2] : r0;
            const float lo1 = odd ? r1 : v[b][1], hi1 = odd ? v[b][3] : r1;
            const int f = R.f0 + 16 * b + (odd ? g + 7 : g);
            const int tok = nt * 8 + 2 * c;
            if (tok < t.n)
                *reinterpret_cast<__nv_bfloat162*>(out + static_cast<long long>(t.out_row0 + tok) *
                                                             a.out_ld + f) =
                    __floats2bfloat162_rn(lo0, hi0);
            if (tok + 1 < t.n)
                *reinterpret_cast<__nv_bfloat162*>(out + static_cast<long long>(t.out_row0 + tok + 1) *
                                                             a.out_ld + f) =
                    __floats2bfloat162_rn(lo1, hi1);
        }
    }
}

// One step of a unit: the MMAs of its P pairs on both row sets and the unit's
// NT token n-tiles (NT = 1: the tile has at most 8 tokens), accumulating into
// acc.  Lanes whose token column is past the tile read the tile's last token
// row instead: MMA columns are independent, and the epilogue stores only the
// tile's own columns, so no load needs a guard.
template <int WF, int NT>
__device__ __forceinline__ void gemv_step(const GemvArgs& a, const GemvCursor& cu,
                                          const uint8_t* codes, const uint8_t* scales,
                                          const int (&e8)[2], float (&acc)[2][2][4], int lane) {
    constexpr int KS = gemv_step_k(WF);
    constexpr int P = KS / 32;                        // MMA pairs per step
    constexpr int PJ = P / 2;                         // pairs per 16-byte chunk of a lane
    const int g = lane >> 2, c = lane & 3;
    const Tile& t = cu.t;
    // token rows of this step: lane slice [st * KS + 8Pc, + 8P)
    const uint4* brow[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int j = min(nt * 8 + g, t.n - 1);
        brow[nt] = reinterpret_cast<const uint4*>(a.b[t.map] +
                                                  static_cast<long long>(t.b_row0 + j) * a.K +
                                                  static_cast<long long>(cu.st) * KS + 8 * P * c);
    }
    // E4M3: the two row sets' multipliers
    Fp8Scale fs[2];
    if constexpr (WF == kGemvFp8) {
#pragma unroll
        for (int so = 0; so < 2; ++so) fs[so] = fp8_scale_m112(e8[so]);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {                     // the lane's two chunks of each row
        uint4 av[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            av[i] = gemv_chunk(codes + (i >> 1) * kGemvSetBytes, g + 8 * (i & 1), 2 * c + j);
        // INT4: the scales of group 2c + j of the lane's four rows
        uint32_t sc[4];
        if constexpr (WF == kGemvInt4) {
            const uint16_t* ss = reinterpret_cast<const uint16_t*>(scales);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // row i: set i / 2, lane row g (+ 8 for odd i) of the box's
                // [group][set][16 rows]; the scale in both halves (v < 2^16,
                // so v * 0x10001 = v | v << 16)
                const uint32_t v = ss[(2 * c + j) * 32 + (i >> 1) * 16 + g + 8 * (i & 1)];
                sc[i] = v * 0x10001u;
            }
        }
#pragma unroll
        for (int pm = 0; pm < PJ; ++pm) {             // pair m = j * PJ + pm
            uint4 bv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) bv[nt] = __ldg(brow[nt] + j * PJ + pm);
#pragma unroll
            for (int so = 0; so < 2; ++so) {
                if constexpr (WF == kGemvInt4) {
                    // each MMA's A fragment in operand order: pairs (0, 1), then
                    // (2, 3), of the lane's rows g and g + 8
                    const uint32_t w0 = u4_word(av[2 * so], pm), w1 = u4_word(av[2 * so + 1], pm);
                    const __nv_bfloat162 s0 = *reinterpret_cast<const __nv_bfloat162*>(&sc[2 * so]);
                    const __nv_bfloat162 s1 = *reinterpret_cast<const __nv_bfloat162*>(&sc[2 * so + 1]);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t a0 = int4_pair_to_bf16x2(w0, 2 * half, s0);
                        const uint32_t a1 = int4_pair_to_bf16x2(w1, 2 * half, s1);
                        const uint32_t a2 = int4_pair_to_bf16x2(w0, 2 * half + 1, s0);
                        const uint32_t a3 = int4_pair_to_bf16x2(w1, 2 * half + 1, s1);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            ptx::mma_16816_bf16(acc[so][nt], a0, a1, a2, a3,
                                                half ? bv[nt].z : bv[nt].x, half ? bv[nt].w : bv[nt].y);
                    }
                } else {
                    uint4 q[2];     // the pair's 8 weights of rows 2 so (g) and 2 so + 1 (g + 8)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int i = 2 * so + h;
                        if constexpr (WF == kGemvFp8) {
                            const uint2 c8 =
                                pm ? make_uint2(av[i].z, av[i].w) : make_uint2(av[i].x, av[i].y);
                            q[h] = fp8x8_to_bf16x8_cvt(c8, fs[so]);
                        } else {
                            q[h] = av[i];
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        ptx::mma_16816_bf16(acc[so][nt], q[0].x, q[1].x, q[0].y, q[1].y, bv[nt].x,
                                            bv[nt].y);
                        ptx::mma_16816_bf16(acc[so][nt], q[0].z, q[1].z, q[0].w, q[1].w, bv[nt].z,
                                            bv[nt].w);
                    }
                }
            }
        }
    }
}

// One launch = the routed tiles (WF kGemvInt4 / kGemvFp8: INT4 / E4M3 codes) or
// the shared expert's tiles (kGemvBF16: bf16 weights) of one of the layer's
// two expert GEMMs: EPI kEpiSwiGLU writes h = silu(gate) * up, kEpiStoreBF16
// writes Y.  The plan lists the shared expert's tiles after the routed ones; a
// launch takes its kind's range.
template <int EPI, int WF>
__global__ void __launch_bounds__(gemv_threads(WF), gemv_ctas_per_sm(WF))
    moe_gemv_kernel(const __grid_constant__ GemvArgs a) {
    extern __shared__ uint8_t gemv_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemv_smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    constexpr int kScale = (WF == kGemvInt4) ? kGemvScaleBytes : 0;
    constexpr int kDepth = gemv_depth(WF);
    constexpr int kWarps = gemv_warps(WF);
    constexpr int kSplit = gemv_split(WF);
    constexpr int kRings = kWarps * kDepth * (kGemvStageBytes + kScale);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this warp's unit of each tile (of kGemvWarps), and the CTA's first tile
    const int warp = (blockIdx.x % kSplit) * kWarps + w;
    uint8_t* codes_ring = smem + w * kDepth * kGemvStageBytes;
    uint8_t* scale_ring = smem + kWarps * kDepth * kGemvStageBytes + w * kDepth * kScale;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRings) + w * kDepth;
    volatile int* abort_flag =
        reinterpret_cast<volatile int*>(smem + kRings + kWarps * kDepth * 8) + w;
    if (lane == 0) {
        for (int s = 0; s < kDepth; ++s) ptx::mbar_init(&full[s], 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&a.a_map);
        if (WF == kGemvInt4) ptx::prefetch_tensormap(&a.s_map);
    }
    __syncwarp();
    // the set-up above touches only shared memory: it may overlap the previous
    // kernel on the stream, whose results are read from here on
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();

    const int first = a.first ? *a.first : 0;
    const int last = *a.last;
    const int nsteps = a.K / gemv_step_k(WF);
    const uint64_t pol = ptx::policy_evict_first();
    const uint64_t tmo = a.timeout_ns;

    GemvCursor pc, cc;          // producer (loads) and consumer (MMAs) positions
    pc.i = first + blockIdx.x / kSplit;
    bool p_ok = gemv_seek<EPI, WF>(a, pc, last, warp);
    cc = pc;
    bool c_ok = p_ok;
    uint32_t qp = 0, qc = 0;    // steps issued / consumed by this warp
    // kDepth - 1 steps in flight before the first is consumed
    for (int s = 0; s < kDepth - 1 && p_ok; ++s) {
        if (lane == 0)
            gemv_issue<WF>(a, pc, codes_ring + (qp % kDepth) * kGemvStageBytes,
                           scale_ring + (qp % kDepth) * kScale, &full[qp % kDepth], pol);
        ++qp;
        p_ok = gemv_advance<EPI, WF>(a, pc, nsteps, last, warp);
    }

    float acc[2][2][4];
    bool ok = true;
    while (c_ok) {
        // refill the stage consumed last (every lane is past it: __syncwarp below)
        if (p_ok) {
            if (lane == 0) {
                ptx::fence_proxy_async_smem();
                gemv_issue<WF>(a, pc, codes_ring + (qp % kDepth) * kGemvStageBytes,
                               scale_ring + (qp % kDepth) * kScale, &full[qp % kDepth], pol);
            }
            ++qp;
            p_ok = gemv_advance<EPI, WF>(a, pc, nsteps, last, warp);
        }
        if (cc.st == 0) {
#pragma unroll
            for (int so = 0; so < 2; ++so)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[so][nt][i] = 0.0f;
        }
        int e8[2] = {0, 0};
        if constexpr (WF == kGemvFp8) {
            // E4M3: the block exponents of the two row sets at this step's K block
            const int kb = a.K / kQuantBlock;
            e8[0] = __ldg(a.exps + static_cast<long long>(cc.R.set0 / kQuantBlock) * kb + cc.st);
            e8[1] = __ldg(a.exps + static_cast<long long>(cc.R.set1 / kQuantBlock) * kb + cc.st);
        }
        const uint32_t stage = qc % kDepth;
        if (!gemv_wait_stage(&full[stage], (qc / kDepth) & 1, abort_flag, tmo, lane)) {
            ok = false;
            break;
        }
        if (cc.t.n > 8)
            gemv_step<WF, 2>(a, cc, codes_ring + stage * kGemvStageBytes,
                             scale_ring + stage * kScale, e8, acc, lane);
        else
            gemv_step<WF, 1>(a, cc, codes_ring + stage * kGemvStageBytes,
                             scale_ring + stage * kScale, e8, acc, lane);
        __syncwarp();                       // every lane is done with the stage
        ++qc;
        if (cc.st == nsteps - 1) gemv_epilogue<EPI>(a, cc, acc, lane);
        c_ok = gemv_advance<EPI, WF>(a, cc, nsteps, last, warp);
    }
    if (!ok && lane == 0) {
        // the loads this warp started land before the CTA exits
        for (uint32_t q = qc; q < qp; ++q)
            wait_bounded(&full[q % kDepth], (q / kDepth) & 1, nullptr, tmo);
    }
}

}  // namespace moe
