// gemm.cuh -- grouped "weights x tokens" GEMM on tcgen05 / TMEM / TMA (sm_100a).
//
// One kernel serves the three contractions of the layer:
//   router     logits[t, e]   = sum_i Wr[e, i] x[t, i]                 (fp32 out)
//   gate|up    h[r, n]        = silu(Wg_e[n,:] . X[r,:]) * (Wu_e[n,:] . X[r,:])
//   down       Y[r, o]        = sum_n Wd_e[o, n] h[r, n]
// ("Kimi K2.5 deep dive", CH10.2 steps 1, 5 and 6; "Kimi K2.5 Q&A", Q8.3).
//
// Orientation: the weight rows (output features) are the MMA's M = 128 lanes,
// the tokens of one expert are its N columns (16..256, a multiple of 16).  A
// tile is therefore (expert, 128 or 256 output features, up to 256 tokens):
// every weight byte is streamed from HBM once per token tile, and an expert
// with few tokens (decode) wastes no weight traffic on padding rows.
//
// Roles inside a 352-thread CTA (one CTA per SM, persistent over tiles):
//   warp 0      weight producer (one lane): A slab(s) 128 x 64 per K step
//   warp 10     token producer  (one lane): B rows N x 64 per K step
//   warp 1      MMA issuer      (one lane): 4 x tcgen05.mma (K=16) per slab per step;
//               the whole warp allocates / frees the 512 TMEM columns
//   warps 2..9  epilogue: two warps per TMEM lane quarter, each taking every
//               other 32-column chunk; tcgen05.ld 32 lanes x 32 columns,
//               convert, store
// FP8-weight mode (480 threads): warps 2..5 are the epilogue (one per lane
// quarter, every chunk), warps 6..9 and 11..14 dequantize E4M3 weight codes
// into the bf16 weight ring (convert_weights).
// FP8-compute mode (352 threads, the roles above): weights and tokens are
// E4M3 codes with one exponent per row; a K step is 128 codes (the same
// 128-byte rows), the MMAs are kind::f8f6f4 (K = 32), and the epilogue scales
// each accumulator by 2^(weight row exponent + token row exponent).
// Weights come from HBM and tokens mostly from L2, so the two operands have
// separate rings: a deep one for weights (their HBM latency needs many bytes
// in flight) and a short one for tokens.  K step q uses weight slot q % SA and
// token slot q % SB (SB <= SA).  The single issuing thread is the bottleneck
// of the MMA side (each tcgen05.mma, commit and barrier wait costs it tens of
// cycles), so it sees one barrier per K step: full[q % SA] counts the arrivals
// of both producers and all their bytes, and one commit to empty[q % SA]
// releases both slots (the token producer waits on the empty barrier of step
// q - SB).  Accumulators (1 or 2 TMEM buffers) have acc_full/acc_empty.
// Every wait is bounded (see wait_bounded).
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace moe {

constexpr int kBK = 64;                       // K elements per pipeline stage (128 B rows)
constexpr int kSlabRows = 128;                // MMA M
constexpr int kSlabBytes = kSlabRows * kBK * 2;
constexpr int kBoxRows = 16;                  // TMA box height for token rows (tail)
constexpr int kBoxRowsBig = 64;               // TMA box height for token rows (bulk)
constexpr int kEpiWarps = 8;                  // two per TMEM lane quarter, splitting the columns
constexpr int kStageRows = 32;                // epilogue staging block: 32 tokens x 32 features
constexpr int kStagingBytes = kEpiWarps * kStageRows * 32 * 2;
constexpr int kMaxN = 256;                    // MMA N limit (router tiles)
// Token rows per tile of the grouped expert GEMMs.  One tile covers a whole
// expert up to 256 tokens, so each weight byte is streamed once per expert.
constexpr int kTileN = 256;
constexpr int kGemmThreads = 352;             // 11 warps: roles below
constexpr int kTokenWarp = 10;
// FP8-weight mode: 15 warps.  Warps 2..5 are the epilogue (one per TMEM lane
// quarter, 4 instead of 8) and warps 6..9 and 11..14 dequantize the weight
// codes into the bf16 ring (two converter warps per SM sub-partition).
constexpr int kEpiWarpsFP8 = 4;
constexpr int kConvWarps = 8;
constexpr int kConvGroups = 2;                // converter groups, on alternating K steps
constexpr int kConvThreads = 32 * kConvWarps / kConvGroups;   // threads per group
constexpr int kGemmThreadsFP8 = 480;
constexpr int kSlabBytes8 = kSlabRows * kBK;  // one FP8 slab per K step (128 rows x 64 codes)
// INT4 slab per K step: 128 rows x 64 codes packed in 32 bytes, then the step's two
// group scales of the 128 rows (bf16, group-major)
constexpr int kSlabCodes4 = kSlabRows * kBK / 2;
constexpr int kSlabBytes4 = kSlabCodes4 + kSlabRows * 2 * 2;
constexpr int kTmemCols = 512;

// Operand formats of a launch.
enum GemmOperands : int {
    kOpsBF16 = 0,       // bf16 weights and tokens (kind::f16)
    kOpsW8Convert = 1,  // routed weights as block-scaled E4M3, dequantized in shared memory
    kOpsFP8 = 2,        // E4M3 weights and tokens with per-row exponents (kind::f8f6f4)
    kOpsW4Convert = 3,  // routed weights as INT4 with group-32 scales, dequantized in shared memory
};

// Modes whose routed weights are converted to bf16 in shared memory, and the
// bytes one weight slab of a K step takes in their code ring.
__host__ __device__ constexpr bool ops_convert(int ops) {
    return ops == kOpsW8Convert || ops == kOpsW4Convert;
}
__host__ __device__ constexpr int code_slab_bytes(int ops) {
    return ops == kOpsW4Convert ? kSlabBytes4 : kSlabBytes8;
}

enum GemmEpilogue : int {
    kEpiSwiGLU = 0,   // 2 slabs (gate, up) -> bf16 silu(gate) * up
    kEpiStoreBF16 = 1,// 1-2 slabs -> bf16
    kEpiStoreF32 = 2, // 1 slab -> fp32 (router logit partials)
};

// A tile as stored in the tile list: two int4.
//   v0 = {a_row0, a_row1, b_row0, n | map << 16}
//   v1 = {out_row0, out_col0, ks0, ks1}
struct Tile {
    int a_row0, a_row1, b_row0, n, map, out_row0, out_col0, ks0, ks1;
};

struct __align__(64) GemmArgs {
    CUtensorMap a_map[2];     // weights: [0] routed (or router), [1] shared expert
    CUtensorMap b_map[2];     // tokens:  [0] permuted rows,       [1] rows in token order
    CUtensorMap b_map64[2];   // the same token matrices read in 64-row boxes
    const int4* tiles;        // grouped tile list (2 x int4 per tile), or null = dense mode
    const int* ntiles_dev;    // grouped mode: number of tiles (device)
    int ntiles_host;          // dense mode: number of tiles
    // dense mode (router): tile i -> (m slab fastest, then token tile, then K split)
    int dense_mslabs, dense_ttiles, dense_tchunk, dense_splits, dense_T, dense_ksteps;
    void* out;                // bf16 or fp32 output, row-major with leading dim out_ld
    long long out_ld;
    int col_limit;            // output features >= col_limit are not stored
    int nslab;                // A slabs per tile (1 or 2)
    int n_max;                // largest tile N of the launch (multiple of 16)
    int stages_a;             // weight ring depth
    int stages_b;             // token ring depth
    int acc_bufs;             // accumulator buffers in TMEM (1 or 2)
    int acc_stride;           // TMEM columns per accumulator buffer
    unsigned long long timeout_ns;
    // FP8-weight mode only: routed tiles (map 0) read E4M3 codes through a8_map
    // ([rows, K] uint8, 64 x 128 boxes) and one int8 exponent per 128 x 128 block
    // (a8_scale[(row / 128) * a8_kblocks + k / 128]); shared tiles (map 1) stay bf16
    // INT4-weight mode: a8_map reads the packed codes ([rows, K/2] bytes, 32 x 128
    // boxes) and a4s_map the group scales ([K/32, rows] bf16, 128 x 2 boxes)
    CUtensorMap a8_map;
    CUtensorMap a4s_map;
    const int8_t* a8_scale;
    int a8_kblocks;
    int stages_a8;            // FP8 code ring depth
    // FP8-compute mode only: one int8 exponent per weight row (a_exp[map],
    // indexed like the A rows) and per token row (b_exp[map], like the B rows)
    const int8_t* a_exp[2];
    const int8_t* b_exp[2];
};

// Tile i of a grouped tile list.
__device__ __forceinline__ Tile tile_at(const int4* tiles, int i) {
    Tile t;
    const int4 v0 = tiles[2 * i];
    const int4 v1 = tiles[2 * i + 1];
    t.a_row0 = v0.x;
    t.a_row1 = v0.y;
    t.b_row0 = v0.z;
    t.n = v0.w & 0xFFFF;
    t.map = (v0.w >> 16) & 1;
    t.out_row0 = v1.x;
    t.out_col0 = v1.y;
    t.ks0 = v1.z;
    t.ks1 = v1.w;
    return t;
}

__device__ __forceinline__ Tile load_tile(const GemmArgs& a, int i) {
    Tile t;
    if (a.tiles != nullptr) {
        t = tile_at(a.tiles, i);
    } else {
        const int m = i % a.dense_mslabs;
        const int r = i / a.dense_mslabs;
        const int tt = r % a.dense_ttiles;
        const int sp = r / a.dense_ttiles;
        t.a_row0 = m * kSlabRows;
        t.a_row1 = t.a_row0 + kSlabRows;
        t.b_row0 = tt * a.dense_tchunk;
        t.n = min(a.dense_tchunk, a.dense_T - t.b_row0);
        t.map = 0;
        t.out_row0 = sp * a.dense_T + t.b_row0;
        t.out_col0 = m * kSlabRows * a.nslab;
        t.ks0 = (int)((long long)sp * a.dense_ksteps / a.dense_splits);
        t.ks1 = (int)((long long)(sp + 1) * a.dense_ksteps / a.dense_splits);
    }
    return t;
}

__device__ __forceinline__ int pad16(int n) { return (n + 15) & ~15; }

// Position in a ring of n slots; the phase bit flips on every wrap.
struct Ring {
    uint32_t stage, phase;
    int n;
    __device__ __forceinline__ void next() {
        if (++stage == static_cast<uint32_t>(n)) {
            stage = 0;
            phase ^= 1;
        }
    }
};

// Writes one warp's block of an output tile: v[j] is the value of token row
// (row0 + j) and feature (fbase + lane), j < ncol.  The block goes through the
// warp's shared staging buffer [32 rows][32 features] so that global memory
// sees 16-byte stores of 8 consecutive features instead of 2-byte ones.  Rows
// >= nrows and features >= col_limit are not written.
__device__ __forceinline__ void store_block_bf16(bf16* stg, const float (&v)[kStageRows], int ncol,
                                                 bf16* out, long long ld, int row0, int nrows,
                                                 int fbase, int col_limit, int lane) {
#pragma unroll
    for (int j = 0; j < kStageRows; ++j)
        if (j < ncol) stg[j * 32 + lane] = __float2bfloat16_rn(v[j]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kStageRows * 4 / 32; ++i) {
        const int vi = lane + 32 * i;
        const int r = vi >> 2, part = vi & 3;
        const int f = fbase + part * 8;
        if (r < nrows && f < col_limit)
            *reinterpret_cast<uint4*>(out + (long long)(row0 + r) * ld + f) =
                *reinterpret_cast<const uint4*>(stg + r * 32 + part * 8);
    }
    __syncwarp();
}

// store_block_bf16 for values already rounded to bf16, two per word: pk[i]
// holds token rows 2i (low half) and 2i + 1 (high half) of feature lane.
__device__ __forceinline__ void store_block_packed(bf16* stg, const uint32_t (&pk)[kStageRows / 2],
                                                   int ncol, bf16* out, long long ld, int row0,
                                                   int nrows, int fbase, int col_limit, int lane) {
    uint16_t* s16 = reinterpret_cast<uint16_t*>(stg);
#pragma unroll
    for (int j = 0; j < kStageRows; ++j)
        if (j < ncol) s16[j * 32 + lane] = static_cast<uint16_t>(pk[j >> 1] >> (16 * (j & 1)));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < kStageRows * 4 / 32; ++i) {
        const int vi = lane + 32 * i;
        const int r = vi >> 2, part = vi & 3;
        const int f = fbase + part * 8;
        if (r < nrows && f < col_limit)
            *reinterpret_cast<uint4*>(out + (long long)(row0 + r) * ld + f) =
                *reinterpret_cast<const uint4*>(stg + r * 32 + part * 8);
    }
    __syncwarp();
}

// Lane 0 waits (bounded) and the warp shares the outcome; after a completed
// wait every lane observes the phase itself (one try_wait, which cannot fail
// then: the barrier cannot complete its next phase before this warp acts), so
// each lane acquires what the phase publishes.
__device__ __forceinline__ bool wait_lane0(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t tmo, int lane) {
    bool ok = true;
    if (lane == 0) ok = wait_bounded(bar, parity, abort_flag, tmo);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) (void)ptx::mbar_try_wait(bar, parity);
    return ok;
}

// Converting modes: the kConvWarps converter warps fill the bf16 weight ring
// in two groups of four warps (one per SM sub-partition each); group g takes
// the K steps q = g mod 2, so two steps are converted at once.  At each of its
// steps every warp of the group waits for the step's code slot (full8: the
// codes landed, or the producer's plain arrival on a shared-expert step) and
// for the bf16 slot (empty: the MMAs of step q - SA done), and the group's
// warps meet on their own named barrier once per step.  The code ring is
// indexed by the global step like the bf16 ring, so every slot use is waited
// on by the group that makes it.  A waiter can never be two phases behind a
// slot's barrier: its previous step needed the MMAs (or codes) of an earlier
// use of every slot, which run in step order.
// Routed step: thread ct (0 .. 127 of its group) converts eight codes at a
// time, units u = ct + 128 i (slab u / 1024, row (u / 8) % 128, chunk u % 8),
// into the 128-byte-swizzled layout a TMA box would have produced (row r at
// byte 128 r, 16-byte chunk c at position c ^ (r % 8)).  Every thread fences
// its stores towards the async proxy before the barrier, and the group's
// thread 0 then publishes the slot (full) and frees the codes (empty8).
// Shared-expert step (bf16 in HBM): after the barrier the group's thread 0
// loads the bf16 weights into the slot with TMA (arrive.expect_tx on full) and
// frees the (unused) code slot.
template <int nslab, int OPS>
__device__ __forceinline__ void convert_weights(const GemmArgs& args, const uint8_t* ring8,
                                                uint8_t* ring_a, int SA, int SA8, uint64_t* full,
                                                uint64_t* empty, uint64_t* full8,
                                                uint64_t* empty8, volatile int* abort_flag,
                                                uint64_t tmo, int ntiles, int grp, int ct) {
    constexpr bool kInt4 = (OPS == kOpsW4Convert);
    constexpr uint32_t a8_bytes = nslab * code_slab_bytes(OPS);
    constexpr uint32_t a_bytes = nslab * kSlabBytes;
    constexpr int kUnits = nslab * kSlabRows * (kBK / 8) / kConvThreads;   // per thread
    static_assert(kUnits == 16 && nslab == 2, "unit geometry: 2 slabs x 8 row blocks");
    const int lane = ct & 31;
    // thread-constant geometry of the units u = ct + 128 j: chunk c = ct % 8,
    // rows r0 + 16 (j % 8) with r0 = ct / 8, slab j / 8; (r0 + 16 i) % 8 == r0 % 8,
    // so the 128-byte swizzle of the destination chunk is a thread constant too
    const int r0 = ct >> 3, cc = ct & 7;
    const uint32_t dst_off = r0 * (kBK * 2) + ((cc ^ (r0 & 7)) << 4);
    const uint32_t code_off = kInt4 ? r0 * (kBK / 2) + cc * 4 : r0 * kBK + cc * 8;
    const uint32_t scale_off = kSlabCodes4 + (cc >> 2) * (kSlabRows * 2) + r0 * 2;
    const uint64_t pol = ptx::policy_evict_first();
    Ring rq{0, 0, SA};          // bf16 slot of step q
    Ring r8{0, 0, SA8};         // code slot of step q
    uint32_t q = 0;
    bool ok = true;
    uint32_t issued = 0, issued_parity = 0;   // thread 0's bf16 loads, for draining
    for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
        const Tile t = load_tile(args, i);
        const bool routed = (t.map == 0);
        const int8_t* sc0 =
            kInt4 ? nullptr : args.a8_scale + (t.a_row0 / kQuantBlock) * args.a8_kblocks;
        const int8_t* sc1 =
            kInt4 ? nullptr : args.a8_scale + (t.a_row1 / kQuantBlock) * args.a8_kblocks;
        for (int ks = t.ks0; ks < t.ks1; ++ks, ++q) {
            if (static_cast<int>(q & 1) != grp) {     // the other group's step
                r8.next();
                rq.next();
                continue;
            }
            bool w_ok = wait_lane0(&full8[r8.stage], r8.phase, abort_flag, tmo, lane) &&
                        wait_lane0(&empty[rq.stage], rq.phase ^ 1, abort_flag, tmo, lane);
            if (kInt4 && routed && w_ok) {
                const uint8_t* src = ring8 + r8.stage * a8_bytes;
                uint8_t* dst = ring_a + rq.stage * a_bytes;
                // unit j: slab j / 8, row r0 + 16 (j % 8), 8-code chunk c (group c / 4):
                // every offset is a thread constant plus a compile-time one
                uint32_t words[kUnits];
#pragma unroll
                for (int j = 0; j < kUnits; ++j)
                    words[j] = *reinterpret_cast<const uint32_t*>(
                        src + code_off + (j / 8) * kSlabBytes4 + (j % 8) * 16 * (kBK / 2));
#pragma unroll
                for (int j = 0; j < kUnits; ++j) {
                    const bf16 sc = *reinterpret_cast<const bf16*>(
                        src + scale_off + (j / 8) * kSlabBytes4 + (j % 8) * 16 * 2);
                    *reinterpret_cast<uint4*>(dst + dst_off + (j / 8) * kSlabBytes +
                                              (j % 8) * 16 * (kBK * 2)) =
                        int4x8_to_bf16x8(words[j], __bfloat162bfloat162(sc));
                }
                ptx::fence_proxy_async_smem();
            } else if (routed && w_ok) {
                const Fp8Scale s0 = fp8_scale_m112(__ldg(sc0 + ks * kBK / kQuantBlock));
                const Fp8Scale s1 =
                    nslab == 2 ? fp8_scale_m112(__ldg(sc1 + ks * kBK / kQuantBlock)) : s0;
                const uint8_t* src = ring8 + r8.stage * a8_bytes;
                uint8_t* dst = ring_a + rq.stage * a_bytes;
                // all of this thread's code loads first, then the conversions:
                // the kUnits chains are independent, so their latencies overlap
                uint2 codes[kUnits];
#pragma unroll
                for (int j = 0; j < kUnits; ++j)
                    codes[j] = *reinterpret_cast<const uint2*>(
                        src + code_off + (j / 8) * kSlabBytes8 + (j % 8) * 16 * kBK);
#pragma unroll
                for (int j = 0; j < kUnits; ++j)
                    *reinterpret_cast<uint4*>(dst + dst_off + (j / 8) * kSlabBytes +
                                              (j % 8) * 16 * (kBK * 2)) =
                        fp8x8_to_bf16x8_cvt(codes[j], j < 8 ? s0 : s1);
                ptx::fence_proxy_async_smem();
            }
            // every thread of the group reaches its barrier once per step of the group
            ok = ptx::bar_red_and(1 + grp, kConvThreads, w_ok);
            if (!ok) break;
            if (ct == 0) {
                ptx::mbar_arrive(&empty8[r8.stage]);
                if (routed) {
                    ptx::mbar_arrive(&full[rq.stage]);
                } else {
                    uint64_t* bar = &full[rq.stage];
                    uint8_t* sa = ring_a + rq.stage * a_bytes;
                    ptx::mbar_arrive_expect_tx(bar, a_bytes);
                    ptx::tma_load_2d_hint(sa, &args.a_map[1], bar, ks * kBK, t.a_row0, pol);
                    if (nslab == 2)
                        ptx::tma_load_2d_hint(sa + kSlabBytes, &args.a_map[1], bar, ks * kBK,
                                              t.a_row1, pol);
                    issued |= 1u << rq.stage;
                    issued_parity = (issued_parity & ~(1u << rq.stage)) | (rq.phase << rq.stage);
                }
            }
            r8.next();
            rq.next();
        }
    }
    if (ct == 0 && !ok) {
        // the bf16 loads this thread started land before the CTA exits
        for (int s = 0; s < SA; ++s)
            if (issued & (1u << s)) wait_bounded(&full[s], (issued_parity >> s) & 1, nullptr, tmo);
    }
}

// OPS (GemmOperands): kOpsW8Convert / kOpsW4Convert have routed weights arrive
// as E4M3 / INT4 codes that the converter warps dequantize in shared memory
// (kGemmThreadsFP8 threads); kOpsBF16 is the all-bf16 kernel and kOpsFP8 the
// FP8-compute one (kGemmThreads threads).
template <int EPI, int OPS>
__global__ void __launch_bounds__(ops_convert(OPS) ? kGemmThreadsFP8 : kGemmThreads, 1)
    moe_gemm_kernel(const __grid_constant__ GemmArgs args) {
    constexpr bool FP8A = ops_convert(OPS);     // a converting mode (E4M3 or INT4 codes)
    constexpr bool kInt4 = (OPS == kOpsW4Convert);
    constexpr bool F8C = (OPS == kOpsFP8);
    constexpr int kStepK = F8C ? 2 * kBK : kBK;   // K elements per step (128-byte rows)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int SA = args.stages_a;
    const int SB = args.stages_b;
    // the router has one weight slab per tile, the expert GEMMs two (gate|up,
    // or two 128-row blocks of down); compile-time so the issuing thread
    // runs no branches on it (the host sets args.nslab to match)
    constexpr int nslab = (EPI == kEpiStoreF32) ? 1 : 2;
    const uint32_t a_bytes = nslab * kSlabBytes;
    const uint32_t b_bytes = args.n_max * kBK * 2;
    static_assert((!FP8A && !F8C) || nslab == 2, "FP8 weights are for the expert GEMMs");
    const int SA8 = FP8A ? args.stages_a8 : 0;
    constexpr uint32_t a8_bytes = nslab * code_slab_bytes(OPS);
    uint8_t* ring_a = smem;                                  // [SA][nslab][128 x 64] bf16
    uint8_t* ring_b = ring_a + SA * a_bytes;                 // [SB][n_max x 64] bf16
    uint8_t* ring8 = ring_b + SB * b_bytes;                  // [SA8][nslab][code slab]
    bf16* staging = reinterpret_cast<bf16*>(ring8 + SA8 * a8_bytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(ring8 + SA8 * a8_bytes + kStagingBytes);
    uint64_t* empty = full + SA;
    uint64_t* acc_full = empty + SA;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* full8 = drain + 1;                             // [SA8] codes landed
    uint64_t* empty8 = full8 + SA8;                          // [SA8] codes converted
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(empty8 + SA8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            ptx::mbar_init(&full[s], 2);     // weight producer + token producer
            ptx::mbar_init(&empty[s], 1);    // one commit of the MMA thread
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], FP8A ? kEpiWarpsFP8 : kEpiWarps);
        }
        ptx::mbar_init(drain, 1);
        for (int s = 0; s < SA8; ++s) {
            ptx::mbar_init(&full8[s], 1);    // the weight producer's codes
            ptx::mbar_init(&empty8[s], 1);   // converter thread 0, after all converted
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&args.a_map[0]);
        ptx::prefetch_tensormap(&args.a_map[1]);
        ptx::prefetch_tensormap(&args.b_map[0]);
        ptx::prefetch_tensormap(&args.b_map[1]);
        ptx::prefetch_tensormap(&args.b_map64[0]);
        ptx::prefetch_tensormap(&args.b_map64[1]);
        if (FP8A) ptx::prefetch_tensormap(&args.a8_map);
        if (kInt4) ptx::prefetch_tensormap(&args.a4s_map);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    // the prologue above touches only this CTA's shared memory and TMEM: it may
    // overlap the previous kernel on the stream; its results are read below
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();

    const int ntiles = args.tiles != nullptr ? *args.ntiles_dev : args.ntiles_host;
    const uint64_t tmo = args.timeout_ns;

    if (warp == 0 || warp == kTokenWarp) {
        // ----------------------------------------------------------- producers
        if (lane == 0) {
            const bool weights = (warp == 0);
            // weights are streamed once; token rows are re-read by the next tiles
            const uint64_t pol = weights ? ptx::policy_evict_first() : ptx::policy_evict_last();
            Ring rq{0, 0, SA};          // K step q: its full barrier / weight slot
            Ring rb{0, 0, SB};          // token slot of step q
            Ring rp{0, 0, SA};          // step q - SB, whose MMAs free token slot q % SB
            Ring r8{0, 0, SA8};         // FP8 code slot of the routed steps
            uint32_t q = 0;
            uint32_t issued = 0, issued_parity = 0;             // per-barrier bits, for draining
            uint32_t issued8 = 0, issued8_parity = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
                const Tile t = load_tile(args, i);
                const int npad = pad16(t.n);
                const uint32_t tx = weights ? a_bytes : npad * kBK * 2;
                for (int ks = t.ks0; ks < t.ks1; ++ks, ++q) {
                    if (FP8A && weights) {
                        // every step takes a code slot: a routed step's codes go
                        // into it, a shared-expert step only completes its phase
                        // (the converter group loads that step's bf16 weights); the
                        // converter warps fill and publish the bf16 slot
                        if (!wait_bounded(&empty8[r8.stage], r8.phase ^ 1, abort_flag, tmo)) {
                            ok = false;
                            break;
                        }
                        if (t.map != 0) {
                            ptx::mbar_arrive(&full8[r8.stage]);
                            r8.next();
                            rq.next();
                            rb.next();
                            continue;
                        }
                        uint64_t* bar8 = &full8[r8.stage];
                        ptx::mbar_arrive_expect_tx(bar8, a8_bytes);
                        uint8_t* s8 = ring8 + r8.stage * a8_bytes;
                        if constexpr (kInt4) {
                            // per slab: 128 rows x 32 code bytes, then 2 groups x 128 scales
                            ptx::tma_load_2d_hint(s8, &args.a8_map, bar8, ks * (kBK / 2), t.a_row0,
                                                  pol);
                            ptx::tma_load_2d_hint(s8 + kSlabCodes4, &args.a4s_map, bar8, t.a_row0,
                                                  ks * (kBK / kInt4Group), pol);
                            ptx::tma_load_2d_hint(s8 + kSlabBytes4, &args.a8_map, bar8,
                                                  ks * (kBK / 2), t.a_row1, pol);
                            ptx::tma_load_2d_hint(s8 + kSlabBytes4 + kSlabCodes4, &args.a4s_map,
                                                  bar8, t.a_row1, ks * (kBK / kInt4Group), pol);
                        } else {
                            ptx::tma_load_2d_hint(s8, &args.a8_map, bar8, ks * kBK, t.a_row0, pol);
                            ptx::tma_load_2d_hint(s8 + kSlabBytes8, &args.a8_map, bar8, ks * kBK,
                                                  t.a_row1, pol);
                        }
                        issued8 |= 1u << r8.stage;
                        issued8_parity = (issued8_parity & ~(1u << r8.stage)) | (r8.phase << r8.stage);
                        r8.next();
                        rq.next();
                        rb.next();
                        continue;
                    }
                    bool free_ok;
                    if (weights) {
                        // weight slot is free once the MMAs of step q - SA are done
                        free_ok = wait_bounded(&empty[rq.stage], rq.phase ^ 1, abort_flag, tmo);
                    } else if (q >= static_cast<uint32_t>(SB)) {
                        free_ok = wait_bounded(&empty[rp.stage], rp.phase, abort_flag, tmo);
                        rp.next();
                    } else {
                        free_ok = true;
                    }
                    if (!free_ok) {
                        ok = false;
                        break;
                    }
                    uint64_t* bar = &full[rq.stage];
                    ptx::mbar_arrive_expect_tx(bar, tx);
                    if (weights) {
                        uint8_t* sa = ring_a + rq.stage * a_bytes;
                        const CUtensorMap* am = &args.a_map[t.map];
                        ptx::tma_load_2d_hint(sa, am, bar, ks * kStepK, t.a_row0, pol);
                        if (nslab == 2)
                            ptx::tma_load_2d_hint(sa + kSlabBytes, am, bar, ks * kStepK, t.a_row1,
                                                  pol);
                    } else {
                        uint8_t* sb = ring_b + rb.stage * b_bytes;
                        int r = 0;
                        for (; r + kBoxRowsBig <= npad; r += kBoxRowsBig)
                            ptx::tma_load_2d_hint(sb + r * kBK * 2, &args.b_map64[t.map], bar,
                                                  ks * kStepK, t.b_row0 + r, pol);
                        for (; r < npad; r += kBoxRows)
                            ptx::tma_load_2d_hint(sb + r * kBK * 2, &args.b_map[t.map], bar,
                                                  ks * kStepK, t.b_row0 + r, pol);
                    }
                    issued |= 1u << rq.stage;
                    issued_parity = (issued_parity & ~(1u << rq.stage)) | (rq.phase << rq.stage);
                    rq.next();
                    rb.next();
                }
            }
            if (!ok) {
                // let every copy this thread started land before the CTA exits (a
                // phase the other producer never joined runs out the bounded wait)
                for (int s = 0; s < SA; ++s)
                    if (issued & (1u << s))
                        wait_bounded(&full[s], (issued_parity >> s) & 1, nullptr, tmo);
                for (int s = 0; s < SA8; ++s)
                    if (issued8 & (1u << s))
                        wait_bounded(&full8[s], (issued8_parity >> s) & 1, nullptr, tmo);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            Ring ra{0, 0, SA}, rb{0, 0, SB};   // K step q: weight slot q % SA, token slot q % SB
            const uint64_t desc_ring_a = ptx::sdesc_k_sw128(ptx::smem_u32(ring_a));
            const uint64_t desc_ring_b = ptx::sdesc_k_sw128(ptx::smem_u32(ring_b));
            uint32_t ab = 0, aphase = 0;
            bool ok = true, any = false;
            for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
                const Tile t = load_tile(args, i);
                const int npad = pad16(t.n);
                const uint32_t idesc = F8C ? ptx::idesc_e4m3_f32(kSlabRows, npad)
                                           : ptx::idesc_bf16_f32(kSlabRows, npad);
                // single-slab tiles of 32+ tokens: two N halves (multiples of 16)
                const int n_lo = (nslab == 1 && npad >= 32) ? pad16(npad / 2) : npad;
                const int n_hi = npad - n_lo;
                const uint32_t idesc_lo = ptx::idesc_bf16_f32(kSlabRows, n_lo);
                const uint32_t idesc_hi = n_hi > 0 ? ptx::idesc_bf16_f32(kSlabRows, n_hi) : idesc;
                if (!wait_bounded(&acc_empty[ab], aphase ^ 1, abort_flag, tmo)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dcol = tmem_base + ab * args.acc_stride;
                for (int ks = t.ks0; ks < t.ks1; ++ks) {
                    if (!wait_bounded(&full[ra.stage], ra.phase, abort_flag, tmo)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    // Consecutive MMAs alternate between two independent accumulators
                    // (the two slabs, or the two N halves of a single-slab tile): back-
                    // to-back MMAs into one accumulator wait on each other.  The
                    // descriptors' start-address field holds (address >> 4), so a slot,
                    // slab or K offset of B bytes is an addition of B >> 4 (one MMA's K,
                    // 16 bf16 or 32 E4M3 elements = 32 B, is +2); shared addresses stay
                    // below 2^18.
                    const uint64_t a0 = desc_ring_a + ra.stage * (a_bytes >> 4);
                    const uint64_t a1 = a0 + (kSlabBytes >> 4);
                    const uint64_t b0 = desc_ring_b + rb.stage * (b_bytes >> 4);
                    const uint64_t b1 = b0 + ((n_lo * kBK * 2) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t acc = (ks > t.ks0 || kk > 0) ? 1u : 0u;
                        if (F8C) {
                            ptx::tc_mma_e4m3(dcol, a0 + 2 * kk, b0 + 2 * kk, idesc, acc);
                            ptx::tc_mma_e4m3(dcol + args.n_max, a1 + 2 * kk, b0 + 2 * kk, idesc, acc);
                        } else if (nslab == 2) {
                            ptx::tc_mma_bf16(dcol, a0 + 2 * kk, b0 + 2 * kk, idesc, acc);
                            ptx::tc_mma_bf16(dcol + args.n_max, a1 + 2 * kk, b0 + 2 * kk, idesc, acc);
                        } else if (n_hi > 0) {
                            ptx::tc_mma_bf16(dcol, a0 + 2 * kk, b0 + 2 * kk, idesc_lo, acc);
                            ptx::tc_mma_bf16(dcol + n_lo, a0 + 2 * kk, b1 + 2 * kk, idesc_hi, acc);
                        } else {
                            ptx::tc_mma_bf16(dcol, a0 + 2 * kk, b0 + 2 * kk, idesc, acc);
                        }
                    }
                    any = true;
                    ptx::tc_commit(&empty[ra.stage]);
                    ra.next();
                    rb.next();
                }
                if (!ok) break;
                ptx::tc_commit(&acc_full[ab]);
                if (++ab == static_cast<uint32_t>(args.acc_bufs)) {
                    ab = 0;
                    aphase ^= 1;
                }
            }
            if (!ok && any) {
                // no MMA may still be writing TMEM when it is freed
                ptx::tc_commit(drain);
                wait_bounded(drain, 0, nullptr, tmo);
            }
        }
    } else if (FP8A && warp >= 2 + kEpiWarpsFP8) {
        // ---------------------------------------------------------- converters
        // group 0: warps 6..9, group 1: warps 11..14 (one warp per sub-partition each)
        if constexpr (FP8A) {
            const int grp = warp < kTokenWarp ? 0 : 1;
            convert_weights<nslab, OPS>(args, ring8, ring_a, SA, SA8, full, empty, full8, empty8,
                                        abort_flag, tmo, ntiles, grp,
                                        32 * (warp - (grp == 0 ? 6 : 11)) + lane);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        // which 32-column chunks the warp takes: every other one when two warps
        // share a lane quarter (bf16 mode), all of them in FP8 mode
        const int half = FP8A ? 0 : (warp - 2) >> 2;
        constexpr int kChunkStep = FP8A ? kStageRows : 2 * kStageRows;
        bf16* stg = staging + (warp - 2) * kStageRows * 32;
        uint32_t ab = 0, aphase = 0;
        for (int i = blockIdx.x; i < ntiles; i += gridDim.x) {
            const Tile t = load_tile(args, i);
            const int npad = pad16(t.n);
            if (!wait_bounded_warp(&acc_full[ab], aphase, abort_flag, tmo)) break;
            ptx::tc_fence_after();
            bool released = false;      // acc_empty already arrived on for this tile
            const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                ab * args.acc_stride;
            if constexpr (EPI == kEpiStoreF32) {
                // lane = output feature: 32 lanes write 128 contiguous bytes per token
                const int f = t.out_col0 + q * 32 + lane;
                const bool fok = f < args.col_limit;
                float* out = static_cast<float*>(args.out) + f;
                for (int c0 = 16 * half; c0 < npad; c0 += 32) {
                    uint32_t v[16];
                    ptx::tmem_ld_x16(tq + c0, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int r = c0 + j;
                        if (r < t.n && fok)
                            out[(long long)(t.out_row0 + r) * args.out_ld] = __uint_as_float(v[j]);
                    }
                }
            } else {
                constexpr bool kSwiGLU = (EPI == kEpiSwiGLU);
                const int nout = kSwiGLU ? 1 : nslab;
                bf16* out = static_cast<bf16*>(args.out);
                // FP8 compute: this lane's weight row exponents (gate and up rows, or
                // the row of each output slab) and the tile's token row exponents
                [[maybe_unused]] const int8_t* bexp = F8C ? args.b_exp[t.map] + t.b_row0 : nullptr;
                int ew0 = 0, ew1 = 0;
                if constexpr (F8C) {
                    const int8_t* aexp = args.a_exp[t.map];
                    const int f0 = t.out_col0 + q * 32 + lane;
                    if (kSwiGLU || f0 < args.col_limit) ew0 = aexp[t.a_row0 + q * 32 + lane];
                    if (kSwiGLU || f0 + kSlabRows < args.col_limit)
                        ew1 = aexp[t.a_row1 + q * 32 + lane];
                }
                // Single-buffered accumulator (tiles of more than 128 tokens): the
                // SwiGLU epilogue first takes all of its warp's columns out of TMEM
                // (h rounded to bf16, two per register), frees the accumulator for
                // the next tile's MMAs, and only then stores.
                if constexpr (kSwiGLU && !FP8A) {
                    if (args.acc_bufs == 1) {
                        constexpr int kMaxChunks = (kMaxN + kChunkStep - 1) / kChunkStep;
                        uint32_t pk[kMaxChunks][kStageRows / 2];
#pragma unroll
                        for (int ci = 0; ci < kMaxChunks; ++ci) {
                            const int c0 = kStageRows * half + ci * kChunkStep;
                            if (c0 >= npad) continue;
                            [[maybe_unused]] const int ex =
                                F8C ? (c0 + lane < t.n ? bexp[c0 + lane] : 0) : 0;
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                if (c0 + 16 * hh >= npad) continue;
                                uint32_t g[16], u[16];
                                ptx::tmem_ld_x16(tq + c0 + 16 * hh, g);
                                ptx::tmem_ld_x16(tq + args.n_max + c0 + 16 * hh, u);
                                ptx::tmem_wait_ld();
#pragma unroll
                                for (int j = 0; j < 16; j += 2) {
                                    float v0, v1;
                                    if constexpr (F8C) {
                                        const int e0 = __shfl_sync(0xffffffffu, ex, 16 * hh + j);
                                        const int e1 = __shfl_sync(0xffffffffu, ex, 16 * hh + j + 1);
                                        v0 = silu_fast(mul_pow2(__uint_as_float(g[j]), ew0 + e0)) *
                                             mul_pow2(__uint_as_float(u[j]), ew1 + e0);
                                        v1 = silu_fast(mul_pow2(__uint_as_float(g[j + 1]), ew0 + e1)) *
                                             mul_pow2(__uint_as_float(u[j + 1]), ew1 + e1);
                                    } else {
                                        v0 = silu_fast(__uint_as_float(g[j])) * __uint_as_float(u[j]);
                                        v1 = silu_fast(__uint_as_float(g[j + 1])) *
                                             __uint_as_float(u[j + 1]);
                                    }
                                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
                                    pk[ci][8 * hh + j / 2] = *reinterpret_cast<const uint32_t*>(&b2);
                                }
                            }
                        }
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
                        released = true;
#pragma unroll
                        for (int ci = 0; ci < kMaxChunks; ++ci) {
                            const int c0 = kStageRows * half + ci * kChunkStep;
                            if (c0 >= npad) continue;
                            const int ncol = min(kStageRows, npad - c0);
                            store_block_packed(stg, pk[ci], ncol, out, args.out_ld, t.out_row0 + c0,
                                               min(ncol, t.n - c0), t.out_col0 + q * 32,
                                               args.col_limit, lane);
                        }
                    }
                }
                for (int s = 0; s < nout && !released; ++s) {
                    const int fbase = t.out_col0 + s * kSlabRows + q * 32;
                    const uint32_t ts = tq + s * args.n_max;
                    [[maybe_unused]] const int ews = s == 0 ? ew0 : ew1;
                    for (int c0 = kStageRows * half; c0 < npad; c0 += kChunkStep) {
                        const int ncol = min(kStageRows, npad - c0);     // 32 or 16 (uniform)
                        float v[kStageRows];
                        if constexpr (kSwiGLU) {
                            uint32_t g[kStageRows], u[kStageRows];
                            if (ncol == kStageRows) {
                                ptx::tmem_ld_x32(ts + c0, g);
                                ptx::tmem_ld_x32(ts + args.n_max + c0, u);
                            } else {
                                ptx::tmem_ld_x16(ts + c0, *reinterpret_cast<uint32_t(*)[16]>(g));
                                ptx::tmem_ld_x16(ts + args.n_max + c0,
                                                 *reinterpret_cast<uint32_t(*)[16]>(u));
                            }
                            ptx::tmem_wait_ld();
                            if constexpr (F8C) {
                                const int ex = c0 + lane < t.n ? bexp[c0 + lane] : 0;
#pragma unroll
                                for (int j = 0; j < kStageRows; ++j) {
                                    const int ej = __shfl_sync(0xffffffffu, ex, j);
                                    v[j] = silu_fast(mul_pow2(__uint_as_float(g[j]), ew0 + ej)) *
                                           mul_pow2(__uint_as_float(u[j]), ew1 + ej);
                                }
                            } else {
#pragma unroll
                                for (int j = 0; j < kStageRows; ++j)
                                    v[j] = silu_fast(__uint_as_float(g[j])) * __uint_as_float(u[j]);
                            }
                        } else {
                            uint32_t r[kStageRows];
                            if (ncol == kStageRows)
                                ptx::tmem_ld_x32(ts + c0, r);
                            else
                                ptx::tmem_ld_x16(ts + c0, *reinterpret_cast<uint32_t(*)[16]>(r));
                            ptx::tmem_wait_ld();
                            if constexpr (F8C) {
                                const int ex = c0 + lane < t.n ? bexp[c0 + lane] : 0;
#pragma unroll
                                for (int j = 0; j < kStageRows; ++j)
                                    v[j] = mul_pow2(__uint_as_float(r[j]),
                                                    ews + __shfl_sync(0xffffffffu, ex, j));
                            } else {
#pragma unroll
                                for (int j = 0; j < kStageRows; ++j) v[j] = __uint_as_float(r[j]);
                            }
                        }
                        store_block_bf16(stg, v, ncol, out, args.out_ld, t.out_row0 + c0,
                                         min(ncol, t.n - c0), fbase, args.col_limit, lane);
                    }
                }
            }
            if (!released) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
            }
            if (++ab == static_cast<uint32_t>(args.acc_bufs)) {
                ab = 0;
                aphase ^= 1;
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Dynamic shared memory the kernel needs for a configuration (code_slab: the
// bytes of one weight slab per K step in the code ring of a converting mode).
inline size_t gemm_smem_bytes(int stages_a, int stages_b, int nslab, int n_max, int stages_a8 = 0,
                              int code_slab = kSlabBytes8) {
    const size_t a = static_cast<size_t>(nslab) * kSlabBytes;
    const size_t b = static_cast<size_t>(n_max) * kBK * 2;
    const size_t a8 = static_cast<size_t>(nslab) * code_slab;
    return 1024 /* alignment slack */ + stages_a * a + stages_b * b + stages_a8 * a8 +
           kStagingBytes + (2 * stages_a + 2 * stages_a8 + 5) * 8 + 16;
}

}  // namespace moe
