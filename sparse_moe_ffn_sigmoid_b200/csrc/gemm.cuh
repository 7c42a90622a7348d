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
// Roles inside a 192-thread CTA (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer   (one lane): A slab(s) 128x64 + B rows Nx64 per stage
//   warp 1      MMA issuer     (one lane): 4 x tcgen05.mma (K=16) per slab per stage;
//               the whole warp allocates / frees the 512 TMEM columns
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 16 columns, convert, store
// Stages are guarded by full/empty mbarriers; accumulators (1 or 2 buffers)
// by acc_full/acc_empty.  Every wait is bounded (see wait_bounded).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kBK = 64;                       // K elements per pipeline stage (128 B rows)
constexpr int kSlabRows = 128;                // MMA M
constexpr int kSlabBytes = kSlabRows * kBK * 2;
constexpr int kBoxRows = 16;                  // TMA box height for token rows
constexpr int kMaxN = 256;                    // MMA N limit
constexpr int kGemmThreads = 192;
constexpr int kTmemCols = 512;

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
    int stages;
    int acc_bufs;             // accumulator buffers in TMEM (1 or 2)
    int acc_stride;           // TMEM columns per accumulator buffer
    unsigned long long timeout_ns;
};

__device__ __forceinline__ Tile load_tile(const GemmArgs& a, int i) {
    Tile t;
    if (a.tiles != nullptr) {
        const int4 v0 = a.tiles[2 * i];
        const int4 v1 = a.tiles[2 * i + 1];
        t.a_row0 = v0.x;
        t.a_row1 = v0.y;
        t.b_row0 = v0.z;
        t.n = v0.w & 0xFFFF;
        t.map = (v0.w >> 16) & 1;
        t.out_row0 = v1.x;
        t.out_col0 = v1.y;
        t.ks0 = v1.z;
        t.ks1 = v1.w;
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

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1) moe_gemm_kernel(const __grid_constant__ GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int S = args.stages;
    const int nslab = args.nslab;
    const uint32_t stage_bytes = nslab * kSlabBytes + args.n_max * kBK * 2;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&acc_full[b], 1);
            ptx::mbar_init(&acc_empty[b], 4);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&args.a_map[0]);
        ptx::prefetch_tensormap(&args.a_map[1]);
        ptx::prefetch_tensormap(&args.b_map[0]);
        ptx::prefetch_tensormap(&args.b_map[1]);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int ntiles = args.tiles != nullptr ? *args.ntiles_dev : args.ntiles_host;
    const uint64_t tmo = args.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = ptx::policy_evict_first();   // weights: streamed once
            const uint64_t pol_x = ptx::policy_evict_last();    // tokens: re-read by tiles
            uint32_t stage = 0, phase = 0;
            uint32_t issued = 0, issued_parity = 0;             // per-stage bits, for draining
            bool ok = true;
            for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
                const Tile t = load_tile(args, i);
                const int npad = pad16(t.n);
                const uint32_t tx = nslab * kSlabBytes + npad * kBK * 2;
                const CUtensorMap* am = &args.a_map[t.map];
                const CUtensorMap* bm = &args.b_map[t.map];
                for (int ks = t.ks0; ks < t.ks1; ++ks) {
                    if (!wait_bounded(&empty[stage], phase ^ 1, abort_flag, tmo)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + stage * stage_bytes;
                    uint8_t* sb = sa + nslab * kSlabBytes;
                    ptx::mbar_arrive_expect_tx(&full[stage], tx);
                    ptx::tma_load_2d_hint(sa, am, &full[stage], ks * kBK, t.a_row0, pol_w);
                    if (nslab == 2)
                        ptx::tma_load_2d_hint(sa + kSlabBytes, am, &full[stage], ks * kBK,
                                              t.a_row1, pol_w);
                    for (int r = 0; r < npad; r += kBoxRows)
                        ptx::tma_load_2d_hint(sb + r * kBK * 2, bm, &full[stage], ks * kBK,
                                              t.b_row0 + r, pol_x);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == static_cast<uint32_t>(S)) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // let every copy this thread started land before the CTA exits
                for (int s = 0; s < S; ++s)
                    if (issued & (1u << s))
                        wait_bounded(&full[s], (issued_parity >> s) & 1, nullptr, tmo);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, ab = 0, aphase = 0;
            bool ok = true, any = false;
            for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
                const Tile t = load_tile(args, i);
                const int npad = pad16(t.n);
                const uint32_t idesc = ptx::idesc_bf16_f32(kSlabRows, npad);
                if (!wait_bounded(&acc_empty[ab], aphase ^ 1, abort_flag, tmo)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dcol = tmem_base + ab * args.acc_stride;
                for (int ks = t.ks0; ks < t.ks1; ++ks) {
                    if (!wait_bounded(&full[stage], phase, abort_flag, tmo)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sa = ptx::smem_u32(smem + stage * stage_bytes);
                    const uint32_t sb = sa + nslab * kSlabBytes;
                    for (int s = 0; s < nslab; ++s) {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint64_t ad = ptx::sdesc_k_sw128(sa + s * kSlabBytes + kk * 32);
                            const uint64_t bd = ptx::sdesc_k_sw128(sb + kk * 32);
                            ptx::tc_mma_bf16(dcol + s * args.n_max, ad, bd, idesc,
                                             (ks > t.ks0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    any = true;
                    ptx::tc_commit(&empty[stage]);
                    if (++stage == static_cast<uint32_t>(S)) {
                        stage = 0;
                        phase ^= 1;
                    }
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
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter of this warp
        uint32_t ab = 0, aphase = 0;
        for (int i = blockIdx.x; i < ntiles; i += gridDim.x) {
            const Tile t = load_tile(args, i);
            const int npad = pad16(t.n);
            if (!wait_bounded(&acc_full[ab], aphase, abort_flag, tmo)) break;
            ptx::tc_fence_after();
            const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                ab * args.acc_stride;
            if constexpr (EPI == kEpiSwiGLU) {
                const int f = t.out_col0 + q * 32 + lane;
                const bool fok = f < args.col_limit;
                bf16* out = static_cast<bf16*>(args.out) + f;
                for (int c0 = 0; c0 < npad; c0 += 16) {
                    uint32_t g[16], u[16];
                    ptx::tmem_ld_x16(tq + c0, g);
                    ptx::tmem_ld_x16(tq + args.n_max + c0, u);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int r = c0 + j;
                        if (r < t.n && fok) {
                            const float gv = __uint_as_float(g[j]);
                            const float uv = __uint_as_float(u[j]);
                            out[(long long)(t.out_row0 + r) * args.out_ld] =
                                __float2bfloat16_rn(silu_f32(gv) * uv);
                        }
                    }
                }
            } else if constexpr (EPI == kEpiStoreBF16) {
                for (int s = 0; s < nslab; ++s) {
                    const int f = t.out_col0 + s * kSlabRows + q * 32 + lane;
                    const bool fok = f < args.col_limit;
                    bf16* out = static_cast<bf16*>(args.out) + f;
                    for (int c0 = 0; c0 < npad; c0 += 16) {
                        uint32_t v[16];
                        ptx::tmem_ld_x16(tq + s * args.n_max + c0, v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int r = c0 + j;
                            if (r < t.n && fok)
                                out[(long long)(t.out_row0 + r) * args.out_ld] =
                                    __float2bfloat16_rn(__uint_as_float(v[j]));
                        }
                    }
                }
            } else {
                const int f = t.out_col0 + q * 32 + lane;
                const bool fok = f < args.col_limit;
                float* out = static_cast<float*>(args.out) + f;
                for (int c0 = 0; c0 < npad; c0 += 16) {
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
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
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

// Dynamic shared memory the kernel needs for a configuration.
inline size_t gemm_smem_bytes(int stages, int nslab, int n_max) {
    const size_t stage = static_cast<size_t>(nslab) * kSlabBytes + static_cast<size_t>(n_max) * kBK * 2;
    return 1024 /* alignment slack */ + stages * stage + (2 * stages + 5) * 8 + 16;
}

}  // namespace moe
