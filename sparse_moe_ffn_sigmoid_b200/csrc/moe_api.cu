// moe_api.cu -- the C ABI of include/moe.h: argument checks, scratch layout,
// TMA descriptors and the launch sequence of the MoE layer forward pass.
//
// Everything here is host code except the kernels it includes; it is built
// as one translation unit (kernels in the *.cuh files next to it).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "moe.h"
#include "combine.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "gemv.cuh"
#include "balance.cuh"
#include "ep.cuh"
#include "permute.cuh"
#include "route.cuh"

// Scratch of moe_layer_forward_noalloc: a fixed array in the library's device
// image, so that entry point never allocates.  Host code must not use this
// name as an address (on the host it is only a stand-in); noalloc_scratch()
// obtains the device address with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_moe_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace moe {
namespace {

constexpr int kTargetCtas = 148;          // SMs of a B200: the router's split heuristic
constexpr int kMaxSplits = 64;
constexpr size_t kMaxDynSmem = 232448;    // 227 KB opt-in per block on sm_100
constexpr size_t kScanSmem = 200 * 1024;  // shared memory for the scan's block counts
constexpr int kTopkBlockTokens = 512;      // top-k launch shape switch (tokens per call)
// Token rows are permuted token by token (each x row read once, written to its
// k rows) from this many tokens on; below it, row by row (one warp per permuted
// row: more warps for a small batch).  Measured on B200: token by token cuts the
// prefill gather from 0.26 to 0.24 ms (bf16) and the FP8 token quantization from
// 0.27 to 0.17 ms, but is slower at decode (64 warps: 16 us against 9 us).
constexpr int kTokenMajorMinT = 1024;

std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_last_launches{0};

// The last CUDA failure this thread met inside the library (moe_last_error_string).
thread_local char t_last_error[256] = "no error";

int record_cuda_failure(const char* where, const char* what) {
    std::snprintf(t_last_error, sizeof(t_last_error), "%s: %s", where, what);
    return MOE_ERR_CUDA;
}

// MOE_OK, or MOE_ERR_CUDA with the launch error recorded, after kernel launches.
int launch_rc(const char* where) {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : record_cuda_failure(where, cudaGetErrorString(e));
}

// Programmatic dependent launch of the library's kernels (moe_set_pdl): each
// kernel may be scheduled while the previous kernel on the stream finishes and
// runs its set-up meanwhile; every kernel waits (griddep_wait) before it reads
// what earlier kernels wrote.
std::atomic<int> g_pdl{0};

// Only a kernel whose predecessor on the stream is this library's previous
// kernel of the same call gets the attribute: the first kernel of every call
// waits for whatever the stream held before (other libraries' kernels, copies).
thread_local bool t_after_own_kernel = false;

struct CallScope {
    CallScope() { t_after_own_kernel = false; }
};

template <typename... KArgs, typename... Args>
void launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
            Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (g_pdl.load() && t_after_own_kernel) ? 1 : 0;
    // a failed launch is left in the thread's error state for launch_rc
    (void)cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    t_after_own_kernel = true;
}

// Kernels of one layer call, in launch order (moe_kernel_name).  gather_rows
// also quantizes the rows in FP8 compute; quantize_h (the activation rows'
// FP8 quantization) runs in FP8 compute only.
constexpr int kLayerKernels = 10;
const char* const kKernelNames[kLayerKernels] = {
    "router_gemm", "topk", "permute_hist", "scan_plan", "permute_scatter",
    "gather_rows", "gemm_gate_up_swiglu", "quantize_h", "gemm_down", "combine"};

// Optional per-kernel CUDA-event timing of layer calls (moe_profile_begin/end).
struct Profile {
    std::mutex mu;
    std::vector<cudaEvent_t> ev;   // [calls][kLayerKernels + 1]
    int max_calls = 0;
    int calls = 0;
} g_prof;

// Counts the kernels a call launches and, when a profile slot is given,
// records an event on the stream after each of them.
struct Recorder {
    cudaEvent_t* ev = nullptr;     // kLayerKernels + 1 events, or null
    int n = 0;                     // slots passed
    int launches = 0;              // kernels launched
    void start(cudaStream_t st) {
        if (ev) cudaEventRecord(ev[0], st);
    }
    void mark(cudaStream_t st) {
        ++launches;
        skip(st);
    }
    // a kernel launched inside a slot that a later mark() closes
    void count() { ++launches; }
    // a slot this call has no kernel for (it times as zero)
    void skip(cudaStream_t st) {
        ++n;
        if (ev && n <= kLayerKernels) cudaEventRecord(ev[n], st);
    }
};

// ------------------------------------------------------------------ checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(int T, int d, int E, int k, int inter) {
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d < 64 || d % 64 != 0 || inter < 64 || inter % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(T) * (k + 1) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(E) * 2 * inter >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(E) * d >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

template <typename... P>
bool all_ok(P... p) {
    return ((p != nullptr && aligned16(p)) && ...);
}

// ------------------------------------------------------------------ layout

// K splits of the router GEMM: more splits fill more SMs when T is small, but
// every split adds one fp32 [T, E] partial that is written and read back.
// Cost model in microseconds: ~0.9 us per 64-deep K step of a tile wave (the
// measured pace of a single-slab router tile on B200), and the partials at
// ~4 TB/s.
int router_splits(int T, int d, int E) {
    const int nt = (T + kMaxN - 1) / kMaxN;
    const int mslabs = (E + kSlabRows - 1) / kSlabRows;
    const int base = std::max(1, nt * mslabs);
    const int ks = d / kBK;
    const double partial_us = static_cast<double>(T) * E * 8.0 / 4e12 * 1e6;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= std::min(ks, kMaxSplits); ++s) {
        const int waves = (base * s + kTargetCtas - 1) / kTargetCtas;
        const double cost = waves * static_cast<double>((ks + s - 1) / s) * 0.9 + s * partial_us;
        if (cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

struct Layout {
    size_t partials, topk_idx, topk_w, blk, counts, offsets, row_token, slot_row;
    size_t tiles1, tiles2, ntiles, xperm, h, y;
    // FP8 compute: the token rows' codes live in xperm (T*k permuted rows, then
    // the T rows in token order); their exponents, the activation's codes and
    // its exponents in regions of their own
    size_t xexp, hq, hexp;
    size_t total;
    int splits, nblk, max_tiles1, max_tiles2;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Largest token tile of the expert GEMMs.  The shared expert's T rows make a
// 256-row tile whenever T >= 256, and the token ring is sized for the largest
// tile; when the routed experts average at most 64 rows (a balanced batch whose
// routed tiles stay far below 192 rows) the tiles are capped at 192 rows, which
// leaves the weight ring a fourth stage (measured on B200 at the DeepSeek-V3
// shape, T = 2048 and 256 experts: 4-5% faster; at 171 rows per expert and with
// skewed loads 192-row tiles were 5-6% slower: more tiles, each with its own
// epilogue wait).
int tile_rows(int T, int E, int k) {
    return (T > kTileN && static_cast<long long>(T) * k <= 64ll * E) ? 192 : kTileN;
}

// Decode-sized batches with INT4 or E4M3 routed weights run the register-
// dequantizing GEMMs of gemv.cuh (token tiles of 16 rows) when the routed experts
// average at most 4 rows and both contraction lengths are multiples of the
// format's step (256 for INT4, 128 for E4M3).
bool gemv_shape(int T, int E, int k) { return static_cast<long long>(T) * k <= 4ll * E; }

bool gemv_ok(int T, int d, int E, int k, int inter, bool int4) {
    const int step = gemv_step_k(int4 ? kGemvInt4 : kGemvFp8);
    return gemv_shape(T, E, k) && d % step == 0 && inter % step == 0;
}

Layout make_layout(int T, int d, int E, int k, int inter, bool fp8_compute = false) {
    Layout L{};
    // tile lists sized for the smallest token tiles any plan of this shape uses
    const int tn = gemv_shape(T, E, k) ? kGemvTileN : tile_rows(T, E, k);
    const size_t Tk = static_cast<size_t>(T) * k;
    const size_t rows = Tk + T;   // routed rows, then the shared expert's rows
    L.splits = router_splits(T, d, E);
    L.nblk = (T + kPermTokens - 1) / kPermTokens;
    const long long token_tiles = static_cast<long long>(Tk / tn) +
                                  std::min<long long>(E, static_cast<long long>(Tk)) + 1 +
                                  (T + tn - 1) / tn;
    L.max_tiles1 = static_cast<int>(token_tiles * ((inter + kSlabRows - 1) / kSlabRows));
    L.max_tiles2 = static_cast<int>(token_tiles * ((d + 2 * kSlabRows - 1) / (2 * kSlabRows)));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.partials = take(static_cast<size_t>(L.splits) * T * E * sizeof(float));
    L.topk_idx = take(Tk * sizeof(int));
    L.topk_w = take(Tk * sizeof(float));
    L.blk = take(static_cast<size_t>(std::max(L.nblk, 1)) * E * sizeof(int));
    L.counts = take(static_cast<size_t>(E) * sizeof(int));
    L.offsets = take(static_cast<size_t>(E + 2) * sizeof(int));
    L.row_token = take(Tk * sizeof(int));
    L.slot_row = take(Tk * sizeof(int));
    L.tiles1 = take(static_cast<size_t>(L.max_tiles1) * 2 * sizeof(int4));
    L.tiles2 = take(static_cast<size_t>(L.max_tiles2) * 2 * sizeof(int4));
    L.ntiles = take(4 * sizeof(int));
    L.xperm = take(Tk * d * sizeof(bf16));
    L.h = take(rows * inter * sizeof(bf16));
    L.y = take(rows * d * sizeof(bf16));
    if (fp8_compute) {
        L.xexp = take(rows);
        L.hq = take(rows * inter);
        L.hexp = take(rows);
    }
    L.total = off;
    return L;
}

// ------------------------------------------------------------- device info

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// Makes sure the calling thread has a current CUDA context before the
// library's driver calls (tensor-map encoding needs one): a thread whose first
// CUDA work is a call into this library may have none yet, and then the
// device's primary context is made current, as the runtime would on its first
// kernel launch.  A context the caller made current is left alone.
int bind_context(int dev) {
    static CtxGetCurrentFn get_current = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext ctx = nullptr;
    if (get_current == nullptr) return record_cuda_failure("cuCtxGetCurrent", "entry point not found");
    if (get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr) return MOE_OK;
    const cudaError_t e = cudaSetDevice(dev);
    return e == cudaSuccess ? MOE_OK : record_cuda_failure("cudaSetDevice", cudaGetErrorString(e));
}

int device_info(DeviceInfo* out) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return record_cuda_failure("cudaGetDevice", cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return record_cuda_failure("cudaGetDevice", "device index >= 64");
    const int brc = bind_context(dev);
    if (brc != MOE_OK) return brc;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return launch_rc("cudaDeviceGetAttribute");
        const int smem = static_cast<int>(kMaxDynSmem);
        const cudaFuncAttribute dyn = cudaFuncAttributeMaxDynamicSharedMemorySize;
        if (cudaFuncSetAttribute(moe_gemm_kernel<kEpiSwiGLU, kOpsBF16>, dyn, smem) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiStoreBF16, kOpsBF16>, dyn, smem) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiStoreF32, kOpsBF16>, dyn, smem) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiSwiGLU, kOpsW8Convert>, dyn, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiStoreBF16, kOpsW8Convert>, dyn, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiSwiGLU, kOpsW4Convert>, dyn, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiStoreBF16, kOpsW4Convert>, dyn, smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiSwiGLU, kOpsFP8>, dyn, smem) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemm_kernel<kEpiStoreBF16, kOpsFP8>, dyn, smem) != cudaSuccess ||
            cudaFuncSetAttribute(scan_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kScanSmem)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiSwiGLU, kGemvInt4>, dyn,
                                 gemv_smem_bytes(kGemvInt4)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiStoreBF16, kGemvInt4>, dyn,
                                 gemv_smem_bytes(kGemvInt4)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiSwiGLU, kGemvFp8>, dyn,
                                 gemv_smem_bytes(kGemvFp8)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiStoreBF16, kGemvFp8>, dyn,
                                 gemv_smem_bytes(kGemvFp8)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiSwiGLU, kGemvBF16>, dyn,
                                 gemv_smem_bytes(kGemvBF16)) != cudaSuccess ||
            cudaFuncSetAttribute(moe_gemv_kernel<kEpiStoreBF16, kGemvBF16>, dyn,
                                 gemv_smem_bytes(kGemvBF16)) != cudaSuccess)
            return launch_rc("cudaFuncSetAttribute");
        di.ready = true;
    }
    *out = di;
    return MOE_OK;
}

// ------------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn g_encode_driver = nullptr;

// cuTensorMapEncodeTiled, recording a failure for moe_last_error_string.
CUresult encode_recording(CUtensorMap* m, CUtensorMapDataType type, cuuint32_t rank, void* base,
                          const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                          const cuuint32_t* estr, CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                          CUtensorMapL2promotion l2, CUtensorMapFloatOOBfill oob) {
    const CUresult r = g_encode_driver(m, type, rank, base, dims, strides, box, estr, il, sw, l2, oob);
    if (r != CUDA_SUCCESS) {
        char what[192];
        std::snprintf(what, sizeof(what), "CUresult %d (base %p, dims %llu x %llu, box %u x %u)",
                      static_cast<int>(r), base, static_cast<unsigned long long>(dims[0]),
                      static_cast<unsigned long long>(rank > 1 ? dims[1] : 1), box[0],
                      rank > 1 ? box[1] : 1u);
        record_cuda_failure("cuTensorMapEncodeTiled", what);
    }
    return r;
}

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_driver = reinterpret_cast<EncodeTiledFn>(p);
    });
    if (g_encode_driver == nullptr) {
        record_cuda_failure("cuTensorMapEncodeTiled", "driver entry point not found");
        return nullptr;
    }
    return encode_recording;
}

// Row-major E4M3 code matrix [rows, cols] (uint8) read in boxes of 128 rows x
// 64 codes, unswizzled (the converter warps read it, not the tensor core).
bool make_map8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(kSlabRows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed INT4 codes [rows, cols / 2] (bytes) read in boxes of 128 rows x 32
// bytes (one K step), and their group scales [cols / 32, rows] (bf16, group-
// major) in boxes of 2 groups x 128 rows; both unswizzled (the converter warps
// read them).
bool make_map_int4(CUtensorMap* codes_map, CUtensorMap* scale_map, const void* codes,
                   const void* scales, uint64_t rows, uint64_t cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t cdims[2] = {cols / 2, rows};
    const cuuint64_t cstrides[1] = {cols / 2};
    const cuuint32_t cbox[2] = {static_cast<cuuint32_t>(kBK / 2), static_cast<cuuint32_t>(kSlabRows)};
    const cuuint64_t sdims[2] = {rows, cols / kInt4Group};
    const cuuint64_t sstrides[1] = {rows * sizeof(bf16)};
    const cuuint32_t sbox[2] = {static_cast<cuuint32_t>(kSlabRows),
                                static_cast<cuuint32_t>(kBK / kInt4Group)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(codes_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), cdims,
               cstrides, cbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
               CUDA_SUCCESS &&
           enc(scale_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(scales), sdims,
               sstrides, sbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
               CUDA_SUCCESS;
}

// Row-major E4M3 code matrix [rows, cols] (uint8) read in boxes of box_rows x
// 128 codes, 128-byte swizzled: the operand layout of the FP8-compute MMAs.
bool make_map_e4m3(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(2 * kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major bf16 matrix [rows, cols] read in boxes of box_rows x 64 columns,
// 128-byte swizzled (the layout the UMMA descriptors expect).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * sizeof(bf16)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of the decode-sized GEMMs (gemv.cuh): weight rows in boxes of 128 bytes x
// 16 rows with the 128-byte swizzle, as uint8 codes [rows, row_bytes] or bf16
// [rows, cols]; INT4 group scales [cols / 32, rows] bf16 in boxes of 16 rows x
// 8 groups (one 256-element step), unswizzled.
// Decode GEMM maps (gemv.cuh): 4-D views (x, row in half, half, expert) of a
// row-major stack of experts of expert_rows rows each.  half_rows > 0 (gate|up:
// the up rows sit half_rows = inter rows after the gate rows): boxes of 16
// rows x 2 halves, a unit's gate rows and the matching up rows in one box;
// half_rows = 0 (down): boxes of 32 rows.
bool make_map_gemv(CUtensorMap* m, CUtensorMapDataType type, size_t esize, const void* base,
                   uint64_t rows, uint64_t cols, uint64_t expert_rows, uint64_t half_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const uint64_t row_bytes = cols * esize;
    const uint64_t in_half = half_rows ? half_rows : expert_rows;
    const cuuint64_t dims[4] = {cols, in_half, half_rows ? 2u : 1u, rows / expert_rows};
    const cuuint64_t strides[3] = {row_bytes, in_half * row_bytes, expert_rows * row_bytes};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(kGemvRowBytes / esize), half_rows ? 16u : 32u,
                               half_rows ? 2u : 1u, 1u};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, type, 4, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// INT4 group scales [cols / 32, rows] bf16 as (row in half, half, expert,
// group): boxes of the same rows as make_map_gemv's x the 8 groups of a step,
// laid out [group][half][rows] in shared memory.
bool make_map_gemv_scales(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                          uint64_t expert_rows, uint64_t half_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const uint64_t in_half = half_rows ? half_rows : expert_rows;
    const cuuint64_t dims[4] = {in_half, half_rows ? 2u : 1u, rows / expert_rows, cols / kInt4Group};
    const cuuint64_t strides[3] = {in_half * sizeof(bf16), expert_rows * sizeof(bf16),
                                   rows * sizeof(bf16)};
    const cuuint32_t box[4] = {half_rows ? 16u : 32u, half_rows ? 2u : 1u, 1u,
                               static_cast<cuuint32_t>(gemv_step_k(kGemvInt4) / kInt4Group)};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- launches

// Ring depths: the token ring gets 3 slots (2 for tiles of <= 64 tokens, whose
// token rows are small), the weight ring every slot that is left, up to 8
// (measured on B200: a 3-slot token ring beat 2 slots on the prefill, skewed
// and DeepSeek-V3 shapes).
void fill_pipeline(GemmArgs& a, int nslab, int n_max) {
    a.nslab = nslab;
    a.n_max = n_max;
    const size_t a_bytes = static_cast<size_t>(nslab) * kSlabBytes;
    const size_t b_bytes = static_cast<size_t>(n_max) * kBK * 2;
    const size_t budget = kMaxDynSmem - 1024 - kStagingBytes - 512;
    a.stages_b = n_max <= 64 ? 2 : 3;
    const int sa = static_cast<int>((budget - a.stages_b * b_bytes) / a_bytes);
    a.stages_a = std::max(a.stages_b, std::min(sa, 8));   // the token ring is never deeper
    a.acc_stride = nslab * n_max;
    a.acc_bufs = (2 * a.acc_stride <= kTmemCols) ? 2 : 1;
    a.timeout_ns = g_timeout_ns.load();
}

// Converting expert GEMMs (FP8 or INT4 weights): a shallow bf16 ring between
// the converter warps and the MMAs, a deep code ring for the weight stream
// (code_slab bytes per slab and step), the token ring as in the bf16 kernel.
void fill_pipeline_fp8(GemmArgs& a, int n_max, int code_slab = kSlabBytes8) {
    fill_pipeline(a, 2, n_max);
    const size_t a_bytes = 2 * static_cast<size_t>(kSlabBytes);
    const size_t a8_bytes = 2 * static_cast<size_t>(code_slab);
    const size_t b_bytes = static_cast<size_t>(n_max) * kBK * 2;
    const size_t budget = kMaxDynSmem - 1024 - kStagingBytes - 1024;
    a.stages_b = (n_max <= 64 || n_max > 128) ? 2 : 3;
    // two converter groups work on alternating steps: at decode each gets two
    // bf16 slots
    a.stages_a = std::max(a.stages_b, n_max <= 64 ? 4 : n_max <= 128 ? 3 : 2);
    const size_t left = budget - a.stages_a * a_bytes - a.stages_b * b_bytes;
    a.stages_a8 = static_cast<int>(std::min<size_t>(12, left / a8_bytes));
}

template <int EPI, int OPS = kOpsBF16>
int launch_gemm(const GemmArgs& a, int grid, cudaStream_t st) {
    constexpr bool FP8A = ops_convert(OPS);
    const size_t smem = gemm_smem_bytes(a.stages_a, a.stages_b, a.nslab, a.n_max,
                                        FP8A ? a.stages_a8 : 0, code_slab_bytes(OPS));
    if (smem > kMaxDynSmem || (FP8A && a.stages_a8 < 2)) return MOE_ERR_UNSUPPORTED_SHAPE;
    launch(moe_gemm_kernel<EPI, OPS>, grid, FP8A ? kGemmThreadsFP8 : kGemmThreads, smem, st, a);
    return launch_rc(__func__);
}

// Router GEMM: fp32 logit partials [splits, T, E] (split-K over d).
int launch_router_gemm(const DeviceInfo& di, const bf16* x, const bf16* wr, int T, int d, int E,
                       float* partials, int splits, cudaStream_t st) {
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    const int nt = (T + kMaxN - 1) / kMaxN;
    const int chunk = (((T + nt - 1) / nt) + 15) & ~15;
    if (!make_map(&a.a_map[0], wr, E, d, kSlabRows) || !make_map(&a.b_map[0], x, T, d, kBoxRows) ||
        !make_map(&a.b_map64[0], x, T, d, kBoxRowsBig))
        return MOE_ERR_CUDA;
    a.a_map[1] = a.a_map[0];
    a.b_map[1] = a.b_map[0];
    a.b_map64[1] = a.b_map64[0];
    a.tiles = nullptr;
    a.dense_mslabs = (E + kSlabRows - 1) / kSlabRows;
    a.dense_ttiles = nt;
    a.dense_tchunk = chunk;
    a.dense_splits = splits;
    a.dense_T = T;
    a.dense_ksteps = d / kBK;
    a.ntiles_host = a.dense_mslabs * nt * splits;
    a.out = partials;
    a.out_ld = E;
    a.col_limit = E;
    fill_pipeline(a, 1, chunk);
    return launch_gemm<kEpiStoreF32>(a, std::min(a.ntiles_host, di.sms), st);
}

int launch_route(const DeviceInfo& di, const bf16* x, const bf16* wr, const float* bias, int T,
                 int d, int E, int k, float scale, int* idx, float* w, float* partials,
                 int splits, cudaStream_t st, Recorder& rec) {
    int rc = launch_router_gemm(di, x, wr, T, d, E, partials, splits, st);
    if (rc != MOE_OK) return rc;
    rec.mark(st);
    const int npl = (E + 31) / 32;
    const long long sstride = static_cast<long long>(T) * E;
    // a block per token while the batch is small (the partial sums then wait
    // on memory, not on selection throughput); a warp per token otherwise
    const bool per_block = T <= kTopkBlockTokens;
#define MOE_TOPK(N)                                                                              \
    do {                                                                                         \
        if (per_block)                                                                           \
            launch(topk_block_kernel<N>, T, 32 * (N), 0, st, partials, splits, sstride, T, E, k,  \
                   bias, scale, idx, w);                                                         \
        else                                                                                     \
            launch(topk_warp_kernel<N>, (T + 7) / 8, 256, 0, st, partials, splits, sstride, T, E, \
                   k, bias, scale, idx, w);                                                      \
    } while (0)
    if (npl <= 1) MOE_TOPK(1);
    else if (npl <= 2) MOE_TOPK(2);
    else if (npl <= 4) MOE_TOPK(4);
    else if (npl <= 8) MOE_TOPK(8);
    else if (npl <= 12) MOE_TOPK(12);
    else if (npl <= 16) MOE_TOPK(16);
    else if (npl <= 24) MOE_TOPK(24);
    else MOE_TOPK(32);
#undef MOE_TOPK
    rec.mark(st);
    return launch_rc(__func__);
}

int launch_permute(const int* idx, int T, int E, int k, int* counts, int* offsets, int* row_token,
                   int* slot_row, int* blk, const PlanArgs& plan, cudaStream_t st, Recorder& rec) {
    const int nblk = (T + kPermTokens - 1) / kPermTokens;
    launch(permute_hist_kernel, nblk, kPermTokens, 4 * E * sizeof(uint32_t), st, idx, T, E, k, blk);
    rec.mark(st);
    // block counts are staged in shared memory when they fit (prefill: 98 KB)
    const long long n = static_cast<long long>(nblk) * E;
    const int smem_counts = n * 4 <= static_cast<long long>(kScanSmem) ? static_cast<int>(n) : 0;
    launch(scan_plan_kernel, 1, 1024, smem_counts * 4, st, blk, nblk, E, counts, offsets, plan, smem_counts);
    rec.mark(st);
    launch(permute_scatter_kernel, nblk, kPermTokens, 8 * E * sizeof(uint32_t), st, idx, T, E, k, blk, row_token, slot_row);
    rec.mark(st);
    return launch_rc(__func__);
}

// Routed experts' weights stored as E4M3 codes with one int8 exponent per
// 128 x 128 block (quant.cuh): gate|up codes [E, 2I, d] + [E, 2I/128, d/128],
// down codes [E, d, I] + [E, d/128, I/128].
struct Fp8Experts {
    const uint8_t* gate_up;
    const int8_t* gate_up_exp;
    const uint8_t* down;
    const int8_t* down_exp;
};

// Routed experts' weights as INT4 (quant.cuh): gate|up codes [E, 2I, d/2] bytes +
// scales [d/32, E*2I] bf16; down codes [E, d, I/2] + scales [I/32, E*d].
struct Int4Experts {
    const uint8_t* gate_up;
    const bf16* gate_up_scale;
    const uint8_t* down;
    const bf16* down_scale;
};

// A second stream of the calling thread in the current context, with a fork
// and a join event: the decode GEMMs run the shared expert's tiles on it beside
// the routed tiles.  One per thread and context, so calls from several threads
// never share events; created on first use and kept for the process.
struct SideStream {
    unsigned long long ctx_id;
    cudaStream_t s;
    cudaEvent_t fork, join;
};
int side_stream(SideStream** out);

// gather + gate|up + down over a planned tile list.
//   rows_b0: rows of the permuted token matrix (T*k); h_rows / y rows: rows_b0 (+ T if shared)
//   f8 / i4: routed weights in FP8 or INT4 (then w_gate_up / w_down are unused),
//   or both null for bf16
int launch_ffn(const DeviceInfo& di, const bf16* x, const int* row_token, const int* slot_row,
               int T, int d, int E,
               int k, int inter, const bf16* w_gate_up, const bf16* w_down,
               const bf16* ws_gate_up, const bf16* ws_down, bool shared, bf16* xperm, bf16* h,
               bf16* y, const int4* tiles1, const int4* tiles2, const int* ntiles,
               int max_tiles1, int max_tiles2, cudaStream_t st, Recorder& rec,
               const Fp8Experts* f8 = nullptr, const Int4Experts* i4 = nullptr,
               int tile_n = kTileN, bool use_gemv = false) {
    if ((f8 != nullptr || i4 != nullptr) && !shared) return MOE_ERR_INVALID_ARG;
    if (use_gemv && i4 == nullptr && f8 == nullptr) return MOE_ERR_INVALID_ARG;
    const int rows_routed = T * k;
    const int rows_all = rows_routed + (shared ? T : 0);
    if (rows_routed > 0) {
        if (slot_row != nullptr && T >= kTokenMajorMinT)   // token by token: x rows read once
            launch(scatter_rows_kernel, (T + 7) / 8, 256, 0, st, x, slot_row, T, k, rows_routed, d, xperm);
        else
            launch(gather_rows_kernel, (rows_routed + 7) / 8, 256, 0, st, x, row_token, T, rows_routed, d, xperm);
        rec.mark(st);
    }
    if (use_gemv) {
        // register-dequantizing GEMMs (gemv.cuh) over the plan's 16-row token
        // tiles: the routed experts' tiles (INT4 or E4M3 codes), then the shared
        // expert's (bf16), whose tile range starts at ntiles[2] / ntiles[3]
        const int shared_tiles1 = ((T + kGemvTileN - 1) / kGemvTileN) * (inter / kSlabRows);
        const int shared_tiles2 = ((T + kGemvTileN - 1) / kGemvTileN) * (d / (2 * kSlabRows));
        const int wf = i4 ? kGemvInt4 : kGemvFp8;
        const int grid_r = gemv_ctas_per_sm(wf) * di.sms;
        const int grid_s = gemv_ctas_per_sm(kGemvBF16) * di.sms;   // a multiple of the split
        SideStream* side = nullptr;
        const int src = side_stream(&side);
        if (src != MOE_OK) return src;
        for (int gemm = 0; gemm < 2; ++gemm) {
            const bool gu = (gemm == 0);
            const uint64_t rows = gu ? static_cast<uint64_t>(E) * 2 * inter
                                     : static_cast<uint64_t>(E) * d;
            const int K = gu ? d : inter;
            GemvArgs v{};
            v.tiles = gu ? tiles1 : tiles2;
            v.first = nullptr;
            v.last = ntiles + (gu ? 2 : 3);
            v.exps = i4 ? nullptr : (gu ? f8->gate_up_exp : f8->down_exp);
            v.b[0] = gu ? (rows_routed > 0 ? xperm : x) : h;
            v.b[1] = gu ? x : h;
            v.out = gu ? h : y;
            v.out_ld = gu ? inter : d;
            v.K = K;
            v.col_limit = gu ? inter : d;
            v.timeout_ns = g_timeout_ns.load();
            // routed tiles: codes (and INT4 scales)
            const uint64_t half = gu ? static_cast<uint64_t>(inter) : 0;
            const uint64_t erows = gu ? 2ull * inter : static_cast<uint64_t>(d);
            v.expert_rows = static_cast<int>(erows);
            const bool maps_ok =
                i4 ? make_map_gemv(&v.a_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                                   gu ? i4->gate_up : i4->down, rows, K / 2, erows, half) &&
                         make_map_gemv_scales(&v.s_map, gu ? i4->gate_up_scale : i4->down_scale,
                                              rows, K, erows, half)
                   : make_map_gemv(&v.a_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                                   gu ? f8->gate_up : f8->down, rows, K, erows, half);
            if (!maps_ok) return record_cuda_failure(__func__, "tensor map encoding failed");
            const int grid1 = std::max(1, std::min(gu ? max_tiles1 : max_tiles2, grid_r));
            // fork: the shared expert's tiles (below) run on the side stream beside
            // the routed ones, which they neither read nor write (x or their own h
            // rows in, their own h or Y rows out); launched after the routed grid,
            // they take the SMs its last wave leaves idle
            if (cudaEventRecord(side->fork, st) != cudaSuccess ||
                cudaStreamWaitEvent(side->s, side->fork, 0) != cudaSuccess)
                return record_cuda_failure(__func__, cudaGetErrorString(cudaGetLastError()));
            if (wf == kGemvInt4) {
                if (gu)
                    launch(moe_gemv_kernel<kEpiSwiGLU, kGemvInt4>, grid1, gemv_threads(wf), gemv_smem_bytes(kGemvInt4), st, v);
                else
                    launch(moe_gemv_kernel<kEpiStoreBF16, kGemvInt4>, grid1, gemv_threads(wf), gemv_smem_bytes(kGemvInt4), st, v);
            } else {
                if (gu)
                    launch(moe_gemv_kernel<kEpiSwiGLU, kGemvFp8>, grid1, gemv_threads(wf), gemv_smem_bytes(kGemvFp8), st, v);
                else
                    launch(moe_gemv_kernel<kEpiStoreBF16, kGemvFp8>, grid1, gemv_threads(wf), gemv_smem_bytes(kGemvFp8), st, v);
            }
            rec.count();
            // the shared expert's tiles: bf16 weights
            if (!make_map_gemv(&v.a_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sizeof(bf16),
                               gu ? ws_gate_up : ws_down, erows, K, erows, half))
                return record_cuda_failure(__func__, "tensor map encoding failed");
            v.first = ntiles + (gu ? 2 : 3);
            v.last = ntiles + (gu ? 0 : 1);
            const int split = gemv_split(kGemvBF16);
            const int grid2 = std::max(1, std::min(gu ? shared_tiles1 : shared_tiles2, grid_s / split)) * split;
            t_after_own_kernel = false;     // first kernel on the side stream: fully ordered
            if (gu)
                launch(moe_gemv_kernel<kEpiSwiGLU, kGemvBF16>, grid2, gemv_threads(kGemvBF16), gemv_smem_bytes(kGemvBF16), side->s, v);
            else
                launch(moe_gemv_kernel<kEpiStoreBF16, kGemvBF16>, grid2, gemv_threads(kGemvBF16), gemv_smem_bytes(kGemvBF16), side->s, v);
            if (launch_rc(__func__) != MOE_OK) return MOE_ERR_CUDA;
            // join: the stream goes on once both halves of this GEMM are done
            if (cudaEventRecord(side->join, side->s) != cudaSuccess ||
                cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess)
                return record_cuda_failure(__func__, cudaGetErrorString(cudaGetLastError()));
            t_after_own_kernel = false;     // the next kernel follows an event wait
            rec.mark(st);
            if (gu) rec.skip(st);   // no activation quantization
        }
        return MOE_OK;
    }

    // largest token tile: an expert never holds more rows than its token count
    const int max_rows = shared ? T : rows_routed;
    const int n_max = std::min(tile_n, (max_rows + 15) & ~15);

    GemmArgs g1;
    std::memset(&g1, 0, sizeof(g1));
    const bf16* xp = rows_routed > 0 ? xperm : x;
    if (i4 != nullptr) {
        // routed tiles read codes and scales; slot 0 of the bf16 maps is never used
        if (!make_map_int4(&g1.a8_map, &g1.a4s_map, i4->gate_up, i4->gate_up_scale,
                           static_cast<uint64_t>(E) * 2 * inter, d) ||
            !make_map(&g1.a_map[0], ws_gate_up, 2ull * inter, d, kSlabRows))
            return MOE_ERR_CUDA;
    } else if (f8 != nullptr) {
        // routed tiles read codes; slot 0 of the bf16 maps is never used
        if (!make_map8(&g1.a8_map, f8->gate_up, static_cast<uint64_t>(E) * 2 * inter, d) ||
            !make_map(&g1.a_map[0], ws_gate_up, 2ull * inter, d, kSlabRows))
            return MOE_ERR_CUDA;
        g1.a8_scale = f8->gate_up_exp;
        g1.a8_kblocks = d / kQuantBlock;
    } else if (!make_map(&g1.a_map[0], w_gate_up, static_cast<uint64_t>(E) * 2 * inter, d,
                         kSlabRows)) {
        return MOE_ERR_CUDA;
    }
    if (!make_map(&g1.b_map[0], xp, std::max(rows_routed, 1), d, kBoxRows) ||
        !make_map(&g1.b_map[1], x, T, d, kBoxRows) ||
        !make_map(&g1.b_map64[0], xp, std::max(rows_routed, 1), d, kBoxRowsBig) ||
        !make_map(&g1.b_map64[1], x, T, d, kBoxRowsBig))
        return MOE_ERR_CUDA;
    if (shared) {
        if (!make_map(&g1.a_map[1], ws_gate_up, 2ull * inter, d, kSlabRows)) return MOE_ERR_CUDA;
    } else {
        g1.a_map[1] = g1.a_map[0];   // no tile refers to slot 1
    }
    g1.tiles = tiles1;
    g1.ntiles_dev = ntiles;
    g1.out = h;
    g1.out_ld = inter;
    g1.col_limit = inter;
    int rc;
    if (i4 != nullptr) {
        fill_pipeline_fp8(g1, n_max, kSlabBytes4);
        rc = launch_gemm<kEpiSwiGLU, kOpsW4Convert>(g1, std::min(max_tiles1, di.sms), st);
    } else if (f8 != nullptr) {
        fill_pipeline_fp8(g1, n_max);
        rc = launch_gemm<kEpiSwiGLU, kOpsW8Convert>(g1, std::min(max_tiles1, di.sms), st);
    } else {
        fill_pipeline(g1, 2, n_max);
        rc = launch_gemm<kEpiSwiGLU>(g1, std::min(max_tiles1, di.sms), st);
    }
    if (rc != MOE_OK) return rc;
    rec.mark(st);
    rec.skip(st);   // no activation quantization

    GemmArgs g2;
    std::memset(&g2, 0, sizeof(g2));
    if (i4 != nullptr) {
        if (!make_map_int4(&g2.a8_map, &g2.a4s_map, i4->down, i4->down_scale,
                           static_cast<uint64_t>(E) * d, inter) ||
            !make_map(&g2.a_map[0], ws_down, d, inter, kSlabRows))
            return MOE_ERR_CUDA;
    } else if (f8 != nullptr) {
        if (!make_map8(&g2.a8_map, f8->down, static_cast<uint64_t>(E) * d, inter) ||
            !make_map(&g2.a_map[0], ws_down, d, inter, kSlabRows))
            return MOE_ERR_CUDA;
        g2.a8_scale = f8->down_exp;
        g2.a8_kblocks = inter / kQuantBlock;
    } else if (!make_map(&g2.a_map[0], w_down, static_cast<uint64_t>(E) * d, inter, kSlabRows)) {
        return MOE_ERR_CUDA;
    }
    if (!make_map(&g2.b_map[0], h, rows_all, inter, kBoxRows) ||
        !make_map(&g2.b_map64[0], h, rows_all, inter, kBoxRowsBig))
        return MOE_ERR_CUDA;
    if (shared) {
        if (!make_map(&g2.a_map[1], ws_down, d, inter, kSlabRows)) return MOE_ERR_CUDA;
    } else {
        g2.a_map[1] = g2.a_map[0];
    }
    g2.b_map[1] = g2.b_map[0];
    g2.b_map64[1] = g2.b_map64[0];
    g2.tiles = tiles2;
    g2.ntiles_dev = ntiles + 1;
    g2.out = y;
    g2.out_ld = d;
    g2.col_limit = d;
    if (i4 != nullptr) {
        fill_pipeline_fp8(g2, n_max, kSlabBytes4);
        rc = launch_gemm<kEpiStoreBF16, kOpsW4Convert>(g2, std::min(max_tiles2, di.sms), st);
    } else if (f8 != nullptr) {
        fill_pipeline_fp8(g2, n_max);
        rc = launch_gemm<kEpiStoreBF16, kOpsW8Convert>(g2, std::min(max_tiles2, di.sms), st);
    } else {
        fill_pipeline(g2, 2, n_max);
        rc = launch_gemm<kEpiStoreBF16>(g2, std::min(max_tiles2, di.sms), st);
    }
    if (rc != MOE_OK) return rc;
    rec.mark(st);
    return MOE_OK;
}

// FP8 compute: every expert's weights (routed and shared) as E4M3 codes with
// one int8 exponent per row (quant.cuh): gate|up [E, 2I, d] + [E, 2I], down
// [E, d, I] + [E, d], shared gate|up [2I, d] + [2I], shared down [d, I] + [d].
struct Fp8Rows {
    const uint8_t* gate_up;
    const int8_t* gate_up_exp;
    const uint8_t* down;
    const int8_t* down_exp;
    const uint8_t* s_gate_up;
    const int8_t* s_gate_up_exp;
    const uint8_t* s_down;
    const int8_t* s_down_exp;
};

// FP8-compute FFN over a planned tile list (tiles with K steps of 2 * kBK):
//   1. the token rows to E4M3 per row: the T*k permuted rows, then the T rows in
//      token order, codes xq, exponents xexp; for large T token by token (each x
//      row quantized once, its codes written to its rows through slot_row), for
//      small T row by row (a gather through row_token)
//   2. gate|up on codes (kind::f8f6f4), SwiGLU epilogue with the exponents -> h
//   3. h's rows to E4M3 per row -> hq, hexp
//   4. down on codes -> y (bf16)
int launch_ffn_fp8(const DeviceInfo& di, const bf16* x, const int* row_token,
                   const int* slot_row, int T, int d,
                   int E, int k, int inter, const Fp8Rows& w, uint8_t* xq, int8_t* xexp, bf16* h,
                   uint8_t* hq, int8_t* hexp, bf16* y, const int4* tiles1, const int4* tiles2,
                   const int* ntiles, int max_tiles1, int max_tiles2, cudaStream_t st,
                   Recorder& rec, int tile_n) {
    const long long rows_routed = static_cast<long long>(T) * k;
    const long long rows_all = rows_routed + T;
    const unsigned qblocks = static_cast<unsigned>((rows_all + kRowQuantWarps - 1) / kRowQuantWarps);
    if (T >= kTokenMajorMinT)
        launch(fp8_quantize_tokens_kernel, (T + kRowQuantWarps - 1) / kRowQuantWarps, 32 * kRowQuantWarps, 0, st, x, slot_row, T, k, rows_routed, d, xq, xexp);
    else
        launch(fp8_quantize_rows_kernel, qblocks, 32 * kRowQuantWarps, 0, st, x, d, row_token, rows_routed, T, rows_all, d, xq, xexp);
    rec.mark(st);
    const int n_max = std::min(tile_n, (T + 15) & ~15);
    const uint8_t* xq_tok = xq + rows_routed * d;

    GemmArgs g1;
    std::memset(&g1, 0, sizeof(g1));
    const uint64_t rr = static_cast<uint64_t>(std::max<long long>(rows_routed, 1));
    if (!make_map_e4m3(&g1.a_map[0], w.gate_up, static_cast<uint64_t>(E) * 2 * inter, d,
                       kSlabRows) ||
        !make_map_e4m3(&g1.a_map[1], w.s_gate_up, 2ull * inter, d, kSlabRows) ||
        !make_map_e4m3(&g1.b_map[0], xq, rr, d, kBoxRows) ||
        !make_map_e4m3(&g1.b_map64[0], xq, rr, d, kBoxRowsBig) ||
        !make_map_e4m3(&g1.b_map[1], xq_tok, T, d, kBoxRows) ||
        !make_map_e4m3(&g1.b_map64[1], xq_tok, T, d, kBoxRowsBig))
        return MOE_ERR_CUDA;
    g1.a_exp[0] = w.gate_up_exp;
    g1.a_exp[1] = w.s_gate_up_exp;
    g1.b_exp[0] = xexp;
    g1.b_exp[1] = xexp + rows_routed;
    g1.tiles = tiles1;
    g1.ntiles_dev = ntiles;
    g1.out = h;
    g1.out_ld = inter;
    g1.col_limit = inter;
    fill_pipeline(g1, 2, n_max);
    int rc = launch_gemm<kEpiSwiGLU, kOpsFP8>(g1, std::min(max_tiles1, di.sms), st);
    if (rc != MOE_OK) return rc;
    rec.mark(st);

    launch(fp8_quantize_rows_kernel, qblocks, 32 * kRowQuantWarps, 0, st, h, inter, nullptr, 0, rows_all, rows_all, inter, hq, hexp);
    rec.mark(st);

    GemmArgs g2;
    std::memset(&g2, 0, sizeof(g2));
    if (!make_map_e4m3(&g2.a_map[0], w.down, static_cast<uint64_t>(E) * d, inter, kSlabRows) ||
        !make_map_e4m3(&g2.a_map[1], w.s_down, d, inter, kSlabRows) ||
        !make_map_e4m3(&g2.b_map[0], hq, rows_all, inter, kBoxRows) ||
        !make_map_e4m3(&g2.b_map64[0], hq, rows_all, inter, kBoxRowsBig))
        return MOE_ERR_CUDA;
    g2.b_map[1] = g2.b_map[0];
    g2.b_map64[1] = g2.b_map64[0];
    g2.a_exp[0] = w.down_exp;
    g2.a_exp[1] = w.s_down_exp;
    g2.b_exp[0] = hexp;
    g2.b_exp[1] = hexp;
    g2.tiles = tiles2;
    g2.ntiles_dev = ntiles + 1;
    g2.out = y;
    g2.out_ld = d;
    g2.col_limit = d;
    fill_pipeline(g2, 2, n_max);
    rc = launch_gemm<kEpiStoreBF16, kOpsFP8>(g2, std::min(max_tiles2, di.sms), st);
    if (rc != MOE_OK) return rc;
    rec.mark(st);
    return launch_rc(__func__);
}

int launch_combine(const bf16* y, const bf16* ysh, const float* w, const int* slot_row, int T,
                   int d, int k, bf16* out, cudaStream_t st, Recorder& rec) {
    // split each row over several blocks only while the batch is small
    const int chunks = (d / 8 + kCombineThreads - 1) / kCombineThreads;
    const dim3 grid(T, std::max(1, std::min(chunks, (2048 + T - 1) / T)));
    launch(combine_kernel, grid, kCombineThreads, 0, st, y, ysh, w, slot_row, T, d, k, static_cast<long long>(T) * k, out);
    rec.mark(st);
    return launch_rc(__func__);
}

__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        // nobody arrives: the bounded wait must give up and record a timeout
        wait_bounded(&bar, 0, nullptr, timeout_ns);
    }
}

int layer_forward(const bf16* x, const bf16* wr, const float* bias, const bf16* wgu,
                  const bf16* wdn, const bf16* sgu, const bf16* sdn, int T, int d, int E, int k,
                  int inter, float scale, bf16* out, void* ws, size_t ws_bytes, cudaStream_t st,
                  const Fp8Experts* f8 = nullptr, const Fp8Rows* f8c = nullptr,
                  const Int4Experts* i4 = nullptr) {
    const Layout L = make_layout(T, d, E, k, inter, f8c != nullptr);
    if (ws == nullptr || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    uint8_t* base = static_cast<uint8_t*>(ws);
    auto P = [&](size_t off) { return base + off; };
    int* idx = reinterpret_cast<int*>(P(L.topk_idx));
    float* w = reinterpret_cast<float*>(P(L.topk_w));
    int* counts = reinterpret_cast<int*>(P(L.counts));
    int* offsets = reinterpret_cast<int*>(P(L.offsets));
    int* row_token = reinterpret_cast<int*>(P(L.row_token));
    int* slot_row = reinterpret_cast<int*>(P(L.slot_row));
    int4* tiles1 = reinterpret_cast<int4*>(P(L.tiles1));
    int4* tiles2 = reinterpret_cast<int4*>(P(L.tiles2));
    int* ntiles = reinterpret_cast<int*>(P(L.ntiles));
    bf16* xperm = reinterpret_cast<bf16*>(P(L.xperm));
    bf16* h = reinterpret_cast<bf16*>(P(L.h));
    bf16* y = reinterpret_cast<bf16*>(P(L.y));
    Recorder rec;
    {
        std::lock_guard<std::mutex> lk(g_prof.mu);
        if (g_prof.calls < g_prof.max_calls) {
            rec.ev = g_prof.ev.data() + static_cast<size_t>(g_prof.calls) * (kLayerKernels + 1);
            ++g_prof.calls;
        }
    }
    rec.start(st);
    rc = launch_route(di, x, wr, bias, T, d, E, k, scale, idx, w,
                      reinterpret_cast<float*>(P(L.partials)), L.splits, st, rec);
    if (rc != MOE_OK) return rc;
    PlanArgs plan{E, 1, T, d, inter, T * k, tiles1, tiles2, ntiles};
    if (f8c != nullptr) plan.kstep = 2 * kBK;
    const bool use_gemv = (i4 != nullptr || f8 != nullptr) && gemv_ok(T, d, E, k, inter, i4 != nullptr);
    plan.tile_n = use_gemv ? kGemvTileN : tile_rows(T, E, k);
    rc = launch_permute(idx, T, E, k, counts, offsets, row_token, slot_row,
                        reinterpret_cast<int*>(P(L.blk)), plan, st, rec);
    if (rc != MOE_OK) return rc;
    if (f8c != nullptr)
        rc = launch_ffn_fp8(di, x, row_token, slot_row, T, d, E, k, inter, *f8c,
                            reinterpret_cast<uint8_t*>(xperm), reinterpret_cast<int8_t*>(P(L.xexp)),
                            h, P(L.hq), reinterpret_cast<int8_t*>(P(L.hexp)), y, tiles1, tiles2,
                            ntiles, L.max_tiles1, L.max_tiles2, st, rec, plan.tile_n);
    else
        rc = launch_ffn(di, x, row_token, slot_row, T, d, E, k, inter, wgu, wdn, sgu, sdn, true,
                        xperm, h,
                        y, tiles1, tiles2, ntiles, L.max_tiles1, L.max_tiles2, st, rec, f8, i4,
                        plan.tile_n, use_gemv);
    if (rc != MOE_OK) return rc;
    rc = launch_combine(y, y + static_cast<size_t>(T) * k * d, w, slot_row, T, d, k, out, st, rec);
    g_last_launches.store(rec.launches);
    return rc;
}

// Library-owned scratch of moe_layer_forward, one buffer per (device, stream).
struct WsEntry {
    int dev;
    cudaStream_t stream;
    void* ptr;
    size_t bytes;
};
std::mutex g_ws_mu;
std::vector<WsEntry> g_ws;

int owned_workspace(cudaStream_t st, size_t need, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (WsEntry& e : g_ws) {
        if (e.dev == dev && e.stream == st) {
            if (e.bytes < need) {
                if (e.ptr) cudaFreeAsync(e.ptr, st);
                e.ptr = nullptr;
                e.bytes = 0;
                if (cudaMallocAsync(&e.ptr, need, st) != cudaSuccess) {
                    cudaGetLastError();
                    return MOE_ERR_NO_MEMORY;
                }
                e.bytes = need;
            }
            *out = e.ptr;
            return MOE_OK;
        }
    }
    void* p = nullptr;
    if (cudaMallocAsync(&p, need, st) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_NO_MEMORY;
    }
    g_ws.push_back({dev, st, p, need});
    *out = p;
    return MOE_OK;
}

// Device address of g_moe_noalloc_scratch in the current CUDA context.  A
// __device__ array has its own address in every context that loads the
// library, so the address is looked up once per context (with that context
// current) and cached under the context's unique id (cuCtxGetId: ids are never
// reused in a process, so a context created after cudaDeviceReset, or a
// non-primary context of the same device, gets its own lookup).
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct NoallocEntry {
    unsigned long long ctx_id;
    void* ptr;
};
std::mutex g_noalloc_mu;
std::vector<NoallocEntry> g_noalloc;

bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

int noalloc_scratch(void** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (have_id)
        for (const NoallocEntry& e : g_noalloc)
            if (e.ctx_id == id) {
                *out = e.ptr;
                return MOE_OK;
            }
    // the lookup also makes the device's primary context current when no
    // context was yet (then the id is read after it)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_noalloc_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (have_id || current_context_id(&id)) g_noalloc.push_back({id, p});
    *out = p;
    return MOE_OK;
}

thread_local std::vector<SideStream> t_side;

int side_stream(SideStream** out) {
    unsigned long long id = 0;
    if (!current_context_id(&id)) return record_cuda_failure(__func__, "no current CUDA context");
    for (SideStream& e : t_side)
        if (e.ctx_id == id) {
            *out = &e;
            return MOE_OK;
        }
    SideStream e{id, nullptr, nullptr, nullptr};
    if (cudaStreamCreateWithFlags(&e.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&e.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&e.join, cudaEventDisableTiming) != cudaSuccess)
        return record_cuda_failure(__func__, cudaGetErrorString(cudaGetLastError()));
    t_side.push_back(e);
    *out = &t_side.back();
    return MOE_OK;
}

// ------------------------------------------------------ expert parallelism

// Scratch of moe_ep_dispatch: router partials, permutation block counts,
// expert offsets and the permuted rows' tokens.
struct EpDispatchLayout {
    size_t partials, blk, offsets, row_token, total;
    int splits;
};

EpDispatchLayout ep_dispatch_layout(int T, int d, int E, int k) {
    EpDispatchLayout L{};
    L.splits = router_splits(T, d, E);
    const int nblk = (T + kPermTokens - 1) / kPermTokens;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.partials = take(static_cast<size_t>(L.splits) * T * E * sizeof(float));
    L.blk = take(static_cast<size_t>(std::max(nblk, 1)) * E * sizeof(int));
    L.offsets = take(static_cast<size_t>(E + 2) * sizeof(int));
    L.row_token = take(static_cast<size_t>(T) * k * sizeof(int));
    L.total = off;
    return L;
}

// Scratch of moe_ep_expert_ffn: the receive maps and expert offsets, then the
// grouped FFN's scratch (the layout of `rows` tokens, E_l experts, k = 1).
struct EpFfnLayout {
    size_t exp_offsets, src_of_exp, exp_of_src, ffn, total;
    Layout F;
};

EpFfnLayout ep_ffn_layout(int rows, int d, int El, int inter) {
    EpFfnLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.exp_offsets = take(static_cast<size_t>(El + 2) * sizeof(int));
    L.src_of_exp = take(static_cast<size_t>(rows) * sizeof(int));
    L.exp_of_src = take(static_cast<size_t>(rows) * sizeof(int));
    L.ffn = off;
    L.F = make_layout(rows, d, El, 1, inter);
    L.total = L.ffn + L.F.total;
    return L;
}

// Scratch of moe_ep_combine: the shared expert's tile lists, h and output rows.
struct EpCombineLayout {
    size_t tiles1, tiles2, ntiles, h, y, total;
    int max_tiles1, max_tiles2;
};

EpCombineLayout ep_combine_layout(int T, int d, int inter) {
    EpCombineLayout L{};
    const int nt = (T + kTileN - 1) / kTileN;
    L.max_tiles1 = nt * ((inter + kSlabRows - 1) / kSlabRows);
    L.max_tiles2 = nt * ((d + 2 * kSlabRows - 1) / (2 * kSlabRows));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.tiles1 = take(static_cast<size_t>(L.max_tiles1) * 2 * sizeof(int4));
    L.tiles2 = take(static_cast<size_t>(L.max_tiles2) * 2 * sizeof(int4));
    L.ntiles = take(4 * sizeof(int));
    L.h = take(static_cast<size_t>(T) * inter * sizeof(bf16));
    L.y = take(static_cast<size_t>(T) * d * sizeof(bf16));
    L.total = off;
    return L;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_NO_MEMORY: return "MOE_ERR_NO_MEMORY";
        default: return "MOE_ERR_UNKNOWN";
    }
}

size_t moe_workspace_size(int T, int d, int E, int k, int inter) {
    if (check_dims(T, d, E, k, inter) != MOE_OK) return 0;
    return make_layout(T, d, E, k, inter).total;
}

int moe_route(const uint16_t* x, const uint16_t* w_router, const float* bias, int T, int d, int E,
              int k, float scale, int32_t* topk_idx, float* topk_w, void* workspace,
              size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, 64);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, topk_idx, topk_w, workspace)) return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    const int splits = router_splits(T, d, E);
    if (workspace_bytes < static_cast<size_t>(splits) * T * E * sizeof(float))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    Recorder rec;
    return launch_route(di, reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                        bias, T, d, E, k, scale, topk_idx, topk_w, static_cast<float*>(workspace),
                        splits, static_cast<cudaStream_t>(stream), rec);
}

int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* row_token, int32_t* slot_row, void* workspace, size_t workspace_bytes,
                void* stream) {
    CallScope scope;
    int rc = check_dims(T, 64, E, k, 64);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(topk_idx, counts, offsets, row_token, slot_row, workspace))
        return MOE_ERR_INVALID_ARG;
    const int nblk = (T + kPermTokens - 1) / kPermTokens;
    if (workspace_bytes < static_cast<size_t>(nblk) * E * sizeof(int)) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;                  // sets the kernels' shared-memory limits on first use
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    PlanArgs none{};
    Recorder rec;
    return launch_permute(topk_idx, T, E, k, counts, offsets, row_token, slot_row,
                          static_cast<int*>(workspace), none, static_cast<cudaStream_t>(stream),
                          rec);
}

int moe_expert_ffn(const uint16_t* x, const int32_t* row_token, const int32_t* offsets,
                   const uint16_t* w_gate_up, const uint16_t* w_down, int T, int d, int E, int k,
                   int inter, uint16_t* y, void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, row_token, offsets, w_gate_up, w_down, y, workspace)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(T, d, E, k, inter);
    if (workspace_bytes < L.total) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int4* tiles1 = reinterpret_cast<int4*>(base + L.tiles1);
    int4* tiles2 = reinterpret_cast<int4*>(base + L.tiles2);
    int* ntiles = reinterpret_cast<int*>(base + L.ntiles);
    PlanArgs plan{E, 0, T, d, inter, T * k, tiles1, tiles2, ntiles};
    launch(plan_kernel, 1, 1024, 0, st, offsets, plan);
    if (launch_rc(__func__) != MOE_OK) return MOE_ERR_CUDA;
    Recorder rec;
    return launch_ffn(di, reinterpret_cast<const bf16*>(x), row_token, nullptr, T, d, E, k, inter,
                      reinterpret_cast<const bf16*>(w_gate_up), reinterpret_cast<const bf16*>(w_down),
                      nullptr, nullptr, false, reinterpret_cast<bf16*>(base + L.xperm),
                      reinterpret_cast<bf16*>(base + L.h), reinterpret_cast<bf16*>(y), tiles1,
                      tiles2, ntiles, L.max_tiles1, L.max_tiles2, st, rec);
}

int moe_combine(const uint16_t* y, const uint16_t* y_shared, const float* topk_w,
                const int32_t* slot_row, int T, int d, int k, uint16_t* out, void* stream) {
    CallScope scope;
    if (T < 0 || k < 1 || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (d < 8 || d % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!all_ok(y, topk_w, slot_row, out)) return MOE_ERR_INVALID_ARG;
    if (y_shared != nullptr && !aligned16(y_shared)) return MOE_ERR_INVALID_ARG;
    Recorder rec;
    return launch_combine(reinterpret_cast<const bf16*>(y), reinterpret_cast<const bf16*>(y_shared),
                          topk_w, slot_row, T, d, k, reinterpret_cast<bf16*>(out),
                          static_cast<cudaStream_t>(stream), rec);
}

int moe_layer_forward_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                         const uint16_t* w_gate_up, const uint16_t* w_down,
                         const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                         int E, int k, int inter, float scale, uint16_t* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, out, workspace))
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    return layer_forward(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                         bias, reinterpret_cast<const bf16*>(w_gate_up),
                         reinterpret_cast<const bf16*>(w_down),
                         reinterpret_cast<const bf16*>(ws_gate_up),
                         reinterpret_cast<const bf16*>(ws_down), T, d, E, k, inter, scale,
                         reinterpret_cast<bf16*>(out), workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream));
}

int moe_layer_forward(const uint16_t* x, const uint16_t* w_router, const float* bias,
                      const uint16_t* w_gate_up, const uint16_t* w_down,
                      const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d, int E,
                      int k, int inter, float scale, uint16_t* out, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, out))
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    const size_t need = make_layout(T, d, E, k, inter).total;
    void* ws = nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = owned_workspace(st, need, &ws);
    if (rc != MOE_OK) return rc;
    return moe_layer_forward_ws(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, T, d, E,
                                k, inter, scale, out, ws, need, stream);
}

int moe_layer_forward_noalloc(const uint16_t* x, const uint16_t* w_router, const float* bias,
                              const uint16_t* w_gate_up, const uint16_t* w_down,
                              const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                              int E, int k, int inter, float scale, uint16_t* out, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, out))
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    if (make_layout(T, d, E, k, inter).total > MOE_NOALLOC_SCRATCH_BYTES)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    void* ws = nullptr;
    rc = noalloc_scratch(&ws);
    if (rc != MOE_OK) return rc;
    return layer_forward(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                         bias, reinterpret_cast<const bf16*>(w_gate_up),
                         reinterpret_cast<const bf16*>(w_down),
                         reinterpret_cast<const bf16*>(ws_gate_up),
                         reinterpret_cast<const bf16*>(ws_down), T, d, E, k, inter, scale,
                         reinterpret_cast<bf16*>(out), ws, MOE_NOALLOC_SCRATCH_BYTES,
                         static_cast<cudaStream_t>(stream));
}

int moe_quantize_fp8(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, int8_t* exps,
                     void* stream) {
    CallScope scope;
    if (rows < 0 || cols < 0 || rows % kQuantBlock != 0 || cols % kQuantBlock != 0 ||
        rows / kQuantBlock > 0x7FFFFFFF || cols / kQuantBlock > 65535)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!all_ok(w, q) || exps == nullptr) return MOE_ERR_INVALID_ARG;
    const dim3 grid(static_cast<unsigned>(rows / kQuantBlock), static_cast<unsigned>(cols / kQuantBlock));
    launch(fp8_quantize_kernel, grid, kQuantThreads, 0, static_cast<cudaStream_t>(stream), reinterpret_cast<const bf16*>(w), cols, q, exps);
    return launch_rc(__func__);
}

int moe_layer_forward_fp8_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                             const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                             const uint8_t* wq_down, const int8_t* wq_down_exp,
                             const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                             int E, int k, int inter, float scale, uint16_t* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (d % kQuantBlock != 0 || inter % kQuantBlock != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_down, ws_gate_up, ws_down, out, workspace) ||
        wq_gate_up_exp == nullptr || wq_down_exp == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    const Fp8Experts f8{wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp};
    return layer_forward(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                         bias, nullptr, nullptr, reinterpret_cast<const bf16*>(ws_gate_up),
                         reinterpret_cast<const bf16*>(ws_down), T, d, E, k, inter, scale,
                         reinterpret_cast<bf16*>(out), workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream), &f8);
}

int moe_layer_forward_fp8(const uint16_t* x, const uint16_t* w_router, const float* bias,
                          const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                          const uint8_t* wq_down, const int8_t* wq_down_exp,
                          const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                          int E, int k, int inter, float scale, uint16_t* out, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (d % kQuantBlock != 0 || inter % kQuantBlock != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_down, ws_gate_up, ws_down, out) ||
        wq_gate_up_exp == nullptr || wq_down_exp == nullptr || !(scale == scale))
        return MOE_ERR_INVALID_ARG;
    const size_t need = make_layout(T, d, E, k, inter).total;
    void* ws = nullptr;
    rc = owned_workspace(static_cast<cudaStream_t>(stream), need, &ws);
    if (rc != MOE_OK) return rc;
    return moe_layer_forward_fp8_ws(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down,
                                    wq_down_exp, ws_gate_up, ws_down, T, d, E, k, inter, scale,
                                    out, ws, need, stream);
}

int moe_quantize_int4(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* codes,
                      uint16_t* scales, void* stream) {
    CallScope scope;
    if (rows < 0 || cols < 0 || cols % kBK != 0 || cols > 0x7FFFFFFF ||
        rows * (cols / kInt4Group) > 0x7FFFFFFFll * kInt4Warps)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!all_ok(w, codes, scales)) return MOE_ERR_INVALID_ARG;
    const long long groups = rows * (cols / kInt4Group);
    const unsigned blocks = static_cast<unsigned>((groups + kInt4Warps - 1) / kInt4Warps);
    launch(int4_quantize_kernel, blocks, 32 * kInt4Warps, 0, static_cast<cudaStream_t>(stream), reinterpret_cast<const bf16*>(w), rows, static_cast<int>(cols), reinterpret_cast<uint32_t*>(codes), reinterpret_cast<bf16*>(scales));
    return launch_rc(__func__);
}

int moe_layer_forward_w4a16_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                               const uint8_t* wq_gate_up, const uint16_t* wq_gate_up_scale,
                               const uint8_t* wq_down, const uint16_t* wq_down_scale,
                               const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                               int E, int k, int inter, float scale, uint16_t* out,
                               void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down, wq_down_scale,
                ws_gate_up, ws_down, out, workspace))
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    const Int4Experts i4{wq_gate_up, reinterpret_cast<const bf16*>(wq_gate_up_scale), wq_down,
                         reinterpret_cast<const bf16*>(wq_down_scale)};
    return layer_forward(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                         bias, nullptr, nullptr, reinterpret_cast<const bf16*>(ws_gate_up),
                         reinterpret_cast<const bf16*>(ws_down), T, d, E, k, inter, scale,
                         reinterpret_cast<bf16*>(out), workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream), nullptr, nullptr, &i4);
}

int moe_layer_forward_w4a16(const uint16_t* x, const uint16_t* w_router, const float* bias,
                            const uint8_t* wq_gate_up, const uint16_t* wq_gate_up_scale,
                            const uint8_t* wq_down, const uint16_t* wq_down_scale,
                            const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                            int E, int k, int inter, float scale, uint16_t* out, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down, wq_down_scale,
                ws_gate_up, ws_down, out) ||
        !(scale == scale))
        return MOE_ERR_INVALID_ARG;
    const size_t need = make_layout(T, d, E, k, inter).total;
    void* ws = nullptr;
    rc = owned_workspace(static_cast<cudaStream_t>(stream), need, &ws);
    if (rc != MOE_OK) return rc;
    return moe_layer_forward_w4a16_ws(x, w_router, bias, wq_gate_up, wq_gate_up_scale, wq_down,
                                      wq_down_scale, ws_gate_up, ws_down, T, d, E, k, inter,
                                      scale, out, ws, need, stream);
}

int moe_quantize_fp8_rows(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q,
                          int8_t* exps, void* stream) {
    CallScope scope;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || cols > 0x7FFFFFFF ||
        rows > 0x7FFFFFFFll * kRowQuantWarps)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!all_ok(w, q) || exps == nullptr) return MOE_ERR_INVALID_ARG;
    const unsigned blocks = static_cast<unsigned>((rows + kRowQuantWarps - 1) / kRowQuantWarps);
    launch(fp8_quantize_rows_kernel, blocks, 32 * kRowQuantWarps, 0, static_cast<cudaStream_t>(stream), reinterpret_cast<const bf16*>(w), cols, nullptr, 0, rows, rows, static_cast<int>(cols), q, exps);
    return launch_rc(__func__);
}

size_t moe_workspace_size_w8a8(int T, int d, int E, int k, int inter) {
    if (check_dims(T, d, E, k, inter) != MOE_OK) return 0;
    return make_layout(T, d, E, k, inter, true).total;
}

int moe_layer_forward_w8a8_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                              const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                              const uint8_t* wq_down, const int8_t* wq_down_exp,
                              const uint8_t* wsq_gate_up, const int8_t* wsq_gate_up_exp,
                              const uint8_t* wsq_down, const int8_t* wsq_down_exp, int T, int d,
                              int E, int k, int inter, float scale, uint16_t* out,
                              void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (d % (2 * kBK) != 0 || inter % (2 * kBK) != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_down, wsq_gate_up, wsq_down, out, workspace) ||
        wq_gate_up_exp == nullptr || wq_down_exp == nullptr || wsq_gate_up_exp == nullptr ||
        wsq_down_exp == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!(scale == scale)) return MOE_ERR_INVALID_ARG;
    const Fp8Rows f8c{wq_gate_up, wq_gate_up_exp, wq_down, wq_down_exp,
                      wsq_gate_up, wsq_gate_up_exp, wsq_down, wsq_down_exp};
    return layer_forward(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                         bias, nullptr, nullptr, nullptr, nullptr, T, d, E, k, inter, scale,
                         reinterpret_cast<bf16*>(out), workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream), nullptr, &f8c);
}

int moe_layer_forward_w8a8(const uint16_t* x, const uint16_t* w_router, const float* bias,
                           const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                           const uint8_t* wq_down, const int8_t* wq_down_exp,
                           const uint8_t* wsq_gate_up, const int8_t* wsq_gate_up_exp,
                           const uint8_t* wsq_down, const int8_t* wsq_down_exp, int T, int d,
                           int E, int k, int inter, float scale, uint16_t* out, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, inter);
    if (rc != MOE_OK) return rc;
    if (d % (2 * kBK) != 0 || inter % (2 * kBK) != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, wq_gate_up, wq_down, wsq_gate_up, wsq_down, out) ||
        wq_gate_up_exp == nullptr || wq_down_exp == nullptr || wsq_gate_up_exp == nullptr ||
        wsq_down_exp == nullptr || !(scale == scale))
        return MOE_ERR_INVALID_ARG;
    const size_t need = make_layout(T, d, E, k, inter, true).total;
    void* ws = nullptr;
    rc = owned_workspace(static_cast<cudaStream_t>(stream), need, &ws);
    if (rc != MOE_OK) return rc;
    return moe_layer_forward_w8a8_ws(x, w_router, bias, wq_gate_up, wq_gate_up_exp, wq_down,
                                     wq_down_exp, wsq_gate_up, wsq_gate_up_exp, wsq_down,
                                     wsq_down_exp, T, d, E, k, inter, scale, out, ws, need,
                                     stream);
}

// Scratch of moe_seq_aux_loss: 1 / (token score sums) [B*S], the per-block
// partial sums [B, ceil(S/256), E] and the selection counts [B, E] (int).
struct AuxLayout {
    size_t inv_tot, part, cnt, total;
    int nsplit;
};

AuxLayout aux_layout(int B, int S, int E) {
    AuxLayout L{};
    const long long T = static_cast<long long>(B) * S;
    L.nsplit = (S + kAuxTokens - 1) / kAuxTokens;
    size_t off = 0;
    L.inv_tot = off;
    off = align256(off + static_cast<size_t>(T) * sizeof(float));
    L.part = off;
    off = align256(off + static_cast<size_t>(B) * L.nsplit * E * sizeof(float));
    L.cnt = off;
    off = align256(off + static_cast<size_t>(B) * E * sizeof(int));
    L.total = off;
    return L;
}

size_t moe_seq_aux_workspace_size(int B, int S, int E) {
    if (B < 0 || S < 1 || E < 1 || E > 1024) return 0;
    return aux_layout(B, S, E).total;
}

int moe_bias_update(const int32_t* counts, int T, int E, int k, float gamma, float* bias,
                    void* stream) {
    CallScope scope;
    if (E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (counts == nullptr || bias == nullptr || !(gamma == gamma)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;           // no rows routed: every expert sits at the mean
    launch(bias_update_kernel, (E + kBalanceThreads - 1) / kBalanceThreads, kBalanceThreads, 0, static_cast<cudaStream_t>(stream), counts, static_cast<long long>(T) * k, E, gamma, bias);
    return launch_rc(__func__);
}

int moe_router_scores(const uint16_t* x, const uint16_t* w_router, int T, int d, int E,
                      float* scores, void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, 1, 64);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, scores, workspace)) return MOE_ERR_INVALID_ARG;
    const int splits = router_splits(T, d, E);
    if (workspace_bytes < static_cast<size_t>(splits) * T * E * sizeof(float))
        return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* partials = static_cast<float*>(workspace);
    rc = launch_router_gemm(di, reinterpret_cast<const bf16*>(x),
                            reinterpret_cast<const bf16*>(w_router), T, d, E, partials, splits, st);
    if (rc != MOE_OK) return rc;
    const long long n = static_cast<long long>(T) * E;
    launch(router_scores_kernel, static_cast<unsigned>((n + kBalanceThreads - 1) / kBalanceThreads), kBalanceThreads, 0, st, partials, splits, n, n, scores);
    return launch_rc(__func__);
}

int moe_seq_aux_loss(const float* scores, const int32_t* topk_idx, int B, int S, int E, int k,
                     float alpha, float* loss, float* f, float* p, void* workspace,
                     size_t workspace_bytes, void* stream) {
    CallScope scope;
    if (E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (B < 0 || S < 1) return MOE_ERR_INVALID_ARG;
    if (B == 0) return MOE_OK;
    if (scores == nullptr || topk_idx == nullptr || loss == nullptr || !(alpha == alpha) ||
        !aligned16(workspace))
        return MOE_ERR_INVALID_ARG;
    const AuxLayout L = aux_layout(B, S, E);
    if (workspace_bytes < L.total || L.nsplit > 65535) return MOE_ERR_INVALID_ARG;
    const long long T = static_cast<long long>(B) * S;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    float* inv_tot = reinterpret_cast<float*>(base + L.inv_tot);
    float* part = reinterpret_cast<float*>(base + L.part);
    int* cnt = reinterpret_cast<int*>(base + L.cnt);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(cnt, 0, static_cast<size_t>(B) * E * sizeof(int), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    launch(token_totals_kernel, static_cast<unsigned>((T + 7) / 8), kBalanceThreads, 0, st, scores, T, E, inv_tot);
    const int nchunk = (E + kAuxExperts - 1) / kAuxExperts;
    launch(seq_aux_partial_kernel, dim3(B, nchunk, L.nsplit), 32 * kAuxWarps, 0, st, scores,
           inv_tot, S, E, part);
    const long long n = T * k;
    launch(seq_aux_count_kernel, static_cast<unsigned>((n + kBalanceThreads - 1) / kBalanceThreads), kBalanceThreads, 0, st, topk_idx, n, S * k, E, cnt);
    launch(seq_aux_finish_kernel, B, kBalanceThreads, 0, st, part, cnt, L.nsplit, S, E, k, alpha, loss, f, p);
    return launch_rc(__func__);
}

// ------------------------------------------------------ expert parallelism

size_t moe_ep_dispatch_workspace_size(int T, int d, int E, int k) {
    if (check_dims(T, d, E, k, 64) != MOE_OK) return 0;
    return ep_dispatch_layout(T, d, E, k).total;
}

int moe_ep_dispatch(const uint16_t* x, const uint16_t* w_router, const float* bias, int T, int d,
                    int E, int k, float scale, int32_t* topk_idx, float* topk_w, int32_t* counts,
                    int32_t* slot_row, uint16_t* send_rows, void* workspace,
                    size_t workspace_bytes, void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, E, k, 64);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(x, w_router, bias, topk_idx, topk_w, counts, slot_row, send_rows, workspace) ||
        !(scale == scale))
        return MOE_ERR_INVALID_ARG;
    const EpDispatchLayout L = ep_dispatch_layout(T, d, E, k);
    if (workspace_bytes < L.total) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int* row_token = reinterpret_cast<int*>(base + L.row_token);
    Recorder rec;
    rc = launch_route(di, reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(w_router),
                      bias, T, d, E, k, scale, topk_idx, topk_w,
                      reinterpret_cast<float*>(base + L.partials), L.splits, st, rec);
    if (rc != MOE_OK) return rc;
    PlanArgs none{};
    rc = launch_permute(topk_idx, T, E, k, counts, reinterpret_cast<int*>(base + L.offsets),
                        row_token, slot_row, reinterpret_cast<int*>(base + L.blk), none, st, rec);
    if (rc != MOE_OK) return rc;
    const int rows = T * k;
    launch(gather_rows_kernel, (rows + 7) / 8, 256, 0, st, reinterpret_cast<const bf16*>(x), row_token, T, rows, d, reinterpret_cast<bf16*>(send_rows));
    return launch_rc(__func__);
}

size_t moe_ep_expert_ffn_workspace_size(int rows, int d, int R, int E_local, int inter) {
    if (R < 1 || E_local < 1 || static_cast<long long>(R) * E_local > 1024) return 0;
    if (check_dims(rows, d, E_local, 1, inter) != MOE_OK) return 0;
    return ep_ffn_layout(rows, d, E_local, inter).total;
}

int moe_ep_expert_ffn(const uint16_t* recv_rows, const int32_t* recv_counts, int rows, int d, int R,
                      int E_local, int inter, const uint16_t* w_gate_up, const uint16_t* w_down,
                      uint16_t* y, void* workspace, size_t workspace_bytes, void* stream) {
    CallScope scope;
    if (R < 1 || E_local < 1 || static_cast<long long>(R) * E_local > 1024)
        return MOE_ERR_UNSUPPORTED_SHAPE;
    int rc = check_dims(rows, d, E_local, 1, inter);
    if (rc != MOE_OK) return rc;
    if (rows == 0) return MOE_OK;
    if (!all_ok(recv_rows, recv_counts, w_gate_up, w_down, y, workspace)) return MOE_ERR_INVALID_ARG;
    const EpFfnLayout L = ep_ffn_layout(rows, d, E_local, inter);
    if (workspace_bytes < L.total) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int* exp_offsets = reinterpret_cast<int*>(base + L.exp_offsets);
    int* src_of_exp = reinterpret_cast<int*>(base + L.src_of_exp);
    int* exp_of_src = reinterpret_cast<int*>(base + L.exp_of_src);
    uint8_t* fb = base + L.ffn;
    int4* tiles1 = reinterpret_cast<int4*>(fb + L.F.tiles1);
    int4* tiles2 = reinterpret_cast<int4*>(fb + L.F.tiles2);
    int* ntiles = reinterpret_cast<int*>(fb + L.F.ntiles);
    bf16* y_exp = reinterpret_cast<bf16*>(fb + L.F.y);
    launch(ep_plan_kernel, 1, 1024, 0, st, recv_counts, R, E_local, rows, exp_offsets, src_of_exp, exp_of_src);
    PlanArgs plan{E_local, 0, rows, d, inter, rows, tiles1, tiles2, ntiles};
    launch(plan_kernel, 1, 1024, 0, st, exp_offsets, plan);
    if (launch_rc(__func__) != MOE_OK) return MOE_ERR_CUDA;
    Recorder rec;
    rc = launch_ffn(di, reinterpret_cast<const bf16*>(recv_rows), src_of_exp, nullptr, rows, d,
                    E_local, 1, inter, reinterpret_cast<const bf16*>(w_gate_up),
                    reinterpret_cast<const bf16*>(w_down), nullptr, nullptr, false,
                    reinterpret_cast<bf16*>(fb + L.F.xperm), reinterpret_cast<bf16*>(fb + L.F.h),
                    y_exp, tiles1, tiles2, ntiles, L.F.max_tiles1, L.F.max_tiles2, st, rec);
    if (rc != MOE_OK) return rc;
    // expert-major output rows back to the received (source-major) order
    launch(gather_rows_kernel, (rows + 7) / 8, 256, 0, st, y_exp, exp_of_src, rows, rows, d, reinterpret_cast<bf16*>(y));
    return launch_rc(__func__);
}

size_t moe_ep_combine_workspace_size(int T, int d, int inter) {
    if (check_dims(T, d, 1, 1, inter) != MOE_OK) return 0;
    return ep_combine_layout(T, d, inter).total;
}

int moe_ep_combine(const uint16_t* y_back, const uint16_t* x, const uint16_t* ws_gate_up,
                   const uint16_t* ws_down, const float* topk_w, const int32_t* slot_row, int T,
                   int d, int k, int inter, uint16_t* out, void* workspace, size_t workspace_bytes,
                   void* stream) {
    CallScope scope;
    int rc = check_dims(T, d, k, k, inter);
    if (rc != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    if (!all_ok(y_back, x, ws_gate_up, ws_down, topk_w, slot_row, out, workspace))
        return MOE_ERR_INVALID_ARG;
    const EpCombineLayout L = ep_combine_layout(T, d, inter);
    if (workspace_bytes < L.total) return MOE_ERR_INVALID_ARG;
    DeviceInfo di;
    rc = device_info(&di);
    if (rc != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    int4* tiles1 = reinterpret_cast<int4*>(base + L.tiles1);
    int4* tiles2 = reinterpret_cast<int4*>(base + L.tiles2);
    int* ntiles = reinterpret_cast<int*>(base + L.ntiles);
    bf16* y_sh = reinterpret_cast<bf16*>(base + L.y);
    // the shared expert alone: a plan with no routed expert (E = 0) and the T
    // token rows in order; its weights also stand in for the (unused) routed slot
    PlanArgs plan{0, 1, T, d, inter, 0, tiles1, tiles2, ntiles};
    launch(plan_kernel, 1, 1024, 0, st, nullptr, plan);
    if (launch_rc(__func__) != MOE_OK) return MOE_ERR_CUDA;
    const bf16* sgu = reinterpret_cast<const bf16*>(ws_gate_up);
    const bf16* sdn = reinterpret_cast<const bf16*>(ws_down);
    Recorder rec;
    rc = launch_ffn(di, reinterpret_cast<const bf16*>(x), nullptr, nullptr, T, d, 1, 0, inter, sgu,
                    sdn, sgu, sdn, true, nullptr, reinterpret_cast<bf16*>(base + L.h), y_sh,
                    tiles1, tiles2, ntiles, L.max_tiles1, L.max_tiles2, st, rec);
    if (rc != MOE_OK) return rc;
    return launch_combine(reinterpret_cast<const bf16*>(y_back), y_sh, topk_w, slot_row, T, d, k,
                          reinterpret_cast<bf16*>(out), st, rec);
}

int moe_device_status(void* stream, int* device_status) {
    if (device_status == nullptr) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    *device_status = v;
    return MOE_OK;
}

void moe_set_pdl(int enable) { g_pdl.store(enable ? 1 : 0); }

void moe_set_wait_timeout_ns(uint64_t timeout_ns) {
    g_timeout_ns.store(timeout_ns == 0 ? 1 : timeout_ns);
}

int moe_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launch_rc(__func__);
}

int moe_last_launch_count(void) { return g_last_launches.load(); }

const char* moe_last_error_string(void) { return t_last_error; }

int moe_profile_begin(int max_calls) {
    if (max_calls < 0) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
    g_prof.ev.clear();
    g_prof.calls = 0;
    g_prof.max_calls = 0;
    const size_t n = static_cast<size_t>(max_calls) * (kLayerKernels + 1);
    g_prof.ev.resize(n);
    for (size_t i = 0; i < n; ++i)
        if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
            for (size_t j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
            g_prof.ev.clear();
            return MOE_ERR_CUDA;
        }
    g_prof.max_calls = max_calls;
    return MOE_OK;
}

int moe_profile_end(float* total_ms, int max_kernels, int* n_calls) {
    if (total_ms == nullptr || n_calls == nullptr || max_kernels < 0) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    for (int i = 0; i < max_kernels; ++i) total_ms[i] = 0.0f;
    int rc = MOE_OK;
    for (int c = 0; c < g_prof.calls; ++c) {
        cudaEvent_t* ev = g_prof.ev.data() + static_cast<size_t>(c) * (kLayerKernels + 1);
        if (cudaEventSynchronize(ev[kLayerKernels]) != cudaSuccess) rc = MOE_ERR_CUDA;
        for (int i = 0; i < std::min(max_kernels, kLayerKernels); ++i) {
            float ms = 0.0f;
            if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) rc = MOE_ERR_CUDA;
            total_ms[i] += ms;
        }
    }
    *n_calls = g_prof.calls;
    for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
    g_prof.ev.clear();
    g_prof.calls = 0;
    g_prof.max_calls = 0;
    return rc == MOE_OK ? kLayerKernels : rc;
}

const char* moe_kernel_name(int i) {
    return (i >= 0 && i < kLayerKernels) ? kKernelNames[i] : "";
}

}  // extern "C"
