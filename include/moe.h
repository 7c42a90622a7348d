/*
 * moe.h -- C ABI of a single-GPU (B200, sm_100a) forward pass of one
 * Kimi-K2-style sparse MoE FFN layer with a sigmoid router.
 *
 * The layer ("Kimi K2.5 deep dive", CH4.2 routing and CH10.2 "MoE 7-step
 * dataflow"; "Kimi K2.5 Q&A", Q8.3; K2 team member's answer, "different"):
 *     s   = sigmoid(x W_r^T)                      scores, [T, E]
 *     b   = s + bias                              selection-only bias
 *     S_t = top-k of b_t over all E experts      (n_group = 1)
 *     w_j = scale * s_j / sum_{i in S_t} s_i      unbiased, renormalised, scaled
 *     out = shared(x) + sum_j w_j * f_{S_t[j]}(x)
 *     f_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x))     SwiGLU expert
 *
 * Conventions for every entry point:
 *   - bf16 tensors are passed as uint16_t* holding bf16 bit patterns;
 *   - every tensor pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned, row-major and densely packed with the shape given;
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); every
 *     call is asynchronous on it and never synchronises the host;
 *   - arguments are checked on the host before anything is launched; on
 *     error nothing is launched and a negative moe_status is returned;
 *   - T == 0 is a no-op that returns MOE_OK;
 *   - limits: 1 <= E <= 1024, 1 <= k <= min(E, 32), d and inter multiples of
 *     64 (>= 64), T * (k + 1) < 2^31;
 *   - kernels never trap: problems they can only see on the device (an
 *     out-of-range expert index, a wait that timed out) are recorded in a
 *     per-device status word that moe_device_status() reads.
 * There is no CPU fallback: a missing GPU or a failed launch is an error.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,       /* null / misaligned pointer, bad count */
    MOE_ERR_UNSUPPORTED_SHAPE = -2, /* d or inter not a multiple of 64, E or k out of range */
    MOE_ERR_CUDA = -3,              /* a CUDA call or launch failed */
    MOE_ERR_TIMEOUT = -4,           /* a device-side wait gave up (see moe_device_status) */
    MOE_ERR_NO_MEMORY = -5          /* workspace growth failed (moe_layer_forward) */
} moe_status;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int status);

/* What the last MOE_ERR_CUDA returned on the calling thread came from: the
 * failing CUDA call or tensor-map encoding and its error (a thread-local string,
 * valid until the thread's next failing call; "no error" before any). */
const char* moe_last_error_string(void);

/*
 * Bytes of device scratch that any staged call below needs for a layer of
 * this size (the largest of their needs).  Routing, permutation and expert
 * calls take the scratch as (workspace, workspace_bytes); its contents are not
 * preserved between calls, and two calls that overlap on the GPU must not
 * share it.
 */
size_t moe_workspace_size(int T, int d, int E, int k, int inter);

/*
 * Router, steps 1-4 ("Kimi K2.5 deep dive", CH4.2; CH10.2 steps 1-4).
 *   x        [T, d]  bf16    hidden states
 *   w_router [E, d]  bf16    router Linear weight (out x in)
 *   bias     [E]     fp32    e_score_correction_bias; affects selection only
 *   scale            fp32    routed_scaling_factor (2.827 for K2, 2.5 for DeepSeek-V3)
 *   topk_idx [T, k]  int32   out: slot j = expert with the j-th largest biased
 *                            score; ties go to the lower expert index
 *   topk_w   [T, k]  fp32    out: scale * s / sum(s) over the selected set,
 *                            s the UNBIASED sigmoid score
 * Logits accumulate in fp32 on tensor cores; selection is taken in fp32.
 */
int moe_route(const uint16_t* x, const uint16_t* w_router, const float* bias, int T, int d, int E,
              int k, float scale, int32_t* topk_idx, float* topk_w, void* workspace,
              size_t workspace_bytes, void* stream);

/*
 * Dispatch: group the T*k (token, slot) pairs by expert ("Kimi K2.5 deep
 * dive", CH10.2 step 6, the per-expert token mask).  Bit-exact and
 * deterministic.
 *   topk_idx  [T, k]  int32  in: k distinct experts in [0, E) per token
 *   counts    [E]     int32  out: rows per expert
 *   offsets   [E+1]   int32  out: exclusive prefix sum of counts, offsets[E] = T*k
 *   row_token [T*k]   int32  out: row -> token; rows of expert e are
 *                            offsets[e] .. offsets[e+1]-1 in ascending token order
 *   slot_row  [T*k]   int32  out: (t*k + j) -> row
 * An index outside [0, E) is skipped and recorded as MOE_ERR_INVALID_ARG in
 * the device status; a token that repeats an expert gives unspecified (but
 * in-bounds) rows.
 */
int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* row_token, int32_t* slot_row, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * Grouped SwiGLU experts ("Kimi K2.5 Q&A", Q8.3 step 5; "Kimi K2.5 deep
 * dive", CH4.3 and CH10.2 step 6): for every row r of expert e,
 *     y[r] = W_down,e ( silu(W_gate,e x[row_token[r]]) * (W_up,e x[row_token[r]]) )
 *   x         [T, d]        bf16
 *   row_token [T*k]         int32  (from moe_permute)
 *   offsets   [E+1]         int32  (from moe_permute), offsets[E] == T*k
 *   w_gate_up [E, 2*inter, d] bf16 rows [0, inter) = gate_proj, [inter, 2*inter) = up_proj
 *   w_down    [E, d, inter] bf16   down_proj
 *   y         [T*k, d]      bf16   out, in row (permuted) order
 * bf16 x bf16 -> fp32 on tcgen05 tensor cores; the intermediate
 * silu(gate) * up is rounded to bf16.  The shared expert is the case E = 1,
 * k = 1, row_token = 0..T-1, offsets = {0, T}.  A row_token entry outside
 * [0, T) is not read: it is recorded as MOE_ERR_INVALID_ARG in the device
 * status, that row of y is unspecified, and every other row is unaffected.
 */
int moe_expert_ffn(const uint16_t* x, const int32_t* row_token, const int32_t* offsets,
                   const uint16_t* w_gate_up, const uint16_t* w_down, int T, int d, int E, int k,
                   int inter, uint16_t* y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Combine, step 7 ("Kimi K2.5 deep dive", CH10.2; "Kimi K2.5 Q&A", Q8.3):
 *     out[t] = y_shared[t] + sum_{j<k} topk_w[t, j] * y[slot_row[t*k + j]]
 * accumulated in fp32 in slot order j = 0..k-1 (deterministic), rounded
 * once to bf16.
 *   y        [T*k, d] bf16   routed expert outputs in row order
 *   y_shared [T, d]   bf16   shared expert output, or NULL for none
 *   topk_w   [T, k]   fp32   (already includes the scaling factor)
 *   slot_row [T*k]    int32
 *   out      [T, d]   bf16
 */
int moe_combine(const uint16_t* y, const uint16_t* y_shared, const float* topk_w,
                const int32_t* slot_row, int T, int d, int k, uint16_t* out, void* stream);

/*
 * The whole layer in one call: route -> permute -> grouped SwiGLU experts
 * (routed and shared in the same grouped launches) -> combine
 * ("Kimi K2.5 deep dive", CH10.2 steps 1-7).
 *   x          [T, d]            bf16
 *   w_router   [E, d]            bf16
 *   bias       [E]               fp32
 *   w_gate_up  [E, 2*inter, d]   bf16  routed experts, gate rows then up rows
 *   w_down     [E, d, inter]     bf16
 *   ws_gate_up [2*inter, d]      bf16  shared expert
 *   ws_down    [d, inter]        bf16
 *   out        [T, d]            bf16
 * Scratch is library-owned: one buffer per (device, stream), grown with
 * cudaMallocAsync on `stream` when a larger layer arrives and kept for later
 * calls (MOE_ERR_NO_MEMORY if growth fails).  Calls on one stream are
 * ordered; calls on different streams use different buffers.
 */
int moe_layer_forward(const uint16_t* x, const uint16_t* w_router, const float* bias,
                      const uint16_t* w_gate_up, const uint16_t* w_down,
                      const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d, int E,
                      int k, int inter, float scale, uint16_t* out, void* stream);

/*
 * moe_layer_forward with caller-owned scratch of at least
 * moe_workspace_size(T, d, E, k, inter) bytes (nothing is allocated).
 * The _ws entries (this one, _fp8_ws, _w4a16_ws, _w8a8_ws) neither allocate nor
 * synchronise the host, so a call can be captured into a CUDA graph on
 * `stream` and replayed; make one call on the device outside the capture first
 * (it sets up the kernels' attributes).  A replay uses the pointers and sizes
 * of the captured call.
 */
int moe_layer_forward_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                         const uint16_t* w_gate_up, const uint16_t* w_down,
                         const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                         int E, int k, int inter, float scale, uint16_t* out, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Size, in bytes, of the scratch array inside the library that
 * moe_layer_forward_noalloc works in (32 MiB). */
#define MOE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * moe_layer_forward for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry point: it exists for deployment.
 *
 * Some callers must not call cudaMalloc / cudaMallocAsync.  A serving engine
 * that has reserved nearly all HBM for weights and its KV cache hands its
 * plugins no allocator.  A latency-critical loop cannot accept the device-wide
 * synchronisation that cudaMalloc may cause.  A deployment with an audited,
 * fixed memory plan forbids allocation after start-up.  Such callers pass
 * only their inputs and outputs (same arguments and layouts as
 * moe_layer_forward), and the scratch comes from one array of
 * MOE_NOALLOC_SCRATCH_BYTES compiled into the library.  Every GPU that loads
 * the library holds that array until the process exits.  This call itself
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 *   - Size limit: if the layer needs more scratch than the array holds
 *     (moe_workspace_size(T, d, E, k, inter) > MOE_NOALLOC_SCRATCH_BYTES), the
 *     call returns MOE_ERR_UNSUPPORTED_SHAPE before launching anything.  With
 *     K2 shapes (d = 7168, E = 384, k = 8, inter = 2048) that allows up to
 *     T = 97 tokens; decode batches fit, prefill batches do not.
 *   - First call in a CUDA context: it looks up the array's device address
 *     with cudaGetSymbolAddress, in the context current on the calling thread,
 *     and caches it under that context's unique id (a non-primary context, or
 *     a context made after cudaDeviceReset, gets a lookup of its own).  Make
 *     that first call before any stream capture begins.
 *   - Sharing: every call on every stream of a device uses the same array, and
 *     the array keeps the previous call's contents.  No kernel reads scratch it
 *     has not written earlier in the same call, so nothing needs clearing.
 *     Calls that overlap on the GPU (different streams, or host threads
 *     launching at the same time) race on the array and corrupt each other's
 *     results: order them on one stream or serialise them.
 */
int moe_layer_forward_noalloc(const uint16_t* x, const uint16_t* w_router, const float* bias,
                              const uint16_t* w_gate_up, const uint16_t* w_down,
                              const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                              int E, int k, int inter, float scale, uint16_t* out, void* stream);

/*
 * FP8 storage of the routed experts' weights ("Kimi K2.5 Q&A", Q7.1: the
 * routed experts' weight storage is quantized while compute stays in BF16;
 * the shared experts are exempt).  The pages give no format; this library
 * uses E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * largest finite 448, NaN at 0x7F/0xFF, no infinities) with one power-of-two
 * scale 2^s per block of 128 rows x 128 columns, s an int8:
 *     s = smallest integer with max|w| <= 448 * 2^s over the block, clamped to
 *         [-124, 127] (0 for an all-zero block);
 *     q = the E4M3 value nearest to w * 2^-s, ties to even.
 * q * 2^s is exactly representable in bf16, so the FP8 layer computes with
 * exactly the weights the codes stand for (bf16 tensor-core math, as in
 * moe_layer_forward).  Weights must be finite with |w| < 2^120.
 *
 * moe_quantize_fp8: w [rows, cols] bf16 row-major (rows and cols multiples of
 * 128, cols / 128 <= 65535) -> q [rows, cols] uint8 codes and
 * exps [rows/128, cols/128] int8 exponents, all device memory owned by the
 * caller, asynchronous on `stream`.  Stacked expert weights quantize in one
 * call: [E, 2*inter, d] as rows = E*2*inter, cols = d (exps [E, 2*inter/128,
 * d/128]); [E, d, inter] as rows = E*d, cols = inter.
 * Returns MOE_ERR_UNSUPPORTED_SHAPE for other shapes, MOE_ERR_INVALID_ARG for
 * null or unaligned (16-byte) pointers.
 */
int moe_quantize_fp8(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, int8_t* exps,
                     void* stream);

/*
 * The layer of moe_layer_forward with the routed experts' weights in FP8
 * (codes and exponents from moe_quantize_fp8):
 *   wq_gate_up [E, 2*inter, d] uint8, wq_gate_up_exp [E, 2*inter/128, d/128] int8
 *   wq_down    [E, d, inter]   uint8, wq_down_exp    [E, d/128, inter/128]   int8
 * Everything else (router, shared expert, activations, output) is as in
 * moe_layer_forward, bf16.  d and inter must be multiples of 128.  Decode-
 * sized batches (T*k <= 4*E) dequantize the routed weights in registers for
 * warp-level tensor-core MMAs; larger batches dequantize them in shared memory
 * just before the tcgen05 tensor cores read them.  Both compute with the same
 * weights, code * 2^s exactly, and nothing in HBM holds a bf16 copy.  Decode-
 * sized batches run the shared expert's tiles on a second stream of the calling
 * thread (created on first use, one per thread and CUDA context), forked from
 * `stream` by an event and joined back into it by another before the combine:
 * the call stays ordered on `stream` and can be captured in a CUDA graph.  Errors as in
 * moe_layer_forward.  The _ws form takes a caller-owned workspace of
 * moe_workspace_size(T, d, E, k, inter) bytes, like moe_layer_forward_ws.
 */
int moe_layer_forward_fp8(const uint16_t* x, const uint16_t* w_router, const float* bias,
                          const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                          const uint8_t* wq_down, const int8_t* wq_down_exp,
                          const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                          int E, int k, int inter, float scale, uint16_t* out, void* stream);
int moe_layer_forward_fp8_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                             const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                             const uint8_t* wq_down, const int8_t* wq_down_exp,
                             const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                             int E, int k, int inter, float scale, uint16_t* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * INT4 storage of the routed experts' weights ("Kimi K2.5 deep dive", CH7.2:
 * the K2.5 quantization config, 4-bit symmetric integers in groups of 32 along
 * K, shared experts exempt; "Kimi K2.5 Q&A", Q7.1: storage quantized, compute
 * BF16).  The config gives no scale rule or type; this library's (per group
 * of 32 consecutive elements of a row):
 *     s = bf16(amax / 7), nearest-even;
 *     q = clamp(nearest integer to w / s, ties to even, -8, 7), 0 when s = 0;
 * and the layer computes with the bf16 weights bf16(q * s) (nearest-even),
 * bf16 tensor-core math as in moe_layer_forward.
 *
 * moe_quantize_int4: w [rows, cols] bf16 row-major (cols a multiple of 64) ->
 *   codes  [rows, cols/2] bytes: in each 32-bit little-endian word j of a row,
 *          element 8j+2i sits in bits 4i..4i+3 and element 8j+2i+1 in bits
 *          16+4i..16+4i+3, each stored as q + 8;
 *   scales [cols/32, rows] bf16, group-major (one row of scales per group).
 * Caller-owned device memory, asynchronous on `stream`.  Stacked experts
 * quantize in one call: [E, 2*inter, d] as rows = E*2*inter (scales
 * [d/32, E*2*inter]); [E, d, inter] as rows = E*d (scales [inter/32, E*d]).
 * MOE_ERR_UNSUPPORTED_SHAPE for other shapes, MOE_ERR_INVALID_ARG for null or
 * unaligned (16-byte) pointers.
 *
 * moe_layer_forward_w4a16: the layer of moe_layer_forward with the routed
 * experts' weights as (codes, scales) from moe_quantize_int4; router, shared
 * expert, activations and output bf16 as there.  Decode-sized batches
 * (T*k <= 4*E, d and inter multiples of 256) dequantize the codes in registers
 * for warp-level tensor-core MMAs; other batches dequantize them in shared
 * memory just before the tcgen05 tensor cores read them.  Both compute with
 * the same weights bf16(q * s).  Decode-sized batches use a second stream for
 * the shared expert's tiles as moe_layer_forward_fp8 does.  Errors as in
 * moe_layer_forward; the _ws form takes moe_workspace_size(T, d, E, k, inter)
 * bytes.
 */
int moe_quantize_int4(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* codes,
                      uint16_t* scales, void* stream);
int moe_layer_forward_w4a16(const uint16_t* x, const uint16_t* w_router, const float* bias,
                            const uint8_t* wq_gate_up, const uint16_t* wq_gate_up_scale,
                            const uint8_t* wq_down, const uint16_t* wq_down_scale,
                            const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                            int E, int k, int inter, float scale, uint16_t* out, void* stream);
int moe_layer_forward_w4a16_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                               const uint8_t* wq_gate_up, const uint16_t* wq_gate_up_scale,
                               const uint8_t* wq_down, const uint16_t* wq_down_scale,
                               const uint16_t* ws_gate_up, const uint16_t* ws_down, int T, int d,
                               int E, int k, int inter, float scale, uint16_t* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * FP8 compute ("Kimi K2.5 Q&A", Q7.1 names DeepSeek-V3's "compute in FP8" next
 * to K2.5's quantized storage; "Kimi K2 deep dive", 3.2: FP8 for speed).  The
 * pages give no format; this library's: E4M3 codes (as above) with one
 * power-of-two exponent per ROW, s an int8 chosen by the rule above over the
 * row (smallest integer with max|row| <= 448 * 2^s, clamped to [-124, 127], 0
 * for an all-zero row), q = E4M3 nearest to w * 2^-s, ties to even.  A weight
 * row is an output channel, an activation row a token, so both exponents
 * factor out of each dot product: the tensor cores multiply codes
 * (E4M3 x E4M3 -> fp32) and the result is scaled by 2^(s_w + s_x) exactly.
 *
 * moe_quantize_fp8_rows: w [rows, cols] bf16 row-major (cols a multiple of 16)
 * -> q [rows, cols] uint8 codes and exps [rows] int8, caller-owned device
 * memory, asynchronous on `stream`.  Stacked experts quantize in one call:
 * [E, 2*inter, d] as rows = E*2*inter (exps [E, 2*inter]), [E, d, inter] as
 * rows = E*d (exps [E, d]).  MOE_ERR_UNSUPPORTED_SHAPE for other shapes,
 * MOE_ERR_INVALID_ARG for null or unaligned (16-byte) w or q, or null exps.
 *
 * moe_layer_forward_w8a8: the layer with FP8 compute in every expert, routed
 * and shared (the router and top-k stay as in moe_layer_forward, bf16 / fp32):
 *   wq_gate_up [E, 2*inter, d] uint8 + wq_gate_up_exp [E, 2*inter] int8
 *   wq_down    [E, d, inter]   uint8 + wq_down_exp    [E, d]       int8
 *   wsq_gate_up   [2*inter, d] uint8 + wsq_gate_up_exp   [2*inter]  int8
 *   wsq_down      [d, inter]   uint8 + wsq_down_exp      [d]        int8
 * all from moe_quantize_fp8_rows (exponents outside [-124, 127] are not
 * supported).  Per expert and token row:
 *   x_t -> per-row E4M3 (codes, s_x);
 *   g_n = 2^(s_gn + s_x) codes . codes, u_n likewise (fp32 accumulation);
 *   h_n = bf16(silu(g_n) * u_n);  h -> per-row E4M3 (codes, s_h);
 *   y_o = 2^(s_do + s_h) codes . codes;
 * then the routing weights combine the y rows as in moe_layer_forward.  d and
 * inter must be multiples of 128.  Errors as in moe_layer_forward.  The _ws
 * form takes a caller-owned workspace of moe_workspace_size_w8a8(T, d, E, k,
 * inter) bytes (0 for unsupported dimensions), 16-byte aligned.
 */
int moe_quantize_fp8_rows(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q,
                          int8_t* exps, void* stream);
size_t moe_workspace_size_w8a8(int T, int d, int E, int k, int inter);
int moe_layer_forward_w8a8(const uint16_t* x, const uint16_t* w_router, const float* bias,
                           const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                           const uint8_t* wq_down, const int8_t* wq_down_exp,
                           const uint8_t* wsq_gate_up, const int8_t* wsq_gate_up_exp,
                           const uint8_t* wsq_down, const int8_t* wsq_down_exp, int T, int d,
                           int E, int k, int inter, float scale, uint16_t* out, void* stream);
int moe_layer_forward_w8a8_ws(const uint16_t* x, const uint16_t* w_router, const float* bias,
                              const uint8_t* wq_gate_up, const int8_t* wq_gate_up_exp,
                              const uint8_t* wq_down, const int8_t* wq_down_exp,
                              const uint8_t* wsq_gate_up, const int8_t* wsq_gate_up_exp,
                              const uint8_t* wsq_down, const int8_t* wsq_down_exp, int T, int d,
                              int E, int k, int inter, float scale, uint16_t* out,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Expert load balancing ("Kimi K2.5 Q&A", Q7.2; "Kimi K2.5 deep dive", CH10.2
 * step 2): the selection bias is a buffer outside the gradient, lowered for
 * over-loaded experts and raised for under-loaded ones, and a weak
 * sequence-level balance loss (aux_loss_alpha = 0.001 in the pages) backs it up.
 *
 * moe_bias_update: one loss-free balancing step from a step's loads.
 *   counts [E] int32 device  rows each expert received (moe_permute's counts;
 *                           they sum to T*k)
 *   bias   [E] fp32  device  updated in place, in fp32:
 *       bias[e] -= gamma  if counts[e] * E > T * k   (above the mean load)
 *       bias[e] += gamma  if counts[e] * E < T * k   (below it)
 *       unchanged         if counts[e] * E == T * k
 * The pages give no rate; gamma is the caller's.  Asynchronous on `stream`.
 * Errors: MOE_ERR_UNSUPPORTED_SHAPE for E or k out of range, MOE_ERR_INVALID_ARG
 * for T < 0, null pointers or a NaN gamma.  T == 0 changes nothing.
 */
int moe_bias_update(const int32_t* counts, int T, int E, int k, float gamma, float* bias,
                    void* stream);

/*
 * moe_router_scores: the unbiased sigmoid scores of every expert,
 *   scores[t, e] = sigmoid(x[t] . w_router[e])   [T, E] fp32, device,
 * the same fp32 values the top-k selection of moe_route starts from (fp32
 * accumulation over d, split-K partials added in a fixed order).  Scratch:
 * workspace of moe_workspace_size(T, d, E, k, inter) bytes for any k, inter.
 * Errors as in moe_route.
 */
int moe_router_scores(const uint16_t* x, const uint16_t* w_router, int T, int d, int E,
                      float* scores, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_seq_aux_loss: the sequence-level balance loss over B sequences of S
 * tokens (rows b*S .. b*S+S-1).  The pages give alpha but no formula; this is
 * the sequence-wise balance loss of the DeepSeek-V3 line that K2 continues:
 *   f_i = E / (k S) * #{t in sequence : i in topk(t)}
 *   P_i = (1 / S) * sum_t scores[t, i] / sum_j scores[t, j]
 *   loss[b] = alpha * sum_i f_i * P_i
 *   scores [B*S, E] fp32 (moe_router_scores), topk_idx [B*S, k] int32 (moe_route);
 *   loss [B] fp32; f, p [B, E] fp32 or NULL; all device memory; workspace of
 *   moe_seq_aux_workspace_size(B, S, E) bytes (16-byte aligned, caller-owned).
 * fp32 with fixed reduction orders (deterministic).  Errors:
 * MOE_ERR_UNSUPPORTED_SHAPE for E or k out of range, MOE_ERR_INVALID_ARG for
 * B < 0, S < 1, null pointers, NaN alpha or a short workspace; an out-of-range
 * index is recorded in the device status and skipped.
 */
size_t moe_seq_aux_workspace_size(int B, int S, int E);
int moe_seq_aux_loss(const float* scores, const int32_t* topk_idx, int B, int S, int E, int k,
                     float alpha, float* loss, float* f, float* p, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the current device's status word:
 * *device_status = MOE_OK, or the first problem a kernel recorded since the
 * last read (MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT).  Returns MOE_OK or
 * MOE_ERR_CUDA if the synchronisation itself failed.
 */
int moe_device_status(void* stream, int* device_status);

/*
 * Upper bound, in nanoseconds, on every device-side wait of the library's
 * kernels (default 2e9 = 2 s).  A wait that runs out records MOE_ERR_TIMEOUT,
 * and the kernel winds down and returns instead of hanging.
 */
void moe_set_wait_timeout_ns(uint64_t timeout_ns);

/*
 * Programmatic dependent launch (default off).  With enable = 1, every kernel of
 * a call after its first may be scheduled while the call's previous kernel is
 * still running; it runs its set-up (barriers, tensor memory, descriptor
 * prefetch) meanwhile and waits for that kernel before reading any result.
 * The first kernel of every call waits for whatever the stream held before,
 * and so does every kernel that follows an event wait (the decode GEMMs' second
 * stream and its join).  Results are the same either way.  Applies to launches
 * issued after the call (process-wide).  With several host threads sharing one
 * stream it is untested and best left off.
 */
void moe_set_pdl(int enable);

/*
 * Failure-detection self-test: launches one block that waits on an mbarrier
 * nobody arrives on, bounded by `timeout_ns`.  The wait runs out, the kernel
 * records MOE_ERR_TIMEOUT and returns; the context stays usable.
 */
int moe_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Kernels the last layer call (any moe_layer_forward* entry) launched. */
int moe_last_launch_count(void);

/*
 * Optional per-kernel timing of layer calls with CUDA events (measurement
 * support; no counterpart in the method).  After moe_profile_begin(n), the
 * next n calls of moe_layer_forward / moe_layer_forward_ws on the current
 * device record one event before their first kernel and one after each
 * kernel, on the call's stream (all moe_layer_forward* entries).
 * moe_profile_end synchronises those events, writes into total_ms[i]
 * (i < max_kernels) the summed time of kernel slot i (moe_kernel_name) over
 * the recorded calls, stores the number of recorded calls in *n_calls, frees
 * the events and returns the number of slots per call (or a negative
 * moe_status).  A slot a call has no kernel for (quantize_h outside FP8
 * compute) sums to zero.
 */
int moe_profile_begin(int max_calls);
int moe_profile_end(float* total_ms, int max_kernels, int* n_calls);

/* Name of kernel slot i of a layer call ("" if out of range). */
const char* moe_kernel_name(int i);

/*
 * Expert parallelism ("K2 inference engineer's answer", 2.1: the deployment
 * spreads the routed experts over many GPUs, EP = 128, two or three experts per
 * rank for DeepSeek-V3 and about 10 GB of expert weights per rank for K2, with
 * data parallelism over tokens; 2.4: n_group = 1, so any token may select any
 * rank's experts).  R ranks; rank q owns the E_l = E / R routed experts
 * [q E_l, (q + 1) E_l) (E a multiple of R); the router, the bias and the shared
 * expert are replicated; every rank routes its own T tokens.  One layer call on
 * every rank is:
 *   1. moe_ep_dispatch: route, permute and gather the rank's token rows into
 *      send_rows [T*k, d], expert-major (expert e's rows from offsets of
 *      `counts`), so the rows for rank q are the contiguous block of experts
 *      [q E_l, (q + 1) E_l);
 *   2. the caller exchanges the per-expert counts ([R][E_l] ints, all-to-all)
 *      and the rows (all-to-all with those splits), e.g. NCCL over NVLink;
 *      the received rows are source-major: source 0's rows grouped by local
 *      expert, then source 1's, ...;
 *   3. moe_ep_expert_ffn: the rank's experts on the received rows, outputs in
 *      the received order;
 *   4. the caller returns the outputs to their sources (the reverse all-to-all);
 *      each source gets back exactly its send_rows' order;
 *   5. moe_ep_combine: the shared expert on the rank's own tokens plus
 *      out[t] = y_shared[t] + sum_j topk_w[t, j] * y_back[slot_row[t*k + j]].
 * Each row's arithmetic is that of moe_layer_forward (same kernels, same K
 * order), so a rank's output equals moe_layer_forward on its own tokens bit
 * for bit.  All pointers are device memory owned by the caller, every call is
 * asynchronous on `stream`, errors as in moe_layer_forward; workspaces are sized
 * by the matching *_workspace_size function (0 for unsupported shapes).
 *
 * moe_ep_dispatch: x [T, d], router and bias as in moe_route -> topk_idx [T, k],
 * topk_w [T, k], counts [E] (rows per expert), slot_row [T*k] (as in
 * moe_permute), send_rows [T*k, d] bf16.
 */
size_t moe_ep_dispatch_workspace_size(int T, int d, int E, int k);
int moe_ep_dispatch(const uint16_t* x, const uint16_t* w_router, const float* bias, int T, int d,
                    int E, int k, float scale, int32_t* topk_idx, float* topk_w, int32_t* counts,
                    int32_t* slot_row, uint16_t* send_rows, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * moe_ep_expert_ffn: recv_rows [rows, d] bf16 as received (source-major) with
 * recv_counts [R, E_l] int32 (device; row counts per source and local expert,
 * summing to `rows`; R * E_l <= 1024), the rank's experts' weights
 * w_gate_up [E_l, 2*inter, d] and w_down [E_l, d, inter] (layouts of
 * moe_layer_forward) -> y [rows, d] bf16, row i = its expert applied to
 * received row i.  Inside: the rows are regrouped expert-major (expert e's rows
 * from source 0, then source 1, ... each in its source's order), run through
 * the grouped SwiGLU GEMMs and put back in the received order.  A count total
 * other than `rows` is recorded in the device status word (MOE_ERR_INVALID_ARG)
 * and y is all zeros.
 */
size_t moe_ep_expert_ffn_workspace_size(int rows, int d, int R, int E_local, int inter);
int moe_ep_expert_ffn(const uint16_t* recv_rows, const int32_t* recv_counts, int rows, int d, int R,
                      int E_local, int inter, const uint16_t* w_gate_up, const uint16_t* w_down,
                      uint16_t* y, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_ep_combine: y_back [T*k, d] bf16 (the expert outputs of this rank's
 * send_rows, in send_rows' order), x [T, d], the shared expert's ws_gate_up
 * [2*inter, d] and ws_down [d, inter], topk_w and slot_row from
 * moe_ep_dispatch -> out [T, d] bf16.
 */
size_t moe_ep_combine_workspace_size(int T, int d, int inter);
int moe_ep_combine(const uint16_t* y_back, const uint16_t* x, const uint16_t* ws_gate_up,
                   const uint16_t* ws_down, const float* topk_w, const int32_t* slot_row, int T,
                   int d, int k, int inter, uint16_t* out, void* workspace, size_t workspace_bytes,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
