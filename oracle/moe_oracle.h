/*
 * moe_oracle.h -- plain, slow, fp64 CPU oracle for one Kimi-K2-style MoE FFN
 * layer (forward pass).  TEST INFRASTRUCTURE ONLY: only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load this library.  The
 * product path (the CUDA library) never calls it and shares no code with it.
 *
 * What it computes, step by step, as the pages give it:
 *   "Kimi K2.5 deep dive", CH4.2 (routing) and CH10.2 (MoE 7-step dataflow):
 *     1. s = sigmoid(x . W_router^T)                       (scoring_func=sigmoid)
 *     2. b = s + e_score_correction_bias                   (selection-only bias)
 *     3. top-k of b over all E experts (n_group = 1, "K2 inference" answer, 2.4)
 *     4. weights = s_sel / sum(s_sel), then * routed_scaling_factor
 *     5. shared expert on every token, unscaled
 *     6. routed experts: SwiGLU y = W_down (silu(W_gate x) * (W_up x))
 *     7. out = shared + sum_j w_j * y_j
 *   "Kimi K2.5 Q&A" Q8.3 gives the same order (router -> shared || routed -> add).
 *
 * Readings where the pages are silent or disagree:
 *   - step 4 uses the UNBIASED sigmoid scores (the bias only picks experts);
 *   - ties in step 3 go to the lower expert index; slot j = j-th largest b;
 *   - no epsilon in the renormalisation (a sum of k sigmoids is > 0);
 *   - every token gets exactly k experts (no capacity, no dropping);
 *   - within an expert, rows are in ascending token order (the per-expert mask
 *     of the pages' dispatch loop visits tokens in order).
 *
 * Precision: bf16 inputs are widened exactly to double; all arithmetic is fp64;
 * results are returned in fp64.  bf16 values travel as their uint16 bit pattern.
 *
 * Parity pins (what checks this oracle against something other than itself)
 * live in tests/test_oracle_pins.py.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 bit pattern -> double (exact). */
double oracle_bf16_to_f64(uint16_t v);
/* double -> bf16 bit pattern, one rounding, to nearest, ties to even. */
uint16_t oracle_f64_to_bf16(double v);
/* bulk version of the rounding above */
void oracle_round_bf16(const double* in, uint16_t* out, size_t n);

double oracle_sigmoid(double z);           /* 1 / (1 + exp(-z)) */
double oracle_silu(double z);              /* z * sigmoid(z) */

/*
 * Router (steps 1-4) for T tokens.
 *   x [T,d] bf16, w_router [E,d] bf16 (Linear out x in), bias [E] fp32.
 *   topk_idx [T,k] int32  (slot j = j-th largest biased score, ties -> lower e)
 *   topk_w   [T,k] double (scale * s_sel / sum s_sel, unbiased s)
 *   scores   [T,E] double sigmoid scores, optional (NULL)
 *   gap      [T]   double b_(k) - b_(k+1) (biased, sorted), +inf if k == E; optional
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_route(const uint16_t* x, const uint16_t* w_router, const float* bias,
                 int T, int d, int E, int k, double scale,
                 int32_t* topk_idx, double* topk_w, double* scores, double* gap,
                 int nthreads);

/*
 * Permutation of the (token, slot) pairs into expert-contiguous rows.
 *   counts[e]   = #{(t,j): idx[t,j] == e}
 *   offsets     = exclusive prefix sum of counts, offsets[E] = T*k
 *   rows of expert e are offsets[e] .. offsets[e+1]-1, in ascending token order
 *   row_token[row] = t,  slot_row[t*k + j] = row
 * Returns 0, or -1 if an index is out of range or a token repeats an expert.
 */
int oracle_permute(const int32_t* topk_idx, int T, int E, int k,
                   int32_t* counts, int32_t* offsets, int32_t* row_token, int32_t* slot_row);

/*
 * One SwiGLU expert on one token row:
 *   y[d] = W_down (silu(W_gate x) * (W_up x)),  w_gate_up [2I,d] (gate rows then
 *   up rows), w_down [d,I].  act (optional) receives the I-vector
 *   silu(W_gate x) * (W_up x).
 */
void oracle_swiglu_row(const uint16_t* xrow, const uint16_t* w_gate_up, const uint16_t* w_down,
                       int d, int inter, double* y, double* act);

/*
 * Combine (step 7) given expert outputs in permuted row order:
 *   out[t] = y_shared[t] + sum_j topk_w[t,j] * y[slot_row[t*k+j]]
 * y [T*k, d], y_shared [T, d] (or NULL), all double.
 */
void oracle_combine(const double* y, const double* y_shared, const double* topk_w,
                    const int32_t* slot_row, int T, int d, int k, double* out);

/*
 * Whole layer on a subset of tokens (rows are independent, so any subset gives
 * the same rows as the full batch).
 *   expert_gate_up[e] -> [2I,d] bf16 of routed expert e, expert_down[e] -> [d,I];
 *   pointers of experts no listed token selects may be NULL.
 *   tokens [n_tokens] : which rows of x to evaluate (NULL = all T, n_tokens = T)
 *   topk_idx/topk_w   : routing of ALL T tokens (from oracle_route)
 *   out [n_tokens, d] double
 * Returns 0, or -1 if a needed expert pointer is NULL.
 */
int oracle_moe_rows(const uint16_t* x, int T, int d, int E, int k, int inter,
                    const int32_t* topk_idx, const double* topk_w,
                    const uint16_t* const* expert_gate_up, const uint16_t* const* expert_down,
                    const uint16_t* shared_gate_up, const uint16_t* shared_down,
                    const int32_t* tokens, int n_tokens, double* out, int nthreads);

/*
 * FP8 storage of the routed experts' weights.
 *
 * "Kimi K2.5 Q&A", Q7.1: what the deployment quantizes is the routed experts'
 * weight storage, while compute stays in BF16 ("storage quantization + high-
 * precision compute"); the shared experts are exempt and stay BF16.  The
 * pages name FP8 as the other storage option ("Kimi K2 deep dive", 3.2:
 * FP8 halves the memory) but give no format.  The format taken here:
 *   - element: FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 *     exponent 0 holds subnormals m * 2^-9; code 0x7F / 0xFF is NaN; largest
 *     finite value 448; no infinities);
 *   - one scale per block of 128 rows x 128 columns (K), a power of two 2^s
 *     with s an int8, so dequantization q * 2^s is exact in bf16;
 *   - s = the smallest integer with amax <= 448 * 2^s (amax = largest |w| of
 *     the block), clamped to [-124, 127]; s = 0 for an all-zero block;
 *   - q = the E4M3 value nearest to w * 2^-s (ties to even; w * 2^-s is exact).
 */

/* E4M3 code of v, nearest value, ties to even; |v| > 448 saturates to +-448,
 * NaN -> 0x7F. */
uint8_t oracle_e4m3_encode(double v);
/* Value of an E4M3 code (NaN for 0x7F / 0xFF). */
double oracle_e4m3_decode(uint8_t code);
/* Block exponent s for a block whose largest magnitude is amax (rule above). */
int oracle_fp8_block_exponent(double amax);
/*
 * Quantize a bf16 matrix w [rows, cols] (row-major; rows and cols multiples of
 * 128) into codes q [rows, cols] and block exponents sexp [rows/128, cols/128].
 * Returns 0, or -1 if a dimension is not a multiple of 128.
 */
int oracle_quantize_fp8(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, int8_t* sexp);
/*
 * Dequantize: w_out[r, c] = bf16( decode(q[r, c]) * 2^sexp[r/128, c/128] ), a
 * value that bf16 holds exactly whenever it is finite.  Returns 0 or -1 as above.
 */
int oracle_dequantize_fp8(const uint8_t* q, const int8_t* sexp, int64_t rows, int64_t cols,
                          uint16_t* w_out);

/*
 * INT4 storage of the routed experts' weights ("Kimi K2.5 deep dive", CH7.2: the
 * K2.5 quantization config, 4-bit integer weights, strategy "group" with
 * group_size 32, symmetric; shared experts on the ignore list stay BF16;
 * "Kimi K2.5 Q&A", Q7.1: storage quantized, compute BF16).  The config gives
 * neither the scale rule nor the scale type; the plainest symmetric reading:
 *   - a group is 32 consecutive K elements of one weight row;
 *   - s = bf16( amax / 7 ) (amax = largest |w| of the group; the quotient taken
 *     in fp64, then rounded to nearest-even bf16);
 *   - q = clamp( nearest integer to w / s, ties to even, -8, 7 ), q = 0 when s = 0;
 *   - the weight the model computes with is bf16( q * s ) (the exact product
 *     rounded to nearest-even bf16), then the bf16 layer as usual.
 * q [rows, cols] int8 in [-8, 7]; scale [rows, cols/32] bf16 bits.
 * Returns 0, or -1 if cols is not a multiple of 32.
 */
int oracle_quantize_int4(const uint16_t* w, int64_t rows, int64_t cols, int8_t* q,
                         uint16_t* scale);
/* w_out[r, c] = bf16( q[r, c] * scale[r, c / 32] ).  Returns 0 or -1 as above. */
int oracle_dequantize_int4(const int8_t* q, const uint16_t* scale, int64_t rows, int64_t cols,
                           uint16_t* w_out);

/*
 * FP8 compute ("Kimi K2.5 Q&A", Q7.1 names V3's "compute in FP8" beside K2.5's
 * quantized storage; "Kimi K2 deep dive", 3.2: FP8 for speed).  The pages give
 * no format.  The one taken for FP8 compute: E4M3 operands with one power-of-two
 * scale per ROW (each weight row = output channel, each activation row = token),
 * chosen by the rule above (s = smallest integer with row amax <= 448 * 2^s,
 * clamped to [-124, 127]); the scales then factor out of every K sum.
 */

/* Per-row quantization: w [rows, cols] bf16 -> q [rows, cols], sexp [rows]. */
void oracle_quantize_fp8_rows(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q,
                              int8_t* sexp);

/*
 * One expert on one token row in FP8 compute:
 *   x row -> (xq, sx) per-row quantization of the bf16 row
 *   g_n = 2^(sg_n + sx) sum_i dec(wq_gu[n, i]) dec(xq_i),  u_n likewise (row inter + n)
 *   h_n = bf16( silu(g_n) * u_n )            (the stored intermediate)
 *   (hq, sh) = per-row quantization of h
 *   y_o = 2^(sd_o + sh) sum_n dec(wq_dn[o, n]) dec(hq_n)
 * wq_gu [2I, d] + s_gu [2I]; wq_dn [d, I] + s_dn [d].  y in fp64.
 */
void oracle_swiglu_row_fp8(const uint16_t* xrow, const uint8_t* wq_gu, const int8_t* s_gu,
                           const uint8_t* wq_dn, const int8_t* s_dn, int d, int inter, double* y);

/*
 * Whole layer, FP8 compute for every expert (routed and shared), on a subset of
 * tokens; routing (topk_idx, topk_w) from oracle_route on the bf16 router.
 * expert_* arrays of pointers as in oracle_moe_rows (NULL for unused experts).
 */
int oracle_moe_rows_fp8(const uint16_t* x, int T, int d, int E, int k, int inter,
                        const int32_t* topk_idx, const double* topk_w,
                        const uint8_t* const* egu_q, const int8_t* const* egu_s,
                        const uint8_t* const* edn_q, const int8_t* const* edn_s,
                        const uint8_t* sgu_q, const int8_t* sgu_s, const uint8_t* sdn_q,
                        const int8_t* sdn_s, const int32_t* tokens, int n_tokens, double* out,
                        int nthreads);

/*
 * Load balancing ("Kimi K2.5 Q&A", Q7.2; "Kimi K2.5 deep dive", CH10.2 step 2).
 *
 * Bias update (noaux_tc): the selection bias is a buffer, not learned; after a
 * step, experts that took more than their share of the step's T*k routed rows
 * have their bias lowered by gamma, experts that took less have it raised, and
 * an expert exactly at the mean T*k/E keeps it.  The pages give neither the
 * rate nor the comparison; the reading: a fixed step gamma (an argument), the
 * load compared with the mean exactly (counts[e]*E against T*k), the update
 * done in the buffer's own precision: bias[e] = fp32(bias[e] -/+ gamma).
 */
void oracle_bias_update(const int32_t* counts, int T, int E, int k, float gamma, float* bias);

/*
 * Sequence-level auxiliary balance loss (seq_aux = true, aux_loss_alpha).  The
 * pages name it and give alpha = 0.001 but not the formula; the reading is the
 * sequence-wise balance loss of the DeepSeek-V3 line the pages say K2 continues:
 * for each sequence b of S tokens,
 *   f_i = E / (k * S) * #{t in b : i in topk(t)}
 *   P_i = (1 / S) * sum_{t in b} s_{t,i} / sum_j s_{t,j}     (sigmoid affinities)
 *   L_b = alpha * sum_i f_i * P_i
 * scores [B*S, E] (sigmoid s), topk_idx [B*S, k]; out: loss [B], and optionally
 * f [B, E], p [B, E].  fp64 throughout.
 */
void oracle_seq_aux_loss(const double* scores, const int32_t* topk_idx, int B, int S, int E,
                         int k, double alpha, double* loss, double* f, double* p);

#ifdef __cplusplus
}
#endif
#endif /* MOE_ORACLE_H */
