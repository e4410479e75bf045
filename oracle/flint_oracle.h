/*
 * flint_oracle.h -- plain fp64 CPU oracle of one Flint MoE layer's decode step.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load or call this library. The product path
 * (libflint_moe.so and its Python binding) never links, imports or runs it, and
 * the two share no code, header, table or constant generator.
 *
 * What it computes, and where the definition comes from:
 *  - Mixture of experts with 256 routed experts, 6 picked per token, plus one
 *    always-on shared expert: "Recursive Flint: 40B Local Coding Model,
 *    Benchmarks", architecture table (Experts row); "Run the Flint coding model
 *    on a CPU VPS", section "What Flint is, from the model card".
 *  - Weight-only NVFP4 (W4A16) experts: "[Model] Add Flint (RecursiveSI/flint)",
 *    section "What happened" (NVFP4 checkpoint served weight-only as W4A16);
 *    NVFP4 is NVIDIA's 4-bit floating-point format ("Run the Flint coding model
 *    on a CPU VPS", section "Which Flint tag to pull on a CPU VPS").
 *  - The pages fix no bit layout, gating, FFN type or shapes. The layer
 *    contract supplies them: E2M1 values, one E4M3 scale per 16 elements along
 *    K, one FP32 tensor scale; softmax over all routed logits, top-k with ties
 *    to the lower index, gates renormalised to sum 1, shared expert weight 1;
 *    SwiGLU experts (gate/up d->I, down I->d, no biases).
 *  - E2M1 / E4M3 bit meanings follow the public OCP Microscaling (MX) v1.0
 *    element formats (FP4 E2M1; FP8 E4M3 "fn": no infinities, S.1111.111 NaN).
 *  - The attention prologue (fused Q/K normalisation + rotary embedding +
 *    KV-cache write): "[Model] Add Flint (RecursiveSI/flint)", section "What
 *    happened"; grouped-query attention with 32 query and 4 key/value heads of
 *    dimension 128, rotary positions on the sliding-window layers and none on
 *    the full-attention layers: "Recursive Flint: 125 tok/s on an M4 Pro",
 *    architecture table. The pages fix no norm type or rotary layout: RMS
 *    normalisation over the head dimension with a learned weight, and rotation
 *    of pairs (i, i + Dh/2) by a caller-supplied cos/sin table.
 *  - Decode attention over the cache (same page and table): grouped-query
 *    softmax attention, query head h reading key/value head h / (Hq / Hkv),
 *    scale 1/sqrt(Dh), over a caller-given range of cache rows per token.
 *
 * Precision: every arithmetic step of the forward pass runs in fp64; weights
 * are decoded exactly (e2m1 * e4m3 * fp32 tensor scale fits in 53 bits).
 * The quantiser runs in IEEE fp32 round-to-nearest (the recipe fixes fp32),
 * built with -ffp-contract=off so no multiply-add is fused.
 */
#ifndef FLINT_ORACLE_H
#define FLINT_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One weight matrix in the oracle's plain ("natural") layout.
 *   kind 0 (NVFP4): codes [rows][cols/2], element 2j in the low nibble of byte j,
 *                   scales [rows][cols/16] E4M3 bytes, block b = elements 16b..16b+15,
 *                   tensor_scale = the fp32 per-tensor scale.
 *   kind 1 (BF16):  bf16 [rows][cols] bit patterns.
 * Unused experts may be left with NULL pointers. */
typedef struct oracle_matrix {
  int32_t kind;
  int32_t rows;
  int32_t cols;
  float tensor_scale;
  const uint8_t* codes;
  const uint8_t* scales;
  const uint16_t* bf16;
} oracle_matrix;

/* ---- element codecs (OCP MX v1.0 element formats) ---- */
double oracle_e2m1_decode(uint8_t code);
double oracle_e4m3_decode(uint8_t code);
/* Round-to-nearest-even, saturating to +-6; the sign of v is kept (so -0 -> 0x8). */
uint8_t oracle_e2m1_encode(float v);
/* Round-to-nearest-even, saturating to +-448; the sign of v is kept. */
uint8_t oracle_e4m3_encode(float v);
/* Round-to-nearest-even fp64 -> bf16 bit pattern (finite inputs). */
uint16_t oracle_bf16_from_double(double v);
double oracle_bf16_to_double(uint16_t bits);

/* ---- NVFP4 quantiser (the recipe, fp32) ----
 * s_t = amax/2688 (1 if amax == 0); per block sb = E4M3((amax_b/6)/s_t);
 * q = E2M1(w / (dec(sb)*s_t)), and q = 0 for every element of a block whose
 * scale decodes to 0. Writes natural-layout planes. Returns 0, or -1 when the
 * shape is not a multiple of 16 along cols or w holds a non-finite value. */
int oracle_quantize_nvfp4(const float* w, int32_t rows, int32_t cols,
                          uint8_t* codes, uint8_t* scales, float* tensor_scale);

/* The same recipe for some rows of a larger tensor whose amax (the largest
 * |w| over the whole tensor) is given: s_t = amax/2688, then the rows' blocks
 * as above. Returns -1 if a row value is non-finite or exceeds amax. */
int oracle_quantize_nvfp4_rows(const float* w, int32_t rows, int32_t cols, float amax,
                               uint8_t* codes, uint8_t* scales, float* tensor_scale);

/* Decode one matrix to fp64 [rows][cols] (NVFP4: e2m1*e4m3*s_t; BF16: exact). */
int oracle_decode_matrix(const oracle_matrix* m, double* out);

/* ---- the product's packed HBM layout, restated from its definition ----
 * Expert e (routed 0..E-1, then the n_shared shared experts) owns a contiguous
 * region in each array. Codes: I units of [gate row u | up row u] (d/2 bytes
 * each), then d down rows of I/2 bytes. Scales: the same rows in the same
 * order, d/16 resp. I/16 bytes per row. Tensor scales: [expert][gate,up,down].
 * mats holds (E+S)*3 natural-layout NVFP4 matrices: gate [I][d], up [I][d],
 * down [d][I] per expert. */
int oracle_pack_layout(const oracle_matrix* mats, int32_t n_experts_total,
                       int32_t d, int32_t inter, uint8_t* packed_codes,
                       uint8_t* packed_scales, float* tensor_scales);
/* The same row order for bf16 weights: [gate row u | up row u] (d bf16 each),
 * then d down rows of I bf16. */
int oracle_pack_layout_bf16(const oracle_matrix* mats, int32_t n_experts_total,
                            int32_t d, int32_t inter, uint16_t* packed);

/* ---- routing ---- */
/* logits[t][e] = sum_j x[t][j] * W_r[e][j] in fp64; x [T][d], W_r [E][d] bf16. */
int oracle_router_logits(const uint16_t* x, int32_t T, const uint16_t* wr,
                         int32_t d, int32_t E, double* logits);
/* Per token: softmax over all E logits; the k experts with the largest logit
 * (ties to the lower index); gates = their probabilities renormalised to 1.
 * gap[t] = p_(k) - p_(k+1) of the full softmax (k-th minus (k+1)-th largest),
 * or +inf when k == E. */
int oracle_topk(const double* logits, int32_t T, int32_t E, int32_t k,
                int32_t* ids, double* gates, double* gap);

/* Grouping of the routed selections by expert (the layer contract's "expert
 * histogram + token permutation"): the experts that at least one token
 * selected, in ascending id order, then the n_shared shared experts E..E+S-1;
 * for each, its (token, slot) pairs as token << 8 | slot in ascending token
 * order (a token selects an expert at most once), the shared experts serving
 * every token in slot k + s; off[a] = index of expert a's first pair, off[n]
 * = total. ids [T][k]. act holds up to E + S entries, off up to E + S + 1,
 * pair T*(k+S). Writes *n_routed (routed experts in use) and returns the
 * number of active experts, or -1 if an id lies outside [0, E) or T > 65536. */
int32_t oracle_group(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t S,
                     int32_t* act, int32_t* off, int32_t* pair, int32_t* n_routed);

/* Expert-parallel dispatch plan (expert parallelism over the GPUs of one node,
 * "[Model] Add Flint (RecursiveSI/flint)", section "What happened"): the send
 * order of the T (k + S) (token, slot) pairs by destination rank (rank r holds
 * routed experts [r E/R, (r+1) E/R); shared slots stay on `rank`), ascending
 * pair index within a rank; per send row its local expert id, gate and
 * source token; per rank its row count; per pair its send position (-1 for an
 * id outside [0, E)). Returns the dropped pairs, or -1 for bad sizes. */
int32_t oracle_ep_plan(const int32_t* ids, const float* gates, int32_t T, int32_t k, int32_t S, int32_t E,
                       int32_t R, int32_t rank, int32_t* send_ids, float* send_gates, int32_t* send_token,
                       int32_t* counts, int32_t* pair_pos);

/* ---- dense NVFP4 matrix-vector product (the 4-bit output head) ----
 * out[t][i] = sum_c w[rows[i]][c] * x[t][c] in fp64, w = e2m1 * e4m3 * s_t of
 * the NVFP4 matrix m (natural layout), x bf16 [T][m->cols]. rows (nullable)
 * picks n_rows of the matrix's rows (all rows in order when NULL, n_rows =
 * m->rows). Returns 0, or -1 on a bad argument. */
int oracle_dense_gemv(const oracle_matrix* m, const uint16_t* x, int32_t T, const int32_t* rows,
                      int32_t n_rows, double* out);

/* ---- experts ---- */
/* Dense SwiGLU FFN of one expert: y = W_d (silu(W_g x) * (W_u x)).
 * mats = {gate [I][d], up [I][d], down [d][I]}. */
int oracle_expert_ffn(const oracle_matrix* mats, int32_t d, int32_t inter,
                      const double* x, double* y);

/* Whole layer. mats: (E+S)*3 matrices (unused experts may be NULL-pointered).
 * out = sum_j gate_j * FFN_{id_j}(xn) + sum_s FFN_{E+s}(xn) (+ residual), fp64,
 * where xn = x, or with input_norm = 1 the weightless RMS normalisation
 * xn = x / sqrt(mean(x^2) + 1e-6) that also feeds the router.
 * ids_override (nullable) forces the routed ids (gates then come from those
 * experts' probabilities, renormalised). ids/gates/gap/logits outputs nullable.
 * n_threads >= 1 spreads the independent (token, expert) FFNs over threads;
 * the arithmetic and its order do not depend on it. */
int oracle_moe_forward(int32_t T, int32_t d, int32_t inter, int32_t E, int32_t k,
                       int32_t S, const uint16_t* x, const uint16_t* wr,
                       const oracle_matrix* mats, const uint16_t* residual,
                       const int32_t* ids_override, int32_t input_norm, int32_t n_threads,
                       int32_t* ids_out, double* gates_out, double* gap_out,
                       double* logits_out, double* out);

/* ---- attention prologue ---- */
/* Fused Q/K RMS normalisation + rotary embedding + key/value pass-through of
 * one layer's QKV projection qkv [T][Hq + 2*Hkv][Dh] bf16 (query heads, key
 * heads, value heads). Query/key heads: y = x / sqrt(mean(x^2) + eps) * w
 * (w = q_w or k_w, bf16 [Dh]); with rope, pairs (i, i + Dh/2) rotated by the
 * position's row of cs [max_pos][Dh] fp32 (cos in columns 0..Dh/2-1, sin in
 * Dh/2..Dh-1). fp64 outputs q [T][Hq][Dh], k, v [T][Hkv][Dh]. Returns 0, or -1
 * on a bad argument or a position outside [0, max_pos). */
int oracle_qk_norm_rope_kv(int32_t T, int32_t Hq, int32_t Hkv, int32_t Dh, const uint16_t* qkv, const uint16_t* q_w,
                           const uint16_t* k_w, const float* cs, int32_t max_pos, const int32_t* positions,
                           int32_t rope, double eps, double* q_out, double* k_out, double* v_out);

/* Decode attention (fp64): query token t, head h attends to cache rows
 * start[t] .. start[t] + len[t] - 1 of key/value head h / (Hq / Hkv):
 * o = softmax(scale * q . k) v. q bf16 [T][Hq][Dh]; k, v bf16 [rows][Hkv][Dh];
 * out fp64 [T][Hq][Dh] (zeros for len 0). Returns 0, or -1 on a bad argument
 * or a range outside [0, rows). */
int oracle_decode_attention(int32_t T, int32_t Hq, int32_t Hkv, int32_t Dh, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, int64_t rows, const int64_t* start, const int32_t* len, double scale,
                            double* out);

#ifdef __cplusplus
}
#endif
#endif
