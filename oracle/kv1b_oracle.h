/*
 * kv1b_oracle.h -- plain, slow CPU oracle for decode attention over a compressed KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call this.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm use it.
 * It shares no code, header, table or constant with the CUDA library under
 * long_context_decode_kv1b_b200/csrc.
 *
 * Sources (web pages; see oracle/kv1b_oracle.cpp for the per-function citations):
 *   - "RaBitQCache: Rotated Binary Quantization for KVCache in Long Context LLM Inference"
 *     (abstract; method sections "core idea", "technical framework", "key design"):
 *     random rotation + binary quantization of keys, binary-INT4 arithmetic for an unbiased
 *     estimate of q.k, adaptive Top-p retrieval.
 *   - "H1B-KV: Hybrid One-Bit Caches for Memory-Efficient Large Language Model Inference"
 *     (abstract; "technical framework", "key design"): 1-bit key sketch by random projection,
 *     4-bit linear quantization of values, attention weights from the sketch then values.
 *   - "Hybrid one-bit cache: H1IB-KV" news article, part 2 item 3 "hardware-friendly storage optimisation":
 *     bitmap storage, bit (i mod 8) of byte (i / 8), bit 1 <-> +1 and bit 0 <-> -1.
 *
 * All arrays are plain host memory, row-major, owned by the caller.  d (head_dim) must be a
 * power of two with d >= 32.  Functions never allocate memory visible to the caller and never
 * throw; invalid sizes return a negative value where a return value exists.
 */
#ifndef KV1B_ORACLE_H
#define KV1B_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* SplitMix64 (Steele, Lea, Flood 2014): advances *state and returns the next output. */
uint64_t ref_splitmix64_next(uint64_t* state);

/* Rotation signs D[0..d): state = seed; D[i] = (next() >> 63) ? -1 : +1. */
void ref_rotation_signs(uint64_t seed, int d, float* signs);

/* Stronger rotation: `rounds` (1..3) successive H * diag(D_r); signs receives 3 x d entries, round r
 * = outputs r d .. r d + d - 1 of one SplitMix64 stream, unused rounds 0.  Every function below
 * that takes `signs` reads 3 x d entries and applies the rounds up to the first all-zero one. */
void ref_rotation_signs_rounds(uint64_t seed, int d, int rounds, float* signs);

/* Unnormalised Walsh-Hadamard transform in natural (Sylvester) order, in place, fp32,
 * butterfly stages h = 1, 2, 4, ..., d/2, each (a, c) -> (a + c, a - c). */
void ref_fwht(float* x, int d);

/* fp32 sum of a[0..d) by the fixed pairwise tree: for h = d/2 .. 1: a[i] += a[i + h], i < h.
 * Works on a copy; returns a[0]. */
float ref_tree_sum(const float* a, int d);

/* Key sketch of one token.  k: d floats.  signs: d floats (+-1).
 * bits: d/32 words, bit i of word w = (y[32w+i] >= 0) with y = FWHT(D*k).
 * norm = sqrt(tree sum k_i^2); cinv = (d*norm) / (tree sum |y_i|), or 1 if that sum is 0. */
void ref_encode_key(const float* k, const float* signs, int d, uint32_t* bits, float* norm, float* cinv);

/* 4-bit value codes of one token.  v: d floats.
 * codes: d/8 words, nibble j of word w = code of channel 8w+j.
 * sm: d/32 words, low half = fp16 bits of scale, high half = fp16 bits of min, per 32-channel group.
 * Returns a flag word: bit 0 = non-finite input, bit 1 = fp16 saturation of min or scale. */
int ref_encode_value(const float* v, int d, uint32_t* codes, uint32_t* sm);

/* The two encoders above applied to L consecutive tokens (rows of K / V, d floats each).
 * ref_encode_values returns the OR of the per-token flag words. */
void ref_encode_keys(const float* K, int64_t L, const float* signs, int d, uint32_t* bits, float* norm, float* cinv);
int ref_encode_values(const float* V, int64_t L, int d, uint32_t* codes, uint32_t* sm);

/* Dequantised value of one token in fp64: out[c] = min_g + scale_g * code_c. */
void ref_dequant_value(const uint32_t* codes, const uint32_t* sm, int d, double* out);

/* fp16 bits -> double (exact). */
double ref_half_to_double(uint16_t h);

/* Query preparation for one head.  q: d floats.
 * z = FWHT(D*q); vl = min z; delta = (max z - vl) / 15; code_i = min(15, floor((z_i - vl)/delta + 0.5))
 * (0 when delta == 0).  planes: 4 x (d/32) words, plane j bit i of word w = bit j of code[32w+i].
 * codes (may be NULL): d bytes.  Sq = sum of codes.  z_out (may be NULL): d floats. */
void ref_query_prep(const float* q, const float* signs, int d, uint32_t* planes, float* vl, float* delta,
                    int32_t* Sq, uint8_t* codes, float* z_out);

/* Binary x INT4 integers for one (token, head): A = sum_j 2^j sum_w popc(bits_w & P_jw),
 * Bc = sum_w popc(bits_w). */
void ref_score_ints(const uint32_t* bits, const uint32_t* planes, int d, int32_t* A, int32_t* Bc);

/* ref_score_ints for L consecutive tokens: bits [L][d/32], A and Bc [L]. */
void ref_score_ints_n(const uint32_t* bits, int64_t L, const uint32_t* planes, int d, int32_t* A, int32_t* Bc);

/* Estimated logit from the integers, fp32, fixed op order:
 * I1 = 2Bc - d, I2 = 2A - Sq, dot = fl(fl(delta*I2) + fl(vl*I1)), s = fl(fl(dot * fl(norm*cinv)) * (scale/d)). */
float ref_logit(int32_t A, int32_t Bc, int32_t Sq, float vl, float delta, float norm, float cinv, float scale, int d);

/* Logits of all L tokens of one (sequence, kv-head) for one query head (planes from ref_query_prep). */
void ref_logits(const uint32_t* bits, const float* norm, const float* cinv, int64_t L, const uint32_t* planes,
                float vl, float delta, int32_t Sq, float scale, int d, float* s_out);

/* Full decode attention for one query head over L encoded tokens, fp64 softmax and accumulation:
 * m = max s; e_t = exp(s_t - m); out = sum_t e_t * vhat_t / sum_t e_t.  L == 0 gives zeros. */
void ref_attend_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                     const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale, int d,
                     double* out);

/* The fp32 coefficient c_k ~ (ln 2)^k / k! used by the Top-p integer weights, k = 0..7. */
float ref_exp2_coef(int k);

/* Integer Top-p weight of one token: t = fl(fl(s - m) * log2e); u = 0 if t < -40, else with
 * n = rint(t), f = t - n, P = Horner(c_7..c_0, f) with fused multiply-adds,
 * u = trunc(P * 2^(32+n)) as an unsigned 64-bit integer. */
uint64_t ref_topp_weight(float s, float m);

/* Top-p selection over logits s[0..L): order (s desc, index asc); U = sum u; T = ceil(p*U) (fp64),
 * clamped to [1, U]; N = smallest k >= 1 whose prefix mass >= T.  sel receives the N selected
 * indices in ascending order; returns N (0 when L == 0, -1 when p is not in (0, 1]). */
int64_t ref_topp_select(const float* s, int64_t L, float p, int64_t* sel);

/* Top-p attention for one query head: selection as ref_topp_select, then fp64 softmax over the
 * selected tokens' logits and their dequantised values.  Returns N (or -1). */
int64_t ref_attend_topp_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                             const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale,
                             float p, int d, int64_t* sel, double* out);

/* Token selection with a mass threshold or a fixed budget, plus an always-kept window (RaBitQCache
 * abstract: adaptive Top-p against a fixed Top-k budget; H1IB-KV article part 2 item 1: a
 * high-precision layer for the important tokens -- read here as the first `sink` and the last
 * `recent` tokens).  W = {t < sink} U {t >= L - recent}.  mode 0 (Top-p): masses u_t as
 * ref_topp_weight with m = max over all L tokens, T = ceil(p U) clamped to [1, U],
 * need = T - sum_{t in W} u_t; the shortest prefix of the other tokens in (s desc, index asc) order
 * whose mass reaches need (nothing when need <= 0).  mode 1 (Top-k): the first min(k, L - |W|) other
 * tokens in that order.  sel receives W and the chosen tokens in ascending order; returns their
 * number, or -1 on an invalid mode / p / k / sink / recent. */
int64_t ref_select(const float* s, int64_t L, int mode, float p, int64_t k, int64_t sink, int64_t recent,
                   int64_t* sel);

/* Attention over a ref_select set for one query head: fp64 softmax over the selected tokens'
 * estimated logits and dequantised values (as ref_attend_topp_head).  Returns the set size or -1. */
int64_t ref_attend_select_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                               const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale,
                               int mode, float p, int64_t k, int64_t sink, int64_t recent, int d, int64_t* sel,
                               double* out);

/* Exact attention over a selected token set (RaBitQCache, abstract / core idea: the proxy scores
 * retrieve the tokens, attention over them is then sparse attention with the exact keys and
 * values).  q: [d]; K, V: [L][d] as fp32 (the exact values of the caller's keys and values);
 * sel: n indices into [0, L) (any order, no repeats).  z_t = scale * sum_c q_c K_tc in fp64;
 * out = sum_t softmax(z)_t V_t in fp64 over t in sel; zeros when n == 0.  Returns 0, or -1 when an
 * index is out of range or d is not positive. */
int ref_attend_exact_selected(const float* q, const float* K, const float* V, int64_t L, int d, const int64_t* sel,
                              int64_t n, float scale, double* out);

#ifdef __cplusplus
}
#endif
#endif
