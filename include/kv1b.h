/*
 * kv1b.h -- C ABI of the B200 (sm_100a) library for decode attention over a compressed KV cache.
 *
 * What the library computes (pages cited by title and section):
 *  - Keys are kept as 1-bit sign sketches of a seeded random rotation, with a per-token norm and
 *    correction scalar ("RaBitQCache: Rotated Binary Quantization for KVCache in Long Context LLM
 *    Inference", abstract and core idea: randomised rotated binary quantisation; "H1B-KV: Hybrid
 *    One-Bit Caches ...", key design: 1-bit sketch by random projection).  The rotation is
 *    y = H * (D (.) k): H the unnormalised 128x128 Walsh-Hadamard matrix in natural order, D a
 *    +-1 vector from SplitMix64(seed).  Bit i of word w is 1 iff y[32w+i] >= 0 (the bitmap rule of
 *    the H1IB-KV news article, part 2 item 3: a set bit stands for +1).
 *  - Values are 4-bit linear codes with an fp16 scale and an fp16 min per 32 channels (H1B-KV,
 *    key design: 4-bit linear quantisation of values).
 *  - Attention logits are estimated with binary x INT4 popcount arithmetic between the key bits
 *    and the 4 bit-planes of the rotated, 4-bit-quantised query (RaBitQCache abstract and key
 *    design); the output is the softmax-weighted sum of the dequantised values (H1B-KV,
 *    technical framework), either over all tokens (kv1b_attend) or over the adaptive Top-p set
 *    (kv1b_attend_topp; RaBitQCache abstract: adaptive Top-p retrieval).
 *
 * Conventions (every entry point):
 *  - All data pointers are DEVICE pointers unless a parameter says "host".  The caller owns every
 *    buffer; the library never allocates device memory and keeps no state outside the
 *    kv1b_cache_t descriptor the caller holds.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every call that
 *    launches work is asynchronous on that stream, except kv1b_read_status (synchronous).
 *  - Return value: KV1B_OK (0) or a negative KV1B_ERR_* code.  Arguments are validated on the
 *    host before any launch; on error nothing is launched and no buffer is written.  No C++
 *    exception crosses the ABI.  Conditions only the device can see (non-finite inputs, fp16
 *    saturation of a value group) set bits in the cache's status word (kv1b_read_status).
 *  - head_dim must be 128.  capacity must be a positive multiple of 128.  batch <= 64.
 *    num_q_heads must be a multiple of num_kv_heads with G = num_q_heads / num_kv_heads <= 8;
 *    query head hq reads KV head hq / G.
 */
#ifndef KV1B_H
#define KV1B_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KV1B_HEAD_DIM 128
#define KV1B_MAX_BATCH 64
#define KV1B_MAX_GROUP 8
#define KV1B_MAX_ROUNDS 3  /* rotation rounds H * diag(D_r) a cache may use (kv1b_cache_init_rounds) */
#define KV1B_CAPACITY_ALIGN 128

/* return codes */
#define KV1B_OK 0
#define KV1B_ERR_INVALID_ARG (-1)      /* null pointer, bad count, p not in (0,1], Hq % Hkv != 0 ... */
#define KV1B_ERR_UNSUPPORTED (-2)      /* head_dim != 128, G > 8, batch > 64 */
#define KV1B_ERR_CAPACITY (-3)         /* an append would exceed the capacity */
#define KV1B_ERR_MISALIGNED (-4)       /* a pointer or stride breaks the alignment rule stated below */
#define KV1B_ERR_WORKSPACE (-5)        /* workspace or cache buffer smaller than required */
#define KV1B_ERR_CUDA (-6)             /* a CUDA launch/runtime error (cudaGetLastError) */

/* element types of K, V and q */
#define KV1B_DTYPE_F32 0
#define KV1B_DTYPE_BF16 1
#define KV1B_DTYPE_F16 2

/* kv1b_attend flags: which engine forms the probability-weighted sum of values */
#define KV1B_ATTEND_TENSOR 0     /* default: integer mma.sync (u8 codes x 32-bit fixed-point weights, exact s32
                                    accumulation) in a persistent kernel, for equal sequence lengths and an
                                    automatic split count (G > 4 as launches of at most 4 query heads, each
                                    streaming the cache); other shapes run the CUDA-core engine */
#define KV1B_ATTEND_CUDA_CORE 1  /* fp32 FMA on the CUDA cores (split-K grid, any shape) */
#define KV1B_ATTEND_WS_CLEAN 2   /* OR-ed into the engine: the workspace's merge counters are zero, as every
                                    kv1b_attend that ran to completion on this workspace with the same cache
                                    shape (batch, kv heads, capacity) and num_q_heads leaves them, so the call
                                    does not zero them first (saves a memset and lets the attend kernel start
                                    while its predecessor in the stream finishes).  Do not pass it for a new
                                    workspace, one used with another shape or written by anything else, or
                                    after KV1B_STATUS_TIMEOUT. */
#define KV1B_ATTEND_PARTIAL 4    /* OR-ed into the engine: out receives log-sum-exp partial rows instead of the
                                    normalised output, f32 [batch][num_q_heads][2 + 128] = (m, l, o[128]) with
                                    l = sum_t 2^(s_t log2(e) - m) and o = sum_t 2^(s_t log2(e) - m) vhat_t for a
                                    reference m in log2 units (the row's largest s_t log2(e), or at most 4 below
                                    it; m = -inf, l = 0, o = 0 for an empty sequence): the attention of this
                                    cache's tokens in a form that kv1b_merge_partials combines with the rows of
                                    other token ranges of the same sequences (a context split over GPUs). */

/* kv1b_attend_select modes */
#define KV1B_SELECT_TOPP 0  /* smallest set reaching a fraction p of the estimated attention mass */
#define KV1B_SELECT_TOPK 1  /* a fixed budget of k tokens */

/* status word bits (kv1b_read_status) */
#define KV1B_STATUS_NONFINITE 1       /* a K or V element appended was NaN or Inf */
#define KV1B_STATUS_FP16_SATURATED 2  /* a value group's min or scale left the binary16 range */
#define KV1B_STATUS_TIMEOUT 4         /* an attend kernel's bounded pipeline wait ran out (results invalid) */
#define KV1B_STATUS_BAD_INDEX 8       /* kv1b_attend_selected_exact met a selected index outside the valid
                                         tokens; that entry was skipped */

/*
 * Cache descriptor.  Filled by kv1b_cache_init; treat as opaque except for reading the fields.
 * Device planes (carved from one caller buffer, token-major within each (sequence, kv-head)):
 *   k_bits  u32 [batch][hkv][capacity][4]     sign bits of the rotated key (16 B / token)
 *   k_norm  f32 [batch][hkv][capacity]        N = ||k|| (fixed pairwise tree sum of squares)
 *   k_cinv  f32 [batch][hkv][capacity]        1/C = 128 N / sum_i |y_i| (1 when the sum is 0)
 *   v_codes u32 [batch][hkv][capacity/128][128][16]  4-bit value codes in 128-token tiles, one
 *           64-byte row per channel: nibble j (bits 4j..4j+3) of word w of row (tile T, channel c)
 *           is the code of token 128T + 8w + j, channel c.  One tile is one TMA box of 4-bit
 *           elements that the tensor-core engine expands to a byte per code in shared memory.
 *   v_sm    u32 [batch][hkv][capacity][4]     per 32-channel group: low half = fp16 scale,
 *           high half = fp16 min; value = min + scale * code
 *   signs   f32 [3][128]                      rotation signs D_r (+-1) of each round; 0 for the
 *                                             rounds past rotation_rounds
 *   d_lengths i32 [batch]                     tokens held per sequence (device copy)
 *   d_status  i32 [1]                         OR of KV1B_STATUS_* bits since init
 * h_lengths is the host mirror of d_lengths; both change only through kv1b_encode_append.
 */
typedef struct kv1b_cache {
  int32_t batch;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t capacity;
  uint64_t rotation_seed;
  uint32_t* k_bits;
  float* k_norm;
  float* k_cinv;
  uint32_t* v_codes;
  uint32_t* v_sm;
  float* signs;
  int32_t* d_lengths;
  int32_t* d_status;
  int64_t h_lengths[KV1B_MAX_BATCH];
  int32_t rotation_rounds;  /* 1 (kv1b_cache_init) to KV1B_MAX_ROUNDS (kv1b_cache_init_rounds) */
  int32_t reserved;
} kv1b_cache_t;

/* Bytes of device memory a cache of this shape needs (0 if the shape is unsupported). */
size_t kv1b_cache_bytes(int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t capacity);

/* Lay a cache out in the caller's device buffer `dev_buf` (256-byte aligned, `bytes` >=
 * kv1b_cache_bytes), zero it, draw the rotation signs from SplitMix64(seed) and set all lengths
 * to 0.  Writes the descriptor *cache (host memory).  Asynchronous on `stream`. */
int kv1b_cache_init(kv1b_cache_t* cache, void* dev_buf, size_t bytes, int32_t batch, int32_t num_kv_heads,
                    int32_t head_dim, int32_t capacity, uint64_t seed, void* stream);

/* kv1b_cache_init with a stronger rotation: `rounds` (1..KV1B_MAX_ROUNDS) successive H * diag(D_r)
 * applied to keys and queries (a closer stand-in for RaBitQ's random orthogonal rotation, whose
 * unbiasedness the RaBitQCache abstract relies on).  Round r's signs are outputs 128 r .. 128 r + 127
 * of the same SplitMix64(seed) stream, so rounds = 1 is kv1b_cache_init.  The estimator needs no
 * other change: C^-1 = 128 N / sum|y| and the query grid both scale with the rotation.  Every later
 * call reads the rounds from the cache.  KV1B_ERR_INVALID_ARG for rounds outside 1..3. */
int kv1b_cache_init_rounds(kv1b_cache_t* cache, void* dev_buf, size_t bytes, int32_t batch, int32_t num_kv_heads,
                           int32_t head_dim, int32_t capacity, uint64_t seed, int32_t rounds, void* stream);

/* Encode and append n_new tokens to every sequence (the same n_new for all).
 * k, v: device arrays of `dtype` (KV1B_DTYPE_*); element (b, t, h, c) of K sits at
 * k[b*stride_b + t*stride_t + h*stride_h + c] (strides in elements, channel stride 1); V uses
 * the same strides.  Alignment rule: k and v 16-byte aligned; stride_b, stride_t, stride_h
 * multiples of 4 elements (so every 4-channel slice is an aligned vector).
 * Per (sequence, token, kv-head): rotation + sign bits + N + 1/C, and 4-bit value codes with an
 * fp16 min (rounded down) and fp16 scale (smallest with 15*scale >= range).  The tokens land at
 * positions h_lengths[b] .. h_lengths[b]+n_new-1, then lengths advance (host mirror and device).
 * Errors: KV1B_ERR_CAPACITY when h_lengths[b] + n_new > capacity for some b. */
int kv1b_encode_append(kv1b_cache_t* cache, const void* k, const void* v, int32_t dtype, int32_t n_new,
                       int64_t stride_b, int64_t stride_t, int64_t stride_h, void* stream);

/* Workspace bytes kv1b_attend (mode 0), kv1b_attend_topp (mode 1) or kv1b_attend_selected_exact
 * (mode 2) needs for this cache and
 * num_q_heads at any length up to the capacity.  0 on invalid arguments. */
size_t kv1b_attend_workspace_bytes(const kv1b_cache_t* cache, int32_t num_q_heads, int32_t mode);

/* Full decode attention over all cached tokens.
 * q: [batch][num_q_heads][128] contiguous, `q_dtype`, 16-byte aligned.
 * out: f32 [batch][num_q_heads][128].  For each (b, hq): with logits s_t estimated from the
 * key sketch (binary x INT4 popcount) and scaled by `scale`, out = sum_t softmax(s)_t * vhat_t,
 * vhat = min + scale_g * code.  A sequence of length 0 gives zeros.
 * ws: device workspace, 256-byte aligned, ws_bytes >= kv1b_attend_workspace_bytes(.., 0).
 * flags: KV1B_ATTEND_TENSOR (default) or KV1B_ATTEND_CUDA_CORE (same result within fp32
 * rounding), optionally | KV1B_ATTEND_WS_CLEAN and | KV1B_ATTEND_PARTIAL (then out is
 * [batch][num_q_heads][2 + 128], see above); any other bit is KV1B_ERR_INVALID_ARG.
 * num_splits: 0 chooses the split-K factor; > 0 forces it (testing).
 * The kernels are launched with programmatic stream serialization: they may be scheduled while the
 * previous kernel in `stream` finishes, and wait for it before touching memory. */
int kv1b_attend(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                float* out, void* ws, size_t ws_bytes, int32_t flags, int32_t num_splits, void* stream);

/* Fixed size of the device array behind kv1b_attend_noalloc (4 MiB on every GPU that loads the
 * library, held until the process exits). */
#define KV1B_NOALLOC_SCRATCH_BYTES (4u << 20)

/* kv1b_attend without a workspace and without any allocation.  (The pages describe nothing like
 * it; it exists for this library's users.)  For callers that can neither allocate device memory
 * (their framework's allocator owns it, or cudaMalloc/cudaFree would synchronise a
 * latency-critical decode loop) nor pass a workspace buffer (a fixed ABI with inputs and outputs
 * only).  Same arguments and result as kv1b_attend minus ws / ws_bytes / num_splits; flags is
 * KV1B_ATTEND_TENSOR or KV1B_ATTEND_CUDA_CORE (KV1B_ATTEND_WS_CLEAN is not accepted).
 * KV1B_ATTEND_TENSOR runs the persistent tensor-core kernel where kv1b_attend would (equal sequence
 * lengths) and its partial rows fit the array, otherwise the CUDA-core split-K
 * engine, which KV1B_ATTEND_CUDA_CORE always runs.  The partial rows and merge counters go to a
 * file-scope device array of KV1B_NOALLOC_SCRATCH_BYTES instead of a workspace; each call zeroes
 * the counters it uses with one small memset on `stream`.
 * The first call on a device (and the first after a new context replaced the old one) looks up that
 * array's device address (cudaGetSymbolAddress, with the device current) and caches it; make that
 * first call before any stream capture.  Every call shares the array: calls whose kernels may
 * overlap on the GPU race, so order them on one stream (or otherwise).  A shape whose split-K
 * partials do not fit (batch * num_q_heads * splits * 520 bytes > the array; splits <= 2 * SMs /
 * (batch * num_kv_heads)) returns KV1B_ERR_WORKSPACE before launching anything.  Calls no
 * cudaMalloc / cudaFree. */
int kv1b_attend_noalloc(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                        float* out, int32_t flags, void* stream);

/* Adaptive Top-p decode attention.  Per (b, hq): integer masses u_t ~ 2^32 exp(s_t - max s)
 * (degree-7 polynomial for 2^f, reproducible bit for bit), T = ceil(p * sum u) in fp64; the
 * selected set is the shortest prefix of the order (s desc, index asc) whose mass reaches T.
 * sel_idx: i32 [batch][num_q_heads][capacity] receives the selected token indices in ascending
 * order (entries past sel_cnt are left unspecified); sel_cnt: i32 [batch][num_q_heads].
 * out: f32 [batch][num_q_heads][128], the softmax over the selected tokens only.
 * p must be in (0, 1].  ws_bytes >= kv1b_attend_workspace_bytes(.., 1). */
int kv1b_attend_topp(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                     float p, float* out, int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                     void* stream);

/* Top-p or Top-k selection plus an always-kept window, then attention over the set.
 * (RaBitQCache abstract: adaptive Top-p, contrasted with a fixed Top-k budget; H1IB-KV article part 2
 * item 1: a high-precision layer for important tokens, read here as the first `sink` and the last
 * `recent` tokens of each sequence.)  Per (b, hq), with W = {t < sink} U {t >= length[b] - recent}
 * and the order (s desc, index asc) of the other tokens:
 *   KV1B_SELECT_TOPP: masses u_t as kv1b_attend_topp (m = max over all tokens), T = ceil(p U) in
 *     fp64 over all tokens, clamped to [1, U]; the set is W plus the shortest prefix of the other
 *     tokens whose mass reaches T - mass(W) (nothing when W already reaches T);
 *   KV1B_SELECT_TOPK: W plus the first min(k, number of other tokens) of them.
 * Outputs and workspace as kv1b_attend_topp (sel_idx ascending, sel_cnt, out = the softmax over the
 * set of the estimated logits with the 4-bit values; ws >= kv1b_attend_workspace_bytes(.., 1)).
 * mode must be one of the two; p in (0, 1] for Top-p; k >= 0 for Top-k; sink, recent >= 0.
 * kv1b_attend_topp(.., p, ..) is kv1b_attend_select(.., KV1B_SELECT_TOPP, p, 0, 0, 0, ..). */
int kv1b_attend_select(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                       int32_t mode, float p, int32_t k, int32_t sink, int32_t recent, float* out, int32_t* sel_idx,
                       int32_t* sel_cnt, void* ws, size_t ws_bytes, void* stream);

/* Exact attention over a selected token set ("RaBitQCache", abstract / core idea: the binary x INT4
 * proxy scores retrieve the tokens -- e.g. kv1b_attend_topp's sel_idx / sel_cnt -- and attention
 * over them uses the exact keys and values).  For each (b, hq), with S = sel_idx[b][hq][0 ..
 * sel_cnt[b][hq]) and kv-head kvh = hq / (num_q_heads / num_kv_heads):
 *   z_t = scale * sum_c q_c k_{b,t,kvh,c},  out[b][hq] = sum_{t in S} softmax(z)_t v_{b,t,kvh}
 * in fp32 (logits in log2 units, online softmax, fixed-order log-sum-exp merge); zeros when S is
 * empty.
 * k, v: the exact keys and values, `kv_dtype` (KV1B_DTYPE_*); element (b, t, h, c) at offset
 *   b*stride_b + t*stride_t + h*stride_h + c elements (channels contiguous); device memory or host
 *   memory the device can address (mapped pinned / managed).  Base addresses 16-byte aligned and
 *   strides multiples of 8 elements; kv_tokens = tokens per sequence the arrays hold.
 * q: [batch][num_q_heads][128] contiguous, `q_dtype`, 16-byte aligned.
 * sel_idx: i32 [batch][num_q_heads][capacity]; sel_cnt: i32 [batch][num_q_heads] (<= capacity).
 *   An index outside [0, min(length[b], kv_tokens)) is skipped and sets KV1B_STATUS_BAD_INDEX.
 * out: f32 [batch][num_q_heads][128].  ws: kv1b_attend_workspace_bytes(.., 2) bytes, 256-aligned.
 * The caller owns every buffer; the call only launches work on `stream`. */
int kv1b_attend_selected_exact(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                               float scale, const void* k, const void* v, int32_t kv_dtype, int64_t kv_tokens,
                               int64_t stride_b, int64_t stride_t, int64_t stride_h, const int32_t* sel_idx,
                               const int32_t* sel_cnt, float* out, void* ws, size_t ws_bytes, void* stream);

/* Test hook for the query preparation step: planes u32 [batch][num_q_heads][4][4] (plane j,
 * word w, bit i = bit j of the code of rotated channel 32w+i), vl / delta f32 [batch][num_q_heads]
 * (grid origin and step), sq i32 [batch][num_q_heads] (sum of codes). */
int kv1b_query_prep(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                    uint32_t* planes, float* vl, float* delta, int32_t* sq, void* stream);

/* Test hook for the proxy score: for every (b, hq) and token t < length[b]:
 * A = sum_j 2^j sum_w popc(k_bits_w & P_jw), Bc = sum_w popc(k_bits_w) (i32) and the fp32 logit
 * (the exact arithmetic kv1b_attend_topp selects with).  A, Bc, s: [batch][num_q_heads][capacity];
 * entries at t >= length[b] are left unspecified. */
int kv1b_scores(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                int32_t* A, int32_t* Bc, float* s, void* stream);

/* Log-sum-exp merge of partial attention rows (KV1B_ATTEND_PARTIAL) of disjoint token ranges of the
 * same sequences -- e.g. one context split over several GPUs, whose rows were gathered into one
 * array: out[r] = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k, M = max_k m_k, in a fixed order
 * (zeros when every l_k is 0).  parts: f32 [nparts][rows][2 + 128] (device, 4-byte aligned), out:
 * f32 [rows][128] (device, 16-byte aligned); 1 <= nparts <= 1024.  Asynchronous on `stream`.
 * (No page describes a multi-GPU split; this is the merge the split-K engines already use, across
 * ranks.) */
int kv1b_merge_partials(const float* parts, int32_t nparts, int64_t rows, float* out, void* stream);

/* kv1b_scores_probe kernels */
#define KV1B_PROBE_POPC 0    /* __popc over AND-ed bit-planes (the kv1b_scores hook) */
#define KV1B_PROBE_ATTEND 1  /* kv1b_attend's persistent tensor-core kernel (the default engine) */
#define KV1B_PROBE_TOPP 2    /* the score pass of kv1b_attend_topp / kv1b_attend_select */

/* Test hook: the proxy-score integers and logits exactly as one of the library's kernels forms them,
 * so that the integers of the kernels kv1b_attend and kv1b_attend_topp really run can be compared
 * bit for bit with A = sum_j 2^j sum_w popc(k_bits_w & P_jw) and Bc = sum_w popc(k_bits_w)
 * ("RaBitQCache", abstract and key design: binary x INT4 arithmetic).  For every (b, hq) and token
 * t < length[b], into A, Bc (i32) and s (f32), each [batch][num_q_heads][capacity]:
 *   KV1B_PROBE_POPC:   A, Bc and the fp32 logit, as kv1b_scores (out, ws, ws_bytes unused);
 *   KV1B_PROBE_ATTEND: the raw integer tensor-core products 8 A and 8 Bc of the persistent kernel
 *                      (an exact multiple of 8 when the products are right) and its logit in log2
 *                      units, s * log2(e) formed in its own fused order (not bit-exact with the fp32
 *                      logit); the call runs the whole attend and writes out like kv1b_attend.
 *                      ws: kv1b_attend_workspace_bytes(.., 0) bytes.  KV1B_ERR_UNSUPPORTED unless
 *                      that kernel would take the call (equal lengths, length > 0);
 *   KV1B_PROBE_TOPP:   the raw products 8 A and 8 Bc of the Top-p score pass and the fp32 logit it
 *                      selects with (bit-exact with the oracle's order).  ws: kv1b_attend_workspace_bytes
 *                      (.., 1) bytes; out unused.
 * Entries at t >= length[b] are left unspecified.  Asynchronous on `stream`. */
int kv1b_scores_probe(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                      int32_t kernel, int32_t* A, int32_t* Bc, float* s, float* out, void* ws, size_t ws_bytes,
                      void* stream);

/* Test hook for the bounded waits of kv1b_attend's persistent kernel: the same call with every
 * pipeline wait limited to `wait_tries` (1 .. 4096, the product default) suspended tries of at most
 * 0.5 ms each and, when stall_stage >= 0, each CTA's copy producer stopping before its stage
 * `stall_stage` as if those copies never arrived.  A CTA whose wait runs out sets
 * KV1B_STATUS_TIMEOUT, stops issuing copies, lets the copies already in flight land and returns;
 * out is then invalid, and the next kv1b_attend on this workspace must not pass
 * KV1B_ATTEND_WS_CLEAN.  KV1B_ERR_UNSUPPORTED unless the persistent kernel would take the call. */
int kv1b_attend_wait_probe(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                           float scale, float* out, void* ws, size_t ws_bytes, int32_t wait_tries,
                           int32_t stall_stage, void* stream);

/* Synchronous: waits for `stream`, then copies the cache's status word to *flags (host). */
int kv1b_read_status(const kv1b_cache_t* cache, int32_t* flags, void* stream);

/* Static string for a return code. */
const char* kv1b_status_string(int code);

/* Library version (major * 10000 + minor * 100 + patch). */
int kv1b_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KV1B_H */
