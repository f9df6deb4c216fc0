// kv1b_launch.h -- internal host<->device interface: kernel parameter blocks and launchers.
#pragma once
#include <atomic>
#include <cuda.h>  // CUtensorMap (the descriptor type only; encoded through the runtime entry point)
#include <cuda_runtime.h>
#include <stdint.h>

#include "kv1b.h"

namespace kv1b {

struct EncodeParams {
  const void* k;
  const void* v;
  int32_t dtype;
  int32_t n_new;
  int64_t sb, st, sh;  // element strides of K/V: sequence, token, kv-head
  int32_t B, Hkv, cap;
  int32_t groups_per_warp;  // prefill form: 8-token groups a warp encodes in turn (set by the launcher)
  uint32_t* k_bits;
  float* k_norm;
  float* k_cinv;
  uint32_t* v_codes;
  uint32_t* v_sm;
  const float* signs;
  int32_t* lengths;
  int32_t* status;
  int64_t L0[KV1B_MAX_BATCH];  // write position per sequence (host mirror before the append)
};

struct CacheView {
  const uint32_t* k_bits;
  const float* k_norm;
  const float* k_cinv;
  const uint32_t* v_codes;
  const uint32_t* v_sm;
  const float* signs;
  int32_t B, Hkv, cap;
};

struct AttendParams {
  CacheView c;
  const void* q;
  int32_t q_dtype;
  int32_t Hq;
  float scale;
  int32_t nsplit;
  float* part;   // [B][Hq][nsplit][2 + 128]: m (log2 units), l, o[128]
  float* out;    // [B][Hq][128], or [B][Hq][2 + 128] partial rows when partial_out
  int32_t partial_out;
  int32_t len[KV1B_MAX_BATCH];
};

struct ScoresParams {
  CacheView c;
  const void* q;
  int32_t q_dtype;
  int32_t Hq;
  float scale;
  int32_t* A;    // optional [B][Hq][cap]
  int32_t* Bc;   // optional [B][Hq][cap]
  float* s;      // [B][Hq][cap]
  int32_t len[KV1B_MAX_BATCH];
};

// Top-p pipeline (kv1b_topp.cu): per row r = b * Hq + hq of the query heads.
struct ToppRowState {
  uint32_t maxkey;           // order-preserving key of the row's largest logit (atomicMax)
  uint32_t ncand;            // tokens in the threshold bucket
  int32_t bstar;             // threshold bucket (-1: the row is empty; -2: the kept window alone suffices)
  uint32_t merged;           // merge blocks of the row done (atomic ticket)
  unsigned long long U;      // integer mass of the tokens outside the kept window (Top-k: their count)
  unsigned long long rem;    // mass still needed inside the threshold bucket
  unsigned long long kstar;  // largest selected 64-bit key of the threshold bucket
  unsigned long long Uw;     // integer mass of the kept window (Top-p)
  unsigned long long pad1[2];
};
constexpr int kToppBuckets = 2048;  // masses by t = (s - m) log2 e: bucket floor(-64 t), t >= -40
constexpr int kToppWinBucket = 0xffff;  // bucket-plane mark of a token of the kept window
constexpr int kToppChunk = 4096;    // tokens per block of the streaming kernels
constexpr int kToppSub = 1024;      // tokens per selected-count entry and per compaction+gather block
constexpr int kToppMergeSplit = 8;  // first-level merge blocks per row

struct ToppParams {
  CacheView c;
  const void* q;
  int32_t q_dtype;
  int32_t Hq;
  float p;
  float scale;
  int32_t mode;              // KV1B_SELECT_TOPP or KV1B_SELECT_TOPK
  int32_t k;                 // Top-k budget (tokens outside the window)
  int32_t sink, recent;      // kept window: the first `sink` and the last `recent` tokens
  uint32_t* planes;          // [R][4][4] query bit-planes, then grid origin, step and code sum per row
  float* qvl;
  float* qdl;
  int32_t* qsq;
  float* s;                  // [R][cap] logits
  uint16_t* bk;              // [R][cap] mass bucket of each token (kToppBuckets: no mass)
  int32_t* cand;             // [R][cap] threshold-bucket candidates (any order)
  ToppRowState* rows;        // [R]
  unsigned long long* hist;  // [R][kToppBuckets] masses per bucket
  uint32_t* sub_cnt;         // [R][nsub] selected tokens per sub-chunk (lower buckets, then candidates)
  uint32_t* sub_off;         // [R][nsub + 1] exclusive prefix of sub_cnt (first output slot per sub-chunk)
  float* part;               // [R][nsub][kPartStride] gather partials per sub-chunk
  float* part2;              // [R][kToppMergeSplit][kPartStride] first-level merge sums
  int32_t nchunk;
  int32_t nsub;
  float* out;
  int32_t* sel_idx;
  int32_t* sel_cnt;
  int32_t* probe_A;          // test hook (probe instantiation of the score pass only): [R][cap] raw
  int32_t* probe_Bc;         //   score products 8 A and 8 Bc
  int32_t len[KV1B_MAX_BATCH];
};

constexpr int kPartStride = 2 + 128;

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) for `func` once per device of the calling thread
// (bit d of *done marks device d; devices past 63 set it on every call).
inline cudaError_t configure_smem(const void* func, int bytes, std::atomic<unsigned long long>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done->load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done->fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// exact attention over a selected token set (kv1b_exact.cu)
constexpr int kExactItem = 256;  // selected entries per work item
struct ExactParams {
  const void* q;
  int32_t q_dtype;
  int32_t Hq, Hkv;
  float qscale;              // scale * log2(e)
  const void* k;             // exact keys / values: element (b, t, h, c) at b sb + t st + h sh + c
  const void* v;
  int32_t kv_dtype;
  int64_t sb, st, sh;
  int64_t kv_tokens;         // tokens per sequence the key / value arrays hold
  const int32_t* sel;        // [R][cap] selected indices
  const int32_t* cnt;        // [R]
  int32_t cap;
  int32_t* item_off;         // [R + 1] first work item of each row
  float* part;               // [items][kPartStride]
  float* out;                // [R][128]
  int32_t* status;
  int32_t len[KV1B_MAX_BATCH];
};

// persistent attend on the integer tensor cores (kv1b_attend_ws.cu)
struct alignas(64) AttendWsParams {
  CUtensorMap codes_map;  // v_codes as [tiles][128 channels][128 4-bit tokens], 16U4_ALIGN16B, 128B swizzle
  CacheView c;
  const void* q;
  int32_t q_dtype;
  int32_t Hq;
  float scale;
  int32_t L;           // tokens per sequence (equal for every sequence)
  int64_t T;           // total 128-token tiles over all (sequence, kv-head) segments
  int64_t Lt;          // tiles per segment
  int32_t ncta;        // CTAs (one per SM)
  int32_t max_pieces;  // partial slots per segment
  float* part;         // [segments][max_pieces][G][2 + 128]: m (log2 units), l, o[128]
  float* out;          // [B][Hq][128]
  int32_t* status;     // cache status word (timeout flag)
  unsigned* counters;  // [B * Hkv] pieces of each segment written so far (zeroed before the launch)
  int32_t partial_out; // the merge writes log-sum-exp rows (m, l, o[128]) to out instead of o / l
  int32_t G_all;       // query heads per kv-head of the call (set by the launcher)
  int32_t head_base;   // first query head (within the kv-head's group) of this launch
  int32_t heads;       // query heads this launch serves (<= the kernel's G)
  int32_t wait_tries;  // suspended tries (<= 0.5 ms each) before a pipeline wait gives up
  int32_t stall_stage; // test hook: each CTA's producer stops before this stage (-1: never)
  int32_t* probe_A;    // test hook (probe instantiation only): [B][Hq][cap] raw score products 8 A,
  int32_t* probe_Bc;   //   8 Bc and the log2-unit logits as the kernel forms them
  float* probe_s;
};
constexpr int kWaitTriesDefault = 4096;

}  // namespace kv1b

cudaError_t kv1b_launch_init(uint64_t seed, int32_t rounds, float* signs, int32_t* lengths, int32_t batch,
                             int32_t* status,
                             cudaStream_t stream);
// Launch with programmatic stream serialization: the kernel may be scheduled while its predecessor
// in the stream finishes, and must call pdl_wait() before it touches memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

cudaError_t kv1b_launch_encode(const kv1b::EncodeParams& p, int64_t max_tiles, cudaStream_t stream);
// The CUDA-core split-K engine (split kernel + merge); the tensor-core engine is kv1b_launch_attend_ws.
cudaError_t kv1b_launch_attend(const kv1b::AttendParams& p, int32_t G, cudaStream_t stream);
cudaError_t kv1b_launch_query_prep(const kv1b::CacheView& c, const void* q, int32_t q_dtype, int32_t Hq,
                                   uint32_t* planes, float* vl, float* delta, int32_t* sq, cudaStream_t stream);
cudaError_t kv1b_launch_scores(const kv1b::ScoresParams& p, int32_t G, int32_t max_len, cudaStream_t stream);
cudaError_t kv1b_launch_topp(const kv1b::ToppParams& p, int32_t G, int32_t max_len, cudaStream_t stream);
// The Top-p pipeline's first two passes only (query preparation, scores), with the score pass writing
// its raw integer products to p.probe_A / probe_Bc and its logits to p.s.
cudaError_t kv1b_launch_topp_scores_probe(const kv1b::ToppParams& p, int32_t G, int32_t max_len, cudaStream_t stream);
size_t kv1b_topp_workspace_bytes(int32_t rows, int32_t cap);
void kv1b_topp_carve(kv1b::ToppParams* p, void* ws, int32_t rows, int32_t cap);
int kv1b_pick_splits(int32_t B, int32_t Hkv, int64_t max_len, int num_sms);
cudaError_t kv1b_launch_merge(const float* part, float* out, int32_t rows, int32_t nsplit, cudaStream_t stream);
// Log-sum-exp merge of nsplit partial rows per output row; partial row k of output row r at
// part + r * row_stride + k * split_stride (floats).  partial_out: write (m, l, o[128]) rows.
cudaError_t kv1b_launch_merge_strided(const float* part, float* out, int64_t rows, int32_t nsplit, int64_t row_stride,
                                      int64_t split_stride, bool partial_out, cudaStream_t stream);
size_t kv1b_exact_workspace_bytes(int32_t rows, int32_t cap);
void kv1b_exact_carve(kv1b::ExactParams* p, void* ws, int32_t rows);
cudaError_t kv1b_launch_exact(const kv1b::ExactParams& p, int32_t rows, int32_t num_sms, cudaStream_t stream);
bool kv1b_ws_supported(int32_t G);
int kv1b_ws_template_group(int32_t G);  // query heads per launch slot of the persistent kernel for G (1, 2 or 4)
int kv1b_attend_ws_buffers(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                           float scale, float* out, float* part, size_t part_bytes, unsigned* counters,
                           cudaStream_t stream);
void kv1b_ws_plan(int32_t B, int32_t Hkv, int64_t L, int num_sms, int64_t* T, int64_t* Lt, int* ncta,
                  int* max_pieces);
cudaError_t kv1b_launch_attend_ws(kv1b::AttendWsParams& p, int32_t G, bool counters_clean, cudaStream_t stream,
                                  bool probe = false);
