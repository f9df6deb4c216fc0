// kv1b_api.cu -- the extern "C" entry points declared in include/kv1b.h: argument validation on
// the host, then kernel launches on the caller's stream.  Nothing here allocates device memory.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "kv1b.h"
#include "kv1b_launch.h"

namespace {

constexpr size_t kAlign = 256;
constexpr int kMinForcedSplits = 64;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  size_t k_bits, k_norm, k_cinv, v_codes, v_sm, signs, lengths, status, total;
};

bool shape_ok(int32_t batch, int32_t hkv, int32_t head_dim, int32_t capacity) {
  return batch >= 1 && batch <= KV1B_MAX_BATCH && hkv >= 1 && head_dim == KV1B_HEAD_DIM && capacity >= 1 &&
         capacity % KV1B_CAPACITY_ALIGN == 0;
}

Layout layout(int32_t batch, int32_t hkv, int32_t capacity) {
  const size_t tok = static_cast<size_t>(batch) * hkv * capacity;
  Layout l;
  size_t off = 0;
  l.k_bits = off;  off += align_up(tok * 16);
  l.k_norm = off;  off += align_up(tok * 4);
  l.k_cinv = off;  off += align_up(tok * 4);
  l.v_codes = off; off += align_up(tok * 64);
  l.v_sm = off;    off += align_up(tok * 16);
  l.signs = off;   off += align_up(KV1B_MAX_ROUNDS * KV1B_HEAD_DIM * 4);
  l.lengths = off; off += align_up(KV1B_MAX_BATCH * 4);
  l.status = off;  off += align_up(4);
  l.total = off;
  return l;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

kv1b::CacheView view(const kv1b_cache_t* c) {
  kv1b::CacheView v;
  v.k_bits = c->k_bits;
  v.k_norm = c->k_norm;
  v.k_cinv = c->k_cinv;
  v.v_codes = c->v_codes;
  v.v_sm = c->v_sm;
  v.signs = c->signs;
  v.B = c->batch;
  v.Hkv = c->num_kv_heads;
  v.cap = c->capacity;
  return v;
}

bool cache_ok(const kv1b_cache_t* c) {
  return c && shape_ok(c->batch, c->num_kv_heads, c->head_dim, c->capacity) && c->k_bits && c->v_codes &&
         c->signs && c->d_lengths && c->d_status;
}

bool dtype_ok(int32_t dt) { return dt == KV1B_DTYPE_F32 || dt == KV1B_DTYPE_BF16 || dt == KV1B_DTYPE_F16; }

int64_t max_length(const kv1b_cache_t* c) {
  int64_t m = 0;
  for (int b = 0; b < c->batch; ++b) m = c->h_lengths[b] > m ? c->h_lengths[b] : m;
  return m;
}

int heads_check(const kv1b_cache_t* c, int32_t num_q_heads) {
  if (num_q_heads < 1 || num_q_heads % c->num_kv_heads != 0) return KV1B_ERR_INVALID_ARG;
  if (num_q_heads / c->num_kv_heads > KV1B_MAX_GROUP) return KV1B_ERR_UNSUPPORTED;
  return KV1B_OK;
}

int32_t max_splits(const kv1b_cache_t* c) {
  const int auto_max = kv1b_pick_splits(c->batch, c->num_kv_heads, c->capacity, num_sms());
  return auto_max > kMinForcedSplits ? auto_max : kMinForcedSplits;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KV1B_OK : KV1B_ERR_CUDA; }

// Partial slots of the persistent kernel: segments x pieces x G x (2 + 128) floats; the piece
// count per segment does not depend on the length, so the capacity-sized plan bounds every call.
size_t ws_bytes_needed(const kv1b_cache_t* c, int32_t num_q_heads) {
  const int Gq = num_q_heads / c->num_kv_heads;
  if (!kv1b_ws_supported(Gq)) return 0;
  const int G = kv1b_ws_template_group(Gq < 4 ? Gq : 4);  // head slots of one launch
  int64_t T, Lt;
  int ncta, pieces;
  kv1b_ws_plan(c->batch, c->num_kv_heads, c->capacity, num_sms(), &T, &Lt, &ncta, &pieces);
  return static_cast<size_t>(c->batch) * c->num_kv_heads * pieces * G * kv1b::kPartStride * 4;
}

// kv1b_attend's workspace: the partial rows of either attend kernel, then one merge counter per
// (sequence, kv-head) for the persistent kernel.
size_t ws_counter_bytes(const kv1b_cache_t* c) { return sizeof(unsigned) * c->batch * c->num_kv_heads; }
size_t ws_counters_offset(const kv1b_cache_t* c, int32_t num_q_heads) {
  const size_t rows = static_cast<size_t>(c->batch) * num_q_heads;
  const size_t split_bytes = rows * static_cast<size_t>(max_splits(c)) * kv1b::kPartStride * 4;
  const size_t ws = ws_bytes_needed(c, num_q_heads);
  return align_up(split_bytes > ws ? split_bytes : ws);
}

bool equal_lengths(const kv1b_cache_t* c) {
  for (int b = 1; b < c->batch; ++b)
    if (c->h_lengths[b] != c->h_lengths[0]) return false;
  return true;
}

// The persistent tensor-core kernel takes the call: one length for every sequence, a non-empty cache
// (G up to 8: launches of at most 4 query heads).
bool ws_engine_applies(const kv1b_cache_t* c, int32_t num_q_heads) {
  return kv1b_ws_supported(num_q_heads / c->num_kv_heads) && equal_lengths(c) && max_length(c) > 0;
}

// Parameters of the persistent kernel for this cache and workspace (KV1B_OK or KV1B_ERR_WORKSPACE).
int ws_params(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale, float* out,
              void* ws, kv1b::AttendWsParams* w) {
  const int Gq = num_q_heads / cache->num_kv_heads;
  const int G = kv1b_ws_template_group(Gq < 4 ? Gq : 4);  // head slots of one launch
  const int64_t maxlen = max_length(cache);
  memset(w, 0, sizeof(*w));
  w->c = view(cache);
  w->q = q;
  w->q_dtype = q_dtype;
  w->Hq = num_q_heads;
  w->scale = scale;
  w->L = static_cast<int32_t>(maxlen);
  int ncta = 0, pieces = 0;
  kv1b_ws_plan(cache->batch, cache->num_kv_heads, maxlen, num_sms(), &w->T, &w->Lt, &ncta, &pieces);
  int64_t Tc, Ltc;
  int nc, pieces_cap;
  kv1b_ws_plan(cache->batch, cache->num_kv_heads, cache->capacity, num_sms(), &Tc, &Ltc, &nc, &pieces_cap);
  w->ncta = ncta;
  w->max_pieces = pieces_cap > pieces ? pieces_cap : pieces;
  if (w->max_pieces > 256 || static_cast<size_t>(cache->batch) * cache->num_kv_heads * w->max_pieces * G *
                                    kv1b::kPartStride * 4 > ws_counters_offset(cache, num_q_heads))
    return KV1B_ERR_WORKSPACE;
  w->part = static_cast<float*>(ws);
  w->out = out;
  w->status = cache->d_status;
  w->counters = reinterpret_cast<unsigned*>(static_cast<char*>(ws) + ws_counters_offset(cache, num_q_heads));
  w->wait_tries = kv1b::kWaitTriesDefault;
  w->stall_stage = -1;
  return KV1B_OK;
}

// Shared argument checks of kv1b_attend and its test hooks.
int attend_args_check(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                      const float* out, const void* ws, size_t ws_bytes) {
  if (!cache_ok(cache) || !q || !out || !ws || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!(scale == scale)) return KV1B_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(ws, kAlign) || !aligned(out, 16)) return KV1B_ERR_MISALIGNED;
  if (ws_bytes < kv1b_attend_workspace_bytes(cache, num_q_heads, 0)) return KV1B_ERR_WORKSPACE;
  return KV1B_OK;
}

}  // namespace

// The persistent tensor-core attend with caller-given partial-row and merge-counter buffers (used by
// kv1b_attend_noalloc).  KV1B_ERR_UNSUPPORTED when that kernel does not take the call,
// KV1B_ERR_WORKSPACE when its partial rows need more than part_bytes.
int kv1b_attend_ws_buffers(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                           float scale, float* out, float* part, size_t part_bytes, unsigned* counters,
                           cudaStream_t stream) {
  if (!cache_ok(cache) || !q || !out || !part || !counters || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!ws_engine_applies(cache, num_q_heads)) return KV1B_ERR_UNSUPPORTED;
  const int Gq = num_q_heads / cache->num_kv_heads;
  const int G = kv1b_ws_template_group(Gq < 4 ? Gq : 4);  // head slots of one launch
  kv1b::AttendWsParams w;
  memset(&w, 0, sizeof(w));
  w.c = view(cache);
  w.q = q;
  w.q_dtype = q_dtype;
  w.Hq = num_q_heads;
  w.scale = scale;
  const int64_t maxlen = max_length(cache);
  w.L = static_cast<int32_t>(maxlen);
  int ncta = 0, pieces = 0;
  kv1b_ws_plan(cache->batch, cache->num_kv_heads, maxlen, num_sms(), &w.T, &w.Lt, &ncta, &pieces);
  w.ncta = ncta;
  w.max_pieces = pieces;
  if (pieces > 256 ||
      static_cast<size_t>(cache->batch) * cache->num_kv_heads * pieces * G * kv1b::kPartStride * 4 > part_bytes)
    return KV1B_ERR_WORKSPACE;
  w.part = part;
  w.out = out;
  w.status = cache->d_status;
  w.counters = counters;
  w.wait_tries = kv1b::kWaitTriesDefault;
  w.stall_stage = -1;
  return cuda_status(kv1b_launch_attend_ws(w, Gq, false, stream));
}

extern "C" {

size_t kv1b_cache_bytes(int32_t batch, int32_t num_kv_heads, int32_t head_dim, int32_t capacity) {
  if (!shape_ok(batch, num_kv_heads, head_dim, capacity)) return 0;
  return layout(batch, num_kv_heads, capacity).total;
}

int kv1b_cache_init(kv1b_cache_t* cache, void* dev_buf, size_t bytes, int32_t batch, int32_t num_kv_heads,
                    int32_t head_dim, int32_t capacity, uint64_t seed, void* stream) {
  return kv1b_cache_init_rounds(cache, dev_buf, bytes, batch, num_kv_heads, head_dim, capacity, seed, 1, stream);
}

int kv1b_cache_init_rounds(kv1b_cache_t* cache, void* dev_buf, size_t bytes, int32_t batch, int32_t num_kv_heads,
                           int32_t head_dim, int32_t capacity, uint64_t seed, int32_t rounds, void* stream) {
  if (!cache || !dev_buf || rounds < 1 || rounds > KV1B_MAX_ROUNDS) return KV1B_ERR_INVALID_ARG;
  if (head_dim != KV1B_HEAD_DIM || batch > KV1B_MAX_BATCH) return KV1B_ERR_UNSUPPORTED;
  if (!shape_ok(batch, num_kv_heads, head_dim, capacity)) return KV1B_ERR_INVALID_ARG;
  if (!aligned(dev_buf, kAlign)) return KV1B_ERR_MISALIGNED;
  const Layout l = layout(batch, num_kv_heads, capacity);
  if (bytes < l.total) return KV1B_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(dev_buf);
  kv1b_cache_t c;
  memset(&c, 0, sizeof(c));
  c.batch = batch;
  c.num_kv_heads = num_kv_heads;
  c.head_dim = head_dim;
  c.capacity = capacity;
  c.rotation_seed = seed;
  c.rotation_rounds = rounds;
  c.k_bits = reinterpret_cast<uint32_t*>(base + l.k_bits);
  c.k_norm = reinterpret_cast<float*>(base + l.k_norm);
  c.k_cinv = reinterpret_cast<float*>(base + l.k_cinv);
  c.v_codes = reinterpret_cast<uint32_t*>(base + l.v_codes);
  c.v_sm = reinterpret_cast<uint32_t*>(base + l.v_sm);
  c.signs = reinterpret_cast<float*>(base + l.signs);
  c.d_lengths = reinterpret_cast<int32_t*>(base + l.lengths);
  c.d_status = reinterpret_cast<int32_t*>(base + l.status);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(dev_buf, 0, l.total, s);
  if (e != cudaSuccess) return KV1B_ERR_CUDA;
  e = kv1b_launch_init(seed, rounds, c.signs, c.d_lengths, batch, c.d_status, s);
  if (e != cudaSuccess) return KV1B_ERR_CUDA;
  *cache = c;
  return KV1B_OK;
}

int kv1b_encode_append(kv1b_cache_t* cache, const void* k, const void* v, int32_t dtype, int32_t n_new,
                       int64_t stride_b, int64_t stride_t, int64_t stride_h, void* stream) {
  if (!cache_ok(cache) || !k || !v || !dtype_ok(dtype) || n_new < 1) return KV1B_ERR_INVALID_ARG;
  if (stride_b < 0 || stride_t < 0 || stride_h < 0) return KV1B_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || stride_b % 4 || stride_t % 4 || stride_h % 4) return KV1B_ERR_MISALIGNED;
  for (int b = 0; b < cache->batch; ++b)
    if (cache->h_lengths[b] + n_new > cache->capacity) return KV1B_ERR_CAPACITY;
  kv1b::EncodeParams p;
  memset(&p, 0, sizeof(p));
  p.k = k;
  p.v = v;
  p.dtype = dtype;
  p.n_new = n_new;
  p.sb = stride_b;
  p.st = stride_t;
  p.sh = stride_h;
  p.B = cache->batch;
  p.Hkv = cache->num_kv_heads;
  p.cap = cache->capacity;
  p.k_bits = cache->k_bits;
  p.k_norm = cache->k_norm;
  p.k_cinv = cache->k_cinv;
  p.v_codes = cache->v_codes;
  p.v_sm = cache->v_sm;
  p.signs = cache->signs;
  p.lengths = cache->d_lengths;
  p.status = cache->d_status;
  int64_t max_tiles = 0;
  for (int b = 0; b < cache->batch; ++b) {
    p.L0[b] = cache->h_lengths[b];
    const int64_t nt = (p.L0[b] + n_new - 1) / 16 - p.L0[b] / 16 + 1;
    max_tiles = nt > max_tiles ? nt : max_tiles;
  }
  const cudaError_t e = kv1b_launch_encode(p, max_tiles, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return KV1B_ERR_CUDA;
  for (int b = 0; b < cache->batch; ++b) cache->h_lengths[b] += n_new;
  return KV1B_OK;
}

size_t kv1b_attend_workspace_bytes(const kv1b_cache_t* cache, int32_t num_q_heads, int32_t mode) {
  if (!cache_ok(cache) || heads_check(cache, num_q_heads) != KV1B_OK) return 0;
  const size_t rows = static_cast<size_t>(cache->batch) * num_q_heads;
  if (mode == 0) return ws_counters_offset(cache, num_q_heads) + align_up(ws_counter_bytes(cache));
  if (mode == 1) return align_up(kv1b_topp_workspace_bytes(static_cast<int32_t>(rows), cache->capacity));
  if (mode == 2) return align_up(kv1b_exact_workspace_bytes(static_cast<int32_t>(rows), cache->capacity));
  return 0;
}

int kv1b_attend(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                float* out, void* ws, size_t ws_bytes, int32_t flags, int32_t num_splits, void* stream) {
  const int ac = attend_args_check(cache, q, q_dtype, num_q_heads, scale, out, ws, ws_bytes);
  if (ac != KV1B_OK) return ac;
  if ((flags & ~(KV1B_ATTEND_CUDA_CORE | KV1B_ATTEND_WS_CLEAN | KV1B_ATTEND_PARTIAL)) != 0) return KV1B_ERR_INVALID_ARG;
  const bool ws_clean = (flags & KV1B_ATTEND_WS_CLEAN) != 0;
  const bool partial = (flags & KV1B_ATTEND_PARTIAL) != 0;
  flags &= KV1B_ATTEND_CUDA_CORE;  // the engine
  if (num_splits < 0 || num_splits > max_splits(cache)) return KV1B_ERR_INVALID_ARG;
  const int64_t maxlen = max_length(cache);
  const int G = num_q_heads / cache->num_kv_heads;
  if (flags == KV1B_ATTEND_TENSOR && num_splits == 0 && ws_engine_applies(cache, num_q_heads)) {
    kv1b::AttendWsParams w;
    const int rc = ws_params(cache, q, q_dtype, num_q_heads, scale, out, ws, &w);
    if (rc != KV1B_OK) return rc;
    w.partial_out = partial ? 1 : 0;
    return cuda_status(kv1b_launch_attend_ws(w, G, ws_clean, static_cast<cudaStream_t>(stream)));
  }
  // this engine does not use the merge counters; they are zeroed here unless the caller says they
  // are, so that every completed call leaves them zero
  if (!ws_clean) {
    const cudaError_t e = cudaMemsetAsync(static_cast<char*>(ws) + ws_counters_offset(cache, num_q_heads), 0,
                                          ws_counter_bytes(cache), static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e);
  }
  kv1b::AttendParams p;
  memset(&p, 0, sizeof(p));
  p.c = view(cache);
  p.q = q;
  p.q_dtype = q_dtype;
  p.Hq = num_q_heads;
  p.scale = scale;
  p.nsplit = num_splits > 0 ? num_splits : kv1b_pick_splits(cache->batch, cache->num_kv_heads, maxlen, num_sms());
  p.part = static_cast<float*>(ws);
  p.out = out;
  p.partial_out = partial ? 1 : 0;
  for (int b = 0; b < cache->batch; ++b) p.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
  return cuda_status(kv1b_launch_attend(p, G, static_cast<cudaStream_t>(stream)));
}

int kv1b_attend_select(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                       int32_t mode, float p, int32_t k, int32_t sink, int32_t recent, float* out, int32_t* sel_idx,
                       int32_t* sel_cnt, void* ws, size_t ws_bytes, void* stream) {
  if (!cache_ok(cache) || !q || !out || !sel_idx || !sel_cnt || !ws || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (mode != KV1B_SELECT_TOPP && mode != KV1B_SELECT_TOPK) return KV1B_ERR_INVALID_ARG;
  if (mode == KV1B_SELECT_TOPP && !(p > 0.0f && p <= 1.0f)) return KV1B_ERR_INVALID_ARG;
  if (mode == KV1B_SELECT_TOPK && k < 0) return KV1B_ERR_INVALID_ARG;
  if (sink < 0 || recent < 0 || !(scale == scale)) return KV1B_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(ws, kAlign)) return KV1B_ERR_MISALIGNED;
  if (ws_bytes < kv1b_attend_workspace_bytes(cache, num_q_heads, 1)) return KV1B_ERR_WORKSPACE;
  const int G = num_q_heads / cache->num_kv_heads;
  kv1b::ToppParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.c = view(cache);
  tp.q = q;
  tp.q_dtype = q_dtype;
  tp.Hq = num_q_heads;
  tp.p = mode == KV1B_SELECT_TOPP ? p : 1.0f;
  tp.scale = scale;
  tp.mode = mode;
  tp.k = k;
  tp.sink = sink;
  tp.recent = recent;
  tp.out = out;
  tp.sel_idx = sel_idx;
  tp.sel_cnt = sel_cnt;
  for (int b = 0; b < cache->batch; ++b) tp.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
  kv1b_topp_carve(&tp, ws, cache->batch * num_q_heads, cache->capacity);
  return cuda_status(
      kv1b_launch_topp(tp, G, static_cast<int32_t>(max_length(cache)), static_cast<cudaStream_t>(stream)));
}

int kv1b_attend_topp(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                     float p, float* out, int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                     void* stream) {
  return kv1b_attend_select(cache, q, q_dtype, num_q_heads, scale, KV1B_SELECT_TOPP, p, 0, 0, 0, out, sel_idx, sel_cnt,
                            ws, ws_bytes, stream);
}

int kv1b_attend_selected_exact(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                               float scale, const void* k, const void* v, int32_t kv_dtype, int64_t kv_tokens,
                               int64_t stride_b, int64_t stride_t, int64_t stride_h, const int32_t* sel_idx,
                               const int32_t* sel_cnt, float* out, void* ws, size_t ws_bytes, void* stream) {
  if (!cache_ok(cache) || !q || !k || !v || !sel_idx || !sel_cnt || !out || !ws || !dtype_ok(q_dtype) ||
      !dtype_ok(kv_dtype))
    return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!(scale == scale) || kv_tokens < 0 || stride_b < 0 || stride_t < 0 || stride_h < 0) return KV1B_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(ws, kAlign) || stride_b % 8 != 0 ||
      stride_t % 8 != 0 || stride_h % 8 != 0)
    return KV1B_ERR_MISALIGNED;
  if (ws_bytes < kv1b_attend_workspace_bytes(cache, num_q_heads, 2)) return KV1B_ERR_WORKSPACE;
  kv1b::ExactParams p;
  memset(&p, 0, sizeof(p));
  p.q = q;
  p.q_dtype = q_dtype;
  p.Hq = num_q_heads;
  p.Hkv = cache->num_kv_heads;
  p.qscale = scale * 1.4426950408889634f;
  p.k = k;
  p.v = v;
  p.kv_dtype = kv_dtype;
  p.sb = stride_b;
  p.st = stride_t;
  p.sh = stride_h;
  p.kv_tokens = kv_tokens;
  p.sel = sel_idx;
  p.cnt = sel_cnt;
  p.cap = cache->capacity;
  p.out = out;
  p.status = cache->d_status;
  for (int b = 0; b < cache->batch; ++b) p.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
  kv1b_exact_carve(&p, ws, cache->batch * num_q_heads);
  return cuda_status(
      kv1b_launch_exact(p, cache->batch * num_q_heads, num_sms(), static_cast<cudaStream_t>(stream)));
}

int kv1b_query_prep(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, uint32_t* planes,
                    float* vl, float* delta, int32_t* sq, void* stream) {
  if (!cache_ok(cache) || !q || !planes || !vl || !delta || !sq || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!aligned(q, 16)) return KV1B_ERR_MISALIGNED;
  return cuda_status(kv1b_launch_query_prep(view(cache), q, q_dtype, num_q_heads, planes, vl, delta, sq,
                                            static_cast<cudaStream_t>(stream)));
}

int kv1b_scores(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                int32_t* A, int32_t* Bc, float* s, void* stream) {
  if (!cache_ok(cache) || !q || !s || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!aligned(q, 16)) return KV1B_ERR_MISALIGNED;
  kv1b::ScoresParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.c = view(cache);
  sp.q = q;
  sp.q_dtype = q_dtype;
  sp.Hq = num_q_heads;
  sp.scale = scale;
  sp.A = A;
  sp.Bc = Bc;
  sp.s = s;
  for (int b = 0; b < cache->batch; ++b) sp.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
  return cuda_status(kv1b_launch_scores(sp, num_q_heads / cache->num_kv_heads, static_cast<int32_t>(max_length(cache)),
                                        static_cast<cudaStream_t>(stream)));
}

int kv1b_scores_probe(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads, float scale,
                      int32_t kernel, int32_t* A, int32_t* Bc, float* s, float* out, void* ws, size_t ws_bytes,
                      void* stream) {
  if (kernel == KV1B_PROBE_POPC) return kv1b_scores(cache, q, q_dtype, num_q_heads, scale, A, Bc, s, stream);
  if (!cache_ok(cache) || !q || !A || !Bc || !s || !ws || !dtype_ok(q_dtype)) return KV1B_ERR_INVALID_ARG;
  const int hc = heads_check(cache, num_q_heads);
  if (hc != KV1B_OK) return hc;
  if (!(scale == scale)) return KV1B_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = num_q_heads / cache->num_kv_heads;
  if (kernel == KV1B_PROBE_ATTEND) {
    const int ac = attend_args_check(cache, q, q_dtype, num_q_heads, scale, out, ws, ws_bytes);
    if (ac != KV1B_OK) return ac;
    if (!ws_engine_applies(cache, num_q_heads)) return KV1B_ERR_UNSUPPORTED;
    kv1b::AttendWsParams w;
    const int rc = ws_params(cache, q, q_dtype, num_q_heads, scale, out, ws, &w);
    if (rc != KV1B_OK) return rc;
    w.probe_A = A;
    w.probe_Bc = Bc;
    w.probe_s = s;
    return cuda_status(kv1b_launch_attend_ws(w, G, false, st, true));
  }
  if (kernel == KV1B_PROBE_TOPP) {
    if (!aligned(q, 16) || !aligned(ws, kAlign)) return KV1B_ERR_MISALIGNED;
    if (ws_bytes < kv1b_attend_workspace_bytes(cache, num_q_heads, 1)) return KV1B_ERR_WORKSPACE;
    kv1b::ToppParams tp;
    memset(&tp, 0, sizeof(tp));
    tp.c = view(cache);
    tp.q = q;
    tp.q_dtype = q_dtype;
    tp.Hq = num_q_heads;
    tp.p = 1.0f;
    tp.scale = scale;
    tp.probe_A = A;
    tp.probe_Bc = Bc;
    for (int b = 0; b < cache->batch; ++b) tp.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
    kv1b_topp_carve(&tp, ws, cache->batch * num_q_heads, cache->capacity);
    const int64_t maxlen = max_length(cache);
    cudaError_t e = kv1b_launch_topp_scores_probe(tp, G, static_cast<int32_t>(maxlen), st);
    if (e == cudaSuccess && maxlen > 0)  // the logits the pass wrote to its plane
      e = cudaMemcpyAsync(s, tp.s, sizeof(float) * static_cast<size_t>(cache->batch) * num_q_heads * cache->capacity,
                          cudaMemcpyDeviceToDevice, st);
    return cuda_status(e);
  }
  return KV1B_ERR_INVALID_ARG;
}

int kv1b_attend_wait_probe(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                           float scale, float* out, void* ws, size_t ws_bytes, int32_t wait_tries,
                           int32_t stall_stage, void* stream) {
  const int ac = attend_args_check(cache, q, q_dtype, num_q_heads, scale, out, ws, ws_bytes);
  if (ac != KV1B_OK) return ac;
  if (wait_tries < 1 || wait_tries > kv1b::kWaitTriesDefault || stall_stage < -1) return KV1B_ERR_INVALID_ARG;
  if (!ws_engine_applies(cache, num_q_heads)) return KV1B_ERR_UNSUPPORTED;
  kv1b::AttendWsParams w;
  const int rc = ws_params(cache, q, q_dtype, num_q_heads, scale, out, ws, &w);
  if (rc != KV1B_OK) return rc;
  w.wait_tries = wait_tries;
  w.stall_stage = stall_stage;
  return cuda_status(kv1b_launch_attend_ws(w, num_q_heads / cache->num_kv_heads, false,
                                           static_cast<cudaStream_t>(stream)));
}

int kv1b_merge_partials(const float* parts, int32_t nparts, int64_t rows, float* out, void* stream) {
  if (!parts || !out || nparts < 1 || nparts > 1024 || rows < 1 || rows > 0x7fffffff) return KV1B_ERR_INVALID_ARG;
  if (!aligned(parts, 4) || !aligned(out, 16)) return KV1B_ERR_MISALIGNED;
  return cuda_status(kv1b_launch_merge_strided(parts, out, rows, nparts, kv1b::kPartStride, rows * kv1b::kPartStride,
                                               false, static_cast<cudaStream_t>(stream)));
}

int kv1b_read_status(const kv1b_cache_t* cache, int32_t* flags, void* stream) {
  if (!cache_ok(cache) || !flags) return KV1B_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, cache->d_status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return KV1B_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KV1B_ERR_CUDA;
  *flags = h;
  return KV1B_OK;
}

const char* kv1b_status_string(int code) {
  switch (code) {
    case KV1B_OK: return "ok";
    case KV1B_ERR_INVALID_ARG: return "invalid argument";
    case KV1B_ERR_UNSUPPORTED: return "unsupported shape (head_dim must be 128, G <= 8, batch <= 64)";
    case KV1B_ERR_CAPACITY: return "append would exceed the cache capacity";
    case KV1B_ERR_MISALIGNED: return "misaligned pointer or stride";
    case KV1B_ERR_WORKSPACE: return "buffer or workspace too small";
    case KV1B_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int kv1b_version(void) { return 100; }

}  // extern "C"
