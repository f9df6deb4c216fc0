// kv1b_noalloc.cu -- kv1b_attend_noalloc: full decode attention for callers that cannot allocate
// device memory and cannot hand the library a workspace buffer.
//
// Who needs this: host frameworks whose own caching allocator owns all device memory and forbids
// outside cudaMalloc calls, fixed plugin ABIs that pass only inputs and outputs, and
// latency-critical decode loops where cudaMalloc / cudaFree would synchronise the device.  They
// still pass the cache, the query and the output buffer; the split-K partial results that
// kv1b_attend keeps in its caller-provided workspace live here in a fixed file-scope device array.
//
// The array occupies KV1B_NOALLOC_SCRATCH_BYTES on every GPU that loads this library, until the
// process exits.  It is shared by all calls and keeps the previous call's contents; every launch
// rewrites all of the partial rows it later reads, so nothing needs clearing, but two calls whose
// kernels overlap on the GPU (different streams, no ordering between them) race on the array.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "kv1b.h"
#include "kv1b_launch.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KV1B_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};  // device address of g_noalloc_scratch, per device ordinal

// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory; the device
// address is looked up once per device (with that device current) and then reused.
int scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KV1B_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KV1B_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return KV1B_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return KV1B_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace

extern "C" int kv1b_attend_noalloc(const kv1b_cache_t* cache, const void* q, int32_t q_dtype, int32_t num_q_heads,
                                   float scale, float* out, int32_t flags, void* stream) {
  if (!cache || !q || !out) return KV1B_ERR_INVALID_ARG;
  if (cache->head_dim != KV1B_HEAD_DIM || cache->batch < 1 || cache->batch > KV1B_MAX_BATCH ||
      cache->num_kv_heads < 1 || cache->capacity < 1 || cache->capacity % KV1B_CAPACITY_ALIGN != 0)
    return KV1B_ERR_INVALID_ARG;
  if (!cache->k_bits || !cache->v_codes || !cache->signs) return KV1B_ERR_INVALID_ARG;
  if (q_dtype != KV1B_DTYPE_F32 && q_dtype != KV1B_DTYPE_BF16 && q_dtype != KV1B_DTYPE_F16) return KV1B_ERR_INVALID_ARG;
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads != 0) return KV1B_ERR_INVALID_ARG;
  const int G = num_q_heads / cache->num_kv_heads;
  if (G > KV1B_MAX_GROUP) return KV1B_ERR_UNSUPPORTED;
  if (flags != KV1B_ATTEND_TENSOR && flags != KV1B_ATTEND_CUDA_CORE) return KV1B_ERR_INVALID_ARG;
  if (!(scale == scale)) return KV1B_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(out) % 16) return KV1B_ERR_MISALIGNED;

  // Split-K partials: rows * nsplit * (2 + 128) floats must fit the fixed array; fewer splits are
  // used when the automatic choice would not fit, and a shape that does not fit even unsplit is
  // refused before anything is launched.
  const size_t row_bytes = static_cast<size_t>(kv1b::kPartStride) * sizeof(float);
  const size_t rows = static_cast<size_t>(cache->batch) * num_q_heads;
  if (rows * row_bytes > KV1B_NOALLOC_SCRATCH_BYTES) return KV1B_ERR_WORKSPACE;
  int64_t maxlen = 0;
  for (int b = 0; b < cache->batch; ++b) maxlen = cache->h_lengths[b] > maxlen ? cache->h_lengths[b] : maxlen;
  int nsplit = kv1b_pick_splits(cache->batch, cache->num_kv_heads, maxlen, sm_count());
  const size_t fit = KV1B_NOALLOC_SCRATCH_BYTES / (rows * row_bytes);
  if (static_cast<size_t>(nsplit) > fit) nsplit = static_cast<int>(fit);

  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != KV1B_OK) return rc;

  kv1b::AttendParams p;
  memset(&p, 0, sizeof(p));
  p.c.k_bits = cache->k_bits;
  p.c.k_norm = cache->k_norm;
  p.c.k_cinv = cache->k_cinv;
  p.c.v_codes = cache->v_codes;
  p.c.v_sm = cache->v_sm;
  p.c.signs = cache->signs;
  p.c.B = cache->batch;
  p.c.Hkv = cache->num_kv_heads;
  p.c.cap = cache->capacity;
  p.q = q;
  p.q_dtype = q_dtype;
  p.Hq = num_q_heads;
  p.scale = scale;
  p.nsplit = nsplit;
  p.part = static_cast<float*>(scratch);
  p.out = out;
  for (int b = 0; b < cache->batch; ++b) p.len[b] = static_cast<int32_t>(cache->h_lengths[b]);
  const cudaError_t e = kv1b_launch_attend(p, G, flags, static_cast<int32_t>(maxlen), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KV1B_OK : KV1B_ERR_CUDA;
}
