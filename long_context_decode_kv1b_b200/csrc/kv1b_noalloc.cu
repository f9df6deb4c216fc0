// kv1b_noalloc.cu -- kv1b_attend_noalloc: full decode attention for callers that cannot allocate
// device memory and cannot hand the library a workspace buffer.
//
// Who needs this: host frameworks whose own caching allocator owns all device memory and forbids
// outside cudaMalloc calls, fixed plugin ABIs that pass only inputs and outputs, and
// latency-critical decode loops where cudaMalloc / cudaFree would synchronise the device.  They
// still pass the cache, the query and the output buffer; the split-K partial results (and the merge
// counters of the persistent kernel) that kv1b_attend keeps in its caller-provided workspace live
// here in a fixed file-scope device array.
//
// The array occupies KV1B_NOALLOC_SCRATCH_BYTES on every GPU that loads this library, until the
// process exits.  It is shared by all calls and keeps the previous call's contents: every launch
// rewrites all of the partial rows it later reads and zeroes the merge counters it uses (one small
// memset on the stream, no allocation), but two calls whose kernels overlap on the GPU (different
// streams, no ordering between them) race on the array.
#include <cuda.h>
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
void* g_scratch_addr[kMaxDevices] = {};                // device address of g_noalloc_scratch, per device ordinal
unsigned long long g_scratch_ctx[kMaxDevices] = {};    // the context it was looked up in (its unique ID)

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique ID of the calling thread's current context (0 if it cannot be read): a device reset or a
// module reload creates a new context, and the array's address must then be looked up again.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    cudaDriverEntryPointQueryResult q1, q2;
    void* f1 = nullptr;
    void* f2 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory; the device
// address is looked up with the device current, once per device and context, and then reused.
int scratch_address(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KV1B_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KV1B_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();  // 0 before the runtime has made a context current
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's context current
    if (e != cudaSuccess || p == nullptr) return KV1B_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
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
  if (!cache->k_bits || !cache->v_codes || !cache->signs || !cache->d_lengths || !cache->d_status)
    return KV1B_ERR_INVALID_ARG;
  if (q_dtype != KV1B_DTYPE_F32 && q_dtype != KV1B_DTYPE_BF16 && q_dtype != KV1B_DTYPE_F16) return KV1B_ERR_INVALID_ARG;
  if (num_q_heads < 1 || num_q_heads % cache->num_kv_heads != 0) return KV1B_ERR_INVALID_ARG;
  const int G = num_q_heads / cache->num_kv_heads;
  if (G > KV1B_MAX_GROUP) return KV1B_ERR_UNSUPPORTED;
  if (flags != KV1B_ATTEND_TENSOR && flags != KV1B_ATTEND_CUDA_CORE) return KV1B_ERR_INVALID_ARG;
  if (!(scale == scale)) return KV1B_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(out) % 16) return KV1B_ERR_MISALIGNED;

  // Split-K partials of the CUDA-core engine: rows * nsplit * (2 + 128) floats.  The split count is
  // at most 2 * SMs / (batch * kv heads) (kv1b_pick_splits), so rows * nsplit <= 2 * SMs * G and the
  // partials stay under 2 * 148 * 8 * 520 B = 1.2 MB on a B200; a shape that does not fit the array
  // (a larger part) is refused before anything is launched.
  const size_t row_bytes = static_cast<size_t>(kv1b::kPartStride) * sizeof(float);
  const size_t rows = static_cast<size_t>(cache->batch) * num_q_heads;
  int64_t maxlen = 0;
  for (int b = 0; b < cache->batch; ++b) maxlen = cache->h_lengths[b] > maxlen ? cache->h_lengths[b] : maxlen;
  const int nsplit = kv1b_pick_splits(cache->batch, cache->num_kv_heads, maxlen, sm_count());
  if (rows * static_cast<size_t>(nsplit) * row_bytes > KV1B_NOALLOC_SCRATCH_BYTES) return KV1B_ERR_WORKSPACE;

  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != KV1B_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (flags == KV1B_ATTEND_TENSOR) {
    // the persistent kernel where kv1b_attend would use it: partial rows from the array's start, one
    // merge counter per (sequence, kv head) at its end (zeroed by the launch)
    const size_t counter_bytes = (static_cast<size_t>(cache->batch) * cache->num_kv_heads * sizeof(unsigned) + 255) / 256 * 256;
    if (counter_bytes < KV1B_NOALLOC_SCRATCH_BYTES) {
      unsigned char* base = static_cast<unsigned char*>(scratch);
      const int wrc = kv1b_attend_ws_buffers(
          cache, q, q_dtype, num_q_heads, scale, out, reinterpret_cast<float*>(base),
          KV1B_NOALLOC_SCRATCH_BYTES - counter_bytes,
          reinterpret_cast<unsigned*>(base + KV1B_NOALLOC_SCRATCH_BYTES - counter_bytes), st);
      if (wrc != KV1B_ERR_UNSUPPORTED && wrc != KV1B_ERR_WORKSPACE) return wrc;
    }
  }

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
  const cudaError_t e = kv1b_launch_attend(p, G, st);
  return e == cudaSuccess ? KV1B_OK : KV1B_ERR_CUDA;
}
