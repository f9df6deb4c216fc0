// kv1b_attend.cu -- split-K decode attention over the compressed cache, its merge, and the
// query-preparation / proxy-score test hooks.
//
// Per (sequence b, kv-head, split) one CTA of 256 threads walks its token range in chunks of 256:
//   phase S  (thread = token): binary x INT4 popcount scores of the G query heads of this kv-head
//            ("RaBitQCache", abstract / key design), online-softmax update in log2 units, and the
//            per-(token, group, head) weights p * scale written to shared memory;
//   phase PV (warp = 16 channels, lane = channel x half of each 16-token step): the
//            probability-weighted sum of the 4-bit values on the CUDA cores in fp32 ("H1B-KV",
//            technical framework: weights from the sketch, then the 4-bit values).
// The dequantised value is min + scale*code = mid + scale*(code - 8) with mid = min + 8 scale;
// the mid term is accumulated per (head, group) in fp32 by phase S.  This kernel serves every
// shape (any G <= 8, unequal lengths, a forced split count); the persistent tensor-core kernel
// (kv1b_attend_ws.cu) takes the common shapes.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

constexpr int kThreads = 256;  // = tokens per chunk
constexpr float kLog2e = 0x1.715476p+0f;  // log2(e) rounded to fp32

__device__ __forceinline__ float exp2_of_int(int e) { return __int_as_float((e + 127) << 23); }

template <int G>
__device__ __forceinline__ float select_head(const float (&v)[G], int h) {
  float r = v[0];
  #pragma unroll
  for (int i = 1; i < G; ++i)
    if (h == i) r = v[i];
  return r;
}

__device__ __forceinline__ void tile_range(int L, int nsplit, int split, int64_t& tok_begin, int64_t& tok_end) {
  const int64_t ntiles = (static_cast<int64_t>(L) + 15) / 16;
  const int64_t t0 = ntiles * split / nsplit, t1 = ntiles * (split + 1) / nsplit;
  tok_begin = 16 * t0;
  tok_end = (16 * t1 < L) ? 16 * t1 : L;
  if (tok_begin > tok_end) tok_begin = tok_end;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 2) attend_kernel(const AttendParams p) {
  extern __shared__ __align__(16) uint8_t smem_dyn[];       // [4 groups][256 tokens][G] weights p * scale
  __shared__ __align__(16) uint32_t s_planes[G][4][4];
  __shared__ float s_vl[G], s_dl[G];
  __shared__ int s_sq[G];
  __shared__ float s_red[kThreads / 32][G + 4];

  const int b = blockIdx.z, kvh = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = p.len[b];
  const CacheView& c = p.c;
  int64_t tok_begin, tok_end;
  tile_range(L, p.nsplit, split, tok_begin, tok_end);

  // ---- prologue: query preparation of the G heads of this kv-head (warp h -> head h)
  if (warp < G) {
    const int hq = kvh * G + warp;
    const QueryPrep qp = query_prep_warp(p.q, (static_cast<int64_t>(b) * p.Hq + hq) * kD, p.q_dtype, c.signs);
    if (lane == 0) {
      #pragma unroll
      for (int j = 0; j < 4; ++j)
        #pragma unroll
        for (int w = 0; w < 4; ++w) s_planes[warp][j][w] = qp.planes[j][w];
      s_vl[warp] = qp.vl;
      s_dl[warp] = qp.delta;
      s_sq[warp] = qp.sq;
    }
  }
  __syncthreads();
  uint32_t P[G][4][4];
  float vl[G], dl[G];
  int sq[G];
  #pragma unroll
  for (int h = 0; h < G; ++h) {
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 pw = *reinterpret_cast<const uint4*>(&s_planes[h][j][0]);
      P[h][j][0] = pw.x; P[h][j][1] = pw.y; P[h][j][2] = pw.z; P[h][j][3] = pw.w;
    }
    vl[h] = s_vl[h];
    dl[h] = s_dl[h];
    sq[h] = s_sq[h];
  }
  const float qs = __fdiv_rn(p.scale, static_cast<float>(kD));

  const int64_t head_tok = (static_cast<int64_t>(b) * c.Hkv + kvh) * c.cap;  // token-major base
  const uint4* kb4 = reinterpret_cast<const uint4*>(c.k_bits) + head_tok;
  const float* kn = c.k_norm + head_tok;
  const float* kc = c.k_cinv + head_tok;
  const uint4* sm4 = reinterpret_cast<const uint4*>(c.v_sm) + head_tok;
  const uint32_t* vcw = c.v_codes + head_tok * 16;  // 128-token tiles of [128 channels][16 words]

  float m_run[G], l_acc[G], mid_acc[G][4];
  #pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_acc[h] = 0.0f;
    #pragma unroll
    for (int g = 0; g < 4; ++g) mid_acc[h][g] = 0.0f;
  }
  float acc[G];        // this lane's channel, its half of every 16-token step
  #pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = 0.0f;

  const int gw = warp >> 1;           // value group owned by this warp in phase PV
  const int ch = 16 * warp + (lane & 15), hf = lane >> 4;

  for (int64_t c0 = tok_begin; c0 < tok_end; c0 += kThreads) {
    // ================= phase S: thread = token
    const int64_t tau = c0 + threadIdx.x;
    const bool valid = tau < tok_end;
    float s2[G], sc[4], mid[4];
    if (valid) {
      const uint4 kb = __ldg(kb4 + tau);
      const float nc = __fmul_rn(__ldg(kn + tau), __ldg(kc + tau));
      const uint4 smv = __ldg(sm4 + tau);
      const uint32_t smw[4] = {smv.x, smv.y, smv.z, smv.w};
      const int32_t Bc = popc_Bc(kb);
      #pragma unroll
      for (int h = 0; h < G; ++h) {
        const int32_t A = popc_A(kb, P[h]);
        s2[h] = __fmul_rn(logit_from_ints(A, Bc, sq[h], vl[h], dl[h], nc, qs), kLog2e);
      }
      #pragma unroll
      for (int g = 0; g < 4; ++g) {
        sc[g] = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[g] & 0xffffu)));
        const float mn = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[g] >> 16)));
        mid[g] = __fmaf_rn(8.0f, sc[g], mn);
      }
    } else {
      #pragma unroll
      for (int h = 0; h < G; ++h) s2[h] = -INFINITY;
      #pragma unroll
      for (int g = 0; g < 4; ++g) sc[g] = mid[g] = 0.0f;
    }
    // chunk maxima of the logits (per head) and of the scales (per group)
    float red[G + 4];
    #pragma unroll
    for (int h = 0; h < G; ++h) red[h] = s2[h];
    #pragma unroll
    for (int g = 0; g < 4; ++g) red[G + g] = sc[g];
    #pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
      #pragma unroll
      for (int i = 0; i < G + 4; ++i) red[i] = fmaxf(red[i], __shfl_xor_sync(kFull, red[i], m));
    if (lane == 0)
      #pragma unroll
      for (int i = 0; i < G + 4; ++i) s_red[warp][i] = red[i];
    __syncthreads();
    #pragma unroll
    for (int i = 0; i < G + 4; ++i) {
      float v = s_red[0][i];
      #pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) v = fmaxf(v, s_red[w][i]);
      red[i] = v;
    }
    float alpha[G], pr[G];
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m_new = fmaxf(m_run[h], red[h]);
      alpha[h] = (m_new == -INFINITY) ? 1.0f : exp2f(m_run[h] - m_new);
      pr[h] = (valid && m_new != -INFINITY) ? exp2f(s2[h] - m_new) : 0.0f;
      m_run[h] = m_new;
      l_acc[h] = __fmaf_rn(l_acc[h], alpha[h], pr[h]);
      #pragma unroll
      for (int g = 0; g < 4; ++g) mid_acc[h][g] = __fmaf_rn(pr[h], mid[g], __fmul_rn(mid_acc[h][g], alpha[h]));
    }
    // weights of this token
    {
      #pragma unroll
      for (int g = 0; g < 4; ++g) {
        float* dst = reinterpret_cast<float*>(smem_dyn) + (g * kThreads + threadIdx.x) * G;
        #pragma unroll
        for (int h = 0; h < G; ++h) dst[h] = __fmul_rn(pr[h], sc[g]);
      }
    }
    __syncthreads();
    // ================= phase PV: warp = channels 16 warp .. 16 warp + 15; lane = (channel, token half)
    const int nsteps = static_cast<int>((tok_end - c0 + 15) / 16) < 16 ? static_cast<int>((tok_end - c0 + 15) / 16) : 16;
    #pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = __fmul_rn(acc[h], alpha[h]);
    const float* wbase = reinterpret_cast<const float*>(smem_dyn) + gw * kThreads * G;
    #pragma unroll 2
    for (int ks = 0; ks < nsteps; ++ks) {
      const int64_t t8 = c0 + 16 * ks + 8 * hf;  // first of this lane's 8 tokens (a multiple of 8)
      const uint32_t w = __ldg(vcw + ((t8 >> 7) * kD + ch) * 16 + ((t8 & 127) >> 3));
      #pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float cv = __int_as_float(0x4B000000 | ((w >> (4 * j)) & 0xFu)) - 8388616.0f;  // c - 8, exact
        const float* wt = wbase + (16 * ks + 8 * hf + j) * G;
        #pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = __fmaf_rn(wt[h], cv, acc[h]);
      }
    }
    __syncthreads();
  }

  // ================= epilogue: CTA sums of l and of the mid terms, then this split's partial
  __shared__ float s_sum[kThreads / 32][G * 5];
  {
    float v[G * 5];
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      v[h * 5] = l_acc[h];
      #pragma unroll
      for (int g = 0; g < 4; ++g) v[h * 5 + 1 + g] = mid_acc[h][g];
    }
    #pragma unroll
    for (int m = 16; m >= 1; m >>= 1)
      #pragma unroll
      for (int i = 0; i < G * 5; ++i) v[i] += __shfl_xor_sync(kFull, v[i], m);
    if (lane == 0)
      #pragma unroll
      for (int i = 0; i < G * 5; ++i) s_sum[warp][i] = v[i];
  }
  __syncthreads();
  const int64_t part_row0 = (static_cast<int64_t>(b) * p.Hq + kvh * G) * p.nsplit + split;  // head 0
  auto part_ptr = [&](int h) { return p.part + (part_row0 + static_cast<int64_t>(h) * p.nsplit) * kPartStride; };
  auto total = [&](int i) {
    float t = 0.0f;
    #pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += s_sum[w][i];
    return t;
  };
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    part_ptr(h)[0] = select_head<G>(m_run, h);
    part_ptr(h)[1] = total(h * 5);
  }
  #pragma unroll
  for (int h = 0; h < G; ++h) acc[h] = __fadd_rn(acc[h], __shfl_xor_sync(kFull, acc[h], 16));
  if (hf == 0) {
    #pragma unroll
    for (int h = 0; h < G; ++h) part_ptr(h)[2 + ch] = __fadd_rn(acc[h], total(h * 5 + 1 + gw));
  }
}

// log-sum-exp merge of the split partials; one block of 128 threads (channels) per (b, hq).
// Split maxima and weights are formed in parallel, then each channel sums the splits with
// independent loads (nsplit <= 1024).  Partial row k of output row r sits at part + r * row_stride +
// k * split_stride; with partial_out the merged row (m, l, o[128]) is written instead of o / l.
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ part, float* __restrict__ out,
                                                    int nsplit, int64_t row_stride, int64_t split_stride,
                                                    int partial_out) {
  __shared__ float s_w[1024];
  __shared__ float s_red[4];
  const int64_t row = blockIdx.x;  // b * Hq + hq
  const float* pr = part + row * row_stride;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float M = -INFINITY;
  for (int k = threadIdx.x; k < nsplit; k += 128) M = fmaxf(M, pr[k * split_stride]);
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, m));
  if (lane == 0) s_red[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();
  float den = 0.0f;
  for (int k = threadIdx.x; k < nsplit; k += 128) {
    const float ms = pr[k * split_stride];
    const float w = (ms != -INFINITY && M != -INFINITY) ? exp2f(ms - M) : 0.0f;
    s_w[k] = w;
    den = __fmaf_rn(w, pr[k * split_stride + 1], den);
  }
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) den += __shfl_xor_sync(kFull, den, m);
  if (lane == 0) s_red[warp] = den;
  __syncthreads();
  den = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
  float num = 0.0f;
  #pragma unroll 8
  for (int k = 0; k < nsplit; ++k) num = __fmaf_rn(s_w[k], pr[k * split_stride + 2 + threadIdx.x], num);
  if (partial_out) {
    float* o = out + row * kPartStride;
    if (threadIdx.x == 0) {
      o[0] = M;
      o[1] = den;
    }
    o[2 + threadIdx.x] = num;
  } else {
    out[row * kD + threadIdx.x] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
  }
}

// ---------------------------------------------------------------------------------------------
// Test hooks.
__global__ void __launch_bounds__(32) query_prep_kernel(const CacheView c, const void* q, int q_dtype, int Hq,
                                                        uint32_t* planes, float* vl, float* delta, int32_t* sq) {
  const int64_t row = blockIdx.x;  // b * Hq + hq
  const QueryPrep qp = query_prep_warp(q, row * kD, q_dtype, c.signs);
  if (threadIdx.x < 16) planes[row * 16 + threadIdx.x] = qp.planes[threadIdx.x >> 2][threadIdx.x & 3];
  if (threadIdx.x == 0) {
    vl[row] = qp.vl;
    delta[row] = qp.delta;
    sq[row] = qp.sq;
  }
}

// Scores of every token of every query head (grid: token blocks x kv-heads x sequences).
__global__ void __launch_bounds__(256) scores_kernel(const ScoresParams p, int G) {
  __shared__ __align__(16) uint32_t s_planes[KV1B_MAX_GROUP][4][4];
  __shared__ float s_vl[KV1B_MAX_GROUP], s_dl[KV1B_MAX_GROUP];
  __shared__ int s_sq[KV1B_MAX_GROUP];
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CacheView& c = p.c;
  if (warp < G) {
    const QueryPrep qp =
        query_prep_warp(p.q, (static_cast<int64_t>(b) * p.Hq + kvh * G + warp) * kD, p.q_dtype, c.signs);
    if (lane == 0) {
      for (int j = 0; j < 4; ++j)
        for (int w = 0; w < 4; ++w) s_planes[warp][j][w] = qp.planes[j][w];
      s_vl[warp] = qp.vl;
      s_dl[warp] = qp.delta;
      s_sq[warp] = qp.sq;
    }
  }
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= p.len[b]) return;
  const int64_t head_tok = (static_cast<int64_t>(b) * c.Hkv + kvh) * c.cap;
  const uint4 kb = __ldg(reinterpret_cast<const uint4*>(c.k_bits) + head_tok + t);
  const float nc = __fmul_rn(__ldg(c.k_norm + head_tok + t), __ldg(c.k_cinv + head_tok + t));
  const int32_t Bc = popc_Bc(kb);
  const float qs = __fdiv_rn(p.scale, static_cast<float>(kD));
  for (int h = 0; h < G; ++h) {
    uint32_t P[4][4];
    for (int j = 0; j < 4; ++j)
      for (int w = 0; w < 4; ++w) P[j][w] = s_planes[h][j][w];
    const int32_t A = popc_A(kb, P);
    const int64_t o = (static_cast<int64_t>(b) * p.Hq + kvh * G + h) * c.cap + t;
    if (p.A) p.A[o] = A;
    if (p.Bc) p.Bc[o] = Bc;
    p.s[o] = logit_from_ints(A, Bc, s_sq[h], s_vl[h], s_dl[h], nc, qs);
  }
}

template <int G>
static cudaError_t launch_attend_t(const AttendParams& p, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(4) * kThreads * G * 4;
  auto kern = attend_kernel<G>;
  static std::atomic<unsigned long long> configured{0};  // per template instance, bit per device
  const cudaError_t e = configure_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem), &configured);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsplit, p.c.Hkv, p.c.B);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace kv1b

using namespace kv1b;

int kv1b_pick_splits(int32_t B, int32_t Hkv, int64_t max_len, int num_sms) {
  const int64_t units = static_cast<int64_t>(B) * Hkv;
  int64_t ns = (2LL * num_sms) / (units > 0 ? units : 1);
  const int64_t by_len = max_len / 512;
  if (ns > by_len) ns = by_len;
  if (ns < 1) ns = 1;
  if (ns > 1024) ns = 1024;
  return static_cast<int>(ns);
}

cudaError_t kv1b_launch_attend(const AttendParams& p, int32_t G, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
#define KV1B_CASE(GG)                      \
  case GG:                                 \
    e = launch_attend_t<GG>(p, stream);    \
    break;
  switch (G) {
    KV1B_CASE(1)
    KV1B_CASE(2)
    KV1B_CASE(3)
    KV1B_CASE(4)
    KV1B_CASE(5)
    KV1B_CASE(6)
    KV1B_CASE(7)
    KV1B_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef KV1B_CASE
  if (e != cudaSuccess) return e;
  merge_kernel<<<p.c.B * p.Hq, 128, 0, stream>>>(p.part, p.out, p.nsplit, static_cast<int64_t>(p.nsplit) * kPartStride,
                                                  kPartStride, p.partial_out);
  return cudaGetLastError();
}

// Log-sum-exp merge of nsplit partial rows (m in log2 units, l, o[128]) per row: [rows][nsplit][2 + 128].
cudaError_t kv1b_launch_merge(const float* part, float* out, int32_t rows, int32_t nsplit, cudaStream_t stream) {
  if (nsplit < 1 || nsplit > 1024 || rows < 1) return cudaErrorInvalidValue;
  merge_kernel<<<rows, 128, 0, stream>>>(part, out, nsplit, static_cast<int64_t>(nsplit) * kPartStride, kPartStride, 0);
  return cudaGetLastError();
}

cudaError_t kv1b_launch_merge_strided(const float* part, float* out, int64_t rows, int32_t nsplit, int64_t row_stride,
                                      int64_t split_stride, bool partial_out, cudaStream_t stream) {
  if (nsplit < 1 || nsplit > 1024 || rows < 1 || rows > 0x7fffffff) return cudaErrorInvalidValue;
  merge_kernel<<<static_cast<unsigned>(rows), 128, 0, stream>>>(part, out, nsplit, row_stride, split_stride,
                                                                partial_out ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t kv1b_launch_query_prep(const CacheView& c, const void* q, int32_t q_dtype, int32_t Hq, uint32_t* planes,
                                   float* vl, float* delta, int32_t* sq, cudaStream_t stream) {
  query_prep_kernel<<<c.B * Hq, 32, 0, stream>>>(c, q, q_dtype, Hq, planes, vl, delta, sq);
  return cudaGetLastError();
}

cudaError_t kv1b_launch_scores(const ScoresParams& p, int32_t G, int32_t max_len, cudaStream_t stream) {
  if (max_len <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((max_len + 255) / 256), p.c.Hkv, p.c.B);
  scores_kernel<<<grid, 256, 0, stream>>>(p, G);
  return cudaGetLastError();
}
