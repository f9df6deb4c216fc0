// kv1b_topp.cu -- adaptive Top-p attention ("RaBitQCache", abstract / core idea: adaptive Top-p
// retrieval whose token budget follows the actual attention sparsity).
//
// One CTA of 1024 threads per (sequence, query head), after the proxy scores of all tokens have
// been written to the workspace by scores_kernel:
//  1. m = max logit; integer masses u_t ~ 2^32 2^((s_t - m) log2 e) from a degree-7 polynomial of
//     2^f (reproducible bit for bit); U = sum u_t; T = ceil(p U) in fp64, clamped to [1, U].
//  2. Block-wide radix select, 8 passes of 8 bits (most significant first), over the unique
//     64-bit keys  (order-preserving descending code of s) << 32 | t  with per-bin MASS histograms:
//     it finds the smallest key K* whose cumulative mass reaches T.  The selected set is
//     {t : key_t <= K*} -- the shortest prefix of the order (s desc, index asc) reaching T, so
//     equal logits are taken in ascending index order.
//  3. Compaction in index order (ballots + a block scan) gives the ascending index list.
//  4. Gather-attend: softmax over the selected tokens' logits, 4-bit values dequantised on the fly,
//     fp32 accumulation, one warp per selected token at a time.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

constexpr int kToppThreads = 1024;
constexpr int kToppWarps = kToppThreads / 32;
constexpr float kL2e = 0x1.715476p+0f;  // log2(e) rounded to fp32

// (ln 2)^k / k!, k = 0..7, each rounded to the nearest fp32 (Taylor coefficients of 2^f).
__constant__ float kExp2Coef[8] = {0x1p+0f,         0x1.62e43p-1f,   0x1.ebfbep-3f,   0x1.c6b08ep-5f,
                                   0x1.3b2ab6p-7f,  0x1.5d87fep-10f, 0x1.430912p-13f, 0x1.ffcbfcp-17f};

__device__ __forceinline__ uint64_t topp_mass(float s, float m) {
  const float t = __fmul_rn(__fsub_rn(s, m), kL2e);
  if (!(t >= -40.0f)) return 0ull;
  const float n = rintf(t);
  const float f = __fsub_rn(t, n);
  float P = kExp2Coef[7];
  #pragma unroll
  for (int k = 6; k >= 0; --k) P = __fmaf_rn(P, f, kExp2Coef[k]);
  const int e = 32 + static_cast<int>(n);                          // in [-8, 32]
  const float scaled = __fmul_rn(P, __int_as_float((e + 127) << 23)); // exact power-of-two scaling
  return __float2ull_rz(scaled);
}

__device__ __forceinline__ uint64_t topp_key(float s, int64_t t) {
  const uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));  // -0 -> +0 so equal logits tie
  const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(~asc) << 32) | static_cast<uint32_t>(t);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__global__ void __launch_bounds__(kToppThreads) topp_kernel(const ToppParams p) {
  __shared__ unsigned long long hist[256];
  __shared__ unsigned long long s_u64[kToppWarps];
  __shared__ float s_f32[kToppWarps];
  __shared__ int s_cnt[kToppWarps];
  __shared__ unsigned long long s_prefix, s_rem;
  __shared__ float s_acc[kToppWarps][kD];
  __shared__ float s_l[kToppWarps];

  const int hq = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CacheView& c = p.c;
  const int G = p.Hq / c.Hkv, kvh = hq / G;
  const int64_t L = p.len[b];
  const int64_t row = static_cast<int64_t>(b) * p.Hq + hq;
  const float* s = p.s + row * c.cap;
  int32_t* sel = p.sel_idx + row * c.cap;
  float* out = p.out + row * kD;
  if (L == 0) {
    if (threadIdx.x < kD) out[threadIdx.x] = 0.0f;
    if (threadIdx.x == 0) p.sel_cnt[row] = 0;
    return;
  }
  // ---- 1. max and total mass
  float m = -INFINITY;
  for (int64_t t = threadIdx.x; t < L; t += kToppThreads) m = fmaxf(m, s[t]);
  #pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  if (lane == 0) s_f32[warp] = m;
  __syncthreads();
  m = s_f32[0];
  for (int w = 1; w < kToppWarps; ++w) m = fmaxf(m, s_f32[w]);
  unsigned long long U = 0;
  for (int64_t t = threadIdx.x; t < L; t += kToppThreads) U += topp_mass(s[t], m);
  U = warp_sum(U);
  if (lane == 0) s_u64[warp] = U;
  __syncthreads();
  U = 0;
  for (int w = 0; w < kToppWarps; ++w) U += s_u64[w];
  unsigned long long T = static_cast<unsigned long long>(ceil(static_cast<double>(p.p) * static_cast<double>(U)));
  if (T > U) T = U;
  if (T < 1) T = 1;
  // ---- 2. radix select over 64-bit keys, mass histograms
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_rem = T;
  }
  for (int d = 7; d >= 0; --d) {
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int64_t t = threadIdx.x; t < L; t += kToppThreads) {
      const float st = s[t];
      const uint64_t key = topp_key(st, t);
      if (d == 7 || (key >> (8 * (d + 1))) == prefix) {
        const uint64_t u = topp_mass(st, m);
        if (u) atomicAdd(&hist[(key >> (8 * d)) & 255u], static_cast<unsigned long long>(u));
      }
    }
    __syncthreads();
    if (warp == 0) {
      const unsigned long long rem = s_rem;
      unsigned long long loc = 0;
      #pragma unroll
      for (int i = 0; i < 8; ++i) loc += hist[8 * lane + i];
      unsigned long long incl = loc;
      #pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned long long excl = incl - loc;
      const unsigned ball = __ballot_sync(kFull, incl >= rem);
      const int first = ball ? __ffs(ball) - 1 : 31;  // the mass invariant guarantees ball != 0
      if (lane == first) {
        unsigned long long cum = excl;
        int bin = 8 * lane + 7;
        for (int i = 0; i < 8; ++i) {
          const unsigned long long hb = hist[8 * lane + i];
          if (cum + hb >= rem) {
            bin = 8 * lane + i;
            break;
          }
          cum += hb;
        }
        s_rem = rem - cum;
        s_prefix = (prefix << 8) | static_cast<unsigned long long>(bin);
      }
    }
    __syncthreads();
  }
  const unsigned long long kstar = s_prefix;
  // ---- 3. compaction of {t : key_t <= K*} in ascending index order
  int base = 0;
  for (int64_t t0 = 0; t0 < L; t0 += kToppThreads) {
    const int64_t t = t0 + threadIdx.x;
    const bool f = t < L && topp_key(s[t], t) <= kstar;
    const unsigned ball = __ballot_sync(kFull, f);
    if (lane == 0) s_cnt[warp] = __popc(ball);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < kToppWarps; ++w) {
      const int cw = s_cnt[w];
      before += (w < warp) ? cw : 0;
      tot += cw;
    }
    if (f) sel[base + before + __popc(ball & ((1u << lane) - 1u))] = static_cast<int32_t>(t);
    base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.sel_cnt[row] = base;
  __syncthreads();  // sel[] written by the whole block before the gather reads it
  // ---- 4. gather-attend over the selected tokens; lane l owns channels 4l..4l+3
  const int64_t head_tok = (static_cast<int64_t>(b) * c.Hkv + kvh) * c.cap;
  const uint32_t* vcw = c.v_codes + head_tok * 16;
  const uint32_t* vsm = c.v_sm + head_tok * 4;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float lsum = 0.0f;
  const int grp = lane >> 3;                // 32-channel group
  for (int i = warp; i < base; i += kToppWarps) {
    const int64_t t = sel[i];
    const float e = exp2f(__fmul_rn(__fsub_rn(s[t], m), kL2e));
    lsum += e;
    // code plane: 128-token tiles, channel-major rows of 16 words, nibble j of word w = token 8w + j
    const uint32_t* row = vcw + ((t >> 7) * kD + 4 * lane) * 16 + ((t & 127) >> 3);
    const int shift = 4 * static_cast<int>(t & 7);
    const uint32_t smw = vsm[t * 4 + grp];
    const float scl = __half2float(__ushort_as_half(static_cast<unsigned short>(smw & 0xffffu)));
    const float mnv = __half2float(__ushort_as_half(static_cast<unsigned short>(smw >> 16)));
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float code = static_cast<float>((row[16 * r] >> shift) & 0xFu);
      acc[r] = __fmaf_rn(e, __fmaf_rn(scl, code, mnv), acc[r]);
    }
  }
  #pragma unroll
  for (int r = 0; r < 4; ++r) s_acc[warp][4 * lane + r] = acc[r];
  if (lane == 0) s_l[warp] = lsum;
  __syncthreads();
  if (threadIdx.x < kD) {
    float num = 0.0f, den = 0.0f;
    for (int w = 0; w < kToppWarps; ++w) {
      num += s_acc[w][threadIdx.x];
      den += s_l[w];
    }
    out[threadIdx.x] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
  }
}

}  // namespace kv1b

using namespace kv1b;

cudaError_t kv1b_launch_topp(const ToppParams& p, cudaStream_t stream) {
  dim3 grid(p.Hq, p.c.B);
  topp_kernel<<<grid, kToppThreads, 0, stream>>>(p);
  return cudaGetLastError();
}
