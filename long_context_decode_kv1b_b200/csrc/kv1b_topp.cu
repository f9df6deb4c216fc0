// kv1b_topp.cu -- adaptive Top-p attention ("RaBitQCache", abstract / core idea: adaptive Top-p
// retrieval whose token budget follows the actual attention sparsity), as a pipeline of
// grid-wide kernels so that a long context is spread over every SM.  Per row r = (sequence,
// query head), with the reproducible integer masses u_t ~ 2^32 2^((s_t - m) log2 e) (degree-7
// polynomial of 2^f, bit for bit the same as the CPU reference) and T = ceil(p U) in fp64:
//  0. query preparation (rotation, 4-bit codes, bit-planes) once per row;
//  1. scores: the binary x INT4 integers A = sum_i bit_i code_i and Bc = sum_i bit_i of every token
//     on the integer tensor cores (exact), then the fp32 logit in the fixed operation order; the row
//     maximum m by atomicMax on an order-preserving key;
//  2. masses: u_t, the row total U, and a histogram of masses over 2048 buckets of
//     t = (s - m) log2 e (bucket floor(-64 t), monotone in s, the last one also holding
//     t in [-40, -32); t < -40 has no mass);
//  3. threshold: the first bucket b* where the cumulative mass reaches T; rem = the mass still
//     needed inside b*;
//  4. candidates: the tokens of bucket b* (any order), and per chunk the count of tokens in lower
//     buckets (all of them selected);
//  5. resolve: a block-wide radix select over the candidates' unique 64-bit keys
//     (order-preserving descending code of s) << 32 | t finds the smallest key K* whose cumulative
//     candidate mass reaches rem, and adds the selected candidates to their chunks' counts;
//  6. the selected set {t : bucket(t) < b*} U {t in b* : key_t <= K*} -- the shortest prefix of the
//     order (s desc, index asc) whose mass reaches T -- is written in ascending index order (chunk
//     offsets from the counts), and in the same pass the chunk's selected tokens are gathered: the
//     softmax numerator and denominator against m, 4-bit values dequantised on the fly, fp32;
//  7. merge: the chunk partials summed in chunk order.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

constexpr float kL2e = 0x1.715476p+0f;  // log2(e) rounded to fp32
constexpr int kStreamThreads = 256;
constexpr int kStreamWarps = kStreamThreads / 32;
constexpr int kTokPerThread = kToppChunk / kStreamThreads;  // contiguous tokens per thread
static_assert(kTokPerThread == 16, "the streaming kernels hold 16 tokens per thread");
constexpr int kScoreTok = 2048;          // tokens per block of the score kernel
constexpr int kResolveThreads = 1024;
constexpr int kResolveSmemCand = 4096;   // candidates whose keys and masses the resolve keeps on chip
                                         // (64 KB: three resolve blocks per SM)
constexpr size_t kResolveSmem = static_cast<size_t>(kResolveSmemCand) * 16;
constexpr int kResolveSmallCand = 128;   // up to this many candidates: direct ranking, no radix passes

__device__ __forceinline__ float topp_t(float s, float m) { return __fmul_rn(__fsub_rn(s, m), kL2e); }

// u = trunc(P(f) 2^(32 + n)), n = rint(t), f = t - n, P the degree-7 Taylor polynomial of 2^f with
// coefficients (ln 2)^k / k! each rounded to the nearest fp32 (Horner, fused multiply-adds); 0 for
// t < -40.  Branch-free: for t in [-40, 0], n in [-40, 0] converts through the 1.5 * 2^23 rounding
// constant (exact), the scaling by 2^(32 + n) is exact, and P 2^(32 + n) <= 2^32 (equal only at
// t = 0, where P(0) = 1), so a 32-bit truncation plus that one case gives the 64-bit value.
__device__ __forceinline__ uint64_t topp_mass_t(float t) {
  const float tc = fmaxf(t, -40.0f);
  const float r = __fadd_rn(tc, 12582912.0f);  // 1.5 * 2^23 + rint(tc)
  const float n = __fsub_rn(r, 12582912.0f);
  const float f = __fsub_rn(tc, n);
  float P = 0x1.ffcbfcp-17f;                   // (ln 2)^7 / 7!
  P = __fmaf_rn(P, f, 0x1.430912p-13f);        // (ln 2)^6 / 6!
  P = __fmaf_rn(P, f, 0x1.5d87fep-10f);        // (ln 2)^5 / 5!
  P = __fmaf_rn(P, f, 0x1.3b2ab6p-7f);         // (ln 2)^4 / 4!
  P = __fmaf_rn(P, f, 0x1.c6b08ep-5f);         // (ln 2)^3 / 3!
  P = __fmaf_rn(P, f, 0x1.ebfbep-3f);          // (ln 2)^2 / 2!
  P = __fmaf_rn(P, f, 0x1.62e43p-1f);          // ln 2
  P = __fmaf_rn(P, f, 1.0f);
  const int ni = __float_as_int(r) - 0x4B400000;                      // rint(tc) as an integer
  const float scaled = __fmul_rn(P, __int_as_float((ni + 32 + 127) << 23)); // exact power-of-two scaling
  const uint64_t u = scaled >= 4294967296.0f ? (1ull << 32) : static_cast<uint64_t>(__float2uint_rz(scaled));
  return t >= -40.0f ? u : 0ull;
}

// Bucket of t = (s - m) log2 e: floor(-64 t) for t in [-40, 0], at most kToppBuckets - 1 (a
// non-decreasing function of -t, hence of the key order); kToppBuckets below -40 (no mass there).
__device__ __forceinline__ int topp_bucket(float t) {
  // floor(-64 t) for -64 t in [0, 2560]: 2^23 + x rounded toward zero is 2^23 + floor(x)
  const int b = __float_as_int(__fadd_rz(__fmul_rn(-fmaxf(t, -40.0f), 64.0f), 8388608.0f)) - 0x4B000000;
  return t >= -40.0f ? (b < kToppBuckets - 1 ? b : kToppBuckets - 1) : kToppBuckets;
}

// Top-k bucket (unit masses, so the logit range matters, not the mass range): the float bits of
// d = m - s >= 0 (non-increasing in s, so non-decreasing in the key order), 128 buckets per binade
// for d in [2^-8, 2^8); smaller d -> 0, larger -> the last bucket.
__device__ __forceinline__ int topk_bucket(float s, float m) {
  const float d = __fsub_rn(m, s);
  const int b = static_cast<int>(__float_as_uint(d) >> 16) - ((127 - 8) << 7);
  return b < 0 ? 0 : (b > kToppBuckets - 1 ? kToppBuckets - 1 : b);
}

__device__ __forceinline__ uint64_t topp_key(float s, int64_t t) {
  const uint32_t u = __float_as_uint(__fadd_rn(s, 0.0f));  // -0 -> +0 so equal logits tie
  const uint32_t asc = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(~asc) << 32) | static_cast<uint32_t>(t);
}
// order-preserving uint32 of a float (for atomicMax) and back
__device__ __forceinline__ uint32_t fkey(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_inv(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}
__device__ __forceinline__ unsigned warp_incl_scan(unsigned v) {
  const int lane = threadIdx.x & 31;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned x = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += x;
  }
  return v;
}

__device__ __forceinline__ int row_len(const ToppParams& p, int64_t r) { return p.len[r / p.Hq]; }

// 16 logits t0 .. t0 + 15 of a row (t0 a multiple of 16; the row holds cap floats, cap a multiple
// of 128, so whole float4s stay inside it); entries at or past t1 are left unspecified.
__device__ __forceinline__ void load16(const float* s, int64_t t0, int64_t t1, float v[16]) {
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (t0 + 4 * q < t1) x = *reinterpret_cast<const float4*>(s + t0 + 4 * q);
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
}


// ---------------------------------------------------------------- 1. logits and row maxima
// Integer MMA D += A B (16 x 32 s8 by 32 x 8 s8 -> s32).
__device__ __forceinline__ void mma_s8(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Sign bits of 16 tokens against 8 operand columns.  Lane (g, t) holds word t (channels 32t..32t+31)
// of tokens g and g + 8.  K-block kb uses the bits at positions 8j + 2kb and 8j + 2kb + 1 of the word
// (after a 4-bit shift for kb >= 2), masked in place so each byte is bit * 2^(position & 3); the
// query column carries code * 2^(3 - (position & 3)) for the same channel, so every product is
// 8 * bit * code and D = 8 * sum_i bit_i code_i exactly (columns of ones give 8 * Bc).
__device__ __forceinline__ void bits_mma(int d[4], uint32_t w0, uint32_t w8, const uint32_t (&bq)[4][2]) {
  d[0] = d[1] = d[2] = d[3] = 0;
  const uint32_t x0[2] = {w0, w0 >> 4}, x8[2] = {w8, w8 >> 4};
  #pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    const uint32_t mlo = 0x01010101u << (2 * (kb & 1)), mhi = mlo << 1;
    const uint32_t a[4] = {x0[kb >> 1] & mlo, x8[kb >> 1] & mlo, x0[kb >> 1] & mhi, x8[kb >> 1] & mhi};
    mma_s8(d, a, bq[kb][0], bq[kb][1]);
  }
}

// Query operand of lane (g, t): column g, k = 4t..4t+3 (register 0) and 16+4t..16+4t+3 (register 1)
// of each k-block.  planes_row: the head's bit-planes for a code column, nullptr otherwise.
__device__ __forceinline__ void build_bq(uint32_t (&bq)[4][2], const uint32_t* planes_row, int t, bool ones_col) {
  uint32_t pw[4] = {0u, 0u, 0u, 0u};
  if (planes_row) {
    #pragma unroll
    for (int j = 0; j < 4; ++j) pw[j] = planes_row[4 * j + t];
  }
  #pragma unroll
  for (int kb = 0; kb < 4; ++kb)
    #pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const int r = 2 * kb + hi;
      const int sh = 3 - (r & 3);
      uint32_t code = 0u;
      #pragma unroll
      for (int j = 0; j < 4; ++j) code |= ((pw[j] >> r) & 0x01010101u) << j;
      bq[kb][hi] = planes_row ? (code << sh) : (ones_col ? (0x01010101u << sh) : 0u);
    }
}

// grid (token blocks of kScoreTok, kv-heads, sequences); warp = 64 tokens at a time, up to 4 NG
// heads as NG groups of 4 operand-column pairs.  PROBE: the test instantiation that also writes the
// raw products 8 A and 8 Bc of every token (p.probe_A / probe_Bc).
template <int NG, bool PROBE>
__global__ void __launch_bounds__(kStreamThreads, NG == 1 ? 4 : 2) topp_scores_kernel(const ToppParams p, int G) {
  pdl_wait();
  __shared__ float s_max[kStreamWarps][8];
  const CacheView& c = p.c;
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int L = p.len[b];
  const int64_t row0 = static_cast<int64_t>(b) * p.Hq + static_cast<int64_t>(kvh) * G;
  const float qs = __fdiv_rn(p.scale, static_cast<float>(kD));
  uint32_t bq[NG][4][2];
  float cdl[NG], cvl[NG];
  int32_t csq[NG];
  bool hv[NG];
  #pragma unroll
  for (int hg = 0; hg < NG; ++hg) {
    const int hc = 4 * hg + (g >> 1);  // head of this lane's operand column
    const bool code_col = (g & 1) == 0 && hc < G;
    build_bq(bq[hg], code_col ? p.planes + (row0 + hc) * 16 : nullptr, t, (g & 1) != 0);
    const int ht = 4 * hg + t;  // head of this lane's output column
    hv[hg] = ht < G;
    cdl[hg] = hv[hg] ? p.qdl[row0 + ht] : 0.0f;
    cvl[hg] = hv[hg] ? p.qvl[row0 + ht] : 0.0f;
    csq[hg] = hv[hg] ? p.qsq[row0 + ht] : 0;
  }
  float mx[NG];
  float* srow[NG];  // this lane's output row per head group
  #pragma unroll
  for (int hg = 0; hg < NG; ++hg) {
    mx[hg] = -INFINITY;
    srow[hg] = p.s + (row0 + (hv[hg] ? 4 * hg + t : 0)) * c.cap;
  }
  const int64_t head_tok = (static_cast<int64_t>(b) * c.Hkv + kvh) * c.cap;
  const uint32_t* kw = c.k_bits + head_tok * 4 + t;
  const float* kn = c.k_norm + head_tok;
  const float* ki = c.k_cinv + head_tok;
  const int tb0 = blockIdx.x * kScoreTok;
  const int tend = tb0 + kScoreTok < L ? tb0 + kScoreTok : L;
  for (int base = tb0 + 64 * warp; base < tend; base += 64 * kStreamWarps) {  // warp-uniform
    uint32_t w[8];
    float nc[8];
    const int nvt = tend - base - g;  // token base + g + 8 i is valid for 8 i < nvt
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tok = base + g + 8 * i;
      const bool v = 8 * i < nvt;
      w[i] = v ? __ldg(kw + 4 * tok) : 0u;
      nc[i] = v ? __fmul_rn(__ldg(kn + tok), __ldg(ki + tok)) : 0.0f;
    }
    #pragma unroll
    for (int hg = 0; hg < NG; ++hg) {
      #pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        int d[4];
        bits_mma(d, w[2 * kk], w[2 * kk + 1], bq[hg]);
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 2 * kk + e;  // token base + g + 8 i
          if (hv[hg] && 8 * i < nvt) {
            const float sv =
                logit_from_ints(d[2 * e] >> 3, d[2 * e + 1] >> 3, csq[hg], cvl[hg], cdl[hg], nc[i], qs);
            srow[hg][base + g + 8 * i] = sv;
            if constexpr (PROBE) {
              const int64_t o = (srow[hg] - p.s) + base + g + 8 * i;
              p.probe_A[o] = d[2 * e];
              p.probe_Bc[o] = d[2 * e + 1];
            }
            mx[hg] = fmaxf(mx[hg], sv);
          }
        }
      }
    }
  }
  #pragma unroll
  for (int hg = 0; hg < NG; ++hg) {
    #pragma unroll
    for (int o = 4; o <= 16; o <<= 1) mx[hg] = fmaxf(mx[hg], __shfl_xor_sync(kFull, mx[hg], o));
    if (g == 0) s_max[warp][4 * hg + t] = mx[hg];
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float m = s_max[0][threadIdx.x];
    for (int w = 1; w < kStreamWarps; ++w) m = fmaxf(m, s_max[w][threadIdx.x]);
    if (m != -INFINITY) atomicMax(&p.rows[row0 + threadIdx.x].maxkey, fkey(m));
  }
}

// ---------------------------------------------------------------- 2. masses and bucket histogram
// grid (chunks of kToppChunk tokens, rows); thread = 16 contiguous tokens.  u < 2^33 is split as
// uh 2^16 + ul (ul < 2^16, uh < 2^17); per bucket the block sums ul and uh separately with 32-bit
// shared reductions (at most 4096 tokens: no overflow), then adds each non-empty bucket's
// (sum uh) 2^16 + sum ul to the row's 64-bit histogram.
template <int MODE>
__global__ void __launch_bounds__(kStreamThreads) topp_mass_kernel(const ToppParams p) {
  constexpr bool topk = MODE == KV1B_SELECT_TOPK;
  pdl_wait();
  __shared__ uint32_t s_lo[kToppBuckets], s_hi[kToppBuckets];  // sums of ul and of uh per bucket
  __shared__ unsigned long long s_u[kStreamWarps], s_w[kStreamWarps];
  const int64_t r = blockIdx.y;
  const int L = row_len(p, r);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kToppChunk;
  if (t0 >= L) return;
  const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
  const int64_t tt0 = t0 + kTokPerThread * threadIdx.x;
  float v[16];
  load16(p.s + r * p.c.cap, tt0, t1, v);
  for (int i = threadIdx.x; i < kToppBuckets; i += kStreamThreads) {
    s_lo[i] = 0u;
    s_hi[i] = 0u;
  }
  __syncthreads();
  const float m = fkey_inv(p.rows[r].maxkey);
  unsigned long long usum = 0ull, wsum = 0ull;
  const int nv = static_cast<int>(t1 - tt0);  // valid tokens of this thread (may be <= 0)
  // the kept window in this thread's local indices: i < wlo or i >= whi
  const int64_t wlo64 = p.sink - tt0, whi64 = static_cast<int64_t>(L) - p.recent - tt0;
  const int wlo = static_cast<int>(wlo64 < 0 ? 0 : (wlo64 > 16 ? 16 : wlo64));
  const int whi = static_cast<int>(whi64 < 0 ? 0 : (whi64 > 16 ? 16 : whi64));
  uint32_t bkw[8];  // the 16 buckets as 16-bit pairs
  // one token outside the window: Top-k gives every token unit mass in its topk_bucket; Top-p its
  // integer mass in its topp_bucket
  auto hist_token = [&](float x) -> int {
    if (topk) {
      const int bk = topk_bucket(x, m);
      atomicAdd(&s_lo[bk], 1u);
      usum += 1ull;
      return bk;
    }
    const float tt = topp_t(x, m);
    const int bk = topp_bucket(tt);
    {
      const uint64_t u = topp_mass_t(tt);
      if (u) {
        atomicAdd(&s_lo[bk], static_cast<uint32_t>(u & 0xffffu));
        atomicAdd(&s_hi[bk], static_cast<uint32_t>(u >> 16));
        usum += u;
      }
    }
    return bk;
  };
  if (nv >= 16 && wlo == 0 && whi == 16) {  // all 16 tokens valid and outside the window
    #pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int bk = hist_token(v[i]);
      if (i & 1) bkw[i >> 1] |= static_cast<uint32_t>(bk) << 16;
      else bkw[i >> 1] = static_cast<uint32_t>(bk);
    }
  } else {
    #pragma unroll
    for (int i = 0; i < 16; ++i) {
      int bk = kToppBuckets;
      if (i < nv) {
        if (i < wlo || i >= whi) {  // kept window: outside the histogram
          bk = kToppWinBucket;
          if (!topk) wsum += topp_mass_t(topp_t(v[i], m));
        } else {
          bk = hist_token(v[i]);
        }
      }
      if (i & 1) bkw[i >> 1] |= static_cast<uint32_t>(bk) << 16;
      else bkw[i >> 1] = static_cast<uint32_t>(bk);
    }
  }
  if (nv > 0) {  // whole 32-byte groups stay inside the row (cap % 128 == 0)
    uint4* bo = reinterpret_cast<uint4*>(p.bk + r * p.c.cap + tt0);
    bo[0] = make_uint4(bkw[0], bkw[1], bkw[2], bkw[3]);
    bo[1] = make_uint4(bkw[4], bkw[5], bkw[6], bkw[7]);
  }
  usum = warp_sum(usum);
  wsum = warp_sum(wsum);
  if ((threadIdx.x & 31) == 0) {
    s_u[threadIdx.x >> 5] = usum;
    s_w[threadIdx.x >> 5] = wsum;
  }
  __syncthreads();
  unsigned long long* hist = p.hist + r * kToppBuckets;
  for (int i = threadIdx.x; i < kToppBuckets; i += kStreamThreads) {
    const unsigned long long h = (static_cast<unsigned long long>(s_hi[i]) << 16) + s_lo[i];
    if (h) atomicAdd(&hist[i], h);
  }
  if (threadIdx.x == 0) {
    unsigned long long tot = 0ull, wtot = 0ull;
    for (int w = 0; w < kStreamWarps; ++w) {
      tot += s_u[w];
      wtot += s_w[w];
    }
    if (tot) atomicAdd(&p.rows[r].U, tot);
    if (wtot) atomicAdd(&p.rows[r].Uw, wtot);
  }
}

// ---------------------------------------------------------------- 3. threshold bucket
// grid (rows), 1024 threads: thread i owns buckets 2i and 2i + 1.
constexpr int kThresholdThreads = kToppBuckets / 2;
__global__ void __launch_bounds__(kThresholdThreads) topp_threshold_kernel(const ToppParams p) {
  pdl_wait();
  __shared__ unsigned long long s_w[kThresholdThreads / 32];
  const int64_t r = blockIdx.x;
  ToppRowState& rs = p.rows[r];
  if (row_len(p, r) == 0) {  // empty row
    if (threadIdx.x == 0) rs.bstar = -1;
    return;
  }
  const unsigned long long U = rs.U, Uw = rs.Uw;
  unsigned long long T;  // mass (Top-k: count) still needed from outside the kept window
  if (p.mode == KV1B_SELECT_TOPK) {
    T = static_cast<unsigned long long>(p.k) < U ? static_cast<unsigned long long>(p.k) : U;
  } else {
    const unsigned long long Ua = U + Uw;
    unsigned long long Tp = static_cast<unsigned long long>(ceil(static_cast<double>(p.p) * static_cast<double>(Ua)));
    if (Tp > Ua) Tp = Ua;
    if (Tp < 1) Tp = 1;
    T = Uw >= Tp ? 0ull : Tp - Uw;
  }
  if (T == 0ull) {  // the kept window alone is the set
    if (threadIdx.x == 0) rs.bstar = -2;
    return;
  }
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const unsigned long long h0 = p.hist[r * kToppBuckets + 2 * i], h1 = p.hist[r * kToppBuckets + 2 * i + 1];
  const unsigned long long loc = h0 + h1;
  unsigned long long incl = loc;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = s_w[lane];
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long v = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += v;
    }
    s_w[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  incl += warp ? s_w[warp - 1] : 0ull;
  const unsigned long long excl = incl - loc;
  // exactly one bucket crosses T (it has mass > 0)
  if (excl < T && T <= excl + h0) {
    rs.bstar = 2 * i;
    rs.rem = T - excl;
  } else if (excl + h0 < T && T <= incl) {
    rs.bstar = 2 * i + 1;
    rs.rem = T - excl - h0;
  }
}

// ---------------------------------------------------------------- 4. candidates and lower-bucket counts
static_assert(kToppChunk % kToppSub == 0 && kToppSub % (32 * kTokPerThread) == 0, "sub-chunks are whole warps");
// grid (chunks, rows); thread = 16 contiguous tokens.
__global__ void __launch_bounds__(kStreamThreads) topp_cand_kernel(const ToppParams p) {
  pdl_wait();
  __shared__ unsigned s_c[kStreamWarps];
  const int64_t r = blockIdx.y;
  const int L = row_len(p, r);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kToppChunk;
  ToppRowState& rs = p.rows[r];
  const int bstar = rs.bstar;
  if (t0 >= L || bstar == -1) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
  const int64_t tt0 = t0 + kTokPerThread * threadIdx.x;
  uint32_t bkw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  const int nv = static_cast<int>(t1 - tt0);  // valid tokens of this thread (may be <= 0)
  if (nv > 0) {
    const uint4* bi = reinterpret_cast<const uint4*>(p.bk + r * p.c.cap + tt0);
    const uint4 a = bi[0], b = bi[1];
    bkw[0] = a.x; bkw[1] = a.y; bkw[2] = a.z; bkw[3] = a.w;
    bkw[4] = b.x; bkw[5] = b.y; bkw[6] = b.z; bkw[7] = b.w;
  }
  unsigned lo = 0, cmask = 0;
  #pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (i < nv) {
      const int bk = static_cast<int>((bkw[i >> 1] >> (16 * (i & 1))) & 0xffffu);
      lo += (bk < bstar) | (bk == kToppWinBucket);  // lower buckets and the kept window are selected
      cmask |= static_cast<unsigned>(bk == bstar) << i;
    }
  }
  const unsigned nc = __popc(cmask);
  const unsigned incl = warp_incl_scan(nc);
  unsigned wbase = 0;
  if (lane == 31 && incl) wbase = atomicAdd(&rs.ncand, incl);
  wbase = __shfl_sync(kFull, wbase, 31);
  int32_t* cand = p.cand + r * p.c.cap + (wbase + incl - nc);
  while (cmask) {
    const int i = __ffs(cmask) - 1;
    cmask &= cmask - 1u;
    *cand++ = static_cast<int32_t>(tt0 + i);
  }
  lo = warp_sum(lo);
  if (lane == 0) s_c[warp] = lo;
  __syncthreads();
  constexpr int kSubsPerChunk = kToppChunk / kToppSub, kWarpsPerSub = kStreamWarps / kSubsPerChunk;
  if (threadIdx.x < kSubsPerChunk) {
    const int64_t sb = static_cast<int64_t>(blockIdx.x) * kSubsPerChunk + threadIdx.x;
    unsigned tot = 0;
    for (int w = 0; w < kWarpsPerSub; ++w) tot += s_c[kWarpsPerSub * threadIdx.x + w];
    if (sb < p.nsub) p.sub_cnt[r * p.nsub + sb] = tot;
  }
}

// ---------------------------------------------------------------- 5. exact resolution inside b*
// grid (rows), 1024 threads: radix select, 8 passes of 8 bits (most significant first), over the
// candidates' unique keys with per-bin mass histograms; K* = the smallest key whose cumulative
// mass (in key order) reaches rem.  Up to kResolveSmemCand candidates keep key and mass on chip.
__global__ void __launch_bounds__(kResolveThreads) topp_resolve_kernel(const ToppParams p) {
  pdl_wait();
  extern __shared__ unsigned long long s_kv[];  // [kResolveSmemCand] keys, then masses
  __shared__ uint32_t h_lo[256], h_hi[256];     // bin masses: wrapping low word + carries
  __shared__ unsigned long long s_prefix, s_rem;
  __shared__ unsigned s_wsum[kResolveThreads / 32];
  __shared__ unsigned s_carry;
  __shared__ unsigned long long s_diff[kResolveThreads / 32];
  const int64_t r = blockIdx.x;
  ToppRowState& rs = p.rows[r];
  const int bstar = rs.bstar;
  if (bstar == -1) {  // empty row
    if (threadIdx.x == 0) p.sel_cnt[r] = 0;
    return;
  }
  if (bstar >= 0) {  // block-uniform
  const int n = static_cast<int>(rs.ncand);
  const bool on_chip = n <= kResolveSmemCand;
  const bool topk = p.mode == KV1B_SELECT_TOPK;
  const float m = fkey_inv(rs.maxkey);
  const float* s = p.s + r * p.c.cap;
  const int32_t* cand = p.cand + r * p.c.cap;
  unsigned long long* skey = s_kv;
  unsigned long long* smass = s_kv + kResolveSmemCand;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (on_chip) {
    for (int i = threadIdx.x; i < n; i += kResolveThreads) {
      const int64_t t = cand[i];
      const float st = s[t];
      skey[i] = topp_key(st, t);
      smass[i] = topk ? 1ull : topp_mass_t(topp_t(st, m));
    }
  }
  if (on_chip && n <= kResolveSmallCand) {  // block-uniform: few candidates (concentrated attention)
    // thread i ranks candidate i: the mass of every candidate whose key is not larger (keys are
    // unique); K* = the smallest key whose cumulative mass reaches rem -- the same key the radix
    // passes below find
    __syncthreads();  // keys and masses are in shared memory
    const unsigned long long rem = rs.rem;
    unsigned long long best = ~0ull;
    if (threadIdx.x < n) {
      const unsigned long long ki = skey[threadIdx.x];
      unsigned long long cum = 0ull;
      for (int j = 0; j < n; ++j) cum += skey[j] <= ki ? smass[j] : 0ull;
      if (cum >= rem) best = ki;
    }
    #pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const unsigned long long x = __shfl_xor_sync(kFull, best, o);
      best = x < best ? x : best;
    }
    if (lane == 0) s_diff[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long b0 = ~0ull;
      for (int w = 0; w < kResolveThreads / 32; ++w) b0 = s_diff[w] < b0 ? s_diff[w] : b0;
      s_prefix = b0;
    }
    __syncthreads();
  } else {
  // leading key bytes shared by every candidate need no pass: start at the highest byte where any
  // candidate differs from the first (on-chip keys only; otherwise all 8 bytes)
  int d_top = 7;
  if (on_chip && n > 0) {
    __syncthreads();  // the keys are in shared memory
    unsigned long long x = 0ull;
    const unsigned long long k0 = skey[0];
    for (int i = threadIdx.x; i < n; i += kResolveThreads) x |= skey[i] ^ k0;
    #pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x |= __shfl_xor_sync(kFull, x, o);
    if (lane == 0) s_diff[warp] = x;
    __syncthreads();
    unsigned long long all = 0ull;
    for (int w = 0; w < kResolveThreads / 32; ++w) all |= s_diff[w];
    d_top = all ? (63 - __clzll(static_cast<long long>(all))) / 8 : 0;
  }
  if (threadIdx.x == 0) {
    s_prefix = d_top == 7 ? 0ull : (skey[0] >> (8 * (d_top + 1)));  // the bytes every candidate shares
    s_rem = rs.rem;
  }
  for (int d = d_top; d >= 0; --d) {
    if (threadIdx.x < 256) {
      h_lo[threadIdx.x] = 0u;
      h_hi[threadIdx.x] = 0u;
    }
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int i = threadIdx.x; i < n; i += kResolveThreads) {
      unsigned long long key, u;
      if (on_chip) {
        key = skey[i];
        u = smass[i];
      } else {
        const int64_t t = cand[i];
        const float st = s[t];
        key = topp_key(st, t);
        u = topk ? 1ull : topp_mass_t(topp_t(st, m));
      }
      if (u && (d == 7 || (key >> (8 * (d + 1))) == prefix)) {  // (every candidate matches above d_top)
        const int bin = static_cast<int>((key >> (8 * d)) & 255u);
        const uint32_t ulo = static_cast<uint32_t>(u);
        const uint32_t old = atomicAdd(&h_lo[bin], ulo);
        const uint32_t inc = static_cast<uint32_t>(u >> 32) + (old + ulo < old ? 1u : 0u);
        if (inc) atomicAdd(&h_hi[bin], inc);
      }
    }
    __syncthreads();
    if (warp == 0) {
      const unsigned long long rem = s_rem;
      unsigned long long loc = 0;
      unsigned long long hb[8];
      #pragma unroll
      for (int i = 0; i < 8; ++i) {
        hb[i] = (static_cast<unsigned long long>(h_hi[8 * lane + i]) << 32) | h_lo[8 * lane + i];
        loc += hb[i];
      }
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
          if (cum + hb[i] >= rem) {
            bin = 8 * lane + i;
            break;
          }
          cum += hb[i];
        }
        s_rem = rem - cum;
        s_prefix = (prefix << 8) | static_cast<unsigned long long>(bin);
      }
    }
    __syncthreads();
  }
  }  // radix passes
  const unsigned long long kstar = s_prefix;
  if (threadIdx.x == 0) rs.kstar = kstar;
  // selected candidates join their sub-chunks' counts (one atomic per sub-chunk and warp)
  uint32_t* cc = p.sub_cnt + r * p.nsub;
  for (int i0 = 0; i0 < n; i0 += kResolveThreads) {  // block-uniform trip count
    const int i = i0 + threadIdx.x;
    int ck = -1;
    if (i < n) {
      const int64_t t = cand[i];
      const unsigned long long key = on_chip ? skey[i] : topp_key(s[t], t);
      if (key <= kstar) ck = static_cast<int>(t / kToppSub);
    }
    const unsigned same = __match_any_sync(kFull, ck);
    if (ck >= 0 && lane == __ffs(same) - 1) atomicAdd(&cc[ck], static_cast<unsigned>(__popc(same)));
  }
  }
  // exclusive prefix of the row's sub-chunk counts -> sub_off[r][0 .. nsub]; sel_cnt = the total
  const int warp_s = threadIdx.x >> 5, lane_s = threadIdx.x & 31;
  const uint32_t* ccs = p.sub_cnt + r * p.nsub;
  uint32_t* off = p.sub_off + r * (p.nsub + 1);
  if (threadIdx.x == 0) s_carry = 0u;
  __syncthreads();  // the candidate counts are in place
  for (int k0 = 0; k0 < p.nsub; k0 += kResolveThreads) {  // block-uniform
    const int k = k0 + threadIdx.x;
    const unsigned c = k < p.nsub ? ccs[k] : 0u;
    const unsigned incl = warp_incl_scan(c);
    if (lane_s == 31) s_wsum[warp_s] = incl;
    __syncthreads();
    unsigned before = s_carry;
    for (int w = 0; w < warp_s; ++w) before += s_wsum[w];
    if (k < p.nsub) off[k] = before + incl - c;
    __syncthreads();
    if (threadIdx.x == kResolveThreads - 1) s_carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    off[p.nsub] = s_carry;
    p.sel_cnt[r] = static_cast<int32_t>(s_carry);
  }
}

// ---------------------------------------------------------------- 6. ordered writes + gather-attend
// grid (sub-chunks of kToppSub tokens, B * Hkv): one block serves the G query heads of a kv-head, so
// each code tile is read once for all of them.  Thread = 4 contiguous tokens, warp = one 128-token
// code tile.  Per head: selection mask, block scan, ordered index writes, softmax weights of the
// selected tokens into shared memory.  Then each warp gathers its tile in slices of 32 tokens (lanes
// 8k .. 8k + 7): for each slice where any head selects a token, lane l loads the slice's 4-bit codes
// of channels 4l..4l+3 (one 16-byte group per channel), the next such slice's loads in flight
// meanwhile, and accumulates, per head, e * (scale * code + min) over that head's selected tokens.
// Each head's (numerator, denominator) against its row maximum goes to part[row][sub-chunk].
template <int GM>
__global__ void __launch_bounds__(kStreamThreads, GM <= 4 ? 3 : 2) topp_write_gather_kernel(const ToppParams p, int G) {
  pdl_wait();
  constexpr int kW = kStreamWarps;
  constexpr int kTok = kToppSub / kStreamThreads;  // contiguous tokens per thread
  constexpr int kPk = (GM + 1) / 2;                // per-thread counts, two heads per 32-bit word
  static_assert(kTok == 4 && kTok * 32 == 128, "a warp covers one 128-token code tile");
  static_assert(kW * kD == kToppSub, "the weight buffer doubles as the cross-warp reduction buffer");
  __shared__ float s_e[GM][kToppSub];               // weights of the selected tokens, then partial sums
  __shared__ unsigned s_cnt[kW][kPk];
  __shared__ __align__(16) float s_scl[kW][32][4];  // per slice token: group scales and minima as fp32
  __shared__ __align__(16) float s_mnv[kW][32][4];
  __shared__ float s_l[kW][GM];
  const CacheView& c = p.c;
  const int z = blockIdx.y;  // b * Hkv + kvh
  const int64_t row0 = static_cast<int64_t>(z) * G;
  const int sub = blockIdx.x;
  const int L = p.len[z / c.Hkv];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(sub) * kToppSub;
  if (t0 >= L) return;  // block-uniform
  const int64_t t1 = t0 + kToppSub < L ? t0 + kToppSub : L;
  const int64_t tt0 = t0 + kTok * threadIdx.x;
  // this sub-chunk's first output slot and selected count per head (prefix sums by the resolve)
  unsigned base[GM], total = 0;
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    base[h] = 0u;
    if (h < G) {
      const uint32_t* off = p.sub_off + (row0 + h) * (p.nsub + 1) + sub;
      base[h] = off[0];
      total += off[1] - off[0];
    }
  }
  if (total == 0u) return;  // block-uniform: nothing selected here for any of the G heads
  unsigned mask[GM];
  uint2 bk4[GM];    // this thread's 4 buckets per head (16 bits each)
  float v[GM][4];   // their logits, loaded where the bucket is at most b*
  float mrow[GM];
  const int nv = static_cast<int>(t1 - tt0);
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    mask[h] = 0u;
    bk4[h] = make_uint2(0xffffffffu, 0xffffffffu);
    mrow[h] = 0.0f;
    if (h < G && nv > 0) bk4[h] = *reinterpret_cast<const uint2*>(p.bk + (row0 + h) * c.cap + tt0);  // inside the row
  }
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h < G && nv > 0) {
      const ToppRowState& rs = p.rows[row0 + h];
      const int bstar = rs.bstar;  // >= 0, or -2 (window only): the row is not empty
      const unsigned long long kstar = rs.kstar;
      mrow[h] = fkey_inv(rs.maxkey);
      const float* srow = p.s + (row0 + h) * c.cap + tt0;
      #pragma unroll
      for (int i = 0; i < kTok; ++i) {
        const int bk = static_cast<int>(((i < 2 ? bk4[h].x : bk4[h].y) >> (16 * (i & 1))) & 0xffffu);
        v[h][i] = 0.0f;
        const bool win = bk == kToppWinBucket;
        if (i < nv && (win || bk <= bstar)) {
          v[h][i] = srow[i];
          const bool f = win || bk < bstar || topp_key(v[h][i], tt0 + i) <= kstar;
          mask[h] |= static_cast<unsigned>(f) << i;
        }
      }
    }
  }
  // one block scan for all heads (counts <= kToppSub fit 16 bits)
  unsigned pk[kPk], incl[kPk];
  #pragma unroll
  for (int w = 0; w < kPk; ++w) pk[w] = 0u;
  #pragma unroll
  for (int h = 0; h < GM; ++h) pk[h >> 1] |= static_cast<unsigned>(__popc(mask[h])) << (16 * (h & 1));
  #pragma unroll
  for (int w = 0; w < kPk; ++w) {
    incl[w] = warp_incl_scan(pk[w]);
    if (lane == 31) s_cnt[warp][w] = incl[w];
  }
  __syncthreads();
  float lsum[GM];
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    lsum[h] = 0.0f;
    if (h < G) {
      const int sh = 16 * (h & 1);
      // lane w < kW holds warp w's count: this warp's prior count within the block
      const unsigned cw = lane < kW ? (s_cnt[lane][h >> 1] >> sh) & 0xffffu : 0u;
      const unsigned prior = __reduce_add_sync(kFull, lane < warp ? cw : 0u);
      const unsigned cnt = __popc(mask[h]);
      unsigned off = base[h] + prior + ((incl[h >> 1] >> sh) & 0xffffu) - cnt;
      int32_t* sel = p.sel_idx + (row0 + h) * c.cap;
      #pragma unroll
      for (int i = 0; i < kTok; ++i) {
        if ((mask[h] >> i) & 1u) {
          sel[off++] = static_cast<int32_t>(tt0 + i);
          const float e = exp2f(__fmul_rn(__fsub_rn(v[h][i], mrow[h]), kL2e));
          s_e[h][kTok * threadIdx.x + i] = e;
          lsum[h] += e;
        }
      }
    }
  }
  __syncwarp();
  // gather over the warp's slices where any head selects a token
  const int64_t head_tok = static_cast<int64_t>(z) * c.cap;
  const uint32_t* vcw = c.v_codes + head_tok * 16;
  const uint4* vsm4 = reinterpret_cast<const uint4*>(c.v_sm) + head_tok;
  const int grp = lane >> 3;  // 32-channel group of this lane's channels
  unsigned pair[GM];          // 32-token slice masks per head, on every lane of the slice's 8 lanes
  unsigned any = 0u;
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    unsigned x = mask[h] << (kTok * (lane & 7));
    x |= __shfl_xor_sync(kFull, x, 1);
    x |= __shfl_xor_sync(kFull, x, 2);
    x |= __shfl_xor_sync(kFull, x, 4);
    pair[h] = x;
    any |= x;
  }
  unsigned active = __ballot_sync(kFull, (lane & 7) == 0 && any != 0u);
  const int64_t wt0 = t0 + 32 * kTok * warp;
  float acc[GM][4], accm[GM];
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    accm[h] = 0.0f;
    #pragma unroll
    for (int q = 0; q < 4; ++q) acc[h][q] = 0.0f;
  }
  uint4 cw_n[4], sm_n = make_uint4(0u, 0u, 0u, 0u);
  int src = active ? __ffs(active) - 1 : -1;
  auto load_slice = [&](int sl) {
    const int64_t ts = wt0 + kTok * sl;  // slice start: a multiple of 32 inside the warp's tile
    const unsigned ball_any = __shfl_sync(kFull, any, sl);
    const uint32_t* cp = vcw + ((ts >> 7) * kD + 4 * lane) * 16 + ((ts & 127) >> 3);
    #pragma unroll
    for (int q = 0; q < 4; ++q) cw_n[q] = __ldg(reinterpret_cast<const uint4*>(cp + 16 * q));
    sm_n = ((ball_any >> lane) & 1u) ? __ldg(vsm4 + ts + lane) : make_uint4(0u, 0u, 0u, 0u);
  };
  if (src >= 0) load_slice(src);
  while (src >= 0) {  // warp-uniform
    const int cur = src;
    uint4 cw[4];
    #pragma unroll
    for (int q = 0; q < 4; ++q) cw[q] = cw_n[q];
    {
      float4 sc, mn;
      sc.x = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.x & 0xffffu)));
      sc.y = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.y & 0xffffu)));
      sc.z = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.z & 0xffffu)));
      sc.w = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.w & 0xffffu)));
      mn.x = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.x >> 16)));
      mn.y = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.y >> 16)));
      mn.z = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.z >> 16)));
      mn.w = __half2float(__ushort_as_half(static_cast<unsigned short>(sm_n.w >> 16)));
      *reinterpret_cast<float4*>(&s_scl[warp][lane][0]) = sc;
      *reinterpret_cast<float4*>(&s_mnv[warp][lane][0]) = mn;
    }
    active &= active - 1u;
    src = active ? __ffs(active) - 1 : -1;
    if (src >= 0) load_slice(src);  // next slice in flight
    __syncwarp();
    #pragma unroll
    for (int h = 0; h < GM; ++h) {
      if (h < G) {
        const unsigned ball = __shfl_sync(kFull, pair[h], cur);
        const float* ew = &s_e[h][32 * kTok * warp + kTok * cur];
        #pragma unroll
        for (int w = 0; w < 4; ++w) {
          unsigned bits = (ball >> (8 * w)) & 0xffu;
          while (bits) {
            const int jj = __ffs(bits) - 1;
            bits &= bits - 1u;
            const int j = 8 * w + jj;
            const float ej = ew[j];
            const float es = __fmul_rn(ej, s_scl[warp][j][grp]);
            accm[h] = __fmaf_rn(ej, s_mnv[warp][j][grp], accm[h]);
            #pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t word = w == 0 ? cw[q].x : (w == 1 ? cw[q].y : (w == 2 ? cw[q].z : cw[q].w));
              // 2^23 + code as a float (exact), minus 2^23: the code as fp32 without an int conversion
              const float code = __fsub_rn(__uint_as_float(((word >> (4 * jj)) & 0xFu) | 0x4B000000u), 8388608.0f);
              acc[h][q] = __fmaf_rn(es, code, acc[h][q]);
            }
          }
        }
      }
    }
    __syncwarp();  // s_scl / s_mnv are rewritten for the next slice
  }
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    const float l = warp_sum(lsum[h]);
    if (lane == 0) s_l[warp][h] = l;
  }
  __syncthreads();  // every warp is done with the weights: s_e becomes [head][warp][channel] sums
  #pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h < G) {
      #pragma unroll
      for (int q = 0; q < 4; ++q) s_e[h][kD * warp + 4 * lane + q] = acc[h][q] + accm[h];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * kD; i += kStreamThreads) {
    const int h = i / kD, ch = i % kD;
    float* row = p.part + ((row0 + h) * p.nsub + sub) * kPartStride;
    float num = 0.0f;
    for (int w = 0; w < kW; ++w) num += s_e[h][kD * w + ch];
    row[2 + ch] = num;
    if (ch == 0) {
      float den = 0.0f;
      for (int w = 0; w < kW; ++w) den += s_l[w][h];
      row[0] = 0.0f;  // every sub-chunk of the row uses the same reference maximum
      row[1] = den;
    }
  }
}

// ---------------------------------------------------------------- 7. merge
// grid (M <= kToppMergeSplit, rows), 128 threads: block j sums the row's sub-chunk partials
// [j n / M, (j + 1) n / M) in order into part2[row][j]; the row's last block to finish (atomic ticket
// after a fence) sums the M first-level sums in order and writes out = numerator / denominator.
// Rows with nothing selected give zeros.
__global__ void __launch_bounds__(kD) topp_merge_kernel(const ToppParams p) {
  pdl_wait();
  const int M = gridDim.x;
  __shared__ bool s_last;
  const int64_t r = blockIdx.y;
  const int j = blockIdx.x;
  const int ch = threadIdx.x;
  const int L = row_len(p, r);
  const int n = p.rows[r].bstar != -1 ? (L + kToppSub - 1) / kToppSub : 0;
  const int k0 = static_cast<int>(static_cast<int64_t>(n) * j / M);
  const int k1 = static_cast<int>(static_cast<int64_t>(n) * (j + 1) / M);
  const float* base = p.part + r * p.nsub * kPartStride;
  const uint32_t* off = p.sub_off + r * (p.nsub + 1);
  float num = 0.0f, den = 0.0f;
  #pragma unroll 4
  for (int k = k0; k < k1; ++k) {
    // a sub-chunk without a selected token of the row wrote no partial: its (allocated, unwritten)
    // entries are read but not used, so the loads of consecutive sub-chunks stay independent
    const bool has = off[k + 1] != off[k];
    const float x = base[k * kPartStride + 2 + ch], y = base[k * kPartStride + 1];
    num = has ? num + x : num;
    den = has ? den + y : den;
  }
  float* q2 = p.part2 + (r * M + j) * kPartStride;
  q2[2 + ch] = num;
  if (ch == 0) q2[1] = den;
  __threadfence();
  __syncthreads();
  if (ch == 0) s_last = atomicAdd(&p.rows[r].merged, 1u) == M - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* b2 = p.part2 + r * M * kPartStride;
  num = 0.0f;
  den = 0.0f;
  for (int k = 0; k < M; ++k) {
    num += __ldcg(b2 + k * kPartStride + 2 + ch);
    den += __ldcg(b2 + k * kPartStride + 1);
  }
  p.out[r * kD + ch] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
}

}  // namespace kv1b

using namespace kv1b;

namespace {
size_t al256(size_t x) { return (x + 255) / 256 * 256; }

struct ToppLayout {
  size_t planes, qvl, qdl, qsq, s, bk, cand, rows, hist, sub_cnt, sub_off, part, part2, total, state_bytes;
};
ToppLayout topp_layout(int32_t rows, int32_t cap) {
  const size_t R = static_cast<size_t>(rows), C = static_cast<size_t>(cap);
  const size_t nsub = (C + kToppSub - 1) / kToppSub;
  ToppLayout l;
  size_t o = 0;
  l.planes = o;    o += al256(R * 16 * 4);
  l.qvl = o;       o += al256(R * 4);
  l.qdl = o;       o += al256(R * 4);
  l.qsq = o;       o += al256(R * 4);
  l.s = o;         o += al256(R * C * 4);
  l.bk = o;        o += al256(R * C * 2);
  l.cand = o;      o += al256(R * C * 4);
  l.rows = o;      o += al256(R * sizeof(ToppRowState));  // rows, hist and sub_cnt: one memset
  l.hist = o;      o += al256(R * kToppBuckets * 8);
  l.sub_cnt = o;   o += al256(R * nsub * 4);
  l.state_bytes = o - l.rows;
  l.sub_off = o;   o += al256(R * (nsub + 1) * 4);
  l.part = o;      o += al256(R * nsub * kPartStride * 4);
  l.part2 = o;     o += al256(R * kToppMergeSplit * kPartStride * 4);
  l.total = o;
  return l;
}
}  // namespace

// Workspace of kv1b_attend_topp (rows = batch x query heads, capacity tokens each).
size_t kv1b_topp_workspace_bytes(int32_t rows, int32_t cap) { return topp_layout(rows, cap).total; }

void kv1b_topp_carve(ToppParams* p, void* ws, int32_t rows, int32_t cap) {
  const ToppLayout l = topp_layout(rows, cap);
  char* w = static_cast<char*>(ws);
  p->planes = reinterpret_cast<uint32_t*>(w + l.planes);
  p->qvl = reinterpret_cast<float*>(w + l.qvl);
  p->qdl = reinterpret_cast<float*>(w + l.qdl);
  p->qsq = reinterpret_cast<int32_t*>(w + l.qsq);
  p->s = reinterpret_cast<float*>(w + l.s);
  p->bk = reinterpret_cast<uint16_t*>(w + l.bk);
  p->cand = reinterpret_cast<int32_t*>(w + l.cand);
  p->rows = reinterpret_cast<ToppRowState*>(w + l.rows);
  p->hist = reinterpret_cast<unsigned long long*>(w + l.hist);
  p->sub_cnt = reinterpret_cast<uint32_t*>(w + l.sub_cnt);
  p->sub_off = reinterpret_cast<uint32_t*>(w + l.sub_off);
  p->part = reinterpret_cast<float*>(w + l.part);
  p->part2 = reinterpret_cast<float*>(w + l.part2);
  p->nchunk = static_cast<int32_t>((static_cast<size_t>(cap) + kToppChunk - 1) / kToppChunk);
  p->nsub = static_cast<int32_t>((static_cast<size_t>(cap) + kToppSub - 1) / kToppSub);
}

cudaError_t kv1b_launch_topp(const ToppParams& p, int32_t G, int32_t max_len, cudaStream_t stream) {
  const int R = p.c.B * p.Hq;
  if (R > 65535 || G > 8) return cudaErrorInvalidValue;  // grid y of the row kernels; two groups of 4 heads
  static std::atomic<unsigned long long> configured{0};  // bit per device
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(topp_resolve_kernel), static_cast<int>(kResolveSmem),
                                 &configured);
  if (e != cudaSuccess) return e;
  const ToppLayout l = topp_layout(R, p.c.cap);
  e = cudaMemsetAsync(p.rows, 0, l.state_bytes, stream);
  if (e != cudaSuccess) return e;
  const dim3 sg(static_cast<unsigned>(p.nchunk), static_cast<unsigned>(R));
  const dim3 bs(kStreamThreads);
  // the first kernel after the memset is a plain launch; the rest overlap their predecessor's tail
  if (max_len > 0) {
    e = kv1b_launch_query_prep(p.c, p.q, p.q_dtype, p.Hq, p.planes, p.qvl, p.qdl, p.qsq, stream);
    if (e != cudaSuccess) return e;
    const dim3 grid((max_len + kScoreTok - 1) / kScoreTok, p.c.Hkv, p.c.B);
    e = G <= 4 ? launch_pdl(topp_scores_kernel<1, false>, grid, bs, 0, stream, p, G)
               : launch_pdl(topp_scores_kernel<2, false>, grid, bs, 0, stream, p, G);
    if (e == cudaSuccess)
      e = p.mode == KV1B_SELECT_TOPK ? launch_pdl(topp_mass_kernel<KV1B_SELECT_TOPK>, sg, bs, 0, stream, p)
                                     : launch_pdl(topp_mass_kernel<KV1B_SELECT_TOPP>, sg, bs, 0, stream, p);
    if (e == cudaSuccess) e = launch_pdl(topp_threshold_kernel, dim3(R), dim3(kThresholdThreads), 0, stream, p);
    if (e == cudaSuccess) e = launch_pdl(topp_cand_kernel, sg, bs, 0, stream, p);
  } else {
    topp_threshold_kernel<<<R, kThresholdThreads, 0, stream>>>(p);  // marks every row empty
    e = cudaGetLastError();
  }
  // select inside the threshold bucket, then every row's sub-chunk offsets and selected count
  if (e == cudaSuccess) e = launch_pdl(topp_resolve_kernel, dim3(R), dim3(kResolveThreads), kResolveSmem, stream, p);
  if (e != cudaSuccess) return e;
  const dim3 gg(static_cast<unsigned>(p.nsub), static_cast<unsigned>(p.c.B * p.c.Hkv));
  e = G <= 4 ? launch_pdl(topp_write_gather_kernel<4>, gg, bs, 0, stream, p, G)
             : launch_pdl(topp_write_gather_kernel<8>, gg, bs, 0, stream, p, G);
  // first-level merge blocks per row: one per 16 sub-chunk partials, at most kToppMergeSplit
  const int nsub_used = (max_len + kToppSub - 1) / kToppSub;
  int msplit = (nsub_used + 15) / 16;
  msplit = msplit < 1 ? 1 : (msplit > kToppMergeSplit ? kToppMergeSplit : msplit);
  if (e == cudaSuccess) e = launch_pdl(topp_merge_kernel, dim3(msplit, R), dim3(kD), 0, stream, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t kv1b_launch_topp_scores_probe(const ToppParams& p, int32_t G, int32_t max_len, cudaStream_t stream) {
  if (G > 8 || !p.probe_A || !p.probe_Bc) return cudaErrorInvalidValue;
  if (max_len <= 0) return cudaSuccess;
  const ToppLayout l = topp_layout(p.c.B * p.Hq, p.c.cap);
  cudaError_t e = cudaMemsetAsync(p.rows, 0, l.state_bytes, stream);
  if (e == cudaSuccess) e = kv1b_launch_query_prep(p.c, p.q, p.q_dtype, p.Hq, p.planes, p.qvl, p.qdl, p.qsq, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid((max_len + kScoreTok - 1) / kScoreTok, p.c.Hkv, p.c.B);
  e = G <= 4 ? launch_pdl(topp_scores_kernel<1, true>, grid, dim3(kStreamThreads), 0, stream, p, G)
             : launch_pdl(topp_scores_kernel<2, true>, grid, dim3(kStreamThreads), 0, stream, p, G);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
