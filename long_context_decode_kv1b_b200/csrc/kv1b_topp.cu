// kv1b_topp.cu -- adaptive Top-p attention ("RaBitQCache", abstract / core idea: adaptive Top-p
// retrieval whose token budget follows the actual attention sparsity), as a pipeline of
// grid-wide kernels so that a long context is spread over every SM.  Per row r = (sequence,
// query head), with the reproducible integer masses u_t ~ 2^32 2^((s_t - m) log2 e) (degree-7
// polynomial of 2^f, bit for bit the same as the CPU reference) and T = ceil(p U) in fp64:
//  1. scores: binary x INT4 popcount logits of every token for the G heads of a kv-head (bit-exact
//     arithmetic), written to the workspace; the row maximum m by atomicMax on an order-preserving
//     key;
//  2. masses: u_t, the row total U, and a histogram of masses over 640 buckets of
//     t = (s - m) log2 e (bucket floor(-16 t), monotone in s; t < -40 has no mass);
//  3. threshold: the first bucket b* where the cumulative mass reaches T; rem = the mass still
//     needed inside b*;
//  4. candidates: the tokens of bucket b* (any order);
//  5. resolve: a block-wide radix select over the candidates' unique 64-bit keys
//     (order-preserving descending code of s) << 32 | t finds the smallest key K* whose cumulative
//     candidate mass reaches rem;
//  6. the selected set {t : bucket(t) < b*} U {t in b* : key_t <= K*} -- the shortest prefix of the
//     order (s desc, index asc) whose mass reaches T -- is compacted in ascending index order
//     (chunk counts, then ordered writes);
//  7. gather-attend, fused with the compaction: the softmax over the selected tokens' logits with
//     the 4-bit values dequantised on the fly, fp32 partials per chunk, summed in chunk order.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

constexpr float kL2e = 0x1.715476p+0f;  // log2(e) rounded to fp32
constexpr int kStreamThreads = 256;

// (ln 2)^k / k!, k = 0..7, each rounded to the nearest fp32 (Taylor coefficients of 2^f).
__constant__ float kExp2Coef[8] = {0x1p+0f,         0x1.62e43p-1f,   0x1.ebfbep-3f,   0x1.c6b08ep-5f,
                                   0x1.3b2ab6p-7f,  0x1.5d87fep-10f, 0x1.430912p-13f, 0x1.ffcbfcp-17f};

__device__ __forceinline__ float topp_t(float s, float m) { return __fmul_rn(__fsub_rn(s, m), kL2e); }

__device__ __forceinline__ uint64_t topp_mass_t(float t) {
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

// Bucket of t = (s - m) log2 e: floor(-16 t) for t in [-40, 0] (639 at most), 640 below.
__device__ __forceinline__ int topp_bucket(float t) {
  if (!(t >= -40.0f)) return 640;
  const int b = static_cast<int>(__fmul_rn(-t, 16.0f));
  return b < 639 ? b : 639;
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

__device__ __forceinline__ int row_len(const ToppParams& p, int64_t r) { return p.len[r / p.Hq]; }

// ---------------------------------------------------------------- 1. logits and row maxima
// grid (token blocks of 256, kv-heads, sequences); thread = token, loops over the G heads.
__global__ void __launch_bounds__(kStreamThreads) topp_scores_kernel(const ToppParams p, int G) {
  __shared__ __align__(16) uint32_t s_planes[KV1B_MAX_GROUP][4][4];
  __shared__ float s_vl[KV1B_MAX_GROUP], s_dl[KV1B_MAX_GROUP];
  __shared__ int s_sq[KV1B_MAX_GROUP];
  __shared__ float s_max[kStreamThreads / 32][KV1B_MAX_GROUP];
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
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kStreamThreads + threadIdx.x;
  const bool valid = t < p.len[b];
  const int64_t head_tok = (static_cast<int64_t>(b) * c.Hkv + kvh) * c.cap;
  uint4 kb = make_uint4(0u, 0u, 0u, 0u);
  float nc = 0.0f;
  if (valid) {
    kb = __ldg(reinterpret_cast<const uint4*>(c.k_bits) + head_tok + t);
    nc = __fmul_rn(__ldg(c.k_norm + head_tok + t), __ldg(c.k_cinv + head_tok + t));
  }
  const int32_t Bc = popc_Bc(kb);
  const float qs = __fdiv_rn(p.scale, static_cast<float>(kD));
  for (int h = 0; h < G; ++h) {
    uint32_t P[4][4];
    for (int j = 0; j < 4; ++j)
      for (int w = 0; w < 4; ++w) P[j][w] = s_planes[h][j][w];
    float sv = -INFINITY;
    if (valid) {
      const int32_t A = popc_A(kb, P);
      sv = logit_from_ints(A, Bc, s_sq[h], s_vl[h], s_dl[h], nc, qs);
      p.s[(static_cast<int64_t>(b) * p.Hq + kvh * G + h) * c.cap + t] = sv;
    }
    #pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sv = fmaxf(sv, __shfl_xor_sync(kFull, sv, o));
    if (lane == 0) s_max[warp][h] = sv;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float mx = s_max[0][threadIdx.x];
    for (int w = 1; w < kStreamThreads / 32; ++w) mx = fmaxf(mx, s_max[w][threadIdx.x]);
    if (mx != -INFINITY) atomicMax(&p.rows[static_cast<int64_t>(b) * p.Hq + kvh * G + threadIdx.x].maxkey, fkey(mx));
  }
}

// ---------------------------------------------------------------- 2. masses and bucket histogram
// grid (chunks of kToppChunk tokens, rows)
__global__ void __launch_bounds__(kStreamThreads) topp_mass_kernel(const ToppParams p) {
  __shared__ unsigned long long sh[kToppBuckets];
  __shared__ unsigned long long s_u[kStreamThreads / 32];
  const int64_t r = blockIdx.y;
  const int L = row_len(p, r);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kToppChunk;
  if (t0 >= L) return;
  const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
  for (int i = threadIdx.x; i < kToppBuckets; i += kStreamThreads) sh[i] = 0ull;
  __syncthreads();
  const float m = fkey_inv(p.rows[r].maxkey);
  const float* s = p.s + r * p.c.cap;
  unsigned long long usum = 0ull;
  for (int64_t t = t0 + threadIdx.x; t < t1; t += kStreamThreads) {
    const float tt = topp_t(s[t], m);
    const uint64_t u = topp_mass_t(tt);
    if (u) {
      atomicAdd(&sh[topp_bucket(tt)], static_cast<unsigned long long>(u));
      usum += u;
    }
  }
  usum = warp_sum(usum);
  if ((threadIdx.x & 31) == 0) s_u[threadIdx.x >> 5] = usum;
  __syncthreads();
  unsigned long long* hist = p.hist + r * kToppBuckets;
  for (int i = threadIdx.x; i < 640; i += kStreamThreads)
    if (sh[i]) atomicAdd(&hist[i], sh[i]);
  if (threadIdx.x == 0) {
    unsigned long long tot = 0ull;
    for (int w = 0; w < kStreamThreads / 32; ++w) tot += s_u[w];
    atomicAdd(&p.rows[r].U, tot);
  }
}

// ---------------------------------------------------------------- 3. threshold bucket
// grid (rows), 1024 threads: thread i owns bucket i.
__global__ void __launch_bounds__(kToppBuckets) topp_threshold_kernel(const ToppParams p) {
  __shared__ unsigned long long s_w[kToppBuckets / 32];
  __shared__ int s_first;
  const int64_t r = blockIdx.x;
  ToppRowState& rs = p.rows[r];
  const unsigned long long U = rs.U;
  if (U == 0ull || row_len(p, r) == 0) {  // empty row
    if (threadIdx.x == 0) rs.bstar = -1;
    return;
  }
  unsigned long long T = static_cast<unsigned long long>(ceil(static_cast<double>(p.p) * static_cast<double>(U)));
  if (T > U) T = U;
  if (T < 1) T = 1;
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const unsigned long long h = p.hist[r * kToppBuckets + i];
  unsigned long long incl = h;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_w[warp] = incl;
  if (i == 0) s_first = kToppBuckets;
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
  if (incl >= T && incl - h < T) atomicMin(&s_first, i);  // exactly one bucket crosses T
  __syncthreads();
  if (i == s_first) {
    rs.bstar = i;
    rs.rem = T - (incl - h);
  }
}

// ---------------------------------------------------------------- 4. candidates of bucket b*
__global__ void __launch_bounds__(kStreamThreads) topp_cand_kernel(const ToppParams p) {
  const int64_t r = blockIdx.y;
  const int L = row_len(p, r);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kToppChunk;
  const int bstar = p.rows[r].bstar;
  if (t0 >= L || bstar < 0) return;
  const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
  const float m = fkey_inv(p.rows[r].maxkey);
  const float* s = p.s + r * p.c.cap;
  int32_t* cand = p.cand + r * p.c.cap;
  const int lane = threadIdx.x & 31;
  for (int64_t tb = t0; tb < t1; tb += kStreamThreads) {
    const int64_t t = tb + threadIdx.x;
    const bool f = t < t1 && topp_bucket(topp_t(s[t], m)) == bstar;
    const unsigned ball = __ballot_sync(kFull, f);
    if (ball) {
      unsigned base = 0;
      if (lane == 0) base = atomicAdd(&p.rows[r].ncand, static_cast<unsigned>(__popc(ball)));
      base = __shfl_sync(kFull, base, 0);
      if (f) cand[base + __popc(ball & ((1u << lane) - 1u))] = static_cast<int32_t>(t);
    }
  }
}

// ---------------------------------------------------------------- 5. exact resolution inside b*
// grid (rows), 1024 threads: radix select, 8 passes of 8 bits (most significant first), over the
// candidates' unique keys with per-bin mass histograms; K* = the smallest key whose cumulative
// mass (in key order) reaches rem.
constexpr int kResolveThreads = 1024;
__global__ void __launch_bounds__(kResolveThreads) topp_resolve_kernel(const ToppParams p) {
  __shared__ unsigned long long hist[256];
  __shared__ unsigned long long s_prefix, s_rem;
  const int64_t r = blockIdx.x;
  ToppRowState& rs = p.rows[r];
  if (rs.bstar < 0) return;
  const int n = static_cast<int>(rs.ncand);
  const float m = fkey_inv(rs.maxkey);
  const float* s = p.s + r * p.c.cap;
  const int32_t* cand = p.cand + r * p.c.cap;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_rem = rs.rem;
  }
  for (int d = 7; d >= 0; --d) {
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int i = threadIdx.x; i < n; i += kResolveThreads) {
      const int64_t t = cand[i];
      const float st = s[t];
      const uint64_t key = topp_key(st, t);
      if (d == 7 || (key >> (8 * (d + 1))) == prefix) {
        const uint64_t u = topp_mass_t(topp_t(st, m));
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
  if (threadIdx.x == 0) rs.kstar = s_prefix;
}

// ---------------------------------------------------------------- 6. ascending compaction
__device__ __forceinline__ bool topp_selected(const ToppRowState& rs, const float* s, float m, int64_t t) {
  const float st = s[t];
  const int bk = topp_bucket(topp_t(st, m));
  return bk < rs.bstar || (bk == rs.bstar && topp_key(st, t) <= rs.kstar);
}

__global__ void __launch_bounds__(kStreamThreads) topp_count_kernel(const ToppParams p) {
  __shared__ unsigned s_c[kStreamThreads / 32];
  const int64_t r = blockIdx.y;
  const int L = row_len(p, r);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kToppChunk;
  const ToppRowState& rs = p.rows[r];
  unsigned cnt = 0;
  if (t0 < L && rs.bstar >= 0) {
    const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
    const float m = fkey_inv(rs.maxkey);
    const float* s = p.s + r * p.c.cap;
    for (int64_t t = t0 + threadIdx.x; t < t1; t += kStreamThreads) cnt += topp_selected(rs, s, m, t);
  }
  cnt = warp_sum(cnt);
  if ((threadIdx.x & 31) == 0) s_c[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned tot = 0;
    for (int w = 0; w < kStreamThreads / 32; ++w) tot += s_c[w];
    p.chunk_cnt[r * p.nchunk + blockIdx.x] = tot;
  }
}

// 6b + 7. ordered writes of the selected indices, fused with the gather-attend of the chunk's selected
// tokens.  grid (G, chunks, B * Hkv): the G query heads of a kv-head and chunk are adjacent in launch
// order, so their value reads share L2.  Warp w owns the 32-token slice tb + 32 w; when any token of
// the slice is selected, lane l loads the slice's 4-bit codes of channels 4l..4l+3 (one 16-byte word
// group per channel) and accumulates e (scale code + min) for every selected token.  The chunk's
// partial (numerator, denominator) against the row maximum goes to part[row][chunk]; the merge sums
// the chunks in order.
__global__ void __launch_bounds__(kStreamThreads) topp_write_gather_kernel(const ToppParams p, int G) {
  constexpr int kW = kStreamThreads / 32;
  __shared__ unsigned s_c[kW];
  __shared__ unsigned s_base;
  __shared__ float s_e[kW][32];
  __shared__ __align__(16) uint32_t s_smw[kW][32][4];  // written as uint4
  __shared__ float s_acc[kW][kD];
  __shared__ float s_l[kW];
  const CacheView& c = p.c;
  const int z = blockIdx.z;  // b * Hkv + kvh
  const int64_t r = static_cast<int64_t>(z) * G + blockIdx.x;
  const int chunk = blockIdx.y;
  const int L = p.len[z / c.Hkv];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ToppRowState& rs = p.rows[r];
  const uint32_t* cc = p.chunk_cnt + r * p.nchunk;
  // offset of this chunk = selected tokens of the chunks before it
  unsigned before = 0;
  for (int k = threadIdx.x; k < chunk; k += kStreamThreads) before += cc[k];
  before = warp_sum(before);
  if (lane == 0) s_c[warp] = before;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned tot = 0;
    for (int w = 0; w < kW; ++w) tot += s_c[w];
    s_base = tot;
    if (chunk == p.nchunk - 1) p.sel_cnt[r] = static_cast<int32_t>(tot + cc[chunk]);
  }
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(chunk) * kToppChunk;
  if (t0 >= L || rs.bstar < 0) return;
  const int64_t t1 = t0 + kToppChunk < L ? t0 + kToppChunk : L;
  const float m = fkey_inv(rs.maxkey);
  const float* s = p.s + r * c.cap;
  int32_t* sel = p.sel_idx + r * c.cap;
  const int64_t head_tok = static_cast<int64_t>(z) * c.cap;
  const uint32_t* vcw = c.v_codes + head_tok * 16;
  const uint4* vsm4 = reinterpret_cast<const uint4*>(c.v_sm) + head_tok;
  const int grp = lane >> 3;  // 32-channel group of this lane's channels
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float accm = 0.0f, lsum = 0.0f;
  unsigned base = s_base;
  for (int64_t tb = t0; tb < t1; tb += kStreamThreads) {
    const int64_t t = tb + threadIdx.x;
    const bool f = t < t1 && topp_selected(rs, s, m, t);
    const unsigned ball = __ballot_sync(kFull, f);
    __syncthreads();  // the previous round's counts are read
    if (lane == 0) s_c[warp] = __popc(ball);
    __syncthreads();
    unsigned off = 0, tot = 0;
    for (int w = 0; w < kW; ++w) {
      off += (w < warp) ? s_c[w] : 0u;
      tot += s_c[w];
    }
    if (f) sel[base + off + __popc(ball & ((1u << lane) - 1u))] = static_cast<int32_t>(t);
    base += tot;
    if (ball) {  // warp-uniform: gather this slice's selected tokens
      float e = 0.0f;
      uint4 smv = make_uint4(0u, 0u, 0u, 0u);
      if (f) {
        e = exp2f(__fmul_rn(__fsub_rn(s[t], m), kL2e));
        smv = __ldg(vsm4 + t);
      }
      lsum += e;
      s_e[warp][lane] = e;
      *reinterpret_cast<uint4*>(&s_smw[warp][lane][0]) = smv;
      const int64_t ts = tb + 32 * warp;  // slice start: a multiple of 32 inside one 128-token tile
      const uint32_t* cp = vcw + ((ts >> 7) * kD + 4 * lane) * 16 + ((ts & 127) >> 3);
      uint4 cw[4];
      #pragma unroll
      for (int q = 0; q < 4; ++q) cw[q] = __ldg(reinterpret_cast<const uint4*>(cp + 16 * q));
      __syncwarp();
      #pragma unroll
      for (int w = 0; w < 4; ++w) {
        unsigned bits = (ball >> (8 * w)) & 0xffu;
        while (bits) {
          const int jj = __ffs(bits) - 1;
          bits &= bits - 1u;
          const int j = 8 * w + jj;
          const float ej = s_e[warp][j];
          const uint32_t smw = s_smw[warp][j][grp];
          const float scl = __half2float(__ushort_as_half(static_cast<unsigned short>(smw & 0xffffu)));
          const float mnv = __half2float(__ushort_as_half(static_cast<unsigned short>(smw >> 16)));
          const float es = __fmul_rn(ej, scl);
          accm = __fmaf_rn(ej, mnv, accm);
          #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t word = w == 0 ? cw[q].x : (w == 1 ? cw[q].y : (w == 2 ? cw[q].z : cw[q].w));
            acc[q] = __fmaf_rn(es, static_cast<float>((word >> (4 * jj)) & 0xFu), acc[q]);
          }
        }
      }
      __syncwarp();  // s_e / s_smw are rewritten by the next slice
    }
  }
  #pragma unroll
  for (int q = 0; q < 4; ++q) s_acc[warp][4 * lane + q] = acc[q] + accm;
  lsum = warp_sum(lsum);
  if (lane == 0) s_l[warp] = lsum;
  __syncthreads();
  if (threadIdx.x < kD) {
    float* row = p.part + (r * p.nchunk + chunk) * kPartStride;
    float num = 0.0f;
    for (int w = 0; w < kW; ++w) num += s_acc[w][threadIdx.x];
    row[2 + threadIdx.x] = num;
    if (threadIdx.x == 0) {
      float den = 0.0f;
      for (int w = 0; w < kW; ++w) den += s_l[w];
      row[0] = 0.0f;  // every chunk of the row uses the same reference maximum
      row[1] = den;
    }
  }
}

// Sum of the row's chunk partials in chunk order; rows with nothing selected give zeros.
__global__ void __launch_bounds__(kD) topp_merge_kernel(const ToppParams p) {
  const int64_t r = blockIdx.x;
  const int ch = threadIdx.x;
  const int L = row_len(p, r);
  const int nch = p.rows[r].bstar >= 0 ? (L + kToppChunk - 1) / kToppChunk : 0;
  const float* base = p.part + r * p.nchunk * kPartStride;
  float num = 0.0f, den = 0.0f;
  for (int k = 0; k < nch; ++k) {
    num += base[k * kPartStride + 2 + ch];
    den += base[k * kPartStride + 1];
  }
  p.out[r * kD + ch] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
}

}  // namespace kv1b

using namespace kv1b;

namespace {
size_t al256(size_t x) { return (x + 255) / 256 * 256; }
}  // namespace

// Workspace of kv1b_attend_topp: logits, candidates, row states, bucket histograms, chunk counts,
// gather partials (rows = batch x query heads, capacity tokens each).
size_t kv1b_topp_workspace_bytes(int32_t rows, int32_t cap) {
  const size_t R = static_cast<size_t>(rows), C = static_cast<size_t>(cap);
  const size_t nchunk = (C + kToppChunk - 1) / kToppChunk;
  return al256(R * C * 4) + al256(R * C * 4) + al256(R * sizeof(ToppRowState)) + al256(R * kToppBuckets * 8) +
         al256(R * nchunk * 4) + al256(R * nchunk * kPartStride * 4);
}

void kv1b_topp_carve(ToppParams* p, void* ws, int32_t rows, int32_t cap) {
  const size_t R = static_cast<size_t>(rows), C = static_cast<size_t>(cap);
  const size_t nchunk = (C + kToppChunk - 1) / kToppChunk;
  char* w = static_cast<char*>(ws);
  p->s = reinterpret_cast<float*>(w);
  w += al256(R * C * 4);
  p->cand = reinterpret_cast<int32_t*>(w);
  w += al256(R * C * 4);
  p->rows = reinterpret_cast<ToppRowState*>(w);  // row states and histograms are contiguous: one memset
  w += al256(R * sizeof(ToppRowState));
  p->hist = reinterpret_cast<unsigned long long*>(w);
  w += al256(R * kToppBuckets * 8);
  p->chunk_cnt = reinterpret_cast<uint32_t*>(w);
  w += al256(R * nchunk * 4);
  p->part = reinterpret_cast<float*>(w);
  p->nchunk = static_cast<int32_t>(nchunk);
}

cudaError_t kv1b_launch_topp(const ToppParams& p, int32_t G, int32_t max_len, cudaStream_t stream) {
  const int R = p.c.B * p.Hq;
  if (p.nchunk > 65535) return cudaErrorInvalidValue;  // grid y limit: capacity above 2^28 tokens
  const size_t state_bytes = al256(static_cast<size_t>(R) * sizeof(ToppRowState)) + static_cast<size_t>(R) * kToppBuckets * 8;
  cudaError_t e = cudaMemsetAsync(p.rows, 0, state_bytes, stream);
  if (e != cudaSuccess) return e;
  const dim3 sg(static_cast<unsigned>(p.nchunk), static_cast<unsigned>(R));
  if (max_len > 0) {
    topp_scores_kernel<<<dim3((max_len + kStreamThreads - 1) / kStreamThreads, p.c.Hkv, p.c.B), kStreamThreads, 0,
                         stream>>>(p, G);
    topp_mass_kernel<<<sg, kStreamThreads, 0, stream>>>(p);
  }
  topp_threshold_kernel<<<R, kToppBuckets, 0, stream>>>(p);
  if (max_len > 0) {
    topp_cand_kernel<<<sg, kStreamThreads, 0, stream>>>(p);
    topp_resolve_kernel<<<R, kResolveThreads, 0, stream>>>(p);
  }
  topp_count_kernel<<<sg, kStreamThreads, 0, stream>>>(p);
  topp_write_gather_kernel<<<dim3(static_cast<unsigned>(G), static_cast<unsigned>(p.nchunk),
                              static_cast<unsigned>(p.c.B * p.c.Hkv)),
                         kStreamThreads, 0, stream>>>(p, G);
  topp_merge_kernel<<<R, kD, 0, stream>>>(p);
  return cudaGetLastError();
}
