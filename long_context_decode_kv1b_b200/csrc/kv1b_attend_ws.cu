// kv1b_attend_ws.cu -- persistent split-K decode attention with tensor-core P.V, one CTA per SM.
//
// Work split: all (sequence, kv-head) segments are laid end to end in 16-token tiles and cut into
// one equal contiguous range per CTA, so every SM streams the same number of compressed bytes
// whatever the batch / head / context mix.  Each CTA walks its range in 512-token chunks that a
// 3-stage shared-memory ring receives by cp.async.bulk (plain bulk copies, no multicast); an
// mbarrier per stage tracks the bytes, and the last warp to finish a stage refills it.
//
// Each of the 16 warps owns a 32-token slice of every chunk and does all of the work for it, so
// warps never wait on one another inside a segment:
//   lane = token: binary x INT4 popcount proxy scores of the G query heads sharing this kv-head
//   ("RaBitQCache", abstract / key design), a warp-local online softmax in log2 units whose
//   reference maximum is raised only when a logit exceeds it by 8 (then the warp's sums are
//   rescaled), and the weights p * scale written as fp16 hi + lo rows;
//   then 2 k-steps x 8 m-tiles of mma.sync m16n8k16: the codes as exact fp16 subnormals straight
//   from the staged code tiles (one AND per register), ldmatrix'd weight B fragments; each chunk's
//   tensor-core partial is added into fp32 accumulators on the CUDA cores (round to nearest), so
//   accumulation error does not build up inside the tensor core ("H1B-KV", technical framework:
//   weights from the sketch, then the 4-bit values).  value = min + scale * code, the min term is
//   summed per (head, group) in fp32 by the score lanes.
// At the end of a segment piece the 16 warps' partials are combined in shared memory and the CTA
// writes one row (m, l, o[128]) per query head; a merge kernel combines the CTA rows of a head
// by log-sum-exp.
//
// Every mbarrier wait is bounded: a wait that runs out sets KV1B_STATUS_TIMEOUT in the cache's
// status word; the CTA then stops issuing copies, later waits return at once, and thread 0
// drains the copies already in flight before the CTA exits.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {
namespace ws {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;            // 512
constexpr int kChunkTiles = 2 * kWarps;          // 32 tiles = 512 tokens per chunk
constexpr int kChunkTok = kChunkTiles * 16;
constexpr int kStages = 3;
constexpr float kTau = 8.0f;                     // lazy-max threshold (log2 units): p <= 2^8
constexpr int kNoExp = 1 << 20;
constexpr long long kSpinLimit = 1LL << 24;

// stage layout (bytes)
constexpr int kOffBits = 0;                                   // u32 [512][4]
constexpr int kOffNorm = kOffBits + kChunkTok * 16;           // f32 [512]
constexpr int kOffCinv = kOffNorm + kChunkTok * 4;            // f32 [512]
constexpr int kOffSm = kOffCinv + kChunkTok * 4;              // u32 [512][4]
constexpr int kOffCodes = kOffSm + kChunkTok * 16;            // u32 [32 tiles][256]
constexpr int kStageBytes = kOffCodes + kChunkTiles * 1024;   // 53248
constexpr int kBRowsPerWarp = 4 * 32 * 16;                    // [4 groups][32 tokens][16 B]
constexpr int kRowF = 6 + 128;                                // per-warp partial: m, l, mid[4], o[128]
constexpr int kPartSmemBytes = kWarps * 4 * kRowF * 4;        // [16 warps][G <= 4 heads][134] floats
constexpr int kSmemBytes = kStages * kStageBytes + kWarps * kBRowsPerWarp + kPartSmemBytes;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait.  Returns false when the CTA has given up (then the caller proceeds on garbage
// data; the status word records the failure and no further copies are issued).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  long long spins = 0;
  while (!mbar_try(bar, parity)) {
    if (*abort_flag) return false;
    if (++spins > kSpinLimit) {
      *abort_flag = 1;
      return false;
    }
    if (spins > 32) __nanosleep(32);
  }
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& b0, uint32_t& b1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(addr));
}
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// One code word (v_codes layout) -> m16n8k16 A fragment holding the codes as exact fp16
// subnormals: rows g get c * 2^-24 (nibbles at bits 0-3 / 16-19 of a half), rows g + 8 get
// 16 c * 2^-24 (their nibbles sit 4 bits higher).  Both scale factors are undone at the end.
__device__ __forceinline__ void codes_to_afrag(uint32_t w, uint32_t a[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = w & 0x000F000Fu;
  a[1] = w & 0x00F000F0u;
  a[2] = w8 & 0x000F000Fu;
  a[3] = w8 & 0x00F000F0u;
}
__device__ __forceinline__ void mma16816_zc(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ int ilog2_pos(float x) { return static_cast<int>((__float_as_uint(x) >> 23) & 0xff) - 127; }
// exact int -> float for |x| < 2^22 without the quarter-rate conversion unit
__device__ __forceinline__ float i2f_exact(int x) { return __int_as_float(x + 0x4B400000) - 12582912.0f; }

// Binary x INT4 integer A = sum_j 2^j sum_w popc(b_w & P_jw); the four words of a plane are first
// folded by a carry-save adder (3 popcounts per plane instead of 4).
__device__ __forceinline__ int popc_A_csa(const uint4 b, const uint4* P) {
  int A = 0;
  #pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 pj = P[j];
    const uint32_t x0 = b.x & pj.x, x1 = b.y & pj.y, x2 = b.z & pj.z, x3 = b.w & pj.w;
    const uint32_t s = x0 ^ x1 ^ x2;
    const uint32_t c = (x0 & x1) | (x2 & (x0 | x1));
    A += (__popc(s) + __popc(x3) + 2 * __popc(c)) << j;
  }
  return A;
}

struct Work {
  int64_t T;   // total tiles
  int64_t Lt;  // tiles per segment
  int n;       // CTAs
};
__device__ __host__ __forceinline__ int64_t tile_begin(const Work& w, int64_t c) { return c * w.T / w.n; }
__device__ __host__ __forceinline__ int64_t cta_of_tile(const Work& w, int64_t t) { return ((t + 1) * w.n - 1) / w.T; }

struct Chunk {
  int seg, lt, nt;
};
__device__ __forceinline__ Chunk chunk_at(const Work& wk, int64_t t, int64_t t_end) {
  Chunk ch;
  ch.seg = static_cast<int>(t / wk.Lt);
  ch.lt = static_cast<int>(t - static_cast<int64_t>(ch.seg) * wk.Lt);
  int64_t lim = static_cast<int64_t>(ch.seg + 1) * wk.Lt;
  if (lim > t_end) lim = t_end;
  const int64_t n = lim - t;
  ch.nt = static_cast<int>(n < kChunkTiles ? n : kChunkTiles);
  return ch;
}

__device__ __forceinline__ void issue_chunk(const CacheView& c, const Chunk& ch, uint8_t* st, uint64_t* bar) {
  const int64_t tok = static_cast<int64_t>(ch.seg) * c.cap + static_cast<int64_t>(ch.lt) * 16;
  const uint32_t ntok = ch.nt * 16;
  mbar_expect_tx(bar, ntok * 104u);
  bulk_g2s(st + kOffBits, c.k_bits + tok * 4, ntok * 16, bar);
  bulk_g2s(st + kOffNorm, c.k_norm + tok, ntok * 4, bar);
  bulk_g2s(st + kOffCinv, c.k_cinv + tok, ntok * 4, bar);
  bulk_g2s(st + kOffSm, c.v_sm + tok * 4, ntok * 16, bar);
  bulk_g2s(st + kOffCodes, c.v_codes + tok * 16, ntok * 64, bar);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  return static_cast<uint64_t>(__float_as_uint(a)) | (static_cast<uint64_t>(__float_as_uint(b)) << 32);
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Tile iterator over a CTA's range: (segment, tile within segment, tiles left), no divisions.
struct TileIt {
  int seg, lt, rem;
  __device__ __forceinline__ int nt(int Lt) const {
    int n = Lt - lt;
    n = n < rem ? n : rem;
    return n < kChunkTiles ? n : kChunkTiles;
  }
  __device__ __forceinline__ void advance(int n, int Lt) {
    lt += n;
    rem -= n;
    if (lt == Lt) {
      lt = 0;
      ++seg;
    }
  }
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1) attend_ws_kernel(const AttendWsParams p) {
  static_assert(G == 1 || G == 2 || G == 4, "one n-tile: (head, hi/lo) columns <= 8");
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ int s_cnt[kStages];
  __shared__ __align__(16) uint4 s_planes[2][G][4];  // double-buffered by segment parity
  __shared__ float s_vl[2][G], s_dl[2][G];
  __shared__ int s_sq[2][G];
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CacheView& c = p.c;
  const Work wk{p.T, p.Lt, static_cast<int>(gridDim.x)};
  const int64_t t_begin = tile_begin(wk, blockIdx.x), t_end = tile_begin(wk, blockIdx.x + 1);
  const int Lt = static_cast<int>(p.Lt);
  const int L = p.L;
  const float qsl = __fmul_rn(__fdiv_rn(p.scale, static_cast<float>(kD)), 0x1.715476p+0f);  // scale/128*log2e
  const int g8 = lane >> 2, t4 = lane & 3;
  uint8_t* brows = smem + kStages * kStageBytes + warp * kBRowsPerWarp;
  const int tloc = warp * 32 + lane;  // this lane's token within every chunk

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      s_cnt[s] = 0;
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  TileIt it;  // consume position
  it.seg = static_cast<int>(t_begin / p.Lt);
  it.lt = static_cast<int>(t_begin - static_cast<int64_t>(it.seg) * p.Lt);
  it.rem = static_cast<int>(t_end - t_begin);
  TileIt is = it;  // issue position (identical on every warp)
  int issued = 0;
  for (int s = 0; s < kStages && is.rem > 0; ++s) {
    const int n = is.nt(Lt);
    if (threadIdx.x == 0) issue_chunk(c, Chunk{is.seg, is.lt, n}, smem + s * kStageBytes, &full_bar[s]);
    is.advance(n, Lt);
    ++issued;
  }

  float m_w[G], l_acc[G], mid_acc[G][4];
  float smax[4];
  int E_w[4];
  float D[8][4];
  auto reset = [&]() {
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      m_w[h] = -INFINITY;
      l_acc[h] = 0.0f;
      #pragma unroll
      for (int g = 0; g < 4; ++g) mid_acc[h][g] = 0.0f;
    }
    #pragma unroll
    for (int g = 0; g < 4; ++g) {
      smax[g] = 0.0f;
      E_w[g] = kNoExp;
    }
    #pragma unroll
    for (int mt = 0; mt < 8; ++mt)
      #pragma unroll
      for (int k = 0; k < 4; ++k) D[mt][k] = 0.0f;
  };

  // Segment piece done: each warp puts its partial (m, l, mid[4], o[128]) per head in shared
  // memory; then thread (head, channel) combines the 16 warps by log-sum-exp and writes the CTA's
  // row (m, l, o[128] with the mid term folded in) for slot (segment, piece).  Every warp reaches
  // this at the same chunk.
  float* spart = reinterpret_cast<float*>(smem + kStages * kStageBytes + kWarps * kBRowsPerWarp);
  auto flush = [&](int seg) {
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
      for (int k = 0; k < G * 5; ++k) v[k] += __shfl_xor_sync(kFull, v[k], m);
    float* mine = spart + warp * 4 * kRowF;
    if (lane < G) {
      float* r = mine + lane * kRowF;
      float mh = m_w[0], lh = v[0], md[4] = {v[1], v[2], v[3], v[4]};
      #pragma unroll
      for (int h = 1; h < G; ++h)
        if (lane == h) {
          mh = m_w[h];
          lh = v[h * 5];
          #pragma unroll
          for (int g = 0; g < 4; ++g) md[g] = v[h * 5 + 1 + g];
        }
      r[0] = mh;
      r[1] = lh;
      #pragma unroll
      for (int g = 0; g < 4; ++g) r[2 + g] = md[g];
    }
    if (t4 < G) {  // D columns 2 t4, 2 t4 + 1 = head t4, hi and lo parts
      float* o = mine + t4 * kRowF + 6;
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int e = E_w[mt >> 1];
        const float un = (e == kNoExp) ? 0.0f : exp2i(24 - e);  // codes were c * 2^-24
        o[16 * mt + g8] = __fmul_rn(__fadd_rn(D[mt][0], D[mt][1]), un);
        o[16 * mt + g8 + 8] = __fmul_rn(__fadd_rn(D[mt][2], D[mt][3]), un * 0.0625f);
      }
    }
    named_bar(1, kThreads);
    const int h = threadIdx.x >> 7, ch = threadIdx.x & 127;
    if (h < G) {
      float M = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, spart[(w * 4 + h) * kRowF]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
        #pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float* r = spart + (w * 4 + h) * kRowF;
          if (r[0] == -INFINITY) continue;
          const float wt = exp2f(r[0] - M);
          den = __fmaf_rn(wt, r[1], den);
          num = __fmaf_rn(wt, __fadd_rn(r[6 + ch], r[2 + (ch >> 5)]), num);
        }
      }
      const int64_t piece = blockIdx.x - cta_of_tile(wk, static_cast<int64_t>(seg) * wk.Lt);
      float* row = p.part + ((static_cast<int64_t>(seg) * p.max_pieces + piece) * G + h) * kPartStride;
      if (ch == 0) {
        row[0] = M;
        row[1] = den;
      }
      row[2 + ch] = num;
    }
    named_bar(1, kThreads);  // the shared partials may be rewritten by the next flush
  };

  // query preparation of a segment's G heads (warp h -> head h) into buffer seg & 1
  auto prep = [&](int seg) {
    const int par = seg & 1;
    if (warp < G) {
      const int b = seg / c.Hkv, kvh = seg - b * c.Hkv;
      const QueryPrep qp =
          query_prep_warp(p.q, (static_cast<int64_t>(b) * p.Hq + kvh * G + warp) * kD, p.q_dtype, c.signs);
      if (lane == 0) {
        #pragma unroll
        for (int j = 0; j < 4; ++j)
          s_planes[par][warp][j] = make_uint4(qp.planes[j][0], qp.planes[j][1], qp.planes[j][2], qp.planes[j][3]);
        s_vl[par][warp] = qp.vl;
        s_dl[par][warp] = qp.delta;
        s_sq[par][warp] = qp.sq;
      }
    }
    named_bar(1, kThreads);  // reached by every warp at the same chunk
  };

  reset();
  int cur_seg = it.seg;
  if (it.rem > 0) prep(cur_seg);
  const uint32_t bbase = smem_u32(brows) + (lane & 15) * 16;
  int s = 0;           // stage of the current chunk
  uint32_t phase = 0;  // parity of the stage's expected completion
  while (it.rem > 0) {
    const int nt = it.nt(Lt);
    if (it.seg != cur_seg) {
      flush(cur_seg);
      reset();
      cur_seg = it.seg;
      prep(cur_seg);
    }
    const int par = cur_seg & 1;
    mbar_wait(&full_bar[s], phase, &s_abort);
    const uint8_t* st = smem + s * kStageBytes;

    // ---------------- scores of this lane's token (invalid lanes read token 0 and are masked)
    const bool valid = tloc < nt * 16 && it.lt * 16 + tloc < L;
    const int tk = valid ? tloc : 0;
    const uint4 kb = *reinterpret_cast<const uint4*>(st + kOffBits + tk * 16);
    const float nc = __fmul_rn(__fmul_rn(reinterpret_cast<const float*>(st + kOffNorm)[tk],
                                         reinterpret_cast<const float*>(st + kOffCinv)[tk]), qsl);
    const uint4 smv = *reinterpret_cast<const uint4*>(st + kOffSm + tk * 16);
    const float i1 = i2f_exact(2 * popc_Bc(kb) - kD);
    float s2[G];
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      const int A = popc_A_csa(kb, s_planes[par][h]);
      const float dot = __fmaf_rn(s_vl[par][h], i1, __fmul_rn(s_dl[par][h], i2f_exact(2 * A - s_sq[par][h])));
      s2[h] = valid ? __fmul_rn(dot, nc) : -INFINITY;
    }
    float sc[4], mid[4];
    {
      const uint32_t smw[4] = {smv.x, smv.y, smv.z, smv.w};
      #pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float scg = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[g] & 0xffffu)));
        const float mn = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[g] >> 16)));
        sc[g] = valid ? scg : 0.0f;
        mid[g] = mn;
      }
    }

    // ---------------- warp-local lazy online softmax: rare path when a logit passes its
    // reference by kTau or a value scale passes the group's running maximum
    bool rare = false;
    #pragma unroll
    for (int h = 0; h < G; ++h) rare |= s2[h] > m_w[h] + kTau;
    #pragma unroll
    for (int g = 0; g < 4; ++g) rare |= sc[g] > smax[g];  // smax = current power-of-two headroom
    if (__any_sync(kFull, rare)) {
      #pragma unroll
      for (int h = 0; h < G; ++h) {
        float mx = s2[h];
        #pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        if (mx > m_w[h] + kTau) {  // warp-uniform
          const float alpha = (m_w[h] == -INFINITY) ? 0.0f : ex2(m_w[h] - mx);
          m_w[h] = mx;
          l_acc[h] = __fmul_rn(l_acc[h], alpha);
          #pragma unroll
          for (int g = 0; g < 4; ++g) mid_acc[h][g] = __fmul_rn(mid_acc[h][g], alpha);
          const float f = (t4 == h) ? alpha : 1.0f;
          #pragma unroll
          for (int mt = 0; mt < 8; ++mt)
            #pragma unroll
            for (int k = 0; k < 4; ++k) D[mt][k] = __fmul_rn(D[mt][k], f);
        }
      }
      #pragma unroll
      for (int g = 0; g < 4; ++g) {
        float mx = sc[g];
        #pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        if (mx > smax[g]) {  // warp-uniform
          const int e_new = 6 - ilog2_pos(mx);
          smax[g] = exp2i(7 - e_new);  // scales up to 2^(7-E) keep p * scale * 2^E <= 2^15
          if (e_new < E_w[g]) {
            if (E_w[g] != kNoExp) {
              const float beta = exp2i(e_new - E_w[g]);
              #pragma unroll
              for (int k = 0; k < 4; ++k) {
                D[2 * g][k] = __fmul_rn(D[2 * g][k], beta);
                D[2 * g + 1][k] = __fmul_rn(D[2 * g + 1][k], beta);
              }
            }
            E_w[g] = e_new;
          }
        }
      }
    }
    float pr[G];
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      pr[h] = valid ? ex2(s2[h] - m_w[h]) : 0.0f;
      l_acc[h] = __fadd_rn(l_acc[h], pr[h]);
      #pragma unroll
      for (int g = 0; g < 4; ++g) mid_acc[h][g] = __fmaf_rn(pr[h], mid[g], mid_acc[h][g]);
    }
    // ---------------- this token's B rows: [group][token][(head, hi/lo) x 8 halves]
    #pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float f = (E_w[g] == kNoExp) ? 0.0f : __fmul_rn(sc[g], exp2i(E_w[g]));
      uint32_t row[4] = {0u, 0u, 0u, 0u};
      #pragma unroll
      for (int h = 0; h < G; h += 2) {
        if (h + 1 < G) {
          const uint64_t w2 = mul2(f2pack(pr[h], pr[h + 1]), f2pack(f, f));
          const uint64_t hi2 = w2 & 0xFFFFE000FFFFE000ull;  // 11 significant bits each
          const uint64_t lo2 = sub2(w2, hi2);
          asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(row[h]) : "f"(__uint_as_float(static_cast<uint32_t>(lo2))),
              "f"(__uint_as_float(static_cast<uint32_t>(hi2))));
          asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(row[h + 1]) : "f"(__uint_as_float(static_cast<uint32_t>(lo2 >> 32))),
              "f"(__uint_as_float(static_cast<uint32_t>(hi2 >> 32))));
        } else {
          const float w = __fmul_rn(pr[h], f);
          const float hi = __uint_as_float(__float_as_uint(w) & 0xFFFFE000u);
          asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(row[h]) : "f"(__fsub_rn(w, hi)), "f"(hi));
        }
      }
      *reinterpret_cast<uint4*>(brows + (g * 32 + lane) * 16) = make_uint4(row[0], row[1], row[2], row[3]);
    }
    __syncwarp();

    // ---------------- P.V: this warp's 2 tiles x 8 m-tiles, chunk partial flushed into D
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(st + kOffCodes) + warp * 512 + lane;
    const int my_tiles = nt - 2 * warp;  // tiles of this chunk owned by this warp (may be <= 0)
    if (my_tiles > 0) {
      uint32_t bf[4][2][2];
      #pragma unroll
      for (int g = 0; g < 4; ++g)
        #pragma unroll
        for (int kk = 0; kk < 2; ++kk) ldsm_x2_trans(bf[g][kk][0], bf[g][kk][1], bbase + (g * 32 + kk * 16) * 16);
      const bool two = my_tiles > 1;
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        float tmp[4];
        codes_to_afrag(codes[mt * 32], a);
        mma16816_zc(tmp, a, bf[mt >> 1][0][0], bf[mt >> 1][0][1]);
        if (two) {
          codes_to_afrag(codes[256 + mt * 32], a);
          mma16816(tmp, a, bf[mt >> 1][1][0], bf[mt >> 1][1][1]);
        }
        #pragma unroll
        for (int k = 0; k < 4; ++k) D[mt][k] = __fadd_rn(D[mt][k], tmp[k]);
      }
    }
    __syncwarp();

    // ---------------- release the stage; the last warp refills it with the chunk kStages ahead
    if (lane == 0) {
      __threadfence_block();
      const int old = atomicAdd(&s_cnt[s], 1);
      if (old == kWarps - 1) {
        s_cnt[s] = 0;
        if (is.rem > 0 && !s_abort) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue_chunk(c, Chunk{is.seg, is.lt, is.nt(Lt)}, smem + s * kStageBytes, &full_bar[s]);
        }
      }
    }
    if (is.rem > 0) {
      is.advance(is.nt(Lt), Lt);
      ++issued;
    }
    it.advance(nt, Lt);
    if (++s == kStages) {
      s = 0;
      phase ^= 1u;
    }
  }
  if (t_end > t_begin) flush(cur_seg);
  if (s_abort && lane == 0) atomicOr(p.status, KV1B_STATUS_TIMEOUT);
  // before the CTA's shared memory is released, every copy issued into the ring must have landed
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = (issued - kStages > 0 ? issued - kStages : 0); j < issued; ++j) {
      long long spins = 0;
      while (!mbar_try(&full_bar[j % kStages], (j / kStages) & 1) && ++spins < kSpinLimit) __nanosleep(64);
    }
  }
}

// Merge: one block of 128 threads (channels) per (b, hq): log-sum-exp over the CTA pieces of the
// query head's segment.  Row maxima and weights are formed in parallel, then every channel sums
// the pieces with independent loads.
__global__ void __launch_bounds__(128) merge_ws_kernel(const AttendWsParams p, int G) {
  __shared__ float s_w[256];
  __shared__ float s_red[4];
  const int row = blockIdx.x;  // b * Hq + hq
  const int b = row / p.Hq, hq = row - b * p.Hq;
  const int kvh = hq / G, h = hq - kvh * G;
  const int seg = b * p.c.Hkv + kvh;
  const Work wk{p.T, p.Lt, p.ncta};
  float* out = p.out + static_cast<int64_t>(row) * kD;
  if (p.Lt == 0 || p.T == 0) {
    out[threadIdx.x] = 0.0f;
    return;
  }
  const int64_t c0 = cta_of_tile(wk, static_cast<int64_t>(seg) * wk.Lt);
  const int64_t c1 = cta_of_tile(wk, static_cast<int64_t>(seg + 1) * wk.Lt - 1);
  const int n = static_cast<int>(c1 - c0 + 1);  // <= max_pieces <= 256 (host-checked)
  const float* base = p.part + (static_cast<int64_t>(seg) * p.max_pieces * G + h) * kPartStride;
  const int stride = G * kPartStride;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float mk[2], lk[2];
  float M = -INFINITY;
  #pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = threadIdx.x + 128 * u;
    mk[u] = k < n ? base[static_cast<int64_t>(k) * stride] : -INFINITY;
    lk[u] = k < n ? base[static_cast<int64_t>(k) * stride + 1] : 0.0f;
    M = fmaxf(M, mk[u]);
  }
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
  if (lane == 0) s_red[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
  __syncthreads();
  float den = 0.0f;
  #pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = threadIdx.x + 128 * u;
    const float wt = (k < n && mk[u] != -INFINITY && M != -INFINITY) ? exp2f(mk[u] - M) : 0.0f;
    if (k < n) s_w[k] = wt;
    den = __fmaf_rn(wt, lk[u], den);
  }
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) den += __shfl_xor_sync(0xffffffffu, den, m);
  if (lane == 0) s_red[warp] = den;
  __syncthreads();
  den = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
  float num = 0.0f;
  #pragma unroll 8
  for (int k = 0; k < n; ++k) num = __fmaf_rn(s_w[k], base[static_cast<int64_t>(k) * stride + 2 + threadIdx.x], num);
  out[threadIdx.x] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
}

template <int G>
static cudaError_t launch_t(const AttendWsParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attend_ws_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  attend_ws_kernel<G><<<p.ncta, kThreads, kSmemBytes, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  merge_ws_kernel<<<p.c.B * p.Hq, 128, 0, stream>>>(p, G);
  return cudaGetLastError();
}

}  // namespace ws
}  // namespace kv1b

using namespace kv1b;

bool kv1b_ws_supported(int32_t G) { return G == 1 || G == 2 || G == 4; }

// CTAs = SMs (fewer when there are fewer tiles); partial rows per segment = pieces x 16 warps.
void kv1b_ws_plan(int32_t B, int32_t Hkv, int32_t G, int64_t L, int num_sms, int64_t* T, int64_t* Lt, int* ncta,
                  int* max_pieces) {
  const int64_t lt = (L + 15) / 16;
  const int64_t tot = static_cast<int64_t>(B) * Hkv * lt;
  int n = num_sms;
  if (tot < n) n = static_cast<int>(tot > 0 ? tot : 1);
  *T = tot;
  *Lt = lt;
  *ncta = n;
  *max_pieces = tot > 0 ? static_cast<int>((lt * n + tot - 1) / tot + 1) : 1;
  (void)G;
}

int kv1b_ws_rows_per_piece() { return ws::kWarps; }

cudaError_t kv1b_launch_attend_ws(const AttendWsParams& p, int32_t G, cudaStream_t stream) {
  switch (G) {
    case 1: return ws::launch_t<1>(p, stream);
    case 2: return ws::launch_t<2>(p, stream);
    case 4: return ws::launch_t<4>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}
