// kv1b_attend_ws.cu -- persistent split-K decode attention with tensor-core P.V, one CTA per SM.
//
// Work split: all (sequence, kv-head) segments are laid end to end in 16-token tiles and cut into
// one equal contiguous range per CTA, so every SM streams the same number of compressed bytes
// whatever the batch / head / context mix.  Each CTA walks its range in 512-token chunks
// streamed into a 3-stage shared-memory ring with cp.async.bulk (five plain bulk copies per chunk,
// one per cache plane, no multicast) and mbarrier completion; every warp owns a 64-token slice of
// each chunk.  A warp done with a stage counts itself out on a shared counter; the warp that
// counts out last issues the refill, so no warp waits for the others except through the ring.
//
// Each warp does all of the work for its slice, one 16-token tile at a time:
//   the binary x INT4 proxy scores of the G query heads sharing this kv-head ("RaBitQCache",
//   abstract / key design) as integer tensor-core products: the key sign bits are the A operand
//   (one AND per register, bits masked in place), the query's 4-bit codes with a per-channel
//   power-of-two correction the B operand, so the s32 accumulator holds 8 * sum_i bit_i * code_i
//   exactly, plus 8 * Bc in the spare columns; each lane then owns one token of the tile and two
//   head slots (and, for the weights, two of the four value groups);
//   a warp-local online softmax in log2 units whose reference maximum is raised only when a logit
//   exceeds it by 8 (then the warp's sums are rescaled), and the weights p * scale written as
//   fp16 hi + lo rows;
//   then 4 k-steps x 8 m-tiles of mma.sync m16n8k16: the codes as exact fp16 subnormals straight
//   from the staged code tiles (one AND per register), ldmatrix'd weight B fragments; each chunk's
//   tensor-core partial is added into fp32 accumulators on the CUDA cores (round to nearest), so
//   accumulation error does not build up inside the tensor core ("H1B-KV", technical framework:
//   weights from the sketch, then the 4-bit values).  value = min + scale * code, the min term is
//   summed per (head, group) in fp32 by the score lanes.
// At the end of a segment piece the 8 warps' partials are combined in shared memory and the CTA
// writes one row (m, l, o[128]) per query head; the CTA that writes a segment's last row merges
// the segment's rows by log-sum-exp into the output (one kernel per attend).
//
// Every mbarrier wait is bounded: a wait that runs out sets KV1B_STATUS_TIMEOUT in the cache's
// status word; the CTA then stops issuing copies, later waits return at once, and thread 0
// drains the copies already in flight before the CTA exits.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {
namespace ws {

constexpr int kWarps = 8;                        // consumer warps; one more warp issues the copies
constexpr int kTPL = 2;                          // tokens per lane per chunk
constexpr int kThreads = kWarps * 32;            // 256 consumer threads
constexpr int kBlock = kThreads + 32;            // + the producer warp
constexpr int kWarpTiles = 2 * kTPL;             // 16-token tiles per warp per chunk
constexpr int kChunkTiles = kWarpTiles * kWarps; // 32 tiles = 512 tokens per chunk
constexpr int kStages = 3;
constexpr float kTau = 8.0f;                     // lazy-max threshold (log2 units): p <= 2^8
constexpr int kNoExp = 100;                     // group exponent before any scale was seen (finite:
                                                 // every product with it meets a zero)
constexpr float kNoMax = -1e30f;                 // reference maximum before any logit was seen
constexpr long long kSpinLimit = 1LL << 24;

// Stage layout (bytes): one 512-token chunk; warp w uses tokens 64w .. 64w + 63 of it.
constexpr int kChunkTok = kChunkTiles * 16;                   // 512
constexpr int kWarpTok = kWarpTiles * 16;                     // 64
constexpr int kOffBits = 0;                                   // u32 [512][4]
constexpr int kOffNorm = kOffBits + kChunkTok * 16;           // f32 [512]
constexpr int kOffCinv = kOffNorm + kChunkTok * 4;            // f32 [512]
constexpr int kOffSm = kOffCinv + kChunkTok * 4;              // u32 [512][4]
constexpr int kOffCodes = kOffSm + kChunkTok * 16;            // u32 [32 tiles][256]
constexpr int kStageBytes = kOffCodes + kChunkTiles * 1024;   // 53248
constexpr int kGroupRows = kWarpTok + 1;                      // 16-B B rows per group (+1 pad: bank shift)
constexpr int kBRowsPerWarp = 4 * kGroupRows * 16;            // [4 groups][65 rows][16 B]
constexpr int kRowF = 6 + 128;                                // per-warp partial: m, l, mid[4], o[128]
static_assert(4 * kRowF * 4 <= kBRowsPerWarp, "a warp's flush partial reuses its B-row area");
constexpr int kSmemBytes = kStages * kStageBytes + kWarps * kBRowsPerWarp;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
// try_wait that lets the hardware suspend the warp (up to ~0.5 ms per try) instead of spinning,
// so waiting warps give their issue slots to working ones.
__device__ __forceinline__ bool mbar_try_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}
constexpr int kWaitTries = 4096;
// Bounded wait.  Returns false when the CTA has given up (then the caller proceeds on garbage
// data; the status word records the failure and no further copies are issued).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (int tries = 0; tries < kWaitTries; ++tries) {
    if (mbar_try_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  return false;
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
  const uint32_t w8 = __umulhi(w, 1u << 24);  // w >> 8 on the multiply pipe (the logic pipe is the busy one)
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
// Integer tensor-core step of the binary x INT4 product: D (s32) += A (16 tokens x 32 channels,
// s8) * B (32 channels x 8 columns, s8).
__device__ __forceinline__ void imma16832(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Score MMA over one 16-token tile.  Lane (g, t) holds word t of the sign bits of tokens g and
// g + 8.  K-block kb (32 channels) takes, from each word, the bits at positions 8j + 2kb (k = 4t+j)
// and 8j + 2kb + 1 (k = 16+4t+j), j = 0..3, each masked in place so that the byte is
// bit * 2^((2kb + hi) & 3); the query operand carries code * 2^(3 - that), so every product is
// 8 * bit * code and D = 8 * sum_i bit_i * code_i exactly (the integer A of the popcount form;
// the column of ones gives 8 * Bc).
__device__ __forceinline__ void imma16832_zc(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}
__device__ __forceinline__ void score_tile(int d[4], uint32_t wg, uint32_t wg8, const uint32_t (&bq)[4][2]) {
  const uint32_t xg[2] = {wg, __umulhi(wg, 1u << 28)}, xg8[2] = {wg8, __umulhi(wg8, 1u << 28)};  // >> 4
  #pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    const uint32_t mlo = 0x01010101u << (2 * (kb & 1)), mhi = mlo << 1;
    const uint32_t a[4] = {xg[kb >> 1] & mlo, xg8[kb >> 1] & mlo, xg[kb >> 1] & mhi, xg8[kb >> 1] & mhi};
    if (kb == 0) imma16832_zc(d, a, bq[kb][0], bq[kb][1]);
    else imma16832(d, a, bq[kb][0], bq[kb][1]);
  }
}
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ int ilog2_pos(float x) { return static_cast<int>((__float_as_uint(x) >> 23) & 0xff) - 127; }
// exact int -> float for |x| < 2^22 without the quarter-rate conversion unit
__device__ __forceinline__ float i2f_exact(int x) { return __int_as_float(x + 0x4B400000) - 12582912.0f; }

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

// Copy chunk `ch` (contiguous tiles of one segment) into a stage: five bulk copies, one per plane.
__device__ __forceinline__ void issue_chunk(const CacheView& c, const Chunk& ch, uint8_t* st, uint64_t* bar) {
  const uint32_t ntok = ch.nt * 16;
  mbar_expect_tx(bar, ntok * 104u);
  const int64_t tok = static_cast<int64_t>(ch.seg) * c.cap + static_cast<int64_t>(ch.lt) * 16;
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
__global__ void __launch_bounds__(kBlock, 1) attend_ws_kernel(const AttendWsParams p) {
  static_assert(G == 1 || G == 2 || G == 4, "one n-tile: (head, hi/lo) columns <= 8");
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];  // all consumer warps released the stage
  __shared__ __align__(16) uint4 s_planes[2][G][4];  // double-buffered by segment parity
  __shared__ float s_vl[2][G], s_dl[2][G];
  __shared__ int s_sq[2][G];
  __shared__ volatile int s_abort;
  __shared__ int s_merge;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CacheView& c = p.c;
  const Work wk{p.T, p.Lt, static_cast<int>(gridDim.x)};
  const int64_t t_begin = tile_begin(wk, blockIdx.x), t_end = tile_begin(wk, blockIdx.x + 1);
  const int Lt = static_cast<int>(p.Lt);
  const int L = p.L;
  const float qsl = __fmul_rn(__fdiv_rn(p.scale, static_cast<float>(kD)), 0x1.715476p+0f);  // scale/128*log2e
  const int g8 = lane >> 2, t4 = lane & 3;
  uint8_t* brows = smem + kStages * kStageBytes + warp * kBRowsPerWarp;
  uint64_t* bars = full_bar;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[s], 1);
      mbar_init(&empty_bar[s], kWarps);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  TileIt it;  // consume position
  it.seg = static_cast<int>(t_begin / p.Lt);
  it.lt = static_cast<int>(t_begin - static_cast<int64_t>(it.seg) * p.Lt);
  it.rem = static_cast<int>(t_end - t_begin);
  if (warp == kWarps) {  // producer: one lane streams the CTA's chunks through the ring
    if (lane == 0) {
      TileIt is = it;
      int j = 0;  // chunks issued
      while (is.rem > 0 && !s_abort) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&empty_bar[st], ((j / kStages) - 1) & 1, &s_abort)) break;
        const int n = is.nt(Lt);
        issue_chunk(c, Chunk{is.seg, is.lt, n}, smem + st * kStageBytes, &bars[st]);
        is.advance(n, Lt);
        ++j;
      }
      // the CTA's shared memory must outlive every copy issued into it (the consumers wait for
      // all of them unless the CTA gave up)
      for (int k = (j - kStages > 0 ? j - kStages : 0); k < j; ++k) {
        long long spins = 0;
        while (!mbar_try(&bars[k % kStages], (k / kStages) & 1) && ++spins < kSpinLimit) __nanosleep(64);
      }
    }
    return;
  }

  // Score lanes.  MMA row g of a tile holds token g + 8 (g >> 2) and row g + 8 holds token g + 4,
  // so that each half-warp's tokens fill 128 contiguous bytes of a B-row group (conflict-free
  // stores) while the key-word loads stay conflict-free too.  Lane (g, t) takes row g (t < 2) or
  // row g + 8 (t >= 2) and the head slots hs0 = 2 (t & 1), hs0 + 1 of the scores (a slot >= G is
  // empty); for the weights the lane pair (t, t ^ 1), which shares the token, splits the value
  // groups: lane t takes groups 2q, 2q + 1 with q = t & 1.
  const int q1 = t4 & 1;
  const int hs0 = 2 * q1;
  const bool upper = (t4 >> 1) != 0;
  const int row_lo = g8 + 8 * (g8 >> 2), row_hi = g8 + 4;
  const int tokr = upper ? row_hi : row_lo;

  float m_w[G], m_thr[G];        // warp-uniform reference maximum and its rare-path threshold
  float m_my[2], thr_my[2];      // the same for this lane's two head slots
  float l_acc[2];                // sum p of this lane's head slots
  float mid_acc[4][2];           // sum p * min, heads 0..3 x this lane's groups 2q, 2q + 1
  float smax[4];                 // per group: scales up to this keep p * scale * 2^E in fp16 range
  int E_w[4];
  float smax_my[2], ef_my[2];    // smax and 2^E of this lane's groups
  float D[8][4];
  uint32_t bq[4][2];             // score-MMA query operand of this segment
  float vl_my[2], dl4_my[2], kq_my[2];
  auto reset = [&]() {
    #pragma unroll
    for (int h = 0; h < G; ++h) {
      m_w[h] = kNoMax;
      m_thr[h] = kNoMax;
    }
    #pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_my[e] = kNoMax;
      thr_my[e] = kNoMax;
      l_acc[e] = 0.0f;
      smax_my[e] = 0.0f;
      ef_my[e] = exp2i(kNoExp);
    }
    #pragma unroll
    for (int h = 0; h < 4; ++h) mid_acc[h][0] = mid_acc[h][1] = 0.0f;
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
  // memory; then thread (head, channel) combines the warps by log-sum-exp and writes the CTA's
  // row (m, l, o[128] with the mid term folded in) for slot (segment, piece).  Every warp reaches
  // this at the same chunk.
  auto part_of = [&](int w) { return reinterpret_cast<float*>(smem + kStages * kStageBytes + w * kBRowsPerWarp); };

  // Log-sum-exp merge of the n CTA rows of segment `seg` (per query head) into the output; the
  // CTA's shared partials are free by now and hold the piece maxima, sums and weights.  All heads
  // at once: thread t takes channel t & 127 of heads (t >> 7) + 2i, with the pieces' loads
  // independent of one another.
  static_assert(kThreads == 256, "two threads per channel in the merge");
  auto merge_segment = [&](int seg, int n) {
    float* sm_m = part_of(0);       // [G][256] piece maxima, then weights
    float* sm_l = sm_m + 4 * 256;   // [G][256] piece sums
    float* sm_d = sm_l + 4 * 256;   // [G] denominators
    const int b = seg / c.Hkv, kvh = seg - b * c.Hkv;
    const int64_t stride = static_cast<int64_t>(G) * kPartStride;  // between pieces
    const float* base = p.part + static_cast<int64_t>(seg) * p.max_pieces * G * kPartStride;
    for (int i = threadIdx.x; i < G * n; i += kThreads) {
      const int h = i / n, k = i - h * n;
      sm_m[h * 256 + k] = base[k * stride + h * kPartStride];
      sm_l[h * 256 + k] = base[k * stride + h * kPartStride + 1];
    }
    named_bar(1, kThreads);
    if (warp < G) {
      float* mw = sm_m + warp * 256;
      const float* lw = sm_l + warp * 256;
      float M = -INFINITY;
      for (int k = lane; k < n; k += 32) M = fmaxf(M, mw[k]);
      #pragma unroll
      for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, m));
      float den = 0.0f;
      for (int k = lane; k < n; k += 32) {
        const float wt = (mw[k] == -INFINITY || M == -INFINITY) ? 0.0f : exp2f(mw[k] - M);
        den = __fmaf_rn(wt, lw[k], den);
        mw[k] = wt;
      }
      #pragma unroll
      for (int m = 16; m >= 1; m >>= 1) den += __shfl_xor_sync(kFull, den, m);
      if (lane == 0) sm_d[warp] = den;
    }
    named_bar(1, kThreads);
    const int ch = threadIdx.x & 127;
    for (int h = threadIdx.x >> 7; h < G; h += 2) {
      const float* w = sm_m + h * 256;
      const float* o = base + h * kPartStride + 2 + ch;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      int k = 0;
      for (; k + 4 <= n; k += 4) {
        #pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = __fmaf_rn(w[k + u], o[(k + u) * stride], acc[u]);
      }
      for (; k < n; ++k) acc[0] = __fmaf_rn(w[k], o[k * stride], acc[0]);
      const float den = sm_d[h];
      p.out[(static_cast<int64_t>(b) * p.Hq + kvh * G + h) * kD + ch] =
          den > 0.0f ? __fdiv_rn(__fadd_rn(__fadd_rn(acc[0], acc[1]), __fadd_rn(acc[2], acc[3])), den) : 0.0f;
    }
  };
  auto flush = [&](int seg) {
    float v[10];  // l of the own head slots, then mid[head][own group]
    v[0] = l_acc[0];
    v[1] = l_acc[1];
    #pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 + 2 * h] = mid_acc[h][0];
      v[3 + 2 * h] = mid_acc[h][1];
    }
    #pragma unroll
    for (int m = 16; m >= 2; m >>= 1)  // lanes with the same t & 1 hold the same slots and groups
      #pragma unroll
      for (int k = 0; k < 10; ++k) v[k] += __shfl_xor_sync(kFull, v[k], m);
    float* mine = part_of(warp);  // this warp's P.V is done with its B rows
    if (lane < 2) {  // lane q: head slots 2q, 2q + 1 and value groups 2q, 2q + 1
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = 2 * lane + e;
        if (h < G) {
          mine[h * kRowF] = m_my[e] == kNoMax ? -INFINITY : m_my[e];
          mine[h * kRowF + 1] = v[e];
        }
      }
      #pragma unroll
      for (int h = 0; h < G; ++h) {
        mine[h * kRowF + 2 + 2 * lane] = v[2 + 2 * h];
        mine[h * kRowF + 3 + 2 * lane] = v[3 + 2 * h];
      }
    }
    if (t4 < G) {  // D columns 2 t4, 2 t4 + 1 = head t4, hi and lo parts
      float* o = mine + t4 * kRowF + 6;
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const float un = exp2i(24 - E_w[mt >> 1]);  // codes were c * 2^-24
        o[16 * mt + g8] = __fmul_rn(__fadd_rn(D[mt][0], D[mt][1]), un);
        o[16 * mt + g8 + 8] = __fmul_rn(__fadd_rn(D[mt][2], D[mt][3]), un * 0.0625f);
      }
    }
    named_bar(1, kThreads);
    const int ch = threadIdx.x & 127;
    for (int h = threadIdx.x >> 7; h < G; h += kThreads / 128) {
      float M = -INFINITY;
      #pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, part_of(w)[h * kRowF]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
        #pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float* r = part_of(w) + h * kRowF;
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
    // The CTA that writes a segment's last piece merges the segment: ticket after the rows are
    // visible device-wide (the counters are zeroed on the stream before the launch).
    __threadfence();
    named_bar(1, kThreads);
    if (threadIdx.x == 0) {
      const int64_t c0 = cta_of_tile(wk, static_cast<int64_t>(seg) * wk.Lt);
      const int64_t c1 = cta_of_tile(wk, static_cast<int64_t>(seg + 1) * wk.Lt - 1);
      const unsigned n = static_cast<unsigned>(c1 - c0 + 1);
      s_merge = (atomicAdd(p.counters + seg, 1u) == n - 1u) ? static_cast<int>(n) : 0;
    }
    named_bar(1, kThreads);
    const int npieces = s_merge;
    if (npieces > 0) {
      __threadfence();
      merge_segment(seg, npieces);
    }
    named_bar(1, kThreads);  // the shared partials may be rewritten by the next flush
  };

  // Query preparation of a segment's G heads (warp h -> head h) into buffer seg & 1, then every
  // lane builds its score-MMA operand: column n = g of B holds head n's codes (n < G), ones
  // (n >= 4, giving Bc) or zeros; k-row 4t + j of k-block kb is channel 32t + 8j + 2kb (+1 for
  // k-rows 16..31), scaled by 2^(3 - ((2kb + hi) & 3)) to undo the in-place bit position.
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
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
    if (g8 < G) {
      #pragma unroll
      for (int j = 0; j < 4; ++j) pw[j] = reinterpret_cast<const uint32_t*>(&s_planes[par][g8][j])[t4];
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
        bq[kb][hi] = (g8 < G) ? (code << sh) : (g8 >= 4 ? (0x01010101u << sh) : 0u);
      }
    #pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = hs0 + e;
      const bool ok = h < G;
      const float dl = ok ? s_dl[par][ok ? h : 0] : 0.0f;
      vl_my[e] = ok ? s_vl[par][ok ? h : 0] : 0.0f;
      dl4_my[e] = 0.25f * dl;
      kq_my[e] = -dl * static_cast<float>(ok ? s_sq[par][ok ? h : 0] : 0);
    }
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
    mbar_wait(&bars[s], phase, &s_abort);
    const uint8_t* st = smem + s * kStageBytes;
    const int my_tiles = nt - kWarpTiles * warp;  // tiles of this chunk owned by this warp (may be <= 0)

    // tokens of this warp's slice below `lim` are real (beyond: other warps' tiles, a ragged
    // segment end, or slots of the stage that were not filled)
    int lim = L - (it.lt * 16 + kWarpTok * warp);
    lim = lim < my_tiles * 16 ? lim : my_tiles * 16;

    // ---------------- scores: one integer MMA chain per tile, then lane (g, t) takes its token's
    // two head slots and Bc from the accumulator columns (heads in columns 0..3, Bc in 4..7)
    bool valid[kWarpTiles];
    float s2[kWarpTiles][2], sc[kWarpTiles][2], mid[kWarpTiles][2];
    #pragma unroll
    for (int kk = 0; kk < kWarpTiles; ++kk) {
      const int tt = kk * 16 + tokr;  // token within the warp slice
      valid[kk] = tt < lim;
      const uint32_t* kbits = reinterpret_cast<const uint32_t*>(st + kOffBits + warp * kWarpTok * 16) + kk * 64 + t4;
      int d[4];
      score_tile(d, kbits[row_lo * 4], kbits[row_hi * 4], bq);
      const int x0 = __shfl_xor_sync(kFull, d[0], 2);
      const int x2 = __shfl_xor_sync(kFull, d[2], 2);
      const int x3 = __shfl_xor_sync(kFull, d[3], 2);
      const int a0 = upper ? x2 : d[0], a1 = upper ? x3 : d[1], bc8 = upper ? d[2] : x0;
      const float nc = __fmul_rn(__fmul_rn(reinterpret_cast<const float*>(st + kOffNorm)[kWarpTok * warp + tt],
                                           reinterpret_cast<const float*>(st + kOffCinv)[kWarpTok * warp + tt]), qsl);
      // the accumulators hold 8 A and 8 Bc: dot = (delta / 4) 8A + (vl (2 Bc - 128) - delta Sq)
      const float i1 = __fmaf_rn(0.25f, __int2float_rn(bc8), -128.0f);
      const int aa[2] = {a0, a1};
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float dot = __fmaf_rn(dl4_my[e], __int2float_rn(aa[e]), __fmaf_rn(vl_my[e], i1, kq_my[e]));
        s2[kk][e] = (valid[kk] && hs0 + e < G) ? __fmul_rn(dot, nc) : -INFINITY;
      }
      // (scale, min) of this lane's two groups; invalid tokens may read a stage slot never filled
      const uint2 smv = *reinterpret_cast<const uint2*>(st + kOffSm + (kWarpTok * warp + tt) * 16 + q1 * 8);
      const uint32_t smw[2] = {valid[kk] ? smv.x : 0u, valid[kk] ? smv.y : 0u};
      #pragma unroll
      for (int j = 0; j < 2; ++j) {
        sc[kk][j] = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[j] & 0xffffu)));
        mid[kk][j] = __half2float(__ushort_as_half(static_cast<unsigned short>(smw[j] >> 16)));
      }
    }

    // ---------------- warp-local lazy online softmax: rare path when a logit passes its
    // reference by kTau or a value scale passes the group's power-of-two headroom
    bool rare = false;
    #pragma unroll
    for (int kk = 0; kk < kWarpTiles; ++kk) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) rare |= s2[kk][e] > thr_my[e];
      #pragma unroll
      for (int j = 0; j < 2; ++j) rare |= sc[kk][j] > smax_my[j];
    }
    if (__any_sync(kFull, rare)) {
      float lm[2];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        lm[e] = s2[0][e];
        #pragma unroll
        for (int kk = 1; kk < kWarpTiles; ++kk) lm[e] = fmaxf(lm[e], s2[kk][e]);
      }
      #pragma unroll
      for (int h = 0; h < G; ++h) {
        // lanes whose slot (h & 1) is head h contribute; the rest give -inf
        float mx = (hs0 == (h & ~1)) ? lm[h & 1] : -INFINITY;
        #pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        if (mx > m_thr[h]) {  // warp-uniform
          const float alpha = ex2(m_w[h] - mx);  // 0 while m_w is still kNoMax
          m_w[h] = mx;
          m_thr[h] = mx + kTau;
          if (hs0 == (h & ~1)) l_acc[h & 1] = __fmul_rn(l_acc[h & 1], alpha);
          mid_acc[h][0] = __fmul_rn(mid_acc[h][0], alpha);
          mid_acc[h][1] = __fmul_rn(mid_acc[h][1], alpha);
          const float f = (t4 == h) ? alpha : 1.0f;
          #pragma unroll
          for (int mt = 0; mt < 8; ++mt)
            #pragma unroll
            for (int k = 0; k < 4; ++k) D[mt][k] = __fmul_rn(D[mt][k], f);
        }
      }
      #pragma unroll
      for (int e = 0; e < 2; ++e) {  // slot e is head e (t & 1 == 0) or head 2 + e
        const float mlo = (e < G) ? m_w[e < G ? e : 0] : kNoMax;
        const float tlo = (e < G) ? m_thr[e < G ? e : 0] : kNoMax;
        const float mhi = (2 + e < G) ? m_w[2 + e < G ? 2 + e : 0] : kNoMax;
        const float thi = (2 + e < G) ? m_thr[2 + e < G ? 2 + e : 0] : kNoMax;
        m_my[e] = hs0 ? mhi : mlo;
        thr_my[e] = hs0 ? thi : tlo;
      }
      #pragma unroll
      for (int g = 0; g < 4; ++g) {
        float mx = 0.0f;  // lanes holding group g contribute their scales
        if (q1 == (g >> 1)) {
          #pragma unroll
          for (int kk = 0; kk < kWarpTiles; ++kk) mx = fmaxf(mx, sc[kk][g & 1]);
        }
        #pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
        if (mx > smax[g]) {  // warp-uniform
          const int e_new = 6 - ilog2_pos(mx);
          smax[g] = exp2i(7 - e_new);  // scales up to 2^(7-E) keep p * scale * 2^E <= 2^15
          if (e_new < E_w[g]) {
            const float beta = exp2i(e_new - E_w[g]);  // D is still 0 while E_w is kNoExp
            #pragma unroll
            for (int k = 0; k < 4; ++k) {
              D[2 * g][k] = __fmul_rn(D[2 * g][k], beta);
              D[2 * g + 1][k] = __fmul_rn(D[2 * g + 1][k], beta);
            }
            E_w[g] = e_new;
          }
        }
      }
      #pragma unroll
      for (int j = 0; j < 2; ++j) {
        smax_my[j] = q1 ? smax[2 + j] : smax[j];
        ef_my[j] = exp2i(q1 ? E_w[2 + j] : E_w[j]);
      }
    }
    #pragma unroll
    for (int kk = 0; kk < kWarpTiles; ++kk) {
      float pr[2];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        pr[e] = ex2(s2[kk][e] - m_my[e]);  // -inf for invalid tokens and empty slots -> 0
        l_acc[e] = __fadd_rn(l_acc[e], pr[e]);
      }
      // p of all four heads for this token: heads 0, 1 from the pair's even lane, 2, 3 from the odd
      float ph[4];
      ph[0] = __shfl_sync(kFull, pr[0], lane & ~1);
      ph[1] = __shfl_sync(kFull, pr[1], lane & ~1);
      ph[2] = G > 2 ? __shfl_sync(kFull, pr[0], lane | 1) : 0.0f;
      ph[3] = G > 2 ? __shfl_sync(kFull, pr[1], lane | 1) : 0.0f;
      #pragma unroll
      for (int h = 0; h < G; ++h) {
        mid_acc[h][0] = __fmaf_rn(ph[h], mid[kk][0], mid_acc[h][0]);
        mid_acc[h][1] = __fmaf_rn(ph[h], mid[kk][1], mid_acc[h][1]);
      }
      // this token's B rows of the lane's two groups: 8 halves (head, hi/lo)
      #pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float f = __fmul_rn(sc[kk][j], ef_my[j]);
        uint32_t row[4];
        #pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
          const uint64_t w2 = mul2(f2pack(ph[2 * hp], ph[2 * hp + 1]), f2pack(f, f));
          const uint64_t hi2 = w2 & 0xFFFFE000FFFFE000ull;  // 11 significant bits each
          const uint64_t lo2 = sub2(w2, hi2);
          asm("cvt.rn.f16x2.f32 %0, %1, %2;"
              : "=r"(row[2 * hp])
              : "f"(__uint_as_float(static_cast<uint32_t>(lo2))), "f"(__uint_as_float(static_cast<uint32_t>(hi2))));
          asm("cvt.rn.f16x2.f32 %0, %1, %2;"
              : "=r"(row[2 * hp + 1])
              : "f"(__uint_as_float(static_cast<uint32_t>(lo2 >> 32))), "f"(__uint_as_float(static_cast<uint32_t>(hi2 >> 32))));
        }
        *reinterpret_cast<uint4*>(brows + ((2 * q1 + j) * kGroupRows + kk * 16 + tokr) * 16) =
            make_uint4(row[0], row[1], row[2], row[3]);
      }
    }
    __syncwarp();

    // ---------------- P.V: this warp's kWarpTiles tiles x 8 m-tiles, chunk partial flushed into D
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(st + kOffCodes + warp * kWarpTiles * 1024) + lane;
    if (my_tiles > 0) {
      float tmp[8][4];
      #pragma unroll
      for (int kk = 0; kk < kWarpTiles; ++kk) {
        if (kk < my_tiles) {
          uint32_t bf[4][2];
          #pragma unroll
          for (int g = 0; g < 4; ++g) ldsm_x2_trans(bf[g][0], bf[g][1], bbase + (g * kGroupRows + kk * 16) * 16);
          #pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            uint32_t a[4];
            codes_to_afrag(codes[kk * 256 + mt * 32], a);
            if (kk == 0) mma16816_zc(tmp[mt], a, bf[mt >> 1][0], bf[mt >> 1][1]);
            else mma16816(tmp[mt], a, bf[mt >> 1][0], bf[mt >> 1][1]);
          }
        }
      }
      #pragma unroll
      for (int mt = 0; mt < 8; ++mt)
        #pragma unroll
        for (int k = 0; k < 4; ++k) D[mt][k] = __fadd_rn(D[mt][k], tmp[mt][k]);
    }
    __syncwarp();

    // ---------------- release the stage to the producer
    if (lane == 0) mbar_arrive(&empty_bar[s]);  // the warp's reads of the stage completed before __syncwarp
    it.advance(nt, Lt);
    if (++s == kStages) {
      s = 0;
      phase ^= 1u;
    }
  }
  if (t_end > t_begin) flush(cur_seg);
  if (s_abort && lane == 0) atomicOr(p.status, KV1B_STATUS_TIMEOUT);
}

template <int G>
static cudaError_t launch_t(const AttendWsParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attend_ws_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaError_t e = cudaMemsetAsync(p.counters, 0, sizeof(unsigned) * p.c.B * p.c.Hkv, stream);
  if (e != cudaSuccess) return e;
  attend_ws_kernel<G><<<p.ncta, kBlock, kSmemBytes, stream>>>(p);
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

cudaError_t kv1b_launch_attend_ws(const AttendWsParams& p, int32_t G, cudaStream_t stream) {
  switch (G) {
    case 1: return ws::launch_t<1>(p, stream);
    case 2: return ws::launch_t<2>(p, stream);
    case 4: return ws::launch_t<4>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}
