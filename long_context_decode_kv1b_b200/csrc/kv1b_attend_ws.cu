// kv1b_attend_ws.cu -- persistent split-K decode attention on the integer tensor cores, one CTA per SM.
//
// Work split: all (sequence, kv-head) segments are laid end to end in 128-token tiles and cut into
// one equal contiguous range per CTA, so every SM streams the same number of compressed bytes
// whatever the batch / head / context mix.  A producer warp walks the CTA's range in stages of up
// to three tiles (384 tokens) of one segment through a 3-deep shared-memory ring: one TMA tensor
// load per tile brings the tile's 4-bit value codes ([128 channels][128 tokens], data type
// 16U4_ALIGN16B: every 8 bytes of packed codes land in a 16-byte slot, 128-byte swizzle), and four
// plain bulk copies bring the key bits, N, 1/C and the fp16 (scale, min) pairs.  Completion is
// tracked by mbarriers with transaction bytes; the 12 compute warps release a stage by arriving on
// its "empty" barrier.  The producer's warpgroup gives most of its registers to the compute
// warpgroups (setmaxnreg), so three compute warps share each SM sub-partition.
//
// The compute warps work in 3 quads; quad q owns tile q of a stage (128 tokens), and warp j of the
// quad owns the 32-token slice j of it for the scores and value group j (channels 32 j .. 32 j + 31)
// for the P.V over all 128 tokens:
//   scores ("RaBitQCache", abstract / key design: binary x INT4 arithmetic): per 16 tokens, four
//     mma.m16n8k32 s8 products of the key sign bits (A, one AND per register: each byte keeps one
//     bit in place) with the query's 4-bit codes (B, column 2h = head h scaled to undo the bit
//     position, column 2h + 1 = ones), so lane (g, t) receives 8 A and 8 Bc of tokens g and g + 8
//     for head t exactly -- the integers of the popcount form;
//   softmax: lane (g, t) turns them into head t's logits (log2 units) and probabilities against a
//     reference maximum shared by the quad and raised only when a logit passes it by kTau (then the
//     accumulators are rescaled), so every p <= 2^kTau;
//   weights ("H1B-KV", technical framework: weights from the sketch, then the 4-bit values): lane
//     (g, t) takes value group t of its tokens for all heads (the heads' p by shuffles within the
//     lane quad) and forms W = rint(p * scale * 2^E) < 2^32; E is a per-group power of two kept in
//     step with the largest scale seen (the quad shares it), so the weights of tokens far below the
//     maximum keep many significant bits (a fixed point with fewer bits would round the long tail
//     of a wide softmax to zero and bias the sum).  stmatrix (.trans, b8) writes the four bytes of
//     every W into the quad's buffer; ldmatrix gathers them as the A operand (rows = (head, byte));
//   P.V: ldmatrix .b8x16.b4x16_p64 expands the staged codes to one byte per code (the B operand,
//     k = tokens), and mma.m16n8k32 u8 x u8 -> s32 accumulates sum_t W * code per (head, byte,
//     channel) EXACTLY in 32-bit integers; value = min + scale * code, the min term is summed per
//     (head, group) in fp32.  The integer accumulators are converted (and rescaled) only when the
//     reference maximum or a group exponent moves, and at the end of a segment piece.
// At the end of a segment piece the quads' partials are combined in shared memory and the CTA
// writes one row (m, l, o[128]) per query head; the CTA that writes a segment's last row merges
// the segment's rows by log-sum-exp into the output (one kernel per attend).
//
// Every mbarrier wait is bounded: a wait that runs out sets KV1B_STATUS_TIMEOUT in the cache's
// status word; the CTA then stops issuing copies, later waits poll once and return, and the
// producer drains the copies already in flight before the CTA exits.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {
namespace ws {

constexpr int kQuads = 3;
constexpr int kWarps = 4 * kQuads;          // compute warps
constexpr int kThreads = kWarps * 32;       // 384 compute threads
constexpr int kBlock = kThreads + 128;      // + the producer warpgroup
constexpr int kComputeRegs = 160;           // setmaxnreg: 384 x 160 + 128 x 24 <= 512 x 128 registers (the producer thread may spill)
constexpr int kProducerRegs = 24;
static_assert(kThreads * kComputeRegs + 128 * kProducerRegs <= 65536, "register split within the launch's registers");
constexpr int kTileTok = 128;               // tokens per code tile (one TMA box)
constexpr int kStageTiles = 3;
constexpr int kStageTok = kStageTiles * kTileTok;
constexpr int kStages = 3;
constexpr int kTau = 4;                     // lazy-max threshold (log2 units): p <= 2^kTau
constexpr int kScaleRoom = 2;               // bits of headroom above the largest scale seen
constexpr int kNoExp = 100;                 // group exponent before any scale was seen
constexpr float kNoMax = -1e30f;            // reference maximum before any logit was seen
constexpr int kMaxAccStages = 4096;         // int32 headroom: 255 * 15 * 128 tokens * 4096 < 2^31
constexpr long long kSpinLimit = 1LL << 24;

// Stage layout (bytes).
constexpr int kTileSmem = kTileTok * 128;                  // 128 channels x 128 B (8 B codes + 8 B gap per 16 tokens)
constexpr int kOffCodes = 0;
constexpr int kOffBits = kStageTiles * kTileSmem;          // u32 [384][4]
constexpr int kOffNorm = kOffBits + kStageTok * 16;        // f32 [384]
constexpr int kOffCinv = kOffNorm + kStageTok * 4;         // f32 [384]
constexpr int kOffSm = kOffCinv + kStageTok * 4;           // u32 [384][4]
constexpr int kStageBytes = (kOffSm + kStageTok * 16 + 1023) / 1024 * 1024;
constexpr int kWSlice = 16 * 128;                          // one warp's 32 tokens: 16 byte matrices of 8 rows x 16 tokens
constexpr int kWQuad = 4 * kWSlice;
constexpr int kOffW = kStages * kStageBytes;
constexpr int kRowL = 1, kRowMid = 5, kRowO = 24;          // quad partial row per head: m, l[4 warps], mid[4 warps][4 groups], -, o[128]
constexpr int kRowQ = kRowO + 128;
constexpr int kSmemUsed = kOffW + kQuads * kWQuad;
constexpr int kSmemBytes = kSmemUsed + 1024;               // + slack to align the base to 1024 B
constexpr uint32_t kTxPerTile = kTileTok * 104;            // packed codes 64 B + 40 B of the other planes per token
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(kOffW % 1024 == 0 && kStageBytes % 1024 == 0, "TMA 128B-swizzle destinations are 1024-B aligned");
static_assert(4 * kRowQ * 4 <= kWQuad, "a quad's partial rows fit its weight buffer");
static_assert(2 * 4 * 256 * 4 + 64 <= kQuads * kWQuad, "the segment merge reuses the weight buffers");

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
// try_wait that lets the hardware suspend the warp (up to ~0.5 ms per try) instead of spinning.
__device__ __forceinline__ bool mbar_try_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}
// Bounded wait: at most `tries` suspended tries.  Returns false when the CTA has given up (then the
// caller proceeds on garbage data; the status word records the failure and no further copies are
// issued); once the CTA has given up, a wait that does not find its phase complete at the first
// poll returns at once.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int tries) {
  if (*abort_flag) return mbar_try(bar, parity);
  for (int i = 0; i < tries; ++i) {
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
// One 128-token code tile: box [128 tokens, 128 channels, 1 tile] at tile index z (no multicast).
__device__ __forceinline__ void tma_codes(void* dst, const CUtensorMap* map, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(0), "r"(0), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Named barrier over n threads that also returns the OR of their predicates c.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool c) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred pc, pr; setp.ne.u32 pc, %3, 0; barrier.cta.red.or.pred pr, %1, %2, pc; selp.u32 %0, 1, 0, pr; }"
      : "=r"(r)
      : "r"(id), "r"(n), "r"(static_cast<uint32_t>(c))
      : "memory");
  return r != 0;
}

// Integer tensor-core products (m16n8k32: A 16 x 32, B 32 x 8, D 16 x 8 s32).
__device__ __forceinline__ void imma_s8(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1, bool zero) {
  if (zero)
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_u8(int d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Four 8 x 16-byte matrices; lane i addresses row i & 7 of matrix i >> 3; register j of lane
// (g, t) receives bytes 4t .. 4t + 3 of row g of matrix j.
__device__ __forceinline__ void ldsm_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Same with rows of 16 packed 4-bit values (8 data bytes, then an 8-byte gap): element e of a row
// becomes byte e of the row, value in bits 0-3 (low nibble = even element).
__device__ __forceinline__ void ldsm_x4_u4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n16.x4.shared.b8x16.b4x16_p64 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Four 16 x 8 byte matrices stored transposed: byte b of register m of lane (g, t) goes to row
// 2t + (b & 1), column g + 8 (b >> 1) of matrix m, whose 16-byte rows lanes 8m .. 8m + 7 address.
__device__ __forceinline__ void stsm_x4_t8(uint32_t addr, const uint32_t r[4]) {
  asm volatile("stmatrix.sync.aligned.m16n8.x4.trans.shared.b8 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Score MMA over one 16-token tile.  Lane (g, t) holds word t of the sign bits of tokens g and
// g + 8.  K-block kb (32 channels) takes, from each word, the bits at positions 8j + 2kb (k = 4t+j)
// and 8j + 2kb + 1 (k = 16+4t+j), j = 0..3, each masked in place so that the byte is
// bit * 2^((2kb + hi) & 3); the query operand carries code * 2^(3 - that), so every product is
// 8 * bit * code and D = 8 * sum_i bit_i * code_i exactly (the integer A of the popcount form;
// the columns of ones give 8 * Bc).  K-blocks 0-1 and 2-3 accumulate separately (two chains of two
// dependent products instead of one of four) and are added at the end.
__device__ __forceinline__ void score_tile(int d[4], uint32_t wg, uint32_t wg8, const uint32_t (&bq)[4][2]) {
  const uint32_t xg[2] = {wg, __umulhi(wg, 1u << 28)}, xg8[2] = {wg8, __umulhi(wg8, 1u << 28)};  // >> 4
  int d2[4];
  #pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    const uint32_t mlo = 0x01010101u << (2 * (kb & 1)), mhi = mlo << 1;
    const uint32_t a[4] = {xg[kb >> 1] & mlo, xg8[kb >> 1] & mlo, xg[kb >> 1] & mhi, xg8[kb >> 1] & mhi};
    imma_s8(kb < 2 ? d : d2, a, bq[kb][0], bq[kb][1], (kb & 1) == 0);
  }
  #pragma unroll
  for (int i = 0; i < 4; ++i) d[i] += d2[i];
}
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ int ilog2_pos(float x) { return static_cast<int>((__float_as_uint(x) >> 23) & 0xff) - 127; }
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <typename T>
__device__ __forceinline__ T sel4(const T (&v)[4], int i) {
  return i == 0 ? v[0] : (i == 1 ? v[1] : (i == 2 ? v[2] : v[3]));
}

struct Work {
  int64_t T;   // total tiles
  int64_t Lt;  // tiles per segment
  int n;       // CTAs
};
__device__ __host__ __forceinline__ int64_t tile_begin(const Work& w, int64_t c) { return c * w.T / w.n; }
__device__ __host__ __forceinline__ int64_t cta_of_tile(const Work& w, int64_t t) { return ((t + 1) * w.n - 1) / w.T; }

// Tile iterator over a CTA's range: (segment, tile within segment, tiles left), no divisions.
struct TileIt {
  int seg, lt, rem;
  __device__ __forceinline__ int nt(int Lt) const {
    int n = Lt - lt;
    n = n < rem ? n : rem;
    return n < kStageTiles ? n : kStageTiles;
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

// Copy a stage: n tiles of segment `seg` starting at tile `lt`.
__device__ __forceinline__ void issue_stage(const AttendWsParams& p, int seg, int lt, int n, uint8_t* st, uint64_t* bar) {
  const CacheView& c = p.c;
  mbar_expect_tx(bar, n * kTxPerTile);
  const int tiles_per_seg = c.cap / kTileTok;
  for (int i = 0; i < n; ++i) tma_codes(st + kOffCodes + i * kTileSmem, &p.codes_map, seg * tiles_per_seg + lt + i, bar);
  const int64_t tok = static_cast<int64_t>(seg) * c.cap + static_cast<int64_t>(lt) * kTileTok;
  const uint32_t ntok = n * kTileTok;
  bulk_g2s(st + kOffBits, c.k_bits + tok * 4, ntok * 16, bar);
  bulk_g2s(st + kOffNorm, c.k_norm + tok, ntok * 4, bar);
  bulk_g2s(st + kOffCinv, c.k_cinv + tok, ntok * 4, bar);
  bulk_g2s(st + kOffSm, c.v_sm + tok * 4, ntok * 16, bar);
}

// PROBE: the test instantiation that also writes every score product and logit it forms
// (p.probe_A / probe_Bc / probe_s); the product kernel is PROBE = false.  FULL: the launch fills all
// G head slots (the head count is then a compile-time constant); otherwise p.heads < G of them.
template <int G, bool PROBE, bool FULL>
__global__ void __launch_bounds__(kBlock, 1) attend_ws_kernel(const __grid_constant__ AttendWsParams p) {
  static_assert(G == 1 || G == 2 || G == 4, "head t of lane (g, t) for t < G");
  // this launch serves query heads head_base .. head_base + NH - 1 of each kv-head's G_all (NH <= G;
  // lanes of absent heads carry no probability, so their weights and sums are zero)
  const int NH = FULL ? G : p.heads;
  const int GA = p.G_all, HB = p.head_base;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];  // all compute warps released the stage
  __shared__ __align__(16) uint4 s_planes[2][4][4];     // double-buffered by segment parity
  __shared__ float s_vl[2][4], s_dl[2][4];
  __shared__ int s_sq[2][4];
  __shared__ float s_xchg[kQuads][4][8];                 // its slice maxima: logits per head, scales per group
  __shared__ volatile int s_abort;
  __shared__ int s_merge;

  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const CacheView& c = p.c;
  const Work wk{p.T, p.Lt, static_cast<int>(gridDim.x)};
  const int64_t t_begin = tile_begin(wk, blockIdx.x), t_end = tile_begin(wk, blockIdx.x + 1);
  const int Lt = static_cast<int>(p.Lt);
  const int L = p.L;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kWarps);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();  // every thread, before any global memory access: q and the cache may come from the previous kernel
  TileIt it;  // consume position
  it.seg = static_cast<int>(t_begin / p.Lt);
  it.lt = static_cast<int>(t_begin - static_cast<int64_t>(it.seg) * p.Lt);
  it.rem = static_cast<int>(t_end - t_begin);
  if (warp >= kWarps) {  // producer warpgroup: one lane streams the CTA's stages through the ring
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
    if (warp == kWarps && lane == 0) {
      TileIt is = it;
      int j = 0;  // stages issued
      while (is.rem > 0 && !s_abort) {
        if (j == p.stall_stage) break;  // test hook: this stage's copies never arrive
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(&empty_bar[st], ((j / kStages) - 1) & 1, &s_abort, p.wait_tries)) break;
        const int n = is.nt(Lt);
        issue_stage(p, is.seg, is.lt, n, smem + st * kStageBytes, &full_bar[st]);
        is.advance(n, Lt);
        ++j;
        // the first stage alone first: every CTA's first stage then lands at once instead of with
        // the ring's other stages, and the compute warps start about 3 us earlier
        if (j == 1 && !mbar_wait(&full_bar[0], 0, &s_abort, p.wait_tries)) break;
      }
      // the CTA's shared memory must outlive every copy issued into it (the compute warps wait
      // for all of them unless the CTA gave up)
      for (int k = (j - kStages > 0 ? j - kStages : 0); k < j; ++k) {
        long long spins = 0;
        while (!mbar_try(&full_bar[k % kStages], (k / kStages) & 1) && ++spins < kSpinLimit) __nanosleep(64);
      }
    }
    return;
  }
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kComputeRegs));

  const int g = lane >> 2, t = lane & 3;
  const int qd = warp >> 2, jw = warp & 3;  // quad; slice and value group of this warp
  const int hh = g & 3;                     // head of this lane's P.V accumulator rows
  const bool lo_bytes = (g >> 2) == 0;       // rows g / g + 8 hold bytes 0 / 2 (else bytes 1 / 3)
  const float qsl = __fmul_rn(__fdiv_rn(p.scale, static_cast<float>(kD)), 0x1.715476p+0f);  // scale/128 * log2 e
  const int tl = qd;                                        // the quad's tile in the stage
  const int sbase = tl * kTileTok + 32 * jw;                // this warp's score slice
  const uint32_t wq_s = smem_u32(smem + kOffW + qd * kWQuad);
  // stmatrix row address of this lane: matrix (kk, head m = lane >> 3, lo/hi), row rho = lane & 7
  // kept in slot (rho + 2 m) & 7 so that the A-operand gathers below are free of bank conflicts
  const uint32_t st_addr = wq_s + jw * kWSlice +
                           static_cast<uint32_t>((lane >> 3) * 2 * 128 + (((lane & 7) + 2 * (lane >> 3)) & 7) * 16);
  // A-operand gather of group jw: lane i addresses A row r = (i & 7) + 8 ((i >> 3) & 1) of k-half
  // kk = i >> 4 of slice ks; row r = (head r & 3, byte r >> 2)
  const int a_r = (lane & 7) + 8 * ((lane >> 3) & 1), a_kk = lane >> 4;
  const int a_head = a_r & 3, a_byte = a_r >> 2;
  const uint32_t a_pre = wq_s + static_cast<uint32_t>(((a_kk * 4 + a_head) * 2 + (a_byte >> 1)) * 128) +
                         static_cast<uint32_t>((((a_byte & 1) + 2 * a_head + 2 * jw) & 7) * 16);
  // code-tile gathers: lanes 8m .. 8m + 7 address channel rows 32 jw + 8 (2 np + (m >> 1)) + (lane & 7)
  // of 16-token chunk 2 ks + (m & 1); 128-byte swizzle: chunk ^ (row & 7) = ((m & 1) ^ (row & 7)) ^ 2 ks
  const uint32_t c_off = static_cast<uint32_t>(tl * kTileSmem + (32 * jw + 8 * (lane >> 4) + (lane & 7)) * 128);
  const uint32_t c_kx0 = static_cast<uint32_t>((((lane >> 3) & 1) ^ (lane & 7)) << 4);
  // weight-rounding dither: a Weyl sequence over the lane's 32-token slices (top byte of
  // n * 0x9E3779B9 + lane * 0x6A09E667, n = slice index in the segment), one value per lane and slice
  const uint32_t weyl_c = static_cast<uint32_t>(lane) * 0x6A09E667u;

  // per-lane state
  float m_w[4], smax_w[4];  // quad-uniform: reference maximum per head, scale bound per group
  int E_w[4];               // quad-uniform: weight exponent per group
  float m_t, thr_t, s2e_t, smax_t;  // the same for this lane's head t / group t
  float l_t;                // sum p of head t over this lane's tokens
  float mid[4];             // sum p * min of group t, heads 0..3
  int D[4][4];              // P.V integer accumulators: n-tile (8 channels) x (rows g, g + 8) x 2 channels
  float F[4][2];            // converted P.V sums of this lane's rows
  uint32_t bq[4][2];        // score-MMA query operand of this segment
  float c1_t, c2_t, c0_t;   // head t logit constants
  bool hv_t;                // head t exists
  int nacc = 0;             // stages accumulated in D since the last conversion

  auto reset = [&]() {
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      m_w[i] = kNoMax;
      smax_w[i] = 0.0f;
      E_w[i] = kNoExp;
      mid[i] = 0.0f;
    }
    m_t = kNoMax;
    thr_t = kNoMax;
    s2e_t = exp2i(kNoExp);
    smax_t = 0.0f;
    l_t = 0.0f;
    #pragma unroll
    for (int n = 0; n < 4; ++n) {
      D[n][0] = D[n][1] = D[n][2] = D[n][3] = 0;
      F[n][0] = F[n][1] = 0.0f;
    }
    nacc = 0;
  };
  // Convert the integer accumulators into F (old exponents), then scale F by alpha of this lane's head.
  auto drain = [&](float al) {
    const float wb0 = lo_bytes ? 1.0f : 256.0f, wb2 = lo_bytes ? 65536.0f : 16777216.0f;
    const float inv = exp2i(-sel4(E_w, jw));
    #pragma unroll
    for (int n = 0; n < 4; ++n) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x = __fmaf_rn(wb2, static_cast<float>(D[n][2 + e]), __fmul_rn(wb0, static_cast<float>(D[n][e])));
        F[n][e] = __fmul_rn(__fmaf_rn(x, inv, F[n][e]), al);
        D[n][e] = 0;
        D[n][2 + e] = 0;
      }
    }
    nacc = 0;
  };

  auto prow = [&](int q, int h) { return reinterpret_cast<float*>(smem + kOffW + q * kWQuad) + h * kRowQ; };

  // Log-sum-exp merge of the n CTA rows of segment `seg` (per query head) into the output; uses
  // the weight buffers as scratch.  All heads at once: thread i takes channel i & 127 of heads
  // (i >> 7) + 3k, with the pieces' loads independent of one another.
  auto merge_segment = [&](int seg, int n) {
    float* sm_m = reinterpret_cast<float*>(smem + kOffW);  // [G][256] piece maxima, then weights
    float* sm_l = sm_m + 4 * 256;                          // [G][256] piece sums
    float* sm_d = sm_l + 4 * 256;                          // [G] denominators
    float* sm_M = sm_d + 4;                                // [G] maxima
    const int b = seg / c.Hkv, kvh = seg - b * c.Hkv;
    const int64_t stride = static_cast<int64_t>(G) * kPartStride;  // between pieces
    const float* base = p.part + static_cast<int64_t>(seg) * p.max_pieces * G * kPartStride;
    for (int i = threadIdx.x; i < NH * n; i += kThreads) {
      const int h = i / n, k = i - h * n;
      sm_m[h * 256 + k] = base[k * stride + h * kPartStride];
      sm_l[h * 256 + k] = base[k * stride + h * kPartStride + 1];
    }
    named_bar(1, kThreads);
    if (warp < NH) {
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
      if (lane == 0) {
        sm_d[warp] = den;
        sm_M[warp] = M;
      }
    }
    named_bar(1, kThreads);
    // thread (h, ch) for h = threadIdx.x >> 7 and h + 3: the pieces' o[ch] of both heads are loaded
    // 16 pieces at a time, all loads issued before the sums (one round trip to L2 per 16 pieces)
    const int ch = threadIdx.x & 127;
    const int ha = threadIdx.x >> 7, hb = ha + kThreads / 128;
    const bool two = hb < NH;
    auto emit = [&](int h, const float (&acc)[4]) {
      const float den = sm_d[h];
      const float num = __fadd_rn(__fadd_rn(acc[0], acc[1]), __fadd_rn(acc[2], acc[3]));
      const int64_t orow = static_cast<int64_t>(b) * p.Hq + kvh * GA + HB + h;
      if (p.partial_out) {  // the segment's log-sum-exp row (m, l, o[128]) for a later merge
        float* o = p.out + orow * kPartStride;
        if (ch == 0) {
          o[0] = sm_M[h];
          o[1] = den;
        }
        o[2 + ch] = num;
      } else {
        p.out[orow * kD + ch] = den > 0.0f ? __fdiv_rn(num, den) : 0.0f;
      }
    };
    if (ha < NH) {
      const float* oa = base + ha * kPartStride + 2 + ch;
      const float* ob = base + (two ? hb : ha) * kPartStride + 2 + ch;
      const float* wa = sm_m + ha * 256;
      const float* wb = sm_m + (two ? hb : ha) * 256;
      float acca[4] = {0.0f, 0.0f, 0.0f, 0.0f}, accb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int k0 = 0; k0 < n; k0 += 16) {
        float xa[16], xb[16];
        #pragma unroll
        for (int u = 0; u < 16; ++u) {
          const bool in = k0 + u < n;
          xa[u] = in ? oa[(k0 + u) * stride] : 0.0f;
          xb[u] = (in && two) ? ob[(k0 + u) * stride] : 0.0f;
        }
        #pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (k0 + u < n) {
            acca[u & 3] = __fmaf_rn(wa[k0 + u], xa[u], acca[u & 3]);
            accb[u & 3] = __fmaf_rn(wb[k0 + u], xb[u], accb[u & 3]);
          }
        }
      }
      emit(ha, acca);
      if (two) emit(hb, accb);
    }
  };

  // Segment piece done: each warp puts its share of the quad's partial (m, l, mid, o) per head in
  // the quad's weight buffer; then thread (head, channel) combines the quads by log-sum-exp and
  // writes the CTA's row (m, l, o[128] with the mid terms folded in) for slot (segment, piece).
  // Every compute warp reaches this at the same stage.
  auto flush = [&](int seg) {
    drain(1.0f);
    #pragma unroll
    for (int n = 0; n < 4; ++n)  // rows g (g < 4) and g + 4 of the same head: bytes {0, 2} and {1, 3}
      #pragma unroll
      for (int e = 0; e < 2; ++e) F[n][e] = __fadd_rn(F[n][e], __shfl_xor_sync(kFull, F[n][e], 16));
    float v[5] = {l_t, mid[0], mid[1], mid[2], mid[3]};
    #pragma unroll
    for (int m = 4; m <= 16; m <<= 1)  // sum over the 8 lanes with the same t
      #pragma unroll
      for (int k = 0; k < 5; ++k) v[k] = __fadd_rn(v[k], __shfl_xor_sync(kFull, v[k], m));
    named_bar(1, kThreads);  // every quad is done with its weight buffer
    if (g == 0) {  // lane t: head t's m and l of this slice, group t's mid of every head
      if (t < NH) {
        if (jw == 0) prow(qd, t)[0] = m_t == kNoMax ? -INFINITY : m_t;
        prow(qd, t)[kRowL + jw] = v[0];
      }
      #pragma unroll
      for (int h = 0; h < G; ++h)
        if (h < NH) prow(qd, h)[kRowMid + 4 * jw + t] = v[1 + h];
    }
    if (g < NH) {  // head g: channels 32 jw + 8n + 2t + e
      float* o = prow(qd, g) + kRowO + 32 * jw + 2 * t;
      #pragma unroll
      for (int n = 0; n < 4; ++n) *reinterpret_cast<float2*>(o + 8 * n) = make_float2(F[n][0], F[n][1]);
    }
    named_bar(1, kThreads);
    const int ch = threadIdx.x & 127;
    for (int h = threadIdx.x >> 7; h < NH; h += kThreads / 128) {
      float M = -INFINITY;
      #pragma unroll
      for (int q = 0; q < kQuads; ++q) M = fmaxf(M, prow(q, h)[0]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
        const int grp = ch >> 5;
        #pragma unroll
        for (int q = 0; q < kQuads; ++q) {
          const float* r = prow(q, h);
          if (r[0] == -INFINITY) continue;
          const float wt = exp2f(r[0] - M);
          den = __fmaf_rn(wt, __fadd_rn(__fadd_rn(r[kRowL], r[kRowL + 1]), __fadd_rn(r[kRowL + 2], r[kRowL + 3])), den);
          const float md = __fadd_rn(__fadd_rn(r[kRowMid + grp], r[kRowMid + 4 + grp]),
                                     __fadd_rn(r[kRowMid + 8 + grp], r[kRowMid + 12 + grp]));
          num = __fmaf_rn(wt, __fadd_rn(r[kRowO + ch], md), num);
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
    // visible device-wide.  The counters are zero at launch (a memset on the stream, or left so by
    // the previous launch on the same workspace): the merging CTA resets its segment's counter.
    __threadfence();
    named_bar(1, kThreads);
    if (threadIdx.x == 0) {
      const int64_t c0 = cta_of_tile(wk, static_cast<int64_t>(seg) * wk.Lt);
      const int64_t c1 = cta_of_tile(wk, static_cast<int64_t>(seg + 1) * wk.Lt - 1);
      const unsigned n = static_cast<unsigned>(c1 - c0 + 1);
      const bool last = atomicAdd(p.counters + seg, 1u) == n - 1u;
      s_merge = last ? static_cast<int>(n) : 0;
      if (last) p.counters[seg] = 0u;  // every piece of the segment has taken its ticket
    }
    named_bar(1, kThreads);
    const int npieces = s_merge;
    if (npieces > 0) {
      __threadfence();
      merge_segment(seg, npieces);
    }
    named_bar(1, kThreads);  // the buffers may be rewritten by the next segment
  };

  // Query preparation of a segment's G heads (warp h -> head h) into buffer seg & 1, then every
  // lane builds its score-MMA operand: column n = g of B holds head g / 2's codes (g even, head
  // < G), ones (g odd, giving Bc) or zeros; k-row 4t + j of k-block kb is channel
  // 32t + 8j + 2kb (+1 for k-rows 16..31), scaled by 2^(3 - ((2kb + hi) & 3)) to undo the
  // in-place bit position.
  // Query preparation of segment `seg`'s head h by the calling warp into buffer seg & 1.
  auto prep_head = [&](int seg, int h) {
    const int par = seg & 1;
    const int b = seg / c.Hkv, kvh = seg - b * c.Hkv;
    const QueryPrep qp =
        query_prep_warp(p.q, (static_cast<int64_t>(b) * p.Hq + kvh * GA + HB + h) * kD, p.q_dtype, c.signs);
    if (lane == 0) {
      #pragma unroll
      for (int j = 0; j < 4; ++j)
        s_planes[par][h][j] = make_uint4(qp.planes[j][0], qp.planes[j][1], qp.planes[j][2], qp.planes[j][3]);
      s_vl[par][h] = qp.vl;
      s_dl[par][h] = qp.delta;
      s_sq[par][h] = qp.sq;
    }
  };
  // next_seg >= 0: warps 4 .. 4 + G - 1 also prepare that segment (the CTA's second one) now, so its
  // switch later skips the preparation (pre = true).
  auto prep = [&](int seg, bool pre, int next_seg) {
    const int par = seg & 1;
    if (!pre && warp < NH) prep_head(seg, warp);
    if (next_seg >= 0 && warp >= 4 && warp < 4 + NH) prep_head(next_seg, warp - 4);
    named_bar(1, kThreads);  // reached by every compute warp at the same stage
    const int hb = g >> 1;
    const bool code_col = (g & 1) == 0 && hb < NH;
    uint32_t pw[4] = {0u, 0u, 0u, 0u};
    if (code_col) {
      #pragma unroll
      for (int j = 0; j < 4; ++j) pw[j] = reinterpret_cast<const uint32_t*>(&s_planes[par][hb][j])[t];
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
        bq[kb][hi] = code_col ? (code << sh) : ((g & 1) ? (0x01010101u << sh) : 0u);
      }
    hv_t = t < NH;
    const int hs = hv_t ? t : 0;
    const float dl = hv_t ? s_dl[par][hs] : 0.0f, vl = hv_t ? s_vl[par][hs] : 0.0f;
    const float sq = hv_t ? static_cast<float>(s_sq[par][hs]) : 0.0f;
    // dot = delta (2A - Sq) + vl (2Bc - 128) = (delta / 4) 8A + (vl / 4) 8Bc - (delta Sq + 128 vl)
    c1_t = __fmul_rn(0.25f * dl, qsl);
    c2_t = __fmul_rn(0.25f * vl, qsl);
    c0_t = __fmul_rn(-__fadd_rn(__fmul_rn(dl, sq), 128.0f * vl), qsl);
  };

  reset();
  int cur_seg = it.seg;
  // the CTA's second segment, if its tiles reach one, is prepared at the start with the first
  const int second_seg = (t_end > t_begin && (t_end - 1) / p.Lt > it.seg) ? it.seg + 1 : -1;
  if (it.rem > 0) prep(cur_seg, false, second_seg);
  int s = 0;           // stage of the current step
  uint32_t phase = 0;  // parity of the stage's expected completion
  while (it.rem > 0) {
    const int nt = it.nt(Lt);
    if (it.seg != cur_seg) {
      flush(cur_seg);
      reset();
      cur_seg = it.seg;
      prep(cur_seg, cur_seg == second_seg, -1);
    }
    if (!mbar_try(&full_bar[s], phase)) mbar_wait(&full_bar[s], phase, &s_abort, p.wait_tries);
    const uint8_t* st = smem + s * kStageBytes;
    const int rel = it.lt * kTileTok + sbase;          // this slice's first token in the segment
    const bool quad_on = tl < nt && L > rel - 32 * jw;  // the quad has real tokens in this stage
    if (quad_on) {
      int lim = L - rel;                                // real tokens of this slice (may be <= 0)
      lim = lim < 32 ? lim : 32;
      if (nacc >= kMaxAccStages) drain(1.0f);
      ++nacc;
      const uint32_t* kbits = reinterpret_cast<const uint32_t*>(st + kOffBits) + sbase * 4 + t;
      const float* knorm = reinterpret_cast<const float*>(st + kOffNorm) + sbase;
      const float* kcinv = reinterpret_cast<const float*>(st + kOffCinv) + sbase;
      const uint32_t* vsm = reinterpret_cast<const uint32_t*>(st + kOffSm) + sbase * 4 + t;
      // ---------------- scores of head t for tokens 16 kk + g + 8 e of the slice
      float s2[2][2], sc[2][2], mn[2][2];
      bool rare = false;
      #pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        int d[4];
        score_tile(d, kbits[(16 * kk + g) * 4], kbits[(16 * kk + g + 8) * 4], bq);
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tt = 16 * kk + g + 8 * e;
          const bool valid = tt < lim && hv_t;
          const float nc = __fmul_rn(knorm[tt], kcinv[tt]);
          const float dot = __fmaf_rn(c1_t, static_cast<float>(d[2 * e]), __fmaf_rn(c2_t, static_cast<float>(d[2 * e + 1]), c0_t));
          s2[kk][e] = valid ? __fmul_rn(dot, nc) : -INFINITY;
          if constexpr (PROBE) {
            if (valid) {
              const int pb = cur_seg / c.Hkv, pkvh = cur_seg - pb * c.Hkv;
              const int64_t o = (static_cast<int64_t>(pb) * p.Hq + pkvh * GA + HB + t) * c.cap + rel + tt;
              p.probe_A[o] = d[2 * e];
              p.probe_Bc[o] = d[2 * e + 1];
              p.probe_s[o] = s2[kk][e];
            }
          }
          const uint32_t smw = vsm[tt * 4];  // (scale, min) of group t; zeros past the end of the cache
          sc[kk][e] = __half2float(__ushort_as_half(static_cast<unsigned short>(smw & 0xffffu)));
          mn[kk][e] = tt < lim ? __half2float(__ushort_as_half(static_cast<unsigned short>(smw >> 16))) : 0.0f;
        }
      }
      rare = (fmaxf(fmaxf(s2[0][0], s2[0][1]), fmaxf(s2[1][0], s2[1][1])) > thr_t) |
             (fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1])) > smax_t);
      // ---------------- rare path (quad-uniform): raise a head's reference maximum or a group's scale
      // bound.  The barrier also tells that the quad's warps are done with the weight buffer.
      if (named_bar_or(2 + qd, 128, rare)) {
        float mx = fmaxf(fmaxf(s2[0][0], s2[0][1]), fmaxf(s2[1][0], s2[1][1]));
        float sx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        #pragma unroll
        for (int m = 4; m <= 16; m <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
          sx = fmaxf(sx, __shfl_xor_sync(kFull, sx, m));
        }
        if (g == 0) {
          s_xchg[qd][jw][t] = mx;
          s_xchg[qd][jw][4 + t] = sx;
        }
        named_bar(2 + qd, 128);
        #pragma unroll
        for (int o = 1; o < 4; ++o) {
          mx = fmaxf(mx, s_xchg[qd][jw ^ o][t]);
          sx = fmaxf(sx, s_xchg[qd][jw ^ o][4 + t]);
        }
        float alpha[4];
        bool changed = false;
        int E_new[4];
        #pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float mh = __shfl_sync(kFull, mx, h);  // lane h has t = h
          const float sh = __shfl_sync(kFull, sx, h);
          alpha[h] = 1.0f;
          if (mh > m_w[h] + static_cast<float>(kTau)) {  // quad-uniform
            alpha[h] = (m_w[h] == kNoMax) ? 0.0f : ex2(m_w[h] - mh);
            m_w[h] = mh;
            changed = true;
          }
          E_new[h] = E_w[h];
          if (sh > smax_w[h]) {  // quad-uniform; group h
            const int k = ilog2_pos(sh);
            smax_w[h] = exp2i(k + 1 + kScaleRoom);  // W = p scale 2^E < 2^kTau 2^(k+1+room) 2^E = 2^32
            E_new[h] = 31 - kTau - kScaleRoom - k;
            changed |= E_new[h] != E_w[h];
          }
        }
        if (changed) {
          drain(sel4(alpha, hh));
          #pragma unroll
          for (int h = 0; h < 4; ++h) E_w[h] = E_new[h];
        }
        l_t = __fmul_rn(l_t, sel4(alpha, t));
        #pragma unroll
        for (int h = 0; h < 4; ++h) mid[h] = __fmul_rn(mid[h], alpha[h]);
        m_t = sel4(m_w, t);
        thr_t = m_t + static_cast<float>(kTau);
        s2e_t = exp2i(sel4(E_w, t));
        smax_t = sel4(smax_w, t);
      }
      // ---------------- probabilities of head t, then every head's p for this lane's tokens
      float ph[2][2][4];
      #pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pr = ex2(s2[kk][e] - m_t);  // -inf for invalid tokens and absent heads -> 0
          l_t = __fadd_rn(l_t, pr);
          #pragma unroll
          for (int h = 0; h < 4; ++h) ph[kk][e][h] = (h < G) ? __shfl_sync(kFull, pr, (lane & ~3) | h) : 0.0f;
        }
      // ---------------- weights of group t: W = rint(p scale 2^E + d) < 2^32, d a dither in [-1/2, 1/2)
      // that makes the rounding unbiased (weights of a long tail far below the maximum are fractions
      // of a unit, which plain rounding would send to zero together)
      // 2^23 + (top byte of the lane's hash for this slice) as a float, then / 256 - 1/2 exactly; the
      // lane's four tokens (and all heads) share it, each draw uniform over the slices
      const uint32_t weyl = static_cast<uint32_t>(rel >> 5) * 0x9E3779B9u + weyl_c;
      const float dz = __fmaf_rn(__uint_as_float(prmt(weyl, 0x4B000000u, 0x7543)), 0x1p-8f, -32768.5f);
      #pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t W[2][4];
        #pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float s2g = __fmul_rn(sc[kk][e], s2e_t);
          #pragma unroll
          for (int h = 0; h < 4; ++h) {
            W[e][h] = __float2uint_rn(__fmaf_rn(ph[kk][e][h], s2g, dz));
            mid[h] = __fmaf_rn(ph[kk][e][h], mn[kk][e], mid[h]);
          }
        }
        uint32_t rlo[4], rhi[4];
        #pragma unroll
        for (int h = 0; h < 4; ++h) {
          rlo[h] = prmt(W[0][h], W[1][h], 0x5410);  // bytes 0, 1 of tokens g, g + 8
          rhi[h] = prmt(W[0][h], W[1][h], 0x7632);  // bytes 2, 3
        }
        stsm_x4_t8(st_addr + (kk * 8) * 128, rlo);
        stsm_x4_t8(st_addr + (kk * 8 + 1) * 128, rhi);
      }
      // ---------------- P.V: value group jw (channels 32 jw .. + 31) over the quad's 128 tokens; the
      // first slice's codes are in the stage already and load while the quad meets at the barrier
      const uint32_t ctile = smem_u32(st) + c_off;
      uint32_t bpre[2][4];
      #pragma unroll
      for (int np = 0; np < 2; ++np) ldsm_x4_u4(bpre[np], ctile + c_kx0 + np * 2048);
      named_bar(5 + qd, 128);  // the four slices' weights are in the quad's buffer
      #pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint32_t cks = ctile + (c_kx0 ^ static_cast<uint32_t>(ks << 5));
        uint32_t a[4];
        ldsm_x4(a, a_pre + ks * kWSlice);
        #pragma unroll
        for (int np = 0; np < 2; ++np) {  // n-tiles 2 np, 2 np + 1
          uint32_t b[4];
          if (ks == 0) {
            #pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = bpre[np][j];
          } else {
            ldsm_x4_u4(b, cks + np * 2048);
          }
          imma_u8(D[2 * np], a, b[0], b[1]);
          imma_u8(D[2 * np + 1], a, b[2], b[3]);
        }
      }
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

template <int G, bool PROBE, bool FULL = true>
static cudaError_t launch_t(const AttendWsParams& p, bool counters_clean, cudaStream_t stream) {
  static std::atomic<unsigned long long> configured{0};  // bit per device
  cudaError_t e = configure_smem(reinterpret_cast<const void*>(attend_ws_kernel<G, PROBE, FULL>), kSmemBytes,
                                 &configured);
  if (e != cudaSuccess) return e;
  if (!counters_clean) {
    e = cudaMemsetAsync(p.counters, 0, sizeof(unsigned) * p.c.B * p.c.Hkv, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(attend_ws_kernel<G, PROBE, FULL>, dim3(p.ncta), dim3(kBlock), kSmemBytes, stream, p);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The code plane as a 3-D tensor of 4-bit elements: [tiles][128 channels][128 tokens], one box per
// tile.  Host-only (no device work); the driver function is looked up once through the runtime.
static cudaError_t encode_codes_map(CUtensorMap* map, const uint32_t* v_codes, int64_t tiles) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) return e != cudaSuccess ? e : cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kTileTok), 128, static_cast<cuuint64_t>(tiles)};
  const cuuint64_t strides[2] = {kTileTok / 2, kTileTok / 2 * 128};  // bytes: one channel row, one tile
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(kTileTok), 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<uint32_t*>(v_codes), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace ws
}  // namespace kv1b

using namespace kv1b;

// Any G up to KV1B_MAX_GROUP: launches of at most 4 query heads each (one for G <= 4), every one
// streaming the whole cache -- the kernel is bound by its per-stage work, not by HBM, so a fused
// 8-head form would not be faster than two 4-head launches.
bool kv1b_ws_supported(int32_t G) { return G >= 1 && G <= KV1B_MAX_GROUP; }
int kv1b_ws_template_group(int32_t G) { return G >= 3 ? 4 : G; }

// CTAs = SMs (fewer when there are fewer tiles); T, Lt in 128-token tiles; partial rows per
// segment = the most CTAs one segment can touch.
void kv1b_ws_plan(int32_t B, int32_t Hkv, int64_t L, int num_sms, int64_t* T, int64_t* Lt, int* ncta,
                  int* max_pieces) {
  const int64_t lt = (L + ws::kTileTok - 1) / ws::kTileTok;
  const int64_t tot = static_cast<int64_t>(B) * Hkv * lt;
  int n = num_sms;
  if (tot < n) n = static_cast<int>(tot > 0 ? tot : 1);
  *T = tot;
  *Lt = lt;
  *ncta = n;
  *max_pieces = tot > 0 ? static_cast<int>((lt * n + tot - 1) / tot + 1) : 1;
}

cudaError_t kv1b_launch_attend_ws(AttendWsParams& p, int32_t G, bool counters_clean, cudaStream_t stream,
                                  bool probe) {
  const int64_t tiles = static_cast<int64_t>(p.c.B) * p.c.Hkv * (p.c.cap / ws::kTileTok);
  const cudaError_t e = ws::encode_codes_map(&p.codes_map, p.c.v_codes, tiles);
  if (e != cudaSuccess) return e;
  if (p.wait_tries < 1 || G < 1 || G > KV1B_MAX_GROUP) return cudaErrorInvalidValue;
  if (probe && (!p.probe_A || !p.probe_Bc || !p.probe_s)) return cudaErrorInvalidValue;
  p.G_all = G;
  // launches of up to 4 heads; the merge counters are zero after each (the first may clear them)
  for (int base = 0; base < G; base += 4) {
    const int nh = G - base < 4 ? G - base : 4;
    const int tg = kv1b_ws_template_group(nh);
    p.head_base = base;
    p.heads = nh;
    const bool clean = counters_clean || base > 0;
    cudaError_t e2;
    switch (tg * 2 + (probe ? 1 : 0) + (nh < tg ? 16 : 0)) {
      case 2: e2 = ws::launch_t<1, false>(p, clean, stream); break;
      case 4: e2 = ws::launch_t<2, false>(p, clean, stream); break;
      case 8: e2 = ws::launch_t<4, false>(p, clean, stream); break;
      case 3: e2 = ws::launch_t<1, true>(p, clean, stream); break;
      case 5: e2 = ws::launch_t<2, true>(p, clean, stream); break;
      case 9: e2 = ws::launch_t<4, true>(p, clean, stream); break;
      case 24: e2 = ws::launch_t<4, false, false>(p, clean, stream); break;  // 3 heads in 4 slots
      case 25: e2 = ws::launch_t<4, true, false>(p, clean, stream); break;
      default: e2 = cudaErrorInvalidValue;
    }
    if (e2 != cudaSuccess) return e2;
  }
  return cudaSuccess;
}
