// kv1b_encode.cu -- cache initialisation and the encode/append kernel.
//
// Keys ("RaBitQCache", abstract / core idea: randomised rotation, then binary quantisation;
// "H1B-KV", key design: a 1-bit sketch by random projection): y = H (D (.) k), one sign bit per
// channel, N = ||k|| and 1/C = 128 N / sum|y_i| for RaBitQ's unbiased estimator.
// Values ("H1B-KV", key design: 4-bit linear quantisation): groups of 32 channels, fp16 min
// rounded down, fp16 scale the smallest with 15 scale >= range, codes = round-half-up.
#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) draws the rotation signs: D_i = -1 iff the top bit
// of the i-th output is set; round r of a stronger rotation takes outputs 128 r .. 128 r + 127 of the
// same stream, and the rounds past `rounds` are zero.  One thread; runs once per cache.
__global__ void init_kernel(uint64_t seed, int rounds, float* signs, int32_t* lengths, int32_t batch,
                            int32_t* status) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    uint64_t st = seed;
    for (int i = 0; i < KV1B_MAX_ROUNDS * kD; ++i) {
      if (i >= rounds * kD) {
        signs[i] = 0.0f;
        continue;
      }
      st += 0x9E3779B97F4A7C15ull;
      uint64_t z = st;
      z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
      z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
      z ^= (z >> 31);
      signs[i] = (z >> 63) ? -1.0f : 1.0f;
    }
    *status = 0;
  }
  if (blockIdx.x == 0 && threadIdx.x < batch) lengths[threadIdx.x] = 0;
}

// One block per (16-token tile touched by the append, kv-head, sequence); warp r < 16 encodes the
// key of tile slot r and warp 16 + r its value, so the two chains run side by side.  Keys and v_sm
// are token-major and written directly; the 4-bit codes of the tile are staged in shared memory and
// then written as whole 32-bit words of the channel-major code plane (read-modify-write keeps the
// nibbles of tokens already in the tile; the old words are read at the start).
__global__ void __launch_bounds__(1024) encode_kernel(const EncodeParams p) {
  __shared__ uint8_t codes[16][kD];
  __shared__ int s_new[16];
  pdl_wait();  // every block, before any memory access: the inputs may come from the previous kernel
  const int b = blockIdx.z, h = blockIdx.y;
  const int64_t L0 = p.L0[b];
  const int64_t first_tile = L0 / 16, last_tile = (L0 + p.n_new - 1) / 16;
  const int64_t tile = first_tile + blockIdx.x;
  if (tile > last_tile) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp & 15;
  const bool value_warp = warp >= 16;
  const int64_t pos = tile * 16 + slot;
  const bool is_new = pos >= L0 && pos < L0 + p.n_new;
  if (lane == 0 && !value_warp) s_new[slot] = is_new;
  const int64_t head_base = (static_cast<int64_t>(b) * p.Hkv + h) * p.cap;  // token index base
  // the code words this block rewrites: thread = (channel, half of the 16 tokens)
  uint32_t* dst = nullptr;
  uint32_t old_word = 0u;
  if (threadIdx.x < 256) {
    const int ch = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int64_t seg = static_cast<int64_t>(b) * p.Hkv + h;
    dst = p.v_codes + ((seg * (p.cap / 128) + tile / 8) * kD + ch) * 16 + (tile & 7) * 2 + half;
    old_word = *dst;
  }

  if (is_new && !value_warp) {
    const int64_t t = pos - L0;
    const int64_t row = static_cast<int64_t>(b) * p.sb + t * p.st + static_cast<int64_t>(h) * p.sh;
    int flags = 0;
    // ---- key sketch
    float x[4], sq[4], y[4], ab[4];
    load4(p.k, row + 4 * lane, p.dtype, x);
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      sq[r] = __fmul_rn(x[r], x[r]);
      if (!isfinite(x[r])) flags |= KV1B_STATUS_NONFINITE;
      y[r] = x[r];
    }
    const float nrm = __fsqrt_rn(tree_sum128(sq));
    rotate_rounds(y, p.signs);
    uint32_t nib = 0;
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      nib |= static_cast<uint32_t>(y[r] >= 0.0f) << r;
      ab[r] = fabsf(y[r]);
    }
    const uint32_t word = pack_word(nib);
    const float sabs = tree_sum128(ab);
    const float cinv = (sabs > 0.0f) ? __fdiv_rn(__fmul_rn(static_cast<float>(kD), nrm), sabs) : 1.0f;
    if ((lane & 7) == 0) p.k_bits[(head_base + pos) * 4 + (lane >> 3)] = word;
    if (lane == 0) {
      p.k_norm[head_base + pos] = nrm;
      p.k_cinv[head_base + pos] = cinv;
    }
    flags = static_cast<int>(__reduce_or_sync(kFull, static_cast<unsigned>(flags)));
    if (lane == 0 && flags) atomicOr(p.status, flags);
  }
  if (is_new && value_warp) {
    const int64_t t = pos - L0;
    const int64_t row = static_cast<int64_t>(b) * p.sb + t * p.st + static_cast<int64_t>(h) * p.sh;
    int flags = 0;
    // ---- value codes
    float v[4];
    load4(p.v, row + 4 * lane, p.dtype, v);
    float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
    float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
    #pragma unroll
    for (int m = 1; m <= 4; m <<= 1) {  // reduce over the 8 lanes of this 32-channel group
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    }
    int sat = 0;
    #pragma unroll
    for (int r = 0; r < 4; ++r)
      if (!isfinite(v[r])) flags |= KV1B_STATUS_NONFINITE;
    const uint32_t min_bits = half_round_down(mn, &sat);
    const uint32_t scale_bits =
        half_scale_up(mx, __half2float(__ushort_as_half(static_cast<unsigned short>(min_bits))), &sat);
    if (sat) flags |= KV1B_STATUS_FP16_SATURATED;
    const float sf = __half2float(__ushort_as_half(static_cast<unsigned short>(scale_bits)));
    const float mf = __half2float(__ushort_as_half(static_cast<unsigned short>(min_bits)));
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      int c = 0;
      if (sf > 0.0f) {
        const float fl = floorf(__fadd_rn(__fdiv_rn(__fsub_rn(v[r], mf), sf), 0.5f));
        c = !(fl > 0.0f) ? 0 : (fl >= 15.0f ? 15 : static_cast<int>(fl));
      }
      codes[slot][4 * lane + r] = static_cast<uint8_t>(c);
    }
    if ((lane & 7) == 0) p.v_sm[(head_base + pos) * 4 + (lane >> 3)] = scale_bits | (min_bits << 16);
    flags = static_cast<int>(__reduce_or_sync(kFull, static_cast<unsigned>(flags)));
    if (lane == 0 && flags) atomicOr(p.status, flags);
  }
  __syncthreads();
  // ---- write the tile's codes: thread = (channel, half of the 16 tokens); the 8 tokens' nibbles
  // form one 32-bit word of the channel's 64-byte row in its 128-token tile (nibble j = token j
  // of the 8), read-modify-write keeps the nibbles of tokens already in the cache.
  if (threadIdx.x < 256) {
    const int ch = threadIdx.x >> 1, half = threadIdx.x & 1;
    uint32_t w = old_word;
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (s_new[8 * half + j]) {
        const uint32_t c = codes[8 * half + j][ch];
        w = (w & ~(0xfu << (4 * j))) | (c << (4 * j));
      }
    }
    *dst = w;
  }
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x < p.B)
    p.lengths[threadIdx.x] = static_cast<int32_t>(p.L0[threadIdx.x] + p.n_new);
}

// ---------------------------------------------------------------------------------------------
// Prefill form (appends of many tokens): one warp per 8-token group of one (sequence, kv-head) --
// the tokens whose codes share one 32-bit word of every channel row -- encoding its tokens one after
// another, the next token's rows in flight while the current one is encoded.
//  - Key: lane l holds channels l + 32 r (r = 0..3).  The fixed tree sums take their two widest
//    levels (h = 64, 32) inside the lane, the rotation its two widest stages (h = 32, 64), and sign
//    word r is the warp's ballot of channel l + 32 r: bit i of word r = channel 32 r + i.  The
//    cross-lane butterfly is one fused multiply-add, sgn * x + partner (sgn = -1 on the upper lane):
//    a single rounding of a + c or a - c, the same value as the sum or difference.
//  - Value: lane l holds channels 4 l .. 4 l + 3 (a 32-channel group on 8 lanes), as the decode form.
//  - Codes: each lane keeps its 4 channels' code words of the group in registers and writes them once
//    (nibbles of tokens outside the append are kept from the old word).
// Every stored bit, code and scalar equals the decode form's (the same operations in the same order).
constexpr int kPrefillWarps = 4;
constexpr int kPrefillMinTokens = 64;  // appends of at least this many tokens per sequence take the prefill form
constexpr int kPrefillGroup = 8;  // tokens per code word

// Fixed pairwise tree over the 128 channels in the strided layout (lane l: channels l + 32 r):
// h = 64 and 32 inside the lane, then h = 16 .. 1 across lanes.  Returns a[0] on every lane.
__device__ __forceinline__ float tree_sum128_strided(const float a[4]) {
  float x = __fadd_rn(__fadd_rn(a[0], a[2]), __fadd_rn(a[1], a[3]));  // h = 64 (r, r + 2), then h = 32
  #pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x = __fadd_rn(x, __shfl_down_sync(kFull, x, off));
  return __shfl_sync(kFull, x, 0);
}

// One round y <- H (D (.) y) in the strided layout: stages h = 1 .. 16 across lanes, 32 and 64 inside.
__device__ __forceinline__ void rotate128_strided(float x[4], const float sg[4]) {
  const int lane = threadIdx.x & 31;
  #pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = (sg[r] < 0.0f) ? -x[r] : x[r];
  #pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    const float sgn = (lane & h) ? -1.0f : 1.0f;
    #pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = __fmaf_rn(sgn, x[r], __shfl_xor_sync(kFull, x[r], h));
  }
  const float a0 = __fadd_rn(x[0], x[1]), a1 = __fsub_rn(x[0], x[1]);  // h = 32: (r, r + 1)
  const float a2 = __fadd_rn(x[2], x[3]), a3 = __fsub_rn(x[2], x[3]);
  x[0] = __fadd_rn(a0, a2);  // h = 64: (r, r + 2)
  x[2] = __fsub_rn(a0, a2);
  x[1] = __fadd_rn(a1, a3);
  x[3] = __fsub_rn(a1, a3);
}

// Channels l + 32 r (r = 0..3) of an fp32 / bf16 / fp16 row as fp32.
__device__ __forceinline__ void load_strided(const void* base, int64_t off, int dtype, float x[4]) {
  const int lane = threadIdx.x & 31;
  #pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t o = off + lane + 32 * r;
    if (dtype == KV1B_DTYPE_F32) {
      x[r] = __ldg(static_cast<const float*>(base) + o);
    } else {
      const uint32_t h = __ldg(static_cast<const unsigned short*>(base) + o);
      x[r] = dtype == KV1B_DTYPE_BF16 ? __uint_as_float(h << 16)
                                      : __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
    }
  }
}

__global__ void __launch_bounds__(32 * kPrefillWarps) encode_prefill_kernel(const EncodeParams p) {
  pdl_wait();
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x < p.B)
    p.lengths[threadIdx.x] = static_cast<int32_t>(p.L0[threadIdx.x] + p.n_new);
  const int64_t L0 = p.L0[b], L1 = L0 + p.n_new;
  const int64_t g0 = ((L0 >> 3) + static_cast<int64_t>(blockIdx.x) * kPrefillWarps + warp) * kPrefillGroup;
  if (g0 >= L1) return;  // warp-uniform
  const int64_t t_lo = g0 > L0 ? g0 : L0, t_hi = g0 + kPrefillGroup < L1 ? g0 + kPrefillGroup : L1;
  const int64_t tok0 = (static_cast<int64_t>(b) * p.Hkv + h) * p.cap + t_lo;  // first token's index in the planes
  // rotation signs of the lane's key channels, round 0; later rounds (rare) are read per token
  float sg[4];
  #pragma unroll
  for (int r = 0; r < 4; ++r) sg[r] = p.signs[lane + 32 * r];
  const bool rotate = p.signs[0] != 0.0f;
  const int rounds = !rotate ? 0 : (p.signs[kD] == 0.0f ? 1 : (p.signs[2 * kD] == 0.0f ? 2 : 3));
  uint32_t cw[4] = {0u, 0u, 0u, 0u};  // code words of channels 4 lane + j for this group
  int flags = 0;
  const int n = static_cast<int>(t_hi - t_lo);
  int64_t row = static_cast<int64_t>(b) * p.sb + (t_lo - L0) * p.st + static_cast<int64_t>(h) * p.sh;
  uint32_t* kbits = p.k_bits + tok0 * 4;
  float* knorm = p.k_norm + tok0;
  float* kcinv = p.k_cinv + tok0;
  uint32_t* vsm = p.v_sm + tok0 * 4 + (lane >> 3);
  float kx[4], vx[4];
  load_strided(p.k, row, p.dtype, kx);
  load4(p.v, row + 4 * lane, p.dtype, vx);
  #pragma unroll 1
  for (int i = 0; i < n; ++i) {
    float x[4], v[4];
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      x[r] = kx[r];
      v[r] = vx[r];
    }
    row += p.st;
    if (i + 1 < n) {  // the next token's rows in flight
      load_strided(p.k, row, p.dtype, kx);
      load4(p.v, row + 4 * lane, p.dtype, vx);
    }
    // ---- key sketch: N, rotation, sign words, 1/C
    float sq[4], ab[4];
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      sq[r] = __fmul_rn(x[r], x[r]);
      flags |= isfinite(x[r]) ? 0 : KV1B_STATUS_NONFINITE;
    }
    const float nrm = __fsqrt_rn(tree_sum128_strided(sq));
    if (rotate) {
      rotate128_strided(x, sg);
      #pragma unroll 1
      for (int rd = 1; rd < rounds; ++rd) {
        float s2[4];
        #pragma unroll
        for (int r = 0; r < 4; ++r) s2[r] = p.signs[rd * kD + lane + 32 * r];
        rotate128_strided(x, s2);
      }
    }
    uint32_t word[4];
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      word[r] = __ballot_sync(kFull, x[r] >= 0.0f);
      ab[r] = fabsf(x[r]);
    }
    const float sabs = tree_sum128_strided(ab);
    const float cinv = (sabs > 0.0f) ? __fdiv_rn(__fmul_rn(static_cast<float>(kD), nrm), sabs) : 1.0f;
    if (lane < 4) kbits[lane] = lane == 0 ? word[0] : (lane == 1 ? word[1] : (lane == 2 ? word[2] : word[3]));
    if (lane == 0) {
      *knorm = nrm;
      *kcinv = cinv;
    }
    kbits += 4;
    ++knorm;
    ++kcinv;
    // ---- value codes: group lane >> 3
    float mn = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
    float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
    #pragma unroll
    for (int m = 1; m <= 4; m <<= 1) {  // reduce over the 8 lanes of this 32-channel group
      mn = fminf(mn, __shfl_xor_sync(kFull, mn, m));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
    }
    int sat = 0;
    #pragma unroll
    for (int r = 0; r < 4; ++r) flags |= isfinite(v[r]) ? 0 : KV1B_STATUS_NONFINITE;
    const uint32_t min_bits = half_round_down(mn, &sat);
    const float mf = __half2float(__ushort_as_half(static_cast<unsigned short>(min_bits)));
    const uint32_t scale_bits = half_scale_up_fast(mx, mf, &sat);
    flags |= sat ? KV1B_STATUS_FP16_SATURATED : 0;
    const float sf = __half2float(__ushort_as_half(static_cast<unsigned short>(scale_bits)));
    const float rs = __frcp_rn(sf);  // correctly rounded; +inf for a zero scale (codes 0 below)
    const uint32_t nsh = 4u * static_cast<uint32_t>((t_lo + i) & 7);
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      // code = clamp(floor(fl(fl(v - min) / scale) + 0.5), 0, 15), 0 for a zero scale
      const float fl = floorf(__fadd_rn(div_markstein(__fsub_rn(v[r], mf), sf, rs), 0.5f));
      const float cl = sf > 0.0f ? fminf(fmaxf(fl, 0.0f), 15.0f) : 0.0f;  // NaN -> 0
      cw[r] |= (__float_as_uint(__fadd_rn(cl, 8388608.0f)) & 0xFu) << nsh;  // the integer in the mantissa
    }
    if ((lane & 7) == 0) *vsm = scale_bits | (min_bits << 16);
    vsm += 4;
  }
  // ---- code words: word (g0 & 127) / 8 of channel rows 4 lane + j in the group's 128-token tile;
  // nibbles of tokens outside [t_lo, t_hi) keep the old word's
  const int64_t seg = static_cast<int64_t>(b) * p.Hkv + h;
  uint32_t* dst = p.v_codes + ((seg * (p.cap / 128) + (g0 >> 7)) * kD + 4 * lane) * 16 + ((g0 & 127) >> 3);
  const int n0 = static_cast<int>(t_lo - g0), n1 = static_cast<int>(t_hi - g0);
  const uint32_t keep = (n0 == 0 && n1 == kPrefillGroup) ? 0u : ~(((n1 == 8 ? 0u : (~0u << (4 * n1))) ^ ~0u) & (~0u << (4 * n0)));
  #pragma unroll
  for (int j = 0; j < 4; ++j) dst[16 * j] = keep ? ((dst[16 * j] & keep) | cw[j]) : cw[j];
  flags = static_cast<int>(__reduce_or_sync(kFull, static_cast<unsigned>(flags)));
  if (lane == 0 && flags) atomicOr(p.status, flags);
}

}  // namespace kv1b

using namespace kv1b;

cudaError_t kv1b_launch_init(uint64_t seed, int32_t rounds, float* signs, int32_t* lengths, int32_t batch,
                             int32_t* status,
                             cudaStream_t stream) {
  init_kernel<<<1, 64, 0, stream>>>(seed, rounds, signs, lengths, batch, status);
  return cudaGetLastError();
}

cudaError_t kv1b_launch_encode(const EncodeParams& p, int64_t max_tiles, cudaStream_t stream) {
  if (p.n_new >= kPrefillMinTokens) {  // prefill: one warp per 8-token group
    int64_t groups = 0;
    for (int b = 0; b < p.B; ++b) {
      const int64_t g = ((p.L0[b] + p.n_new - 1) >> 3) - (p.L0[b] >> 3) + 1;
      groups = g > groups ? g : groups;
    }
    const dim3 grid(static_cast<unsigned>((groups + kPrefillWarps - 1) / kPrefillWarps), p.Hkv, p.B);
    return launch_pdl(encode_prefill_kernel, grid, dim3(32 * kPrefillWarps), 0, stream, p);
  }
  const dim3 grid(static_cast<unsigned>(max_tiles), p.Hkv, p.B);
  return launch_pdl(encode_kernel, grid, dim3(1024), 0, stream, p);
}
