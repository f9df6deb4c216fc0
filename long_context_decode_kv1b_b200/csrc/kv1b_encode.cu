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
  pdl_launch_dependents();  // the attend that usually follows sets up on the SMs this grid leaves free
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
// the tokens whose codes share one 32-bit word of every channel row -- with 4 lanes per token
// (lane = 4 tau + j: token tau of the group, part j) and all 8 tokens at once.
//  - Key: lane j holds channels j + 4 r (r = 0..31).  The fixed tree sums take levels h = 64 .. 4
//    inside the lane (pairs r, r + h / 4) and h = 2, 1 across the token's lanes; the rotation takes
//    stages h = 1, 2 across them (one fused multiply-add, sgn * x + partner: a single rounding of
//    a + c or a - c) and h = 4 .. 64 inside (pairs r, r + h / 4), in the order h = 1, 2, 4, ..., 64.
//    Sign word w of a token: bit i is channel 32 w + i, i.e. lane i & 3 at r = 8 w + (i >> 2) -- one
//    ballot per r gives every token's bits, and lane j assembles word j of its token.
//  - Value: lane j holds value group j (channels 32 j .. 32 j + 31): min / max and the binary16
//    searches inside the lane; codes from one correctly rounded reciprocal per group and Markstein's
//    correction, packed 8 per word token-major, then an 8 x 8 transpose of nibbles across the group's
//    8 token lanes turns them into the channel-major code words (nibble tau = token tau).
// Every stored bit, code and scalar equals the decode form's (the same operations in the same order).
constexpr int kPrefillWarps = 4;
constexpr int kPrefillMinTokens = 64;  // appends of at least this many tokens per sequence take the prefill form
constexpr int kPrefillGroup = 8;       // tokens per code word

// 32-bit mask of the rotation signs of lane j's key channels j + 4 r (bit r set: D = -1) for round rd:
// four coalesced loads, one ballot each (bit l of ballot i = channel 32 i + l), then the stride-4
// bits j, j + 4, .., j + 28 of each ballot packed into byte i.
__device__ __forceinline__ uint32_t sign_mask(const float* signs, int rd, int j) {
  const int lane = threadIdx.x & 31;
  uint32_t m = 0u;
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t x = (__ballot_sync(kFull, __ldg(signs + rd * kD + 32 * i + lane) < 0.0f) >> j) & 0x11111111u;
    x = (x | (x >> 3)) & 0x03030303u;
    x = (x | (x >> 6)) & 0x000F000Fu;
    x = (x | (x >> 12)) & 0x000000FFu;
    m |= x << (8 * i);
  }
  return m;
}

// One round y <- H (D (.) y): stages h = 1, 2 across the token's 4 lanes, h = 4 .. 64 inside.
__device__ __forceinline__ void rotate_q4(float x[32], uint32_t smask, int j) {
  #pragma unroll
  for (int r = 0; r < 32; ++r)  // D: flip the sign bit where the mask has a 1
    x[r] = __int_as_float(__float_as_int(x[r]) ^ static_cast<int>((smask << (31 - r)) & 0x80000000u));
  #pragma unroll
  for (int h = 1; h <= 2; h <<= 1) {
    const float sgn = (j & h) ? -1.0f : 1.0f;  // the lane of the pair's upper element forms a - c
    #pragma unroll
    for (int r = 0; r < 32; ++r) x[r] = __fmaf_rn(sgn, x[r], __shfl_xor_sync(kFull, x[r], h));
  }
  #pragma unroll
  for (int hr = 1; hr <= 16; hr <<= 1) {
    #pragma unroll
    for (int r = 0; r < 32; ++r) {
      if (r & hr) continue;
      const float a = x[r], c = x[r + hr];
      x[r] = __fadd_rn(a, c);
      x[r + hr] = __fsub_rn(a, c);
    }
  }
}

// Fixed pairwise tree over the token's 128 channels (lane j: channels j + 4 r); h = 64 .. 4 inside
// the lane, 2 and 1 across lanes.  Returns the sum on each of the token's lanes.  a is overwritten.
__device__ __forceinline__ float tree_sum_q4(float a[32]) {
  #pragma unroll
  for (int hr = 16; hr >= 1; hr >>= 1)
    #pragma unroll
    for (int r = 0; r < hr; ++r) a[r] = __fadd_rn(a[r], a[r + hr]);
  float x = a[0];
  x = __fadd_rn(x, __shfl_xor_sync(kFull, x, 2));  // h = 2: lanes j < 2 add lane j + 2
  x = __fadd_rn(x, __shfl_xor_sync(kFull, x, 1));  // h = 1: lane 0 adds lane 1
  return __shfl_sync(kFull, x, (threadIdx.x & 31) & ~3);
}

// Element types of the K / V rows (the kernel is compiled once per type).
template <int DT> struct Elem;
template <> struct Elem<KV1B_DTYPE_F32> {
  typedef float T;
  static __device__ __forceinline__ float get(float x) { return x; }
};
template <> struct Elem<KV1B_DTYPE_BF16> {
  typedef unsigned short T;
  static __device__ __forceinline__ float get(unsigned short x) { return __uint_as_float(static_cast<uint32_t>(x) << 16); }
};
template <> struct Elem<KV1B_DTYPE_F16> {
  typedef unsigned short T;
  static __device__ __forceinline__ float get(unsigned short x) { return __half2float(__ushort_as_half(x)); }
};

// sum over i = 0..7 of (0x4B000000 << 4 i) modulo 2^32: the exponent bits of 2^23 + code, shifted
// into each nibble's place (only i = 0, 1 keep any bits)
constexpr uint32_t kMagicPacked = 0x4B000000u + (0x4B000000u << 4);
constexpr int kPrefillMaxGroupsPerWarp = 4;  // 8-token groups a warp encodes one after another, at most

template <int DT>
__global__ void __launch_bounds__(32 * kPrefillWarps, 4) encode_prefill_kernel(const EncodeParams p) {
  typedef typename Elem<DT>::T T;
  pdl_wait();
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tau = lane >> 2, j = lane & 3;
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x < p.B)
    p.lengths[threadIdx.x] = static_cast<int32_t>(p.L0[threadIdx.x] + p.n_new);
  const int64_t L0 = p.L0[b], L1 = L0 + p.n_new;
  const int gpw = p.groups_per_warp;
  const int64_t gw = ((L0 >> 3) + (static_cast<int64_t>(blockIdx.x) * kPrefillWarps + warp) * gpw) *
                     kPrefillGroup;  // the warp's first group
  if (gw >= L1) return;  // warp-uniform
  // rotation: round 0's sign mask of this lane's key channels (the rounds and their masks are the
  // same for every token)
  const bool rotate = p.signs[0] != 0.0f;
  const int rounds = !rotate ? 0 : (p.signs[kD] == 0.0f ? 1 : (p.signs[2 * kD] == 0.0f ? 2 : 3));
  const uint32_t smask0 = sign_mask(p.signs, 0, j);
  const int64_t seg = static_cast<int64_t>(b) * p.Hkv + h;
  int flags = 0;
  #pragma unroll 1
  for (int gi = 0; gi < gpw; ++gi) {
    const int64_t g0 = gw + gi * kPrefillGroup;
    if (g0 >= L1) break;  // warp-uniform
    const int64_t pos = g0 + tau;
    const bool full = g0 >= L0 && g0 + kPrefillGroup <= L1;  // warp-uniform: every token of the group is new
    const bool on = pos >= L0 && pos < L1;                   // this token is appended now (its 4 lanes agree)
    const int64_t rowk = static_cast<int64_t>(b) * p.sb + (pos - L0) * p.st + static_cast<int64_t>(h) * p.sh;
    const T* krow = static_cast<const T*>(p.k) + rowk + j;       // channels j + 4 r at krow[4 r]
    const int64_t tok = seg * p.cap + pos;                       // the token's index in the planes

    // ---- key sketch: N, rotation, sign words, 1/C
    {
      float x[32], a[32];
      if (full) {
        #pragma unroll
        for (int r = 0; r < 32; ++r) x[r] = Elem<DT>::get(__ldg(krow + 4 * r));
      } else {
        #pragma unroll
        for (int r = 0; r < 32; ++r) x[r] = on ? Elem<DT>::get(__ldg(krow + 4 * r)) : 0.0f;
      }
      bool fin = true;
      #pragma unroll
      for (int r = 0; r < 32; ++r) {
        fin &= isfinite(x[r]);
        a[r] = __fmul_rn(x[r], x[r]);
      }
      flags |= fin ? 0 : KV1B_STATUS_NONFINITE;
      const float nrm = __fsqrt_rn(tree_sum_q4(a));
      if (rotate) {  // a zero first sign: no rotation (as the decode form)
        rotate_q4(x, smask0, j);
        #pragma unroll 1
        for (int rd = 1; rd < rounds; ++rd) rotate_q4(x, sign_mask(p.signs, rd, j), j);
      }
      uint32_t word = 0u;  // sign word j of this lane's token
      #pragma unroll
      for (int r = 0; r < 32; ++r) {
        const uint32_t bal = __ballot_sync(kFull, x[r] >= 0.0f);  // bit 4 tau' + j' = channel j' + 4 r of token tau'
        if ((r >> 3) == j) word |= ((bal >> (4 * tau)) & 0xFu) << (4 * (r & 7));
        a[r] = fabsf(x[r]);
      }
      const float sabs = tree_sum_q4(a);
      const float cinv = (sabs > 0.0f) ? __fdiv_rn(__fmul_rn(static_cast<float>(kD), nrm), sabs) : 1.0f;
      if (on) {
        p.k_bits[tok * 4 + j] = word;
        if (j == 0) {
          p.k_norm[tok] = nrm;
          p.k_cinv[tok] = cinv;
        }
      }
    }

    // ---- value codes: group j
    float v[32];
    if (full) {
      #pragma unroll
      for (int q = 0; q < 8; ++q) load4(p.v, rowk + 32 * j + 4 * q, DT, v + 4 * q);
    } else {
      #pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (on) {
          load4(p.v, rowk + 32 * j + 4 * q, DT, v + 4 * q);
        } else {
          v[4 * q] = v[4 * q + 1] = v[4 * q + 2] = v[4 * q + 3] = 0.0f;
        }
      }
    }
    float mn = v[0], mx = v[0];
    bool fin = true;
    #pragma unroll
    for (int i = 0; i < 32; ++i) {
      fin &= isfinite(v[i]);
      mn = fminf(mn, v[i]);
      mx = fmaxf(mx, v[i]);
    }
    flags |= fin ? 0 : KV1B_STATUS_NONFINITE;
    int sat = 0;
    const uint32_t min_bits = half_round_down(mn, &sat);
    const float mf = __half2float(__ushort_as_half(static_cast<unsigned short>(min_bits)));
    const uint32_t scale_bits = half_scale_up_fast(mx, mf, &sat);
    flags |= (sat && on) ? KV1B_STATUS_FP16_SATURATED : 0;
    const float sf = __half2float(__ushort_as_half(static_cast<unsigned short>(scale_bits)));
    const float rs = __frcp_rn(sf);  // correctly rounded; +inf for a zero scale (codes 0 below)
    uint32_t cw[4];  // token-major: nibble i of word k = channel 32 j + 8 k + i of this token
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
      // code = clamp(floor(y), 0, 15) with y = fl(fl(v - min) / scale) + 0.5, 0 for a zero scale.
      // floor(clamp(y, 0, 15.5)) is the same integer (NaN -> 0), and adding 2^23 rounded toward
      // -inf leaves it exactly in the low mantissa bits: the float's bits are 0x4B000000 + code.
      // Shifted by 4 i and summed modulo 2^32, the eight words give the packed codes plus the
      // shifted constants, which one subtraction removes.
      uint32_t w = 0u - kMagicPacked;
      #pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float y = __fadd_rn(div_markstein(__fsub_rn(v[8 * k + i], mf), sf, rs), 0.5f);
        const float c = fminf(fmaxf(y, 0.0f), 15.5f);
        w += __float_as_uint(__fadd_rd(c, 8388608.0f)) << (4 * i);
      }
      cw[k] = (on && sf > 0.0f) ? w : 0u;  // sf NaN or 0: codes 0
    }
    if (on) p.v_sm[tok * 4 + j] = scale_bits | (min_bits << 16);
    // transpose the 8 x 8 nibbles of each word across the 8 token lanes of group j: afterwards
    // nibble tau' of lane tau's word k is the code of channel 32 j + 8 k + tau of token tau'
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t x = cw[k];
      uint32_t y = __shfl_xor_sync(kFull, x, 16);  // token tau ^ 4
      x = (tau & 4) ? ((x & 0xFFFF0000u) | (y >> 16)) : ((x & 0x0000FFFFu) | (y << 16));
      y = __shfl_xor_sync(kFull, x, 8);            // token tau ^ 2
      x = (tau & 2) ? ((x & 0xFF00FF00u) | ((y >> 8) & 0x00FF00FFu)) : ((x & 0x00FF00FFu) | ((y & 0x00FF00FFu) << 8));
      y = __shfl_xor_sync(kFull, x, 4);            // token tau ^ 1
      x = (tau & 1) ? ((x & 0xF0F0F0F0u) | ((y >> 4) & 0x0F0F0F0Fu)) : ((x & 0x0F0F0F0Fu) | ((y & 0x0F0F0F0Fu) << 4));
      cw[k] = x;
    }
    // ---- code words: word (g0 & 127) / 8 of channel rows 32 j + 8 k + tau in the group's 128-token
    // tile; nibbles of tokens outside the append keep the old word's
    uint32_t* dst = p.v_codes + ((seg * (p.cap / 128) + (g0 >> 7)) * kD + 32 * j + tau) * 16 + ((g0 & 127) >> 3);
    if (full) {
      #pragma unroll
      for (int k = 0; k < 4; ++k) dst[8 * 16 * k] = cw[k];
    } else {
      const int n0 = static_cast<int>((g0 > L0 ? g0 : L0) - g0), n1 = static_cast<int>((g0 + 8 < L1 ? g0 + 8 : L1) - g0);
      const uint32_t keep = ~(((n1 == 8 ? 0u : (~0u << (4 * n1))) ^ ~0u) & (~0u << (4 * n0)));
      #pragma unroll
      for (int k = 0; k < 4; ++k) dst[8 * 16 * k] = (dst[8 * 16 * k] & keep) | cw[k];
    }
  }
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
    // several groups per warp amortise the warp's set-up (sign masks, row bases) once there are
    // about two waves of warps at 16 resident per SM without it
    const int64_t warps = groups * p.Hkv * p.B;
    const int64_t wave2 = 2LL * 148 * 16;
    EncodeParams q = p;
    q.groups_per_warp = static_cast<int32_t>(warps >= kPrefillMaxGroupsPerWarp * wave2 ? kPrefillMaxGroupsPerWarp
                                             : (warps >= 2 * wave2 ? 2 : 1));
    const int64_t per_block = static_cast<int64_t>(kPrefillWarps) * q.groups_per_warp;
    const dim3 grid(static_cast<unsigned>((groups + per_block - 1) / per_block), p.Hkv, p.B);
    switch (p.dtype) {
      case KV1B_DTYPE_F32: return launch_pdl(encode_prefill_kernel<KV1B_DTYPE_F32>, grid, dim3(32 * kPrefillWarps), 0, stream, q);
      case KV1B_DTYPE_BF16: return launch_pdl(encode_prefill_kernel<KV1B_DTYPE_BF16>, grid, dim3(32 * kPrefillWarps), 0, stream, q);
      default: return launch_pdl(encode_prefill_kernel<KV1B_DTYPE_F16>, grid, dim3(32 * kPrefillWarps), 0, stream, q);
    }
  }
  const dim3 grid(static_cast<unsigned>(max_tiles), p.Hkv, p.B);
  return launch_pdl(encode_kernel, grid, dim3(1024), 0, stream, p);
}
