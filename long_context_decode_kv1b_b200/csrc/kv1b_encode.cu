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
    const double range = static_cast<double>(mx) - half_bits_to_double(min_bits);
    const uint32_t scale_bits = half_scale_up(range, &sat);
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

}  // namespace kv1b

using namespace kv1b;

cudaError_t kv1b_launch_init(uint64_t seed, int32_t rounds, float* signs, int32_t* lengths, int32_t batch,
                             int32_t* status,
                             cudaStream_t stream) {
  init_kernel<<<1, 64, 0, stream>>>(seed, rounds, signs, lengths, batch, status);
  return cudaGetLastError();
}

cudaError_t kv1b_launch_encode(const EncodeParams& p, int64_t max_tiles, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(max_tiles), p.Hkv, p.B);
  return launch_pdl(encode_kernel, grid, dim3(1024), 0, stream, p);
}
