// kv1b_device.cuh -- device-side building blocks shared by the encode, attend and Top-p kernels.
//
// Warp convention used throughout: a warp owns one 128-channel vector; lane l holds channels
// 4l .. 4l+3 in registers x[0..3].
//
// Every floating-point step that decides a stored bit, code or integer is written with explicit
// round-to-nearest intrinsics (__fadd_rn, __fmul_rn, __fdiv_rn, __fsqrt_rn) so the compiler can
// neither contract nor reorder it; the library is also compiled with --fmad=false.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kv1b.h"

namespace kv1b {

// Programmatic dependent launch: a kernel launched with the programmatic-serialization attribute may
// be scheduled while its predecessor in the stream is still running; griddepcontrol.wait returns once
// every prerequisite grid has completed and its memory is visible (a no-op for a plain launch).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel in the stream be scheduled now (its CTAs take free SM slots and run up to
// their own griddepcontrol.wait, which still waits for this whole grid to complete).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

constexpr int kD = 128;
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------------------------
// Loads: 4 consecutive channels of an fp32 / bf16 / fp16 row as fp32 (exact conversions).
__device__ __forceinline__ void load4(const void* base, int64_t elem_off, int dtype, float x[4]) {
  if (dtype == KV1B_DTYPE_F32) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + elem_off));
    const uint32_t h[4] = {u.x & 0xffffu, u.x >> 16, u.y & 0xffffu, u.y >> 16};
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (dtype == KV1B_DTYPE_BF16) x[r] = __uint_as_float(h[r] << 16);
      else x[r] = __half2float(__ushort_as_half(static_cast<unsigned short>(h[r])));
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Random-sign Walsh-Hadamard rotation ("RaBitQCache": randomised rotation before binarisation).
// y = H (D (.) x), H the unnormalised Hadamard matrix in natural (Sylvester) order, computed with
// butterfly stages h = 1, 2, 4, ..., 64; each stage maps the pair (a at index i, c at i + h) to
// (a + c, a - c).  Stages 1 and 2 are inside a lane, stages 4..64 pair lane l with lane l ^ (h/4).
__device__ __forceinline__ void rotate128(float x[4], const float sgn[4]) {
  #pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = (sgn[r] < 0.0f) ? -x[r] : x[r];
  const float a0 = __fadd_rn(x[0], x[1]), a1 = __fsub_rn(x[0], x[1]);
  const float a2 = __fadd_rn(x[2], x[3]), a3 = __fsub_rn(x[2], x[3]);
  x[0] = __fadd_rn(a0, a2);
  x[2] = __fsub_rn(a0, a2);
  x[1] = __fadd_rn(a1, a3);
  x[3] = __fsub_rn(a1, a3);
  const int lane = threadIdx.x & 31;
  #pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float o = __shfl_xor_sync(kFull, x[r], m);
      x[r] = upper ? __fsub_rn(o, x[r]) : __fadd_rn(x[r], o);
    }
  }
}

// Several rounds y <- H (D_r (.) y) (a stronger rotation): signs holds KV1B_MAX_ROUNDS x 128 entries
// and a round whose first sign is 0 ends the rotation (one round unless the cache asked for more).
__device__ __forceinline__ void rotate_rounds(float x[4], const float* signs) {
  static_assert(KV1B_MAX_ROUNDS == 3, "three round markers below");
  const int lane = threadIdx.x & 31;
  // the rounds' first signs (the same addresses for every lane: warp-uniform), read together with
  // round 0's signs so that the count costs no extra dependent load
  const float f1 = signs[kD], f2 = signs[2 * kD];
  float sg[4];
  #pragma unroll
  for (int j = 0; j < 4; ++j) sg[j] = signs[4 * lane + j];
  if (signs[0] == 0.0f) return;
  rotate128(x, sg);  // round 0, straight-line (every cache has it)
  const int rounds = f1 == 0.0f ? 1 : (f2 == 0.0f ? 2 : 3);
  #pragma unroll 1
  for (int r = 1; r < rounds; ++r) {
    #pragma unroll
    for (int j = 0; j < 4; ++j) sg[j] = signs[r * kD + 4 * lane + j];
    rotate128(x, sg);
  }
}

// Fixed pairwise tree over the 128 channels: for h = 64, 32, ..., 1: a[i] += a[i + h] (i < h).
// Returns a[0] on every lane.
__device__ __forceinline__ float tree_sum128(const float a_in[4]) {
  float a[4] = {a_in[0], a_in[1], a_in[2], a_in[3]};
  #pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {  // h = 64, 32, 16, 8, 4  <->  lane offsets 16..1
    #pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float o = __shfl_down_sync(kFull, a[r], off);
      a[r] = __fadd_rn(a[r], o);
    }
  }
  // lane 0 now holds a[0..3] after the h = 4 stage
  a[0] = __fadd_rn(a[0], a[2]);  // h = 2
  a[1] = __fadd_rn(a[1], a[3]);
  a[0] = __fadd_rn(a[0], a[1]);  // h = 1
  return __shfl_sync(kFull, a[0], 0);
}

// Pack one bit per channel: bit i of word w = bit of channel 32w + i ("H1IB-KV" bitmap order).
// nib = this lane's 4 bits (bit r = channel 4l + r).  Returns word (lane >> 3) on every lane.
__device__ __forceinline__ uint32_t pack_word(uint32_t nib) {
  const int lane = threadIdx.x & 31;
  uint32_t v = nib << (4 * (lane & 7));
  v |= __shfl_xor_sync(kFull, v, 1);
  v |= __shfl_xor_sync(kFull, v, 2);
  v |= __shfl_xor_sync(kFull, v, 4);
  return v;
}

// ---------------------------------------------------------------------------------------------
// Query preparation for one head (one warp): rotate, quantise to 4 bits between min and max,
// and build the 4 bit-planes ("RaBitQCache": binary x INT4 arithmetic).
struct QueryPrep {
  uint32_t planes[4][4];  // [plane j][word w], valid on every lane
  float vl, delta;
  int32_t sq;
};

__device__ __forceinline__ QueryPrep query_prep_warp(const void* q, int64_t row_off, int dtype, const float* signs) {
  const int lane = threadIdx.x & 31;
  float x[4];
  load4(q, row_off + 4 * lane, dtype, x);
  rotate_rounds(x, signs);
  float lo = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
  float hi = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  #pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(kFull, lo, m));
    hi = fmaxf(hi, __shfl_xor_sync(kFull, hi, m));
  }
  const float dl = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
  int code[4];
  int csum = 0;
  #pragma unroll
  for (int r = 0; r < 4; ++r) {
    int c = 0;
    if (dl > 0.0f) {
      const float fl = floorf(__fadd_rn(__fdiv_rn(__fsub_rn(x[r], lo), dl), 0.5f));
      c = !(fl > 0.0f) ? 0 : (fl >= 15.0f ? 15 : static_cast<int>(fl));
    }
    code[r] = c;
    csum += c;
  }
  QueryPrep qp;
  #pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t nib = 0;
    #pragma unroll
    for (int r = 0; r < 4; ++r) nib |= static_cast<uint32_t>((code[r] >> j) & 1) << r;
    const uint32_t word = pack_word(nib);
    #pragma unroll
    for (int w = 0; w < 4; ++w) qp.planes[j][w] = __shfl_sync(kFull, word, 8 * w);
  }
  qp.vl = lo;
  qp.delta = dl;
  qp.sq = __reduce_add_sync(kFull, csum);
  return qp;
}

// ---------------------------------------------------------------------------------------------
// Proxy score of one (token, head): binary x INT4 popcounts, then the fp32 logit in the fixed
// order  dot = fl(fl(delta * I2) + fl(vl * I1)),  s = fl(fl(dot * fl(N * cinv)) * qs),
// I1 = 2 Bc - 128, I2 = 2 A - Sq, qs = scale / 128.
__device__ __forceinline__ int32_t popc_A(const uint4 b, const uint32_t P[4][4]) {
  int32_t A = 0;
  #pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int32_t pj = __popc(b.x & P[j][0]) + __popc(b.y & P[j][1]) + __popc(b.z & P[j][2]) + __popc(b.w & P[j][3]);
    A += pj << j;
  }
  return A;
}

__device__ __forceinline__ int32_t popc_Bc(const uint4 b) {
  return __popc(b.x) + __popc(b.y) + __popc(b.z) + __popc(b.w);
}

__device__ __forceinline__ float logit_from_ints(int32_t A, int32_t Bc, int32_t sq, float vl, float delta, float nc,
                                                 float qs) {
  const int32_t I1 = 2 * Bc - kD;
  const int32_t I2 = 2 * A - sq;
  const float dot = __fadd_rn(__fmul_rn(delta, static_cast<float>(I2)), __fmul_rn(vl, static_cast<float>(I1)));
  return __fmul_rn(__fmul_rn(dot, nc), qs);
}

// ---------------------------------------------------------------------------------------------
// binary16 helpers for the value quantiser.
__device__ __forceinline__ double half_bits_to_double(uint32_t hb) {
  return static_cast<double>(__half2float(__ushort_as_half(static_cast<unsigned short>(hb))));
}

// Smallest non-negative finite binary16 h with 15*h >= D (15*h is exact in fp64); 0x7bff and
// *sat on overflow.  Starts next to the answer (a float estimate of D / 15, within a binary16 step
// of it) and walks at most a few steps, each checked exactly in fp64.
__device__ __forceinline__ uint32_t half_scale_up_f64(double D, int* sat) {
  if (!(D > 0.0)) return 0u;
  if (D > 15.0 * 65504.0) { *sat = 1; return 0x7bffu; }
  uint32_t hb = __half_as_ushort(__float2half_rz(__fmul_rz(__double2float_rz(D), 0x1.111112p-4f)));
  if (hb > 0x7bffu) hb = 0x7bffu;
  #pragma unroll 1
  for (int i = 0; i < 8 && 15.0 * half_bits_to_double(hb) < D; ++i) ++hb;
  #pragma unroll 1
  for (int i = 0; i < 8 && hb > 0u && 15.0 * half_bits_to_double(hb - 1u) >= D; --hb, ++i) {}
  return hb;
}

// The same for D = fl64(mx - mn) (mn a binary16 value, mx >= mn), in fp32 arithmetic: TwoSum (Knuth)
// gives D = hi + lo exactly; when that sum fits the 53 bits of a double (always, unless lo is below
// hi's 29th bit: then the fp64 rounding of D matters and the fp64 form runs), 15 h >= D is decided
// exactly as 15 h - hi >= lo: 15 h is exact, and 15 h - hi is exact whenever 15 h and hi are within a
// factor of two (Sterbenz) and otherwise far from lo on the right side.
__device__ __forceinline__ uint32_t half_scale_up(float mx, float mn, int* sat) {
  const float hi = __fsub_rn(mx, mn);
  const float bb = __fsub_rn(hi, mx);
  const float lo = __fadd_rn(__fsub_rn(mx, __fsub_rn(hi, bb)), __fsub_rn(-mn, bb));
  if (lo != 0.0f && fabsf(lo) < __fmul_rn(hi, 0x1p-28f))
    return half_scale_up_f64(static_cast<double>(mx) - static_cast<double>(mn), sat);
  if (!(hi > 0.0f)) return 0u;
  if (hi > 982560.0f || (hi == 982560.0f && lo > 0.0f)) { *sat = 1; return 0x7bffu; }  // 15 * 65504
  auto covers = [&](uint32_t hb) {
    const float h15 = __fmul_rn(15.0f, __half2float(__ushort_as_half(static_cast<unsigned short>(hb))));
    return __fsub_rn(h15, hi) >= lo;
  };
  uint32_t hb = __half_as_ushort(__float2half_rz(__fmul_rz(hi, 0x1.111112p-4f)));
  if (hb > 0x7bffu) hb = 0x7bffu;
  #pragma unroll 1
  for (int i = 0; i < 8 && !covers(hb); ++i) ++hb;
  #pragma unroll 1
  for (int i = 0; i < 8 && hb > 0u && covers(hb - 1u); --hb, ++i) {}
  return hb;
}

// The smallest non-negative finite binary16 h with 15 h >= D for D = fl64(mx - mn), as half_scale_up,
// without a data-dependent loop in the common case: the float estimate e of D / 15 is at most two
// binary16 steps below the answer and never above it, so the answer is e, e + 1 or e + 2 unless
// e - 1 already covers D; only then (or for e + 2 failing) does the warp take the walking form.
__device__ __forceinline__ uint32_t half_scale_up_fast(float mx, float mn, int* sat) {
  const float hi = __fsub_rn(mx, mn);
  const float bb = __fsub_rn(hi, mx);
  const float lo = __fadd_rn(__fsub_rn(mx, __fsub_rn(hi, bb)), __fsub_rn(-mn, bb));
  const bool exact = !(lo != 0.0f && fabsf(lo) < __fmul_rn(hi, 0x1p-28f));
  auto covers = [&](uint32_t hb) {
    const float h15 = __fmul_rn(15.0f, __half2float(__ushort_as_half(static_cast<unsigned short>(hb))));
    return __fsub_rn(h15, hi) >= lo;
  };
  uint32_t e = __half_as_ushort(__float2half_rz(__fmul_rz(hi, 0x1.111112p-4f)));
  e = e > 0x7bfdu ? 0x7bfdu : e;
  const bool cm = e > 0u && covers(e - 1u), c0 = covers(e), c1 = covers(e + 1u), c2 = covers(e + 2u);
  const bool normal = exact && hi >= 0.0f && hi < 982560.0f && !cm && c2;  // hi = 0: a constant group, scale 0
  uint32_t hb = c0 ? e : (c1 ? e + 1u : e + 2u);
  if (__any_sync(kFull, !normal)) {  // rare: saturation, an inexact fp64 range, or an estimate off by more
    const uint32_t slow = half_scale_up(mx, mn, sat);
    hb = normal ? hb : slow;
  }
  return hb;
}

// Correctly rounded x / y from r = RN(1 / y): q0 = RN(x r) is within an ulp of x / y, the residual
// x - y q0 is exact in a fused multiply-add, and RN(q0 + (x - y q0) r) = RN(x / y) when nothing
// underflows or overflows (Markstein's correction theorem: P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34 (1), 1990).
__device__ __forceinline__ float div_markstein(float x, float y, float r) {
  const float q0 = __fmul_rn(x, r);
  return __fmaf_rn(__fmaf_rn(-y, q0, x), r, q0);
}

// Largest finite binary16 <= x (saturates at -65504 with *sat).
__device__ __forceinline__ uint32_t half_round_down(float x, int* sat) {
  uint32_t hb = __half_as_ushort(__float2half_rd(x));
  if (hb == 0xfc00u) { *sat = 1; return 0xfbffu; }  // -inf: below the binary16 range
  if (hb == 0x8000u) hb = 0u;                      // -0 -> +0
  return hb;
}

}  // namespace kv1b
