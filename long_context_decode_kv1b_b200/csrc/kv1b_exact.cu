// kv1b_exact.cu -- exact attention over a selected token set ("RaBitQCache", abstract / core idea:
// the proxy scores retrieve the tokens, and attention over them is then sparse attention with the
// exact keys and values).  The keys and values are the caller's own (bf16 / fp16 / fp32, any
// token / head / sequence strides, device memory or host memory the device can read).
//
// Row r = (sequence b, query head hq) reads kv-head hq / G.  The work is sized by the selected counts,
// which only the device knows:
//  1. plan: one block turns the rows' counts n_r into work items of kExactItem selected entries
//     (item_off[r] = sum over earlier rows of ceil(n_r / kExactItem));
//  2. a persistent grid (a few blocks per SM) strides over the items: each of a block's 8 warps takes
//     every 8th entry of the item (its 32 token indices fetched at once, one per lane), in rounds of
//     8 tokens (4 for fp32 rows) with the next round's loads in flight; lane l loads channels
//     4l..4l+3 of the token's
//     key and value row (fp32 after exact conversion), the logit z = (scale log2 e) q.k is a butterfly
//     sum (the same bits in every lane), and an online softmax in log2 units accumulates
//     sum 2^(z - m) v; the warps combine into one partial (m, l, o[128]) per item;
//  3. merge: per row, log-sum-exp over its items in a fixed order, out = o / l (zeros for an empty
//     set).
// An index outside [0, min(length[b], kv_tokens)) is skipped and flagged in the cache status word;
// no memory outside the given rows is read.
#include <type_traits>

#include "kv1b_device.cuh"
#include "kv1b_launch.h"

namespace kv1b {

constexpr int kExactWarps = 8;
constexpr int kPlanThreads = 1024;

__device__ __forceinline__ int row_count(const ExactParams& p, int64_t r) {
  const int n = p.cnt[r];
  return n < 0 ? 0 : (n > p.cap ? p.cap : n);
}

// ---------------------------------------------------------------- 1. plan
__global__ void __launch_bounds__(kPlanThreads) exact_plan_kernel(const ExactParams p, int rows) {
  __shared__ int s_w[kPlanThreads / 32];
  __shared__ int s_carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int r0 = 0; r0 < rows; r0 += kPlanThreads) {  // block-uniform
    const int r = r0 + threadIdx.x;
    const int items = r < rows ? (row_count(p, r) + kExactItem - 1) / kExactItem : 0;
    int incl = items;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    int before = s_carry;
    for (int w = 0; w < warp; ++w) before += s_w[w];
    if (r < rows) p.item_off[r] = before + incl - items;
    __syncthreads();
    if (threadIdx.x == kPlanThreads - 1) s_carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) p.item_off[rows] = s_carry;
}

// ---------------------------------------------------------------- 2. items
// One token's 4 channels of this lane, raw: 8 bytes for 16-bit rows, 16 bytes for fp32 rows.
template <int KVD>
struct RawRow {
  using T = typename std::conditional<KVD == KV1B_DTYPE_F32, float4, uint2>::type;
  static __device__ __forceinline__ T load(const void* base, int64_t elem_off) {
    if constexpr (KVD == KV1B_DTYPE_F32) {
      return __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off));
    } else {
      return __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + elem_off));
    }
  }
  static __device__ __forceinline__ void to_f32(const T& r, float x[4]) {
    if constexpr (KVD == KV1B_DTYPE_F32) {
      x[0] = r.x; x[1] = r.y; x[2] = r.z; x[3] = r.w;
    } else {
      const uint32_t h[4] = {r.x & 0xffffu, r.x >> 16, r.y & 0xffffu, r.y >> 16};
      #pragma unroll
      for (int c = 0; c < 4; ++c) {
        if constexpr (KVD == KV1B_DTYPE_BF16) x[c] = __uint_as_float(h[c] << 16);
        else x[c] = __half2float(__ushort_as_half(static_cast<unsigned short>(h[c])));
      }
    }
  }
};

// Each warp takes entries e0 + warp + 8 j (j < 32) of its item: lane j holds entry j's token index;
// rounds of U tokens are loaded one round ahead of the one being reduced.
template <int KVD>
__global__ void __launch_bounds__(kExactWarps * 32) exact_kernel(const ExactParams p, int rows) {
  constexpr int U = KVD == KV1B_DTYPE_F32 ? 4 : 8;  // tokens per round (registers for 2 rounds in flight)
  using R = RawRow<KVD>;
  using Raw = typename R::T;
  static_assert(kExactItem == kExactWarps * 32, "a warp holds its item entries' indices one per lane");
  __shared__ float s_m[kExactWarps], s_l[kExactWarps];
  __shared__ float s_acc[kExactWarps][kD];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.item_off[rows];
  bool bad = false;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {  // block-uniform
    // the row holding this item: the last r with item_off[r] <= item (binary search)
    int lo = 0, hi = rows - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.item_off[mid] <= item) lo = mid;
      else hi = mid - 1;
    }
    const int64_t r = lo;
    const int b = static_cast<int>(r / p.Hq), hq = static_cast<int>(r - static_cast<int64_t>(b) * p.Hq);
    const int kvh = hq / (p.Hq / p.Hkv);
    const int n = row_count(p, r);
    const int e0 = (item - p.item_off[r]) * kExactItem;
    const int e1 = e0 + kExactItem < n ? e0 + kExactItem : n;
    const int64_t lim = p.len[b] < p.kv_tokens ? p.len[b] : p.kv_tokens;
    // this warp's entries: e0 + warp + 8 j for j < cnt
    const int cnt = e1 - e0 - warp > 0 ? (e1 - e0 - warp + kExactWarps - 1) / kExactWarps : 0;
    const int64_t my_t = lane < cnt ? static_cast<int64_t>(p.sel[r * p.cap + e0 + warp + kExactWarps * lane]) : -1;
    const bool my_ok = lane < cnt && my_t >= 0 && my_t < lim;
    bad |= lane < cnt && !my_ok;
    float qv[4];
    load4(p.q, r * kD + 4 * lane, p.q_dtype, qv);
    #pragma unroll
    for (int c = 0; c < 4; ++c) qv[c] = __fmul_rn(qv[c], p.qscale);  // logits in log2 units
    const int64_t kv_off = static_cast<int64_t>(b) * p.sb + static_cast<int64_t>(kvh) * p.sh + 4 * lane;
    float m = -INFINITY, l = 0.0f;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    Raw kr[U], vr[U];
    bool ok[U];
    auto issue = [&](int j0) {  // loads of entries j0 .. j0 + U - 1 of this warp
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u;
        const int64_t t = __shfl_sync(kFull, my_t, j & 31);
        ok[u] = __shfl_sync(kFull, my_ok, j & 31) && j < cnt;
        if (ok[u]) {
          kr[u] = R::load(p.k, kv_off + t * p.st);
          vr[u] = R::load(p.v, kv_off + t * p.st);
        }
      }
    };
    if (cnt > 0) issue(0);
    for (int j0 = 0; j0 < cnt; j0 += U) {  // warp-uniform
      Raw kc[U], vc[U];
      bool okc[U];
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        kc[u] = kr[u];
        vc[u] = vr[u];
        okc[u] = ok[u];
      }
      if (j0 + U < cnt) issue(j0 + U);  // the next round in flight
      float z[U];
      float mx = m;
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        float kx[4];
        R::to_f32(kc[u], kx);
        float d = __fmul_rn(qv[0], kx[0]);
        #pragma unroll
        for (int c = 1; c < 4; ++c) d = __fmaf_rn(qv[c], kx[c], d);
        #pragma unroll
        for (int o = 16; o >= 1; o >>= 1) d = __fadd_rn(d, __shfl_xor_sync(kFull, d, o));  // same in every lane
        z[u] = okc[u] ? d : -INFINITY;
        mx = fmaxf(mx, z[u]);
      }
      if (mx > m) {  // warp-uniform: rescale to the new reference
        const float al = (m == -INFINITY) ? 0.0f : exp2f(__fsub_rn(m, mx));
        l = __fmul_rn(l, al);
        #pragma unroll
        for (int c = 0; c < 4; ++c) acc[c] = __fmul_rn(acc[c], al);
        m = mx;
      }
      #pragma unroll
      for (int u = 0; u < U; ++u) {
        if (okc[u]) {
          float vx[4];
          R::to_f32(vc[u], vx);
          const float pu = exp2f(__fsub_rn(z[u], m));
          l = __fadd_rn(l, pu);
          #pragma unroll
          for (int c = 0; c < 4; ++c) acc[c] = __fmaf_rn(pu, vx[c], acc[c]);
        }
      }
    }
    __syncthreads();  // the previous item's partial sums are read
    if (lane == 0) {
      s_m[warp] = m;
      s_l[warp] = l;
    }
    #pragma unroll
    for (int c = 0; c < 4; ++c) s_acc[warp][4 * lane + c] = acc[c];
    __syncthreads();
    if (threadIdx.x < kD) {
      const int ch = threadIdx.x;
      float M = -INFINITY;
      for (int w = 0; w < kExactWarps; ++w) M = fmaxf(M, s_m[w]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
        for (int w = 0; w < kExactWarps; ++w) {
          if (s_m[w] == -INFINITY) continue;
          const float wt = exp2f(__fsub_rn(s_m[w], M));
          num = __fmaf_rn(wt, s_acc[w][ch], num);
          den = __fmaf_rn(wt, s_l[w], den);
        }
      }
      float* part = p.part + static_cast<int64_t>(item) * kPartStride;
      if (ch == 0) {
        part[0] = M;
        part[1] = den;
      }
      part[2 + ch] = num;
    }
  }
  if (__any_sync(kFull, bad) && lane == 0) atomicOr(p.status, KV1B_STATUS_BAD_INDEX);
}

// ---------------------------------------------------------------- 3. merge
// grid (rows), 1024 threads: the row's reference maximum and denominator by block reductions (fixed
// tree order), then thread group g = tid / 128 sums the numerators of items g, g + 8, ... for channel
// tid % 128, and the 8 group sums are added in order.
constexpr int kMergeThreads = 1024;
constexpr int kMergeGroups = kMergeThreads / kD;
__global__ void __launch_bounds__(kMergeThreads) exact_merge_kernel(const ExactParams p) {
  __shared__ float s_red[kMergeThreads / 32];
  __shared__ float s_num[kMergeGroups][kD];
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k0 = p.item_off[r], k1 = p.item_off[r + 1];
  float M = -INFINITY;
  for (int k = k0 + tid; k < k1; k += kMergeThreads) M = fmaxf(M, p.part[static_cast<int64_t>(k) * kPartStride]);
  #pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
  if (lane == 0) s_red[warp] = M;
  __syncthreads();
  M = s_red[0];
  for (int w = 1; w < kMergeThreads / 32; ++w) M = fmaxf(M, s_red[w]);
  __syncthreads();  // s_red is reused
  float den = 0.0f;
  if (M != -INFINITY) {
    for (int k = k0 + tid; k < k1; k += kMergeThreads) {
      const float* part = p.part + static_cast<int64_t>(k) * kPartStride;
      if (part[0] != -INFINITY) den = __fmaf_rn(exp2f(__fsub_rn(part[0], M)), part[1], den);
    }
  }
  #pragma unroll
  for (int o = 16; o >= 1; o >>= 1) den = __fadd_rn(den, __shfl_xor_sync(kFull, den, o));
  if (lane == 0) s_red[warp] = den;
  const int g = tid / kD, ch = tid % kD;
  float num = 0.0f;
  if (M != -INFINITY) {
    #pragma unroll 4
    for (int k = k0 + g; k < k1; k += kMergeGroups) {
      const float* part = p.part + static_cast<int64_t>(k) * kPartStride;
      const float mk = part[0];
      if (mk != -INFINITY) num = __fmaf_rn(exp2f(__fsub_rn(mk, M)), part[2 + ch], num);
    }
  }
  s_num[g][ch] = num;
  __syncthreads();
  if (tid < kD) {
    float tot = 0.0f, dsum = 0.0f;
    for (int j = 0; j < kMergeGroups; ++j) tot = __fadd_rn(tot, s_num[j][tid]);
    for (int w = 0; w < kMergeThreads / 32; ++w) dsum = __fadd_rn(dsum, s_red[w]);
    p.out[r * kD + tid] = dsum > 0.0f ? __fdiv_rn(tot, dsum) : 0.0f;
  }
}

}  // namespace kv1b

using namespace kv1b;

size_t kv1b_exact_workspace_bytes(int32_t rows, int32_t cap) {
  const size_t R = static_cast<size_t>(rows);
  const size_t items = R * ((static_cast<size_t>(cap) + kExactItem - 1) / kExactItem);
  return ((R + 1) * 4 + 255) / 256 * 256 + items * kPartStride * 4;  // item offsets, item partials
}

void kv1b_exact_carve(ExactParams* p, void* ws, int32_t rows) {
  char* w = static_cast<char*>(ws);
  p->item_off = reinterpret_cast<int32_t*>(w);
  p->part = reinterpret_cast<float*>(w + ((static_cast<size_t>(rows) + 1) * 4 + 255) / 256 * 256);
}

cudaError_t kv1b_launch_exact(const ExactParams& p, int32_t rows, int32_t num_sms, cudaStream_t stream) {
  if (rows < 1) return cudaErrorInvalidValue;
  exact_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p, rows);
  const unsigned grid = 4u * static_cast<unsigned>(num_sms > 0 ? num_sms : 1);
  if (p.kv_dtype == KV1B_DTYPE_F32)
    exact_kernel<KV1B_DTYPE_F32><<<grid, kExactWarps * 32, 0, stream>>>(p, rows);
  else if (p.kv_dtype == KV1B_DTYPE_BF16)
    exact_kernel<KV1B_DTYPE_BF16><<<grid, kExactWarps * 32, 0, stream>>>(p, rows);
  else
    exact_kernel<KV1B_DTYPE_F16><<<grid, kExactWarps * 32, 0, stream>>>(p, rows);
  exact_merge_kernel<<<rows, kMergeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}
