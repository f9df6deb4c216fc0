/*
 * kv1b_oracle.cpp -- plain, slow, obviously-correct CPU oracle (C++17, single thread).
 *
 * TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference arm may load it.  It shares no code with the CUDA library.
 *
 * Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC
 * (no contraction of a*b+c into fma, so every fp32 step below is one IEEE round-to-nearest op;
 * fmaf() is used only where the algorithm states a fused multiply-add).
 *
 * Which page fixes what (page title, then section):
 *  - RaBitQCache (abstract; "core idea"; "technical framework"; "key design"): keys are randomly
 *    rotated then binary-quantised; a binary x INT4 computation gives an unbiased proxy score;
 *    adaptive Top-p picks the smallest token set by estimated attention.
 *  - H1B-KV (abstract; "technical framework"; "key design"): 1-bit key sketch by random projection,
 *    4-bit linear value quantisation; weights from the sketch, then the 4-bit values give the output.
 *  - H1IB-KV news article, part 2 (architecture), item 3 "hardware-friendly storage optimisation": bitmap storage with bit
 *    (i mod 8) of byte (i/8); bit 1 stands for +1 and bit 0 for -1.  Packing bit (i mod 32) of
 *    32-bit word (i/32) is the same bit order on a little-endian machine.
 * Where the pages leave a step open, the reading taken is stated beside the step.
 */
#include "kv1b_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

namespace {

bool valid_d(int d) { return d >= 32 && (d & (d - 1)) == 0; }

int popcount32(uint32_t x) {
  int c = 0;
  for (int i = 0; i < 32; ++i) c += (x >> i) & 1u;
  return c;
}

/* ---- binary16, from the IEEE 754 definition: 1 sign bit, 5 exponent bits (bias 15),
 *      10 fraction bits; exponent 0 = subnormal, exponent 31 = inf/nan. ---- */
double half_value(uint16_t h) {
  const int sign = h >> 15, e = (h >> 10) & 0x1f, m = h & 0x3ff;
  double v;
  if (e == 0) v = std::ldexp(static_cast<double>(m), -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp(static_cast<double>(m | 0x400), e - 25);
  return sign ? -v : v;
}

/* All finite binary16 values except -0, sorted ascending (value, bits). Built once. */
const std::vector<std::pair<double, uint16_t>>& finite_halves() {
  static std::vector<std::pair<double, uint16_t>> t;
  if (t.empty()) {
    for (uint32_t b = 0; b < 65536u; ++b) {
      const uint16_t h = static_cast<uint16_t>(b);
      if (((h >> 10) & 0x1f) == 31) continue;  // inf / nan
      if (h == 0x8000) continue;               // -0 (keep +0)
      t.emplace_back(half_value(h), h);
    }
    std::sort(t.begin(), t.end());
  }
  return t;
}

/* Largest finite half <= x; saturates at -65504 (sets *sat). */
uint16_t half_round_down(double x, int* sat) {
  const auto& t = finite_halves();
  if (x < t.front().first) { *sat = 1; return t.front().second; }
  // last element with value <= x
  std::size_t lo = 0, hi = t.size();  // invariant: t[lo].first <= x, answer in [lo, hi)
  while (hi - lo > 1) {
    const std::size_t mid = (lo + hi) / 2;
    if (t[mid].first <= x) lo = mid; else hi = mid;
  }
  return t[lo].second;
}

/* Smallest non-negative finite half h with 15*h >= D (15*h is exact in fp64); saturates. */
uint16_t half_scale_up(double D, int* sat) {
  const auto& t = finite_halves();
  static const std::size_t i = static_cast<std::size_t>(
      std::lower_bound(t.begin(), t.end(), std::make_pair(0.0, static_cast<uint16_t>(0))) - t.begin());  // +0
  if (15.0 * t.back().first < D) { *sat = 1; return t.back().second; }
  std::size_t lo = i, hi = t.size() - 1;  // answer in [lo, hi]
  while (lo < hi) {
    const std::size_t mid = (lo + hi) / 2;
    if (15.0 * t[mid].first >= D) hi = mid; else lo = mid + 1;
  }
  return t[lo].second;
}

// Up to kRefMaxRounds rounds y <- H (D_r (.) y); signs holds kRefMaxRounds x d entries, and a
// round whose signs are 0 ends the rotation (one round unless a stronger rotation was asked for).
constexpr int kRefMaxRounds = 3;

void rotate(const float* x, const float* signs, int d, float* y) {
  for (int i = 0; i < d; ++i) y[i] = x[i];
  for (int r = 0; r < kRefMaxRounds; ++r) {
    const float* sg = signs + static_cast<int64_t>(r) * d;
    if (sg[0] == 0.0f) break;
    for (int i = 0; i < d; ++i) y[i] = (sg[i] < 0.0f) ? -y[i] : y[i];
    ref_fwht(y, d);
  }
}

}  // namespace

extern "C" {

/* SplitMix64, Steele, Lea & Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014.
 * Reading (the pages name no generator): the rotation's random signs come from this generator. */
uint64_t ref_splitmix64_next(uint64_t* state) {
  *state += 0x9E3779B97F4A7C15ull;
  uint64_t z = *state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* RaBitQCache abstract / "core idea": a seeded random rotation.  Reading: R = H * diag(D) with
 * D_i = +-1 from the top bit of successive SplitMix64 outputs, one sign vector per cache. */
void ref_rotation_signs(uint64_t seed, int d, float* signs) {
  uint64_t st = seed;
  for (int i = 0; i < d; ++i) signs[i] = (ref_splitmix64_next(&st) >> 63) ? -1.0f : 1.0f;
}

/* Stronger rotation (RaBitQCache, abstract / key design: a randomised rotation; RaBitQ proves its
 * estimator for a random orthogonal one, which several H D rounds approach): `rounds`
 * successive H * diag(D_r), the signs of round r being outputs r d .. r d + d - 1 of the same
 * SplitMix64 stream (round 0 equals ref_rotation_signs).  signs: kRefMaxRounds x d entries, the
 * unused rounds zero. */
void ref_rotation_signs_rounds(uint64_t seed, int d, int rounds, float* signs) {
  uint64_t st = seed;
  for (int r = 0; r < kRefMaxRounds; ++r)
    for (int i = 0; i < d; ++i)
      signs[r * d + i] = r < rounds ? ((ref_splitmix64_next(&st) >> 63) ? -1.0f : 1.0f) : 0.0f;
}

/* Walsh-Hadamard transform, natural order, unnormalised (H H = d I). */
void ref_fwht(float* x, int d) {
  for (int h = 1; h < d; h *= 2) {
    for (int i = 0; i < d; i += 2 * h) {
      for (int j = i; j < i + h; ++j) {
        const float a = x[j];
        const float c = x[j + h];
        x[j] = a + c;
        x[j + h] = a - c;
      }
    }
  }
}

float ref_tree_sum(const float* a, int d) {
  std::vector<float> t(a, a + d);
  for (int h = d / 2; h >= 1; h /= 2)
    for (int i = 0; i < h; ++i) t[i] = t[i] + t[i + h];
  return t[0];
}

/* H1B-KV abstract / "key design": each key becomes a 1-bit sketch of a random projection.
 * RaBitQCache: rotation then binary quantisation, with an unbiased estimator.  Reading of the
 * per-token scalars (the pages print no formula): RaBitQ's norm ||k|| and the correction
 * <xbar, k'> with xbar = sign(y)/sqrt(d), k' = y/(sqrt(d)||k||), i.e. C = sum|y_i| / (d ||k||);
 * we store N = ||k|| and cinv = 1/C = d N / sum|y_i| (one IEEE division).  Sign of 0 -> bit 1. */
void ref_encode_key(const float* k, const float* signs, int d, uint32_t* bits, float* norm, float* cinv) {
  if (!valid_d(d)) return;
  std::vector<float> sq(d), y(d), ab(d);
  for (int i = 0; i < d; ++i) sq[i] = k[i] * k[i];
  const float n = std::sqrt(ref_tree_sum(sq.data(), d));
  rotate(k, signs, d, y.data());
  for (int w = 0; w < d / 32; ++w) {
    uint32_t word = 0;
    for (int i = 0; i < 32; ++i)
      if (y[32 * w + i] >= 0.0f) word |= (1u << i);
    bits[w] = word;
  }
  for (int i = 0; i < d; ++i) ab[i] = std::fabs(y[i]);
  const float sabs = ref_tree_sum(ab.data(), d);
  const float dn = static_cast<float>(d) * n;
  *norm = n;
  *cinv = (sabs > 0.0f) ? dn / sabs : 1.0f;
}

/* H1B-KV "key design": values by 4-bit linear quantisation.  Reading: asymmetric, groups of 32
 * channels, fp16 min rounded down and fp16 scale rounded up so that every value of the group lies
 * in [min, min + 15 scale]; code = clamp(floor((v - min)/scale + 0.5), 0, 15) in fp32. */
int ref_encode_value(const float* v, int d, uint32_t* codes, uint32_t* sm) {
  if (!valid_d(d)) return -1;
  int flags = 0;
  for (int i = 0; i < d; ++i)
    if (!std::isfinite(v[i])) flags |= 1;
  for (int w = 0; w < d / 8; ++w) codes[w] = 0;
  for (int g = 0; g < d / 32; ++g) {
    const float* x = v + 32 * g;
    float mn = x[0], mx = x[0];
    for (int i = 1; i < 32; ++i) {
      if (x[i] < mn) mn = x[i];
      if (x[i] > mx) mx = x[i];
    }
    int sat = 0;
    const uint16_t min_bits = half_round_down(static_cast<double>(mn), &sat);
    const double minv = half_value(min_bits);
    const double D = static_cast<double>(mx) - minv;
    const uint16_t scale_bits = half_scale_up(D, &sat);
    if (sat) flags |= 2;
    const float sf = static_cast<float>(half_value(scale_bits));
    const float mf = static_cast<float>(minv);
    sm[g] = static_cast<uint32_t>(scale_bits) | (static_cast<uint32_t>(min_bits) << 16);
    for (int i = 0; i < 32; ++i) {
      int code = 0;
      if (sf > 0.0f) {
        const float t1 = x[i] - mf;
        const float t2 = t1 / sf;
        const float t3 = t2 + 0.5f;
        const float fl = std::floor(t3);
        code = !(fl > 0.0f) ? 0 : (fl >= 15.0f ? 15 : static_cast<int>(fl));  // NaN -> 0
      }
      const int c = 32 * g + i;
      codes[c / 8] |= static_cast<uint32_t>(code) << (4 * (c % 8));
    }
  }
  return flags;
}

void ref_encode_keys(const float* K, int64_t L, const float* signs, int d, uint32_t* bits, float* norm,
                     float* cinv) {
  for (int64_t t = 0; t < L; ++t)
    ref_encode_key(K + t * d, signs, d, bits + t * (d / 32), norm + t, cinv + t);
}

int ref_encode_values(const float* V, int64_t L, int d, uint32_t* codes, uint32_t* sm) {
  int flags = 0;
  for (int64_t t = 0; t < L; ++t) flags |= ref_encode_value(V + t * d, d, codes + t * (d / 8), sm + t * (d / 32));
  return flags;
}

double ref_half_to_double(uint16_t h) { return half_value(h); }

void ref_dequant_value(const uint32_t* codes, const uint32_t* sm, int d, double* out) {
  for (int c = 0; c < d; ++c) {
    const uint32_t code = (codes[c / 8] >> (4 * (c % 8))) & 0xfu;
    const uint32_t s = sm[c / 32];
    const double scale = half_value(static_cast<uint16_t>(s & 0xffffu));
    const double mn = half_value(static_cast<uint16_t>(s >> 16));
    out[c] = mn + scale * static_cast<double>(code);
  }
}

/* RaBitQCache abstract / "key design": the INT4 side of binary-INT4 arithmetic is the rotated
 * query quantised to 4 bits.  Reading: uniform min/max quantiser, deterministic round-half-up,
 * codes held as 4 bit-planes. */
void ref_query_prep(const float* q, const float* signs, int d, uint32_t* planes, float* vl, float* delta,
                    int32_t* Sq, uint8_t* codes, float* z_out) {
  if (!valid_d(d)) return;
  std::vector<float> z(d);
  rotate(q, signs, d, z.data());
  float lo = z[0], hi = z[0];
  for (int i = 1; i < d; ++i) {
    if (z[i] < lo) lo = z[i];
    if (z[i] > hi) hi = z[i];
  }
  const float range = hi - lo;
  const float dl = range / 15.0f;
  std::vector<int> c(d, 0);
  int32_t sum = 0;
  for (int i = 0; i < d; ++i) {
    int code = 0;
    if (dl > 0.0f) {
      const float t1 = z[i] - lo;
      const float t2 = t1 / dl;
      const float t3 = t2 + 0.5f;
      const float fl = std::floor(t3);
      code = !(fl > 0.0f) ? 0 : (fl >= 15.0f ? 15 : static_cast<int>(fl));  // NaN -> 0
    }
    c[i] = code;
    sum += code;
  }
  for (int j = 0; j < 4; ++j)
    for (int w = 0; w < d / 32; ++w) {
      uint32_t word = 0;
      for (int i = 0; i < 32; ++i)
        if ((c[32 * w + i] >> j) & 1) word |= (1u << i);
      planes[j * (d / 32) + w] = word;
    }
  *vl = lo;
  *delta = dl;
  *Sq = sum;
  if (codes)
    for (int i = 0; i < d; ++i) codes[i] = static_cast<uint8_t>(c[i]);
  if (z_out)
    for (int i = 0; i < d; ++i) z_out[i] = z[i];
}

/* RaBitQCache abstract: "binary-INT4 arithmetic": sum_i b_i code_i by AND + popcount per plane. */
void ref_score_ints(const uint32_t* bits, const uint32_t* planes, int d, int32_t* A, int32_t* Bc) {
  const int nw = d / 32;
  int32_t a = 0, b = 0;
  for (int j = 0; j < 4; ++j) {
    int32_t pj = 0;
    for (int w = 0; w < nw; ++w) pj += popcount32(bits[w] & planes[j * nw + w]);
    a += pj << j;
  }
  for (int w = 0; w < nw; ++w) b += popcount32(bits[w]);
  *A = a;
  *Bc = b;
}

/* The same integers for L consecutive tokens (one call instead of L). */
void ref_score_ints_n(const uint32_t* bits, int64_t L, const uint32_t* planes, int d, int32_t* A, int32_t* Bc) {
  const int nw = d / 32;
  for (int64_t t = 0; t < L; ++t) ref_score_ints(bits + t * nw, planes, d, A + t, Bc + t);
}

/* RaBitQ estimator in unnormalised variables: q.k ~ N cinv sum_i (2 b_i - 1) z_i / d, with the
 * quantised z_i = vl + delta code_i, so sum_i (2b_i - 1) z_i = delta (2A - Sq) + vl (2Bc - d).
 * The logit is that estimate times the softmax scale. */
float ref_logit(int32_t A, int32_t Bc, int32_t Sq, float vl, float delta, float norm, float cinv, float scale,
                int d) {
  const int32_t I1 = 2 * Bc - d;
  const int32_t I2 = 2 * A - Sq;
  const float t1 = delta * static_cast<float>(I2);
  const float t2 = vl * static_cast<float>(I1);
  const float dot = t1 + t2;
  const float nc = norm * cinv;
  const float qs = scale / static_cast<float>(d);
  const float t3 = dot * nc;
  return t3 * qs;
}

void ref_logits(const uint32_t* bits, const float* norm, const float* cinv, int64_t L, const uint32_t* planes,
                float vl, float delta, int32_t Sq, float scale, int d, float* s_out) {
  const int nw = d / 32;
  for (int64_t t = 0; t < L; ++t) {
    int32_t A, Bc;
    ref_score_ints(bits + t * nw, planes, d, &A, &Bc);
    s_out[t] = ref_logit(A, Bc, Sq, vl, delta, norm[t], cinv[t], scale, d);
  }
}

/* H1B-KV "technical framework": attention weights from the 1-bit sketch, then the output from the
 * 4-bit values.  Full (non-Top-p) mode: softmax over all estimated logits, fp64. */
void ref_attend_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                     const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale, int d,
                     double* out) {
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (!valid_d(d) || L <= 0) return;
  std::vector<uint32_t> planes(4 * (d / 32));
  float vl, dl;
  int32_t Sq;
  ref_query_prep(q, signs, d, planes.data(), &vl, &dl, &Sq, nullptr, nullptr);
  std::vector<float> s(L);
  ref_logits(bits, norm, cinv, L, planes.data(), vl, dl, Sq, scale, d, s.data());
  double m = s[0];
  for (int64_t t = 1; t < L; ++t) m = std::max(m, static_cast<double>(s[t]));
  std::vector<double> acc(d, 0.0), vh(d);
  double l = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const double e = std::exp(static_cast<double>(s[t]) - m);
    l += e;
    ref_dequant_value(codes + t * (d / 8), sm + t * (d / 32), d, vh.data());
    for (int c = 0; c < d; ++c) acc[c] += e * vh[c];
  }
  for (int c = 0; c < d; ++c) out[c] = acc[c] / l;
}

/* Coefficients of the degree-7 Taylor polynomial of 2^f = e^(f ln 2): (ln 2)^k / k!, as fp32. */
float ref_exp2_coef(int k) {
  double c = 1.0;
  for (int i = 1; i <= k; ++i) c = c * 0.6931471805599453094 / static_cast<double>(i);
  return static_cast<float>(c);
}

/* RaBitQCache: Top-p over estimated attention probabilities.  Reading: so that the selection is
 * reproducible bit for bit, probabilities are turned into integer masses u ~ 2^32 exp(s - m). */
uint64_t ref_topp_weight(float s, float m) {
  const float log2e = static_cast<float>(1.4426950408889634074);
  const float diff = s - m;
  const float t = diff * log2e;
  if (!(t >= -40.0f)) return 0;
  const float n = std::rint(t);
  const float f = t - n;
  float P = ref_exp2_coef(7);
  for (int k = 6; k >= 0; --k) P = std::fmaf(P, f, ref_exp2_coef(k));
  const float scaled = std::ldexp(P, 32 + static_cast<int>(n));
  return static_cast<uint64_t>(std::trunc(scaled));
}

/* RaBitQCache abstract: adaptive Top-p retrieval -- the token budget follows the actual sparsity:
 * the smallest set of highest-scoring tokens whose estimated probability mass reaches p. */
int64_t ref_topp_select(const float* s, int64_t L, float p, int64_t* sel) {
  if (!(p > 0.0f && p <= 1.0f)) return -1;
  if (L <= 0) return 0;
  float m = s[0];
  for (int64_t t = 1; t < L; ++t) m = std::max(m, s[t]);
  std::vector<uint64_t> u(L);
  uint64_t U = 0;
  for (int64_t t = 0; t < L; ++t) {
    u[t] = ref_topp_weight(s[t], m);
    U += u[t];
  }
  const double Tp = std::ceil(static_cast<double>(p) * static_cast<double>(U));
  uint64_t T = static_cast<uint64_t>(Tp);
  if (T > U) T = U;
  if (T < 1) T = 1;
  std::vector<int64_t> order(L);
  for (int64_t t = 0; t < L; ++t) order[t] = t;
  std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return a < b;
  });
  uint64_t acc = 0;
  int64_t n = 0;
  while (n < L) {
    acc += u[order[n]];
    ++n;
    if (acc >= T) break;
  }
  std::vector<int64_t> chosen(order.begin(), order.begin() + n);
  std::sort(chosen.begin(), chosen.end());
  for (int64_t i = 0; i < n; ++i) sel[i] = chosen[i];
  return n;
}

int64_t ref_attend_topp_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                             const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale,
                             float p, int d, int64_t* sel, double* out) {
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (!valid_d(d)) return -1;
  if (!(p > 0.0f && p <= 1.0f)) return -1;
  if (L <= 0) return 0;
  std::vector<uint32_t> planes(4 * (d / 32));
  float vl, dl;
  int32_t Sq;
  ref_query_prep(q, signs, d, planes.data(), &vl, &dl, &Sq, nullptr, nullptr);
  std::vector<float> s(L);
  ref_logits(bits, norm, cinv, L, planes.data(), vl, dl, Sq, scale, d, s.data());
  const int64_t n = ref_topp_select(s.data(), L, p, sel);
  double m = s[sel[0]];
  for (int64_t i = 1; i < n; ++i) m = std::max(m, static_cast<double>(s[sel[i]]));
  std::vector<double> acc(d, 0.0), vh(d);
  double l = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    const int64_t t = sel[i];
    const double e = std::exp(static_cast<double>(s[t]) - m);
    l += e;
    ref_dequant_value(codes + t * (d / 8), sm + t * (d / 32), d, vh.data());
    for (int c = 0; c < d; ++c) acc[c] += e * vh[c];
  }
  for (int c = 0; c < d; ++c) out[c] = acc[c] / l;
  return n;
}

/* RaBitQCache abstract (adaptive Top-p, and the fixed Top-k budget it is contrasted with) and the
 * H1IB-KV article, part 2 item 1 (a high-precision layer for important tokens; here the first
 * `sink` and last `recent` tokens are always kept). */
int64_t ref_select(const float* s, int64_t L, int mode, float p, int64_t k, int64_t sink, int64_t recent,
                   int64_t* sel) {
  if (mode != 0 && mode != 1) return -1;
  if (mode == 0 && !(p > 0.0f && p <= 1.0f)) return -1;
  if (mode == 1 && k < 0) return -1;
  if (sink < 0 || recent < 0) return -1;
  if (L <= 0) return 0;
  std::vector<char> win(L, 0);
  for (int64_t t = 0; t < L; ++t) win[t] = (t < sink || t >= L - recent) ? 1 : 0;
  std::vector<int64_t> order;
  for (int64_t t = 0; t < L; ++t)
    if (!win[t]) order.push_back(t);
  std::sort(order.begin(), order.end(), [&](int64_t a, int64_t b) {
    if (s[a] != s[b]) return s[a] > s[b];
    return a < b;
  });
  int64_t n_extra = 0;
  if (mode == 1) {
    n_extra = std::min<int64_t>(k, static_cast<int64_t>(order.size()));
  } else {
    float m = s[0];
    for (int64_t t = 1; t < L; ++t) m = std::max(m, s[t]);
    uint64_t U = 0, Uw = 0;
    for (int64_t t = 0; t < L; ++t) {
      const uint64_t u = ref_topp_weight(s[t], m);
      U += u;
      if (win[t]) Uw += u;
    }
    uint64_t T = static_cast<uint64_t>(std::ceil(static_cast<double>(p) * static_cast<double>(U)));
    if (T > U) T = U;
    if (T < 1) T = 1;
    if (Uw < T) {
      const uint64_t need = T - Uw;
      uint64_t acc = 0;
      while (n_extra < static_cast<int64_t>(order.size())) {
        acc += ref_topp_weight(s[order[n_extra]], m);
        ++n_extra;
        if (acc >= need) break;
      }
    }
  }
  std::vector<int64_t> chosen(order.begin(), order.begin() + n_extra);
  for (int64_t t = 0; t < L; ++t)
    if (win[t]) chosen.push_back(t);
  std::sort(chosen.begin(), chosen.end());
  for (size_t i = 0; i < chosen.size(); ++i) sel[i] = chosen[i];
  return static_cast<int64_t>(chosen.size());
}

int64_t ref_attend_select_head(const uint32_t* bits, const float* norm, const float* cinv, const uint32_t* codes,
                               const uint32_t* sm, int64_t L, const float* q, const float* signs, float scale,
                               int mode, float p, int64_t k, int64_t sink, int64_t recent, int d, int64_t* sel,
                               double* out) {
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (!valid_d(d)) return -1;
  if (L <= 0) return ref_select(nullptr, 0, mode, p, k, sink, recent, sel);
  std::vector<uint32_t> planes(4 * (d / 32));
  float vl, dl;
  int32_t Sq;
  ref_query_prep(q, signs, d, planes.data(), &vl, &dl, &Sq, nullptr, nullptr);
  std::vector<float> s(L);
  ref_logits(bits, norm, cinv, L, planes.data(), vl, dl, Sq, scale, d, s.data());
  const int64_t n = ref_select(s.data(), L, mode, p, k, sink, recent, sel);
  if (n <= 0) return n;
  double m = s[sel[0]];
  for (int64_t i = 1; i < n; ++i) m = std::max(m, static_cast<double>(s[sel[i]]));
  std::vector<double> acc(d, 0.0), vh(d);
  double l = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    const int64_t t = sel[i];
    const double e = std::exp(static_cast<double>(s[t]) - m);
    l += e;
    ref_dequant_value(codes + t * (d / 8), sm + t * (d / 32), d, vh.data());
    for (int c = 0; c < d; ++c) acc[c] += e * vh[c];
  }
  for (int c = 0; c < d; ++c) out[c] = acc[c] / l;
  return n;
}

/* RaBitQCache abstract / core idea: after the proxy scores pick the token set, attention is taken
 * over that set alone with the exact keys and values (sparse attention).  Plain fp64 softmax. */
int ref_attend_exact_selected(const float* q, const float* K, const float* V, int64_t L, int d, const int64_t* sel,
                              int64_t n, float scale, double* out) {
  if (d <= 0) return -1;
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  for (int64_t i = 0; i < n; ++i)
    if (sel[i] < 0 || sel[i] >= L) return -1;
  if (n <= 0) return 0;
  std::vector<double> z(n);
  for (int64_t i = 0; i < n; ++i) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += static_cast<double>(q[c]) * static_cast<double>(K[sel[i] * d + c]);
    z[i] = static_cast<double>(scale) * dot;
  }
  double m = z[0];
  for (int64_t i = 1; i < n; ++i) m = std::max(m, z[i]);
  double l = 0.0;
  std::vector<double> acc(d, 0.0);
  for (int64_t i = 0; i < n; ++i) {
    const double e = std::exp(z[i] - m);
    l += e;
    for (int c = 0; c < d; ++c) acc[c] += e * static_cast<double>(V[sel[i] * d + c]);
  }
  for (int c = 0; c < d; ++c) out[c] = acc[c] / l;
  return 0;
}

}  // extern "C"
