// moe_oracle.cpp -- plain fp64 CPU oracle for the W4A8 MoE decode step.
//
// TEST INFRASTRUCTURE ONLY: used by the test suite, the smoke check and the
// benchmark's CPU-baseline leg, never by the product path. Shares no code with
// the CUDA library. See moe_oracle.h for sources, layouts and pin status.
//
// Build: g++ -std=c++17 -O2 -ffp-contract=off -fPIC -shared (no fast-math, so
// float arithmetic is IEEE round-to-nearest-even on SSE).
#include "moe_oracle.h"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <vector>

namespace {

const double kNaN = std::numeric_limits<double>::quiet_NaN();

// Nibble j (0-based, along K) of a packed E2M1 row: byte j/2, low nibble for
// even j, high nibble for odd j (layout stated in moe_oracle.h).
int nibble(const uint8_t* row, int j) {
  uint8_t b = row[j / 2];
  return (j % 2 == 0) ? (b & 0xF) : (b >> 4);
}

// Decoded MXFP4 weight element [MX]: E2M1 value times the block's E8M0 scale.
double mx_element(const uint8_t* codes_row, const uint8_t* scales_row, int j) {
  return oracle_e2m1_value(nibble(codes_row, j)) *
         oracle_e8m0_value(scales_row[j / 32]);
}

bool has_nan_scale(const uint8_t* scales, size_t n) {
  for (size_t i = 0; i < n; ++i)
    if (scales[i] == 0xFF) return true;
  return false;
}

}  // namespace

extern "C" {

// [MX] E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN.
// Exponent field 0 is subnormal: value = m * 2^(1-1) * 0.5.
double oracle_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// [MX] E8M0: an 8-bit biased exponent, value 2^(b-127); 0xFF encodes NaN.
double oracle_e8m0_value(int byte) {
  if (byte == 0xFF) return kNaN;
  return std::ldexp(1.0, byte - 127);
}

// [OFP8] E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.
// Exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities.
double oracle_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0xF && m == 7) return kNaN;
  double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// [OFP8] E4M3 encode with round-to-nearest-even and saturation to the largest
// finite magnitude (448). Written as a nearest-value search over the 127
// non-negative finite codes 0x00..0x7E; consecutive codes are consecutive
// values, so "even" on a tie is the code with mantissa bit 0 clear.
int oracle_e4m3_encode(float v) {
  if (std::isnan(v)) return 0x7F;
  int sign = std::signbit(v) ? 0x80 : 0x00;
  double a = std::fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  int best = 0;
  double best_err = a;  // distance to code 0 (value 0)
  for (int c = 1; c <= 0x7E; ++c) {
    double err = std::fabs(a - oracle_e4m3_value(c));
    if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      best_err = err;
    }
  }
  return sign | best;
}

// bfloat16: the upper 16 bits of an IEEE fp32.
double oracle_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round an fp64 value to the nearest bf16 (ties to even), by comparing the
// two bf16 neighbours that bracket it. Values beyond the finite range become
// +-Inf; NaN stays NaN.
uint16_t oracle_bf16_round(double v) {
  if (std::isnan(v)) return 0x7FC0;
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  // Largest bf16 whose magnitude is <= a: search the 0x7F80 positive patterns
  // by bisection (monotone in the bit pattern).
  uint32_t lo = 0, hi = 0x7F80;  // 0x7F80 = +Inf
  while (hi - lo > 1) {
    uint32_t mid = (lo + hi) / 2;
    if (oracle_bf16_value((uint16_t)mid) <= a) lo = mid; else hi = mid;
  }
  double vlo = oracle_bf16_value((uint16_t)lo);
  if (vlo == a) return sign | (uint16_t)lo;
  // Upper neighbour: pattern lo+1; the step after the largest finite bf16
  // (0x7F7F) is Inf, rounded as if the exponent range continued.
  double vhi = (lo + 1 == 0x7F80) ? std::ldexp(1.0, 128) : oracle_bf16_value((uint16_t)(lo + 1));
  double dlo = a - vlo, dhi = vhi - a;
  uint32_t pick = (dlo < dhi) ? lo : (dhi < dlo) ? lo + 1 : ((lo & 1) ? lo + 1 : lo);
  return sign | (uint16_t)pick;
}

// A1 -- per-token FP8 E4M3 activation quantisation ("W4A8": 4-bit weights,
// 8-bit activations [MTP "Why is MoE decoding ... memory-bound?"]).
// amax = max|x|; inv = fl32(448/amax); code = E4M3_RNE_sat(fl32(x*inv));
// s = fl32(amax/448). Both fl32 steps are IEEE fp32 so codes are exact.
// amax == 0 gives all-zero codes and s = 1.
int oracle_quantize(int M, int H, const uint16_t* x, uint8_t* q, float* s) {
  if (M < 0 || H <= 0 || (!x && M > 0)) return -1;
  for (int m = 0; m < M; ++m) {
    const uint16_t* xm = x + (size_t)m * H;
    float amax = 0.0f;
    for (int h = 0; h < H; ++h) amax = std::max(amax, (float)std::fabs(oracle_bf16_value(xm[h])));
    if (amax == 0.0f) {
      for (int h = 0; h < H; ++h) q[(size_t)m * H + h] = 0;
      s[m] = 1.0f;
      continue;
    }
    volatile float inv = 448.0f / amax;  // fp32 division, round to nearest even
    for (int h = 0; h < H; ++h) {
      volatile float v = (float)oracle_bf16_value(xm[h]) * inv;  // fp32 multiply
      q[(size_t)m * H + h] = (uint8_t)oracle_e4m3_encode(v);
    }
    volatile float sm = amax / 448.0f;
    s[m] = sm;
  }
  return 0;
}

// A2 -- router logits l[m][e] = sum_h x[m][h] * Wr[e][h], fp64, from the bf16
// activations (not the FP8 codes).
int oracle_router_logits(int M, int H, int E, const uint16_t* x,
                         const float* router_w, double* logits) {
  if (M < 0 || H <= 0 || E <= 0) return -1;
  for (int m = 0; m < M; ++m)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += oracle_bf16_value(x[(size_t)m * H + h]) * (double)router_w[(size_t)e * H + h];
      logits[(size_t)m * E + e] = acc;
    }
  return 0;
}

// A3 -- top-k of E routed experts per token ("routes a token to 8 of ...
// routed experts" [MTP "What is Ling 3.0 ..."]). Ranked by logit descending,
// ties to the lower expert index; weights are a softmax over the k kept
// logits, so they sum to 1.
int oracle_topk(int M, int E, int k, const double* logits, int32_t* ids, double* weights) {
  if (M < 0 || E <= 0 || k <= 0 || k > E) return -1;
  std::vector<int> order(E);
  for (int m = 0; m < M; ++m) {
    const double* l = logits + (size_t)m * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [&](int a, int b) {
      if (l[a] != l[b]) return l[a] > l[b];
      return a < b;
    });
    double lmax = l[order[0]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += std::exp(l[order[j]] - lmax);
    for (int j = 0; j < k; ++j) {
      ids[(size_t)m * k + j] = order[j];
      weights[(size_t)m * k + j] = std::exp(l[order[j]] - lmax) / z;
    }
  }
  return 0;
}

// A4 -- the expert union over M tokens. A 4-token verify step can touch as
// many as 32 distinct experts where a single token touches 8 [MTP "What are
// the 3 optimizations?"].
int oracle_union(int M, int E, int k, const int32_t* ids, int32_t* union_ids,
                 int32_t* pair_off, int32_t* pair_tok, int32_t* pair_slot) {
  if (M < 0 || E <= 0 || k <= 0) return -1;
  std::vector<int> count(E, 0);
  for (int i = 0; i < M * k; ++i) {
    if (ids[i] < 0 || ids[i] >= E) return -2;
    count[ids[i]]++;
  }
  int U = 0;
  for (int e = 0; e < E; ++e)
    if (count[e] > 0) union_ids[U++] = e;
  int pos = 0;
  for (int u = 0; u < U; ++u) {
    pair_off[u] = pos;
    for (int m = 0; m < M; ++m)
      for (int j = 0; j < k; ++j)
        if (ids[(size_t)m * k + j] == union_ids[u]) {
          pair_tok[pos] = m;
          pair_slot[pos] = j;
          ++pos;
        }
  }
  pair_off[U] = pos;
  return U;
}

// A5-A7 -- one token through one MXFP4 expert, fp64:
//   g_n  = s * sum_h W13[n][h]   * e4m3(q[h])   (gate, n < I)
//   up_n = s * sum_h W13[I+n][h] * e4m3(q[h])   (up)
//   h_n  = silu(g_n) * up_n, silu(z) = z / (1 + e^-z)  (no requantisation)
//   d_r  = sum_n W2[r][n] * h_n
// with W = E2M1(code) * 2^(E8M0 - 127) per block of 32 along K [MX].
int oracle_expert(int H, int I, const uint8_t* q_m, float s_m,
                  const uint8_t* w13_codes, const uint8_t* w13_scales,
                  const uint8_t* w2_codes, const uint8_t* w2_scales,
                  double* h_out, double* d_out) {
  if (H <= 0 || I <= 0 || H % 32 || I % 32) return -1;
  if (!q_m || !w13_codes || !w13_scales || !w2_codes || !w2_scales || !d_out) return -1;
  if (has_nan_scale(w13_scales, (size_t)2 * I * (H / 32)) ||
      has_nan_scale(w2_scales, (size_t)H * (I / 32)))
    return -3;
  std::vector<double> a(H), hv(I);
  for (int j = 0; j < H; ++j) a[j] = oracle_e4m3_value(q_m[j]);
  for (int n = 0; n < I; ++n) {
    double g = 0.0, u = 0.0;
    const uint8_t* gc = w13_codes + (size_t)n * (H / 2);
    const uint8_t* gs = w13_scales + (size_t)n * (H / 32);
    const uint8_t* uc = w13_codes + (size_t)(I + n) * (H / 2);
    const uint8_t* us = w13_scales + (size_t)(I + n) * (H / 32);
    for (int j = 0; j < H; ++j) {
      g += mx_element(gc, gs, j) * a[j];
      u += mx_element(uc, us, j) * a[j];
    }
    g *= (double)s_m;
    u *= (double)s_m;
    hv[n] = g / (1.0 + std::exp(-g)) * u;
  }
  for (int r = 0; r < H; ++r) {
    const uint8_t* dc = w2_codes + (size_t)r * (I / 2);
    const uint8_t* ds = w2_scales + (size_t)r * (I / 32);
    double acc = 0.0;
    for (int n = 0; n < I; ++n) acc += mx_element(dc, ds, n) * hv[n];
    d_out[r] = acc;
  }
  if (h_out)
    for (int n = 0; n < I; ++n) h_out[n] = hv[n];
  return 0;
}

// A1-A8 -- the whole decode step; A8 combines y[m] = sum_slot w[m][slot] *
// d[m][slot] in fp64 and also rounds it to bf16.
int oracle_moe_decode(int H, int I, int E, int k, int M,
                      const uint16_t* x, const float* router_w,
                      const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                      const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                      uint8_t* q, float* s, double* logits, int32_t* ids,
                      double* weights, double* y64, uint16_t* y_bf16) {
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || M < 0 || !y64) return -1;
  std::vector<uint8_t> qv((size_t)M * H);
  std::vector<float> sv(M);
  std::vector<double> lv((size_t)M * E), wv((size_t)M * k), d(H);
  std::vector<int32_t> iv((size_t)M * k);
  int rc = oracle_quantize(M, H, x, qv.data(), sv.data());
  if (rc) return rc;
  rc = oracle_router_logits(M, H, E, x, router_w, lv.data());
  if (rc) return rc;
  rc = oracle_topk(M, E, k, lv.data(), iv.data(), wv.data());
  if (rc) return rc;
  for (int m = 0; m < M; ++m) {
    for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] = 0.0;
    for (int j = 0; j < k; ++j) {
      int e = iv[(size_t)m * k + j];
      rc = oracle_expert(H, I, qv.data() + (size_t)m * H, sv[m], w13_codes[e], w13_scales[e],
                         w2_codes[e], w2_scales[e], nullptr, d.data());
      if (rc) return rc;
      double w = wv[(size_t)m * k + j];
      for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] += w * d[r];
    }
  }
  if (q) std::memcpy(q, qv.data(), qv.size());
  if (s) std::memcpy(s, sv.data(), sv.size() * sizeof(float));
  if (logits) std::memcpy(logits, lv.data(), lv.size() * sizeof(double));
  if (ids) std::memcpy(ids, iv.data(), iv.size() * sizeof(int32_t));
  if (weights) std::memcpy(weights, wv.data(), wv.size() * sizeof(double));
  if (y_bf16)
    for (size_t i = 0; i < (size_t)M * H; ++i) y_bf16[i] = oracle_bf16_round(y64[i]);
  return 0;
}

// The routed step, then the shared expert's output added with weight 1.
int oracle_moe_decode_shared(int H, int I, int E, int k, int M,
                             const uint16_t* x, const float* router_w,
                             const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                             const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                             const uint8_t* sh_w13_codes, const uint8_t* sh_w13_scales,
                             const uint8_t* sh_w2_codes, const uint8_t* sh_w2_scales,
                             uint8_t* q, float* s, double* logits, int32_t* ids, double* weights,
                             double* y64) {
  if (!sh_w13_codes || !sh_w13_scales || !sh_w2_codes || !sh_w2_scales || M < 0 || H <= 0) return -1;
  std::vector<uint8_t> qv((size_t)M * H);
  std::vector<float> sv(M);
  int rc = oracle_moe_decode(H, I, E, k, M, x, router_w, w13_codes, w13_scales, w2_codes, w2_scales,
                             qv.data(), sv.data(), logits, ids, weights, y64, nullptr);
  if (rc) return rc;
  if (q) std::copy(qv.begin(), qv.end(), q);
  if (s) std::copy(sv.begin(), sv.end(), s);
  std::vector<double> d(H);
  for (int m = 0; m < M; ++m) {
    rc = oracle_expert(H, I, qv.data() + (size_t)m * H, sv[m], sh_w13_codes, sh_w13_scales, sh_w2_codes,
                       sh_w2_scales, nullptr, d.data());
    if (rc) return rc;
    for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] += d[r];
  }
  return 0;
}

// The A1 steps of oracle_quantize, on fp32 input.
int oracle_quantize_f32(int n, const float* v, uint8_t* q, float* s) {
  if (n <= 0 || !v || !q || !s) return -1;
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0f) {
    for (int i = 0; i < n; ++i) q[i] = 0;
    *s = 1.0f;
    return 0;
  }
  volatile float inv = 448.0f / amax;  // fp32 division, round to nearest even
  for (int i = 0; i < n; ++i) {
    volatile float t = v[i] * inv;  // fp32 multiply
    q[i] = (uint8_t)oracle_e4m3_encode(t);
  }
  volatile float sm = amax / 448.0f;
  *s = sm;
  return 0;
}

// h in fp64 from oracle_expert, rounded to fp32, quantised; then the down
// projection of the dequantised codes in fp64.
int oracle_expert_a8(int H, int I, const uint8_t* q_m, float s_m,
                     const uint8_t* w13_codes, const uint8_t* w13_scales,
                     const uint8_t* w2_codes, const uint8_t* w2_scales,
                     uint8_t* hq_out, float* hs_out, double* d_out) {
  if (!d_out || H <= 0 || I <= 0) return -1;
  std::vector<double> h(I), dtmp(H);
  int rc = oracle_expert(H, I, q_m, s_m, w13_codes, w13_scales, w2_codes, w2_scales, h.data(), dtmp.data());
  if (rc) return rc;
  std::vector<float> hf(I);
  for (int n = 0; n < I; ++n) hf[n] = (float)h[n];
  std::vector<uint8_t> hq(I);
  float hs = 1.0f;
  rc = oracle_quantize_f32(I, hf.data(), hq.data(), &hs);
  if (rc) return rc;
  std::vector<double> hd(I);
  for (int n = 0; n < I; ++n) hd[n] = oracle_e4m3_value(hq[n]);
  for (int r = 0; r < H; ++r) {
    const uint8_t* dc = w2_codes + (size_t)r * (I / 2);
    const uint8_t* ds = w2_scales + (size_t)r * (I / 32);
    double acc = 0.0;
    for (int n = 0; n < I; ++n) acc += mx_element(dc, ds, n) * hd[n];
    d_out[r] = (double)hs * acc;
  }
  if (hq_out) std::copy(hq.begin(), hq.end(), hq_out);
  if (hs_out) *hs_out = hs;
  return 0;
}

// A1-A4 as in oracle_moe_decode, then every expert through oracle_expert_a8;
// y = sum_slot w * d (+ the shared expert's d with weight 1).
int oracle_moe_decode_a8(int H, int I, int E, int k, int M,
                         const uint16_t* x, const float* router_w,
                         const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                         const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                         const uint8_t* sh_w13_codes, const uint8_t* sh_w13_scales,
                         const uint8_t* sh_w2_codes, const uint8_t* sh_w2_scales,
                         uint8_t* q, float* s, double* logits, int32_t* ids, double* weights,
                         double* y64) {
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || M < 0 || !y64) return -1;
  const bool shared = sh_w13_codes || sh_w13_scales || sh_w2_codes || sh_w2_scales;
  if (shared && !(sh_w13_codes && sh_w13_scales && sh_w2_codes && sh_w2_scales)) return -1;
  std::vector<uint8_t> qv((size_t)M * H);
  std::vector<float> sv(M);
  std::vector<double> lv((size_t)M * E), wv((size_t)M * k), d(H);
  std::vector<int32_t> iv((size_t)M * k);
  int rc = oracle_quantize(M, H, x, qv.data(), sv.data());
  if (rc) return rc;
  rc = oracle_router_logits(M, H, E, x, router_w, lv.data());
  if (rc) return rc;
  rc = oracle_topk(M, E, k, lv.data(), iv.data(), wv.data());
  if (rc) return rc;
  for (int m = 0; m < M; ++m) {
    const uint8_t* qm = qv.data() + (size_t)m * H;
    for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] = 0.0;
    for (int j = 0; j < k; ++j) {
      const int e = iv[(size_t)m * k + j];
      rc = oracle_expert_a8(H, I, qm, sv[m], w13_codes[e], w13_scales[e], w2_codes[e], w2_scales[e], nullptr,
                            nullptr, d.data());
      if (rc) return rc;
      const double w = wv[(size_t)m * k + j];
      for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] += w * d[r];
    }
    if (shared) {
      rc = oracle_expert_a8(H, I, qm, sv[m], sh_w13_codes, sh_w13_scales, sh_w2_codes, sh_w2_scales, nullptr,
                            nullptr, d.data());
      if (rc) return rc;
      for (int r = 0; r < H; ++r) y64[(size_t)m * H + r] += d[r];
    }
  }
  if (q) std::copy(qv.begin(), qv.end(), q);
  if (s) std::copy(sv.begin(), sv.end(), s);
  if (logits) std::copy(lv.begin(), lv.end(), logits);
  if (ids) std::copy(iv.begin(), iv.end(), ids);
  if (weights) std::copy(wv.begin(), wv.end(), weights);
  return 0;
}

// Brute force over all E experts: expert e is kept for token m when fewer
// than k experts rank above it (higher logit, or equal logit and lower index);
// the kept experts' weights are exp(l_e - max) renormalised over the kept set.
int oracle_moe_dense(int H, int I, int E, int k, int M,
                     const uint16_t* x, const float* router_w,
                     const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                     const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                     double* y64) {
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || M < 0 || !y64) return -1;
  std::vector<uint8_t> qv((size_t)M * H);
  std::vector<float> sv(M);
  std::vector<double> lv((size_t)M * E), d((size_t)E * H);
  int rc = oracle_quantize(M, H, x, qv.data(), sv.data());
  if (rc) return rc;
  rc = oracle_router_logits(M, H, E, x, router_w, lv.data());
  if (rc) return rc;
  for (int m = 0; m < M; ++m) {
    const double* l = lv.data() + (size_t)m * E;
    for (int e = 0; e < E; ++e) {
      rc = oracle_expert(H, I, qv.data() + (size_t)m * H, sv[m], w13_codes[e], w13_scales[e],
                         w2_codes[e], w2_scales[e], nullptr, d.data() + (size_t)e * H);
      if (rc) return rc;
    }
    std::vector<int> keep(E, 0);
    double lmax = -std::numeric_limits<double>::infinity();
    for (int e = 0; e < E; ++e) lmax = std::max(lmax, l[e]);
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      int above = 0;
      for (int f = 0; f < E; ++f)
        if (l[f] > l[e] || (l[f] == l[e] && f < e)) ++above;
      keep[e] = above < k;
      if (keep[e]) z += std::exp(l[e] - lmax);
    }
    for (int r = 0; r < H; ++r) {
      double acc = 0.0;
      for (int e = 0; e < E; ++e)
        acc += keep[e] ? (std::exp(l[e] - lmax) / z) * d[(size_t)e * H + r] : 0.0;
      y64[(size_t)m * H + r] = acc;
    }
  }
  return 0;
}

// A9 -- RMSNorm with unit weight between stacked layers, fp64, rounded to
// bf16: out = y / sqrt(mean(y^2) + eps).
int oracle_rmsnorm(int M, int H, const uint16_t* y, double eps, uint16_t* out) {
  if (M < 0 || H <= 0) return -1;
  for (int m = 0; m < M; ++m) {
    double ss = 0.0;
    for (int h = 0; h < H; ++h) {
      double v = oracle_bf16_value(y[(size_t)m * H + h]);
      ss += v * v;
    }
    double r = 1.0 / std::sqrt(ss / H + eps);
    for (int h = 0; h < H; ++h)
      out[(size_t)m * H + h] = oracle_bf16_round(oracle_bf16_value(y[(size_t)m * H + h]) * r);
  }
  return 0;
}

// FP8 LM head: per-row quantisation is the A1 rule applied to each row of
// the output matrix (one fp32 scale per row, the reading stated in
// moe_oracle.h).
int oracle_lm_quantize(int V, int H, const uint16_t* w, uint8_t* codes, float* scales) {
  if (V < 0 || H <= 0 || !w || !codes || !scales) return -1;
  return oracle_quantize(V, H, w, codes, scales);
}

// logits[m][v] = s_v * sum_h e4m3(code[v][h]) * x[m][h], fp64.
int oracle_lm_head(int V, int H, int M, const uint8_t* codes, const float* scales, const uint16_t* x,
                   double* logits) {
  if (V < 0 || H <= 0 || M < 0 || !codes || !scales || !x || !logits) return -1;
  for (int m = 0; m < M; ++m)
    for (int v = 0; v < V; ++v) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += oracle_e4m3_value(codes[(size_t)v * H + h]) * oracle_bf16_value(x[(size_t)m * H + h]);
      logits[(size_t)m * V + v] = acc * (double)scales[v];
    }
  return 0;
}

}  // extern "C"
