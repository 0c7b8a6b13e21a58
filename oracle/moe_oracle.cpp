// Oracle of the sparse MoE layer forward in plain C++ (FP64, OpenMP over tokens and rows).
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, plain CPU statement of what the layer
// computes; it shares no code with the CUDA library (no common header, helper or table), and
// only the tests, the smoke check and the benchmark's CPU-baseline leg may load it.
//
// Sources (cited by page title and section):
//   [PR]     vLLM PR "Day-0 support for Reflection's Beam-1.0": "Status" (router GEMM for
//            hidden 5120 -> 256 experts; the TP all-reduce fused with Beam's sandwich norms and
//            the MoE finalize), "Remaining work" (moe_finalize).
//   [RECIPE] vLLM recipe "reflection/Beam-1.0-501B-A23B": "Overview" (8 of 256 routed experts),
//            "Variants" (only the routed experts are NVFP4, run W4A4 on Blackwell; an FP8
//            checkpoint is the second variant).
//   [NEWS]   "vLLM adds day-zero Reflection Beam serving after agent-driven kernel
//            optimization": "Agents worked on the serving path" (an FP32 router kernel; fused
//            normalisation and residual kernels).
// The rest are the layer's stated conventions: softmax over all experts, renormalisation over
// the chosen k, SwiGLU experts, NVFP4 = E2M1 values with one E4M3 scale per 16 values and an
// FP32 tensor scale, post-norm RMSNorm with eps 1e-6.  Readings where the pages are silent:
// equal logits go to the lower expert index; the chosen slots are in descending weight; gate
// rows are the first I rows of the stored [2I][H] gate/up weight; no bias, clamp or shared
// expert; RMSNorm is gamma * x_hat; the output is rounded to BF16 once.  The FP8 variant is
// read as MXFP8: E4M3 values, one power-of-two scale per 32 values (the smallest 2^e with
// amax <= 448 * 2^e, e >= -127), no tensor scale.
//
// Steps of one forward, in order:
//   1  l = x W_r^T (x BF16 and W_r FP32 taken exactly, FP64 sums)            [PR], [NEWS]
//   2  p = softmax over all E; 3 the k largest p (ties: lower index), descending
//   4  w_j = p_j / sum of the chosen p                                         [RECIPE]
//   5  histogram, exclusive scan, permutation (expert-major, ascending tokens)
//   6  A1 = Q(x, alpha_a1)          7  G, U = deq(A1) deq(W_gate / W_up)^T   [RECIPE]
//   8  h = G sigmoid(G) U, rounded to FP32     9  A2 = Q(h, alpha_a2)
//  10  y = deq(A2) deq(W_down)^T   11  m = sum_j w_j y_j                      [PR]
//  12  n = m / sqrt(mean(m^2) + eps) * gamma   13  out = bf16(residual + n)   [PR], [NEWS]
//
// Number formats are decoded from their bit layouts and encoded as "the nearest value of the
// format, ties to the even code", found by a binary search over the sorted table of the
// format's values (E4M3: 1 sign, 4 exponent bits of bias 7, 3 mantissa bits, subnormal step
// 2^-9, largest 448, 0x7F NaN; E2M1: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ------------------------------------------------------------------ number formats
double e4m3_value(int code) {  // unsigned code 0..126
  const int e = (code >> 3) & 15, m = code & 7;
  if (e == 0) return std::ldexp(static_cast<double>(m), -9);
  return std::ldexp(1.0 + m / 8.0, e - 7);
}

const std::vector<double>& e4m3_table() {  // value of codes 0..126, ascending
  static const std::vector<double> t = [] {
    std::vector<double> v(127);
    for (int c = 0; c < 127; ++c) v[c] = e4m3_value(c);
    return v;
  }();
  return t;
}

// The nearest entry of an ascending table (entry index = code), ties to the even code;
// values past the last entry saturate to it.
int nearest_code(const double* table, int n, double a) {
  if (a >= table[n - 1]) return n - 1;
  const int hi = static_cast<int>(std::upper_bound(table, table + n, a) - table);  // table[hi] > a
  if (hi == 0) return 0;
  const int lo = hi - 1;
  const double dl = a - table[lo], dh = table[hi] - a;
  if (dl < dh) return lo;
  if (dh < dl) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

uint8_t e4m3_encode_unsigned(float s) {  // s >= 0, finite
  return static_cast<uint8_t>(nearest_code(e4m3_table().data(), 127, static_cast<double>(s)));
}

const double kE2m1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

uint8_t e2m1_encode(float v) {  // sign bit 3 copies the sign of v (so -0 -> 8)
  const int mag = nearest_code(kE2m1, 8, std::fabs(static_cast<double>(v)));
  return static_cast<uint8_t>(mag | (std::signbit(v) ? 8 : 0));
}

double e2m1_value(int code) { return (code & 8) ? -kE2m1[code & 7] : kE2m1[code & 7]; }

uint8_t e4m3_encode_signed(double v) {  // MXFP8 codes: sign bit 7 copies the sign of v
  const int mag = nearest_code(e4m3_table().data(), 127, std::fabs(v));
  return static_cast<uint8_t>(mag | (std::signbit(v) ? 0x80 : 0));
}

double e4m3_signed_value(int code) { return (code & 0x80) ? -e4m3_value(code & 0x7F) : e4m3_value(code & 0x7F); }

// FP64 -> the nearest BF16 value (8 significant bits), ties to even, as FP64.
double bf16_round(double z) {
  if (z == 0.0 || !std::isfinite(z)) return z;
  int ex = 0;
  std::frexp(z, &ex);                        // |z| in [2^(ex-1), 2^ex)
  const int step = std::max(ex - 8, -133);   // 8 significant bits; BF16 subnormal step 2^-133
  return std::ldexp(std::nearbyint(std::ldexp(z, -step)), step);  // default rounding: ties to even
}

uint16_t bf16_bits_of(double v) {  // v already a BF16 value
  const float f = static_cast<float>(v);
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return static_cast<uint16_t>(u >> 16);
}

double bf16_to_double(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// ------------------------------------------------------------------ quantisers
// NVFP4 Q of one row (cols % 16 == 0), every step an IEEE FP32 operation:
// s = amax / (6 alpha); S = E4M3(s); S == 0 zeroes the block; d = S alpha; q = E2M1(v / d).
void quantize_row_nvfp4(const float* v, int64_t cols, float alpha, uint8_t* packed, uint8_t* sf) {
  const float six_alpha = 6.0f * alpha;
  for (int64_t b = 0; b < cols / 16; ++b) {
    const float* blk = v + 16 * b;
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(blk[i]));
    const float s = amax / six_alpha;
    const uint8_t scode = e4m3_encode_unsigned(s);
    sf[b] = scode;
    uint8_t q[16];
    if (scode == 0) {
      std::memset(q, 0, 16);
    } else {
      const float d = static_cast<float>(e4m3_value(scode)) * alpha;
      for (int i = 0; i < 16; ++i) q[i] = e2m1_encode(blk[i] / d);
    }
    for (int i = 0; i < 8; ++i) packed[8 * b + i] = static_cast<uint8_t>((q[2 * i] & 15) | ((q[2 * i + 1] & 15) << 4));
  }
}

void dequantize_row_nvfp4(const uint8_t* packed, const uint8_t* sf, int64_t cols, float alpha, double* out) {
  for (int64_t j = 0; j < cols; ++j) {
    const int code = (j & 1) ? (packed[j / 2] >> 4) : (packed[j / 2] & 15);
    out[j] = e2m1_value(code) * e4m3_value(sf[j / 16]) * static_cast<double>(alpha);
  }
}

// MXFP8 of one row (cols % 32 == 0): X = 2^e, e the smallest integer with amax <= 448 2^e
// (at least -127); q = E4M3(v / X) with v / X exact; scale byte e + 127.
void quantize_row_mxfp8(const float* v, int64_t cols, uint8_t* codes, uint8_t* sf) {
  for (int64_t b = 0; b < cols / 32; ++b) {
    const float* blk = v + 32 * b;
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(static_cast<double>(blk[i])));
    int e = -127;
    while (amax > std::ldexp(448.0, e)) ++e;  // the smallest e that holds amax
    sf[b] = static_cast<uint8_t>(e + 127);
    for (int i = 0; i < 32; ++i) codes[32 * b + i] = e4m3_encode_signed(std::ldexp(static_cast<double>(blk[i]), -e));
  }
}

void dequantize_row_mxfp8(const uint8_t* codes, const uint8_t* sf, int64_t cols, double* out) {
  for (int64_t j = 0; j < cols; ++j) out[j] = e4m3_signed_value(codes[j]) * std::ldexp(1.0, sf[j / 32] - 127);
}

}  // namespace

// ------------------------------------------------------------------ C ABI
extern "C" {

typedef int (*orc_expert_fp32_fn)(void* ctx, int32_t expert, float* w_gu, float* w_d);

uint8_t orc_e4m3_encode(float s) { return e4m3_encode_unsigned(s); }
double orc_e4m3_decode(uint8_t c) { return e4m3_value(c & 0x7F); }
uint8_t orc_e2m1_encode(float v) { return e2m1_encode(v); }
double orc_e2m1_decode(uint8_t c) { return e2m1_value(c & 15); }
uint8_t orc_e4m3_encode_signed(float v) { return e4m3_encode_signed(static_cast<double>(v)); }
double orc_bf16_round(double z) { return bf16_round(z); }

// Tensor scale of a weight tensor: fl32(amax / 2688), 2688 = 6 * 448.
float orc_tensor_scale(const float* w, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::max(amax, std::fabs(w[i]));
  return amax / 2688.0f;
}

void orc_quantize_nvfp4(const float* v, int64_t rows, int64_t cols, float alpha, uint8_t* packed, uint8_t* sf) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) quantize_row_nvfp4(v + r * cols, cols, alpha, packed + r * cols / 2, sf + r * cols / 16);
}

void orc_quantize_mxfp8(const float* v, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* sf) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) quantize_row_mxfp8(v + r * cols, cols, codes + r * cols, sf + r * cols / 32);
}

// Steps 1-4 for T tokens: logits [T][E] (FP64), ids [T][k], w [T][k] (FP64) and near_tie[T]
// (the k-th and (k+1)-th largest logits differ by less than 1e-5 max(|l_k|, |l_k+1|, 1)).
void orc_route(const uint16_t* x, const float* router_w, int32_t T, int32_t H, int32_t E, int32_t k, double* logits,
               int32_t* ids, double* w, uint8_t* near_tie) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int32_t t = 0; t < T; ++t) {
    double* l = logits + static_cast<int64_t>(t) * E;
    for (int32_t e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int32_t h = 0; h < H; ++h)
        acc += bf16_to_double(x[static_cast<int64_t>(t) * H + h]) * static_cast<double>(router_w[static_cast<int64_t>(e) * H + h]);
      l[e] = acc;
    }
    double lmax = l[0];
    for (int32_t e = 1; e < E; ++e) lmax = std::max(lmax, l[e]);
    std::vector<double> p(E);
    double z = 0.0;
    for (int32_t e = 0; e < E; ++e) z += (p[e] = std::exp(l[e] - lmax));
    for (int32_t e = 0; e < E; ++e) p[e] /= z;
    std::vector<int32_t> order(E);
    for (int32_t e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return p[a] > p[b]; });
    double psum = 0.0;
    for (int32_t j = 0; j < k; ++j) psum += p[order[j]];
    for (int32_t j = 0; j < k; ++j) {
      ids[static_cast<int64_t>(t) * k + j] = order[j];
      w[static_cast<int64_t>(t) * k + j] = p[order[j]] / psum;
    }
    if (k < E) {
      std::vector<double> s(l, l + E);
      std::sort(s.begin(), s.end(), [](double a, double b) { return a > b; });
      const double a = s[k - 1], b = s[k];
      near_tie[t] = (a - b) < 1e-5 * std::max(std::max(std::fabs(a), std::fabs(b)), 1.0);
    } else {
      near_tie[t] = 0;
    }
  }
}

// Step 5: counts [E], offsets [E + 1], perm_src / perm_slot [T k] (token and slot of each
// permuted row: expert-major, ascending tokens within an expert), inv [T][k].
void orc_permute(const int32_t* ids, int32_t T, int32_t k, int32_t E, int64_t* counts, int64_t* offsets, int32_t* perm_src,
                 int32_t* perm_slot, int32_t* inv) {
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < static_cast<int64_t>(T) * k; ++i) ++counts[ids[i]];
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int64_t> fill(offsets, offsets + E);
  for (int32_t t = 0; t < T; ++t)      // ascending tokens ...
    for (int32_t j = 0; j < k; ++j) {  // ... each token's slots in order
      const int32_t e = ids[static_cast<int64_t>(t) * k + j];
      const int64_t r = fill[e]++;
      perm_src[r] = t;
      perm_slot[r] = j;
      inv[static_cast<int64_t>(t) * k + j] = static_cast<int32_t>(r);
    }
}

// The whole forward for T tokens (steps 1-4 and 6-13).  fmt 0: NVFP4 (alpha_a1, alpha_a2
// used); fmt 1: MXFP8.  Expert weights come as FP32 (w_gu [2I][H], rows 0..I-1 gate; w_d
// [H][I]) from get(ctx, e) and are quantised here with this oracle's quantisers (NVFP4
// tensor scales amax / 2688).  Outputs: ids [T][k], w [T][k], near_tie [T], m [T][H] (may be
// null), out_pre [T][H] (FP64, before rounding), out_bf16 [T][H] (BF16 bits).  Returns 0, or
// nonzero if get() failed.
int orc_moe_forward(int32_t T, int32_t H, int32_t E, int32_t k, int32_t I, int32_t fmt, const uint16_t* x,
                    const uint16_t* residual, const float* router_w, const uint16_t* gamma, float alpha_a1,
                    float alpha_a2, double eps, orc_expert_fp32_fn get, void* ctx, int32_t* ids, double* w,
                    uint8_t* near_tie, double* m_out, double* out_pre, uint16_t* out_bf16) {
  const bool mx = fmt == 1;
  std::vector<double> logits(static_cast<size_t>(T) * E);
  orc_route(x, router_w, T, H, E, k, logits.data(), ids, w, near_tie);
  // step 6: A1 of every token, dequantised (a token's k rows share it)
  std::vector<float> x32(static_cast<size_t>(T) * H);
  for (size_t i = 0; i < x32.size(); ++i) x32[i] = static_cast<float>(bf16_to_double(x[i]));
  std::vector<double> a1(static_cast<size_t>(T) * H);
  {
    std::vector<uint8_t> codes(static_cast<size_t>(T) * H), sf(static_cast<size_t>(T) * H / 16);
    for (int32_t t = 0; t < T; ++t) {
      const float* row = x32.data() + static_cast<size_t>(t) * H;
      if (mx) {
        quantize_row_mxfp8(row, H, codes.data() + static_cast<size_t>(t) * H, sf.data() + static_cast<size_t>(t) * H / 32);
        dequantize_row_mxfp8(codes.data() + static_cast<size_t>(t) * H, sf.data() + static_cast<size_t>(t) * H / 32, H,
                             a1.data() + static_cast<size_t>(t) * H);
      } else {
        quantize_row_nvfp4(row, H, alpha_a1, codes.data() + static_cast<size_t>(t) * H / 2,
                           sf.data() + static_cast<size_t>(t) * H / 16);
        dequantize_row_nvfp4(codes.data() + static_cast<size_t>(t) * H / 2, sf.data() + static_cast<size_t>(t) * H / 16, H,
                             alpha_a1, a1.data() + static_cast<size_t>(t) * H);
      }
    }
  }
  // steps 7-11, expert by expert over the tokens that chose it
  std::vector<double> m(static_cast<size_t>(T) * H, 0.0);
  std::vector<float> wgu(static_cast<size_t>(2) * I * H), wd(static_cast<size_t>(H) * I);
  std::vector<double> dgu(static_cast<size_t>(2) * I * H), dd(static_cast<size_t>(H) * I);
  for (int32_t e = 0; e < E; ++e) {
    std::vector<std::pair<int32_t, double>> rows;  // (token, routing weight)
    for (int32_t t = 0; t < T; ++t)
      for (int32_t j = 0; j < k; ++j)
        if (ids[static_cast<int64_t>(t) * k + j] == e) rows.emplace_back(t, w[static_cast<int64_t>(t) * k + j]);
    if (rows.empty()) continue;
    if (get(ctx, e, wgu.data(), wd.data()) != 0) return 1;
    // this oracle's quantisation of the expert, then its exact FP64 values
    if (mx) {
      std::vector<uint8_t> c(static_cast<size_t>(2) * I * H), s(static_cast<size_t>(2) * I * H / 32);
      orc_quantize_mxfp8(wgu.data(), 2 * I, H, c.data(), s.data());
#pragma omp parallel for schedule(static)
      for (int64_t r = 0; r < 2 * I; ++r) dequantize_row_mxfp8(c.data() + r * H, s.data() + r * H / 32, H, dgu.data() + r * H);
      std::vector<uint8_t> c2(static_cast<size_t>(H) * I), s2(static_cast<size_t>(H) * I / 32);
      orc_quantize_mxfp8(wd.data(), H, I, c2.data(), s2.data());
#pragma omp parallel for schedule(static)
      for (int64_t r = 0; r < H; ++r) dequantize_row_mxfp8(c2.data() + r * I, s2.data() + r * I / 32, I, dd.data() + r * I);
    } else {
      const float a_gu = orc_tensor_scale(wgu.data(), static_cast<int64_t>(2) * I * H);
      const float a_d = orc_tensor_scale(wd.data(), static_cast<int64_t>(H) * I);
      std::vector<uint8_t> c(static_cast<size_t>(I) * H), s(static_cast<size_t>(2) * I * H / 16);
      orc_quantize_nvfp4(wgu.data(), 2 * I, H, a_gu, c.data(), s.data());
#pragma omp parallel for schedule(static)
      for (int64_t r = 0; r < 2 * I; ++r)
        dequantize_row_nvfp4(c.data() + r * H / 2, s.data() + r * H / 16, H, a_gu, dgu.data() + r * H);
      std::vector<uint8_t> c2(static_cast<size_t>(H) * I / 2), s2(static_cast<size_t>(H) * I / 16);
      orc_quantize_nvfp4(wd.data(), H, I, a_d, c2.data(), s2.data());
#pragma omp parallel for schedule(static)
      for (int64_t r = 0; r < H; ++r) dequantize_row_nvfp4(c2.data() + r * I / 2, s2.data() + r * I / 16, I, a_d, dd.data() + r * I);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < static_cast<int64_t>(rows.size()); ++q) {
      const int32_t t = rows[q].first;
      const double* a = a1.data() + static_cast<size_t>(t) * H;
      std::vector<float> h32(I);
      for (int32_t f = 0; f < I; ++f) {  // steps 7-8
        const double* wg = dgu.data() + static_cast<size_t>(f) * H;
        const double* wu = dgu.data() + static_cast<size_t>(I + f) * H;
        double g = 0.0, u = 0.0;
        for (int32_t hh = 0; hh < H; ++hh) {
          g += a[hh] * wg[hh];
          u += a[hh] * wu[hh];
        }
        h32[f] = static_cast<float>(g / (1.0 + std::exp(-g)) * u);
      }
      std::vector<double> a2(I);  // step 9
      if (mx) {
        std::vector<uint8_t> c(I), s(I / 32);
        quantize_row_mxfp8(h32.data(), I, c.data(), s.data());
        dequantize_row_mxfp8(c.data(), s.data(), I, a2.data());
      } else {
        std::vector<uint8_t> c(I / 2), s(I / 16);
        quantize_row_nvfp4(h32.data(), I, alpha_a2, c.data(), s.data());
        dequantize_row_nvfp4(c.data(), s.data(), I, alpha_a2, a2.data());
      }
      double* mt = m.data() + static_cast<size_t>(t) * H;  // steps 10-11 (each token once per expert)
      for (int32_t n = 0; n < H; ++n) {
        const double* wrow = dd.data() + static_cast<size_t>(n) * I;
        double y = 0.0;
        for (int32_t f = 0; f < I; ++f) y += a2[f] * wrow[f];
        mt[n] += rows[q].second * y;
      }
    }
  }
  // steps 12-13
#pragma omp parallel for schedule(static)
  for (int32_t t = 0; t < T; ++t) {
    const double* mt = m.data() + static_cast<size_t>(t) * H;
    double ss = 0.0;
    for (int32_t n = 0; n < H; ++n) ss += mt[n] * mt[n];
    const double rms = std::sqrt(ss / H + eps);
    for (int32_t n = 0; n < H; ++n) {
      const size_t i = static_cast<size_t>(t) * H + n;
      const double pre = bf16_to_double(residual[i]) + mt[n] / rms * bf16_to_double(gamma[n]);
      out_pre[i] = pre;
      out_bf16[i] = bf16_bits_of(bf16_round(pre));
      if (m_out) m_out[i] = mt[n];
    }
  }
  return 0;
}

}  // extern "C"
