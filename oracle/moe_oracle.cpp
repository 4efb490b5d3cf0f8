// The MoE decode layer in plain C++17, float64 -- TEST INFRASTRUCTURE ONLY.
//
// Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg load
// this library (oracle/liboracle.so, through oracle/cpp.py); the product
// path never does, and this file shares no code with the CUDA library.  It
// computes what oracle/moe.py computes, step by step, written from the same
// definitions:
//
//  * routing: 8 of 512 routed experts plus 1 shared expert per MoE layer
//    ("NVIDIA 在单台 DGX Spark 上叠加三项优化，Ling-3.0-flash 的 MoE 推理吞吐提升
//    42.5%", tanhow.com, section "Ling 3.0 是什么", sparse-MoE bullet);
//  * the W4A8 recipe, MXFP4 weights and 8-bit activations (same page,
//    "为什么 DGX Spark 上的 MoE 解码是内存受限的？"; devotd.net retelling,
//    section 2: MXFP4 is a blocked 4-bit float format);
//  * expert width 768 and hidden 2560 (tanhow.com, "三项优化是什么？" items 1, 2);
//  * the MXFP4 block (32 E2M1 elements sharing one E8M0 scale) from the OCP
//    Microscaling Formats v1.0 specification; E4M3 from the OCP 8-bit
//    floating point specification (bias 7, largest finite 448).
//
// Readings where the pages are silent (the same as oracle/moe.py): softmax
// over float32 logits, top-k by descending logit with ties to the lower
// index, renormalised over the k; logits summed in float64 and rounded once
// to float32, then the float32 bias added; FP8 scale amax/448 per token
// (IEEE float32 division, 1 when amax is 0), codes rounded to nearest even
// with saturation; SwiGLU experts, h rounded to float32 and re-quantised per
// (token, expert); shared experts added with weight 1; the float64 output
// rounded once to BF16.
//
// Parallelism: the rows of a matrix-vector product are independent and each
// row's sum runs sequentially over K, so the result does not depend on the
// number of OpenMP threads.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- formats --

// BF16 bits -> value (exact).
double bf16_value(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// E2M1 code (OCP MX): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
// mantissa; exponent 0 is subnormal (0 or 0.5).
double e2m1_value(unsigned c) {
  const unsigned e = (c >> 1) & 3u, m = c & 1u;
  const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, static_cast<int>(e) - 1);
  return (c & 8u) ? -mag : mag;
}

// E8M0 scale (OCP MX): 2^(e - 127); 255 (NaN) is outside the layer's inputs.
double e8m0_value(unsigned e) { return e == 255 ? std::nan("") : std::ldexp(1.0, static_cast<int>(e) - 127); }

// E4M3 code (OCP OFP8): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0
// mantissa; exponent 0 subnormal; S.1111.111 is NaN.
double e4m3_value(uint8_t c) {
  const unsigned e = (c >> 3) & 15u, m = c & 7u;
  if (e == 15 && m == 7) return std::nan("");
  const double mag = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, static_cast<int>(e) - 7);
  return (c & 0x80u) ? -mag : mag;
}

// float32 -> E4M3 code: round to nearest, ties to the even code, saturate to
// +-448.  Every E4M3 magnitude is a multiple of its binade's step (2^-9 below
// 2^-6, 2^(e-3) in the binade [2^e, 2^(e+1))), so rounding |v| to that step
// and mapping the result back to bits is exact.
uint8_t e4m3_encode(float v) {
  const double a = std::fabs(static_cast<double>(v));
  const uint8_t sign = std::signbit(v) ? 0x80u : 0u;
  if (a >= 448.0) return sign | 0x7Eu;
  int ex;
  std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
  const int e = std::max(ex - 1, -6);  // binade exponent (subnormals share -6)
  const double step = std::ldexp(1.0, e - 3);
  double q = a / step;  // exact: a is a float32, step a power of two
  const double fl = std::floor(q), fr = q - fl;
  q = fr > 0.5 ? fl + 1 : fr < 0.5 ? fl : (std::fmod(fl, 2.0) == 0.0 ? fl : fl + 1);
  const double r = q * step;  // the rounded magnitude
  if (r >= 448.0) return sign | 0x7Eu;
  if (r == 0.0) return sign;
  int rex;
  std::frexp(r, &rex);
  const int re = rex - 1;
  if (re < -6) return sign | static_cast<uint8_t>(r / std::ldexp(1.0, -9));  // subnormal: m * 2^-9
  const unsigned mant = static_cast<unsigned>(r / std::ldexp(1.0, re - 3)) - 8u;  // 8..15 -> 0..7
  return sign | static_cast<uint8_t>(((re + 7) << 3) | mant);
}

// float64 -> BF16 bits, one rounding to nearest even.
uint16_t bf16_round(double v) {
  if (std::isnan(v)) return 0x7FC0u;
  const double a = std::fabs(v);
  const uint16_t sign = std::signbit(v) ? 0x8000u : 0u;
  // largest finite BF16 is (2 - 2^-7) * 2^127; half a step above it rounds to inf
  if (a >= std::ldexp(2.0 - std::ldexp(1.0, -8), 127)) return sign | 0x7F80u;
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);
  const int e = std::max(ex - 1, -126);
  const double step = std::ldexp(1.0, e - 7);
  double q = a / step;
  const double fl = std::floor(q), fr = q - fl;
  q = fr > 0.5 ? fl + 1 : fr < 0.5 ? fl : (std::fmod(fl, 2.0) == 0.0 ? fl : fl + 1);
  const double r = q * step;
  const float rf = static_cast<float>(r);  // exact: r has at most 8 significant bits
  uint32_t u;
  std::memcpy(&u, &rf, 4);
  return sign | static_cast<uint16_t>(u >> 16);
}

// -------------------------------------------------------- per-row FP8 quant --

// s = amax / 448 (IEEE float32 division; 1 when amax is 0), q = E4M3(v / s).
float quantize_row(const float* v, int K, uint8_t* q) {
  float amax = 0.f;
  for (int k = 0; k < K; ++k) amax = std::max(amax, std::fabs(v[k]));
  const float s = amax == 0.f ? 1.f : amax / 448.f;
  for (int k = 0; k < K; ++k) q[k] = e4m3_encode(v[k] / s);
  return s;
}

// out[r] = s * sum_b 2^(E[r,b]-127) * sum_{k in b} e2m1(c[r,k]) * e4m3(q[k]),
// one float64 sum per row, sequential over k (rows in parallel).
void mxfp4_matvec(const uint8_t* codes, const uint8_t* scales, int R, int K, const uint8_t* q, float s,
                  double* out) {
  std::vector<double> a(K);
  for (int k = 0; k < K; ++k) a[k] = e4m3_value(q[k]);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    const uint8_t* cr = codes + static_cast<size_t>(r) * (K / 2);
    const uint8_t* sr = scales + static_cast<size_t>(r) * (K / 32);
    double acc = 0.0;
    for (int k = 0; k < K; ++k) {
      const unsigned c = (k & 1) ? (cr[k >> 1] >> 4) : (cr[k >> 1] & 15u);  // element 2j: low nibble
      acc += e2m1_value(c) * e8m0_value(sr[k / 32]) * a[k];
    }
    out[r] = static_cast<double>(s) * acc;
  }
}

}  // namespace

extern "C" {

// Threads the following calls may use (OpenMP); returns the number set.
int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n < 1) n = omp_get_num_procs();
  omp_set_num_threads(n);
  return n;
#else
  (void)n;
  return 1;
#endif
}

// Router: x [T][H] and W [E][H] BF16 bits, bias [E] float32 or null ->
// logits [T][E] float32, ids [T][k] (descending logit, ties to the lower
// index), w [T][k] float32 (softmax over the selected logits, float64).
void oracle_route(const uint16_t* x, int T, int H, const uint16_t* Wr, const float* bias, int E, int k,
                  float* logits, int32_t* ids, float* w) {
  for (int t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c)
        acc += bf16_value(x[static_cast<size_t>(t) * H + c]) * bf16_value(Wr[static_cast<size_t>(e) * H + c]);
      float l = static_cast<float>(acc);
      if (bias) l = l + bias[e];
      logits[static_cast<size_t>(t) * E + e] = l;
    }
    std::vector<int> order(E);
    for (int e = 0; e < E; ++e) order[e] = e;
    const float* lt = logits + static_cast<size_t>(t) * E;
    std::stable_sort(order.begin(), order.end(), [lt](int i, int j) { return lt[i] > lt[j]; });
    const double top = lt[order[0]];
    double z[64], sum = 0.0;
    for (int i = 0; i < k; ++i) {
      z[i] = std::exp(static_cast<double>(lt[order[i]]) - top);
      sum += z[i];
    }
    for (int i = 0; i < k; ++i) {
      ids[static_cast<size_t>(t) * k + i] = order[i];
      w[static_cast<size_t>(t) * k + i] = static_cast<float>(z[i] / sum);
    }
  }
}

// Experts and combine: y[t] = bf16( sum_i w[t,i] FFN_{ids[t,i]}(x_t) +
// sum_s FFN_{E+s}(x_t) ).  Expert e's canonical weights are w13c[e]
// [2I][H/2], w13s[e] [2I][H/32], w2c[e] [H][I/2], w2s[e] [H][I/32] (rows
// 0..I-1 gate, I..2I-1 up); only the experts the call touches need to be set.
// Outputs: y [T][H] BF16 bits; optional (may be null) xq [T][H], xs [T],
// per (token, slot) h [T][k+S][I], qh [T][k+S][I], sh [T][k+S] with slots in
// ids order followed by the shared experts, and y64 [T][H].
void oracle_forward(const uint16_t* x, int T, int H, int I, int E, int k, int n_shared, const int32_t* ids,
                    const float* w, const uint8_t* const* w13c, const uint8_t* const* w13s,
                    const uint8_t* const* w2c, const uint8_t* const* w2s, uint16_t* y, uint8_t* xq_out,
                    float* xs_out, float* h_out, uint8_t* qh_out, float* sh_out, double* y64_out) {
  const int S = k + n_shared;
  std::vector<float> x32(H), h32(I);
  std::vector<uint8_t> xq(H), qh(I);
  std::vector<double> gu(2 * static_cast<size_t>(I)), d(H), y64(H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) x32[c] = static_cast<float>(bf16_value(x[static_cast<size_t>(t) * H + c]));
    const float xs = quantize_row(x32.data(), H, xq.data());
    if (xq_out) std::memcpy(xq_out + static_cast<size_t>(t) * H, xq.data(), H);
    if (xs_out) xs_out[t] = xs;
    std::fill(y64.begin(), y64.end(), 0.0);
    for (int si = 0; si < S; ++si) {
      const int e = si < k ? ids[static_cast<size_t>(t) * k + si] : E + (si - k);
      const double we = si < k ? static_cast<double>(w[static_cast<size_t>(t) * k + si]) : 1.0;
      mxfp4_matvec(w13c[e], w13s[e], 2 * I, H, xq.data(), xs, gu.data());
      for (int j = 0; j < I; ++j) {
        const double g = gu[j], u = gu[I + j];
        h32[j] = static_cast<float>(g / (1.0 + std::exp(-g)) * u);  // SwiGLU
      }
      const float sh = quantize_row(h32.data(), I, qh.data());
      mxfp4_matvec(w2c[e], w2s[e], H, I, qh.data(), sh, d.data());
      for (int n = 0; n < H; ++n) y64[n] += we * d[n];
      const size_t slot = static_cast<size_t>(t) * S + si;
      if (h_out) std::memcpy(h_out + slot * I, h32.data(), sizeof(float) * I);
      if (qh_out) std::memcpy(qh_out + slot * I, qh.data(), I);
      if (sh_out) sh_out[slot] = sh;
    }
    for (int n = 0; n < H; ++n) y[static_cast<size_t>(t) * H + n] = bf16_round(y64[n]);
    if (y64_out) std::memcpy(y64_out + static_cast<size_t>(t) * H, y64.data(), sizeof(double) * H);
  }
}

// The two format conversions on their own (for the format pins).
uint8_t oracle_e4m3_encode(float v) { return e4m3_encode(v); }
uint16_t oracle_bf16_round(double v) { return bf16_round(v); }

}  // extern "C"
