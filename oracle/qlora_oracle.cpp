// qlora_oracle.cpp -- plain, slow, fp64 CPU oracle for the 4-bit-base unmerged-LoRA linear.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
// leg may load this library.  The product path (bit_quantized_base_b200/) never links, imports
// or calls it, and this file shares no code, table or header with the CUDA kernels: every decode
// table below is typed in here from the format specification and pinned by tests/.
//
// What it computes (the plain definition, no blocking, fusion or reordering):
//   * Decode of each frozen 4-bit weight element to bf16:
//       NF4   : w = bf16_rne( fp32( level[code] * absmax ) ), one fp32 absmax per 64 along K
//               ("Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §3 "The three QLoRA
//               tricks", items 1 and 2).
//       MXFP4 : w = bf16_rne( fp32( e2m1(code) * 2^(e-127) ) ), one E8M0 per 32 along K
//       NVFP4 : w = bf16_rne( fp32( fp32( e2m1(code) * e4m3(s_blk) ) * s_tensor ) ), one E4M3 per
//               16 along K plus one fp32 tensor scale
//               ("Fine-Tuning 4-Bit Models: Adapting a Base That Only Ships Quantized", "Case 2:
//               An NVFP4 deployment checkpoint is what you were handed").
//       NF4 with double quantisation: as NF4 with absmax = fp32( e4m3(c1) * s2[g] ): the 64-block
//               absmax is stored as an 8-bit E4M3 code c1, and every 256 consecutive first-level
//               codes of the weight (row-major [N, K/64] order) share one fp32 second-level
//               scale s2 ("Training LLMs on a Budget", §3 "The three QLoRA tricks", item 2:
//               "8-bit FP8 with a second-level absmax over blocks of 256 first-level constants").
//     Every multiply is IEEE binary32 round-to-nearest-even, subnormals kept (no FTZ).
//   * The layer, in fp64 on the exact bf16/fp32 input values, with s = alpha/r (or alpha/sqrt r)
//     multiplying every LoRA term ("Training LLMs on a Budget", §2 "The math": y = Wx + (a/r)BAx,
//     and the scaling "reappears wherever BA does"; §2 "Initialization matters" for the gradient
//     chain dL/dA = B^T (dL/dy) x^T and dL/dB = (dL/dy) x^T A^T), written for a batch of rows:
//       T  = X A^T                 [M,r]
//       Y  = X Wd^T + s T B^T      [M,N]
//       U  = dY B                  [M,r]
//       dX = dY Wd + s U A         [M,K]
//       dA = s U^T X               [r,K]
//       dB = s dY^T T              [N,r]
//     No dW: the base weight is frozen ("Quantized weights, full precision: The math behind 75%
//     cheaper fine-tuning", "Backward pass and optimizer step in training").
//
// Built with plain g++ -O2 -fopenmp -ffp-contract=off (no fast-math), so float products are the
// IEEE products the definition names.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <limits>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------------------------------------
// Scalar conversions
// ---------------------------------------------------------------------------------------------

float f32_from_bits(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
uint32_t bits_from_f32(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

float bf16_to_f32(uint16_t h) { return f32_from_bits(static_cast<uint32_t>(h) << 16); }

// Round-to-nearest-even of a binary32 value to bfloat16 (1 sign, 8 exponent, 7 fraction bits).
// The 16 dropped fraction bits decide: above half rounds up, below half rounds down, exactly
// half rounds to the even result.  NaN stays NaN (quiet bit forced so it cannot round to inf).
uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = bits_from_f32(f);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
    return static_cast<uint16_t>((u >> 16) | 0x0040u);
  uint32_t upper = u >> 16;
  uint32_t lower = u & 0xffffu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;  // carries into exponent
  return static_cast<uint16_t>(upper);
}

// ---------------------------------------------------------------------------------------------
// Format tables, typed in from the format definitions
// ---------------------------------------------------------------------------------------------

// The 16 NF4 levels as binary32 bit patterns, code 0 (-1) .. code 15 (+1), ascending; code 7 is
// exact zero.  Construction: quantiles of N(0,1) ("16 quantile points drawn from the inverse CDF
// of a standard normal", "Training LLMs on a Budget", §3 "The three QLoRA tricks", item 1), 8 on
// the positive side and 7 on the negative side plus an exact zero, normalised to [-1, 1].  The
// probabilities are evenly spaced from 1-d down to 1/2 with d = (1/30 + 1/32)/2 (9 points for the
// positive side, 8 for the negative, dropping 1/2 each time).  oracle_nf4_levels_as241 recomputes
// them from Phi^-1; tests/ pin the two against each other and against an independent Phi^-1.
const uint32_t kNF4LevelBits[16] = {
    0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
    0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
    0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};

float nf4_level(uint32_t code) { return f32_from_bits(kNF4LevelBits[code & 15u]); }

// E2M1 (OCP MX element type FP4): bit layout s e1 e0 m, exponent bias 1, exponent field 0 is
// subnormal with value 0.5*m.  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; code 8 is -0.  No inf/NaN.
float e2m1_value(uint32_t code) {
  const uint32_t s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  float mag;
  if (e == 0u) mag = 0.5f * static_cast<float>(m);
  else mag = std::ldexp(1.0f + 0.5f * static_cast<float>(m), static_cast<int>(e) - 1);
  return s ? -mag : mag;
}

// E8M0 (OCP MX scale type): unsigned power of two 2^(e-127); e = 255 is NaN.  e = 0 gives 2^-127,
// a binary32 subnormal, exact.
float e8m0_value(uint32_t e) {
  e &= 0xffu;
  if (e == 255u) return std::numeric_limits<float>::quiet_NaN();
  return std::ldexp(1.0f, static_cast<int>(e) - 127);
}

// E4M3 "FN" (OCP FP8): s eeee mmm, bias 7, no infinities, S.1111.111 is NaN, maximum 448,
// exponent field 0 is subnormal (m/8 * 2^-6).
float e4m3_value(uint32_t b) {
  b &= 0xffu;
  const uint32_t s = b >> 7, e = (b >> 3) & 15u, m = b & 7u;
  if (e == 15u && m == 7u) return std::numeric_limits<float>::quiet_NaN();
  float mag;
  if (e == 0u) mag = std::ldexp(static_cast<float>(m) / 8.0f, -6);
  else mag = std::ldexp(1.0f + static_cast<float>(m) / 8.0f, static_cast<int>(e) - 7);
  return s ? -mag : mag;
}

// ---------------------------------------------------------------------------------------------
// Inverse standard normal CDF, Wichura's algorithm AS 241 (PPND16, Applied Statistics 37(3),
// 1988): rational approximations in three regions, relative accuracy about 1e-16.
// ---------------------------------------------------------------------------------------------
double poly(const double* c, int n, double x) {  // c[0] + c[1] x + ... + c[n-1] x^(n-1)
  double r = 0.0;
  for (int i = n - 1; i >= 0; --i) r = r * x + c[i];
  return r;
}

double norm_ppf(double p) {
  static const double a[8] = {3.3871328727963666080e0, 1.3314166789178437745e+2,
                              1.9715909503065514427e+3, 1.3731693765509461125e+4,
                              4.5921953931549871457e+4, 6.7265770927008700853e+4,
                              3.3430575583588128105e+4, 2.5090809287301226727e+3};
  static const double b[8] = {1.0,
                              4.2313330701600911252e+1, 6.8718700749205790830e+2,
                              5.3941960214247511077e+3, 2.1213794301586595867e+4,
                              3.9307895800092710610e+4, 2.8729085735721942674e+4,
                              5.2264952788528545610e+3};
  static const double c[8] = {1.42343711074968357734e0, 4.63033784615654529590e0,
                              5.76949722146069140550e0, 3.64784832476320460504e0,
                              1.27045825245236838258e0, 2.41780725177450611770e-1,
                              2.27238449892691845833e-2, 7.74545014278341407640e-4};
  static const double d[8] = {1.0,
                              2.05319162663775882187e0, 1.67638483018380384940e0,
                              6.89767334985100004550e-1, 1.48103976427480074590e-1,
                              1.51986665636164571966e-2, 5.47593808499534494600e-4,
                              1.05075007164441684324e-9};
  static const double e[8] = {6.65790464350110377720e0, 5.46378491116411436990e0,
                              1.78482653991729133580e0, 2.96560571828504891230e-1,
                              2.65321895265761230930e-2, 1.24266094738807843860e-3,
                              2.71155556874348757815e-5, 2.01033439929228813265e-7};
  static const double f[8] = {1.0,
                              5.99832206555887937690e-1, 1.36929880922735805310e-1,
                              1.48753612908506148525e-2, 7.86869131145613259100e-4,
                              1.84631831751005468180e-5, 1.42151175831644588870e-7,
                              2.04426310338993978564e-15};
  if (!(p > 0.0 && p < 1.0)) {
    if (p == 0.0) return -std::numeric_limits<double>::infinity();
    if (p == 1.0) return std::numeric_limits<double>::infinity();
    return std::numeric_limits<double>::quiet_NaN();
  }
  const double q = p - 0.5;
  if (std::fabs(q) <= 0.425) {
    const double r = 0.180625 - q * q;
    return q * poly(a, 8, r) / poly(b, 8, r);
  }
  double r = (q < 0.0) ? p : 1.0 - p;
  r = std::sqrt(-std::log(r));
  double x;
  if (r <= 5.0) {
    r -= 1.6;
    x = poly(c, 8, r) / poly(d, 8, r);
  } else {
    r -= 5.0;
    x = poly(e, 8, r) / poly(f, 8, r);
  }
  return (q < 0.0) ? -x : x;
}

// Formats: 0 NF4, 1 MXFP4, 2 NVFP4, 3 NF4 with double-quantised absmax.
constexpr int kFmtNf4Dq = 3;
constexpr int64_t kDqGroup = 256;   // first-level constants per second-level scale

// Block size along K of the scale of each format.
int block_size(int fmt) { return (fmt == 0 || fmt == kFmtNf4Dq) ? 64 : (fmt == 1 ? 32 : 16); }

// Second-level scales of one [N, K] NF4-DQ weight: ceil(N * K/64 / 256).
int64_t dq_groups(int64_t N, int64_t K) { return (N * (K / 64) + kDqGroup - 1) / kDqGroup; }

uint32_t code_at(const uint8_t* codes, int64_t K, int64_t n, int64_t k) {
  const uint8_t byte = codes[n * (K / 2) + k / 2];
  return (k & 1) ? (byte >> 4) : (byte & 15u);  // element 2j in the low nibble, 2j+1 in the high
}

// One weight element per the definition at the top of this file.  with_tensor_scale = 0 stops
// the NVFP4 chain before the tensor scale (the micro-block decode alone).
uint16_t dequant_element(int fmt, const uint8_t* codes, const void* scales, const float* scales2,
                         float tensor_scale, int with_tensor_scale, int64_t K, int64_t n,
                         int64_t k) {
  const uint32_t c = code_at(codes, K, n, k);
  const int64_t nb = K / block_size(fmt);
  const int64_t blk = k / block_size(fmt);
  if (fmt == 0) {
    const float absmax = static_cast<const float*>(scales)[n * nb + blk];
    const float p = nf4_level(c) * absmax;
    return f32_to_bf16_rne(p);
  }
  if (fmt == kFmtNf4Dq) {
    const int64_t f = n * nb + blk;   // first-level constant, row-major
    const float absmax = e4m3_value(static_cast<const uint8_t*>(scales)[f]) * scales2[f / kDqGroup];
    const float p = nf4_level(c) * absmax;
    return f32_to_bf16_rne(p);
  }
  if (fmt == 1) {
    const uint8_t e = static_cast<const uint8_t*>(scales)[n * nb + blk];
    const float p = e2m1_value(c) * e8m0_value(e);
    return f32_to_bf16_rne(p);
  }
  const uint8_t sb = static_cast<const uint8_t*>(scales)[n * nb + blk];
  float p = e2m1_value(c) * e4m3_value(sb);
  if (with_tensor_scale) p = p * tensor_scale;
  return f32_to_bf16_rne(p);
}

bool valid_shape(int fmt, int64_t N, int64_t K) {
  if (fmt < 0 || fmt > kFmtNf4Dq || N < 0 || K < 0) return false;
  return K % block_size(fmt) == 0;
}

// ---------------------------------------------------------------------------------------------
// Encoders (float weight -> stored codes and scales).  The pages give no rounding rules, so the
// encode is this build's reading, stated once here and in the header (include/qlora.h):
//   NF4    : absmax = max |v| over the 64-block (binary32, exact); absmax == 0 -> every code 7
//            (level 0); else code = the number of level midpoints m_i = (L_i + L_{i+1}) / 2 that
//            are < x = v / absmax, x and m_i in binary64 (ties go to the lower code).
//   NF4-DQ : the 64-block absmax a as above; per group of 256 consecutive blocks (row-major)
//            s2 = fp32(gmax / 448) (gmax = the group's largest a; s2 = 1 if gmax == 0);
//            c1 = E4M3 nearest to a / s2 (binary64 quotient; ties to the even code; saturating
//            at 448); the element codes as NF4 against the decoded absmax fp32(e4m3(c1) * s2).
//   MXFP4  : amax = max |v| over the 32-block; e = clamp(floor(log2 amax) - 2 + 127, 0, 254)
//            (amax == 0 -> e = 0); code = E2M1 nearest to v / 2^(e-127) (binary64), ties to the
//            even code (mantissa bit 0), magnitude saturating at 6, sign bit only on a non-zero
//            magnitude.
//   NVFP4  : tensor amax T; s_t = fp32(T / 2688) (1 if T == 0); per 16-block s_b = E4M3 nearest
//            to amax_b / (6 s_t) (binary64, ties to even, saturating at 448); code = E2M1 nearest
//            to v / (e4m3(s_b) * s_t) (binary64 divisor; a zero divisor gives code 0).
// Inputs must be finite.
// ---------------------------------------------------------------------------------------------

// Nearest E2M1 code of x (binary64), ties to even, saturating, sign only on non-zero magnitude.
uint32_t e2m1_encode(double x) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double a = std::fabs(x) < 6.0 ? std::fabs(x) : 6.0;
  uint32_t c = 0;
  for (uint32_t i = 0; i < 7; ++i) {
    const double mid = 0.5 * (mag[i] + mag[i + 1]);
    if (a > mid || (a == mid && (i & 1u))) c = i + 1;   // past the midpoint, or a tie toward even
  }
  return (c != 0u && std::signbit(x)) ? (c | 8u) : c;
}

// Nearest positive E4M3 code of q >= 0 (binary64), ties to the even code, saturating at 448.
uint32_t e4m3_encode_pos(double q) {
  uint32_t best = 0;
  for (uint32_t c = 1; c <= 0x7Eu; ++c) {
    const double lo = e4m3_value(c - 1), hi = e4m3_value(c);
    const double mid = 0.5 * (lo + hi);
    if (q > mid || (q == mid && (c & 1u) == 0u)) best = c;
  }
  return best;
}

// NF4 code of v against absmax a (> 0).
uint32_t nf4_encode(float v, float a) {
  const double x = static_cast<double>(v) / static_cast<double>(a);
  uint32_t c = 0;
  for (uint32_t i = 0; i < 15; ++i) {
    const double mid = 0.5 * (static_cast<double>(nf4_level(i)) + static_cast<double>(nf4_level(i + 1)));
    if (mid < x) c = i + 1;
  }
  return c;
}

void put_code(uint8_t* codes, int64_t K, int64_t n, int64_t k, uint32_t c) {
  uint8_t& b = codes[n * (K / 2) + k / 2];
  b = (k & 1) ? static_cast<uint8_t>((b & 0x0Fu) | (c << 4)) : static_cast<uint8_t>((b & 0xF0u) | c);
}

}  // namespace

extern "C" {

// Encode a float weight v [N,K] (binary32, row-major) per the rules above.  Outputs: codes
// [N,K/2]; scales (NF4 float [N,K/64], NF4-DQ uint8 E4M3 [N,K/64], MXFP4 uint8 [N,K/32], NVFP4
// uint8 [N,K/16]); *tensor_scale (NVFP4, else untouched); scales2 (NF4-DQ [ceil(N*K/64/256)]).
// Returns 0, or -1 on a bad argument.
int oracle_encode(int fmt, int64_t N, int64_t K, const float* v, uint8_t* codes, void* scales,
                  float* tensor_scale, float* scales2) {
  if (!valid_shape(fmt, N, K) || (N * K > 0 && (!v || !codes || !scales))) return -1;
  if (fmt == 2 && !tensor_scale) return -1;
  if (fmt == kFmtNf4Dq && N * K > 0 && !scales2) return -1;
  const int bs = block_size(fmt);
  const int64_t nb = K / bs;
  std::vector<float> amax(static_cast<size_t>(N * nb), 0.0f);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < nb; ++b) {
      float a = 0.0f;
      for (int i = 0; i < bs; ++i) a = std::fmax(a, std::fabs(v[n * K + b * bs + i]));
      amax[static_cast<size_t>(n * nb + b)] = a;
    }
  if (fmt == 0 || fmt == kFmtNf4Dq) {
    std::vector<float> dec(amax);   // the absmax the element codes are taken against
    if (fmt == kFmtNf4Dq) {
      const int64_t G = dq_groups(N, K);
      for (int64_t g = 0; g < G; ++g) {
        const int64_t f0 = g * kDqGroup, f1 = (f0 + kDqGroup < N * nb) ? f0 + kDqGroup : N * nb;
        float gmax = 0.0f;
        for (int64_t f = f0; f < f1; ++f) gmax = std::fmax(gmax, amax[static_cast<size_t>(f)]);
        const float s2 = gmax > 0.0f ? gmax / 448.0f : 1.0f;
        scales2[g] = s2;
        for (int64_t f = f0; f < f1; ++f) {
          const uint32_t c1 = e4m3_encode_pos(static_cast<double>(amax[static_cast<size_t>(f)]) /
                                              static_cast<double>(s2));
          static_cast<uint8_t*>(scales)[f] = static_cast<uint8_t>(c1);
          dec[static_cast<size_t>(f)] = e4m3_value(c1) * s2;
        }
      }
    } else {
      for (int64_t f = 0; f < N * nb; ++f) static_cast<float*>(scales)[f] = amax[static_cast<size_t>(f)];
    }
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) {
        const float a = dec[static_cast<size_t>(n * nb + k / 64)];
        put_code(codes, K, n, k, a > 0.0f ? nf4_encode(v[n * K + k], a) : 7u);
      }
    return 0;
  }
  if (fmt == 1) {
    for (int64_t f = 0; f < N * nb; ++f) {
      const float a = amax[static_cast<size_t>(f)];
      uint32_t e = 0;
      if (a > 0.0f) {
        int p = 0;
        std::frexp(a, &p);                       // a = m 2^p, m in [0.5, 1): floor(log2 a) = p - 1
        const int ee = (p - 1) - 2 + 127;
        e = static_cast<uint32_t>(ee < 0 ? 0 : (ee > 254 ? 254 : ee));
      }
      static_cast<uint8_t*>(scales)[f] = static_cast<uint8_t>(e);
    }
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) {
        const uint32_t e = static_cast<const uint8_t*>(scales)[n * nb + k / 32];
        const double sc = std::ldexp(1.0, static_cast<int>(e) - 127);
        put_code(codes, K, n, k, e2m1_encode(static_cast<double>(v[n * K + k]) / sc));
      }
    return 0;
  }
  // NVFP4
  float T = 0.0f;
  for (int64_t i = 0; i < N * K; ++i) T = std::fmax(T, std::fabs(v[i]));
  const float st = T > 0.0f ? static_cast<float>(static_cast<double>(T) / 2688.0) : 1.0f;
  *tensor_scale = st;
  for (int64_t f = 0; f < N * nb; ++f)
    static_cast<uint8_t*>(scales)[f] = static_cast<uint8_t>(
        e4m3_encode_pos(static_cast<double>(amax[static_cast<size_t>(f)]) / (6.0 * static_cast<double>(st))));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const double d = static_cast<double>(e4m3_value(static_cast<const uint8_t*>(scales)[n * nb + k / 16])) *
                       static_cast<double>(st);
      put_code(codes, K, n, k, d > 0.0 ? e2m1_encode(static_cast<double>(v[n * K + k]) / d) : 0u);
    }
  return 0;
}

// ---- scalar access for the spec tests ------------------------------------------------------
void oracle_nf4_levels_spec(float* out16) {
  for (int i = 0; i < 16; ++i) out16[i] = nf4_level(static_cast<uint32_t>(i));
}

// The NF4 construction recomputed in fp64 with AS 241 and normalised by the largest level.
void oracle_nf4_levels_as241(double* out16) {
  const double dlt = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  std::vector<double> v;
  for (int i = 0; i < 8; ++i) {  // 9 evenly spaced points from 1-d to 1/2, last one dropped
    const double p = (1.0 - dlt) + (0.5 - (1.0 - dlt)) * static_cast<double>(i) / 8.0;
    v.push_back(norm_ppf(p));
  }
  for (int i = 0; i < 7; ++i) {  // 8 evenly spaced points from 1-d to 1/2, last one dropped
    const double p = (1.0 - dlt) + (0.5 - (1.0 - dlt)) * static_cast<double>(i) / 7.0;
    v.push_back(-norm_ppf(p));
  }
  v.push_back(0.0);
  // sort ascending (insertion sort: 16 items)
  for (size_t i = 1; i < v.size(); ++i)
    for (size_t j = i; j > 0 && v[j - 1] > v[j]; --j) std::swap(v[j - 1], v[j]);
  double mx = 0.0;
  for (double x : v) mx = std::fabs(x) > mx ? std::fabs(x) : mx;
  for (int i = 0; i < 16; ++i) out16[i] = v[static_cast<size_t>(i)] / mx;
}

double oracle_norm_ppf(double p) { return norm_ppf(p); }
float oracle_decode_e2m1(uint32_t code) { return e2m1_value(code); }
float oracle_decode_e8m0(uint32_t code) { return e8m0_value(code); }
float oracle_decode_e4m3(uint32_t code) { return e4m3_value(code); }
uint16_t oracle_f32_to_bf16(float x) { return f32_to_bf16_rne(x); }
float oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

// Bytes of one stored weight: codes + block scales (+ 4 for the NVFP4 tensor scale; + 4 per 256
// first-level constants for NF4 with double quantisation).
int64_t oracle_weight_bytes(int fmt, int64_t N, int64_t K) {
  if (!valid_shape(fmt, N, K)) return -1;
  const int64_t codes = N * K / 2;
  const int64_t nb = N * (K / block_size(fmt));
  if (fmt == 0) return codes + 4 * nb;
  if (fmt == kFmtNf4Dq) return codes + nb + 4 * dq_groups(N, K);
  if (fmt == 1) return codes + nb;
  return codes + nb + 4;
}

// Decode a whole weight [N,K] to bf16 bit patterns.  scales2: NF4-DQ second-level scales
// [ceil(N * K/64 / 256)], else unused.  Returns 0, or -1 on a bad argument.
int oracle_dequant(int fmt, int64_t N, int64_t K, const uint8_t* codes, const void* scales,
                   const float* scales2, float tensor_scale, int with_tensor_scale,
                   uint16_t* out) {
  if (!valid_shape(fmt, N, K) || (N * K > 0 && (!codes || !scales || !out))) return -1;
  if (fmt == kFmtNf4Dq && N * K > 0 && !scales2) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      out[n * K + k] = dequant_element(fmt, codes, scales, scales2, tensor_scale,
                                       with_tensor_scale, K, n, k);
  return 0;
}

// The layer forward and backward in fp64 (see the header of this file).
//   X [M,K], A [r,K], B [N,r], dY [M,N]: bf16 bit patterns, row-major.
//   rows / nrows: the rows of Y and dX to produce (rows == NULL: all M rows, in order).
//   Outputs (each may be NULL to skip it): Y_rows [nrows,N], dX_rows [nrows,K], T [M,r],
//   U [M,r], dA [r,K], dB [N,r].  T, U, dA and dB always cover all M rows.
// Returns 0, or -1 on a bad argument.
int oracle_layer(int fmt, int64_t M, int64_t N, int64_t K, int r, double s,
                 const uint8_t* codes, const void* scales, const float* scales2, float tensor_scale,
                 const uint16_t* X, const uint16_t* A, const uint16_t* B, const uint16_t* dY,
                 const int64_t* rows, int64_t nrows,
                 double* Y_rows, double* dX_rows, double* T_out, double* U_out,
                 double* dA, double* dB) {
  if (!valid_shape(fmt, N, K) || M < 0 || r < 0) return -1;
  if (!rows) nrows = M;
  for (int64_t i = 0; rows && i < nrows; ++i)
    if (rows[i] < 0 || rows[i] >= M) return -1;

  // Wd = decoded weight (values exactly representable in float).
  std::vector<float> Wd(static_cast<size_t>(N * K));
  {
    std::vector<uint16_t> wb(static_cast<size_t>(N * K));
    if (N * K > 0 &&
        oracle_dequant(fmt, N, K, codes, scales, scales2, tensor_scale, 1, wb.data()) != 0)
      return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N * K; ++i) Wd[static_cast<size_t>(i)] = bf16_to_f32(wb[static_cast<size_t>(i)]);
  }
  auto x = [&](int64_t m, int64_t k) { return static_cast<double>(bf16_to_f32(X[m * K + k])); };
  auto a = [&](int64_t j, int64_t k) { return static_cast<double>(bf16_to_f32(A[j * K + k])); };
  auto b = [&](int64_t n, int64_t j) { return static_cast<double>(bf16_to_f32(B[n * r + j])); };
  auto g = [&](int64_t m, int64_t n) { return static_cast<double>(bf16_to_f32(dY[m * N + n])); };

  // T = X A^T (all rows: dB needs every row of T).
  std::vector<double> T(static_cast<size_t>(M * r), 0.0);
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += x(m, k) * a(j, k);
      T[static_cast<size_t>(m * r + j)] = acc;
    }

  // U = dY B (all rows: dA needs every row of U).
  std::vector<double> U;
  const bool need_bwd = dY && (dX_rows || U_out || dA || dB);
  if (need_bwd) {
    U.assign(static_cast<size_t>(M * r), 0.0);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
      for (int j = 0; j < r; ++j) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) acc += g(m, n) * b(n, j);
        U[static_cast<size_t>(m * r + j)] = acc;
      }
  }

  // Y rows: Y[m,n] = sum_k X[m,k] Wd[n,k] + s sum_j T[m,j] B[n,j].
  if (Y_rows) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      const int64_t m = rows ? rows[i] : i;
      std::vector<double> xr(static_cast<size_t>(K));
      for (int64_t k = 0; k < K; ++k) xr[static_cast<size_t>(k)] = x(m, k);
      for (int64_t n = 0; n < N; ++n) {
        const float* wr = &Wd[static_cast<size_t>(n * K)];
        double base = 0.0;
        for (int64_t k = 0; k < K; ++k) base += xr[static_cast<size_t>(k)] * static_cast<double>(wr[k]);
        double lora = 0.0;
        for (int j = 0; j < r; ++j) lora += T[static_cast<size_t>(m * r + j)] * b(n, j);
        Y_rows[i * N + n] = base + s * lora;
      }
    }
  }

  // dX rows: dX[m,k] = sum_n dY[m,n] Wd[n,k] + s sum_j U[m,j] A[j,k].
  if (dX_rows && need_bwd) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
      const int64_t m = rows ? rows[i] : i;
      std::vector<double> acc(static_cast<size_t>(K), 0.0);
      for (int64_t n = 0; n < N; ++n) {
        const double gv = g(m, n);
        const float* wr = &Wd[static_cast<size_t>(n * K)];
        for (int64_t k = 0; k < K; ++k) acc[static_cast<size_t>(k)] += gv * static_cast<double>(wr[k]);
      }
      for (int64_t k = 0; k < K; ++k) {
        double lora = 0.0;
        for (int j = 0; j < r; ++j) lora += U[static_cast<size_t>(m * r + j)] * a(j, k);
        dX_rows[i * K + k] = acc[static_cast<size_t>(k)] + s * lora;
      }
    }
  }

  // dA[j,k] = s sum_m U[m,j] X[m,k].  Each (j,k) sums over m = 0..M-1 in order; the loop nest
  // only walks k innermost so that rows of X are read contiguously.
  if (dA && need_bwd) {
    const int64_t kc = 256;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k0 = 0; k0 < K; k0 += kc) {
      const int64_t k1 = (k0 + kc < K) ? k0 + kc : K;
      std::vector<double> acc(static_cast<size_t>(r * (k1 - k0)), 0.0);
      for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
          const double u = U[static_cast<size_t>(m * r + j)];
          for (int64_t k = k0; k < k1; ++k) acc[static_cast<size_t>(j * (k1 - k0) + (k - k0))] += u * x(m, k);
        }
      for (int j = 0; j < r; ++j)
        for (int64_t k = k0; k < k1; ++k)
          dA[static_cast<int64_t>(j) * K + k] = s * acc[static_cast<size_t>(j * (k1 - k0) + (k - k0))];
    }
  }

  // dB[n,j] = s sum_m dY[m,n] T[m,j].  Each (n,j) sums over m = 0..M-1 in order.
  if (dB && need_bwd) {
    const int64_t nc = 256;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n0 = 0; n0 < N; n0 += nc) {
      const int64_t n1 = (n0 + nc < N) ? n0 + nc : N;
      std::vector<double> acc(static_cast<size_t>((n1 - n0) * r), 0.0);
      for (int64_t m = 0; m < M; ++m)
        for (int64_t n = n0; n < n1; ++n) {
          const double gv = g(m, n);
          for (int j = 0; j < r; ++j) acc[static_cast<size_t>((n - n0) * r + j)] += gv * T[static_cast<size_t>(m * r + j)];
        }
      for (int64_t n = n0; n < n1; ++n)
        for (int j = 0; j < r; ++j) dB[n * r + j] = s * acc[static_cast<size_t>((n - n0) * r + j)];
    }
  }

  if (T_out) std::memcpy(T_out, T.data(), sizeof(double) * static_cast<size_t>(M * r));
  if (U_out && need_bwd) std::memcpy(U_out, U.data(), sizeof(double) * static_cast<size_t>(M * r));
  return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
