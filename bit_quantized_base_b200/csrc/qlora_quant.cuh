// qlora_quant.cuh -- the quantiser (float weight -> stored 4-bit codes and scales) and the merge
// of a trained adapter into a stored weight with requantisation, W' = Q(deq(W) + s B A).
//
// "Training LLMs on a Budget: LoRA, QLoRA, and LoftQ": the base is quantised once, before
// training (§3 "The setup", "What QLoRA leaves open"); merging a trained adapter, W' = W +
// (alpha/r) B A, into a quantised base means dequantise, add, requantise (§2 "Deployment: keep or
// merge").  "Fine-Tuning 4-Bit Models: Adapting a Base That Only Ships Quantized": the merged
// result is requantised to NVFP4 ("Case 2") or back to MXFP4, where how much of the adapter
// survives has to be measured ("Case 3").  The pages give no rounding rules; the encode
// rules are this library's (include/qlora.h, qlora_quantize):
//   NF4    : absmax = max |v| of the 64-block; code = number of NF4 level midpoints below
//            v / absmax (binary64), ties to the lower code; a zero block is all code 7 (level 0).
//   NF4-DQ : as NF4 against the decoded absmax fp32(e4m3(c1) * s2), with s2 = fp32(group max /
//            448) per 256 consecutive blocks (1 for an all-zero group) and c1 = nearest E4M3 of
//            absmax / s2.
//   MXFP4  : e = clamp(floor(log2 amax) - 2 + 127, 0, 254) (0 for a zero block); code = nearest
//            E2M1 of v / 2^(e-127), ties to the even code, saturating at 6.
//   NVFP4  : s_t = fp32(T / 2688) from the tensor's max |v| (1 if zero); s_b = nearest E4M3 of
//            amax_b / (6 s_t); code = nearest E2M1 of v / (e4m3(s_b) s_t) (binary64).
// Every quotient and comparison is binary64 (IEEE, no contraction), every E4M3 tie goes to the
// even code and saturates at 448, so the result is exactly reproducible.
//
// Work split: one CTA of 256 threads per 256 consecutive scale blocks (row-major over [N, K/bs]),
// one block per thread -- NF4-DQ's second-level groups are exactly these CTAs.
#pragma once
#include <cuda_bf16.h>
#include "qlora_dequant.cuh"

namespace qlora {
namespace quant {
constexpr int kBlocksPerCta = 256;
__host__ __device__ constexpr int block_size(int fmt) {
  return (fmt == kFmtNF4 || fmt == kFmtNF4DQ) ? 64 : (fmt == kFmtMXFP4 ? 32 : 16);
}
}  // namespace quant

// E2M1 element value (binary32, exact).
__device__ __forceinline__ float e2m1_f32(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const float mag = e == 0u ? 0.5f * float(m) : __uint_as_float(((e + 126u) << 23) | (m << 22));
  return (c & 8u) ? -mag : mag;
}

// Division-free comparisons.  The rules compare a binary64 quotient x = fl64(v / d) (d > 0)
// with the midpoint m of two neighbouring grid values.  In every use v has at most 24
// significant bits, d at most 28 and m at most 25, so the product m d is exact in binary64; and
// fl64(v / d) cannot round onto m unless v / d equals m, because a non-zero v - m d is at least
// 2^-49 of m d in magnitude, while rounding moves a quotient by at most 2^-53 of it.  So
// "x > m" has the outcome of "v > m d", and "x == m" that of "v == m d".

// Nearest E2M1 code of v / d (d > 0, at most 28 significant bits): ties to the even code
// (mantissa bit 0), magnitude saturating at 6, sign bit only on a non-zero magnitude.
__device__ __forceinline__ uint32_t e2m1_encode_scaled(float v, double d) {
  constexpr double mids[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  const double a = fabs(double(v));
  uint32_t c = 0;
#pragma unroll
  for (uint32_t i = 0; i < 7; ++i) {
    const double t = mids[i] * d;
    if (a > t || (a == t && (i & 1u))) c = i + 1;
  }
  return (c != 0u && signbit(v)) ? (c | 8u) : c;
}

// Nearest positive E4M3 code of q >= 0, ties to the even code, saturating at 448.  "q is past
// the midpoint below code c" (strictly, or on it with c even) holds for c = 1..best and for no
// larger c, so a binary search over c finds best in 7 steps.
__device__ __forceinline__ uint32_t e4m3_encode_pos(double q) {
  uint32_t lo = 0, hi = 0x7Fu;
#pragma unroll
  for (int it = 0; it < 7; ++it) {
    const uint32_t c = (lo + hi) >> 1;
    const double mid = 0.5 * (double(e4m3_f32(c - 1u)) + double(e4m3_f32(c)));
    if (q > mid || (q == mid && (c & 1u) == 0u)) lo = c;
    else hi = c;
  }
  return lo;
}

// NF4 code of v against absmax a > 0: the number of level midpoints m with m < v / a, as
// m a < v (exact, see above).  The midpoints are compile-time constants (the sum of two
// neighbouring binary32 levels is exact in binary64).
__device__ __forceinline__ uint32_t nf4_encode(float v, float a) {
  const double vv = double(v), aa = double(a);
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) {
    const double mid = 0.5 * (double(nf4_level_dev(i)) + double(nf4_level_dev(i + 1)));
    if (mid * aa < vv) c = uint32_t(i + 1);
  }
  return c;
}

struct QuantParams {
  const void* v;          // [N, K] fp32 or bf16 (row-major)
  int v_bf16;
  uint8_t* codes;         // [N, K/2]
  void* scales;           // NF4 float [N, K/64]; NF4-DQ / NVFP4 / MXFP4 uint8
  float* scales2;         // NF4-DQ [ceil(N K/64 / 256)]
  float* tensor_scale;    // NVFP4: holds max |v| (as bits) on entry, s_t written by the last kernel
  int N, K;
};


// max |v| over the tensor into *bits (non-negative binary32 values order like their bit
// patterns); 16-byte loads (N K is a multiple of 64, v 16-byte aligned).
__global__ void __launch_bounds__(256) qlora_quant_amax_kernel(const QuantParams p, unsigned* bits) {
  const size_t n = size_t(p.N) * size_t(p.K);
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  float a = 0.0f;
  if (p.v_bf16) {
    const uint4* src = reinterpret_cast<const uint4*>(p.v);
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n / 8; i += stride) {
      const uint4 q = src[i];
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h)
        a = fmaxf(a, fmaxf(fabsf(__uint_as_float(u[h] << 16)),
                           fabsf(__uint_as_float(u[h] & 0xFFFF0000u))));
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(p.v);
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n / 4; i += stride) {
      const float4 q = src[i];
      a = fmaxf(a, fmaxf(fmaxf(fabsf(q.x), fabsf(q.y)), fmaxf(fabsf(q.z), fabsf(q.w))));
    }
  }
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(bits, __float_as_uint(a));
}

// s_t = fp32(T / 2688), 1 for an all-zero tensor, replacing T in place (one thread, after the
// encode kernel has read T).
__global__ void qlora_quant_tensor_scale_kernel(float* ts) {
  const float T = *ts;
  *ts = T > 0.0f ? __double2float_rn(__ddiv_rn(double(T), 2688.0)) : 1.0f;
}

template <int FMT>
__global__ void __launch_bounds__(quant::kBlocksPerCta)
qlora_quant_encode_kernel(const QuantParams p) {
  constexpr int BS = quant::block_size(FMT);
  __shared__ float red[quant::kBlocksPerCta / 32];
  const int nb = p.K / BS;
  const size_t nblocks = size_t(p.N) * size_t(nb);
  const size_t f = size_t(blockIdx.x) * quant::kBlocksPerCta + threadIdx.x;
  const bool have = f < nblocks;
  const size_t n = have ? f / size_t(nb) : 0;
  const int b = have ? int(f % size_t(nb)) : 0;
  const size_t base = n * size_t(p.K) + size_t(b) * BS;
  float v[BS];
  float amax = 0.0f;
  if (have) {
    if (p.v_bf16) {                          // 8 bf16 per 16-byte load
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(p.v) + base);
#pragma unroll
      for (int w = 0; w < BS / 8; ++w) {
        const uint4 q = src[w];
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          v[8 * w + 2 * h] = __uint_as_float(u[h] << 16);
          v[8 * w + 2 * h + 1] = __uint_as_float(u[h] & 0xFFFF0000u);
        }
      }
    } else {                                 // 4 fp32 per 16-byte load
      const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.v) + base);
#pragma unroll
      for (int w = 0; w < BS / 4; ++w) {
        const float4 q = src[w];
        v[4 * w] = q.x;
        v[4 * w + 1] = q.y;
        v[4 * w + 2] = q.z;
        v[4 * w + 3] = q.w;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < BS; ++i) v[i] = 0.0f;
  }
#pragma unroll
  for (int i = 0; i < BS; ++i) amax = fmaxf(amax, fabsf(v[i]));
  uint32_t packed[BS / 8];
#pragma unroll
  for (int w = 0; w < BS / 8; ++w) packed[w] = 0u;
  auto put = [&](int i, uint32_t c) { packed[i >> 3] |= c << (4 * (i & 7)); };

  if constexpr (FMT == kFmtNF4 || FMT == kFmtNF4DQ) {
    float a = amax;
    if constexpr (FMT == kFmtNF4DQ) {
      // group max over the CTA's 256 blocks -> s2, c1, decoded absmax
      float g = amax;
      for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
      if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = g;
      __syncthreads();
      g = red[0];
#pragma unroll
      for (int w = 1; w < quant::kBlocksPerCta / 32; ++w) g = fmaxf(g, red[w]);
      const float s2 = g > 0.0f ? __fdiv_rn(g, 448.0f) : 1.0f;
      if (threadIdx.x == 0) p.scales2[blockIdx.x] = s2;
      const uint32_t c1 = e4m3_encode_pos(__ddiv_rn(double(amax), double(s2)));
      if (have) static_cast<uint8_t*>(p.scales)[f] = uint8_t(c1);
      a = __fmul_rn(e4m3_f32(c1), s2);
    } else {
      if (have) static_cast<float*>(p.scales)[f] = amax;
    }
#pragma unroll
    for (int i = 0; i < BS; ++i) put(i, a > 0.0f ? nf4_encode(v[i], a) : 7u);
  } else if constexpr (FMT == kFmtMXFP4) {
    uint32_t e = 0;
    if (amax > 0.0f) {
      int pe = 0;
      frexp(double(amax), &pe);                 // amax = m 2^pe, m in [0.5, 1)
      const int ee = (pe - 1) - 2 + 127;
      e = uint32_t(ee < 0 ? 0 : (ee > 254 ? 254 : ee));
    }
    if (have) static_cast<uint8_t*>(p.scales)[f] = uint8_t(e);
    const double sc = ldexp(1.0, int(e) - 127);
#pragma unroll
    for (int i = 0; i < BS; ++i) put(i, e2m1_encode_scaled(v[i], sc));
  } else {
    const float T = *p.tensor_scale;
    const float st = T > 0.0f ? __double2float_rn(__ddiv_rn(double(T), 2688.0)) : 1.0f;
    const uint32_t sb = e4m3_encode_pos(__ddiv_rn(double(amax), __dmul_rn(6.0, double(st))));
    if (have) static_cast<uint8_t*>(p.scales)[f] = uint8_t(sb);
    const double d = double(e4m3_f32(sb)) * double(st);   // exact: 4 x 24 significant bits
#pragma unroll
    for (int i = 0; i < BS; ++i) put(i, d > 0.0 ? e2m1_encode_scaled(v[i], d) : 0u);
  }
  if (have) {
    uint8_t* dst = p.codes + n * size_t(p.K / 2) + size_t(b) * (BS / 2);
    if constexpr (BS == 64) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    } else if constexpr (BS == 32) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else {
      reinterpret_cast<uint2*>(dst)[0] = make_uint2(packed[0], packed[1]);
    }
  }
}

// ---------------------------------------------------------------------------- merge
// The merged value of element (n, k): fp32( deq(W)[n,k] + s * sum_j B[n,j] A[j,k] ), the sum over
// j = 0..r-1 in that order in binary64 (each bf16 product exact), plus and times in binary64
// without contraction, one rounding to binary32 at the end.  deq(W) is the weight's full decode
// (for NVFP4 including the tensor scale).
// A stored weight as the element decode reads it.
struct StoredView {
  const uint8_t* codes;
  const void* scales;
  const float* scales2;
  const float* tensor_scale;
  int K;
};

struct MergeParams {
  StoredView w;
  const __nv_bfloat16* A;   // [r, K]
  const __nv_bfloat16* B;   // [N, r]
  float* out;               // [N, K]
  int N, K, r;
  float s;
};

// Element (n, k) of the decoded weight as the layer's GEMMs see it: the bf16 value of the format's
// decode chain (NVFP4 including the tensor scale), widened to fp32.
template <int FMT>
__device__ __forceinline__ float decode_element(const StoredView& w, int n, int k) {
  const uint8_t byte = w.codes[size_t(n) * (w.K / 2) + k / 2];
  const uint32_t c = (k & 1) ? uint32_t(byte >> 4) : uint32_t(byte & 15u);
  if constexpr (FMT == kFmtNF4 || FMT == kFmtNF4DQ) {
    const size_t fb = size_t(n) * (w.K / 64) + k / 64;
    const float a = FMT == kFmtNF4
                        ? static_cast<const float*>(w.scales)[fb]
                        : __fmul_rn(e4m3_f32(static_cast<const uint8_t*>(w.scales)[fb]),
                                    w.scales2[fb / 256]);
    float lv = 0.0f;                       // select, not an indexed local array
#pragma unroll
    for (int i = 0; i < 16; ++i) lv = c == uint32_t(i) ? nf4_level_dev(i) : lv;
    return __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv, a)));
  } else if constexpr (FMT == kFmtMXFP4) {
    const uint32_t e = static_cast<const uint8_t*>(w.scales)[size_t(n) * (w.K / 32) + k / 32];
    const float sc = e == 255u ? __uint_as_float(0x7FC00000u)
                               : (e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23));
    return __bfloat162float(__float2bfloat16_rn(__fmul_rn(e2m1_f32(c), sc)));
  } else {
    const uint32_t sb = static_cast<const uint8_t*>(w.scales)[size_t(n) * (w.K / 16) + k / 16];
    const float prod = __fmul_rn(__fmul_rn(e2m1_f32(c), e4m3_f32(sb)), *w.tensor_scale);
    return __bfloat162float(__float2bfloat16_rn(prod));
  }
}

template <int FMT>
__global__ void __launch_bounds__(256) qlora_merge_values_kernel(const MergeParams p) {
  const size_t total = size_t(p.N) * size_t(p.K);
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += size_t(gridDim.x) * blockDim.x) {
    const int n = int(i / size_t(p.K)), k = int(i % size_t(p.K));
    double lora = 0.0;
    for (int j = 0; j < p.r; ++j)
      lora = __dadd_rn(lora, __dmul_rn(double(__bfloat162float(p.B[size_t(n) * p.r + j])),
                                       double(__bfloat162float(p.A[size_t(j) * p.K + k]))));
    const double v = __dadd_rn(double(decode_element<FMT>(p.w, n, k)), __dmul_rn(double(p.s), lora));
    p.out[i] = __double2float_rn(v);
  }
}

}  // namespace qlora
