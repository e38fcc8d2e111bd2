// qlora_dequant.cuh -- 4-bit weight decode to bf16 in registers, for the dequant warps of the
// fused GEMM kernels (sm_100a).
//
// One "item" is 64 consecutive elements of one weight row (32 code bytes).  The decoded item is
// written as 8 chunks of 16 bytes (8 bf16) into a swizzled shared-memory tile that the tensor core
// reads directly.
//
// Decode definitions (per element, code c, block scale s):
//   NF4   : bf16_rne( fp32( level[c] * absmax ) )           -- one fp32 absmax per 64 along K
//           ("Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §3 "The three QLoRA tricks",
//           items 1-2).  For each item the 16 possible products are formed once in binary32 and
//           rounded to bf16 (exactly the definition), then every element is a table lookup done
//           with byte permutes from registers.
//   MXFP4 : e2m1(c) * 2^(e-127)                              -- one E8M0 per 32 along K
//   NVFP4 : e2m1(c) * e4m3(s)                                -- one E4M3 per 16 along K
//           ("Fine-Tuning 4-Bit Models: Adapting a Base That Only Ships Quantized", "Case 2").
//           Both products are exact in bf16 (at most 2 x 4 significant bits, exponent inside the
//           bf16 range or overflowing to inf), so one packed bf16 multiply of the decoded E2M1 pair
//           by the decoded scale gives the exact result.  The NVFP4 fp32 tensor scale is NOT applied
//           here: it is uniform over the weight, so the GEMM epilogue multiplies the fp32
//           accumulator by it instead.
#pragma once
#include <cstdint>
#include "qlora_ptx.cuh"

namespace qlora {

// The kernel's own copy of the 16 NF4 levels (binary32 bit patterns, code 0..15 ascending, code 7
// is exact zero): quantiles of N(0,1) normalised to [-1, 1].
__device__ __forceinline__ float nf4_level_dev(int i) {
  constexpr uint32_t bits[16] = {
      0xbf800000u, 0xbf3239b1u, 0xbf066b2eu, 0xbeca329eu, 0xbe91a24bu, 0xbe3d353du,
      0xbdba7869u, 0x00000000u, 0x3da2fb01u, 0x3e24cadfu, 0x3e7c04dau, 0x3ead0336u,
      0x3ee1a4b5u, 0x3f1007a9u, 0x3f3913b0u, 0x3f800000u};
  return __uint_as_float(bits[i]);
}

// 16-entry bf16 lookup table split into byte planes: lo[q] holds the low bytes of entries
// 4q..4q+3, hi[q] the high bytes.
struct Lut16 {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ Lut16 nf4_lut(float absmax) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = __fmul_rn(nf4_level_dev(2 * i), absmax);
    const float b = __fmul_rn(nf4_level_dev(2 * i + 1), absmax);
    p[i] = ptx::cvt_bf16x2(a, b);            // entry 2i in the low half, 2i+1 in the high half
  }
  Lut16 t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = ptx::prmt(p[2 * q], p[2 * q + 1], 0x6420u);
    t.hi[q] = ptx::prmt(p[2 * q], p[2 * q + 1], 0x7531u);
  }
  return t;
}

// Look up 8 codes (the 8 nibbles of w, element 0 in the low nibble) in a 16-entry table.
// out[i] = { t[code 2i] (low half), t[code 2i+1] (high half) }.
__device__ __forceinline__ void lut16_lookup8(const Lut16& t, uint32_t w, uint32_t (&out)[4]) {
  const uint32_t sel3 = w & 0x77777777u;                 // low 3 bits of each code
  const uint32_t b3 = w & 0x88888888u;                   // bit 3 of each code
  const uint32_t msel = b3 | (b3 >> 3);                  // nibble 0 -> byte 0 (0x00), 9 -> sign of byte 1 (0xFF)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? (sel3 >> 16) : sel3;
    const uint32_t ms = h ? (msel >> 16) : msel;
    const uint32_t m = ptx::prmt(0x00008000u, 0u, ms);  // byte i = 0xFF where code i >= 8
    const uint32_t lo0 = ptx::prmt(t.lo[0], t.lo[1], s);
    const uint32_t lo1 = ptx::prmt(t.lo[2], t.lo[3], s);
    const uint32_t hi0 = ptx::prmt(t.hi[0], t.hi[1], s);
    const uint32_t hi1 = ptx::prmt(t.hi[2], t.hi[3], s);
    const uint32_t lo = (lo0 & ~m) | (lo1 & m);
    const uint32_t hi = (hi0 & ~m) | (hi1 & m);
    out[2 * h] = ptx::prmt(lo, hi, 0x5140u);
    out[2 * h + 1] = ptx::prmt(lo, hi, 0x7362u);
  }
}

// E2M1 codes -> unscaled bf16.  Magnitude (3 low bits) through byte tables, sign from bit 3.
//   magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 = bf16 0x0000 3F00 3F80 3FC0 4000 4040 4080 40C0
__device__ __forceinline__ void e2m1_decode8(uint32_t w, uint32_t (&out)[4]) {
  constexpr uint32_t kLoA = 0xC0800000u, kLoB = 0xC0804000u;   // low bytes, entries 0-3 / 4-7
  constexpr uint32_t kHiA = 0x3F3F3F00u, kHiB = 0x40404040u;   // high bytes
  const uint32_t sel3 = w & 0x77777777u;
  const uint32_t b3 = w & 0x88888888u;
  const uint32_t msel = b3 | (b3 >> 3);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? (sel3 >> 16) : sel3;
    const uint32_t ms = h ? (msel >> 16) : msel;
    const uint32_t m = ptx::prmt(0x00008000u, 0u, ms);
    const uint32_t lo = ptx::prmt(kLoA, kLoB, s);
    const uint32_t hi = ptx::prmt(kHiA, kHiB, s) | (m & 0x80808080u);
    out[2 * h] = ptx::prmt(lo, hi, 0x5140u);
    out[2 * h + 1] = ptx::prmt(lo, hi, 0x7362u);
  }
}

// E8M0 scale -> bf16 bit pattern (exact): 2^(e-127); e = 0 is the bf16 subnormal 2^-127;
// e = 255 is NaN.
__device__ __forceinline__ uint32_t e8m0_bf16(uint32_t e) {
  e &= 0xFFu;
  if (e == 0u) return 0x0040u;
  if (e == 255u) return 0x7FC0u;
  return e << 7;
}

// E4M3 ("FN": bias 7, no inf, S.1111.111 NaN) -> binary32 (exact).
__device__ __forceinline__ float e4m3_f32(uint32_t b) {
  b &= 0xFFu;
  const uint32_t s = b >> 7, e = (b >> 3) & 15u, m = b & 7u;
  if (e == 15u && m == 7u) return __uint_as_float(0x7FC00000u);
  float mag;
  if (e == 0u) mag = __fmul_rn(static_cast<float>(m), 0.001953125f);   // m/8 * 2^-6
  else mag = __uint_as_float(((e + 120u) << 23) | (m << 20));
  return __uint_as_float(__float_as_uint(mag) | (s << 31));
}
// ... and its bf16 bit pattern (exact: at most 4 significant bits).
__device__ __forceinline__ uint32_t e4m3_bf16(uint32_t b) { return __float_as_uint(e4m3_f32(b)) >> 16; }

// kFmtNF4DQ: NF4 whose 64-block absmax is an E4M3 code times an fp32 second-level scale (one per
// 256 consecutive codes); once the absmax is formed the decode is NF4's.
enum : int { kFmtNF4 = 0, kFmtMXFP4 = 1, kFmtNVFP4 = 2, kFmtNF4DQ = 3 };

// Per-item scale material, loaded from global memory one step ahead of use.
struct ItemScale {
  uint32_t raw;   // NF4 / NF4DQ: fp32 bits of the absmax; MXFP4: 2 E8M0 bytes; NVFP4: 4 E4M3 bytes
};

// The absmax of an NF4DQ block: fp32( e4m3(c1) * s2 ), binary32 round-to-nearest-even.
__device__ __forceinline__ ItemScale nf4dq_item_scale(uint32_t c1, float s2) {
  ItemScale s;
  s.raw = __float_as_uint(__fmul_rn(e4m3_f32(c1), s2));
  return s;
}

// Decode one item (64 elements: code words cw[0..7], 8 elements each) and store it as eight
// 16-byte chunks: chunk j goes to shared address row_base + ((j ^ swz) << 4).
template <int FMT>
__device__ __forceinline__ void dequant_item_store(const uint32_t (&cw)[8], ItemScale sc,
                                                   uint32_t row_base, uint32_t swz) {
  if constexpr (FMT == kFmtNF4 || FMT == kFmtNF4DQ) {
    const Lut16 t = nf4_lut(__uint_as_float(sc.raw));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t o[4];
      lut16_lookup8(t, cw[j], o);
      ptx::st_shared_v4(row_base + ((static_cast<uint32_t>(j) ^ swz) << 4), o[0], o[1], o[2], o[3]);
    }
  } else {
    uint32_t s2[4];   // bf16x2 scale per 16-element quarter of the item
    if constexpr (FMT == kFmtMXFP4) {
      const uint32_t a = e8m0_bf16(sc.raw & 0xFFu), b = e8m0_bf16((sc.raw >> 8) & 0xFFu);
      s2[0] = s2[1] = a | (a << 16);
      s2[2] = s2[3] = b | (b << 16);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t v = e4m3_bf16((sc.raw >> (8 * q)) & 0xFFu);
        s2[q] = v | (v << 16);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t o[4];
      e2m1_decode8(cw[j], o);
      const uint32_t s = s2[j >> 1];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = ptx::mul_bf16x2(o[i], s);
      ptx::st_shared_v4(row_base + ((static_cast<uint32_t>(j) ^ swz) << 4), o[0], o[1], o[2], o[3]);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Short-batch decoders.  On sm_100a the byte-permute, logic and shift instructions share one
// 64-lane-per-clock pipe, while integer multiply-add and packed bf16 multiplies share another of
// the same width, so the decoders below move shifts onto the multiply pipe: a right shift by n is
// the high word of a multiply by 2^(32-n), a left shift a multiply by 2^n.  The multipliers come
// from a run-time 1 (a kernel argument) so the compiler cannot turn them back into shifts.
struct DecodeMul {
  uint32_t hi16, hi28, hi29;   // 2^16, 2^28, 2^29: high words give >> 16, >> 4, >> 3
  uint32_t x63, x64;           // 63, 64
};
__device__ __forceinline__ DecodeMul decode_mul(uint32_t one) {
  DecodeMul k;
  k.hi16 = one << 16;
  k.hi28 = one << 28;
  k.hi29 = one << 29;
  k.x63 = one * 63u;
  k.x64 = one << 6;
  return k;
}

// NF4: 8 codes of w through the item's 16-entry table; out[i] = {t[code 2i], t[code 2i+1]}.
// Same selection as lut16_lookup8, with the selector shifts done as multiply-high.
__device__ __forceinline__ void nf4_lookup8_mul(const Lut16& t, uint32_t w, const DecodeMul& k,
                                                uint32_t (&out)[4]) {
  const uint32_t b3 = w & 0x88888888u;                 // bit 3 of each code
  const uint32_t sel3 = w ^ b3;                        // low 3 bits of each code
  const uint32_t msel = __umulhi(b3, k.hi29) + b3;     // b3 | (b3 >> 3): 9 where code >= 8
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? __umulhi(sel3, k.hi16) : sel3;
    const uint32_t ms = h ? __umulhi(msel, k.hi16) : msel;
    const uint32_t m = ptx::prmt(0x00008000u, 0u, ms);  // byte i = 0xFF where code i >= 8
    const uint32_t lo0 = ptx::prmt(t.lo[0], t.lo[1], s);
    const uint32_t lo1 = ptx::prmt(t.lo[2], t.lo[3], s);
    const uint32_t hi0 = ptx::prmt(t.hi[0], t.hi[1], s);
    const uint32_t hi1 = ptx::prmt(t.hi[2], t.hi[3], s);
    const uint32_t lo = (lo0 & ~m) | (lo1 & m);
    const uint32_t hi = (hi0 & ~m) | (hi1 & m);
    out[2 * h] = ptx::prmt(lo, hi, 0x5140u);
    out[2 * h + 1] = ptx::prmt(lo, hi, 0x7362u);
  }
}

// E2M1 bit placement: for a code c = s e1 e0 m the bf16 pattern (c & 7) << 6 | (c & 8) << 12 puts
// e1 e0 in the two lowest exponent bits and m in the top mantissa bit, which is exactly
// e2m1(c) * 2^-126 (e1 e0 = 0 lands on the bf16 subnormals 0 and 2^-127, matching E2M1's own
// subnormal 0.5 m), with the sign in place.  One packed bf16 multiply by (block scale * 2^126)
// then gives e2m1(c) * scale exactly whenever that product is representable.
// out[i] = {pattern(code 2i), pattern(code 2i+1)}.
__device__ __forceinline__ void e2m1_pattern8(uint32_t w, const DecodeMul& k, uint32_t (&out)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;                        // codes 2i in byte i
  const uint32_t hi = __umulhi(w, k.hi28) & 0x0F0F0F0Fu;      // codes 2i+1 in byte i
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // byte 0 <- code 2i, byte 2 <- code 2i+1, bytes 1 and 3 <- the sign of a byte whose top bit
    // is 0, i.e. zero: each 16-bit lane holds one bare code
    const uint32_t x = ptx::prmt(lo, hi, uint32_t(i) | 0x80u | (uint32_t(4 + i) << 8) | 0x8000u);
    const uint32_t sg = x & 0x00080008u;
    out[i] = (x + sg * k.x63) * k.x64;                        // mag << 6 | sign << 12
  }
}

// Packed bf16 scale operands for the bit-placement decode.
//   MXFP4: 2^(e-1) (= 2^(e-127) * 2^126), exact for e <= 128; bit 0 of *slow* is set when an
//          E8M0 exponent is above 128 (the product no longer fits: decode in two multiplies).
//   NVFP4: e4m3(s) * 2^118, exact for every E4M3 byte (NaN stays NaN): the decoded element is
//          e2m1 * e4m3 * 2^-8, and the kernel multiplies its accumulator by 2^8 * tensor scale.
__device__ __forceinline__ uint32_t mx_fast_scale(uint32_t e) {
  const uint32_t v = ((e & 0xFFu) + 126u) << 7;
  return v | (v << 16);
}
__device__ __forceinline__ uint32_t nv_shifted_scale(uint32_t b) {
  const uint32_t v = __float_as_uint(__fmul_rn(e4m3_f32(b), 3.3230699894622896e+35f)) >> 16;  // 2^118
  return v | (v << 16);
}
// 2^126 in both halves, and the exact E8M0 scale in both halves.
constexpr uint32_t kBf16x2Pow126 = 0x7E807E80u;
__device__ __forceinline__ uint32_t mx_exact_scale(uint32_t e) {
  const uint32_t v = e8m0_bf16(e);
  return v | (v << 16);
}

// Decode one 64-element item into 32 packed words (word j = elements 2j, 2j+1), for operands kept
// in tensor memory.  NVFP4 elements come out times 2^-8 (see nv_shifted_scale).
template <int FMT>
__device__ __forceinline__ void decode_item_regs(const uint32_t (&cw)[8], ItemScale sc,
                                                 const DecodeMul& k, uint32_t (&o)[32]) {
  if constexpr (FMT == kFmtNF4 || FMT == kFmtNF4DQ) {
    const Lut16 t = nf4_lut(__uint_as_float(sc.raw));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t q[4];
      nf4_lookup8_mul(t, cw[j], k, q);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[4 * j + i] = q[i];
    }
  } else if constexpr (FMT == kFmtMXFP4) {
    const uint32_t e0 = sc.raw & 0xFFu, e1 = (sc.raw >> 8) & 0xFFu;
    if (e0 <= 128u && e1 <= 128u) {
      const uint32_t s0 = mx_fast_scale(e0), s1 = mx_fast_scale(e1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t q[4];
        e2m1_pattern8(cw[j], k, q);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[4 * j + i] = ptx::mul_bf16x2(q[i], j < 4 ? s0 : s1);
      }
    } else {
      const uint32_t s0 = mx_exact_scale(e0), s1 = mx_exact_scale(e1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t q[4];
        e2m1_pattern8(cw[j], k, q);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          o[4 * j + i] = ptx::mul_bf16x2(ptx::mul_bf16x2(q[i], kBf16x2Pow126), j < 4 ? s0 : s1);
      }
    }
  } else {
    uint32_t s[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) s[q4] = nv_shifted_scale((sc.raw >> (8 * q4)) & 0xFFu);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t q[4];
      e2m1_pattern8(cw[j], k, q);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[4 * j + i] = ptx::mul_bf16x2(q[i], s[j >> 1]);
    }
  }
}

// The same decode stored as eight swizzled 16-byte chunks (chunk j at row_base + ((j ^ swz) << 4)),
// for operands kept in shared memory.  NVFP4 elements come out times 2^-8.
template <int FMT>
__device__ __forceinline__ void decode_item_store(const uint32_t (&cw)[8], ItemScale sc,
                                                  const DecodeMul& k, uint32_t row_base,
                                                  uint32_t swz) {
  if constexpr (FMT == kFmtNF4 || FMT == kFmtNF4DQ) {
    const Lut16 t = nf4_lut(__uint_as_float(sc.raw));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t q[4];
      nf4_lookup8_mul(t, cw[j], k, q);
      ptx::st_shared_v4(row_base + ((uint32_t(j) ^ swz) << 4), q[0], q[1], q[2], q[3]);
    }
  } else {
    uint32_t s[4];
    bool slow = false;
    if constexpr (FMT == kFmtMXFP4) {
      const uint32_t e0 = sc.raw & 0xFFu, e1 = (sc.raw >> 8) & 0xFFu;
      slow = e0 > 128u || e1 > 128u;
      s[0] = s[1] = slow ? mx_exact_scale(e0) : mx_fast_scale(e0);
      s[2] = s[3] = slow ? mx_exact_scale(e1) : mx_fast_scale(e1);
    } else {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) s[q4] = nv_shifted_scale((sc.raw >> (8 * q4)) & 0xFFu);
    }
    if (!slow) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t q[4];
        e2m1_pattern8(cw[j], k, q);
        const uint32_t sj = s[j >> 1];
        ptx::st_shared_v4(row_base + ((uint32_t(j) ^ swz) << 4), ptx::mul_bf16x2(q[0], sj),
                          ptx::mul_bf16x2(q[1], sj), ptx::mul_bf16x2(q[2], sj),
                          ptx::mul_bf16x2(q[3], sj));
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t q[4];
        e2m1_pattern8(cw[j], k, q);
        const uint32_t sj = s[j >> 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = ptx::mul_bf16x2(ptx::mul_bf16x2(q[i], kBf16x2Pow126), sj);
        ptx::st_shared_v4(row_base + ((uint32_t(j) ^ swz) << 4), q[0], q[1], q[2], q[3]);
      }
    }
  }
}

// Store 64 zeros (an item outside the weight).
__device__ __forceinline__ void zero_item_store(uint32_t row_base) {
#pragma unroll
  for (int j = 0; j < 8; ++j) ptx::st_shared_v4(row_base + (static_cast<uint32_t>(j) << 4), 0, 0, 0, 0);
}

}  // namespace qlora
