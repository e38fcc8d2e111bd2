// Opt-in native block-scaled forward for MXFP4 weights (W4A8):
//
//   Y = deq8(X) deq(W)^T + s T B^T,   T = X A^T (from the bf16 X)
//
// where deq8(X) is X quantised to MXFP8 (E4M3 elements, one E8M0 scale per 32 along K) and
// deq(W) is the exact E2M1 x E8M0 block product of the stored weight.  The tensor cores multiply
// the stored 4-bit weight codes by the 8-bit activation codes with both block scales
// (tcgen05.mma kind::mxf8f6f4 block_scale, fp32 accumulation): no weight is decoded by the SMs at
// all ("Quantized weights, full precision", "LoRA operations and quantization": Blackwell runs
// mxfp4-native ops; "Fine-Tuning 4-Bit Models", "Case 3": a W4AFP8 variant of a 4-bit model).
//
// Two kernels besides the LoRA down-projection:
//   qlora_mxfp8_quant_kernel  X [M,K] bf16 -> codes [M,K] E4M3 + scales [M,K/32] E8M0, one
//                             thread per 32-element block (memory-bound, ~3 bytes per element).
//   qlora_w4a8_gemm_kernel    persistent, one CTA per SM, 128 x 192 output tiles (batch rows x
//                             weight rows), 128-deep K steps in a 4-stage ring:
//     warp 0     TMA: the step's activation codes (box 128 x 128 bytes, 128B swizzle) and weight
//                codes (packed 4-bit type: 16 codes per 16-byte chunk, 8 bytes of gap, the layout
//                the MMA reads E2M1 operands in), then the LoRA step's Zs and B tiles;
//     warp 1     MMA: per step four 32-deep block-scaled MMAs (scale-factor id 0..3 picks the
//                byte of each scale cell), then the LoRA step as bf16 MMAs into the same
//                accumulator; two accumulators of 192 columns alternate between tiles;
//     warps 4-7  scale factors: each lane quarter writes the step's 128 activation and 192
//                weight scale words (4 E8M0 bytes = the step's 4 blocks of a row) into the
//                stage's tensor-memory slot with tcgen05.st, replicated in every lane quarter,
//                row m of a 128-row block at lane 32 q + m % 32, column base + m / 32 (weight
//                rows 128..191 at base + 4, 5); the words of 4 steps arrive in one 16-byte load,
//                fetched one group of steps ahead;
//     warps 8-11 epilogue: accumulator -> bf16 -> Y, then release the accumulator.
// Every wait is bounded (QLORA_ERR_DEVICE_TIMEOUT in the status word, abort flag).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "qlora_ptx.cuh"

namespace qlora {

// ------------------------------------------------------------------------------ MXFP8 quantiser
struct Mxfp8Params {
  const __nv_bfloat16* x;    // [M, K]
  uint8_t* codes;            // [M, K] E4M3
  uint8_t* scales;           // [M, K/32] E8M0
  long long blocks;          // M * K / 32
};

// Two binary32 values to E4M3 (round to nearest even, saturating at +-448), packed lo | hi << 8.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// One 32-element block: the shared exponent e = clamp(floor(log2 amax) - 8 + 127, 0, 254) (8 is
// E4M3's largest normal exponent; an all-zero block gets 0), elements the nearest E4M3 of
// x / 2^(e-127), ties to even, saturating at 448, a zero magnitude without its sign (the OCP MX
// shared-exponent rule; the pages fix no rule of their own).  floor(log2 amax) of a bf16 amax is
// its exponent field minus 127 (a subnormal or zero amax clamps e to 0), and x / 2^(e-127) is a
// multiplication by an exact power of two, so the decision matches the fp64 definition.
__global__ void __launch_bounds__(256) qlora_mxfp8_quant_kernel(const __grid_constant__ Mxfp8Params p) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= p.blocks) return;
  const uint4* src = reinterpret_cast<const uint4*>(p.x) + b * 4;
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(src + i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  uint32_t amax = 0;                 // bf16 magnitudes order as integers
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = max(amax, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  int e = int(amax >> 7) - 8;
  e = e < 0 ? 0 : (e > 254 ? 254 : e);
  // 2^(127 - e): a normal binary32 for e <= 253, the subnormal 2^-127 for e = 254
  const float inv = e <= 253 ? __uint_as_float(uint32_t(254 - e) << 23) : __uint_as_float(0x00400000u);
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = w[2 * i], c = w[2 * i + 1];
    const uint32_t lo = cvt_e4m3x2(__uint_as_float(a << 16) * inv, __uint_as_float(a & 0xFFFF0000u) * inv);
    const uint32_t hi = cvt_e4m3x2(__uint_as_float(c << 16) * inv, __uint_as_float(c & 0xFFFF0000u) * inv);
    uint32_t v = lo | (hi << 16);
    // a magnitude that rounded to zero keeps no sign: 0x80 -> 0x00 in every byte
    const uint32_t mag0 = ((v & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & 0x80808080u;   // 0x80 where nonzero
    v &= mag0 | 0x7F7F7F7Fu;
    out[i] = v;
  }
  uint4* dst = reinterpret_cast<uint4*>(p.codes + b * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  p.scales[b] = uint8_t(e);
}

// ------------------------------------------------------------------------------ block-scaled GEMM
namespace w4a8 {
constexpr int BM = 128, BN = 192, BK = 128;   // tile rows (batch), tile columns (weight rows), K step
constexpr int NS = 4;
constexpr int A_BYTES = BM * BK;              // 16 KB of E4M3 codes (or the LoRA step's Zs tile)
constexpr int B_BYTES = BN * BK;              // 24 KB shared-memory footprint of the weight codes
constexpr int B_TX = BN * BK / 2;             // 12 KB of packed codes the copy delivers
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int kTmaWarp = 0, kMmaWarp = 1, kSfWarp0 = 4, kEpiWarp0 = 8;
constexpr int kThreads = 12 * 32;
constexpr int kTmemCols = 512;
constexpr int SF_COL0 = 2 * BN;               // scale slots of 32 columns per stage after the
                                              // accumulators: activation scales at +0, weight at +16
constexpr int kBarBytes = 1024;
__host__ __device__ constexpr size_t smem_bytes() { return 1024 + size_t(NS) * STAGE + kBarBytes; }
}  // namespace w4a8

struct W4a8Params {
  CUtensorMap tm_xq;     // quantised X [M, K] u8, box {128, 128}, 128B swizzle
  CUtensorMap tm_w;      // codes [N, K] packed 4-bit (16U4_ALIGN16B), box {128, 192}, 128B swizzle
  CUtensorMap tm_zs;     // Zs [M, r] bf16, box {64, 128}, 128B swizzle (zero fill beyond r)
  CUtensorMap tm_b;      // B [N, r] bf16, box {64, 192}, 128B swizzle (zero fill beyond r)
  const uint8_t* xs;     // [M, K/32] E8M0
  const uint8_t* wsc;    // [N, K/32] E8M0 (the MXFP4 block scales)
  __nv_bfloat16* out;    // Y [M, N]
  int* status;
  int M, N, K, rpad, num_m, num_n, num_k;
};

__global__ void __launch_bounds__(w4a8::kThreads, 1)
qlora_w4a8_gemm_kernel(const __grid_constant__ W4a8Params p) {
  using namespace w4a8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(NS) * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t b0 = ptx::smem_u32(bars);
  auto full = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  auto acc_full = [&](uint32_t b) { return b0 + 8u * (2 * NS + b); };
  auto acc_empty = [&](uint32_t b) { return b0 + 8u * (2 * NS + 2 + b); };
  auto stage = [&](uint32_t s) { return ptx::smem_u32(smem) + s * uint32_t(STAGE); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = p.num_m * p.num_n;
  const int steps = p.num_k + 1;                 // the K steps, then the LoRA step
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(full(s), 1 + 4);            // the copy's expect-tx arrive + 4 scale warps
      ptx::mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(acc_full(b), 1);
      ptx::mbar_init(acc_empty(b), 4);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    ptx::prefetch_tmap(&p.tm_xq);
    ptx::prefetch_tmap(&p.tm_w);
    ptx::prefetch_tmap(&p.tm_zs);
    ptx::prefetch_tmap(&p.tm_b);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the quantised activations, Zs and the previous users of Y come from the kernels before
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ copies
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int mt = t % p.num_m, nt = t / p.num_m;
        for (int st = 0; st < steps; ++st) {
          if (!ptx::mbar_wait_idle(empty(s), ph ^ 1u, p.status, abort_flag)) { ok = false; break; }
          if (st < p.num_k) {
            ptx::mbar_arrive_expect_tx(full(s), uint32_t(A_BYTES + B_TX));
            if (ptx::dcheck(ptx::tma_x_ok(st * BK, 1), p.status)) {
              ptx::tma_load_2d(stage(s), &p.tm_xq, full(s), st * BK, mt * BM);
              ptx::tma_load_2d(stage(s) + A_BYTES, &p.tm_w, full(s), st * BK, nt * BN);
            }
          } else {
            ptx::mbar_arrive_expect_tx(full(s), uint32_t(A_BYTES + BN * 128));
            ptx::tma_load_2d(stage(s), &p.tm_zs, full(s), 0, mt * BM);
            ptx::tma_load_2d(stage(s) + A_BYTES, &p.tm_b, full(s), 0, nt * BN);
          }
          if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      int lt = 0;
      bool ok = true;
      const uint32_t id_lora = ptx::idesc_bf16(BM, BN, 0u, 0u);
      const int lora_kk = p.rpad / 16;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++lt) {
        const uint32_t b = uint32_t(lt & 1), bph = uint32_t((lt >> 1) & 1);
        if (!ptx::mbar_wait(acc_empty(b), bph ^ 1u, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + b * uint32_t(BN);
        for (int st = 0; st < steps; ++st) {
          if (!ptx::mbar_wait(full(s), ph, p.status, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t ad = ptx::smem_desc(stage(s), 16, 1024, ptx::kSw128);
          const uint64_t bd = ptx::smem_desc(stage(s) + A_BYTES, 16, 1024, ptx::kSw128);
          if (st < p.num_k) {
            const uint32_t sfa = tmem + uint32_t(SF_COL0) + 32u * s;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_mx(d, ad + uint64_t(kk) * 2u, bd + uint64_t(kk) * 2u,
                          ptx::idesc_mx_e4m3_e2m1(BM, BN, uint32_t(kk)), (st | kk) ? 1u : 0u, sfa,
                          sfa + 16u);
          } else {
            for (int kk = 0; kk < lora_kk; ++kk)
              ptx::mma_bf16(d, ad + uint64_t(kk) * 2u, bd + uint64_t(kk) * 2u, id_lora, 1u);
          }
          ptx::mma_commit(empty(s));
          if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
        }
        if (ok) ptx::mma_commit(acc_full(b));
      }
    }
  } else if (warp >= kSfWarp0 && warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale factors
    // The scale words of 4 consecutive K steps (16 blocks of a row) are fetched together, one
    // group ahead of the steps that use them, so the global-load latency stays off the steps.
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const int kb = p.K / 32;                     // scale bytes per row
    const bool vec = (kb & 15) == 0;             // rows of scales 16-byte aligned
    const int ng = (p.num_k + 3) / 4;            // groups of 4 steps per tile
    uint32_t ca[4][4], cb[8][4], na[4][4], nb[8][4];
    auto load_group = [&](int t, int g, uint32_t (&a)[4][4], uint32_t (&b)[8][4]) {
      const int mt = t % p.num_m, nt = t / p.num_m;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int m = mt * BM + 32 * c + lane;
        const uint8_t* row = p.xs + size_t(m) * kb + g * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m < p.M) {
          if (vec) {
            v = __ldg(reinterpret_cast<const uint4*>(row));
          } else {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(row);
            v.x = __ldg(w);
            if (g * 4 + 1 < p.num_k) v.y = __ldg(w + 1);
            if (g * 4 + 2 < p.num_k) v.z = __ldg(w + 2);
            if (g * 4 + 3 < p.num_k) v.w = __ldg(w + 3);
          }
        }
        a[c][0] = v.x; a[c][1] = v.y; a[c][2] = v.z; a[c][3] = v.w;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int nl = 128 * j + 32 * c + lane, n = nt * BN + nl;
          const uint8_t* row = p.wsc + size_t(n) * kb + g * 16;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (nl < BN && n < p.N) {
            if (vec) {
              v = __ldg(reinterpret_cast<const uint4*>(row));
            } else {
              const uint32_t* w = reinterpret_cast<const uint32_t*>(row);
              v.x = __ldg(w);
              if (g * 4 + 1 < p.num_k) v.y = __ldg(w + 1);
              if (g * 4 + 2 < p.num_k) v.z = __ldg(w + 2);
              if (g * 4 + 3 < p.num_k) v.w = __ldg(w + 3);
            }
          }
          b[4 * j + c][0] = v.x; b[4 * j + c][1] = v.y; b[4 * j + c][2] = v.z; b[4 * j + c][3] = v.w;
        }
    };
    uint32_t s = 0, ph = 0;
    bool ok = true;
    if (int(blockIdx.x) < num_tiles) load_group(blockIdx.x, 0, ca, cb);
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      for (int g = 0; g < ng && ok; ++g) {
        if (g + 1 < ng) load_group(t, g + 1, na, nb);
        else if (t + int(gridDim.x) < num_tiles) load_group(t + gridDim.x, 0, na, nb);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (g * 4 + j >= p.num_k) break;
          if (!ptx::mbar_wait_idle(empty(s), ph ^ 1u, p.status, abort_flag)) { ok = false; break; }
          uint32_t va[8] = {ca[0][j], ca[1][j], ca[2][j], ca[3][j], 0u, 0u, 0u, 0u};
          uint32_t vb[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) vb[i] = cb[i][j];
          const uint32_t col = tmem + lane_base + uint32_t(SF_COL0) + 32u * s;
          ptx::tmem_st_32x32b_x8(col, va);          // columns 0-3 used
          ptx::tmem_st_32x32b_x8(col + 16u, vb);
          ptx::tmem_st_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(full(s));
          if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 4; ++j) ca[c][j] = na[c][j];
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int j = 0; j < 4; ++j) cb[c][j] = nb[c][j];
      }
      if (!ok) break;
      // the LoRA step needs no scale factors; its arrival completes the stage's barrier
      if (!ptx::mbar_wait_idle(empty(s), ph ^ 1u, p.status, abort_flag)) break;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full(s));
      if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    int lt = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++lt) {
      const int mt = t % p.num_m, nt = t / p.num_m;
      const uint32_t b = uint32_t(lt & 1), bph = uint32_t((lt >> 1) & 1);
      if (!ptx::mbar_wait_idle(acc_full(b), bph, p.status, abort_flag)) break;
      ptx::tc_fence_after();
      const int m = mt * BM + q * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tmem + lane_base + b * uint32_t(BN) + uint32_t(c * 32), v);
        ptx::tmem_ld_wait(v);
        const int n0 = nt * BN + c * 32;
        if (m < p.M && ptx::dcheck(n0 >= 0, p.status)) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + size_t(m) * p.N + n0);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (n0 + 8 * u < p.N) {
              uint4 o;
              o.x = ptx::cvt_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1]));
              o.y = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3]));
              o.z = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5]));
              o.w = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7]));
              dst[u] = o;
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace qlora
