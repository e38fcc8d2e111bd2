// qlora_debug.cuh -- test-only kernels: the dequant stage run on its own (decoded tiles written
// back un-swizzled), and a bounded wait that is meant to run out.
#pragma once
#include <cuda_bf16.h>
#include "qlora_fused.cuh"
#include "qlora_short.cuh"

namespace qlora {

struct DebugDequantParams {
  CUtensorMap tm_codes;  // same tensor map shape as the fused kernel's
  const void* scales;
  const float* scales2;  // NF4DQ second-level scales, else unused
  __nv_bfloat16* out;    // [N, K]
  int* status;
  int N, K;
};

// One CTA = one pipeline step of the fused kernel's weight operand: forward tiling = 128 weight
// rows x 64 columns (K-major tile), dX tiling = 64 weight rows x 128 columns (MN-major tile).
// 128 threads, one 64-element item each, exactly as in the fused kernel's dequant group.
template <int FMT, bool DX>
__global__ void __launch_bounds__(128)
qlora_debug_dequant_kernel(const __grid_constant__ DebugDequantParams p) {
  __shared__ __align__(1024) uint8_t wtile[fused::W_BYTES];
  __shared__ __align__(1024) uint8_t ctile[fused::C_BYTES];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const int tg = threadIdx.x;
  const int c0 = blockIdx.x * fused::HN;    // forward: first weight row; dX: first column
  const int ks = blockIdx.y;                 // forward: column step;     dX: row step
  const uint32_t b = ptx::smem_u32(&bar);
  if (tg == 0) {
    ptx::mbar_init(b, 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  if (tg == 0) {
    ptx::mbar_arrive_expect_tx(b, fused::C_BYTES);
    if (!DX) ptx::tma_load_2d(ptx::smem_u32(ctile), &p.tm_codes, b, ks * (fused::BK / 2), c0);
    else ptx::tma_load_2d(ptx::smem_u32(ctile), &p.tm_codes, b, c0 / 2, ks * fused::BK);
  }
  const ItemGeom<DX> geo(tg);
  const int n = DX ? ks * fused::BK + geo.row : c0 + geo.row;
  const int kcol = DX ? c0 + geo.chunk * 64 : ks * fused::BK;
  const bool valid = n < p.N && kcol < p.K;
  ItemScale sc{0u};
  if (valid) {
    if constexpr (FMT == kFmtNF4DQ) sc = load_item_scale_dq(p.scales, p.scales2, 0, p.N, n, kcol, p.K);
    else sc = load_item_scale<FMT>(p.scales, n, kcol, p.K);
  }
  if (!ptx::mbar_wait(b, 0, p.status, &abort_flag)) return;
  const uint32_t cb = ptx::smem_u32(ctile);
  const uint4 lo = ptx::ld_shared_v4(cb + geo.code_off(0));
  const uint4 hi = ptx::ld_shared_v4(cb + geo.code_off(1));
  const uint32_t cw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  const uint32_t rb = geo.op_row_base(ptx::smem_u32(wtile));
  if (valid) dequant_item_store<FMT>(cw, sc, rb, geo.swz());
  else zero_item_store(rb);
  __syncthreads();
  // read back a DIFFERENT thread's item (the next row of the same chunk) through the swizzle
  const ItemGeom<DX> g2((tg & ~63) | ((tg + 1) & 63));
  const int n2 = DX ? ks * fused::BK + g2.row : c0 + g2.row;
  const int k2 = DX ? c0 + g2.chunk * 64 : ks * fused::BK;
  if (n2 < p.N && k2 < p.K) {
    const uint32_t rb2 = g2.op_row_base(ptx::smem_u32(wtile));
    for (int j = 0; j < 8; ++j) {
      const uint4 v = ptx::ld_shared_v4(rb2 + ((uint32_t(j) ^ g2.swz()) << 4));
      *reinterpret_cast<uint4*>(p.out + size_t(n2) * p.K + k2 + j * 8) = v;
    }
  }
}

// The short-batch kernels' decoders run on their own: one thread per 64-element item (row n,
// columns [64 c, 64 c + 64)), with the item's codes and block scale.
// REGS = true: decode_item_regs (the forward's tensor-memory form), written straight out;
// REGS = false: decode_item_store into a swizzled shared-memory row, read back through the swizzle.
// NVFP4 elements come out times 2^-8, as those kernels use them.
template <int FMT, bool REGS>
__global__ void __launch_bounds__(128)
qlora_debug_short_decode_kernel(const __grid_constant__ ShortParams p) {
  __shared__ __align__(1024) uint8_t rows[128 * 128];
  const int item = int(blockIdx.x) * 128 + int(threadIdx.x);
  const int per_row = p.K / 64;
  if (item >= p.N * per_row) return;
  const int n = item / per_row, kcol = (item - n * per_row) * 64;
  const uint4* cp = reinterpret_cast<const uint4*>(p.codes + size_t(n) * size_t(p.K / 2) + size_t(kcol / 2));
  const uint4 c0 = cp[0], c1 = cp[1];
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  ItemScale sc = load_item_scale<FMT>(p.scales, n, kcol, p.K);
  const DecodeMul km = decode_mul(p.one);
  uint4* dst = reinterpret_cast<uint4*>(p.out + size_t(n) * p.K + kcol);
  if constexpr (REGS) {
    uint32_t o[32];
    decode_item_regs<FMT>(cw, sc, km, o);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
  } else {
    const uint32_t rb = ptx::smem_u32(rows) + threadIdx.x * 128u;
    const uint32_t swz = threadIdx.x & 7u;
    decode_item_store<FMT>(cw, sc, km, rb, swz);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = ptx::ld_shared_v4(rb + ((uint32_t(j) ^ swz) << 4));
  }
}

// Decode throughput of the short-batch kernels' dequant stage on one SM, the bound of the
// short-batch path: 512 threads (the short-batch kernels' 16 dequant warps) each decode `iters`
// 64-element items with decode_item_store into a swizzled operand tile, fresh codes every item
// (one xor per code word).  cycles[b] = the CTA's clock cycles for the loop.
template <int FMT>
__global__ void __launch_bounds__(512, 1)
qlora_debug_decode_rate_kernel(int iters, unsigned long long* cycles, uint32_t* sink, uint32_t one) {
  __shared__ __align__(1024) uint8_t tile[2][fused::W_BYTES];
  const int tg = threadIdx.x & 127;
  const ItemGeom<false> geo(tg);
  const uint32_t rb = geo.op_row_base(ptx::smem_u32(tile[(threadIdx.x >> 7) & 1]));
  const DecodeMul km = decode_mul(one);
  uint32_t cw[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) cw[j] = (threadIdx.x * 8u + j + blockIdx.x * 7919u) * 0x9E3779B1u;
  ItemScale sc;
  sc.raw = FMT == kFmtNF4 ? __float_as_uint(0.01f + 0.001f * float(tg & 7))
                          : (FMT == kFmtMXFP4 ? 0x7C7Du : 0x38393A3Bu);
  __syncthreads();
  const unsigned long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
    decode_item_store<FMT>(cw, sc, km, rb, geo.swz());
#pragma unroll
    for (int j = 0; j < 8; ++j) cw[j] ^= 0x9E3779B1u + uint32_t(it);
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  const uint32_t v = ptx::ld_shared_v4(rb).x;
  if (v == 0x12345678u) sink[0] = v;   // keeps the stores live
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

__global__ void qlora_debug_wait_kernel(int* status, unsigned long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the wait must give up and record the timeout
    ptx::mbar_wait(ptx::smem_u32(&bar), 0, status, &abort_flag, limit_cycles);
  }
}

}  // namespace qlora
