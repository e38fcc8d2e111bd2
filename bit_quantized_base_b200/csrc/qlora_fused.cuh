// qlora_fused.cuh -- the fused dequant-GEMM kernel of the layer (forward Y and backward dX).
//
//   forward : Y  = ( X  deq(W)^T + (s/ts) T B^T ) * ts     contraction over K, tile over (M, N)
//   backward: dX = ( dY deq(W)   + (s/ts) U A   ) * ts     contraction over N, tile over (M, K)
//
// ts is the NVFP4 tensor scale (1 for NF4 and MXFP4).  The LoRA term enters as one extra step of
// the same tcgen05 pipeline: its A operand is Zs = bf16(Z * s/ts) (Z = T or U, written by the
// lora_down kernel), its B operand the rows of B (forward) or A (backward), so it accumulates into
// the same fp32 tensor-memory accumulator as the base product and the epilogue only scales by ts.
//
// Per CTA tile: 256 rows (two M=128 UMMA halves sharing one B operand) x 128 output columns,
// 64-deep contraction steps.  Warp roles (448 threads, one CTA per SM, persistent over tiles):
//   warps 0-3   epilogue: tensor memory -> registers -> * ts -> bf16 -> global
//   warp  4     TMA producer: activation tiles (SW128, K-major) and packed-code tiles
//   warp  5     tensor-memory allocation and the single thread that issues tcgen05.mma
//   warps 6-13  dequant: two groups of 4 warps taking alternate steps; each thread decodes one
//               64-element item of W per step into the swizzled operand tile
// The weight tile is K-major for the forward pass (rows of W are rows of the operand) and
// MN-major for dX (rows of W run along the contraction); in both cases a 64-element item is one
// 128-byte swizzled row, so the decode stage is the same code.
#pragma once
#include <cuda_bf16.h>
#include "qlora_ptx.cuh"
#include "qlora_dequant.cuh"

namespace qlora {
namespace fused {
constexpr int BM = 256, BN = 128, BK = 64;
constexpr int NX = 4, NW = 4, NC = 6;
constexpr int X_BYTES = BM * BK * 2;   // 32 KB: two 128-row boxes
constexpr int W_BYTES = BN * BK * 2;   // 16 KB
constexpr int C_BYTES = BN * BK / 2;   // 4 KB of packed codes
constexpr int kEpiWarps = 4, kTmaWarp = 4, kMmaWarp = 5, kDqWarp0 = 6, kDqWarps = 8;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kTmemCols = 512;         // 2 buffers x 2 halves x 128 columns
constexpr int GM = 8;                  // m-tiles per raster group
constexpr int kNumBars = 2 * NX + 2 * NW + 2 * NC + 4;
constexpr size_t kSmemBytes = 1024 + size_t(NX) * X_BYTES + size_t(NW) * W_BYTES +
                              size_t(NC) * C_BYTES + 1024;
}  // namespace fused

struct FusedParams {
  CUtensorMap tm_act;    // activations [M, Kc] bf16, box {64, 128}, SW128
  CUtensorMap tm_codes;  // codes [N, K/2] u8: fwd box {32, 128} SW32; dX box {64, 64} SW64
  CUtensorMap tm_zs;     // Zs [M, r] bf16, box {64, 128}, SW128 (zero fill beyond r)
  const void* scales;
  const float* tensor_scale;         // NVFP4 device scalar, else nullptr
  const __nv_bfloat16* lora_up;      // fwd: B [N, r]; dX: A [r, K]
  __nv_bfloat16* out;                // fwd: Y [M, N]; dX: dX [M, K]
  int* status;
  int M, N, K, r;
  int num_m, num_n, num_k;           // tiles over rows, over output columns; contraction steps
};

__device__ __forceinline__ void fused_tile_coords(int t, int num_m, int num_n, int& mt, int& nt) {
  const int per_group = fused::GM * num_n;
  const int g = t / per_group;
  const int within = t - g * per_group;
  const int m_base = g * fused::GM;
  const int gm = min(fused::GM, num_m - m_base);
  mt = m_base + within % gm;
  nt = within / gm;
}

// Block-scale word of the item that starts at weight element (n, kcol).
template <int FMT>
__device__ __forceinline__ ItemScale load_item_scale(const void* scales, int n, int kcol, int K) {
  ItemScale s;
  if constexpr (FMT == kFmtNF4) {
    s.raw = __ldg(reinterpret_cast<const uint32_t*>(scales) + size_t(n) * (K / 64) + kcol / 64);
  } else if constexpr (FMT == kFmtMXFP4) {
    s.raw = __ldg(reinterpret_cast<const uint16_t*>(scales) + (size_t(n) * (K / 32) + kcol / 32) / 2);
  } else {
    s.raw = __ldg(reinterpret_cast<const uint32_t*>(scales) + (size_t(n) * (K / 16) + kcol / 16) / 4);
  }
  return s;
}

// Shared-memory geometry of one dequant item (thread tg = 0..127 of a dequant group).
//   forward: item = weight row (c0 + tg), columns [ks*64, ks*64+64): operand row tg of the
//            K-major tile; code bytes: row tg of a 128 x 32-byte SW32 tile.
//   dX     : item = weight row (ks*64 + tg%64), columns [c0 + 64*(tg/64), +64): row tg%64 of
//            operand block tg/64 of the MN-major tile; code bytes: row tg%64, bytes
//            32*(tg/64).. of a 64 x 64-byte SW64 tile.
template <bool DX>
struct ItemGeom {
  int row, chunk;
  __device__ __forceinline__ explicit ItemGeom(int tg) {
    row = DX ? (tg & 63) : tg;
    chunk = DX ? (tg >> 6) : 0;
  }
  __device__ __forceinline__ uint32_t op_row_base(uint32_t wslot) const {
    return wslot + uint32_t(chunk) * 8192u + uint32_t(row) * 128u;
  }
  __device__ __forceinline__ uint32_t swz() const { return uint32_t(row) & 7u; }
  __device__ __forceinline__ uint32_t code_off(int half) const {
    if (!DX) {
      const uint32_t o = uint32_t(row) * 32u + uint32_t(half) * 16u;
      return o ^ (((o >> 7) & 1u) << 4);
    } else {
      const uint32_t o = uint32_t(row) * 64u + uint32_t(chunk) * 32u + uint32_t(half) * 16u;
      return o ^ (((o >> 7) & 3u) << 4);
    }
  }
};

template <int FMT, bool DX>
__global__ void __launch_bounds__(fused::kThreads, 1)
qlora_fused_gemm_kernel(const __grid_constant__ FusedParams p) {
  using namespace fused;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint8_t* wsm = xs + NX * X_BYTES;
  uint8_t* cs = wsm + NW * W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(cs + NC * C_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t b0 = ptx::smem_u32(bars);
  auto full_x = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty_x = [&](uint32_t s) { return b0 + 8u * (NX + s); };
  auto full_w = [&](uint32_t s) { return b0 + 8u * (2 * NX + s); };
  auto empty_w = [&](uint32_t s) { return b0 + 8u * (2 * NX + NW + s); };
  auto full_c = [&](uint32_t s) { return b0 + 8u * (2 * NX + 2 * NW + s); };
  auto empty_c = [&](uint32_t s) { return b0 + 8u * (2 * NX + 2 * NW + NC + s); };
  auto acc_full = [&](uint32_t b) { return b0 + 8u * (2 * NX + 2 * NW + 2 * NC + b); };
  auto acc_empty = [&](uint32_t b) { return b0 + 8u * (2 * NX + 2 * NW + 2 * NC + 2 + b); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NX; ++s) { ptx::mbar_init(full_x(s), 1); ptx::mbar_init(empty_x(s), 1); }
    for (int s = 0; s < NW; ++s) { ptx::mbar_init(full_w(s), kDqWarps / 2); ptx::mbar_init(empty_w(s), 1); }
    for (int s = 0; s < NC; ++s) { ptx::mbar_init(full_c(s), 1); ptx::mbar_init(empty_c(s), kDqWarps / 2); }
    for (int b = 0; b < 2; ++b) { ptx::mbar_init(acc_full(b), 1); ptx::mbar_init(acc_empty(b), kEpiWarps); }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    ptx::prefetch_tmap(&p.tm_act);
    ptx::prefetch_tmap(&p.tm_codes);
    ptx::prefetch_tmap(&p.tm_zs);
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int num_tiles = p.num_m * p.num_n;
  const int nk = p.num_k;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t i = 0, j = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        int mt, nt;
        fused_tile_coords(t, p.num_m, p.num_n, mt, nt);
        const int m0 = mt * BM, c0 = nt * BN;
        for (int ks = 0; ks <= nk; ++ks, ++i) {
          const uint32_t sx = i % NX, px = (i / NX) & 1u;
          if (!ptx::mbar_wait(empty_x(sx), px ^ 1u, p.status, abort_flag)) goto producer_done;
          ptx::mbar_arrive_expect_tx(full_x(sx), X_BYTES);
          const uint32_t xd = ptx::smem_u32(xs + sx * X_BYTES);
          if (ks < nk) {
            ptx::tma_load_2d(xd, &p.tm_act, full_x(sx), ks * BK, m0);
            ptx::tma_load_2d(xd + X_BYTES / 2, &p.tm_act, full_x(sx), ks * BK, m0 + 128);
          } else {
            ptx::tma_load_2d(xd, &p.tm_zs, full_x(sx), 0, m0);
            ptx::tma_load_2d(xd + X_BYTES / 2, &p.tm_zs, full_x(sx), 0, m0 + 128);
          }
          if (ks < nk) {
            const uint32_t sc = j % NC, pc = (j / NC) & 1u;
            if (!ptx::mbar_wait(empty_c(sc), pc ^ 1u, p.status, abort_flag)) goto producer_done;
            ptx::mbar_arrive_expect_tx(full_c(sc), C_BYTES);
            const uint32_t cd = ptx::smem_u32(cs + sc * C_BYTES);
            if (!DX) ptx::tma_load_2d(cd, &p.tm_codes, full_c(sc), ks * (BK / 2), c0);
            else ptx::tma_load_2d(cd, &p.tm_codes, full_c(sc), c0 / 2, ks * BK);
            ++j;
          }
        }
      }
    producer_done:;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16(128, BN, 0, DX ? 1u : 0u);
      const int lora_kk = (p.r + 15) / 16;
      uint32_t i = 0, tc = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tc) {
        const uint32_t buf = tc & 1u;
        if (!ptx::mbar_wait(acc_empty(buf), ((tc >> 1) & 1u) ^ 1u, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t d0 = tmem + buf * 2u * BN, d1 = d0 + BN;
        bool ok = true;
        for (int ks = 0; ks <= nk; ++ks, ++i) {
          const uint32_t sx = i % NX, sw = i % NW;
          if (!ptx::mbar_wait(full_x(sx), (i / NX) & 1u, p.status, abort_flag) ||
              !ptx::mbar_wait(full_w(sw), (i / NW) & 1u, p.status, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t xa = ptx::smem_u32(xs + sx * X_BYTES);
          const uint32_t wb = ptx::smem_u32(wsm + sw * W_BYTES);
          const int nkk = ks < nk ? BK / 16 : lora_kk;
          for (int kk = 0; kk < nkk; ++kk) {
            const uint64_t a0 = ptx::smem_desc(xa + kk * 32, 16, 1024, ptx::kSw128);
            const uint64_t a1 = ptx::smem_desc(xa + X_BYTES / 2 + kk * 32, 16, 1024, ptx::kSw128);
            const uint64_t bd = DX ? ptx::smem_desc(wb + kk * 2048, 8192, 1024, ptx::kSw128)
                                   : ptx::smem_desc(wb + kk * 32, 16, 1024, ptx::kSw128);
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            ptx::mma_bf16(d0, a0, bd, idesc, acc);
            ptx::mma_bf16(d1, a1, bd, idesc, acc);
          }
          ptx::mma_commit(empty_x(sx));
          ptx::mma_commit(empty_w(sw));
        }
        if (!ok) break;
        ptx::mma_commit(acc_full(buf));
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp;  // tensor-memory lanes 32q .. 32q+31
    const float ts = (FMT == kFmtNVFP4 && p.tensor_scale) ? __ldg(p.tensor_scale) : 1.0f;
    const int ncols = DX ? p.K : p.N;
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tc) {
      int mt, nt;
      fused_tile_coords(t, p.num_m, p.num_n, mt, nt);
      const int m0 = mt * BM, c0 = nt * BN;
      const uint32_t buf = tc & 1u;
      if (!ptx::mbar_wait(acc_full(buf), (tc >> 1) & 1u, p.status, abort_flag)) break;
      ptx::tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int row = m0 + h * 128 + q * 32 + lane;
#pragma unroll 1
        for (int cb = 0; cb < BN / 32; ++cb) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(tmem + (uint32_t(q * 32) << 16) + (buf * 2u + h) * BN + cb * 32, v);
          ptx::tmem_ld_wait();
          if (row < p.M) {
            __nv_bfloat16* orow = p.out + size_t(row) * ncols;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int col = c0 + cb * 32 + g * 8;
              if (col < ncols) {
                uint4 o;
                o.x = ptx::cvt_bf16x2(__uint_as_float(v[g * 8 + 0]) * ts, __uint_as_float(v[g * 8 + 1]) * ts);
                o.y = ptx::cvt_bf16x2(__uint_as_float(v[g * 8 + 2]) * ts, __uint_as_float(v[g * 8 + 3]) * ts);
                o.z = ptx::cvt_bf16x2(__uint_as_float(v[g * 8 + 4]) * ts, __uint_as_float(v[g * 8 + 5]) * ts);
                o.w = ptx::cvt_bf16x2(__uint_as_float(v[g * 8 + 6]) * ts, __uint_as_float(v[g * 8 + 7]) * ts);
                *reinterpret_cast<uint4*>(orow + col) = o;
              }
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(buf));
    }
  } else {
    // ------------------------------------------------------------------ dequant
    const int dw = warp - kDqWarp0;
    const int grp = dw >> 2;
    const int tg = (dw & 3) * 32 + lane;
    const ItemGeom<DX> geo(tg);
    uint32_t i = 0, j = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      int mt, nt;
      fused_tile_coords(t, p.num_m, p.num_n, mt, nt);
      const int c0 = nt * BN;
      for (int ks = 0; ks <= nk; ++ks, ++i) {
        const bool real = ks < nk;
        if (int(i & 1u) == grp) {
          const uint32_t sw = i % NW, pw = (i / NW) & 1u;
          const uint32_t rb = geo.op_row_base(ptx::smem_u32(wsm + sw * W_BYTES));
          if (real) {
            const int n = DX ? ks * BK + geo.row : c0 + geo.row;
            const int kcol = DX ? c0 + geo.chunk * 64 : ks * BK;
            const bool valid = n < p.N && kcol < p.K;
            ItemScale sc{0u};
            if (valid) sc = load_item_scale<FMT>(p.scales, n, kcol, p.K);
            const uint32_t scs = j % NC;
            if (!ptx::mbar_wait(full_c(scs), (j / NC) & 1u, p.status, abort_flag)) { ok = false; break; }
            const uint32_t cb = ptx::smem_u32(cs + scs * C_BYTES);
            const uint4 c_lo = ptx::ld_shared_v4(cb + geo.code_off(0));
            const uint4 c_hi = ptx::ld_shared_v4(cb + geo.code_off(1));
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty_c(scs));
            const uint32_t cw[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
            if (!ptx::mbar_wait(empty_w(sw), pw ^ 1u, p.status, abort_flag)) { ok = false; break; }
            if (valid) dequant_item_store<FMT>(cw, sc, rb, geo.swz());
            else zero_item_store(rb);
          } else {
            // LoRA step: rows of B (forward, K-major) or of A (dX, MN-major), zero padded.
            uint4 v[8];
            if (!DX) {
              const int n = c0 + geo.row;
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                v[jj] = (n < p.N && jj * 8 < p.r)
                            ? __ldg(reinterpret_cast<const uint4*>(p.lora_up + size_t(n) * p.r + jj * 8))
                            : make_uint4(0, 0, 0, 0);
            } else {
              const int rj = geo.row, kc = c0 + geo.chunk * 64;
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                v[jj] = (rj < p.r && kc < p.K)
                            ? __ldg(reinterpret_cast<const uint4*>(p.lora_up + size_t(rj) * p.K + kc + jj * 8))
                            : make_uint4(0, 0, 0, 0);
            }
            if (!ptx::mbar_wait(empty_w(sw), pw ^ 1u, p.status, abort_flag)) { ok = false; break; }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              ptx::st_shared_v4(rb + ((uint32_t(jj) ^ geo.swz()) << 4), v[jj].x, v[jj].y, v[jj].z, v[jj].w);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(full_w(sw));
        }
        if (real) ++j;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace qlora
