// qlora_stream.cuh -- the dequant-GEMM for short batches (M <= 256 rows): weight streaming.
//
//   forward : Y  = ( X  deq(W)^T + (s/ts) T B^T ) * ts     contraction over K, tiles over N
//   backward: dX = ( dY deq(W)   + (s/ts) U A   ) * ts     contraction over N, tiles over K
//
// With few rows the layer is a stream over the 4-bit weight: every weight element is decoded once
// and meets only M activation rows, so the work is the decode, not the tensor-core math.  The
// pair-tiled kernel (qlora_fused.cuh) would give such a batch one tile row, ceil(N/256) tiles, and
// leave most SMs idle; here the whole (output tile, contraction step) iteration space is instead
// cut into equal contiguous ranges, one per CTA (one CTA per SM), so every SM decodes the same
// number of weight elements.  A range may start or end inside an output tile; each piece of a tile
// (a segment) is accumulated in tensor memory and stored as an fp32 partial, and a second small
// kernel adds the partials of each tile in range order (a fixed order: results are deterministic),
// applies the NVFP4 tensor scale and writes bf16.
//
// A tile is 256 output columns (two 128-column weight halves, each decoded exactly as one CTA's
// half in the pair kernel) by all M rows.  Up to 128 rows (MT = 1) the activation rows are the A
// operand (M = 128; lanes past the batch are never read) and the whole decoded 256-row weight tile
// the B operand (N = 256): one MMA per 16-deep sub-step, an N at which the tensor core runs at
// its proportional rate.  Above 128 rows (MT = 2) the operands are swapped: each weight half is an
// A operand and the batch rows the B operand (N = M rounded up to 16), and the accumulator holds
// the tile transposed (tensor-memory lane = output column, column = batch row).
// The LoRA term is one extra step per tile (operands rows of B or A, and Zs), as in the pair
// kernel.  Every step has one operand stage (activation rows + weight tile) with one full and one
// empty barrier.
//
// Warp roles (480 threads, one CTA per SM):
//   warps 0-3   epilogue: tensor memory -> fp32 partial (global, L2-resident)
//   warp  4     TMA producer of the activation blocks (and Zs for the LoRA step)
//   warp  5     TMA producer of the packed-code tiles, on its own deeper ring
//   warp  6     tensor-memory allocation and the single MMA-issuing thread
//   warps 7-14  dequant: two groups of 4 warps taking alternate steps; thread tg of a group
//               decodes 64-element item tg of both 128-column weight halves of its step (a row of
//               the forward tile, or a row x column chunk of the dX tile); block scales are copied
//               asynchronously into a shared ring four own steps ahead of their use
#pragma once
#include <cuda_bf16.h>
#include "qlora_ptx.cuh"
#include "qlora_dequant.cuh"
#include "qlora_fused.cuh"

namespace qlora {
namespace stream {
constexpr int BN = 256, HN = 128, BK = 64;
constexpr int W_BYTES = BN * BK * 2;      // 32 KB (two 16 KB halves)
constexpr int HW_BYTES = HN * BK * 2;     // 16 KB
constexpr int C_BYTES = BN * BK / 2;      // 8 KB of packed codes (two 4 KB halves)
constexpr int HC_BYTES = HN * BK / 2;
constexpr int kEpiWarps = 4, kTmaWarp = 4, kCodeWarp = 5, kMmaWarp = 6, kDqWarp0 = 7, kDqWarps = 8;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kTmemCols = 512;
constexpr int kMaxRows = 256;
constexpr int SCALE_RING_BYTES = 4 * 2 * 256 * 4;   // kPf slots x 2 halves x 256 threads
// Operand stages: xrows activation rows (M rounded up to 16) plus one weight tile; the stage count
// depends on xrows, so every role tracks its stage index and phase incrementally.  MT = 1 for
// xrows <= 128 (double-buffered accumulators: 2 x 256 tensor-memory columns), 2 above (one
// accumulator: 2 halves x xrows columns).
__host__ __device__ constexpr int num_stages(int xrows) { return xrows <= 64 ? 4 : (xrows <= 128 ? 3 : 2); }
constexpr int kMaxStages = 4;
constexpr int NC = 6;                     // code stages
__host__ __device__ constexpr size_t smem_bytes(int xrows) {
  return 1024 + size_t(num_stages(xrows)) * (size_t(xrows) * 128 + W_BYTES) + size_t(NC) * C_BYTES +
         SCALE_RING_BYTES + 1024;
}
}  // namespace stream

struct StreamParams {
  CUtensorMap tm_act;    // activations [M, Kc] bf16, box {64, xrows}, SW128
  CUtensorMap tm_codes;  // codes [N, K/2] u8, per weight half: fwd box {32, 128} SW32; dX box {64, 64} SW64
  CUtensorMap tm_zs;     // Zs [M, r] bf16, box {64, xrows}, SW128
  const void* scales;                // [N, K/bs]
  const __nv_bfloat16* lora_up;      // fwd: B [N, r]; dX: A [r, K]
  float* partial;                    // [segments][M][256] fp32
  int* status;
  int M, N, K, r;
  int num_k;                         // contraction steps of 64 (the LoRA step comes after them)
  int num_tiles;                     // 256-column output tiles
  int iters;                         // L: (tile, step) iterations per CTA
  long long lcm;                     // lcm(L, num_k + 1)
  int xrows;                         // M rounded up to 16: activation rows per stage, MMA N
  uint32_t zero;                     // 0 (see zero_after)
  int segments;                      // partial segments the workspace holds
};

// Segments are the pieces of the iteration space between consecutive CTA-range starts (multiples
// of L) and tile starts (multiples of nk1); a segment's index is the number of such starts below
// its own start `st` (multiples of both counted once).
__device__ __forceinline__ int stream_segment(long long st, int L, int nk1, long long lcm) {
  return int((st + L - 1) / L + (st + nk1 - 1) / nk1 - (st + lcm - 1) / lcm);
}

// Segment bookkeeping shared by the producer, MMA and epilogue roles: iteration g of the flat
// (tile, step) space is tile g / (num_k + 1), step g % (num_k + 1).
struct StreamRange {
  int g0, g1, nk1;
  __device__ __forceinline__ int tile(int g) const { return g / nk1; }
  __device__ __forceinline__ int step(int g) const { return g - (g / nk1) * nk1; }
  __device__ __forceinline__ bool seg_end(int g) const { return g + 1 == g1 || step(g) == nk1 - 1; }
};

template <int FMT, bool DX, int MT>
__global__ void __launch_bounds__(stream::kThreads, 1)
qlora_stream_gemm_kernel(const __grid_constant__ StreamParams p) {
  using namespace stream;
  constexpr int NB = MT == 1 ? 2 : 1;          // accumulator buffers
  const int NS = num_stages(p.xrows);
  const uint32_t XSTAGE = uint32_t(p.xrows) * 128u;   // bytes of one activation stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* xst = smem;                         // NS activation stages, then NS weight tiles
  uint8_t* wst = xst + NS * XSTAGE;
  uint8_t* cs = wst + NS * W_BYTES;
  uint8_t* scr = cs + NC * C_BYTES;            // scale ring: kPf slots x 2 halves x 256 threads x 4 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(scr + SCALE_RING_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMaxStages + 2 * NC + 2 * NB);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t b0 = ptx::smem_u32(bars);
  auto full_s = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty_s = [&](uint32_t s) { return b0 + 8u * (kMaxStages + s); };
  auto full_c = [&](uint32_t s) { return b0 + 8u * (2 * kMaxStages + s); };
  auto empty_c = [&](uint32_t s) { return b0 + 8u * (2 * kMaxStages + NC + s); };
  auto acc_full = [&](uint32_t b) { return b0 + 8u * (2 * kMaxStages + 2 * NC + b); };
  auto acc_empty = [&](uint32_t b) { return b0 + 8u * (2 * kMaxStages + 2 * NC + NB + b); };
  auto xs = [&](uint32_t s) { return ptx::smem_u32(xst) + s * XSTAGE; };
  auto wsm = [&](uint32_t s) { return ptx::smem_u32(wst) + s * uint32_t(W_BYTES); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.num_k;
  const int total = p.num_tiles * (nk + 1);
  StreamRange rg;
  rg.nk1 = nk + 1;
  rg.g0 = int(blockIdx.x) * p.iters;
  rg.g1 = min(rg.g0 + p.iters, total);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(full_s(s), 1 + kDqWarps / 2);   // producer's expect-tx arrive + one dequant group
      ptx::mbar_init(empty_s(s), 1);
    }
    for (int s = 0; s < NC; ++s) { ptx::mbar_init(full_c(s), 1); ptx::mbar_init(empty_c(s), kDqWarps / 2); }
    for (int b = 0; b < NB; ++b) { ptx::mbar_init(acc_full(b), 1); ptx::mbar_init(acc_empty(b), kEpiWarps); }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    ptx::prefetch_tmap(&p.tm_act);
    ptx::prefetch_tmap(&p.tm_zs);
  }
  if (warp == kCodeWarp && lane == 0) ptx::prefetch_tmap(&p.tm_codes);
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The previous kernel of the stream (the lora_down launch that writes Zs, on SMs this launch
  // leaves free) may still be running: only the Zs loads of the LoRA steps wait for it.
  // Everything else this kernel reads was complete before that kernel let this one launch.
  ptx::griddep_launch_dependents();

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ activation producer
    if (lane == 0) {
      uint32_t s = 0, ph = 0;
      int ks = rg.step(rg.g0);
      bool waited = false;
      for (int g = rg.g0; g < rg.g1; ++g) {
        if (ks == nk && !waited) {
          ptx::griddep_wait();
          waited = true;
        }
        if (!ptx::mbar_wait_idle(empty_s(s), ph ^ 1u, p.status, abort_flag)) break;
        ptx::mbar_arrive_expect_tx(full_s(s), XSTAGE);
        if (ks < nk) {
          if (ptx::dcheck(ptx::tma_x_ok(ks * BK, 2), p.status))
            ptx::tma_load_2d(xs(s), &p.tm_act, full_s(s), ks * BK, 0);
        } else {
          ptx::tma_load_2d(xs(s), &p.tm_zs, full_s(s), 0, 0);
        }
        if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
        if (++ks == rg.nk1) ks = 0;
      }
    }
  } else if (warp == kCodeWarp) {
    // ------------------------------------------------------------------ code producer
    if (lane == 0) {
      uint32_t sc = 0, ph = 0;
      int ks = rg.step(rg.g0), c0 = rg.tile(rg.g0) * BN;
      for (int g = rg.g0; g < rg.g1; ++g) {
        if (ks < nk) {
          if (!ptx::mbar_wait_idle(empty_c(sc), ph ^ 1u, p.status, abort_flag)) break;
          ptx::mbar_arrive_expect_tx(full_c(sc), C_BYTES);
          const uint32_t cd = ptx::smem_u32(cs + sc * C_BYTES);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int cx = !DX ? ks * (BK / 2) : (c0 + h * HN) / 2;
            if (!ptx::dcheck(ptx::tma_x_ok(cx, 1), p.status)) continue;
            if (!DX) ptx::tma_load_2d(cd + h * HC_BYTES, &p.tm_codes, full_c(sc), cx, c0 + h * HN);
            else ptx::tma_load_2d(cd + h * HC_BYTES, &p.tm_codes, full_c(sc), cx, ks * BK);
          }
          if (++sc == uint32_t(NC)) { sc = 0; ph ^= 1u; }
        }
        if (++ks == rg.nk1) { ks = 0; c0 += BN; }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Lean issue loop (the thread shares its SM sub-partition with busy dequant warps):
      // descriptors are stage-0 descriptors plus constant offsets, the 16-deep sub-steps unrolled.
      const int lora_kk = (p.r + 15) / 16;
      const uint64_t x0 = ptx::smem_desc(xs(0), 16, 1024, ptx::kSw128);
      const uint64_t w0 = DX ? ptx::smem_desc(wsm(0), 8192, 1024, ptx::kSw128)
                             : ptx::smem_desc(wsm(0), 16, 1024, ptx::kSw128);
      const uint64_t kXStage = XSTAGE >> 4;
      constexpr uint64_t kWStage = W_BYTES >> 4, kWHalf = HW_BYTES >> 4;
      constexpr uint64_t kXkk = 32 >> 4, kWkk = DX ? (2048 >> 4) : (32 >> 4);
      // MT == 1: the activation rows are the A operand (M = 128: rows past xrows read whatever
      // follows in shared memory and land in accumulator lanes nobody reads) and the whole
      // 256-row weight tile the B operand (N = 256), one MMA per 16-deep sub-step; accumulator
      // buffer b = tensor-memory columns [256 b, 256 b + 256), lane = batch row.
      // MT == 2: each 128-row weight half is the A operand and the batch rows the B operand
      // (N = xrows), two MMAs per sub-step; the accumulator holds the tile transposed.
      const uint32_t idesc = MT == 1 ? ptx::idesc_bf16(128, 256, 0u, DX ? 1u : 0u)
                                     : ptx::idesc_bf16(128, uint32_t(p.xrows), DX ? 1u : 0u, 0u);
      const uint32_t xr = uint32_t(p.xrows);
      uint32_t b = 0, bph = 0, s = 0, ph = 0;
      int ks = rg.step(rg.g0);
      bool first = true;
      for (int g = rg.g0; g < rg.g1; ++g) {
        if (first) {
          if (!ptx::mbar_wait(acc_empty(b), bph ^ 1u, p.status, abort_flag)) break;
          ptx::tc_fence_after();
        }
        if (!ptx::mbar_wait(full_s(s), ph, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint64_t xd = x0 + s * kXStage, wd = w0 + s * kWStage;
        const uint32_t acc0 = first ? 0u : 1u;
        const int nkk = ks < nk ? BK / 16 : lora_kk;
        if constexpr (MT == 1) {
          const uint32_t d0 = tmem + b * uint32_t(BN);
          if (nkk == BK / 16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              ptx::mma_bf16(d0, xd + kk * kXkk, wd + kk * kWkk, idesc, kk ? 1u : acc0);
          } else {
            for (int kk = 0; kk < nkk; ++kk)
              ptx::mma_bf16(d0, xd + kk * kXkk, wd + kk * kWkk, idesc, kk ? 1u : acc0);
          }
        } else {
          const uint32_t d0 = tmem + b * 2u * xr;
          if (nkk == BK / 16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              ptx::mma_bf16(d0, wd + kk * kWkk, xd + kk * kXkk, idesc, kk ? 1u : acc0);
              ptx::mma_bf16(d0 + xr, wd + kWHalf + kk * kWkk, xd + kk * kXkk, idesc, kk ? 1u : acc0);
            }
          } else {
            for (int kk = 0; kk < nkk; ++kk) {
              ptx::mma_bf16(d0, wd + kk * kWkk, xd + kk * kXkk, idesc, kk ? 1u : acc0);
              ptx::mma_bf16(d0 + xr, wd + kWHalf + kk * kWkk, xd + kk * kXkk, idesc, kk ? 1u : acc0);
            }
          }
        }
        ptx::mma_commit(empty_s(s));
        first = false;
        if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
        const bool end = g + 1 == rg.g1 || ks == nk;
        if (++ks == rg.nk1) ks = 0;
        if (end) {
          ptx::mma_commit(acc_full(b));
          if (++b == uint32_t(NB)) { b = 0; bph ^= 1u; }
          first = true;
        }
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp;
    uint32_t b = 0, bph = 0;
    for (int g = rg.g0; g < rg.g1; ++g) {
      if (!rg.seg_end(g)) continue;
      if (!ptx::mbar_wait_idle(acc_full(b), bph, p.status, abort_flag)) break;
      ptx::tc_fence_after();
      const long long st = max((long long)rg.g0, (long long)rg.tile(g) * rg.nk1);
      const int seg = stream_segment(st, p.iters, rg.nk1, p.lcm);
      if (!ptx::dcheck(seg >= 0 && seg < p.segments, p.status)) break;
      float* base = p.partial + size_t(seg) * size_t(p.M) * BN;
      if constexpr (MT == 1) {
        // Tensor-memory lane 32q + lane holds batch row 32q + lane; its 256 columns are the tile's
        // output columns.  Warps whose rows are all past the batch have nothing to store.
        const int m = q * 32 + lane;
        if (q * 32 < p.M) {
          const uint32_t trow = tmem + (uint32_t(q * 32) << 16) + b * uint32_t(BN);
          float* row = base + size_t(m) * BN;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t v[32];
            ptx::tmem_ld_32x32b_x32(trow + uint32_t(c0), v);
            ptx::tmem_ld_wait(v);
            if (m < p.M) {
#pragma unroll
              for (int u = 0; u < 32; u += 4)
                __stcg(reinterpret_cast<float4*>(row + c0 + u),
                       make_float4(__uint_as_float(v[u]), __uint_as_float(v[u + 1]),
                                   __uint_as_float(v[u + 2]), __uint_as_float(v[u + 3])));
            }
          }
        }
      } else {
        // Tensor-memory lane 32q + lane holds output column hh * 128 + 32q + lane of the tile; its
        // accumulator columns are the batch rows.  Each store instruction writes 32 consecutive
        // floats of one partial row.
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t tcol = tmem + (uint32_t(q * 32) << 16) + b * 2u * uint32_t(p.xrows) + hh * uint32_t(p.xrows);
          float* col = base + hh * HN + q * 32 + lane;
#pragma unroll 1
          for (int m0 = 0; m0 < p.xrows; m0 += 16) {
            uint32_t v[16];
            ptx::tmem_ld_32x32b_x16(tcol + m0, v);
            ptx::tmem_ld_wait(v);
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (m0 + u < p.M) __stcg(col + size_t(m0 + u) * BN, __uint_as_float(v[u]));
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
      if (++b == uint32_t(NB)) { b = 0; bph ^= 1u; }
    }
  } else {
    // ------------------------------------------------------------------ dequant
    // Two groups of 4 warps take alternate steps, so one group's barrier waits and bookkeeping
    // overlap the other's decode; thread tg of a group decodes item tg of both weight halves.
    const int dt = threadIdx.x - kDqWarp0 * 32;   // 0..255
    const int grp = dt >> 7;
    const ItemGeom<DX> geo(dt & 127);
    // Block scales travel global -> shared by per-thread 4-byte asynchronous copies issued kPf own
    // steps ahead of their use (one copy group per own step, empty for steps without a scale), so
    // the decode never waits on a global load.  Positions advance incrementally (no divisions on
    // the decode path).
    constexpr int kPf = 4;
    const uint32_t sring = ptx::smem_u32(scr) + uint32_t(dt) * 4u;   // (slot, half) at + (2 slot + half) * 1024
    struct Cursor {
      int g, t, ks;
      uint32_t i, j;   // step index within the range; code-step index within the range
    };
    auto advance1 = [&](Cursor& c) {
      if (c.ks < nk) ++c.j;
      ++c.g;
      ++c.i;
      if (++c.ks == rg.nk1) { c.ks = 0; ++c.t; }
    };
    auto advance2 = [&](Cursor& c) { advance1(c); advance1(c); };
    // weight row n and first column kcol of this thread's item in weight half hh at cursor c
    auto item_at = [&](const Cursor& c, int hh, int& n, int& kcol) {
      const int h0 = c.t * BN + hh * HN;
      n = DX ? c.ks * BK + geo.row : h0 + geo.row;
      kcol = DX ? h0 + geo.chunk * 64 : c.ks * BK;
    };
    auto scale_fetch = [&](const Cursor& c, uint32_t slot, uint32_t dep) {
      if (c.g < rg.g1 && c.ks < nk) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          int n, kcol;
          item_at(c, hh, n, kcol);
          uint32_t sh;
          if (n < p.N && kcol < p.K)
            ptx::cp_async_4(sring + (2u * slot + hh) * 1024u + dep,
                            item_scale_word<FMT>(p.scales, n, kcol, p.K, 0, sh));
        }
      }
      ptx::cp_async_commit();
    };
    Cursor cur{rg.g0, rg.g0 / rg.nk1, rg.g0 - (rg.g0 / rg.nk1) * rg.nk1, 0u, 0u};
    if (grp) advance1(cur);
    Cursor pf = cur;
#pragma unroll
    for (int d = 0; d < kPf; ++d) {
      scale_fetch(pf, uint32_t(d), 0u);
      advance2(pf);
    }
    uint32_t slot = 0;
    uint32_t s = cur.i, pw = 0;   // operand stage of the step and its phase (own steps are 2 apart)
    if (s >= uint32_t(NS)) { s -= NS; pw ^= 1u; }
    for (; cur.g < rg.g1; advance2(cur), advance2(pf)) {
      ptx::cp_async_wait<kPf - 1>();
      uint32_t sdep = 0;   // zero, but only once the slot has been read: orders the refill after it
      bool ok = true;
      if (cur.ks < nk) {
        const uint32_t scs = cur.j % NC;
        if (!ptx::mbar_wait(full_c(scs), (cur.j / NC) & 1u, p.status, abort_flag)) break;
        uint32_t used = 0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          int n, kcol;
          item_at(cur, hh, n, kcol);
          uint32_t sh = 0;
          if (FMT == kFmtMXFP4) item_scale_word<FMT>(p.scales, n, kcol, p.K, 0, sh);
          ItemScale sc;
          sc.raw = ptx::ld_shared_u32(sring + (2u * slot + hh) * 1024u) >> sh;
          sdep |= sc.raw;
          const uint32_t cb = ptx::smem_u32(cs + scs * C_BYTES) + hh * HC_BYTES;
          const uint4 c_lo = ptx::ld_shared_v4(cb + geo.code_off(0));
          const uint4 c_hi = ptx::ld_shared_v4(cb + geo.code_off(1));
          const uint32_t cw[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
          if (hh == 0 && !ptx::mbar_wait(empty_s(s), pw ^ 1u, p.status, abort_flag)) { ok = false; break; }
          const uint32_t rb = geo.op_row_base(wsm(s) + hh * HW_BYTES);
          if (n < p.N && kcol < p.K) dequant_item_store<FMT>(cw, sc, rb, geo.swz());
          else zero_item_store(rb);
          used ^= (c_lo.x ^ c_lo.y ^ c_lo.z ^ c_lo.w) ^ (c_hi.x ^ c_hi.y ^ c_hi.z ^ c_hi.w);
        }
        if (!ok) break;
        // release the code stage only once the loaded words have been consumed
        const uint32_t dep = ptx::zero_after(used, p.zero);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(empty_c(scs) + dep);
      } else {
        // LoRA step: rows of B (forward, K-major) or of A (dX, MN-major), zero padded
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const int h0 = cur.t * BN + hh * HN;
          uint4 v[8];
          if (!DX) {
            const int n = h0 + geo.row;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              v[jj] = (n < p.N && jj * 8 < p.r)
                          ? __ldg(reinterpret_cast<const uint4*>(p.lora_up + size_t(n) * p.r + jj * 8))
                          : make_uint4(0, 0, 0, 0);
          } else {
            const int rj = geo.row, kc = h0 + geo.chunk * 64;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              v[jj] = (rj < p.r && kc < p.K)
                          ? __ldg(reinterpret_cast<const uint4*>(p.lora_up + size_t(rj) * p.K + kc + jj * 8))
                          : make_uint4(0, 0, 0, 0);
          }
          if (hh == 0 && !ptx::mbar_wait(empty_s(s), pw ^ 1u, p.status, abort_flag)) { ok = false; break; }
          const uint32_t rb = geo.op_row_base(wsm(s) + hh * HW_BYTES);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            ptx::st_shared_v4(rb + ((uint32_t(jj) ^ geo.swz()) << 4), v[jj].x, v[jj].y, v[jj].z, v[jj].w);
        }
        if (!ok) break;
      }
      sdep = ptx::zero_after(sdep, p.zero);
      scale_fetch(pf, slot, sdep);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full_s(s));
      slot = slot + 1 == kPf ? 0 : slot + 1;
      s += 2;
      if (s >= uint32_t(NS)) { s -= NS; pw ^= 1u; }
    }
    ptx::cp_async_wait<0>();
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

// out[m, c] = bf16( ts * sum over the segments of tile c / 256, in range order ), for m < M and
// c < ncols.  One thread per 4 consecutive columns of one row.  The segments of tile t are the
// consecutive indices from the rank of its first iteration t * nk1 to the rank of (t+1) * nk1.
struct StreamReduceParams {
  const float* partial;
  const float* tensor_scale;   // NVFP4: device float, else nullptr
  __nv_bfloat16* out;          // [M, ncols]
  int M, ncols, num_tiles, nk1, iters, lcm, segments;   // lcm clamped to at most total + 1
};

__device__ __forceinline__ int stream_rank32(int st, int L, int nk1, int lcm) {
  return (st + L - 1) / L + (st + nk1 - 1) / nk1 - (st + lcm - 1) / lcm;
}

__global__ void __launch_bounds__(256)
qlora_stream_reduce_kernel(const __grid_constant__ StreamReduceParams p) {
  constexpr int BN = stream::BN, Q4 = BN / 4;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int idx = int(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = p.num_tiles * Q4;
  if (idx >= per_row * p.M) return;
  const int m = idx / per_row;
  const int rem = idx - m * per_row;
  const int t = rem / Q4, col = (rem - t * Q4) * 4;
  if (t * BN + col >= p.ncols) return;
  const int seg0 = stream_rank32(t * p.nk1, p.iters, p.nk1, p.lcm);
  const int seg1 = t + 1 == p.num_tiles ? p.segments
                                        : stream_rank32((t + 1) * p.nk1, p.iters, p.nk1, p.lcm);
  if (!ptx::dcheck(seg0 >= 0 && seg1 <= p.segments && seg0 <= seg1, nullptr)) return;
  const float* src = p.partial + (size_t(seg0) * p.M + m) * BN + col;
  const size_t sstride = size_t(p.M) * BN;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sg = seg0; sg < seg1; sg += 4) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (sg + u < seg1) v[u] = __ldcg(reinterpret_cast<const float4*>(src + size_t(sg - seg0 + u) * sstride));
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (sg + u < seg1) { acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w; }
  }
  const float ts = p.tensor_scale ? __ldg(p.tensor_scale) : 1.0f;
  uint2 o;
  o.x = ptx::cvt_bf16x2(acc.x * ts, acc.y * ts);
  o.y = ptx::cvt_bf16x2(acc.z * ts, acc.w * ts);
  *reinterpret_cast<uint2*>(p.out + size_t(m) * p.ncols + t * BN + col) = o;
}

}  // namespace qlora
