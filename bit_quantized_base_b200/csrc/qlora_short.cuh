// qlora_short.cuh -- the dequant-GEMM for batches of at most 64 rows, where each pass streams the
// 4-bit weight once and the decode, not the tensor core, sets the pace.
//
//   forward : Y  = ( X  deq(W)^T + (s/ts') T B^T ) * ts'     contraction over K, tiles over N
//   backward: dX = ( dY deq(W)   + (s/ts') U A   ) * ts'     contraction over N, tiles over K
//
// ts' is the NVFP4 tensor scale times 2^8 (the decode below yields NVFP4 elements times 2^-8,
// exactly; lora_down scales Zs to match), 1 for NF4 and MXFP4.
//
// Work split: the flat space of (output tile, contraction iteration) pairs, plus one LoRA
// iteration per tile, is cut into equal contiguous ranges, one per CTA, so every SM decodes the
// same number of weight elements.  A tile that one CTA covers entirely is written straight from
// its accumulator; the pieces of a tile split between CTAs are stored as fp32 partials and the CTA
// that finishes a tile's last piece (arrival counters per tile and epilogue warp in the workspace
// header, reset by that CTA) adds the pieces in piece order -- a fixed order, so results are
// deterministic -- and writes the tile.
//
// One iteration covers 128 weight rows x 256 weight columns: 512 items of 64 elements, one per
// dequant thread, whose packed codes (128 rows x 128 bytes) arrive by one TMA box into a swizzled
// shared-memory ring.  The issuing thread then waits once and commits once per 16 (forward) or 8
// (dX) MMAs: its fixed cost per barrier round is several hundred cycles, larger than the tensor
// work of a single 64-deep step at these batch sizes.
//
// Forward (tcgen05 with the weight in tensor memory): a tile is 128 weight rows, the rows of the
// MMA's A operand, which the dequant warps write straight into tensor memory (lane = weight row,
// two bf16 per column along K); the batch rows (padded to a multiple of 16) are the N operand,
// staged in shared memory by TMA.  The accumulator holds the tile transposed (lane = output column,
// column = batch row).  An A operand read from tensor memory costs the tensor core about 45 cycles
// per 128 x 16 block of weights whatever N is, against about 64 from shared memory.
// dX (tcgen05 with the weight in shared memory): the contraction runs over weight rows, which the
// decode cannot lay out along tensor-memory lanes, so the decoded weight is the MN-major B operand
// (N = 256 output columns) in shared memory, as in the tiled kernel, and the batch rows the M = 128
// A operand (its rows past 64 read the next region of the stage and land in accumulator lanes that
// are never stored).
//
// Warp roles (736 threads, one CTA per SM):
//   warps 0-3   epilogue: tensor memory -> bf16 output, or fp32 partials and the tile reduction
//   warp  4     TMA producer of the activation tiles (and Zs for the LoRA iterations)
//   warp  5     tensor-memory allocation and the single MMA-issuing thread
//   warp  6     TMA producer of the packed-code tiles, on its own deeper ring
//   warps 7-22  dequant: every warp takes part in every iteration, one item per thread (forward:
//               warp w decodes k-block (w-7)/4 of the rows of its tensor-memory lane quarter w%4;
//               dX: chunk (w-7)/4 of rows 32((w-7)%4) .. +32); block scales are loaded from global
//               memory one iteration ahead.
#pragma once
#include <cuda_bf16.h>
#include "qlora_ptx.cuh"
#include "qlora_dequant.cuh"
#include "qlora_fused.cuh"

namespace qlora {
namespace shortk {
constexpr int KB = 64;                    // elements per item (one k-block)
constexpr int IW = 4;                     // items per weight row per iteration (256 elements)
constexpr int kMaxRows = 64;
constexpr int kEpiWarps = 4, kXWarp = 4, kMmaWarp = 5, kCodeWarp = 6, kDqWarp0 = 7, kDqWarps = 16;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kTmemCols = 512;
constexpr int kMaxTiles = 496;            // 4 arrival counters per tile in the workspace header
constexpr int C_BYTES = 128 * 128;        // packed codes of one iteration: 128 rows x 128 bytes
// forward: tile = 128 weight rows; iteration = 256 weight columns
constexpr int F_TILE = 128, F_NS = 3, F_NC = 4;
constexpr int F_ACC_COLS = 64;            // accumulator buffers at tensor-memory columns 0 and 64
constexpr int F_A_COL0 = 128;             // A slots of 128 columns at 128 + 128 s
// dX: tile = 256 output columns; iteration = 128 weight rows, two 64-deep slabs
constexpr int D_TILE = 256, D_NS = 2, D_NC = 3;
constexpr int D_A_SLAB = 64 * 128;        // rows 0-63 of one slab of the activation operand
constexpr int D_W_SLAB = D_TILE * 64 * 2; // one 64-deep slab of the decoded weight operand
constexpr int D_STAGE = 2 * D_A_SLAB + 2 * D_W_SLAB;
constexpr int kBarBytes = 2048;           // barriers, flags and the MMA descriptor table
constexpr int kTabOff = 1024;             // descriptor table offset inside that region
__host__ __device__ constexpr size_t fwd_smem_bytes(int xrows) {
  return 1024 + size_t(F_NC) * C_BYTES + size_t(F_NS) * IW * size_t(xrows) * 128 + kBarBytes;
}
__host__ __device__ constexpr size_t dx_smem_bytes() {
  return 1024 + size_t(D_NC) * C_BYTES + size_t(D_NS) * D_STAGE + kBarBytes;
}
}  // namespace shortk

struct ShortParams {
  CUtensorMap tm_act;    // X [M, K] (forward) or dY [M, N] (dX) bf16, box {64, xrows}, SW128
  CUtensorMap tm_zs;     // Zs [M, r] bf16, box {64, xrows}, SW128 (zero fill beyond r)
  CUtensorMap tm_codes;  // codes [N, K/2] u8, box {128, 128}, SW128
  const uint8_t* codes;              // the same codes (for the decoder's stand-alone export)
  const void* scales;                // [N, K/bs]
  const float* tensor_scale;         // NVFP4: device float, else nullptr
  const __nv_bfloat16* lora_up;      // forward: B [N, r]; dX: A [r, K]
  __nv_bfloat16* out;                // forward: Y [M, N]; dX: dX [M, K]
  float* partial;                    // [tiles][max_pieces][M][tile columns] fp32
  unsigned* counters;                // [tiles][4] arrival counters, zero between launches
  int* status;
  int M, N, K, r, rpad, xrows;
  int num_k;                         // contraction iterations per tile (the LoRA one follows them)
  int num_tiles;
  int iters;                         // L: iterations per CTA
  int max_pieces;
  float ts_mul;                      // 2^8 for NVFP4, else 1
  uint32_t one;                      // 1 (see decode_mul)
  uint32_t zero;                     // 0 (see zero_after)
};

namespace shortk {
// The CTAs whose ranges cover tile t: [first, last].
__device__ __forceinline__ void tile_pieces(int t, int nk1, int L, int& first, int& last) {
  first = (t * nk1) / L;
  last = (t * nk1 + nk1 - 1) / L;
}

// The 32 code bytes of item (row, chunk) of a 128 x 128-byte code tile stored with the 128-byte
// swizzle (16-byte unit u of row r at u ^ (r % 8)): conflict-free for 32 consecutive rows.
__device__ __forceinline__ void load_codes(uint32_t tile, int row, int chunk, uint32_t (&cw)[8]) {
  const uint32_t rb = tile + uint32_t(row) * 128u, sw = uint32_t(row) & 7u;
  const uint4 lo = ptx::ld_shared_v4(rb + ((uint32_t(2 * chunk) ^ sw) << 4));
  const uint4 hi = ptx::ld_shared_v4(rb + ((uint32_t(2 * chunk + 1) ^ sw) << 4));
  cw[0] = lo.x; cw[1] = lo.y; cw[2] = lo.z; cw[3] = lo.w;
  cw[4] = hi.x; cw[5] = hi.y; cw[6] = hi.z; cw[7] = hi.w;
}

// Release a code slot once the words loaded from it have arrived: the arrive's address takes a
// zero computed from every loaded word (zero_after), so it cannot issue before the shared-memory
// loads have returned, and the producer's next TMA into the slot cannot overtake them.  (Without
// the dependency that race garbled whole 32-column groups of the decoded weight in long runs.)
__device__ __forceinline__ void release_codes(uint32_t bar, const uint32_t (&cw)[8], int lane,
                                              uint32_t zero) {
  const uint32_t used = (cw[0] ^ cw[1] ^ cw[2] ^ cw[3]) ^ (cw[4] ^ cw[5] ^ cw[6] ^ cw[7]);
  const uint32_t dep = ptx::zero_after(used, zero);
  __syncwarp();
  if (lane == 0) ptx::mbar_arrive(bar + dep);
}

// Epilogue bookkeeping shared by both kernels.  Each epilogue warp owns the same slice of every
// tile in every CTA (its lane quarter), so the pieces of a slice are counted per (tile, warp): after
// the warp has stored its slice of a split tile's piece it counts it in and learns whether this
// CTA was the last to arrive, in which case it adds the slice's pieces and resets the counter.
// No barrier between the epilogue warps is needed.
__device__ __forceinline__ bool arrive_piece(unsigned* counter, int pieces) {
  __threadfence();                                       // this thread's piece stores, device-wide
  __syncwarp();
  unsigned last = 0u;
  if ((threadIdx.x & 31) == 0) last = atomicAdd(counter, 1u) == unsigned(pieces - 1) ? 1u : 0u;
  last = __shfl_sync(0xFFFFFFFFu, last, 0);
  if (last) __threadfence();
  return last != 0u;
}
}  // namespace shortk

// ============================================================================= forward
template <int FMT>
__global__ void __launch_bounds__(shortk::kThreads, 1)
qlora_short_fwd_kernel(const __grid_constant__ ShortParams p) {
  using namespace shortk;
  constexpr int NS = F_NS, NC = F_NC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t XB = uint32_t(p.xrows) * 128u;         // one 64-wide activation box
  uint8_t* cst = smem;                                  // NC code tiles
  uint8_t* xst = cst + NC * C_BYTES;                    // NS stages of IW activation boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(xst + NS * IW * XB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2 * NC + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t b0 = ptx::smem_u32(bars);
  auto full = [&](uint32_t s) { return b0 + 8u * s; };
  auto done = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  auto cfull = [&](uint32_t c) { return b0 + 8u * (2 * NS + c); };
  auto cempty = [&](uint32_t c) { return b0 + 8u * (2 * NS + NC + c); };
  auto acc_full = [&](uint32_t b) { return b0 + 8u * (2 * NS + 2 * NC + b); };
  auto acc_empty = [&](uint32_t b) { return b0 + 8u * (2 * NS + 2 * NC + 2 + b); };
  auto xs = [&](uint32_t s) { return ptx::smem_u32(xst) + s * uint32_t(IW) * XB; };
  auto cs = [&](uint32_t c) { return ptx::smem_u32(cst) + c * uint32_t(C_BYTES); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.num_k, nk1 = nk + 1;
  const int kblocks = p.K / KB;
  const int total = p.num_tiles * nk1;
  const int g0 = int(blockIdx.x) * p.iters;
  const int g1 = min(g0 + p.iters, total);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(full(s), 1 + kDqWarps);   // activation producer's expect-tx arrive + dequant warps
      ptx::mbar_init(done(s), 1);
    }
    for (int c = 0; c < NC; ++c) {
      ptx::mbar_init(cfull(c), 1);
      ptx::mbar_init(cempty(c), kDqWarps);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(acc_full(b), 1);
      ptx::mbar_init(acc_empty(b), kEpiWarps);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kXWarp && lane == 0) {
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
  // The previous kernel of the stream (lora_down, writing Zs, on SMs this grid leaves free) may
  // still run: the Zs loads wait for it, and so does the epilogue (arrival counters and partials
  // of the launch before it).  Everything else this kernel reads was complete before then.
  ptx::griddep_launch_dependents();

  if (warp == kXWarp) {
    // ------------------------------------------------------------------ activation producer
    if (lane == 0) {
      bool waited = false;
      uint32_t s = 0, ph = 0;
      int st = g0 % nk1;
      for (int g = g0; g < g1; ++g) {
        if (st == nk && !waited) {
          ptx::griddep_wait();
          waited = true;
        }
        if (!ptx::mbar_wait_idle(done(s), ph ^ 1u, p.status, abort_flag)) break;
        if (st < nk) {
          ptx::mbar_arrive_expect_tx(full(s), uint32_t(IW) * XB);
#pragma unroll
          for (int kb = 0; kb < IW; ++kb)
            if (ptx::dcheck(ptx::tma_x_ok((st * IW + kb) * KB, 2), p.status))
              ptx::tma_load_2d(xs(s) + uint32_t(kb) * XB, &p.tm_act, full(s), (st * IW + kb) * KB, 0);
        } else {
          ptx::mbar_arrive_expect_tx(full(s), XB);
          ptx::tma_load_2d(xs(s), &p.tm_zs, full(s), 0, 0);
        }
        if (++st == nk1) st = 0;
        if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == kCodeWarp) {
    // ------------------------------------------------------------------ code producer
    if (lane == 0) {
      uint32_t c = 0, ph = 0;
      int st = g0 % nk1, t = g0 / nk1;
      for (int g = g0; g < g1; ++g) {
        if (st < nk) {
          if (!ptx::mbar_wait_idle(cempty(c), ph ^ 1u, p.status, abort_flag)) break;
          ptx::mbar_arrive_expect_tx(cfull(c), C_BYTES);
          if (ptx::dcheck(ptx::tma_x_ok(st * (IW * KB / 2), 1) && t < p.num_tiles, p.status))
            ptx::tma_load_2d(cs(c), &p.tm_codes, cfull(c), st * (IW * KB / 2), t * F_TILE);
          if (++c == uint32_t(NC)) { c = 0; ph ^= 1u; }
        }
        if (++st == nk1) { st = 0; ++t; }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16(128, uint32_t(p.xrows), 0u, 0u);
      const uint64_t xd0 = ptx::smem_desc(xs(0), 16, 1024, ptx::kSw128);
      const uint64_t xbox = uint64_t(XB >> 4), xstage = uint64_t(IW) * xbox;
      const uint32_t a0 = tmem + uint32_t(F_A_COL0);
      const int lora_kk = p.rpad / 16;
      // descriptor table: entry (stage, k-block, 16-deep sub-step) = {B descriptor, A address};
      // the issue loop reads it instead of computing (see mma4_bf16_ts)
      const uint32_t tab = ptx::smem_u32(bars) + uint32_t(kTabOff);
      for (int ss = 0; ss < NS; ++ss)
        for (int kb = 0; kb < IW; ++kb)
          for (int kk = 0; kk < 4; ++kk)
            ptx::st_shared_v2_u64(tab + uint32_t((ss * IW + kb) * 4 + kk) * 16u,
                                  xd0 + uint64_t(ss) * xstage + uint64_t(kb) * xbox + uint64_t(kk) * 2u,
                                  uint64_t(a0 + uint32_t(ss) * 128u + uint32_t(kb) * 32u + uint32_t(kk) * 8u));
      uint32_t b = 0, bph = 0, s = 0, ph = 0, a = a0, ts = tab;
      uint64_t xd = xd0;
      int st = g0 % nk1;
      bool first = true;
      for (int g = g0; g < g1; ++g) {
        if (first) {
          if (!ptx::mbar_wait(acc_empty(b), bph ^ 1u, p.status, abort_flag)) break;
          ptx::tc_fence_after();
        }
        if (!ptx::mbar_wait(full(s), ph, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + b * uint32_t(F_ACC_COLS);
        const int nb = st < nk ? min(IW, kblocks - st * IW) : 0;
        if (nb == IW) {
#pragma unroll
          for (int kb = 0; kb < IW; ++kb) {
            uint32_t av[4];
            uint64_t xv[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              uint64_t aa;
              ptx::ld_shared_v2_u64(ts + uint32_t(kb * 4 + kk) * 16u, xv[kk], aa);
              av[kk] = uint32_t(aa);
            }
            ptx::mma4_bf16_ts(d, av, xv, idesc, (kb || !first) ? 1u : 0u);
          }
        } else if (st < nk) {
          for (int kb = 0; kb < nb; ++kb)
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_bf16_ts(d, a + uint32_t(kb * 32 + kk * 8), xd + uint64_t(kb) * xbox + uint64_t(kk) * 2u,
                               idesc, (kb || kk || !first) ? 1u : 0u);
        } else {
          for (int kk = 0; kk < lora_kk; ++kk)
            ptx::mma_bf16_ts(d, a + uint32_t(kk) * 8u, xd + uint64_t(kk) * 2u, idesc,
                             (kk || !first) ? 1u : 0u);
        }
        ptx::mma_commit(done(s));
        first = false;
        const bool end = g + 1 == g1 || st == nk;
        if (++st == nk1) st = 0;
        if (end) {
          ptx::mma_commit(acc_full(b));
          b ^= 1u;
          if (b == 0u) bph ^= 1u;
          first = true;
        }
        if (++s == uint32_t(NS)) {
          s = 0;
          ph ^= 1u;
          a = a0;
          xd = xd0;
          ts = tab;
        } else {
          a += 128u;
          xd += xstage;
          ts += uint32_t(IW * 4 * 16);
        }
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    ptx::griddep_wait();
    const int q = warp;
    const int nl = q * 32 + lane;                        // tile row = output column in the tile
    const float tse = (p.tensor_scale ? __ldg(p.tensor_scale) : 1.0f) * p.ts_mul;
    const size_t piece_elems = size_t(p.M) * F_TILE;
    uint32_t b = 0, bph = 0;
    int st = g0 % nk1, t = g0 / nk1;
    for (int g = g0; g < g1; ++g) {
      const bool end = g + 1 == g1 || st == nk;
      const int tile = t;
      if (++st == nk1) { st = 0; ++t; }
      if (!end) continue;
      if (!ptx::mbar_wait_idle(acc_full(b), bph, p.status, abort_flag)) break;
      ptx::tc_fence_after();
      int first, last;
      tile_pieces(tile, nk1, p.iters, first, last);
      const int n = tile * F_TILE + nl;
      const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + b * uint32_t(F_ACC_COLS);
      // this CTA's piece of the tile and the tile's arrival counter lie inside their regions
      const bool seg_ok = ptx::dcheck(tile < p.num_tiles && p.num_tiles <= kMaxTiles &&
                                      int(blockIdx.x) >= first &&
                                      int(blockIdx.x) - first < p.max_pieces, p.status);
      float* piece = p.partial + (size_t(tile) * p.max_pieces + size_t(int(blockIdx.x) - first)) * piece_elems;
#pragma unroll 1
      for (int c0 = 0; c0 < p.xrows; c0 += 16) {
        uint32_t v[16];
        ptx::tmem_ld_32x32b_x16(tbase + uint32_t(c0), v);
        ptx::tmem_ld_wait(v);
        if (first == last) {
          if (n < p.N) {
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (c0 + u < p.M)
                p.out[size_t(c0 + u) * p.N + n] = __float2bfloat16_rn(__uint_as_float(v[u]) * tse);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (seg_ok && c0 + u < p.M) __stcg(piece + size_t(c0 + u) * F_TILE + nl, __uint_as_float(v[u]));
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
      b ^= 1u;
      if (b == 0u) bph ^= 1u;
      if (seg_ok && first != last && arrive_piece(p.counters + tile * 4 + q, last - first + 1)) {
        // add the pieces in piece order, 16 batch rows at a time, two pieces' loads in flight
        // before their sums
        const float* p0 = p.partial + size_t(tile) * p.max_pieces * piece_elems + nl;
        const int np = last - first + 1;
#pragma unroll 1
        for (int m0 = 0; m0 < p.M; m0 += 16) {
          float a[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) a[u] = 0.0f;
#pragma unroll 1
          for (int j = 0; j < np; j += 2) {
            float v0[16], v1[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const bool ok = m0 + u < p.M;
              v0[u] = ok ? __ldcg(p0 + size_t(j) * piece_elems + size_t(m0 + u) * F_TILE) : 0.0f;
              v1[u] = ok && j + 1 < np ? __ldcg(p0 + size_t(j + 1) * piece_elems + size_t(m0 + u) * F_TILE) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              a[u] += v0[u];
              if (j + 1 < np) a[u] += v1[u];
            }
          }
          if (n < p.N) {
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (m0 + u < p.M) p.out[size_t(m0 + u) * p.N + n] = __float2bfloat16_rn(a[u] * tse);
          }
        }
        if (lane == 0) p.counters[tile * 4 + q] = 0u;
      }
    }
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------------ dequant
    const int q = warp & 3;                              // the lane quarter this warp may access
    const int chunk = (warp - kDqWarp0) >> 2;            // k-block of the iteration
    const int trow = q * 32 + lane;
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    const DecodeMul km = decode_mul(p.one);
    uint32_t s = 0, ph = 0, c = 0, cph = 0;
    int st = g0 % nk1, t = g0 / nk1;
    // block scale of this thread's item of iteration (tt, ss), loaded one iteration ahead
    auto scale_of = [&](int tt, int ss) -> uint32_t {
      const int n = tt * F_TILE + trow, kb = ss * IW + chunk;
      return (ss < nk && kb < kblocks && n < p.N) ? load_item_scale<FMT>(p.scales, n, kb * KB, p.K).raw : 0u;
    };
    uint32_t sc_next = scale_of(t, st);
    for (int g = g0; g < g1; ++g) {
      const uint32_t sc_cur = sc_next;
      const int tt = t, ss = st;
      if (++st == nk1) { st = 0; ++t; }
      if (g + 1 < g1) sc_next = scale_of(t, st);
      // the decode runs ahead of the tensor core by design: while a stage is still in use the
      // warp sleeps between polls, leaving issue slots to the MMA thread of its sub-partition
      if (!ptx::mbar_wait_idle(done(s), ph ^ 1u, p.status, abort_flag)) break;
      const uint32_t dst = tmem + lane_base + uint32_t(F_A_COL0) + s * 128u + uint32_t(chunk) * 32u;
      if (ss < nk) {
        if (!ptx::mbar_wait(cfull(c), cph, p.status, abort_flag)) break;
        uint32_t cw[8];
        load_codes(cs(c), trow, chunk, cw);
        release_codes(cempty(c), cw, lane, p.zero);
        if (++c == uint32_t(NC)) { c = 0; cph ^= 1u; }
        if (ss * IW + chunk < kblocks) {                 // warp-uniform: the store is collective
          ItemScale sc;
          sc.raw = sc_cur;
          uint32_t o[32];
          decode_item_regs<FMT>(cw, sc, km, o);
          __syncwarp();
          ptx::tmem_st_32x32b_x32(dst, o);
        }
      } else if (chunk == 0) {
        // LoRA iteration: row n of B (r values), zero padded to rpad
        const int n = tt * F_TILE + trow;
        uint32_t o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
        if (n < p.N) {
          const uint4* src = reinterpret_cast<const uint4*>(p.lora_up + size_t(n) * p.r);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j * 8 < p.r) {
              const uint4 v = __ldg(src + j);
              o[4 * j] = v.x; o[4 * j + 1] = v.y; o[4 * j + 2] = v.z; o[4 * j + 3] = v.w;
            }
        }
        __syncwarp();
        if (p.rpad == 16) {
          uint32_t o8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) o8[j] = o[j];
          ptx::tmem_st_32x32b_x8(dst, o8);
        } else if (p.rpad == 32) {
          uint32_t o16[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) o16[j] = o[j];
          ptx::tmem_st_32x32b_x16(dst, o16);
        } else {
          ptx::tmem_st_32x32b_x32(dst, o);
        }
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full(s));
      if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ============================================================================= dX
template <int FMT>
__global__ void __launch_bounds__(shortk::kThreads, 1)
qlora_short_dx_kernel(const __grid_constant__ ShortParams p) {
  using namespace shortk;
  constexpr int NS = D_NS, NC = D_NC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* cst = smem;
  uint8_t* stg = cst + NC * C_BYTES;                    // NS stages: [A slab 0][A slab 1][W slab 0][W slab 1]
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + NS * D_STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 2 * NC + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* s_defer = reinterpret_cast<volatile int*>(tmem_slot + 3);   // tile reduced at the end
  const uint32_t b0 = ptx::smem_u32(bars);
  auto full = [&](uint32_t s) { return b0 + 8u * s; };
  auto done = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  auto cfull = [&](uint32_t c) { return b0 + 8u * (2 * NS + c); };
  auto cempty = [&](uint32_t c) { return b0 + 8u * (2 * NS + NC + c); };
  auto acc_full = [&](uint32_t b) { return b0 + 8u * (2 * NS + 2 * NC + b); };
  auto acc_empty = [&](uint32_t b) { return b0 + 8u * (2 * NS + 2 * NC + 2 + b); };
  const uint32_t epi_a = b0 + 8u * (2 * NS + 2 * NC + 4);   // the 4 epilogue warps' pieces stored
  const uint32_t epi_b = epi_a + 8u;                         // this CTA's arrival counted
  auto xs = [&](uint32_t s) { return ptx::smem_u32(stg) + s * uint32_t(D_STAGE); };
  auto wsm = [&](uint32_t s) { return ptx::smem_u32(stg) + s * uint32_t(D_STAGE) + 2u * D_A_SLAB; };
  auto cs = [&](uint32_t c) { return ptx::smem_u32(cst) + c * uint32_t(C_BYTES); };
  const uint32_t XB = uint32_t(p.xrows) * 128u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.num_k, nk1 = nk + 1;
  const int total = p.num_tiles * nk1;
  const int g0 = int(blockIdx.x) * p.iters;
  const int g1 = min(g0 + p.iters, total);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(full(s), 1 + kDqWarps);
      ptx::mbar_init(done(s), 1);
    }
    for (int c = 0; c < NC; ++c) {
      ptx::mbar_init(cfull(c), 1);
      ptx::mbar_init(cempty(c), kDqWarps);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(acc_full(b), 1);
      ptx::mbar_init(acc_empty(b), kEpiWarps);
    }
    ptx::mbar_init(epi_a, kEpiWarps);
    ptx::mbar_init(epi_b, 1);
    *abort_flag = 0;
    *s_defer = -1;
    ptx::fence_mbarrier_init();
  }
  if (warp == kXWarp && lane == 0) {
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
  ptx::griddep_launch_dependents();

  if (warp == kXWarp) {
    // ------------------------------------------------------------------ activation producer
    if (lane == 0) {
      bool waited = false;
      uint32_t s = 0, ph = 0;
      int st = g0 % nk1;
      for (int g = g0; g < g1; ++g) {
        if (st == nk && !waited) {
          ptx::griddep_wait();
          waited = true;
        }
        if (!ptx::mbar_wait_idle(done(s), ph ^ 1u, p.status, abort_flag)) break;
        if (st < nk) {
          ptx::mbar_arrive_expect_tx(full(s), 2u * XB);
          if (ptx::dcheck(ptx::tma_x_ok(st * 128, 2), p.status)) {
            ptx::tma_load_2d(xs(s), &p.tm_act, full(s), st * 128, 0);
            ptx::tma_load_2d(xs(s) + D_A_SLAB, &p.tm_act, full(s), st * 128 + 64, 0);
          }
        } else {
          ptx::mbar_arrive_expect_tx(full(s), XB);
          ptx::tma_load_2d(xs(s), &p.tm_zs, full(s), 0, 0);
        }
        if (++st == nk1) st = 0;
        if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == kCodeWarp) {
    // ------------------------------------------------------------------ code producer
    if (lane == 0) {
      uint32_t c = 0, ph = 0;
      int st = g0 % nk1, t = g0 / nk1;
      for (int g = g0; g < g1; ++g) {
        if (st < nk) {
          if (!ptx::mbar_wait_idle(cempty(c), ph ^ 1u, p.status, abort_flag)) break;
          ptx::mbar_arrive_expect_tx(cfull(c), C_BYTES);
          if (ptx::dcheck(ptx::tma_x_ok(t * (D_TILE / 2), 1) && t < p.num_tiles, p.status))
            ptx::tma_load_2d(cs(c), &p.tm_codes, cfull(c), t * (D_TILE / 2), st * 128);
          if (++c == uint32_t(NC)) { c = 0; ph ^= 1u; }
        }
        if (++st == nk1) { st = 0; ++t; }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // batch rows as the M = 128 A operand, the decoded weight slab, MN-major, as the N = 256 B
      // operand; two 64-deep slabs per iteration
      const uint32_t idesc = ptx::idesc_bf16(128, D_TILE, 0u, 1u);
      const uint64_t x0 = ptx::smem_desc(xs(0), 16, 1024, ptx::kSw128);
      const uint64_t w0 = ptx::smem_desc(wsm(0), 8192, 1024, ptx::kSw128);
      constexpr uint64_t kStage = uint64_t(D_STAGE) >> 4, kWkk = 2048 >> 4;
      constexpr uint64_t kASlab = uint64_t(D_A_SLAB) >> 4, kWSlab = uint64_t(D_W_SLAB) >> 4;
      const int lora_kk = p.rpad / 16;
      // descriptor table: entry (stage, slab, 16-deep sub-step) = {A descriptor, B descriptor}
      const uint32_t tab = ptx::smem_u32(bars) + uint32_t(kTabOff);
      for (int ss = 0; ss < NS; ++ss)
        for (int sl = 0; sl < 2; ++sl)
          for (int kk = 0; kk < 4; ++kk)
            ptx::st_shared_v2_u64(tab + uint32_t((ss * 2 + sl) * 4 + kk) * 16u,
                                  x0 + uint64_t(ss) * kStage + uint64_t(sl) * kASlab + uint64_t(kk) * 2u,
                                  w0 + uint64_t(ss) * kStage + uint64_t(sl) * kWSlab + uint64_t(kk) * kWkk);
      uint32_t b = 0, bph = 0, s = 0, ph = 0, ts = tab;
      uint64_t xd = x0, wd = w0;
      int st = g0 % nk1;
      bool first = true;
      for (int g = g0; g < g1; ++g) {
        if (first) {
          if (!ptx::mbar_wait(acc_empty(b), bph ^ 1u, p.status, abort_flag)) break;
          ptx::tc_fence_after();
        }
        if (!ptx::mbar_wait(full(s), ph, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + b * uint32_t(D_TILE);
        if (st < nk) {
          const int nsl = min(2, (p.N - st * 128 + 63) / 64);   // slabs holding weight rows
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            if (sl < nsl) {
              uint64_t xv[4], wv[4];
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) ptx::ld_shared_v2_u64(ts + uint32_t(sl * 4 + kk) * 16u, xv[kk], wv[kk]);
              ptx::mma4_bf16_ss(d, xv, wv, idesc, (sl || !first) ? 1u : 0u);
            }
          }
        } else {
          for (int kk = 0; kk < lora_kk; ++kk)
            ptx::mma_bf16(d, xd + uint64_t(kk) * 2u, wd + uint64_t(kk) * kWkk, idesc,
                          (kk || !first) ? 1u : 0u);
        }
        ptx::mma_commit(done(s));
        first = false;
        const bool end = g + 1 == g1 || st == nk;
        if (++st == nk1) st = 0;
        if (end) {
          ptx::mma_commit(acc_full(b));
          b ^= 1u;
          if (b == 0u) bph ^= 1u;
          first = true;
        }
        if (++s == uint32_t(NS)) {
          s = 0;
          ph ^= 1u;
          xd = x0;
          wd = w0;
          ts = tab;
        } else {
          xd += kStage;
          wd += kStage;
          ts += uint32_t(2 * 4 * 16);
        }
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    ptx::griddep_wait();
    const int q = warp;
    const int m = q * 32 + lane;                         // batch row = accumulator lane
    const bool active = q * 32 < p.M;
    const float tse = (p.tensor_scale ? __ldg(p.tensor_scale) : 1.0f) * p.ts_mul;
    const size_t piece_elems = size_t(p.M) * D_TILE;
    uint32_t b = 0, bph = 0, ephase = 0;
    int st = g0 % nk1, t = g0 / nk1;
    for (int g = g0; g < g1; ++g) {
      const bool end = g + 1 == g1 || st == nk;
      const int tile = t;
      if (++st == nk1) { st = 0; ++t; }
      if (!end) continue;
      if (!ptx::mbar_wait_idle(acc_full(b), bph, p.status, abort_flag)) break;
      ptx::tc_fence_after();
      int first, last;
      tile_pieces(tile, nk1, p.iters, first, last);
      const int k0 = tile * D_TILE;
      const bool seg_ok = ptx::dcheck(tile < p.num_tiles && p.num_tiles <= kMaxTiles &&
                                      int(blockIdx.x) >= first &&
                                      int(blockIdx.x) - first < p.max_pieces, p.status);
      float* piece = p.partial + (size_t(tile) * p.max_pieces + size_t(int(blockIdx.x) - first)) * piece_elems;
      if (active) {
        const uint32_t tbase = tmem + (uint32_t(q * 32) << 16) + b * uint32_t(D_TILE);
#pragma unroll 1
        for (int c = 0; c < D_TILE / 32; ++c) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(tbase + uint32_t(c * 32), v);
          ptx::tmem_ld_wait(v);
          if (seg_ok && m < p.M && k0 + c * 32 < p.K) {
            if (first == last) {
              uint4* dst = reinterpret_cast<uint4*>(p.out + size_t(m) * p.K + k0 + c * 32);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                uint4 w;
                w.x = ptx::cvt_bf16x2(__uint_as_float(v[8 * u]) * tse, __uint_as_float(v[8 * u + 1]) * tse);
                w.y = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 2]) * tse, __uint_as_float(v[8 * u + 3]) * tse);
                w.z = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 4]) * tse, __uint_as_float(v[8 * u + 5]) * tse);
                w.w = ptx::cvt_bf16x2(__uint_as_float(v[8 * u + 6]) * tse, __uint_as_float(v[8 * u + 7]) * tse);
                dst[u] = w;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(piece + size_t(m) * D_TILE + c * 32);
#pragma unroll
              for (int u = 0; u < 8; ++u)
                __stcg(dst + u, make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                            __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3])));
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
      b ^= 1u;
      if (b == 0u) bph ^= 1u;
      if (seg_ok && first != last) {
        // Split tile: the 4 warps' row slices of this piece are stored; count the CTA's piece
        // once (thread 0), and if it was the last to arrive, all 128 epilogue threads add the
        // tile's pieces in piece order (each thread 4 columns of every other batch row).  The
        // rendezvous uses bounded mbarrier waits, so a stalled pipeline cannot hang it.
        __threadfence();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(epi_a);
        if (!ptx::mbar_wait(epi_a, ephase, p.status, abort_flag)) break;
        if (threadIdx.x == 0) {
          const unsigned old = atomicAdd(p.counters + tile * 4, 1u);
          *s_last = old == unsigned(last - first) ? 1 : 0;
          __threadfence();
          ptx::mbar_arrive(epi_b);
        }
        if (!ptx::mbar_wait(epi_b, ephase, p.status, abort_flag)) break;
        ephase ^= 1u;
        if (*s_last && g + 1 == g1) {
          // the tile of the range's last segment: every thread of the CTA adds it once all roles
          // are done (below), with 5.75 times the epilogue warps' loads in flight
          if (threadIdx.x == 0) *s_defer = tile;
        } else if (*s_last) {
          __threadfence();
          const int e = int(threadIdx.x);                     // 0..127
          const int c0 = (e & 63) * 4, rh = e >> 6;
          const float* p0 = p.partial + size_t(tile) * p.max_pieces * piece_elems + c0;
          const int np = last - first + 1;
          if (k0 + c0 < p.K) {
#pragma unroll 1
            for (int mb = rh; mb < p.M; mb += 16) {
              float4 a[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
              for (int j = 0; j < np; j += 2) {
                float4 v0[8], v1[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const int mm = mb + 2 * u;
                  const bool ok = mm < p.M;
                  v0[u] = ok ? __ldcg(reinterpret_cast<const float4*>(p0 + size_t(j) * piece_elems + size_t(mm) * D_TILE))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
                  v1[u] = ok && j + 1 < np
                              ? __ldcg(reinterpret_cast<const float4*>(p0 + size_t(j + 1) * piece_elems + size_t(mm) * D_TILE))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  a[u].x += v0[u].x; a[u].y += v0[u].y; a[u].z += v0[u].z; a[u].w += v0[u].w;
                  if (j + 1 < np) {
                    a[u].x += v1[u].x; a[u].y += v1[u].y; a[u].z += v1[u].z; a[u].w += v1[u].w;
                  }
                }
              }
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int mm = mb + 2 * u;
                if (mm < p.M) {
                  uint2 w;
                  w.x = ptx::cvt_bf16x2(a[u].x * tse, a[u].y * tse);
                  w.y = ptx::cvt_bf16x2(a[u].z * tse, a[u].w * tse);
                  *reinterpret_cast<uint2*>(p.out + size_t(mm) * p.K + k0 + c0) = w;
                }
              }
            }
          }
          if (threadIdx.x == 0) p.counters[tile * 4] = 0u;
        }
      }
    }
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------------ dequant
    const int dq = warp - kDqWarp0;
    const int row = (dq & 3) * 32 + lane;                // weight row of the iteration (0..127)
    const int chunk = dq >> 2;                           // 64-column chunk of the tile
    const int slab = row >> 6, rs = row & 63;
    const uint32_t swz = uint32_t(rs) & 7u;
    const DecodeMul km = decode_mul(p.one);
    uint32_t s = 0, ph = 0, c = 0, cph = 0;
    int st = g0 % nk1, t = g0 / nk1;
    auto scale_of = [&](int tt, int ss) -> uint32_t {
      const int n = ss * 128 + row, kc = tt * D_TILE + chunk * KB;
      return (ss < nk && n < p.N && kc < p.K) ? load_item_scale<FMT>(p.scales, n, kc, p.K).raw : 0u;
    };
    uint32_t sc_next = scale_of(t, st);
    for (int g = g0; g < g1; ++g) {
      const uint32_t sc_cur = sc_next;
      const int tt = t, ss = st;
      if (++st == nk1) { st = 0; ++t; }
      if (g + 1 < g1) sc_next = scale_of(t, st);
      if (!ptx::mbar_wait_idle(done(s), ph ^ 1u, p.status, abort_flag)) break;
      const uint32_t rb = wsm(s) + uint32_t(slab) * D_W_SLAB + uint32_t(chunk) * 8192u + uint32_t(rs) * 128u;
      const int kc = tt * D_TILE + chunk * KB;
      if (ss < nk) {
        if (!ptx::mbar_wait(cfull(c), cph, p.status, abort_flag)) break;
        uint32_t cw[8];
        load_codes(cs(c), row, chunk, cw);
        release_codes(cempty(c), cw, lane, p.zero);
        if (++c == uint32_t(NC)) { c = 0; cph ^= 1u; }
        const int n = ss * 128 + row;
        if (n < p.N && kc < p.K) {
          ItemScale sc;
          sc.raw = sc_cur;
          decode_item_store<FMT>(cw, sc, km, rb, swz);
        } else {
          zero_item_store(rb);
        }
      } else if (slab == 0) {
        // LoRA iteration: row `rs` of A, columns [kc, kc + 64), zero padded to rpad rows
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          v[j] = (rs < p.r && kc < p.K)
                     ? __ldg(reinterpret_cast<const uint4*>(p.lora_up + size_t(rs) * p.K + kc + j * 8))
                     : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          ptx::st_shared_v4(rb + ((uint32_t(j) ^ swz) << 4), v[j].x, v[j].y, v[j].z, v[j].w);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full(s));
      if (++s == uint32_t(NS)) { s = 0; ph ^= 1u; }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);

  // This CTA was the last to arrive at the tile of its final segment: add the tile's pieces in
  // piece order (the order of the epilogue's own reduction, so the result is the same bit for
  // bit) with all threads, two 4-column groups of a row per thread and four pieces of each in
  // flight, then reset the tile's counter.
  const int dtile = *s_defer;
  if (dtile >= 0) {
    int first, last;
    tile_pieces(dtile, nk1, p.iters, first, last);
    const int np = last - first + 1;
    if (*abort_flag == 0 && ptx::dcheck(dtile < p.num_tiles && np <= p.max_pieces, p.status)) {
      __threadfence();
      const int k0 = dtile * D_TILE;
      const float tse = (p.tensor_scale ? __ldg(p.tensor_scale) : 1.0f) * p.ts_mul;
      const size_t piece_elems = size_t(p.M) * D_TILE;
      const float* base = p.partial + size_t(dtile) * p.max_pieces * piece_elems;
      const int items = p.M * (D_TILE / 4);              // (batch row, 4-column group)
      const int T = int(blockDim.x);
      auto item_ptr = [&](int i) { return base + size_t(i >> 6) * D_TILE + (i & 63) * 4; };
      auto write4 = [&](int i, const float4& a) {
        const int mm = i >> 6, c0 = (i & 63) * 4;
        if (k0 + c0 < p.K) {
          uint2 w;
          w.x = ptx::cvt_bf16x2(a.x * tse, a.y * tse);
          w.y = ptx::cvt_bf16x2(a.z * tse, a.w * tse);
          *reinterpret_cast<uint2*>(p.out + size_t(mm) * p.K + k0 + c0) = w;
        }
      };
#pragma unroll 1
      for (int i0 = int(threadIdx.x); i0 < items; i0 += 2 * T) {
        const int i1 = i0 + T;
        const bool two = i1 < items;
        const float* q0 = item_ptr(i0);
        const float* q1 = item_ptr(two ? i1 : i0);
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 1
        for (int j = 0; j < np; j += 4) {
          float4 v0[4], v1[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool ok = j + u < np;
            v0[u] = ok ? __ldcg(reinterpret_cast<const float4*>(q0 + size_t(j + u) * piece_elems))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
            v1[u] = ok && two ? __ldcg(reinterpret_cast<const float4*>(q1 + size_t(j + u) * piece_elems))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (j + u < np) {
              a0.x += v0[u].x; a0.y += v0[u].y; a0.z += v0[u].z; a0.w += v0[u].w;
              a1.x += v1[u].x; a1.y += v1[u].y; a1.z += v1[u].z; a1.w += v1[u].w;
            }
        }
        write4(i0, a0);
        if (two) write4(i1, a1);
      }
    }
    if (threadIdx.x == 0) p.counters[dtile * 4] = 0u;
  }
}

}  // namespace qlora
