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
// The kernel runs on CTA pairs (clusters of 2) issuing tcgen05.mma.cta_group::2 of M=256, N=256.
// A pair tile is 512 rows x 256 output columns: two MMA blocks of 256 rows share each 16-deep
// step's dequantised weight operand.  CTA rank r holds rows [256b + 128r, 256b + 128r + 128) of
// activation block b and output columns [128r, 128r+128) of the weight operand, and receives rows
// [256b + 128r, +128) x all 256 columns of block b's fp32 accumulator in its own tensor memory
// (2 blocks x 256 columns, all 512 columns, single buffered).  Each weight element is decoded once
// per 512 rows (8 decoded weights per clock per SM keep the MMA at full rate), and each step issues
// 8 pair MMAs per barrier round, which keeps the fixed per-step cost of the issuing thread small
// against the 1024 cycles of tensor work.  The epilogue of one tile delays the next tile's first
// MMA (the accumulator is not double buffered); the dequant warps keep decoding into free stages
// meanwhile.
//
// Warp roles per CTA (480 threads, one CTA per SM, persistent over pair tiles):
//   warps 0-3   epilogue: tensor memory (both blocks) -> registers -> * ts -> bf16 -> a per-warp
//               staging tile in shared memory -> coalesced 64-byte row segments to global
//   warp  4     TMA producer of this CTA's activation half (completion counted on the leader's
//               barrier)
//   warp  6     TMA producer of this CTA's packed-code tiles, running ahead of the activation
//               stream on its own deeper ring so the decode never waits for codes
//   warp  5     tensor-memory allocation; in the leader CTA the single thread that issues the
//               pair MMA and commits (arriving on both CTAs' barriers); in the other CTA one
//               thread that forwards "weight half ready" to the leader, one cluster-scope arrive
//               per step (the dequant warps themselves only arrive on their own CTA's barrier)
// An operand stage holds this CTA's activation half and weight half of one 64-deep step.  The
// leader's stage-full barrier collects everything the pair MMA needs -- the activation bytes of
// both CTAs (TMA transaction count), the leader's 4 dequant warps and the other CTA's relayed
// arrive -- so the MMA thread waits once and commits once per step (a commit plus several waits
// per step cost the tensor pipe up to a third of its rate).
//   warps 7-14  dequant: two groups of 4 warps taking alternate steps; each thread decodes one
//               64-element item of its CTA's weight half per step into the swizzled operand tile;
//               its block scale is loaded from global memory two of its own steps ahead
// Barriers that only the pair's tensor core (commit) or local threads complete are waited on with
// CTA-scope acquire; the two that threads of the other CTA arrive on (the leader's stage-full and
// accumulator-empty barriers) are waited on with cluster-scope acquire.
// The weight tile is K-major for the forward pass (rows of W are rows of the operand) and
// MN-major for dX (rows of W run along the contraction); in both cases a 64-element item is one
// 128-byte swizzled row, so the decode stage is the same code.
#pragma once
#include <cuda_bf16.h>
#include "qlora_ptx.cuh"
#include "qlora_dequant.cuh"
#include "qlora_groups.cuh"

namespace qlora {
namespace fused {
constexpr int BM = 512, BN = 256;      // pair tile
constexpr int HM = 128, HN = 128;      // per-CTA rows of one MMA block; per-CTA weight half
constexpr int MB = 2;                  // MMA blocks of 256 rows per pair tile
constexpr int BK = 64;
constexpr int NS = 4, NC = 4;         // operand stages (activation blocks + weight half), code stages
constexpr int X_BYTES = HM * BK * 2;   // 16 KB per block
constexpr int W_BYTES = HN * BK * 2;   // 16 KB
constexpr int C_BYTES = HN * BK / 2;   // 4 KB of packed codes
constexpr int kEpiWarps = 4, kTmaWarp = 4, kMmaWarp = 5, kCodeWarp = 6, kDqWarp0 = 7, kDqWarps = 8;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kTmemCols = 512;         // 2 blocks x 256 columns
constexpr int GM = 8;                  // m-tiles per raster group
constexpr int kNumBars = 2 * NS + 2 * NC + 2;
// epilogue staging: per epilogue warp one tile of 32 rows x 32 output columns (bf16)
constexpr int STG_BYTES = 32 * 32 * 2;
constexpr size_t kStgOff = size_t(NS) * (MB * X_BYTES + W_BYTES) + size_t(NC) * C_BYTES + 1024;
constexpr size_t kSmemBase = 1024 + kStgOff + size_t(kEpiWarps) * STG_BYTES;
// plus the expert table: 2 x (E + 1) ints
__host__ __device__ constexpr size_t smem_bytes(int E) { return kSmemBase + size_t(2) * (E + 1) * 4; }
}  // namespace fused

struct FusedParams {
  CUtensorMap tm_act;    // activations [M, Kc] bf16, box {64, 128}, SW128
  CUtensorMap tm_codes;  // codes [E*N, K/2] u8: fwd box {32, 128} SW32; dX box {64, 64} SW64
  CUtensorMap tm_zs;     // Zs [M, r] bf16, box {64, 128}, SW128 (zero fill beyond r)
  const void* scales;                // [E, N, K/bs]
  const float* scales2;              // NF4DQ: second-level scales [E, ceil(N * K/64 / 256)]
  const float* tensor_scale;         // NVFP4: [E] device floats, else nullptr
  const __nv_bfloat16* lora_up;      // fwd: B [E, N, r]; dX: A [E, r, K]
  __nv_bfloat16* out;                // fwd: Y [M, N]; dX: dX [M, K]
  const int32_t* offsets;            // grouped: device [E+1] row offsets; nullptr: one expert
  int* status;
  unsigned* ticket;                  // pair-rank ticket, 0 between launches (wraps back to 0)
  int M, N, K, r, E;                 // M: all rows (packed over experts)
  int num_n, num_k;                  // pair tiles over output columns; contraction steps
  int tail_split;                    // the last tail_split 512-row tiles run as 2 x 256-row tiles
  uint32_t zero;                     // 0 (see zero_after)
};

// Tile t of an expert's (m-tile, n-tile) grid, in raster groups of `group_m` m-tiles.  The
// forward takes groups of GM: a wave then shares each weight tile among several row blocks.  dX
// takes groups of 1 (the n-tiles of one row block consecutive): the num_n tiles that read the same
// dY row block (up to 15 MB) run in the same wave and share it through L2, instead of reading it
// again a wave later.
__device__ __forceinline__ void fused_tile_coords(int t, int num_m, int num_n, int group_m, int& mt,
                                                  int& nt) {
  const int per_group = group_m * num_n;
  const int g = t / per_group;
  const int within = t - g * per_group;
  const int m_base = g * group_m;
  const int gm = min(group_m, num_m - m_base);
  mt = m_base + within % gm;
  nt = within / gm;
}

// Block-scale word of the item that starts at element (n, kcol) of the weight whose rows begin
// at row `nrow0` of the (stacked) scale array.
template <int FMT>
__device__ __forceinline__ ItemScale load_item_scale(const void* scales, int n, int kcol, int K,
                                                     size_t nrow0 = 0) {
  ItemScale s;
  const size_t row = nrow0 + size_t(n);
  if constexpr (FMT == kFmtNF4) {
    s.raw = __ldg(reinterpret_cast<const uint32_t*>(scales) + row * (K / 64) + kcol / 64);
  } else if constexpr (FMT == kFmtMXFP4) {
    s.raw = __ldg(reinterpret_cast<const uint16_t*>(scales) + (row * (K / 32) + kcol / 32) / 2);
  } else {
    s.raw = __ldg(reinterpret_cast<const uint32_t*>(scales) + (row * (K / 16) + kcol / 16) / 4);
  }
  return s;
}

// NF4DQ: the absmax of the block of element (n, kcol) of expert e's weight, from its first-level
// E4M3 code and the second-level scale of its group of 256 consecutive first-level codes in the
// expert's row-major [N, K/64] array.
__device__ __forceinline__ ItemScale load_item_scale_dq(const void* scales, const float* scales2,
                                                        int e, int N, int n, int kcol, int K) {
  const size_t nb = size_t(K) / 64;
  const size_t f = size_t(n) * nb + size_t(kcol) / 64;
  const size_t groups = (size_t(N) * nb + 255) / 256;
  const uint32_t c1 = __ldg(static_cast<const uint8_t*>(scales) + size_t(e) * size_t(N) * nb + f);
  return nf4dq_item_scale(c1, __ldg(scales2 + size_t(e) * groups + f / 256));
}

// The 4-byte word of the scale array that holds the block-scale material of the item starting at
// element (n, kcol), and the right shift that brings it to the low bits (for an asynchronous
// 4-byte copy into shared memory): NF4 the fp32 absmax; MXFP4 the two E8M0 bytes (2-byte
// aligned, so the word is the aligned one around them); NVFP4 the four E4M3 bytes.
template <int FMT>
__device__ __forceinline__ const void* item_scale_word(const void* scales, int n, int kcol, int K,
                                                       size_t nrow0, uint32_t& shift) {
  const size_t row = nrow0 + size_t(n);
  shift = 0;
  if constexpr (FMT == kFmtNF4) {
    return reinterpret_cast<const uint32_t*>(scales) + row * (K / 64) + kcol / 64;
  } else if constexpr (FMT == kFmtMXFP4) {
    const size_t off = row * (K / 32) + kcol / 32;
    shift = uint32_t(off & 2u) * 8u;
    return reinterpret_cast<const uint8_t*>(scales) + (off & ~size_t(3));
  } else {
    return reinterpret_cast<const uint8_t*>(scales) + row * (K / 16) + kcol / 16;
  }
}

// Pair tile t of a (grouped) launch: expert e, rows [row0, row0 + 256) of which rows below
// row_end belong to the expert, output-column tile nt.
struct PairTile {
  int e, row0, row_end, nt, nb;   // nb: MMA blocks of 256 rows in the tile (2, or 1 for a split tile)
};
// Tiles [0, total - tail) are the 512-row tiles of the table; when the last wave of tiles would
// leave most pairs idle, the host asks for the last `tail` of them to be split in two 256-row
// tiles each, scheduled after all others (indices total - tail .. total + tail - 1).
template <bool DX>
__device__ __forceinline__ PairTile pair_tile_at(const GroupView& g, int t, int num_n, int tail) {
  PairTile pt;
  int half = -1;
  const int nbig = g.total() - tail;
  if (t >= nbig) {
    half = (t - nbig) & 1;
    t = nbig + ((t - nbig) >> 1);
  }
  pt.e = g.expert_of(t);
  const int local = t - g.first[pt.e];
  const int rows = g.off[pt.e + 1] - g.off[pt.e];
  const int mtiles = (rows + fused::BM - 1) / fused::BM;
  int mt, nt;
  fused_tile_coords(local, mtiles, num_n, DX ? 1 : fused::GM, mt, nt);
  pt.row0 = g.off[pt.e] + mt * fused::BM;
  pt.row_end = g.off[pt.e + 1];
  pt.nt = nt;
  pt.nb = fused::MB;
  if (half >= 0) {
    pt.row0 += half * 2 * fused::HM;
    pt.row_end = min(pt.row_end, pt.row0 + 2 * fused::HM);
    pt.nb = 1;
  }
  return pt;
}

// Shared-memory geometry of one dequant item (thread tg = 0..127 of a dequant group) in a CTA's
// 128-column weight half whose first weight row (forward) or column (dX) is h0:
//   forward: item = weight row (h0 + tg), columns [ks*64, ks*64+64): operand row tg of the
//            K-major tile; code bytes: row tg of a 128 x 32-byte SW32 tile.
//   dX     : item = weight row (ks*64 + tg%64), columns [h0 + 64*(tg/64), +64): row tg%64 of
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(fused::kThreads, 1)
qlora_fused_gemm_kernel(const __grid_constant__ FusedParams p) {
  using namespace fused;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* xs = smem;                      // NS stages of this CTA's MB activation blocks
  uint8_t* wsm = xs + NS * MB * X_BYTES;   // NS weight halves
  uint8_t* cs = wsm + NS * W_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(cs + NC * C_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* pair_slot = tmem_slot + 2;
  int* s_off = reinterpret_cast<int*>(smem + (kSmemBase - 1024));
  int* s_first = s_off + (p.E + 1);

  const uint32_t b0 = ptx::smem_u32(bars);
  auto full_s = [&](uint32_t s) { return b0 + 8u * s; };
  auto empty_s = [&](uint32_t s) { return b0 + 8u * (NS + s); };
  auto full_c = [&](uint32_t s) { return b0 + 8u * (2 * NS + s); };
  auto empty_c = [&](uint32_t s) { return b0 + 8u * (2 * NS + NC + s); };
  const uint32_t acc_full = b0 + 8u * (2 * NS + 2 * NC);
  const uint32_t acc_empty = b0 + 8u * (2 * NS + 2 * NC + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int npairs = int(gridDim.x >> 1);
  if (threadIdx.x == 0 && rank == 0) {
    // Pair ranks in order of arrival: pairs that start late (their SMs still held by the previous
    // kernel) get the last ranks, whose static share of tiles is the smaller one.  atomicInc
    // wraps at npairs, so the npairs tickets of a launch are a permutation of 0..npairs-1 and
    // leave the ticket where it started.
    const uint32_t r = atomicInc(p.ticket, unsigned(npairs - 1));
    if (r >= uint32_t(npairs) && p.status)   // the workspace header was never zeroed
      atomicCAS(p.status, 0, 1 /* QLORA_ERR_INVALID_ARG */);
    *pair_slot = r;
    ptx::st_cluster_u32(ptx::mapa(ptx::smem_u32(pair_slot), 1), r);
  }
  if (threadIdx.x == 0) {
    // stage full: leader = producer's expect-tx arrive + 4 dequant warps + 1 relayed arrive;
    // other CTA = its 4 dequant warps (waited on by its relay).  acc_empty is used in the leader.
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(full_s(s), rank == 0 ? 2 + kDqWarps / 2 : kDqWarps / 2);
      ptx::mbar_init(empty_s(s), 1);
    }
    for (int s = 0; s < NC; ++s) { ptx::mbar_init(full_c(s), 1); ptx::mbar_init(empty_c(s), kDqWarps / 2); }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 2 * kEpiWarps);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    ptx::prefetch_tmap(&p.tm_act);
    ptx::prefetch_tmap(&p.tm_zs);
  }
  if (warp == kCodeWarp && lane == 0) ptx::prefetch_tmap(&p.tm_codes);
  if (warp == kMmaWarp) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  const GroupView grp_view =
      build_group_view(p.offsets, p.E, p.M, BM, p.num_n, s_off, s_first, p.status);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int pair = int(*pair_slot) % npairs;
  // The previous kernel of the stream (the lora_down launch that writes Zs) may still be running:
  // only the Zs loads of the LoRA steps wait for it (griddep_wait in the activation producer).
  // Everything else this kernel reads was complete before that kernel let this one launch.
  ptx::griddep_launch_dependents();

  const int num_tiles = grp_view.total() + p.tail_split;
  const int nk = p.num_k;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ activation producer
    if (lane == 0) {
      uint32_t i = 0;
      bool waited = false;
      for (int t = pair; t < num_tiles; t += npairs) {
        const PairTile pt = pair_tile_at<DX>(grp_view, t, p.num_n, p.tail_split);
        const int m0 = pt.row0 + int(rank) * HM;      // this CTA's rows of block 0 (+256: block 1)
        bool ok = true;
        for (int ks = 0; ks <= nk; ++ks, ++i) {
          const uint32_t sx = i % NS, px = (i / NS) & 1u;
          if (!ptx::mbar_wait(empty_s(sx), px ^ 1u, p.status, abort_flag)) { ok = false; break; }
          if (ks == nk && !waited) {
            ptx::griddep_wait();
            waited = true;
          }
          if (rank == 0) ptx::mbar_arrive_expect_tx(full_s(sx), 2 * pt.nb * X_BYTES);
          const uint32_t fx = ptx::mapa(full_s(sx), 0);
          for (int blk = 0; blk < pt.nb; ++blk) {
            const uint32_t xd = ptx::smem_u32(xs + (sx * MB + blk) * X_BYTES);
            if (ks < nk) {
              if (ptx::dcheck(ptx::tma_x_ok(ks * BK, 2), p.status))
                ptx::tma_load_2d_pair(xd, &p.tm_act, fx, ks * BK, m0 + blk * 2 * HM);
            } else {
              ptx::tma_load_2d_pair(xd, &p.tm_zs, fx, 0, m0 + blk * 2 * HM);
            }
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == kCodeWarp) {
    // ------------------------------------------------------------------ code producer
    if (lane == 0) {
      uint32_t j = 0;
      for (int t = pair; t < num_tiles; t += npairs) {
        const PairTile pt = pair_tile_at<DX>(grp_view, t, p.num_n, p.tail_split);
        const int h0 = pt.nt * BN + int(rank) * HN;   // this CTA's weight half
        const int wrow0 = pt.e * p.N;                 // the expert's first row of the codes
        bool ok = true;
        for (int ks = 0; ks < nk; ++ks, ++j) {
          const uint32_t sc = j % NC, pc = (j / NC) & 1u;
          if (!ptx::mbar_wait(empty_c(sc), pc ^ 1u, p.status, abort_flag)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(full_c(sc), C_BYTES);
          const uint32_t cd = ptx::smem_u32(cs + sc * C_BYTES);
          const int cx = !DX ? ks * (BK / 2) : h0 / 2;
          if (!ptx::dcheck(ptx::tma_x_ok(cx, 1) && pt.e < p.E, p.status)) continue;
          if (!DX) ptx::tma_load_2d(cd, &p.tm_codes, full_c(sc), cx, wrow0 + h0);
          else ptx::tma_load_2d(cd, &p.tm_codes, full_c(sc), cx, wrow0 + ks * BK);
        }
        if (!ok) break;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      // Lean issue loop: the issuing thread shares its SM sub-partition with busy dequant warps, so
      // every instruction between two steps' MMAs costs several cycles of tensor-pipe time.
      // Descriptors are the stage-0 descriptors plus constant offsets (the 14-bit address field
      // never carries), the four 16-deep sub-steps are unrolled, and the stage ring is a power of 2.
      static_assert((NS & (NS - 1)) == 0, "stage count must be a power of two");
      const uint32_t idesc = ptx::idesc_bf16(256, BN, 0, DX ? 1u : 0u);
      const int lora_kk = (p.r + 15) / 16;
      const uint64_t a0 = ptx::smem_desc(ptx::smem_u32(xs), 16, 1024, ptx::kSw128);
      const uint64_t b0d = DX ? ptx::smem_desc(ptx::smem_u32(wsm), 8192, 1024, ptx::kSw128)
                              : ptx::smem_desc(ptx::smem_u32(wsm), 16, 1024, ptx::kSw128);
      constexpr uint64_t kAStage = (MB * X_BYTES) >> 4, kBStage = W_BYTES >> 4;
      constexpr uint64_t kABlk = X_BYTES >> 4, kAkk = 32 >> 4, kBkk = DX ? (2048 >> 4) : (32 >> 4);
      uint32_t i = 0, tc = 0;
      for (int t = pair; t < num_tiles; t += npairs, ++tc) {
        const int nb = pair_tile_at<DX>(grp_view, t, p.num_n, p.tail_split).nb;
        if (!ptx::mbar_wait_cluster(acc_empty, (tc & 1u) ^ 1u, p.status, abort_flag)) break;
        ptx::tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks <= nk; ++ks, ++i) {
          const uint32_t st = i & (NS - 1);
          if (!ptx::mbar_wait_cluster(full_s(st), (i / NS) & 1u, p.status, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint64_t a = a0 + st * kAStage, b = b0d + st * kBStage;
          if (ks < nk) {
            const uint32_t acc0 = ks > 0 ? 1u : 0u;
            if (nb == 2) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) {
                ptx::mma_bf16_pair(tmem, a + kk * kAkk, b + kk * kBkk, idesc, kk ? 1u : acc0);
                ptx::mma_bf16_pair(tmem + BN, a + kABlk + kk * kAkk, b + kk * kBkk, idesc, kk ? 1u : acc0);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                ptx::mma_bf16_pair(tmem, a + kk * kAkk, b + kk * kBkk, idesc, kk ? 1u : acc0);
            }
          } else {
            for (int kk = 0; kk < lora_kk; ++kk) {
              ptx::mma_bf16_pair(tmem, a + kk * kAkk, b + kk * kBkk, idesc, 1u);
              if (nb == 2) ptx::mma_bf16_pair(tmem + BN, a + kABlk + kk * kAkk, b + kk * kBkk, idesc, 1u);
            }
          }
          ptx::mma_commit_pair(empty_s(st), 3);
        }
        if (!ok) break;
        ptx::mma_commit_pair(acc_full, 3);
      }
    } else if (lane == 0) {
      // relay (other CTA): this CTA's weight half of step i is complete -> tell the leader
      const uint32_t full_leader0 = ptx::mapa(full_s(0), 0);
      uint32_t i = 0;
      for (int t = pair; t < num_tiles; t += npairs) {
        bool ok = true;
        for (int ks = 0; ks <= nk; ++ks, ++i) {
          const uint32_t st = i % NS;
          if (!ptx::mbar_wait(full_s(st), (i / NS) & 1u, p.status, abort_flag)) { ok = false; break; }
          ptx::mbar_arrive_remote(full_leader0 + 8u * st);
        }
        if (!ok) break;
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------------ epilogue
    // Each warp drains its 32 accumulator lanes (rows) 32 columns at a time: scaled, rounded to
    // bf16 and written as one row per lane into a 32 x 32 staging tile (16-byte chunks XOR-swizzled
    // by row, so neither the row writes nor the column reads conflict), then read back 8 rows x
    // 64 bytes per warp instruction, so each global store covers 8 row segments of 64 contiguous
    // bytes instead of 32 scattered 16-byte pieces.
    const int q = warp;  // tensor-memory lanes 32q .. 32q+31
    const int ncols = DX ? p.K : p.N;
    const uint32_t acc_empty_leader = ptx::mapa(acc_empty, 0);
    const uint32_t stg = ptx::smem_u32(smem + kStgOff) + uint32_t(q) * STG_BYTES;
    const uint32_t wsw = (uint32_t(lane) >> 1) & 3u;             // write swizzle of row `lane`
    const int rr0 = lane >> 2, rc = lane & 3;                     // read: row rr0 + 8 it, chunk rc
    uint32_t tc = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++tc) {
      const PairTile pt = pair_tile_at<DX>(grp_view, t, p.num_n, p.tail_split);
      const int c0 = pt.nt * BN;
      const float ts = (FMT == kFmtNVFP4 && p.tensor_scale) ? __ldg(p.tensor_scale + pt.e) : 1.0f;
      if (!ptx::mbar_wait(acc_full, tc & 1u, p.status, abort_flag)) break;
      ptx::tc_fence_after();
#pragma unroll 1
      for (int blk = 0; blk < pt.nb; ++blk) {
        const int rbase = pt.row0 + blk * 2 * HM + int(rank) * HM + q * 32;
        if (rbase >= pt.row_end) continue;   // warp-uniform
        const uint32_t tb = tmem + (uint32_t(q * 32) << 16) + uint32_t(blk * BN);
#pragma unroll 1
        for (int cb = 0; cb < BN / 32; ++cb) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(tb + uint32_t(cb) * 32u, v);
          ptx::tmem_ld_wait(v);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float lo = __uint_as_float(v[g * 8 + 2 * j]), hi = __uint_as_float(v[g * 8 + 2 * j + 1]);
              if constexpr (FMT == kFmtNVFP4) { lo *= ts; hi *= ts; }
              w[j] = ptx::cvt_bf16x2(lo, hi);
            }
            ptx::st_shared_v4(stg + uint32_t(lane) * 64u + ((uint32_t(g) ^ wsw) << 4), w[0], w[1], w[2], w[3]);
          }
          __syncwarp();
          uint4 o[4];
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const uint32_t rr = uint32_t(it * 8 + rr0);
            o[it] = ptx::ld_shared_v4(stg + rr * 64u + ((uint32_t(rc) ^ ((rr >> 1) & 3u)) << 4));
          }
          __syncwarp();
          const int col = c0 + cb * 32 + rc * 8;
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int row = rbase + it * 8 + rr0;
            if (row < pt.row_end && col < ncols && ptx::dcheck(row >= 0 && pt.row_end <= p.M, p.status))
              *reinterpret_cast<uint4*>(p.out + size_t(row) * ncols + col) = o[it];
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_remote(acc_empty_leader);
    }
  } else {
    // ------------------------------------------------------------------ dequant
    const int dw = warp - kDqWarp0;
    const int grp = dw >> 2;
    const int tg = (dw & 3) * 32 + lane;
    const ItemGeom<DX> geo(tg);
    // Cursor over this group's steps (every other step of the CTA's pipeline): tile t (the lt-th
    // of this pair), step ks of the tile (ks == nk is the LoRA step), weight-half origin h0.
    struct Cursor {
      int t, lt, ks, h0, e;
    };
    auto set_tile = [&](Cursor& c) {
      if (c.t < num_tiles) {
        const PairTile pt = pair_tile_at<DX>(grp_view, c.t, p.num_n, p.tail_split);
        c.h0 = pt.nt * BN + int(rank) * HN;
        c.e = pt.e;
      }
    };
    auto advance2 = [&](Cursor& c) {
      c.ks += 2;
      if (c.ks > nk) {
        c.ks -= nk + 1;
        c.t += npairs;
        ++c.lt;
        set_tile(c);
      }
    };
    auto scale_for = [&](const Cursor& c) {
      ItemScale sc{0u};
      if (c.t < num_tiles && c.ks < nk) {
        const int n = DX ? c.ks * BK + geo.row : c.h0 + geo.row;
        const int kcol = DX ? c.h0 + geo.chunk * 64 : c.ks * BK;
        if (n < p.N && kcol < p.K) {
          if constexpr (FMT == kFmtNF4DQ) sc = load_item_scale_dq(p.scales, p.scales2, c.e, p.N, n, kcol, p.K);
          else sc = load_item_scale<FMT>(p.scales, n, kcol, p.K, size_t(c.e) * p.N);
        }
      }
      return sc;
    };
    Cursor cur{pair, 0, grp, 0, 0};
    set_tile(cur);
    Cursor pf = cur;
    advance2(pf);
    ItemScale s_cur = scale_for(cur), s_next = scale_for(pf);
    advance2(pf);
    while (cur.t < num_tiles) {
      const ItemScale s_pref = scale_for(pf);   // two own steps ahead
      advance2(pf);
      const uint32_t i = uint32_t(cur.lt * (nk + 1) + cur.ks);     // pipeline step
      const uint32_t sw = i % NS, pw = (i / NS) & 1u;
      const uint32_t rb = geo.op_row_base(ptx::smem_u32(wsm + sw * W_BYTES));
      if (cur.ks < nk) {
        const int n = DX ? cur.ks * BK + geo.row : cur.h0 + geo.row;
        const int kcol = DX ? cur.h0 + geo.chunk * 64 : cur.ks * BK;
        const bool valid = n < p.N && kcol < p.K;
        const uint32_t j = uint32_t(cur.lt * nk + cur.ks);          // code step
        const uint32_t scs = j % NC;
        if (!ptx::mbar_wait(full_c(scs), (j / NC) & 1u, p.status, abort_flag)) break;
        const uint32_t cb = ptx::smem_u32(cs + scs * C_BYTES);
        const uint4 c_lo = ptx::ld_shared_v4(cb + geo.code_off(0));
        const uint4 c_hi = ptx::ld_shared_v4(cb + geo.code_off(1));
        const uint32_t cw[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
        if (!ptx::mbar_wait(empty_s(sw), pw ^ 1u, p.status, abort_flag)) break;
        if (valid) dequant_item_store<FMT>(cw, s_cur, rb, geo.swz());
        else zero_item_store(rb);
        // release the code stage only once the loaded code words have been consumed: the
        // producer's next TMA into this stage must not overtake the loads above
        const uint32_t used = (c_lo.x ^ c_lo.y ^ c_lo.z ^ c_lo.w) ^ (c_hi.x ^ c_hi.y ^ c_hi.z ^ c_hi.w);
        const uint32_t dep = ptx::zero_after(used, p.zero);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(empty_c(scs) + dep);
      } else {
        // LoRA step: rows of B (forward, K-major) or of A (dX, MN-major), zero padded.
        uint4 v[8];
        const __nv_bfloat16* up = p.lora_up + size_t(cur.e) * size_t(p.r) * (DX ? p.K : p.N);
        if (!DX) {
          const int n = cur.h0 + geo.row;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            v[jj] = (n < p.N && jj * 8 < p.r)
                        ? __ldg(reinterpret_cast<const uint4*>(up + size_t(n) * p.r + jj * 8))
                        : make_uint4(0, 0, 0, 0);
        } else {
          const int rj = geo.row, kc = cur.h0 + geo.chunk * 64;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            v[jj] = (rj < p.r && kc < p.K)
                        ? __ldg(reinterpret_cast<const uint4*>(up + size_t(rj) * p.K + kc + jj * 8))
                        : make_uint4(0, 0, 0, 0);
        }
        if (!ptx::mbar_wait(empty_s(sw), pw ^ 1u, p.status, abort_flag)) break;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          ptx::st_shared_v4(rb + ((uint32_t(jj) ^ geo.swz()) << 4), v[jj].x, v[jj].y, v[jj].z, v[jj].w);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full_s(sw));
      s_cur = s_next;
      s_next = s_pref;
      advance2(cur);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == kMmaWarp) ptx::tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace qlora
